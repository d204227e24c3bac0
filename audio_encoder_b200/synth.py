"""Seeded synthetic inputs: PCM clips and a random-init weight blob.

This module holds only input synthesis. It does none of the encoder's
arithmetic (no STFT, mel, convolution, attention or layer math), so both the
CUDA path and the CPU oracle can take their inputs from it.

PCM recipe (16 kHz mono fp32):
  * "tones" clip: the sum of three sines, each with a frequency uniform in
    [100, 6000] Hz, an amplitude uniform in [0.1, 0.3] and a phase uniform in
    [0, 2*pi), plus white Gaussian noise of standard deviation 0.01.
  * "30 s" clip: a tones clip plus, over seconds 12-17, white Gaussian noise of
    standard deviation 0.05 band-passed to 300-3400 Hz by zeroing FFT bins.
  * "long" clip: tones whose three frequencies, amplitudes and phases are
    redrawn every 2 s, plus the same white noise.
  * batch clip i: seed i, a length drawn uniformly from [160000, 480000]
    samples (10-30 s), then a tones clip of that length.

Weight recipe: every tensor in the documented blob order (``weight_manifest``)
is drawn from one PCG64 stream seeded with ``seed``: matrices and conv kernels
N(0, 1/fan_in), biases N(0, 0.01^2), LayerNorm gamma = 1 and beta = 0; then
rounded once to bf16 (round to nearest even). The blob is a flat little-endian
array of bf16 bit patterns (uint16).
"""
from __future__ import annotations

import numpy as np

SAMPLE_RATE = 16000

# Encoder widths (Qwen3-Omni AuT tower as described on the MOSS-Transcribe
# GGUF card, "Architecture" table).
D_MODEL = 1280
N_HEADS = 20
HEAD_DIM = 64
D_FFN = 5120
C_STEM = 480
F_STEM = 16          # mel bins after three stride-2 convs (128 -> 16)
D_OUT = 2048         # proj2 output width
D_ADAPTER = 8192     # SwiGLU hidden width


def weight_manifest(n_layers: int):
    """List of (name, shape, kind) in blob order.

    kind is "w" (matrix / conv kernel, N(0, 1/fan_in)), "b" (bias,
    N(0, 0.01^2)), "g" (LayerNorm gamma, ones) or "beta" (LayerNorm beta,
    zeros). Shapes follow PyTorch conventions: linear [out, in], conv
    [out, in, k_freq, k_time].
    """
    m = [
        ("conv1.weight", (C_STEM, 1, 3, 3), "w"),
        ("conv1.bias", (C_STEM,), "b"),
        ("conv2.weight", (C_STEM, C_STEM, 3, 3), "w"),
        ("conv2.bias", (C_STEM,), "b"),
        ("conv3.weight", (C_STEM, C_STEM, 3, 3), "w"),
        ("conv3.bias", (C_STEM,), "b"),
        ("conv_out.weight", (D_MODEL, C_STEM * F_STEM), "w"),
    ]
    for i in range(n_layers):
        p = f"layers.{i}."
        m += [
            (p + "ln1.weight", (D_MODEL,), "g"),
            (p + "ln1.bias", (D_MODEL,), "beta"),
            (p + "q.weight", (D_MODEL, D_MODEL), "w"),
            (p + "q.bias", (D_MODEL,), "b"),
            (p + "k.weight", (D_MODEL, D_MODEL), "w"),
            (p + "k.bias", (D_MODEL,), "b"),
            (p + "v.weight", (D_MODEL, D_MODEL), "w"),
            (p + "v.bias", (D_MODEL,), "b"),
            (p + "o.weight", (D_MODEL, D_MODEL), "w"),
            (p + "o.bias", (D_MODEL,), "b"),
            (p + "ln2.weight", (D_MODEL,), "g"),
            (p + "ln2.bias", (D_MODEL,), "beta"),
            (p + "fc1.weight", (D_FFN, D_MODEL), "w"),
            (p + "fc1.bias", (D_FFN,), "b"),
            (p + "fc2.weight", (D_MODEL, D_FFN), "w"),
            (p + "fc2.bias", (D_MODEL,), "b"),
        ]
    m += [
        ("ln_post.weight", (D_MODEL,), "g"),
        ("ln_post.bias", (D_MODEL,), "beta"),
        ("proj1.weight", (D_MODEL, D_MODEL), "w"),
        ("proj1.bias", (D_MODEL,), "b"),
        ("proj2.weight", (D_OUT, D_MODEL), "w"),
        ("proj2.bias", (D_OUT,), "b"),
        ("adapter.gate.weight", (D_ADAPTER, D_OUT), "w"),
        ("adapter.gate.bias", (D_ADAPTER,), "b"),
        ("adapter.up.weight", (D_ADAPTER, D_OUT), "w"),
        ("adapter.up.bias", (D_ADAPTER,), "b"),
        ("adapter.down.weight", (D_OUT, D_ADAPTER), "w"),
        ("adapter.down.bias", (D_OUT,), "b"),
    ]
    return m


def weight_offsets(n_layers: int):
    """{name: (offset_in_elements, shape)} and the total element count."""
    off = 0
    table = {}
    for name, shape, _ in weight_manifest(n_layers):
        table[name] = (off, shape)
        off += int(np.prod(shape))
    return table, off


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp32 to bf16 (nearest, ties to even); returns uint16 bit patterns."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    rounding = ((u >> 16) & 1) + np.uint32(0x7FFF)
    return ((u + rounding) >> 16).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def make_weights(n_layers: int, seed: int = 1234) -> np.ndarray:
    """The whole weight blob as a flat uint16 array of bf16 bits."""
    rng = np.random.Generator(np.random.PCG64(seed))
    table, total = weight_offsets(n_layers)
    blob = np.empty(total, dtype=np.uint16)
    for name, shape, kind in weight_manifest(n_layers):
        off, _ = table[name]
        n = int(np.prod(shape))
        if kind == "w":
            fan_in = int(np.prod(shape[1:]))
            v = rng.standard_normal(n, dtype=np.float32) * np.float32(1.0 / np.sqrt(fan_in))
        elif kind == "b":
            v = rng.standard_normal(n, dtype=np.float32) * np.float32(0.01)
        elif kind == "g":
            v = np.ones(n, dtype=np.float32)
        else:
            v = np.zeros(n, dtype=np.float32)
        blob[off:off + n] = f32_to_bf16_bits(v)
    return blob


def head_manifest():
    """(name, shape, kind) of one head + adapter set: the tail of the blob
    after the layers, which is also the layout of one layer tap's set."""
    m = weight_manifest(0)
    first = [name for name, _, _ in m].index("ln_post.weight")
    return m[first:]


def make_tap_weights(n_taps: int, seed: int = 4321) -> np.ndarray:
    """n_taps consecutive head + adapter sets (bf16 bits), initialised like
    the blob's own: N(0, 1/fan_in) matrices, N(0, 0.01^2) biases, LayerNorm
    gamma 1 and beta 0."""
    rng = np.random.Generator(np.random.PCG64(seed))
    parts = []
    for _ in range(n_taps):
        for _name, shape, kind in head_manifest():
            n = int(np.prod(shape))
            if kind == "w":
                v = rng.standard_normal(n, dtype=np.float32) * np.float32(1.0 / np.sqrt(int(np.prod(shape[1:]))))
            elif kind == "b":
                v = rng.standard_normal(n, dtype=np.float32) * np.float32(0.01)
            elif kind == "g":
                v = np.ones(n, dtype=np.float32)
            else:
                v = np.zeros(n, dtype=np.float32)
            parts.append(f32_to_bf16_bits(v))
    return np.concatenate(parts) if parts else np.empty(0, dtype=np.uint16)


def _tones(rng, n: int, t0: int = 0) -> np.ndarray:
    t = (np.arange(n, dtype=np.float64) + t0) / SAMPLE_RATE
    freqs = rng.uniform(100.0, 6000.0, size=3)
    amps = rng.uniform(0.1, 0.3, size=3)
    phases = rng.uniform(0.0, 2.0 * np.pi, size=3)
    x = np.zeros(n, dtype=np.float64)
    for f, a, p in zip(freqs, amps, phases):
        x += a * np.sin(2.0 * np.pi * f * t + p)
    return x


def pcm_tones(seed: int, n_samples: int) -> np.ndarray:
    """Three sines plus N(0, 0.01^2) noise (the Tiny recipe)."""
    rng = np.random.Generator(np.random.PCG64(seed))
    x = _tones(rng, n_samples)
    x += rng.standard_normal(n_samples) * 0.01
    return x.astype(np.float32)


def pcm_30s(seed: int = 1, n_samples: int = 480000) -> np.ndarray:
    """Tones plus 5 s of 300-3400 Hz band-limited noise over seconds 12-17."""
    rng = np.random.Generator(np.random.PCG64(seed))
    x = _tones(rng, n_samples)
    x += rng.standard_normal(n_samples) * 0.01
    a, b = 12 * SAMPLE_RATE, min(17 * SAMPLE_RATE, n_samples)
    if b > a:
        seg = rng.standard_normal(b - a) * 0.05
        spec = np.fft.rfft(seg)
        f = np.fft.rfftfreq(b - a, 1.0 / SAMPLE_RATE)
        spec[(f < 300.0) | (f > 3400.0)] = 0.0
        x[a:b] += np.fft.irfft(spec, n=b - a)
    return x.astype(np.float32)


def pcm_long(seed: int, n_samples: int, segment_s: float = 2.0) -> np.ndarray:
    """Tones redrawn every ``segment_s`` seconds plus N(0, 0.01^2) noise."""
    rng = np.random.Generator(np.random.PCG64(seed))
    seg = int(segment_s * SAMPLE_RATE)
    out = np.empty(n_samples, dtype=np.float32)
    for s in range(0, n_samples, seg):
        e = min(s + seg, n_samples)
        out[s:e] = _tones(rng, e - s, t0=s)
    out += (rng.standard_normal(n_samples, dtype=np.float32) * np.float32(0.01))
    return out


def batch_lengths(n_clips: int = 16):
    return [int(np.random.Generator(np.random.PCG64(i)).integers(160000, 480001))
            for i in range(n_clips)]


def pcm_batch(n_clips: int = 16):
    """Clip i: seed i, length uniform in [160000, 480000] samples, tones recipe."""
    clips = []
    for i in range(n_clips):
        rng = np.random.Generator(np.random.PCG64(i))
        n = int(rng.integers(160000, 480001))
        x = _tones(rng, n)
        x += rng.standard_normal(n) * 0.01
        clips.append(x.astype(np.float32))
    return clips


# Workloads by name: (description, builder returning a list of clips, n_layers)
WORKLOADS = {
    "tiny_1s": ("1 s tones clip, 4 layers", lambda: [pcm_tones(0, 16000)], 4),
    "single_30s": ("one 30 s clip with band noise, 32 layers", lambda: [pcm_30s(1)], 32),
    "batch16_10to30s": ("16 clips of 10-30 s, 32 layers", lambda: pcm_batch(16), 32),
    "clip_10min": ("one 10-min clip, tones redrawn every 2 s, 32 layers",
                   lambda: [pcm_long(2, 9_600_000)], 32),
    "clip_60min_streamed": ("one 60-min clip in 64 s pieces, 32 layers",
                            lambda: [pcm_long(3, 57_600_000)], 32),
}
