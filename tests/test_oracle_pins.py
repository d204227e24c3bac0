"""Pins for the CPU oracle: page facts, closed forms, library routines and
invariants. None of these reads the CUDA path."""
import json
import os

import numpy as np
import pytest
import torch

import oracle
from audio_encoder_b200 import synth
from conftest import oracle_model, weights

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def facts():
    with open(os.path.join(GOLDEN, "page_facts.json")) as f:
        return json.load(f)


# ----------------------------------------------------------------- counts

def test_token_counts_match_pages():
    fx = facts()
    for n, t in fx["workload_token_counts"]["value"].items():
        assert oracle.num_tokens(int(n)) == t


def test_frames_drop_trailing_stft_frame():
    # n // hop frames: a centred STFT gives n//hop + 1, the last is dropped.
    for n in [0, 1, 159, 160, 161, 16000, 16159, 480000, 480001]:
        assert oracle.num_frames(n) == n // 160


def test_token_rate_is_12_5_hz():
    rate = facts()["token_rate_hz"]["value"]
    for seconds in [8, 16, 64, 600, 3600]:
        assert oracle.num_tokens(16000 * seconds) == rate * seconds


def test_chunk_tokens_are_ceil_div_8():
    # three stride-2 convs: 100 frames/s -> 12.5 tokens/s
    for fc in range(0, 801):
        assert oracle.chunk_tokens(fc) == -(-fc // 8)


def test_parameter_count_matches_pages():
    fx = facts()
    n_enc = oracle.weight_count(32)
    table, total = synth.weight_offsets(32)
    assert total == n_enc
    adapter = sum(int(np.prod(s)) for name, (o, s) in table.items() if name.startswith("adapter"))
    enc = total - adapter
    assert abs(enc / 1e9 - fx["encoder_params_billion"]["value"]) < 0.005
    w = fx["conv_out_in_width"]
    assert table["conv_out.weight"][1] == (fx["d_model"]["value"], w["value"])
    assert w["factors"][0] * w["factors"][1] == w["value"]


# ------------------------------------------------------------- front end

def test_hann_is_periodic():
    import scipy.signal
    np.testing.assert_allclose(oracle.hann(), scipy.signal.get_window("hann", 400), atol=1e-15)


def test_tone_on_bin_closed_form():
    # A cosine on bin k with amplitude A: the periodic-Hann DFT has weights
    # 1/2, -1/4, -1/4 on bins k, k+-1, so |X_k|^2 = (100 A)^2 and
    # |X_{k+-1}|^2 = (50 A)^2, zero elsewhere (frames fully inside the clip).
    A, k = 0.25, 37
    n = np.arange(16000)
    pcm = (A * np.cos(2 * np.pi * 40.0 * k * n / 16000 + 0.3)).astype(np.float32)
    P = oracle.frame_power(pcm, 20)
    assert P[k] == pytest.approx((100 * A) ** 2, rel=1e-5)
    assert P[k - 1] == pytest.approx((50 * A) ** 2, rel=1e-4)
    assert P[k + 1] == pytest.approx((50 * A) ** 2, rel=1e-4)
    rest = np.delete(P, [k - 1, k, k + 1])
    assert rest.max() < 1e-6 * P[k]


def test_frame_power_vs_numpy_rfft_with_reflect_pad():
    pcm = synth.pcm_tones(5, 4000)
    padded = np.pad(pcm.astype(np.float64), 200, mode="reflect")
    w = np.hanning(401)[:-1]
    for t in [0, 1, 2, 12, 23, 24]:
        ref = np.abs(np.fft.rfft(padded[160 * t:160 * t + 400] * w)) ** 2
        np.testing.assert_allclose(oracle.frame_power(pcm, t), ref, rtol=1e-9, atol=1e-12)


def test_impulse_lands_in_frames_within_200_samples():
    n = 8000
    for s in [1000, 1160, 4321]:
        pcm = np.zeros(n, dtype=np.float32)
        pcm[s] = 1.0
        for t in range(n // 160):
            e = oracle.frame_power(pcm, t).sum()
            assert (e > 0) == (abs(160 * t - s) < 200), (s, t)


def test_mel_filters_vs_torchaudio():
    import torchaudio
    ref = torchaudio.functional.melscale_fbanks(201, 0.0, 8000.0, 128, 16000, norm="slaney",
                                                mel_scale="slaney").double().numpy().T
    np.testing.assert_allclose(oracle.mel_filters(), ref, rtol=1e-5, atol=5e-7)  # torchaudio builds it in fp32


def test_mel_filter_area_and_scale():
    W = oracle.mel_filters()
    f = 40.0 * np.arange(201)
    centroid = (W * f).sum(1) / W.sum(1)
    # area normalisation: each wide triangle integrates to 1 over Hz
    # (sampled at 40 Hz, so only approximately for the narrower ones)
    assert np.all(np.abs(W[centroid > 2000].sum(1) * 40.0 - 1.0) < 0.1)
    assert np.all(np.abs(W[centroid > 5000].sum(1) * 40.0 - 1.0) < 0.02)
    # Slaney scale: linear spacing below 1 kHz, constant ratio above
    # (below 1 kHz the triangles are narrower than a 40 Hz bin, so centroids
    # are quantised: check a straight-line fit to within half a bin)
    m = np.arange(128)
    lo = (centroid > 200) & (centroid < 900)
    fit = np.polyval(np.polyfit(m[lo], centroid[lo], 1), m[lo])
    assert np.abs(fit - centroid[lo]).max() < 20.0
    hi = centroid > 2000
    fit = np.polyval(np.polyfit(m[hi], np.log(centroid[hi]), 1), m[hi])
    assert np.abs(fit - np.log(centroid[hi])).max() < 0.01


def test_pure_tone_lands_in_predicted_mel_bin():
    # Predicted bin: the filter whose centre (on the Slaney scale, 128
    # filters over 0..8 kHz, centre m at mel (m+1) * mel(8000)/129) is the
    # tone frequency.  Above 1 kHz the scale is 15 + 27 ln(f/1000)/ln(6.4).
    mel_max = 15.0 + 27.0 * np.log(8.0) / np.log(6.4)
    n = np.arange(16000)
    for m in [40, 60, 80, 100, 120]:
        mm = (m + 1) * mel_max / 129.0
        f = 1000.0 * np.exp((mm - 15.0) * np.log(6.4) / 27.0)
        pcm = (0.2 * np.sin(2 * np.pi * f * n / 16000)).astype(np.float32)
        raw = oracle.logmel_raw(pcm, 40, 60)
        assert np.all(raw.argmax(1) == m), (m, f, raw.argmax(1))


def test_logmel_of_silence_is_minus_1_5():
    mel, mx = oracle.logmel(np.zeros(4800, dtype=np.float32))
    assert mx == pytest.approx(-10.0)
    np.testing.assert_array_equal(mel, np.full((30, 128), -1.5, dtype=np.float32))


def test_logmel_closed_form_on_bin_tone():
    # mel_m = sum_k W[m,k] P_k with P from the on-bin closed form; log10.
    A, k = 0.2, 50
    n = np.arange(16000)
    pcm = (A * np.cos(2 * np.pi * 40.0 * k * n / 16000)).astype(np.float32)
    W = oracle.mel_filters()
    P = np.zeros(201)
    P[k], P[k - 1], P[k + 1] = (100 * A) ** 2, (50 * A) ** 2, (50 * A) ** 2
    mel = W @ P
    ref = np.log10(np.maximum(mel, 1e-10))
    raw = oracle.logmel_raw(pcm, 10, 11)[0]
    big = mel > 1e-3
    np.testing.assert_allclose(raw[big], ref[big], atol=1e-5)


def test_floor_and_scale():
    raw = np.array([[0.0, -3.0, -8.0, -9.5, -20.0]], dtype=np.float32)
    out = oracle.normalize(raw, 0.0)
    np.testing.assert_allclose(out[0], [1.0, 0.25, -1.0, -1.0, -1.0])


@pytest.mark.parametrize("n", [16000, 16100, 480000])
def test_logmel_vs_whisper_feature_extractor(n):
    from transformers import WhisperFeatureExtractor
    fe = WhisperFeatureExtractor(feature_size=128)
    pcm = synth.pcm_30s(1, n) if n == 480000 else synth.pcm_tones(3, n)
    ref = fe(pcm, sampling_rate=16000, return_tensors="np", padding="longest")["input_features"][0].T
    mel, _ = oracle.logmel(pcm)
    assert mel.shape == ref.shape == (n // 160, 128)
    np.testing.assert_allclose(mel, ref, atol=1e-4)  # the extractor works in fp32


# ------------------------------------------------------------- positions

def test_positions_special_cases():
    for p in [0, 1, 7, 99]:
        assert oracle.position(p, 0) == pytest.approx(np.sin(p), abs=1e-15)
        assert oracle.position(p, 640) == pytest.approx(np.cos(p), abs=1e-15)
        assert oracle.position(p, 639) == pytest.approx(np.sin(p / 10000.0), abs=1e-15)
        assert oracle.position(p, 1279) == pytest.approx(np.cos(p / 10000.0), abs=1e-15)
    for c in range(640):
        assert oracle.position(0, c) == 0.0
        assert oracle.position(0, 640 + c) == 1.0


def test_positions_pair_channels_and_geometric_frequencies():
    # every channel c < 640 and its partner 640 + c are the sine and cosine of
    # one angle (sin^2 + cos^2 = 1, and the angle grows linearly with the
    # position), and the angle rates fall geometrically from 1 to 1/10000
    # over the 640 channels (log-rate linear in c with step ln(10^4)/639)
    rates = np.empty(640)
    for c in range(640):
        s1, c1 = oracle.position(1, c), oracle.position(1, 640 + c)
        assert s1 * s1 + c1 * c1 == pytest.approx(1.0, abs=1e-12)
        rates[c] = np.arctan2(s1, c1)  # angle at p = 1 (below pi: rates <= 1)
        s3, c3 = oracle.position(3, c), oracle.position(3, 640 + c)
        assert np.arctan2(s3, c3) == pytest.approx(np.angle(np.exp(3j * rates[c])), abs=1e-12)
    steps = np.diff(np.log(rates))
    np.testing.assert_allclose(steps, -np.log(10000.0) / 639.0, rtol=1e-9)
    assert rates[0] == pytest.approx(1.0, abs=1e-15) and rates[639] == pytest.approx(1e-4, rel=1e-12)


# ----------------------------------------------------- model vs library

def _tref(n_layers):
    from torch_ref import TorchRef
    return TorchRef(weights(n_layers), n_layers)


@pytest.fixture(scope="module")
def tref4():
    return _tref(4)


@pytest.mark.parametrize("fc", [800, 100, 37])
def test_stem_vs_torch_conv2d(om4, tref4, fc):
    rng = np.random.default_rng(fc)
    mel = rng.uniform(-1.0, 1.5, size=(fc, 128)).astype(np.float32)
    got = om4.stem_chunk(mel)
    ref = tref4.stem_chunk(mel).numpy()
    assert got.shape == ref.shape == (-(-fc // 8), 1280)
    np.testing.assert_allclose(got, ref, rtol=1e-4, atol=1e-4)


def test_stem_tail_is_zero_padding(om4):
    rng = np.random.default_rng(7)
    mel = rng.uniform(-1.0, 1.5, size=(203, 128)).astype(np.float32)
    padded = np.zeros((800, 128), dtype=np.float32)
    padded[:203] = mel
    a = om4.stem_chunk(mel)
    b = om4.stem_chunk(padded)[: a.shape[0]]
    np.testing.assert_array_equal(a, b)


def test_layers_vs_torch(om4, tref4):
    rng = np.random.default_rng(1)
    x = rng.standard_normal((57, 1280)).astype(np.float32)
    windows = [0, 20, 21, 57]
    got = om4.layers(x, windows)
    ref = tref4.layers(torch.from_numpy(x.astype(np.float64)), windows).numpy()
    np.testing.assert_allclose(got, ref, rtol=1e-4, atol=1e-4)


def test_blockdiag_equals_full_masked(om4):
    rng = np.random.default_rng(2)
    x = rng.standard_normal((130, 1280)).astype(np.float32)
    windows = [0, 100, 101, 130]
    a = om4.layers(x, windows, attn_full=False)
    b = om4.layers(x, windows, attn_full=True)
    np.testing.assert_allclose(a, b, rtol=0, atol=1e-6)


def test_head_and_adapter_vs_torch(om4, tref4):
    rng = np.random.default_rng(3)
    x = rng.standard_normal((9, 1280)).astype(np.float32) * 2
    h = om4.head(x)
    href = tref4.head(torch.from_numpy(x.astype(np.float64)))
    np.testing.assert_allclose(h, href.numpy(), rtol=1e-4, atol=1e-4)
    y = om4.adapter(h)
    yref = tref4.adapter(torch.from_numpy(h.astype(np.float64))).numpy()
    np.testing.assert_allclose(y, yref, rtol=1e-4, atol=2e-4)


# ------------------------------------------------------------- invariants

def test_locality_per_window(om4):
    # Perturbing the audio of chunk 1 (away from its 200-sample halo) leaves the
    # rows of chunks 0 and 2 unchanged when the log-mel maximum is held fixed.
    n = 128000 * 2 + 48000
    pcm = synth.pcm_tones(11, n)
    gmax = oracle.clip_log_max(pcm)
    base = om4.encode(pcm, gmax=gmax)
    p2 = pcm.copy()
    p2[128000 + 1000:256000 - 1000] *= 0.5
    pert = om4.encode(p2, gmax=gmax)
    np.testing.assert_array_equal(base[:100], pert[:100])
    np.testing.assert_array_equal(base[200:], pert[200:])
    assert np.abs(base[100:200] - pert[100:200]).max() > 1e-3


def test_chunk_ranges_concatenate_to_whole_clip(om4):
    n = 128000 + 30000
    pcm = synth.pcm_tones(12, n)
    whole = om4.encode(pcm)
    parts = np.concatenate([om4.encode_chunks(pcm, 0, 1), om4.encode_chunks(pcm, 1, 2)])
    np.testing.assert_array_equal(whole, parts)
    assert whole.shape == (oracle.num_tokens(n), 2048)


def test_deterministic(om4):
    pcm = synth.pcm_tones(0, 16000)
    a = om4.encode(pcm)
    b = om4.encode(pcm)
    np.testing.assert_array_equal(a, b)
    assert a.shape == (13, 2048)


def test_empty_and_short_clips(om4):
    for n in [0, 100, 159]:
        out = om4.encode(np.zeros(n, dtype=np.float32) + 0.01)
        assert out.shape == (0, 2048)
    out = om4.encode(synth.pcm_tones(4, 170))
    assert out.shape == (1, 2048)
    assert np.isfinite(out).all()


def test_stored_tiny_rows_regression(om4):
    # Rows written by tests/golden/make_golden.py, which calls only the oracle.
    path = os.path.join(GOLDEN, "tiny_oracle_rows.json")
    with open(path) as f:
        g = json.load(f)
    out = om4.encode(synth.pcm_tones(0, 16000))
    np.testing.assert_allclose(out[:, :8], np.array(g["rows_first8"]), rtol=1e-5, atol=1e-5)
    np.testing.assert_allclose(np.linalg.norm(out, axis=1), np.array(g["row_norms"]), rtol=1e-5)
