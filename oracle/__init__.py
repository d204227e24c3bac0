"""Python handle on the CPU oracle (``moss_oracle.c``).

Test infrastructure only: the tests, the smoke check and the benchmark's
CPU-baseline leg use it. The product path never imports this package.
``build()`` compiles the C file into ``oracle/libmoss_oracle.so`` with gcc.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moss_oracle.c")
_LIB = os.path.join(_HERE, "libmoss_oracle.so")

N_MELS = 128
N_BINS = 201
D_MODEL = 1280
D_OUT = 2048
CHUNK_FRAMES = 800

_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (-O3, OpenMP, AVX2 baseline)."""
    if not force and os.path.exists(_LIB) and os.path.getmtime(_LIB) >= os.path.getmtime(_SRC):
        return _LIB
    tmp = _LIB + f".tmp{os.getpid()}"
    cmd = ["gcc", "-std=gnu11", "-O3", "-march=x86-64-v3", "-fopenmp", "-fPIC", "-shared",
           "-o", tmp, _SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB)
    return _LIB


def lib():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        L = _lib
        i64, i32, f32 = ctypes.c_int64, ctypes.c_int, ctypes.c_float
        vp = ctypes.c_void_p
        L.oracle_num_frames.restype = i64
        L.oracle_num_frames.argtypes = [i64]
        L.oracle_num_tokens.restype = i64
        L.oracle_num_tokens.argtypes = [i64]
        L.oracle_num_chunks.restype = i64
        L.oracle_num_chunks.argtypes = [i64]
        L.oracle_chunk_tokens.restype = i64
        L.oracle_chunk_tokens.argtypes = [i64]
        L.oracle_hann.argtypes = [vp]
        L.oracle_mel_filters.argtypes = [vp]
        L.oracle_frame_power.argtypes = [vp, i64, i64, vp]
        L.oracle_logmel_raw.argtypes = [vp, i64, i64, i64, vp]
        L.oracle_max.restype = f32
        L.oracle_max.argtypes = [vp, i64]
        L.oracle_normalize.argtypes = [vp, i64, f32]
        L.oracle_clip_log_max.restype = f32
        L.oracle_clip_log_max.argtypes = [vp, i64]
        L.oracle_logmel.restype = f32
        L.oracle_logmel.argtypes = [vp, i64, vp]
        L.oracle_position.restype = ctypes.c_double
        L.oracle_position.argtypes = [i32, i32]
        L.oracle_model_create.restype = vp
        L.oracle_model_create.argtypes = [vp, i32]
        L.oracle_model_destroy.argtypes = [vp]
        L.oracle_weight_count.restype = i64
        L.oracle_weight_count.argtypes = [i32]
        L.oracle_stem_chunk.restype = i32
        L.oracle_stem_chunk.argtypes = [vp, vp, i32, vp]
        L.oracle_layers.restype = i32
        L.oracle_layers.argtypes = [vp, vp, i32, vp, i32, i32, i32, i32]
        L.oracle_head.restype = i32
        L.oracle_head.argtypes = [vp, vp, i32, vp]
        L.oracle_adapter.restype = i32
        L.oracle_adapter.argtypes = [vp, vp, i32, vp]
        L.oracle_encode_chunks.restype = i64
        L.oracle_encode_chunks.argtypes = [vp, vp, i64, i64, i64, f32, i32, vp, vp, vp, vp]
        L.oracle_model_create_bits.restype = vp
        L.oracle_model_create_bits.argtypes = [vp, i32, i32]
        L.oracle_quant_rtn4.argtypes = [vp, i32, i32, vp, vp, vp]
        L.oracle_e4m3.restype = f32
        L.oracle_e4m3.argtypes = [f32]
        L.oracle_quant_e4m3_rows.argtypes = [vp, i32, i32, vp, vp]
        L.oracle_e2m1.restype = f32
        L.oracle_e2m1.argtypes = [f32]
        L.oracle_quant_nvfp4.argtypes = [vp, i64, i32, i32, vp, vp, vp, vp]
        L.oracle_model_create_nvfp4.restype = vp
        L.oracle_model_create_nvfp4.argtypes = [vp, i32]
        L.oracle_set_threads.argtypes = [i32]
        L.oracle_max_threads.restype = i32
    return _lib


def _p(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _f32(a):
    return np.ascontiguousarray(a, dtype=np.float32)


def set_threads(n: int) -> None:
    lib().oracle_set_threads(int(n))


def max_threads() -> int:
    return int(lib().oracle_max_threads())


def num_frames(n: int) -> int:
    return int(lib().oracle_num_frames(n))


def num_tokens(n: int) -> int:
    return int(lib().oracle_num_tokens(n))


def num_chunks(n: int) -> int:
    return int(lib().oracle_num_chunks(n))


def chunk_tokens(frames: int) -> int:
    return int(lib().oracle_chunk_tokens(frames))


def hann() -> np.ndarray:
    w = np.empty(400, dtype=np.float64)
    lib().oracle_hann(_p(w))
    return w


def mel_filters() -> np.ndarray:
    W = np.empty((N_MELS, N_BINS), dtype=np.float64)
    lib().oracle_mel_filters(_p(W))
    return W


def frame_power(pcm, t: int) -> np.ndarray:
    pcm = _f32(pcm)
    P = np.empty(N_BINS, dtype=np.float64)
    lib().oracle_frame_power(_p(pcm), pcm.size, int(t), _p(P))
    return P


def logmel_raw(pcm, f0: int = 0, f1: int | None = None) -> np.ndarray:
    pcm = _f32(pcm)
    if f1 is None:
        f1 = num_frames(pcm.size)
    out = np.empty((max(f1 - f0, 0), N_MELS), dtype=np.float32)
    if f1 > f0:
        lib().oracle_logmel_raw(_p(pcm), pcm.size, int(f0), int(f1), _p(out))
    return out


def normalize(raw: np.ndarray, gmax: float) -> np.ndarray:
    out = np.array(raw, dtype=np.float32, copy=True, order="C")
    lib().oracle_normalize(_p(out), out.size, float(gmax))
    return out


def clip_log_max(pcm) -> float:
    pcm = _f32(pcm)
    return float(lib().oracle_clip_log_max(_p(pcm), pcm.size))


def logmel(pcm):
    """Normalised log-mel [F][128] and the clip's log-mel maximum."""
    pcm = _f32(pcm)
    F = num_frames(pcm.size)
    out = np.empty((F, N_MELS), dtype=np.float32)
    if F == 0:
        return out, float("-inf")
    mx = lib().oracle_logmel(_p(pcm), pcm.size, _p(out))
    return out, float(mx)


def position(p: int, c: int) -> float:
    return float(lib().oracle_position(p, c))


def weight_count(n_layers: int) -> int:
    return int(lib().oracle_weight_count(n_layers))


def quant_rtn4(w: np.ndarray):
    """4-bit round-to-nearest quantisation in groups of 128 along the last
    axis of a bf16 matrix (uint16 bits) [rows][cols]: returns (w' as bf16
    bits, codes q + 8 as uint8, scales [rows][cols / 128] fp32)."""
    w = np.ascontiguousarray(w, dtype=np.uint16)
    rows, cols = w.shape
    if cols % 128:
        raise ValueError("cols must be a multiple of 128")
    deq = np.empty_like(w)
    codes = np.empty((rows, cols), dtype=np.uint8)
    scales = np.empty((rows, cols // 128), dtype=np.float32)
    lib().oracle_quant_rtn4(_p(w), rows, cols, _p(deq), _p(codes), _p(scales))
    return deq, codes, scales


def e4m3(x: float) -> float:
    """The nearest e4m3 value (ties to even, saturating at +-448)."""
    return float(lib().oracle_e4m3(float(x)))


def quant_e4m3_rows(w: np.ndarray):
    """Per-row e4m3 quantisation of a bf16 matrix (uint16 bits) [rows][cols]:
    returns (e4m3 values as bf16 bits, scales [rows] fp32), row max -> 448."""
    w = np.ascontiguousarray(w, dtype=np.uint16)
    rows, cols = w.shape
    q = np.empty_like(w)
    s = np.empty(rows, dtype=np.float32)
    lib().oracle_quant_e4m3_rows(_p(w), rows, cols, _p(q), _p(s))
    return q, s


def e2m1(x: float) -> float:
    """The nearest E2M1 value (ties to even, saturating at +-6)."""
    return float(lib().oracle_e2m1(float(x)))


def quant_nvfp4(x: np.ndarray, per_row: bool):
    """NVFP4 quantisation of x [rows][cols] (cols a multiple of 16): returns
    (units q * s_b [rows][cols] fp32, g [rows] or [1] fp32, E2M1 codes
    [rows][cols] uint8 (sign bit 3), block scales [rows][cols / 16] fp32)."""
    x = _f32(x)
    rows, cols = x.shape
    if cols % 16:
        raise ValueError("cols must be a multiple of 16")
    unit = np.empty_like(x)
    g = np.empty(rows if per_row else 1, dtype=np.float32)
    codes = np.empty((rows, cols), dtype=np.uint8)
    bs = np.empty((rows, cols // 16), dtype=np.float32)
    lib().oracle_quant_nvfp4(_p(x), rows, cols, int(per_row), _p(unit), _p(g), _p(codes), _p(bs))
    return unit, g, codes, bs


class Model:
    """The oracle's copy of a bf16 weight blob (uint16 bit patterns);
    weight_bits=4 gives the model with 4-bit quantised linear layers, 8 the
    model whose q, k, v and fc1 GEMMs take e4m3 operands; nvfp4=True the model
    whose q, k, v and fc1 GEMMs take NVFP4 operands."""

    def __init__(self, blob: np.ndarray, n_layers: int, weight_bits: int = 16, nvfp4: bool = False):
        blob = np.ascontiguousarray(blob, dtype=np.uint16)
        if blob.size != weight_count(n_layers):
            raise ValueError(f"blob has {blob.size} elements, expected {weight_count(n_layers)}")
        self._blob = blob  # the model points into it
        self.n_layers = n_layers
        if nvfp4:
            self._h = lib().oracle_model_create_nvfp4(_p(blob), n_layers)
        else:
            self._h = lib().oracle_model_create_bits(_p(blob), n_layers, int(weight_bits))

    def close(self):
        if self._h:
            lib().oracle_model_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def stem_chunk(self, mel_norm) -> np.ndarray:
        mel_norm = _f32(mel_norm)
        fc = mel_norm.shape[0]
        out = np.empty((chunk_tokens(fc), D_MODEL), dtype=np.float32)
        lib().oracle_stem_chunk(self._h, _p(mel_norm), fc, _p(out))
        return out

    def layers(self, x, windows, l0: int = 0, l1: int | None = None, attn_full: bool = False):
        """Run layers [l0, l1) in place on a copy of x; windows = token offsets."""
        x = np.array(x, dtype=np.float32, copy=True, order="C")
        win = np.ascontiguousarray(windows, dtype=np.int32)
        l1 = self.n_layers if l1 is None else l1
        lib().oracle_layers(self._h, _p(x), x.shape[0], _p(win), win.size - 1, l0, l1,
                            int(attn_full))
        return x

    def head(self, x) -> np.ndarray:
        x = _f32(x)
        out = np.empty((x.shape[0], D_OUT), dtype=np.float32)
        lib().oracle_head(self._h, _p(x), x.shape[0], _p(out))
        return out

    def adapter(self, h) -> np.ndarray:
        h = _f32(h)
        out = np.empty((h.shape[0], D_OUT), dtype=np.float32)
        lib().oracle_adapter(self._h, _p(h), h.shape[0], _p(out))
        return out

    def encode_chunks(self, pcm, c0: int = 0, c1: int | None = None, gmax: float = float("nan"),
                      attn_full: bool = False, dumps: bool = False):
        """Rows [T][2048] of chunks [c0, c1) of one clip (optionally with dumps)."""
        pcm = _f32(pcm)
        nc = num_chunks(pcm.size)
        c1 = nc if c1 is None else min(c1, nc)
        F = num_frames(pcm.size)
        T = 0
        for c in range(c0, c1):
            T += chunk_tokens(min(800, F - 800 * c))
        out = np.empty((T, D_OUT), dtype=np.float32)
        ds = de = dh = None
        if dumps:
            ds = np.empty((T, D_MODEL), dtype=np.float32)
            de = np.empty((T, D_MODEL), dtype=np.float32)
            dh = np.empty((T, D_OUT), dtype=np.float32)
        got = lib().oracle_encode_chunks(
            self._h, _p(pcm), pcm.size, c0, c1, float(gmax), int(attn_full), _p(out),
            _p(ds) if dumps else None, _p(de) if dumps else None, _p(dh) if dumps else None)
        assert got == T, (got, T)
        if dumps:
            return out, {"stem": ds, "enc": de, "head": dh}
        return out

    def encode(self, pcm, **kw):
        return self.encode_chunks(pcm, 0, None, **kw)
