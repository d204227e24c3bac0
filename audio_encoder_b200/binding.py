"""Thin ctypes binding of the moss_enc C ABI (``include/moss_enc.h``).

Argument marshalling only: every step of the encoder runs in the CUDA
library.  PyTorch provides device memory and the stream.  Loading fails
loudly if ``libmoss_enc.so`` has not been built; there is no fallback.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libmoss_enc.so")

OK = 0
STATUS = {0: "ok", 1: "invalid argument", 2: "capacity", 3: "out of memory", 4: "cuda error",
          5: "device timeout"}
OUT_F32, OUT_BF16 = 0, 1
STAGE_STEM, STAGE_LAYERS, STAGE_HEAD, STAGE_ADAPTER = 0, 1, 2, 3
D_MODEL, D_OUT = 1280, 2048

EXPORTED = [
    "moss_enc_weight_count", "moss_enc_num_frames", "moss_enc_num_tokens", "moss_enc_range_tokens",
    "moss_enc_create", "moss_enc_set_stream", "moss_enc_synchronize", "moss_enc_destroy",
    "moss_enc_status_string", "moss_enc_last_error", "moss_enc_logmel", "moss_enc_log_max",
    "moss_enc_range_log_max",
    "moss_enc_forward", "moss_enc_forward_stage", "moss_enc_forward_host",
    "moss_enc_tap_weight_count", "moss_enc_set_taps", "moss_enc_forward_taps",
    "moss_enc_profile_enable", "moss_enc_profile_read", "moss_enc_launch_count",
    "moss_enc_logmel_static", "moss_enc_gemm", "moss_enc_gemm_q4", "moss_enc_gemm_f8", "moss_enc_gemm_nvf4", "moss_enc_nvf4_quant_rows",
    "moss_enc_nvf4_quant_weights",
    "moss_enc_selftest_gelu",
    "moss_enc_selftest_timeout",
]
WEIGHTS_4BIT = 4
STATIC_MAX_CLIPS = 64


class MossEncError(RuntimeError):
    def __init__(self, status: int, msg: str = ""):
        super().__init__(f"moss_enc status {status} ({STATUS.get(status, '?')}): {msg}")
        self.status = status


class Config(ctypes.Structure):
    _fields_ = [("n_layers", ctypes.c_int), ("max_samples", ctypes.c_int64),
                ("max_clips", ctypes.c_int), ("out_dtype", ctypes.c_int), ("weight_bits", ctypes.c_int),
                ("fp8", ctypes.c_int), ("nvfp4", ctypes.c_int)]


class KernelStat(ctypes.Structure):
    _fields_ = [("name", ctypes.c_char * 32), ("launches", ctypes.c_int64), ("ms", ctypes.c_double),
                ("flops", ctypes.c_double), ("bytes", ctypes.c_double)]


class Clip(ctypes.Structure):
    _fields_ = [("pcm", ctypes.c_void_p), ("n_samples", ctypes.c_int64), ("begin", ctypes.c_int64),
                ("end", ctypes.c_int64), ("log_max", ctypes.c_void_p)]


_lib = None


def lib():
    """The loaded library (raises if it is missing)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is not built; run `python -m audio_encoder_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        i64, i32, vp = ctypes.c_int64, ctypes.c_int, ctypes.c_void_p
        L.moss_enc_weight_count.restype = i64
        L.moss_enc_weight_count.argtypes = [i32]
        L.moss_enc_num_frames.restype = i64
        L.moss_enc_num_frames.argtypes = [i64]
        L.moss_enc_num_tokens.restype = i64
        L.moss_enc_num_tokens.argtypes = [i64]
        L.moss_enc_range_tokens.restype = i64
        L.moss_enc_range_tokens.argtypes = [i64, i64, i64]
        L.moss_enc_create.restype = i32
        L.moss_enc_create.argtypes = [ctypes.POINTER(Config), vp, ctypes.c_size_t, i32, vp, ctypes.POINTER(vp)]
        L.moss_enc_set_stream.restype = i32
        L.moss_enc_set_stream.argtypes = [vp, vp]
        L.moss_enc_synchronize.restype = i32
        L.moss_enc_synchronize.argtypes = [vp]
        L.moss_enc_destroy.restype = None
        L.moss_enc_destroy.argtypes = [vp]
        L.moss_enc_status_string.restype = ctypes.c_char_p
        L.moss_enc_status_string.argtypes = [i32]
        L.moss_enc_last_error.restype = ctypes.c_char_p
        L.moss_enc_last_error.argtypes = [vp]
        L.moss_enc_logmel.restype = i32
        L.moss_enc_logmel.argtypes = [vp, ctypes.POINTER(Clip), vp, ctypes.POINTER(i64), vp]
        L.moss_enc_log_max.restype = i32
        L.moss_enc_log_max.argtypes = [vp, vp, i64, vp]
        L.moss_enc_range_log_max.restype = i32
        L.moss_enc_range_log_max.argtypes = [vp, vp, i64, i64, i64, vp]
        L.moss_enc_forward.restype = i32
        L.moss_enc_forward.argtypes = [vp, ctypes.POINTER(Clip), i32, vp, ctypes.POINTER(i64)]
        L.moss_enc_forward_stage.restype = i32
        L.moss_enc_forward_stage.argtypes = [vp, ctypes.POINTER(Clip), i32, i32, vp, ctypes.POINTER(i64)]
        L.moss_enc_forward_host.restype = i32
        L.moss_enc_forward_host.argtypes = [vp, ctypes.POINTER(vp), ctypes.POINTER(i64), i32, vp,
                                            ctypes.POINTER(i64)]
        L.moss_enc_tap_weight_count.restype = i64
        L.moss_enc_tap_weight_count.argtypes = []
        L.moss_enc_set_taps.restype = i32
        L.moss_enc_set_taps.argtypes = [vp, ctypes.POINTER(i32), i32, vp, ctypes.c_size_t, i32]
        L.moss_enc_forward_taps.restype = i32
        L.moss_enc_forward_taps.argtypes = [vp, ctypes.POINTER(Clip), i32, vp, ctypes.POINTER(vp),
                                            ctypes.POINTER(i64)]
        L.moss_enc_profile_enable.restype = i32
        L.moss_enc_profile_enable.argtypes = [vp, i32]
        L.moss_enc_profile_read.restype = i32
        L.moss_enc_profile_read.argtypes = [vp, ctypes.POINTER(KernelStat), i32]
        L.moss_enc_launch_count.restype = i64
        L.moss_enc_launch_count.argtypes = [vp]
        L.moss_enc_selftest_timeout.restype = i32
        L.moss_enc_selftest_timeout.argtypes = [vp, i32]
        L.moss_enc_selftest_gelu.restype = i32
        L.moss_enc_selftest_gelu.argtypes = [vp, ctypes.POINTER(ctypes.c_float)]
        L.moss_enc_gemm.restype = i32
        L.moss_enc_gemm.argtypes = [vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32]
        L.moss_enc_gemm_q4.restype = i32
        L.moss_enc_gemm_q4.argtypes = [vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, i32]
        L.moss_enc_gemm_f8.restype = i32
        L.moss_enc_gemm_f8.argtypes = [vp, vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, i32]
        L.moss_enc_gemm_nvf4.restype = i32
        L.moss_enc_gemm_nvf4.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i32, i32, i32, i32]
        L.moss_enc_nvf4_quant_rows.restype = i32
        L.moss_enc_nvf4_quant_rows.argtypes = [vp, vp, vp, vp, vp, i32]
        L.moss_enc_nvf4_quant_weights.restype = i32
        L.moss_enc_nvf4_quant_weights.argtypes = [vp, i32, i32, i32, vp, vp, vp]
        L.moss_enc_logmel_static.restype = i32
        L.moss_enc_logmel_static.argtypes = [ctypes.POINTER(Clip), i32, ctypes.POINTER(vp), vp, vp]
        _lib = L
    return _lib


def weight_count(n_layers: int) -> int:
    return int(lib().moss_enc_weight_count(n_layers))


def num_frames(n: int) -> int:
    return int(lib().moss_enc_num_frames(n))


def num_tokens(n: int) -> int:
    return int(lib().moss_enc_num_tokens(n))


def range_tokens(n: int, begin: int, end: int) -> int:
    return int(lib().moss_enc_range_tokens(n, begin, end))


def nvf4_quant_weights(w: np.ndarray, parts: int = 1):
    """The create-time NVFP4 quantisation of a bf16 matrix (uint16 bits)
    [n][k] in `parts` row ranges (host only): (codes [n][k/2] uint8, scale
    atoms uint8, g [n] fp32)."""
    w = np.ascontiguousarray(w, dtype=np.uint16)
    n, k = w.shape
    codes = np.empty((n, k // 2), dtype=np.uint8)
    sfa = np.empty(n * k // 16, dtype=np.uint8)
    g = np.empty(n, dtype=np.float32)
    st = lib().moss_enc_nvf4_quant_weights(w.ctypes.data_as(ctypes.c_void_p), n, k, parts,
                                           codes.ctypes.data_as(ctypes.c_void_p), sfa.ctypes.data_as(ctypes.c_void_p),
                                           g.ctypes.data_as(ctypes.c_void_p))
    if st != OK:
        raise MossEncError(st, "nvf4_quant_weights")
    return codes, sfa, g


def tap_weight_count() -> int:
    return int(lib().moss_enc_tap_weight_count())


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else None


class Encoder:
    """One moss_enc handle on the current CUDA device.

    blob: uint16 numpy array of bf16 bits (host) or a torch uint16/int16 CUDA
    tensor.  Work is enqueued on ``stream`` (default: torch's current stream).
    """

    def __init__(self, blob, n_layers: int, max_samples: int, max_clips: int = 1,
                 out_dtype: int = OUT_F32, stream=None, weight_bits: int = 16, fp8: bool = False,
                 nvfp4: bool = False):
        import torch
        self.torch = torch
        self.n_layers = n_layers
        self.out_dtype = out_dtype
        cfg = Config(n_layers, int(max_samples), int(max_clips), int(out_dtype), int(weight_bits), int(bool(fp8)),
                     int(bool(nvfp4)))
        if stream is None:
            stream = torch.cuda.current_stream()
        self.stream = stream
        h = ctypes.c_void_p()
        if isinstance(blob, np.ndarray):
            blob = np.ascontiguousarray(blob, dtype=np.uint16)
            st = lib().moss_enc_create(ctypes.byref(cfg), blob.ctypes.data_as(ctypes.c_void_p),
                                       blob.nbytes, 0, ctypes.c_void_p(stream.cuda_stream), ctypes.byref(h))
        else:
            st = lib().moss_enc_create(ctypes.byref(cfg), ctypes.c_void_p(blob.data_ptr()),
                                       blob.numel() * 2, 1, ctypes.c_void_p(stream.cuda_stream),
                                       ctypes.byref(h))
        if st != OK:
            raise MossEncError(st, "create failed")
        self.h = h

    def close(self):
        if getattr(self, "h", None):
            lib().moss_enc_destroy(self.h)
            self.h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def _check(self, st):
        if st != OK:
            msg = lib().moss_enc_last_error(self.h) or b""
            raise MossEncError(st, msg.decode())

    def set_stream(self, stream):
        self.stream = stream
        self._check(lib().moss_enc_set_stream(self.h, ctypes.c_void_p(stream.cuda_stream)))

    def synchronize(self):
        self._check(lib().moss_enc_synchronize(self.h))

    def profile_enable(self, max_launches: int):
        self._check(lib().moss_enc_profile_enable(self.h, int(max_launches)))

    def profile_read(self):
        """{category: dict(launches, ms, flops, bytes)} since the last read."""
        arr = (KernelStat * 64)()
        n = lib().moss_enc_profile_read(self.h, arr, 64)
        if n < 0:
            raise MossEncError(4, "profile_read failed")
        return {arr[i].name.decode(): dict(launches=arr[i].launches, ms=arr[i].ms, flops=arr[i].flops,
                                           bytes=arr[i].bytes) for i in range(n)}

    def gemm(self, A, B, bias, out, epilogue: int, block_n: int, cta_pair: bool = True):
        """out = epi(A @ B.T + bias) on the tensor cores (A [M][K], B [N][K] bf16)."""
        M, K = A.shape
        N = B.shape[0]
        self._check(lib().moss_enc_gemm(self.h, _ptr(A), _ptr(B), _ptr(bias), _ptr(out), M, N, K,
                                        int(epilogue), int(block_n), int(bool(cta_pair))))
        return out

    def gemm_q4(self, A, Bq, Bs, bias, out, epilogue: int, block_n: int):
        """out = epi(A @ B.T + bias) with B as 4-bit codes Bq [N][K/2] (uint8,
        even k in the low nibble, code q + 8) and group scales Bs [K/128][N]."""
        M, K = A.shape
        N = Bq.shape[0]
        self._check(lib().moss_enc_gemm_q4(self.h, _ptr(A), _ptr(Bq), _ptr(Bs), _ptr(bias), _ptr(out), M, N, K,
                                           int(epilogue), int(block_n)))
        return out

    def gemm_f8(self, A8, B8, sa, sb, bias, out, epilogue: int, block_n: int):
        """out = epi((A8 @ B8.T) * sa[:, None] * sb[None, :] + bias) on e4m3
        operands (uint8 bits) A8 [M][K], B8 [N][K]."""
        M, K = A8.shape
        N = B8.shape[0]
        self._check(lib().moss_enc_gemm_f8(self.h, _ptr(A8), _ptr(B8), _ptr(sa), _ptr(sb), _ptr(bias), _ptr(out),
                                           M, N, K, int(epilogue), int(block_n)))
        return out

    def gemm_nvf4(self, A4, sfa, ga, B4, sfb, gb, bias, out, epilogue: int):
        """out = epi((a @ b.T) * ga[:, None] * gb[None, :] + bias) on NVFP4
        operands: A4 [M][K/2], B4 [N][K/2] packed E2M1 codes (uint8), sfa, sfb
        their E4M3 block-scale atoms (uint8), ga [M], gb [N] fp32."""
        M, K2 = A4.shape
        N = B4.shape[0]
        if B4.shape[1] != K2 or sfa.numel() < (M + 127) // 128 * (2 * K2 // 64) * 512 or \
                sfb.numel() < (N + 127) // 128 * (2 * K2 // 64) * 512 or ga.numel() < M or gb.numel() < N:
            raise ValueError("A4 [M][K/2], B4 [N][K/2], their scale atoms, ga [M], gb [N]")
        self._check(lib().moss_enc_gemm_nvf4(self.h, _ptr(A4), _ptr(sfa), _ptr(ga), _ptr(B4), _ptr(sfb), _ptr(gb),
                                             _ptr(bias), _ptr(out), M, N, 2 * K2, int(epilogue)))
        return out

    def nvf4_quant_rows(self, x, codes, sfa, g):
        """NVFP4 codes, scale atoms and per-row g of fp32 rows x [M][1280]."""
        M = x.shape[0]
        if (x.dim() != 2 or x.shape[1] != D_MODEL or not x.is_contiguous() or tuple(codes.shape) != (M, D_MODEL // 2)
                or sfa.numel() < (M + 127) // 128 * 20 * 512 or g.numel() < M):
            raise ValueError("x [M][1280] fp32, codes [M][640], sfa ceil(M/128)*20*512 bytes, g [M]")
        self._check(lib().moss_enc_nvf4_quant_rows(self.h, _ptr(x), _ptr(codes), _ptr(sfa), _ptr(g), M))

    def selftest_timeout(self, limit_ms: int = 50):
        self._check(lib().moss_enc_selftest_timeout(self.h, int(limit_ms)))

    def selftest_gelu(self) -> float:
        e = ctypes.c_float()
        self._check(lib().moss_enc_selftest_gelu(self.h, ctypes.byref(e)))
        return float(e.value)

    def launch_count(self) -> int:
        return int(lib().moss_enc_launch_count(self.h))

    @staticmethod
    def _clip(pcm, begin=0, end=None, log_max=None):
        n = pcm.numel()
        return Clip(pcm.data_ptr(), n, int(begin), int(n if end is None else end),
                    log_max.data_ptr() if log_max is not None else None)

    def log_max(self, pcm):
        out = self.torch.empty(1, dtype=self.torch.float32, device=pcm.device)
        self._check(lib().moss_enc_log_max(self.h, _ptr(pcm), pcm.numel(), _ptr(out)))
        return out

    def range_log_max(self, pcm, begin=0, end=None):
        """Log-mel maximum over the frames of samples [begin, end) (device [1])."""
        n = pcm.numel()
        out = self.torch.empty(1, dtype=self.torch.float32, device=pcm.device)
        self._check(lib().moss_enc_range_log_max(self.h, _ptr(pcm), n, int(begin), int(n if end is None else end),
                                                 _ptr(out)))
        return out

    def logmel(self, pcm, begin=0, end=None, log_max=None):
        """Normalised log-mel [frames][128] fp32 and the log-mel maximum (device)."""
        n = pcm.numel()
        end = n if end is None else end
        fb = begin // 160
        fe = num_frames(n) if end == n else end // 160
        mel = self.torch.empty((max(fe - fb, 0), 128), dtype=self.torch.float32, device=pcm.device)
        mx = self.torch.empty(1, dtype=self.torch.float32, device=pcm.device)
        c = self._clip(pcm, begin, end, log_max)
        nf = ctypes.c_int64()
        self._check(lib().moss_enc_logmel(self.h, ctypes.byref(c), _ptr(mel) if mel.numel() else None,
                                          ctypes.byref(nf), _ptr(mx)))
        assert nf.value == mel.shape[0]
        return mel, mx

    def _clips(self, clips):
        arr = (Clip * max(len(clips), 1))()
        total = 0
        for i, c in enumerate(clips):
            if isinstance(c, tuple):
                pcm, begin, end, lm = (list(c) + [None, None, None])[:4]
                n = pcm.numel()
                arr[i] = self._clip(pcm, begin or 0, n if end is None else end, lm)
                total += max(0, range_tokens(n, begin or 0, n if end is None else end))
            else:
                arr[i] = self._clip(c)
                total += num_tokens(c.numel())
        return arr, total

    def forward(self, clips, out=None, stage: int = STAGE_ADAPTER):
        """Encode clips (device fp32 tensors, or (pcm, begin, end, log_max) tuples).

        Returns (rows, row_offsets): rows [T][2048] (or [T][1280] for the stem
        and layer stages), row_offsets a Python list of n_clips + 1 ints.
        """
        torch = self.torch
        arr, T = self._clips(clips)
        width = D_MODEL if stage in (STAGE_STEM, STAGE_LAYERS) else D_OUT
        if stage == STAGE_ADAPTER:
            dt = torch.float32 if self.out_dtype == OUT_F32 else torch.bfloat16
        else:
            dt = torch.float32
        dev = clips[0][0].device if isinstance(clips[0], tuple) else clips[0].device
        if out is None:
            out = torch.empty((T, width), dtype=dt, device=dev)
        offs = (ctypes.c_int64 * (len(clips) + 1))()
        if stage == STAGE_ADAPTER:
            st = lib().moss_enc_forward(self.h, arr, len(clips), _ptr(out) if T else None, offs)
        else:
            st = lib().moss_enc_forward_stage(self.h, arr, len(clips), stage, _ptr(out) if T else None, offs)
        self._check(st)
        return out, list(offs)

    def set_taps(self, layers, weights=None):
        """Layer taps: 0-based encoder layers, each with its own head + adapter
        set (``weights``: uint16 numpy array or torch uint16/int16 CUDA tensor
        of len(layers) * tap_weight_count() bf16 bits), or None to share the
        encoder's own head and adapter."""
        n = len(layers)
        arr = (ctypes.c_int * max(n, 1))(*[int(l) for l in layers])
        if weights is None:
            st = lib().moss_enc_set_taps(self.h, arr, n, None, 0, 0)
        elif isinstance(weights, np.ndarray):
            w = np.ascontiguousarray(weights, dtype=np.uint16)
            st = lib().moss_enc_set_taps(self.h, arr, n, w.ctypes.data_as(ctypes.c_void_p), w.nbytes, 0)
        else:
            st = lib().moss_enc_set_taps(self.h, arr, n, ctypes.c_void_p(weights.data_ptr()),
                                         weights.numel() * 2, 1)
        self._check(st)
        self.n_taps = n

    def forward_taps(self, clips, out=None, taps=None):
        """Final rows plus one [T][2048] tensor per tap set by set_taps.

        Returns (rows, [tap rows], row_offsets)."""
        torch = self.torch
        arr, T = self._clips(clips)
        dt = torch.float32 if self.out_dtype == OUT_F32 else torch.bfloat16
        dev = clips[0][0].device if isinstance(clips[0], tuple) else clips[0].device
        n = getattr(self, "n_taps", 0)
        if out is None:
            out = torch.empty((T, D_OUT), dtype=dt, device=dev)
        if taps is None:
            taps = [torch.empty((T, D_OUT), dtype=dt, device=dev) for _ in range(n)]
        ptrs = (ctypes.c_void_p * max(n, 1))(*[t.data_ptr() for t in taps])
        offs = (ctypes.c_int64 * (len(clips) + 1))()
        self._check(lib().moss_enc_forward_taps(self.h, arr, len(clips), _ptr(out) if T else None,
                                                ptrs if n else None, offs))
        return out, taps, list(offs)

    def forward_host(self, clips_host, rows_host=None):
        """End-to-end from host fp32 arrays to host rows (synchronises)."""
        n = len(clips_host)
        ptrs = (ctypes.c_void_p * max(n, 1))()
        lens = (ctypes.c_int64 * max(n, 1))()
        T = 0
        for i, c in enumerate(clips_host):
            ptrs[i] = c.data_ptr() if hasattr(c, "data_ptr") else c.ctypes.data
            lens[i] = c.numel() if hasattr(c, "numel") else c.size
            T += num_tokens(lens[i])
        if rows_host is None:
            dt = np.float32 if self.out_dtype == OUT_F32 else np.uint16
            rows_host = np.empty((T, D_OUT), dtype=dt)
        rp = rows_host.data_ptr() if hasattr(rows_host, "data_ptr") else rows_host.ctypes.data
        offs = (ctypes.c_int64 * (n + 1))()
        self._check(lib().moss_enc_forward_host(self.h, ptrs, lens, n, ctypes.c_void_p(rp), offs))
        return rows_host, list(offs)


def logmel_static(clips, stream=None):
    """Allocation-free log-mel of up to STATIC_MAX_CLIPS clips (no handle).

    clips: device fp32 tensors or (pcm, begin, end, log_max) tuples.  The
    output tensors are made here by PyTorch on the caller's behalf; the
    library call itself allocates nothing.  Returns (list of [frames][128]
    tensors, log_max tensor [n_clips]).
    """
    import torch
    n = len(clips)
    arr = (Clip * max(n, 1))()
    outs = []
    for i, c in enumerate(clips):
        pcm, begin, end, lm = (list(c) + [None, None, None])[:4] if isinstance(c, tuple) else (c, 0, None, None)
        ns = pcm.numel()
        end = ns if end is None else end
        arr[i] = Clip(pcm.data_ptr(), ns, int(begin or 0), int(end), lm.data_ptr() if lm is not None else None)
        fb = (begin or 0) // 160
        fe = num_frames(ns) if end == ns else end // 160
        outs.append(torch.empty((max(fe - fb, 0), 128), dtype=torch.float32, device=pcm.device))
    ptrs = (ctypes.c_void_p * max(n, 1))(*[o.data_ptr() if o.numel() else None for o in outs])
    dev = clips[0][0].device if isinstance(clips[0], tuple) else clips[0].device
    mx = torch.empty(max(n, 1), dtype=torch.float32, device=dev)
    if stream is None:
        stream = torch.cuda.current_stream()
    st = lib().moss_enc_logmel_static(arr, n, ptrs, ctypes.c_void_p(mx.data_ptr()),
                                      ctypes.c_void_p(stream.cuda_stream))
    if st != OK:
        raise MossEncError(st, "logmel_static failed")
    return outs, mx[:n]
