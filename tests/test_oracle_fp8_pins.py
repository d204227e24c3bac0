"""Pins for the oracle's FP8 (e4m3) operands (page "Ossicle-4B", "Quantized:
NVFP4 and INT4 in vLLM": low-precision weights and activations for the
encoder): the rounding against PyTorch's float8_e4m3fn conversion and its
closed forms (every e4m3 value is a fixed point, ties go to even, +-448
saturates, the step below 2^-6 is 2^-9), the per-row scales, and the FP8
layers against the same layers written with PyTorch routines.  None of
these reads the CUDA path."""
import numpy as np
import pytest
import torch

import oracle
from audio_encoder_b200 import synth
from conftest import weights
from torch_ref import TorchRef


def e4m3_values():
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8).view(torch.float8_e4m3fn)
    v = codes.to(torch.float32).numpy()
    return np.unique(v[np.isfinite(v)])


def test_every_e4m3_value_is_a_fixed_point():
    v = e4m3_values()
    assert v.max() == 448.0 and v.min() == -448.0 and len(v) == 253  # 254 finite codes, +0 and -0 merge
    for x in v:
        assert oracle.e4m3(float(x)) == x


def test_rounding_matches_torch_float8_conversion():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.uniform(-460, 460, 4000), rng.standard_normal(4000) * 0.01,
                        rng.standard_normal(2000) * 2.0 ** -8]).astype(np.float32)
    got = np.array([oracle.e4m3(float(a)) for a in x], dtype=np.float32)
    ref = torch.from_numpy(np.clip(x, -448, 448)).to(torch.float8_e4m3fn).to(torch.float32).numpy()
    np.testing.assert_array_equal(got, ref)


def test_ties_go_to_even_and_saturation():
    v = e4m3_values()
    pos = v[v > 0]
    for lo, hi in zip(pos[:-1], pos[1:]):
        mid = float(np.float32((lo + hi) / 2))
        got = oracle.e4m3(mid)
        # the neighbour whose last mantissa bit is 0
        lo_code = int(torch.tensor([lo]).to(torch.float8_e4m3fn).view(torch.uint8).item())
        want = lo if lo_code % 2 == 0 else hi
        assert got == want, (lo, hi, got)
    assert oracle.e4m3(464.0) == 448.0 and oracle.e4m3(1e9) == 448.0 and oracle.e4m3(-1e9) == -448.0
    assert oracle.e4m3(2.0 ** -10) == 0.0 and oracle.e4m3(3 * 2.0 ** -11) == 2.0 ** -9


def test_row_scales_map_each_row_max_to_448():
    rng = np.random.default_rng(1)
    w = synth.f32_to_bf16_bits((rng.standard_normal((8, 256)) * rng.uniform(0.01, 5, (8, 1))).astype(np.float32))
    w[3] = 0
    q, s = oracle.quant_e4m3_rows(w)
    qv = synth.bf16_bits_to_f32(q)
    wv = synth.bf16_bits_to_f32(w)
    for r in range(8):
        if r == 3:
            assert s[r] == 0 and np.all(qv[r] == 0)
            continue
        k = np.argmax(np.abs(wv[r]))
        assert abs(qv[r, k]) == 448.0
        assert s[r] == np.float32(np.abs(wv[r]).max()) / np.float32(448.0)


def test_fp8_layers_vs_torch():
    # q, k, v and fc1 on e4m3 operands, against the same layers with PyTorch's
    # LayerNorm, float8 conversion, attention and GELU
    blob = weights(1)
    om = oracle.Model(blob, 1, weight_bits=8)
    tr = TorchRef(blob, 1)
    rng = np.random.default_rng(3)
    x = rng.standard_normal((37, 1280)).astype(np.float32)
    windows = [0, 30, 37]
    got = om.layers(x, windows)
    ref = tr.layers(torch.from_numpy(x.astype(np.float64)), windows, fp8=True).numpy()
    np.testing.assert_allclose(got, ref, rtol=2e-3, atol=2e-3)
    # and the e4m3 operands move the result (it is not the bf16 model)
    ref16 = tr.layers(torch.from_numpy(x.astype(np.float64)), windows).numpy()
    assert np.abs(ref16 - ref).max() > 1e-2
    om.close()
