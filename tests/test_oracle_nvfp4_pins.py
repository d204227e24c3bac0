"""Pins for the oracle's NVFP4 operands (page "Ossicle-4B", "Quantized:
NVFP4 and INT4 in vLLM": NVFP4 weights and activations for the encoder):
the E2M1 grid and its rounding by brute force (every value a fixed point,
ties to the even code, +-6 saturates), the two-level scales (g = amax / 2688,
the block holding the tensor's or row's maximum gets the E4M3 scale 448 and
its maximum maps to +-6), zero rows, and the NVFP4 layers against the same
layers written with PyTorch routines.  None of these reads the CUDA path."""
import numpy as np
import torch

import oracle
from conftest import weights
from torch_ref import TorchRef

GRID = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0], dtype=np.float32)


def nearest_even(y):
    # brute force: the closest grid magnitude, on a tie the one with the even code
    a = np.abs(y)
    d = np.abs(a[:, None] - GRID[None, :])
    best = d.min(axis=1)
    pick = np.empty_like(a)
    for i in range(len(a)):
        cand = np.nonzero(d[i] == best[i])[0]
        even = [c for c in cand if c % 2 == 0]
        pick[i] = GRID[even[0] if even else cand[0]]
    return np.sign(y) * pick


def test_every_e2m1_value_is_a_fixed_point():
    for v in np.concatenate([GRID, -GRID]):
        assert oracle.e2m1(float(v)) == v
    assert len(np.unique(np.concatenate([GRID, -GRID]))) == 15  # +0 and -0 merge


def test_rounding_is_nearest_with_ties_to_even():
    rng = np.random.default_rng(0)
    mids = (GRID[:-1] + GRID[1:]) / 2
    y = np.concatenate([rng.uniform(-7, 7, 3000), mids, -mids, mids + 1e-6, mids - 1e-6,
                        [6.0, 6.5, 1e6, -1e6]]).astype(np.float32)
    got = np.array([oracle.e2m1(float(v)) for v in y], dtype=np.float32)
    np.testing.assert_array_equal(np.abs(got), np.abs(nearest_even(y)))
    assert oracle.e2m1(0.25) == 0.0 and oracle.e2m1(0.75) == 1.0 and oracle.e2m1(2.5) == 2.0
    assert oracle.e2m1(5.0) == 4.0 and oracle.e2m1(5.5) == 6.0 and oracle.e2m1(100.0) == 6.0


def test_two_level_scales():
    rng = np.random.default_rng(1)
    x = (rng.standard_normal((6, 128)) * rng.uniform(0.01, 30, (6, 1))).astype(np.float32)
    x[4] = 0.0
    unit, g, codes, bs = oracle.quant_nvfp4(x, per_row=True)
    for r in range(6):
        if r == 4:
            assert g[r] == 0 and np.all(unit[r] == 0) and np.all(bs[r] == 0)
            continue
        amax = np.float32(np.abs(x[r]).max())
        assert g[r] == amax / np.float32(2688.0)
        k = int(np.argmax(np.abs(x[r])))
        assert bs[r, k // 16] == 448.0
        assert abs(unit[r, k]) == 6.0 * 448.0
        # every element is its block's nearest E2M1 value times the block scale
        for b in range(8):
            sg = np.float32(bs[r, b]) * g[r]
            y = (x[r, 16 * b:16 * b + 16] / sg).astype(np.float32)
            np.testing.assert_array_equal(np.abs(unit[r, 16 * b:16 * b + 16]), np.abs(nearest_even(y)) * bs[r, b])
        # and the codes index the grid with the sign in bit 3
        mag = GRID[codes[r] & 7] * np.where(codes[r] & 8, -1, 1)
        np.testing.assert_array_equal(np.abs(mag * bs[r][np.arange(128) // 16]), np.abs(unit[r]))
    # one g for the whole matrix
    unit_t, g_t, _, _ = oracle.quant_nvfp4(x, per_row=False)
    assert g_t.shape == (1,) and g_t[0] == np.float32(np.abs(x).max()) / np.float32(2688.0)


def test_nvfp4_layers_vs_torch():
    # q, k, v and fc1 on NVFP4 operands, against the same layers with
    # PyTorch's LayerNorm, float8 conversion of the block scales, attention
    # and GELU
    blob = weights(1)
    om = oracle.Model(blob, 1, nvfp4=True)
    tr = TorchRef(blob, 1)
    rng = np.random.default_rng(3)
    x = rng.standard_normal((37, 1280)).astype(np.float32)
    windows = [0, 30, 37]
    got = om.layers(x, windows)
    ref = tr.layers(torch.from_numpy(x.astype(np.float64)), windows, nvfp4=True).numpy()
    np.testing.assert_allclose(got, ref, rtol=2e-3, atol=2e-3)
    # the NVFP4 operands move the result (it is neither the bf16 nor the FP8 model)
    ref16 = tr.layers(torch.from_numpy(x.astype(np.float64)), windows).numpy()
    ref8 = tr.layers(torch.from_numpy(x.astype(np.float64)), windows, fp8=True).numpy()
    assert np.abs(ref16 - ref).max() > 3e-2 and np.abs(ref8 - ref).max() > 3e-2
    om.close()
