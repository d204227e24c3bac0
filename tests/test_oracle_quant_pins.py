"""Pins for the oracle's 4-bit weight quantisation (round to nearest, groups
of 128; page "Ossicle-4B", "Long Audio", the note under the table): closed
forms on values whose codes are known, the round-to-nearest error bound, the
ties-to-even rule, group independence, and the quantised model against the
bf16 model on weights the quantiser reproduces exactly.  None of these reads
the CUDA path."""
import numpy as np
import pytest

import oracle
from audio_encoder_b200 import synth

LINEARS = ("q", "k", "v", "o", "fc1", "fc2")
HEAD_LINEARS = ("proj1", "proj2", "adapter.gate", "adapter.up", "adapter.down")


def bits(x):
    return synth.f32_to_bf16_bits(np.asarray(x, dtype=np.float32))


def vals(b):
    return synth.bf16_bits_to_f32(b)


def test_values_on_the_grid_come_back_exactly():
    # w = q * 2^e with |q| <= 7 and some |q| = 7 in every group: the scale is
    # 7 * 2^e / 7 = 2^e exactly, every code is q, and w' = w
    rng = np.random.default_rng(0)
    q = rng.integers(-7, 8, size=(3, 384))
    for g in range(3):
        q[:, 128 * g + 5] = 7 * (1 if g % 2 == 0 else -1)
    e = np.array([[-3.0, 0.0, 2.0], [-10.0, -1.0, 4.0], [1.0, 1.0, -6.0]])
    w = q * np.repeat(2.0 ** e, 128, axis=1)
    deq, codes, scales = oracle.quant_rtn4(bits(w))
    np.testing.assert_array_equal(vals(deq), w.astype(np.float32))
    np.testing.assert_array_equal(codes.astype(int) - 8, q)
    np.testing.assert_array_equal(scales, (2.0 ** e).astype(np.float32))


def test_ties_round_to_even():
    # largest magnitude 7: the scale is exactly 1, so codes are rint(w)
    w = np.zeros((1, 128), dtype=np.float32)
    w[0, :8] = [7.0, 2.5, 3.5, -2.5, 0.5, 1.5, 6.5, -0.5]
    deq, codes, scales = oracle.quant_rtn4(bits(w))
    assert scales[0, 0] == 1.0
    np.testing.assert_array_equal(codes[0, :8].astype(int) - 8, [7, 2, 4, -2, 0, 2, 6, 0])
    np.testing.assert_array_equal(vals(deq)[0, :8], [7.0, 2.0, 4.0, -2.0, 0.0, 2.0, 6.0, 0.0])


def test_zero_group_and_group_independence():
    rng = np.random.default_rng(1)
    w = rng.standard_normal((2, 256)).astype(np.float32) * 0.05
    w[1, 128:] = 0.0
    deq, codes, scales = oracle.quant_rtn4(bits(w))
    assert scales[1, 1] == 0.0
    assert np.all(vals(deq)[1, 128:] == 0.0) and np.all(codes[1, 128:] == 8)
    # changing one group leaves every other group's codes and scales alone
    w2 = w.copy()
    w2[0, 128:] *= 3.0
    deq2, codes2, scales2 = oracle.quant_rtn4(bits(w2))
    np.testing.assert_array_equal(deq2[:, :128], deq[:, :128])
    np.testing.assert_array_equal(deq2[1], deq[1])
    np.testing.assert_array_equal(scales2[:, 0], scales[:, 0])


def test_round_to_nearest_error_bound():
    # |w - w'| <= s/2 (nearest code) plus half a bf16 unit of w' (the final
    # rounding); codes stay in [-7, 7]; the scale is the group's largest
    # magnitude over 7 (to fp32 rounding)
    rng = np.random.default_rng(2)
    w = vals(bits(rng.standard_normal((64, 1280)) * rng.uniform(0.001, 3.0, size=(64, 1))))
    deq, codes, scales = oracle.quant_rtn4(bits(w))
    d = vals(deq)
    s = np.repeat(scales, 128, axis=1)
    half_ulp = np.abs(d) * 2.0 ** -8  # half a unit in the last place of an 8-bit significand
    assert np.all(np.abs(w - d) <= s / 2 * (1 + 1e-6) + half_ulp)
    assert codes.min() >= 1 and codes.max() <= 15
    amax = np.abs(w.reshape(64, 10, 128)).max(axis=2)
    np.testing.assert_allclose(scales, amax / 7, rtol=1e-7)


def _grid_blob(n_layers, axis_in=True):
    """The seeded blob with every quantised linear weight moved onto the
    4-bit grid of its groups along the input axis (axis_in) or, to check the
    axis, along the output axis (128 consecutive rows of one column)."""
    blob = synth.make_weights(n_layers).copy()
    offs, _ = synth.weight_offsets(n_layers)
    names = [f"layers.{l}.{n}.weight" for l in range(n_layers) for n in LINEARS] + \
            [f"{n}.weight" for n in HEAD_LINEARS]
    for name in names:
        o, shape = offs[name]
        w = vals(blob[o:o + int(np.prod(shape))]).reshape(shape).astype(np.float64)
        m = w if axis_in else w.T
        g = m.reshape(m.shape[0], -1, 128)
        amax = np.abs(g).max(axis=2, keepdims=True)
        s = 2.0 ** np.floor(np.log2(amax / 7.0))
        q = np.clip(np.rint(g / s), -7, 7)
        q[:, :, 0] = 7  # every group reaches 7: its scale is s exactly
        m2 = (q * s).reshape(m.shape)
        w2 = m2 if axis_in else m2.T
        blob[o:o + w2.size] = bits(w2.astype(np.float32)).ravel()
    return blob


def test_quantised_model_is_lossless_on_grid_weights():
    # on weights the quantiser reproduces exactly, the 4-bit model's rows are
    # the bf16 model's bit for bit; the same grid taken along the wrong axis
    # does change them (the groups run along the input features)
    pcm = synth.pcm_tones(0, 16000)
    blob = _grid_blob(1)
    a = oracle.Model(blob, 1, weight_bits=4).encode(pcm)
    b = oracle.Model(blob, 1, weight_bits=16).encode(pcm)
    np.testing.assert_array_equal(a, b)
    blob_t = _grid_blob(1, axis_in=False)
    c = oracle.Model(blob_t, 1, weight_bits=4).encode(pcm)
    d = oracle.Model(blob_t, 1, weight_bits=16).encode(pcm)
    assert np.abs(c - d).max() > 1e-3 * np.abs(d).max()
