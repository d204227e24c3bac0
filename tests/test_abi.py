"""The C-ABI library loads and exports every symbol its header declares;
the pure host functions agree with the oracle's counts.  No GPU needed."""
import os
import re

import numpy as np
import pytest

import oracle
from audio_encoder_b200 import binding, synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_symbols():
    with open(os.path.join(ROOT, "include", "moss_enc.h")) as f:
        text = f.read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(moss_enc_[a-z_]+)\s*\(", text)))


def test_header_declares_the_documented_calls():
    syms = declared_symbols()
    for s in ["moss_enc_create", "moss_enc_logmel", "moss_enc_forward", "moss_enc_destroy"]:
        assert s in syms


def test_library_exports_every_declared_symbol():
    L = binding.lib()
    for s in declared_symbols():
        assert hasattr(L, s), s
    assert set(declared_symbols()) <= set(binding.EXPORTED)


def test_weight_count_matches_generator_and_oracle():
    for n in [1, 4, 32]:
        _, total = synth.weight_offsets(n)
        assert binding.weight_count(n) == total == oracle.weight_count(n)


def test_tap_weight_count_is_one_head_and_adapter_set():
    # a layer tap's weights are laid out like the blob's tail after the layers
    count = binding.tap_weight_count()
    assert count == sum(int(np.prod(shape)) for _, shape, _ in synth.head_manifest())
    names = [name for name, _, _ in synth.weight_manifest(0)]
    stem = sum(int(np.prod(shape)) for _, shape, _ in synth.weight_manifest(0)[:names.index("ln_post.weight")])
    assert binding.weight_count(0) == stem + count
    assert synth.make_tap_weights(2).size == 2 * count


@pytest.mark.parametrize("n", [0, 1, 159, 160, 161, 16000, 16159, 127999, 128000, 128160, 480000,
                               9_600_000, 57_600_000, 1_024_000, 160 * 801])
def test_counts_match_oracle(n):
    assert binding.num_frames(n) == oracle.num_frames(n)
    assert binding.num_tokens(n) == oracle.num_tokens(n)


def test_range_tokens_add_up_over_pieces():
    n = 57_600_000
    piece = 1_024_000
    total = sum(binding.range_tokens(n, b, min(b + piece, n)) for b in range(0, n, piece))
    assert total == binding.num_tokens(n) == 45000
    assert binding.range_tokens(n, 0, n) == 45000
    assert binding.range_tokens(n, 1000, n) == -1          # begin not chunk-aligned
    assert binding.range_tokens(n, 0, 1000) == -1          # end neither n nor aligned
    assert binding.range_tokens(n, 128000, 128000) == 0


def test_create_rejects_bad_arguments_before_touching_a_device():
    import ctypes
    L = binding.lib()
    h = ctypes.c_void_p()
    cfg = binding.Config(0, 1000, 1, 0)  # n_layers 0
    blob = np.zeros(4, dtype=np.uint16)
    st = L.moss_enc_create(ctypes.byref(cfg), blob.ctypes.data_as(ctypes.c_void_p), 8, 0, None, ctypes.byref(h))
    assert st == 1 and not h.value
    assert L.moss_enc_create(None, None, 0, 0, None, ctypes.byref(h)) == 1
    cfg = binding.Config(4, 1000, 1, 0)
    st = L.moss_enc_create(ctypes.byref(cfg), blob.ctypes.data_as(ctypes.c_void_p), 8, 0, None, ctypes.byref(h))
    assert st == 1  # blob size does not match 4 layers
    # weight_bits must be 16 (or 0) or 4: refused before the blob is read
    # weight_bits 16/0/4; fp8 0/1, not with 4-bit weights; nvfp4 0/1, with
    # neither fp8 nor 4-bit weights
    for bits, fp8, nvfp4 in [(8, 0, 0), (4, 1, 0), (16, 2, 0), (16, 0, 2), (16, 1, 1), (4, 0, 1)]:
        cfg = binding.Config(1, 1000, 1, 0, bits, fp8, nvfp4)
        assert L.moss_enc_create(ctypes.byref(cfg), blob.ctypes.data_as(ctypes.c_void_p), 2 * binding.weight_count(1),
                                 0, None, ctypes.byref(h)) == 1
    assert L.moss_enc_status_string(2) == b"request exceeds capacity"


def test_static_logmel_rejects_a_clip_without_samples_pointer():
    # A clip with samples but no pcm pointer is refused before anything is
    # enqueued, even when its encoded range is empty (the whole-clip maximum
    # would read the samples); no device is touched.
    import ctypes
    L = binding.lib()
    arr = (binding.Clip * 1)()
    arr[0] = binding.Clip(None, 16000, 0, 0, None)
    outs = (ctypes.c_void_p * 1)(None)
    assert L.moss_enc_logmel_static(arr, 1, outs, None, None) == 1
    arr[0] = binding.Clip(None, 16000, 0, 16000, None)
    assert L.moss_enc_logmel_static(arr, 1, outs, None, None) == 1


def test_nvf4_weight_quantiser_matches_oracle():
    # the create-time NVFP4 quantisation of a weight matrix (host code of the
    # library) against the oracle's, part by part: g, block scales and codes
    # bit for bit (a zero may carry either sign); no device is touched
    import oracle
    import torch
    from audio_encoder_b200 import synth
    rng = np.random.default_rng(11)
    n, k, parts = 384, 256, 3
    w = (rng.standard_normal((n, k)) * np.repeat([0.02, 0.3, 5.0], n // parts)[:, None]).astype(np.float32)
    w[5, :32] = 0.0
    wb = synth.f32_to_bf16_bits(w)
    codes, sfa, g = binding.nvf4_quant_weights(wb, parts)
    got = np.empty((n, k), dtype=np.uint8)
    got[:, 0::2] = codes & 15
    got[:, 1::2] = codes >> 4
    atoms = sfa.reshape(n // 128, k // 64, 512)
    r = np.arange(n)[:, None]
    b = np.arange(k // 16)[None, :]
    e4 = atoms[r // 128, b // 4, (r % 32) * 16 + ((r % 128) // 32) * 4 + b % 4]
    bs = torch.from_numpy(np.ascontiguousarray(e4)).view(torch.float8_e4m3fn).to(torch.float32).numpy()
    wf = synth.bf16_bits_to_f32(wb)
    rows = n // parts
    for p in range(parts):
        sl = slice(p * rows, (p + 1) * rows)
        _, g_ref, c_ref, bs_ref = oracle.quant_nvfp4(wf[sl], per_row=False)
        assert np.all(g[sl] == g_ref[0])
        np.testing.assert_array_equal(bs[sl], bs_ref)
        np.testing.assert_array_equal(got[sl] & 7, c_ref & 7)
        nz = (c_ref & 7) != 0
        np.testing.assert_array_equal((got[sl] & 8)[nz], (c_ref & 8)[nz])
    # exact ties: with the part's maximum 2688 (g = 1) and a block maximum of
    # 2688 (scale 448), x = m * 448 lands exactly on every E2M1 midpoint m;
    # each tie must go to the even code, as in the oracle
    mids = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0], dtype=np.float32)
    t = np.zeros((128, 64), dtype=np.float32)
    t[0, 0] = 2688.0
    t[0, 1:8] = mids * 448.0
    t[0, 8:15] = -mids * 448.0
    tb = synth.f32_to_bf16_bits(t)
    assert np.array_equal(synth.bf16_bits_to_f32(tb), t)  # every value is exact in bf16
    c, _, gt = binding.nvf4_quant_weights(tb, 1)
    mag = np.empty(64, dtype=np.uint8)
    mag[0::2] = c[0] & 15
    mag[1::2] = c[0] >> 4
    assert gt[0] == 1.0 and mag[0] == 7  # 2688 / 448 = 6
    np.testing.assert_array_equal(mag[1:8] & 7, [0, 2, 2, 4, 4, 6, 6])  # 0, 1, 1, 2, 2, 4, 4
    np.testing.assert_array_equal(mag[9:15] & 7, [2, 2, 4, 4, 6, 6])
    assert np.all(mag[9:15] & 8)  # negative
    _, _, c_ref, _ = oracle.quant_nvfp4(t, per_row=False)
    np.testing.assert_array_equal(mag[:15] & 7, c_ref[0, :15] & 7)
    with pytest.raises(binding.MossEncError):
        binding.nvf4_quant_weights(wb[:, :100], 1)  # k not a multiple of 64
