"""Layer taps (the cross-layer adapter: page "MOSS-Audio-4B-Instruct on an
RTX 5070", opening paragraph) through the C ABI against the CPU oracle.

A tap's rows are its own head + adapter set applied to the residual stream
after one encoder layer; the oracle computes them as its layers [0, l + 1)
followed by the head and adapter of a model holding the tap's set."""
import numpy as np
import pytest

import oracle
from audio_encoder_b200 import binding, synth
from conftest import oracle_model, weights
from metrics import assert_rows_close

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


def dev(x):
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).cuda()


def tap_oracles(n_layers, tap_blob, n_taps):
    """One oracle model per tap set: the main blob's stem with 0 layers and
    the tap's head + adapter."""
    count = binding.tap_weight_count()
    stem = weights(n_layers)[:oracle.weight_count(0) - count]
    return [oracle.Model(np.concatenate([stem, tap_blob[t * count:(t + 1) * count]]), 0) for t in range(n_taps)]


def oracle_taps(om, pcm_list, layers, tap_models, n_chunks=None):
    """Reference tap rows of clips encoded independently (rows concatenated);
    n_chunks limits each clip to its first windows (whole-clip maximum)."""
    outs = [[] for _ in layers]
    for pcm in pcm_list:
        _, d = om.encode_chunks(pcm, 0, n_chunks, dumps=True)
        T = d["stem"].shape[0]
        win = [0]
        F = oracle.num_frames(pcm.size)
        nc = oracle.num_chunks(pcm.size) if n_chunks is None else min(n_chunks, oracle.num_chunks(pcm.size))
        for c in range(nc):
            win.append(win[-1] + oracle.chunk_tokens(min(800, F - 800 * c)))
        assert win[-1] == T
        for t, l in enumerate(layers):
            x = om.layers(d["stem"], win, 0, l + 1)
            tm = tap_models[t]
            outs[t].append(tm.adapter(tm.head(x)))
    return [np.concatenate(o) for o in outs]


def test_tap_weight_count_matches_blob_tail():
    count = binding.tap_weight_count()
    assert count == sum(int(np.prod(s)) for _, s, _ in synth.head_manifest())
    assert oracle.weight_count(1) - oracle.weight_count(0) + count < oracle.weight_count(1)


def test_taps_own_weights_tiny_clip():
    n_layers, layers = 4, [0, 2, 3]
    pcm = synth.pcm_tones(0, 16000)
    enc = binding.Encoder(weights(n_layers), n_layers, 600_000, 2)
    try:
        plain, offs0 = enc.forward([dev(pcm)])
        tw = synth.make_tap_weights(len(layers))
        enc.set_taps(layers, tw)
        rows, taps, offs = enc.forward_taps([dev(pcm)])
        torch.cuda.synchronize()
        assert offs == offs0 == [0, 13]
        # the taps leave the final rows untouched
        np.testing.assert_array_equal(rows.cpu().numpy(), plain.cpu().numpy())
        refs = oracle_taps(oracle_model(n_layers), [pcm], layers, tap_oracles(n_layers, tw, len(layers)))
        for t, l in enumerate(layers):
            assert_rows_close(taps[t].cpu().numpy(), refs[t], f"tap after layer {l}")
    finally:
        enc.close()


def test_taps_shared_weights_equal_final_rows_at_last_layer():
    # with the encoder's own head set, a tap after the last layer is the
    # final output, launch for launch
    n_layers = 4
    pcm = synth.pcm_30s(1, 480000)
    enc = binding.Encoder(weights(n_layers), n_layers, 600_000, 1)
    try:
        enc.set_taps([n_layers - 1, 1])
        rows, taps, offs = enc.forward_taps([dev(pcm)])
        torch.cuda.synchronize()
        assert offs == [0, 375]
        np.testing.assert_array_equal(taps[0].cpu().numpy(), rows.cpu().numpy())
        om = oracle_model(n_layers)
        ref = oracle_taps(om, [pcm], [1], [om], n_chunks=2)[0]
        assert_rows_close(taps[1].cpu().numpy()[:ref.shape[0]], ref, "shared-weight tap after layer 1")
    finally:
        enc.close()


def test_taps_batch_ragged_and_graph_replay():
    # two clips (3 + 2 windows, ragged tails: 588 rows over three 256-row
    # tiles), own weights, on a side stream: the first call runs launch by
    # launch, the repeated one is captured as a CUDA graph and run from it
    n_layers, layers = 4, [1, 3]
    clips = [synth.pcm_30s(1, 480000), synth.pcm_tones(5, 17 * 16000 + 123)]
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        enc = binding.Encoder(weights(n_layers), n_layers, 1_000_000, 2, stream=s)
        try:
            tw = synth.make_tap_weights(len(layers), seed=99)
            enc.set_taps(layers, torch.from_numpy(tw.view(np.int16)).cuda())
            d = [dev(c) for c in clips]
            rows, taps, offs = enc.forward_taps(d)
            first = [t.clone() for t in taps]
            rows2, taps2, _ = enc.forward_taps(d, out=rows, taps=taps)
            s.synchronize()
        finally:
            enc.close()
    assert offs == [0, 375, 375 + oracle.num_tokens(clips[1].size)]
    for a, b in zip(first, taps2):
        np.testing.assert_array_equal(a.cpu().numpy(), b.cpu().numpy())
    refs = oracle_taps(oracle_model(n_layers), clips, layers, tap_oracles(n_layers, tw, len(layers)))
    for t, l in enumerate(layers):
        assert_rows_close(taps[t].cpu().numpy(), refs[t], f"batch tap after layer {l}")


def test_tap_arguments_checked():
    n_layers = 2
    enc = binding.Encoder(weights(n_layers), n_layers, 100_000, 1)
    try:
        with pytest.raises(binding.MossEncError):
            enc.set_taps([2])  # past the last layer
        with pytest.raises(binding.MossEncError):
            enc.set_taps([-1])
        with pytest.raises(binding.MossEncError):
            enc.set_taps([0], np.zeros(10, np.uint16))  # wrong size
        with pytest.raises(binding.MossEncError):
            enc.set_taps([0] * 9)  # more than 8 taps
        enc.set_taps([])
        pcm = dev(synth.pcm_tones(3, 32000))
        rows, taps, offs = enc.forward_taps([pcm])
        plain, _ = enc.forward([pcm])
        torch.cuda.synchronize()
        assert taps == [] and offs == [0, 25]
        np.testing.assert_array_equal(rows.cpu().numpy(), plain.cpu().numpy())
    finally:
        enc.close()
