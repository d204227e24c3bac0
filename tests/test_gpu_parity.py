"""Parity of the CUDA path (through the C ABI) against the CPU oracle.

Small cases are compared whole, element by element (mel) or row by row
(embeddings).  The full-size workloads run on the GPU in the launch
configuration the benchmark times and are compared on sampled windows the
oracle computes one by one (every 800-frame chunk is independent given the
clip's log-mel maximum)."""
import numpy as np
import pytest

import oracle
from audio_encoder_b200 import binding, shard, synth
from conftest import oracle_model, weights
from metrics import MEL_ATOL, assert_rows_close

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")

_ENC = {}


def encoder(n_layers, max_samples, max_clips=1, out_dtype=binding.OUT_F32):
    key = (n_layers, max_samples, max_clips, out_dtype)
    if key not in _ENC:
        for k in list(_ENC):
            if k[0] != n_layers or k[1] * k[2] > 4 * 10**8:
                _ENC.pop(k).close()
        _ENC[key] = binding.Encoder(weights(n_layers), n_layers, max_samples, max_clips, out_dtype)
    return _ENC[key]


def dev(x):
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).cuda()


# ------------------------------------------------------------------ log-mel

@pytest.mark.parametrize("n", [170, 400, 16000, 16001, 16159, 48000 + 77, 480000])
def test_logmel_matches_oracle(n):
    enc = encoder(1, 600_000)
    pcm = synth.pcm_30s(1, n) if n == 480000 else synth.pcm_tones(n % 97, n)
    mel, mx = enc.logmel(dev(pcm))
    ref, rmx = oracle.logmel(pcm)
    torch.cuda.synchronize()
    assert mel.shape == ref.shape == (n // 160, 128)
    assert abs(float(mx.item()) - rmx) < 1e-4
    np.testing.assert_allclose(mel.cpu().numpy(), ref, rtol=0, atol=MEL_ATOL)


def test_logmel_silence_and_empty():
    enc = encoder(1, 600_000)
    mel, mx = enc.logmel(dev(np.zeros(3200, np.float32)))
    np.testing.assert_array_equal(mel.cpu().numpy(), np.full((20, 128), -1.5, np.float32))
    mel, _ = enc.logmel(dev(np.zeros(100, np.float32) + 0.1))
    assert mel.shape == (0, 128)


def test_logmel_output_without_16_byte_alignment():
    # the rows leave by bulk copies only when the output buffer allows them;
    # a float buffer at a 4-byte offset takes the plain-store path, same values
    import ctypes
    enc = encoder(1, 600_000)
    pcm = dev(synth.pcm_tones(3, 48000))
    ref, _ = enc.logmel(pcm)
    buf = torch.zeros(300 * 128 + 1, dtype=torch.float32, device="cuda")
    view = buf[1:]
    mx = torch.empty(1, dtype=torch.float32, device="cuda")
    c = enc._clip(pcm)
    nf = ctypes.c_int64()
    enc._check(binding.lib().moss_enc_logmel(enc.h, ctypes.byref(c), ctypes.c_void_p(view.data_ptr()),
                                             ctypes.byref(nf), ctypes.c_void_p(mx.data_ptr())))
    torch.cuda.synchronize()
    assert nf.value == 300 and float(buf[0]) == 0.0
    np.testing.assert_array_equal(view.view(300, 128).cpu().numpy(), ref.cpu().numpy())


def test_logmel_range_uses_whole_clip_max():
    enc = encoder(1, 600_000)
    n = 128000 * 3 + 5000
    pcm = synth.pcm_long(4, n)
    whole, mx = enc.logmel(dev(pcm))
    part, mx2 = enc.logmel(dev(pcm), 128000, 256000)
    torch.cuda.synchronize()
    assert float(mx.item()) == float(mx2.item())
    np.testing.assert_array_equal(part.cpu().numpy(), whole.cpu().numpy()[800:1600])


def test_logmel_10min_bandwidth_workload():
    # the full 10-min clip in the benchmark's configuration, checked against
    # oracle frames sampled across it (start, the 2 s tone changes, the end)
    enc = encoder(1, 9_600_000)
    pcm = synth.pcm_long(2, 9_600_000)
    mel, mx = enc.logmel(dev(pcm))
    gmax = oracle.clip_log_max(pcm)
    assert abs(float(mx.item()) - gmax) < 1e-4
    m = mel.cpu().numpy()
    for f0 in [0, 199, 30000, 59968]:
        ref = oracle.normalize(oracle.logmel_raw(pcm, f0, f0 + 32), gmax)
        np.testing.assert_allclose(m[f0:f0 + 32], ref, rtol=0, atol=MEL_ATOL)


# ---------------------------------------------------------- module boundaries

@pytest.fixture(scope="module")
def tiny_case():
    pcm = synth.pcm_tones(0, 16000)
    out, d = oracle_model(4).encode(pcm, dumps=True)
    return pcm, out, d


def test_tiny_stem_boundary(tiny_case):
    pcm, _, d = tiny_case
    enc = encoder(4, 600_000)
    x, offs = enc.forward([dev(pcm)], stage=binding.STAGE_STEM)
    assert offs == [0, 13]
    assert_rows_close(x.cpu().numpy(), d["stem"], "post-stem")


def test_tiny_layers_boundary(tiny_case):
    pcm, _, d = tiny_case
    enc = encoder(4, 600_000)
    x, _ = enc.forward([dev(pcm)], stage=binding.STAGE_LAYERS)
    assert_rows_close(x.cpu().numpy(), d["enc"], "after 4 layers")


def test_tiny_head_boundary(tiny_case):
    pcm, _, d = tiny_case
    enc = encoder(4, 600_000)
    x, _ = enc.forward([dev(pcm)], stage=binding.STAGE_HEAD)
    assert_rows_close(x.cpu().numpy(), d["head"], "after proj2")


def test_tiny_final_rows(tiny_case):
    pcm, out, _ = tiny_case
    enc = encoder(4, 600_000)
    y, offs = enc.forward([dev(pcm)])
    assert y.shape == (13, 2048) and offs == [0, 13]
    assert_rows_close(y.cpu().numpy(), out, "tiny rows")


def test_one_layer_from_oracle_stem():
    # layer 0 alone (conv + windowed attention), three chunks with a ragged tail
    n = 128000 * 2 + 40000
    pcm = synth.pcm_tones(21, n)
    om = oracle_model(1)
    ref, d = om.encode(pcm, dumps=True)
    enc = encoder(1, 600_000)
    x, offs = enc.forward([dev(pcm)], stage=binding.STAGE_LAYERS)
    assert offs == [0, oracle.num_tokens(n)]
    assert_rows_close(x.cpu().numpy(), d["enc"], "after layer 0")
    y, _ = enc.forward([dev(pcm)])
    assert_rows_close(y.cpu().numpy(), ref, "1-layer rows")


def test_bf16_output_matches_f32_output(tiny_case):
    pcm, out, _ = tiny_case
    enc = encoder(4, 600_000, out_dtype=binding.OUT_BF16)
    y, _ = enc.forward([dev(pcm)])
    assert y.dtype == torch.bfloat16
    assert_rows_close(y.float().cpu().numpy(), out, "bf16 rows")


# ------------------------------------------------------- full-size workloads

def test_single_30s_clip_full():
    pcm = synth.pcm_30s(1)
    enc = encoder(32, 9_600_000, 16)
    y, offs = enc.forward([dev(pcm)])
    assert offs == [0, 375] and y.shape == (375, 2048)
    ref = oracle_model(32).encode(pcm)
    assert_rows_close(y.cpu().numpy(), ref, "30 s rows")


def test_batch16_sampled_windows_and_invariance():
    clips = synth.pcm_batch(16)
    enc = encoder(32, 9_600_000, 16)
    y, offs = enc.forward([dev(c) for c in clips])
    assert offs[-1] == sum(oracle.num_tokens(c.size) for c in clips)
    Y = y.cpu().numpy()
    om = oracle_model(32)
    # one window of every clip: its first, its last (ragged) or a middle one
    for i in range(16):
        pcm = clips[i]
        nc = oracle.num_chunks(pcm.size)
        c = [0, nc - 1, nc // 2][i % 3]
        ref = om.encode_chunks(pcm, c, c + 1)
        t0 = offs[i] + 100 * c
        assert_rows_close(Y[t0:t0 + ref.shape[0]], ref, f"clip {i} chunk {c}")
    # a clip encoded alone gives the same rows as inside the batch
    for i in [3, 15]:
        yi, _ = enc.forward([dev(clips[i])])
        np.testing.assert_array_equal(yi.cpu().numpy(), Y[offs[i]:offs[i + 1]])


def test_10min_clip_sampled_windows():
    pcm = synth.pcm_long(2, 9_600_000)
    enc = encoder(32, 9_600_000, 16)
    y, offs = enc.forward([dev(pcm)])
    assert offs == [0, 7500]
    Y = y.cpu().numpy()
    om = oracle_model(32)
    gmax = oracle.clip_log_max(pcm)
    for c in list(range(0, 75, 8)) + [37, 74]:  # 12 of the 75 windows, spread over the clip
        ref = om.encode_chunks(pcm, c, c + 1, gmax=gmax)
        assert_rows_close(Y[100 * c:100 * c + 100], ref, f"10-min window {c}")


def test_60min_streamed_equals_whole_clip_and_oracle():
    n = 57_600_000
    pcm = synth.pcm_long(3, n)
    enc = encoder(32, 57_600_000, 1)
    x = dev(pcm)
    whole, offs = enc.forward([x])
    assert offs == [0, 45000]
    lm = enc.log_max(x)
    piece = 1_024_000
    rows = []
    for b in range(0, n, piece):
        e = min(b + piece, n)
        y, o = enc.forward([(x, b, e, lm)])
        assert o[1] == (800 if e - b == piece else 200)
        rows.append(y)
    streamed = torch.cat(rows)
    torch.cuda.synchronize()
    W = whole.cpu().numpy()
    # the same frames, chunks and per-row arithmetic: the rows agree bit for
    # bit (the tile widths differ with the row count, which changes no
    # element's arithmetic)
    np.testing.assert_array_equal(streamed.cpu().numpy(), W)
    om = oracle_model(32)
    gmax = oracle.clip_log_max(pcm)
    assert abs(float(lm.item()) - gmax) < 1e-4
    for c in [0, 79, 80, 225, 447, 448, 449]:  # ends, piece boundaries, the middle and the 200-token tail
        ref = om.encode_chunks(pcm, c, c + 1, gmax=gmax)
        assert_rows_close(W[100 * c:100 * c + ref.shape[0]], ref, f"60-min window {c}")


# ---------------------------------------------------------------- edge cases

def test_long_clip_split_over_ranks_equals_whole_clip():
    # three ranks simulated on one GPU: each takes its range's log-mel maximum,
    # the maxima are max-reduced (here on the host, over NCCL/gloo across
    # processes), each range is encoded against the common maximum, and the
    # ranks' rows, in rank order, are the whole clip's rows bit for bit
    n = 5 * 128000 + 37000
    pcm = synth.pcm_long(3, n)
    enc = encoder(4, 1_024_000)
    x = dev(pcm)
    whole, _ = enc.forward([x])
    whole = whole.cpu().numpy()
    world = 3
    maxima = [float(enc.range_log_max(x, b, e).item()) for b, e in shard.chunk_ranges(n, world)]
    gmax = max(maxima)
    assert gmax == float(enc.log_max(x).item())
    parts = []
    for r in range(world):
        rows, first = shard.encode_range(enc, x, r, world, lambda t: t.fill_(gmax))
        assert first == sum(p.shape[0] for p in parts)
        parts.append(rows.cpu().numpy())
    np.testing.assert_array_equal(np.concatenate(parts), whole)


def test_ragged_batch_with_empty_and_tiny_clips():
    enc = encoder(4, 600_000, 8)
    lens = [0, 170, 16000, 128000, 128160, 100]
    clips = [synth.pcm_tones(30 + i, n) for i, n in enumerate(lens)]
    y, offs = enc.forward([dev(c) if c.size else torch.empty(0, device="cuda") for c in clips])
    assert offs == list(np.cumsum([0] + [oracle.num_tokens(n) for n in lens]))
    om = oracle_model(4)
    Y = y.cpu().numpy()
    for i, c in enumerate(clips):
        ref = om.encode(c)
        assert_rows_close(Y[offs[i]:offs[i + 1]], ref, f"clip of {lens[i]} samples")


def test_deterministic_and_prompt_independent(tiny_case):
    pcm, _, _ = tiny_case
    enc = encoder(4, 600_000)
    a, _ = enc.forward([dev(pcm)])
    b, _ = enc.forward([dev(pcm)])
    assert torch.equal(a, b)


def test_host_end_to_end_matches_device_path(tiny_case):
    pcm, _, _ = tiny_case
    enc = encoder(4, 600_000, 4)
    clips = [pcm, synth.pcm_tones(5, 30000)]
    yd, od = enc.forward([dev(c) for c in clips])
    yh, oh = enc.forward_host(clips)
    assert od == oh
    np.testing.assert_array_equal(yh, yd.cpu().numpy())


def test_capacity_and_range_errors():
    enc = encoder(4, 600_000, 2)
    x = dev(synth.pcm_tones(1, 700_000))
    with pytest.raises(binding.MossEncError) as e:
        enc.forward([x])
    assert e.value.status == 2
    with pytest.raises(binding.MossEncError) as e:
        enc.forward([(x, 1000, 700_000, None)])
    assert e.value.status == 1
    with pytest.raises(binding.MossEncError) as e:
        enc.forward([x[:1000]] * 3)
    assert e.value.status == 2
    enc.synchronize()


def test_graph_replay_matches_eager_launches(tiny_case):
    # On a non-default stream a request that repeats the previous one is
    # captured as one CUDA graph and replayed after that; a new request runs
    # launch by launch (no capture for a stream of distinct requests); with
    # profiling on, every request runs launch by launch.
    pcm, out, _ = tiny_case
    s = torch.cuda.Stream()
    enc = binding.Encoder(weights(4), 4, 600_000, 2, stream=s)
    xa, xb = dev(pcm), dev(synth.pcm_tones(8, 40000))
    with torch.cuda.stream(s):
        ya = torch.empty((13, 2048), dtype=torch.float32, device="cuda")
        yb = torch.empty((13 + binding.num_tokens(40000), 2048), dtype=torch.float32, device="cuda")
    torch.cuda.synchronize()
    got = []
    with torch.cuda.stream(s):        # the copies below follow the forwards on their stream
        for _ in range(3):            # launched, captured, replayed
            enc.forward([xa], out=ya)
            got.append(ya.clone())
        enc.forward([xa, xb], out=yb)  # a new request: launched
        yb1 = yb.clone()
        enc.forward([xa], out=ya)     # the captured request again: replayed
        got.append(ya.clone())
        enc.profile_enable(2000)
        enc.forward([xa], out=ya)     # launched one by one
        got.append(ya.clone())
        enc.forward([xa, xb], out=yb)
        stats = enc.profile_read()
        enc.profile_enable(0)
    enc.synchronize()
    torch.cuda.synchronize()
    for g in got[1:]:
        assert torch.equal(got[0], g)
    assert torch.equal(yb1, yb)
    assert torch.equal(yb1[:13], got[0])
    assert "gemm_fc1" in stats and stats["gemm_fc1"]["launches"] == 2 * 4
    assert_rows_close(got[0].cpu().numpy(), out, "graph rows")
    enc.close()


def test_pieces_of_one_shape_share_a_graph():
    # Pieces of one long clip with the same chunk structure are one request
    # shape: the first runs launch by launch, the second is captured, the
    # rest replay that graph with their own tables and output ranges.  The
    # rows are the whole clip's bit for bit.
    n = 5 * 128000 + 37000
    pcm = synth.pcm_long(5, n)
    s = torch.cuda.Stream()
    enc = binding.Encoder(weights(4), 4, n, 1, stream=s)
    x = dev(pcm)
    with torch.cuda.stream(s):
        whole, _ = enc.forward([x])
        lm = enc.log_max(x)
        out = torch.empty_like(whole)
        o = 0
        for b in range(0, n, 128000):
            e = min(b + 128000, n)
            t = binding.range_tokens(n, b, e)
            enc.forward([(x, b, e, lm)], out=out[o:o + t])
            o += t
    enc.synchronize()
    torch.cuda.synchronize()
    assert o == whole.shape[0]
    assert torch.equal(out, whole)
    enc.close()


def test_bounded_wait_reports_timeout_and_context_survives(tiny_case):
    pcm, out, _ = tiny_case
    enc = encoder(4, 600_000)
    enc.selftest_timeout(50)
    with pytest.raises(binding.MossEncError) as e:
        enc.synchronize()
    assert e.value.status == 5
    enc.synchronize()  # flag cleared
    y, _ = enc.forward([dev(pcm)])
    assert_rows_close(y.cpu().numpy(), out, "rows after a device timeout")
