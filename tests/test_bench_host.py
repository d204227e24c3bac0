"""Host-side arithmetic of bench.py (no device): the method's FLOP count
per token that every roofline fraction divides by, derived here again from
the layer shapes of the page "MOSS-Transcribe-preview-2B - GGUF"
("Architecture" table); the gate that reports committed ncu DRAM bytes only
for the GEMM sources they were captured from; and the weak-scaling total."""
import bench


def test_model_flops_matches_the_layer_shapes():
    d, dqkv, dff, heads, hd, win = 1280, 3840, 5120, 20, 64, 100
    # per token of a full 100-token window
    layer = 2 * d * dqkv + 2 * d * d + 2 * d * dff + 2 * dff * d + 2 * 2 * heads * hd * win
    head = 2 * d * d + 2 * d * 2048
    adapter = 2 * 2048 * 8192 * 2 + 2 * 8192 * 2048
    # the stem per 800-frame chunk (100 tokens): conv1 1 -> 480 on 400 x 64
    # outputs, conv2 / conv3 480 -> 480 (3 x 3) on 200 x 32 and 100 x 16,
    # conv_out 7680 -> 1280 on 100 rows
    stem = (400 * 64 * 480 * 9 * 2 + 200 * 32 * 480 * 480 * 9 * 2 + 100 * 16 * 480 * 480 * 9 * 2
            + 100 * 7680 * 1280 * 2) / 100
    for n_layers in (1, 4, 32):
        want = stem + n_layers * layer + head + adapter
        assert abs(bench.model_flops(1, n_layers) - want) <= 1e-3 * want
    # a layer tap adds one head + adapter set
    assert abs(bench.model_flops(1, 32, 1) - bench.model_flops(1, 32) - (head + adapter)) <= 1e-3 * (head + adapter)


def test_traffic_is_reported_only_for_the_captured_sources(monkeypatch):
    got = bench.profiled_traffic("gemm_fc2")
    assert got is None or got > 0
    monkeypatch.setattr(bench, "gemm_source_hash", lambda: "not-the-captured-hash")
    assert bench.profiled_traffic("gemm_fc2") is None
    assert bench.profiled_traffic("no_such_kernel") is None


def test_weak_scaling_counts_every_rank():
    assert bench.weak_scaling_throughput(1, 4608, 8.0) == 4608 / 8e-3
    assert bench.weak_scaling_throughput(8, 4608, 8.0) == 8 * 4608 / 8e-3
