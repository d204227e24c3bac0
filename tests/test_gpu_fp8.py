"""FP8 GEMMs (page "Ossicle-4B", "Quantized: NVFP4 and INT4 in vLLM": the
low-precision builds quantise the audio encoder's weights and activations).

The e4m3 GEMM (kind::f8f6f4) against a PyTorch fp32 matmul of the same e4m3
operands and scales; the e4m3 LayerNorm against the oracle's quantisation of
the same rows; and the FP8 encoder (q/k/v and fc1 on e4m3 operands) against
the oracle's FP8 model on the 1 s / 4-layer case and the single 30 s clip."""
import numpy as np
import pytest

import oracle
from audio_encoder_b200 import binding, synth
from conftest import weights
from metrics import FP8_ROW_COS, FP8_ROW_MAXERR_RMS, assert_rows_close, row_metrics

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def enc():
    e = binding.Encoder(weights(1), 1, max_samples=16000, max_clips=1)
    yield e
    e.close()


def e4m3_rows(x):
    """Per-row e4m3 operands (uint8 bits) and scales of an fp32 matrix, by
    PyTorch's float8 conversion (row max -> 448)."""
    s = x.abs().amax(dim=1) / 448.0
    q = (x / s[:, None]).clamp(-448, 448).to(torch.float8_e4m3fn)
    return q.view(torch.uint8), s


@pytest.mark.parametrize("block_n", [128, 256])
@pytest.mark.parametrize("epi", [0, 1])
@pytest.mark.parametrize("M,K,N", [(1, 256, 512), (300, 1280, 3840), (1000, 1280, 5120)])
def test_e4m3_gemm_vs_torch(enc, block_n, epi, M, K, N):
    g = torch.Generator().manual_seed(M + K + N + epi + block_n)
    A = torch.randn(M, K, generator=g) * 2.0
    W = torch.randn(N, K, generator=g) / K ** 0.5
    a8, sa = e4m3_rows(A)
    w8, sw = e4m3_rows(W)
    bias = torch.randn(N, generator=g) * 0.1
    out = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    enc.gemm_f8(a8.cuda(), w8.cuda(), sa.cuda(), sw.cuda(), bias.cuda(), out, epi, block_n)
    enc.synchronize()
    ref = (a8.view(torch.float8_e4m3fn).float() @ w8.view(torch.float8_e4m3fn).float().T) * sa[:, None] * sw[None, :] + bias
    if epi == 1:
        ref = torch.nn.functional.gelu(ref)
    err = (out.float().cpu() - ref).abs().max().item()
    assert err <= 1e-2 * max(ref.abs().max().item(), 1.0), err


@pytest.fixture(scope="module")
def tiny_f8():
    blob = weights(4)
    pcm = synth.pcm_tones(0, 16000)
    return blob, pcm, oracle.Model(blob, 4, weight_bits=8).encode(pcm)


def test_fp8_tiny_encoder_matches_oracle_fp8_model(tiny_f8):
    blob, pcm, ref = tiny_f8
    e = binding.Encoder(blob, 4, 16000, 1, fp8=True)
    rows, offs = e.forward([torch.from_numpy(pcm).cuda()])
    e.synchronize()
    assert offs == [0, 13]
    got = rows.cpu().numpy()
    ref16 = oracle.Model(blob, 4).encode(pcm)
    c8, e8 = row_metrics(got, ref)
    c16, e16 = row_metrics(got, ref16)
    print(f"FP8 tiny: vs FP8 oracle min cos {c8.min():.6f} max err/rms {e8.max():.4f}; "
          f"vs bf16 oracle min cos {c16.min():.6f} max err/rms {e16.max():.4f}")
    assert_rows_close(got, ref, "FP8 tiny rows", FP8_ROW_COS, FP8_ROW_MAXERR_RMS)
    assert e8.max() < e16.max()  # the rows follow the FP8 model, not the bf16 one
    e.close()


def test_fp8_single_30s_clip_matches_oracle_fp8_model():
    blob = weights(32)
    pcm = synth.pcm_30s(1)
    e = binding.Encoder(blob, 32, 480000, 1, fp8=True)
    rows, offs = e.forward([torch.from_numpy(pcm).cuda()])
    e.synchronize()
    assert offs == [0, 375]
    om = oracle.Model(blob, 32, weight_bits=8)
    ref = om.encode(pcm)
    om.close()
    om16 = oracle.Model(blob, 32)
    ref16 = om16.encode(pcm)
    om16.close()
    got = rows.cpu().numpy()
    c8, e8 = row_metrics(got, ref)
    c16, e16 = row_metrics(got, ref16)
    print(f"FP8 30 s: vs FP8 oracle min cos {c8.min():.6f} max err/rms {e8.max():.4f} (mean {e8.mean():.4f}); "
          f"vs bf16 oracle min cos {c16.min():.6f} max err/rms {e16.max():.4f} (mean {e16.mean():.4f})")
    assert_rows_close(got, ref, "FP8 30 s rows", FP8_ROW_COS, FP8_ROW_MAXERR_RMS)
    assert e8.mean() < 0.5 * e16.mean()  # the rows follow the FP8 model, not the bf16 one
    e.close()


def test_fp8_batch_invariance(tiny_f8):
    # the e4m3 LayerNorm rows and their scales are per row: a clip's rows are
    # the same alone and in a batch (tile widths change no element's sum)
    blob, pcm, _ = tiny_f8
    e = binding.Encoder(blob, 4, 600_000, 2, fp8=True)
    x = torch.from_numpy(pcm).cuda()
    alone, _ = e.forward([x])
    both, _ = e.forward([x, torch.from_numpy(synth.pcm_tones(9, 480000)).cuda()])
    e.synchronize()
    assert torch.equal(both[:13], alone)
    e.close()
