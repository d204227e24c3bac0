"""The tensor-core GEMM with each fused epilogue against a plain PyTorch
fp32 matmul of the same bf16 operands (ragged M, several tiles, each tile
width)."""
import pytest

from audio_encoder_b200 import binding
from conftest import weights

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def enc():
    e = binding.Encoder(weights(1), 1, max_samples=16000, max_clips=1)
    yield e
    e.close()


@pytest.mark.parametrize("pair,block_n", [(False, 128), (False, 160), (False, 192), (False, 256), (True, 128),
                                          (True, 160), (True, 192), (True, 256), (True, 320)])
@pytest.mark.parametrize("epi", [0, 1, 2, 5])
@pytest.mark.parametrize("M,K", [(1, 64), (300, 1280), (1000, 4608), (4608, 1280)])
def test_gemm_epilogues(enc, pair, block_n, epi, M, K):
    N = {128: 1280, 160: 480, 192: 3840, 256: 2048, 320: 1280}[block_n]
    g = torch.Generator().manual_seed(M * 7 + K + epi + block_n)
    A = (torch.randn(M, K, generator=g) / K ** 0.25).bfloat16()
    B = (torch.randn(N, K, generator=g) / K ** 0.25).bfloat16()
    bias = torch.randn(N, generator=g) * 0.1
    ref = A.float() @ B.float().T + bias
    if epi == 1:
        ref = torch.nn.functional.gelu(ref)
    base = torch.randn(M, N, generator=g)
    if epi == 2:
        ref = ref + base
    if epi in (0, 1):
        out = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    else:
        out = base.clone().cuda() if epi == 2 else torch.empty(M, N, device="cuda")
    enc.gemm(A.cuda(), B.cuda(), bias.cuda(), out, epi, block_n, pair)
    enc.synchronize()
    got = out.float().cpu()
    tol = 2e-2 if epi in (0, 1) else 1e-3
    err = (got - ref).abs().max().item()
    scale = ref.abs().max().item()
    assert err <= tol * max(scale, 1.0), (err, scale)


@pytest.mark.parametrize("M,K,N,epi", [(375, 1280, 3840, 0), (512, 1280, 3840, 0), (375, 8192, 2048, 0),
                                       (1000, 8192, 2048, 5)])
def test_gemm_does_not_depend_on_tile_width(enc, M, K, N, epi):
    # QKV of a batch of at most 512 tokens and the adapter's down-projection
    # of a small batch run on 128-wide tiles, larger ones on 256-wide: same
    # arithmetic per output element, same bits
    g = torch.Generator().manual_seed(M + K + 1)
    A = (torch.randn(M, K, generator=g) / K ** 0.25).bfloat16().cuda()
    B = (torch.randn(N, K, generator=g) / K ** 0.25).bfloat16().cuda()
    bias = (torch.randn(N, generator=g) * 0.1).cuda()
    outs = []
    for block_n in (128, 256):
        out = torch.empty(M, N, dtype=torch.bfloat16 if epi == 0 else torch.float32, device="cuda")
        enc.gemm(A, B, bias, out, epi, block_n, True)
        outs.append(out)
    torch.cuda.synchronize()
    assert torch.equal(outs[0], outs[1])


@pytest.mark.parametrize("M,K", [(375, 1280), (800, 5120), (4608, 1280)])
def test_residual_gemm_does_not_depend_on_tile_width(enc, M, K):
    # the forward picks 128-, 160- or 320-wide tiles for the N = 1280 residual
    # GEMMs by batch size; every output element's sum over K runs through the
    # same MMA k-steps whatever the width, so the results agree bit for bit
    # (which keeps a clip's rows the same alone and in a batch)
    N = 1280
    g = torch.Generator().manual_seed(M + K)
    A = (torch.randn(M, K, generator=g) / K ** 0.25).bfloat16().cuda()
    B = (torch.randn(N, K, generator=g) / K ** 0.25).bfloat16().cuda()
    bias = (torch.randn(N, generator=g) * 0.1).cuda()
    base = torch.randn(M, N, generator=g).cuda()
    outs = []
    for block_n in (128, 160, 320):
        out = base.clone()
        enc.gemm(A, B, bias, out, 2, block_n, True)
        outs.append(out)
    torch.cuda.synchronize()
    assert torch.equal(outs[0], outs[1]) and torch.equal(outs[0], outs[2])


def test_fast_gelu_matches_erff(enc):
    # Abramowitz & Stegun 7.1.28 erf against CUDA's erff
    assert enc.selftest_gelu() <= 1e-6
