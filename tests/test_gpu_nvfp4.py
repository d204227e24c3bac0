"""NVFP4 GEMMs (page "Ossicle-4B", section "Quantized: NVFP4 and INT4 in
vLLM"): the block-scaled FP4 tensor-core GEMM against an fp64 product of the
same quantised operands.  The operands come from the oracle's NVFP4
quantiser (pinned in test_oracle_nvfp4_pins.py) and are packed here into the
library's layout: two E2M1 codes per byte (even k low), E4M3 scales in
512-byte atoms of 128 rows x 64 k."""
import numpy as np
import pytest

import oracle
from audio_encoder_b200 import binding
from conftest import weights

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")

GRID = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


@pytest.fixture(scope="module")
def enc():
    e = binding.Encoder(weights(1), 1, max_samples=16000, max_clips=1)
    yield e
    e.close()


def pack(x, per_row):
    """NVFP4 operands of x [rows][K]: (codes [rows][K/2] uint8, scale atoms
    uint8, g, units) with rows padded to 128 in the atoms."""
    unit, g, codes, bs = oracle.quant_nvfp4(x, per_row)
    rows, K = x.shape
    packed = (codes[:, 0::2] | (codes[:, 1::2] << 4)).astype(np.uint8)
    rb = (rows + 127) // 128
    atoms = np.zeros((rb, K // 64, 512), dtype=np.uint8)
    e4 = torch.from_numpy(bs).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(torch.from_numpy(e4).view(torch.float8_e4m3fn).to(torch.float32).numpy(), bs)
    r = np.arange(rows)[:, None]
    b = np.arange(K // 16)[None, :]
    off = (r % 32) * 16 + ((r % 128) // 32) * 4 + (b % 4)
    atoms[r // 128, b // 4, off] = e4
    return packed, atoms.reshape(-1), g, unit


@pytest.mark.parametrize("M,N,K", [(128, 128, 256), (300, 256, 1280), (1000, 384, 2048)])
@pytest.mark.parametrize("epi", [0, 1])
def test_nvfp4_gemm_vs_fp64(enc, M, N, K, epi):
    rng = np.random.default_rng(M + N + K + epi)
    A = (rng.standard_normal((M, K)) * rng.uniform(0.2, 3.0, (M, 1))).astype(np.float32)
    A[M // 3] = 0.0  # a zero row: g = 0, codes 0
    B = (rng.standard_normal((N, K)) * 0.05).astype(np.float32)
    bias = (rng.standard_normal(N) * 0.1).astype(np.float32)
    a4, sfa, ga, ua = pack(A, True)
    b4, sfb, gb, ub = pack(B, False)
    ref = (ua.astype(np.float64) @ ub.astype(np.float64).T) * ga[:, None].astype(np.float64) * float(gb[0]) + bias
    if epi == 1:
        ref = torch.nn.functional.gelu(torch.from_numpy(ref)).numpy()
    dev = "cuda"
    out = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    enc.gemm_nvf4(torch.from_numpy(a4).to(dev), torch.from_numpy(sfa).to(dev), torch.from_numpy(ga).to(dev),
                  torch.from_numpy(b4).to(dev), torch.from_numpy(sfb).to(dev),
                  torch.full((N,), float(gb[0]), device=dev), torch.from_numpy(bias).to(dev), out, epi)
    enc.synchronize()
    got = out.float().cpu().numpy().astype(np.float64)
    scale = max(np.abs(ref).max(), 1.0)
    err = np.abs(got - ref).max()
    assert err <= 1e-2 * scale, (err, scale)
    # the zero row is the bias (through the epilogue)
    np.testing.assert_allclose(got[M // 3], ref[M // 3], rtol=1e-2, atol=1e-2)
