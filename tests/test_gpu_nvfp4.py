"""NVFP4 GEMMs (page "Ossicle-4B", section "Quantized: NVFP4 and INT4 in
vLLM"): the block-scaled FP4 tensor-core GEMM against an fp64 product of the
same quantised operands (which come from the oracle's NVFP4 quantiser,
pinned in test_oracle_nvfp4_pins.py, packed here into the library's layout:
two E2M1 codes per byte, even k low, E4M3 scales in 512-byte atoms of 128
rows x 64 k); the activation quantiser against the oracle's bit for bit; and
the NVFP4 encoder (q/k/v and fc1 on NVFP4 operands) against the oracle's
NVFP4 model on the 1 s / 4-layer case and the single 30 s clip."""
import numpy as np
import pytest

import oracle
from audio_encoder_b200 import binding, synth
from conftest import weights
from metrics import NVFP4_ROW_COS, NVFP4_ROW_MAXERR_RMS, assert_rows_close, row_metrics

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


def test_nvf4_quant_rows_match_oracle(enc):
    # the activation quantiser (what the NVFP4 LayerNorm kernel applies after
    # the norm) against the oracle's, on the same fp32 rows: g, block scales
    # and codes bit for bit (a zero may carry either sign)
    rng = np.random.default_rng(5)
    M = 300
    x = (rng.standard_normal((M, 1280)) * rng.uniform(0.05, 40, (M, 1))).astype(np.float32)
    x[7] = 0.0
    x[8, :16] = 1e-30  # a block far below its row's maximum: scale 0, codes 0
    _, g_ref, codes_ref, bs_ref = oracle.quant_nvfp4(x, True)
    dev = "cuda"
    rb = (M + 127) // 128
    codes = torch.zeros((M, 640), dtype=torch.uint8, device=dev)
    sfa = torch.zeros(rb * 20 * 512, dtype=torch.uint8, device=dev)
    g = torch.empty(M, device=dev)
    enc.nvf4_quant_rows(torch.from_numpy(x).to(dev), codes, sfa, g)
    enc.synchronize()
    np.testing.assert_array_equal(g.cpu().numpy(), g_ref)
    c = codes.cpu().numpy()
    got = np.empty((M, 1280), dtype=np.uint8)
    got[:, 0::2] = c & 15
    got[:, 1::2] = c >> 4
    mag_g, mag_r = got & 7, codes_ref & 7
    np.testing.assert_array_equal(mag_g, mag_r)
    nz = mag_r != 0
    np.testing.assert_array_equal((got & 8)[nz], (codes_ref & 8)[nz])
    a = sfa.cpu().numpy().reshape(rb, 20, 512)
    r = np.arange(M)[:, None]
    b = np.arange(80)[None, :]
    e4 = a[r // 128, b // 4, (r % 32) * 16 + ((r % 128) // 32) * 4 + b % 4]
    bs = torch.from_numpy(np.ascontiguousarray(e4)).view(torch.float8_e4m3fn).to(torch.float32).numpy()
    np.testing.assert_array_equal(bs, bs_ref)


@pytest.fixture(scope="module")
def tiny_f4():
    blob = weights(4)
    pcm = synth.pcm_tones(0, 16000)
    return blob, pcm, oracle.Model(blob, 4, nvfp4=True).encode(pcm)


def test_nvfp4_tiny_encoder_matches_oracle_nvfp4_model(tiny_f4):
    blob, pcm, ref = tiny_f4
    e = binding.Encoder(blob, 4, 16000, 1, nvfp4=True)
    rows, offs = e.forward([torch.from_numpy(pcm).cuda()])
    e.synchronize()
    assert offs == [0, 13]
    got = rows.cpu().numpy()
    ref16 = oracle.Model(blob, 4).encode(pcm)
    c4, e4 = row_metrics(got, ref)
    c16, e16 = row_metrics(got, ref16)
    print(f"NVFP4 tiny: vs NVFP4 oracle min cos {c4.min():.6f} max err/rms {e4.max():.4f}; "
          f"vs bf16 oracle min cos {c16.min():.6f} max err/rms {e16.max():.4f}")
    assert_rows_close(got, ref, "NVFP4 tiny rows", NVFP4_ROW_COS, NVFP4_ROW_MAXERR_RMS)
    assert e4.max() < e16.max()  # the rows follow the NVFP4 model, not the bf16 one
    e.close()


def test_nvfp4_single_30s_clip_matches_oracle_nvfp4_model():
    blob = weights(32)
    pcm = synth.pcm_30s(1)
    e = binding.Encoder(blob, 32, 480000, 1, nvfp4=True)
    rows, offs = e.forward([torch.from_numpy(pcm).cuda()])
    e.synchronize()
    assert offs == [0, 375]
    om = oracle.Model(blob, 32, nvfp4=True)
    ref = om.encode(pcm)
    om.close()
    om16 = oracle.Model(blob, 32)
    ref16 = om16.encode(pcm)
    om16.close()
    got = rows.cpu().numpy()
    c4, e4 = row_metrics(got, ref)
    c16, e16 = row_metrics(got, ref16)
    print(f"NVFP4 30 s: vs NVFP4 oracle min cos {c4.min():.6f} max err/rms {e4.max():.4f} (mean {e4.mean():.4f}); "
          f"vs bf16 oracle min cos {c16.min():.6f} max err/rms {e16.max():.4f} (mean {e16.mean():.4f})")
    assert_rows_close(got, ref, "NVFP4 30 s rows", NVFP4_ROW_COS, NVFP4_ROW_MAXERR_RMS)
    assert e4.mean() < 0.5 * e16.mean()  # the rows follow the NVFP4 model, not the bf16 one
    e.close()


def test_nvfp4_batch_invariance(tiny_f4):
    # the activation g and block scales are per row: a clip's rows are the
    # same alone and in a batch
    blob, pcm, _ = tiny_f4
    e = binding.Encoder(blob, 4, 600_000, 2, nvfp4=True)
    x = torch.from_numpy(pcm).cuda()
    alone, _ = e.forward([x])
    both, _ = e.forward([x, torch.from_numpy(synth.pcm_tones(9, 480000)).cuda()])
    e.synchronize()
    assert torch.equal(both[:13], alone)
    e.close()
