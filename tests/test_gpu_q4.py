"""4-bit weights (page "Ossicle-4B", "Long Audio", the note under the table:
4-bit weights for the audio encoder, round to nearest, groups of 128).

The 4-bit GEMM against the bf16 GEMM on the oracle's dequantised weights (the
converter produces exactly those bf16 values, so the products and their
order are the same: bit for bit), and against a PyTorch fp32 matmul; the
4-bit encoder against the oracle's 4-bit model on the 1 s / 4-layer case and
the single 30 s clip; and the weight memory it saves."""
import numpy as np
import pytest

import oracle
from audio_encoder_b200 import binding, synth
from conftest import weights
from metrics import assert_rows_close

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")


def packed(codes, scales):
    """Codes [N][K] (q + 8) -> [N][K/2] bytes (even k low nibble); scales
    [N][K/128] -> [K/128][N]."""
    c = codes.astype(np.uint8)
    return (c[:, 0::2] | (c[:, 1::2] << 4)).astype(np.uint8), np.ascontiguousarray(scales.T)


@pytest.fixture(scope="module")
def enc():
    e = binding.Encoder(weights(1), 1, max_samples=16000, max_clips=1)
    yield e
    e.close()


@pytest.mark.parametrize("block_n", [128, 160, 256, 320])
@pytest.mark.parametrize("epi", [0, 1, 2, 5])
@pytest.mark.parametrize("M,K", [(1, 128), (300, 1280), (1000, 5120)])
def test_q4_gemm_equals_bf16_gemm_on_dequantised_weights(enc, block_n, epi, M, K):
    N = {128: 1280, 160: 480, 256: 2048, 320: 1280}[block_n]
    g = torch.Generator().manual_seed(M + K + epi + block_n)
    A = (torch.randn(M, K, generator=g) / K ** 0.25).bfloat16()
    W = (torch.randn(N, K, generator=g) / K ** 0.5).bfloat16()
    deq, codes, scales = oracle.quant_rtn4(W.view(torch.int16).numpy().view(np.uint16))
    bq, bs = packed(codes, scales)
    Wd = torch.from_numpy(deq.view(np.int16)).view(torch.bfloat16)
    bias = torch.randn(N, generator=g) * 0.1
    base = torch.randn(M, N, generator=g)
    dt = torch.bfloat16 if epi in (0, 1) else torch.float32
    outs = []
    for q4 in (True, False):
        out = base.clone().cuda() if epi == 2 else torch.empty(M, N, dtype=dt, device="cuda")
        if q4:
            enc.gemm_q4(A.cuda(), torch.from_numpy(bq).cuda(), torch.from_numpy(bs).cuda(), bias.cuda(), out, epi, block_n)
        else:
            enc.gemm(A.cuda(), Wd.cuda(), bias.cuda(), out, epi, block_n, True)
        outs.append(out)
    enc.synchronize()
    assert torch.equal(outs[0], outs[1])
    ref = A.float() @ Wd.float().T + bias
    if epi == 1:
        ref = torch.nn.functional.gelu(ref)
    if epi == 2:
        ref = ref + base
    tol = 2e-2 if epi in (0, 1) else 1e-3
    err = (outs[0].float().cpu() - ref).abs().max().item()
    assert err <= tol * max(ref.abs().max().item(), 1.0)


@pytest.fixture(scope="module")
def tiny_q4():
    blob = weights(4)
    pcm = synth.pcm_tones(0, 16000)
    ref = oracle.Model(blob, 4, weight_bits=4).encode(pcm)
    return blob, pcm, ref


def test_q4_tiny_encoder_matches_oracle_4bit_model(tiny_q4):
    blob, pcm, ref = tiny_q4
    e = binding.Encoder(blob, 4, 16000, 1, weight_bits=4)
    rows, offs = e.forward([torch.from_numpy(pcm).cuda()])
    e.synchronize()
    assert offs == [0, 13]
    assert_rows_close(rows.cpu().numpy(), ref, "4-bit tiny rows")
    # and it is not the bf16 model: the quantisation moves the rows
    ref16 = oracle.Model(blob, 4).encode(pcm)
    assert np.abs(ref16 - ref).max() > 1e-3 * np.abs(ref16).max()
    e.close()


def test_q4_single_30s_clip_matches_oracle_and_saves_memory():
    blob = weights(32)
    pcm = synth.pcm_30s(1)
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    e4 = binding.Encoder(blob, 32, 480000, 1, weight_bits=4)
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    e16 = binding.Encoder(blob, 32, 480000, 1)
    torch.cuda.synchronize()
    free2, _ = torch.cuda.mem_get_info()
    used4, used16 = free0 - free1, free1 - free2
    x = torch.from_numpy(pcm).cuda()
    rows, offs = e4.forward([x])
    e4.synchronize()
    assert offs == [0, 375]
    om = oracle.Model(blob, 32, weight_bits=4)
    ref = om.encode(pcm)
    assert_rows_close(rows.cpu().numpy(), ref, "4-bit 30 s rows")
    om.close()
    # weights + workspace: the 4-bit handle holds well under half the memory
    assert used4 < 0.5 * used16, (used4, used16)
    e4.close()
    e16.close()


def test_q4_fused_and_expanded_paths_agree_bit_for_bit(tiny_q4):
    # a batch of one 256-row tile expands the codes inside the GEMM; a larger
    # batch expands each matrix once into a scratch and runs the bf16 GEMM:
    # the same weight values and arithmetic, so a clip's rows are the same
    blob, pcm, _ = tiny_q4
    e = binding.Encoder(blob, 4, 600_000, 2, weight_bits=4)
    x = torch.from_numpy(pcm).cuda()
    alone, _ = e.forward([x])
    other = torch.from_numpy(synth.pcm_tones(9, 480000)).cuda()
    both, offs = e.forward([x, other])
    e.synchronize()
    assert offs[-1] > 256
    assert torch.equal(both[:13], alone)
    e.close()
