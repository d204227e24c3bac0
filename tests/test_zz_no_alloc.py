"""The allocation-free log-mel entry point (moss_enc_logmel_static).

Some callers cannot allocate device memory: a process whose GPU memory is
owned by another framework's pool, or a real-time front end that must not
allocate once running.  moss_enc_logmel_static serves them with scratch in a
static device array.  Here it is called through the C ABI twice in a row and
compared with the handle-based moss_enc_logmel on the same clips.

This file is collected last on purpose, so that a run stopping at the first
failure has run every other test first.
"""
import numpy as np
import pytest

from audio_encoder_b200 import binding, synth
from conftest import weights
from metrics import MEL_ATOL

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


def test_static_logmel_matches_handle_logmel_twice():
    enc = binding.Encoder(weights(1), 1, max_samples=600_000, max_clips=1)
    n_long = 128000 * 2 + 30000
    pcms = [synth.pcm_tones(40, 16000), synth.pcm_30s(1), synth.pcm_long(41, n_long), synth.pcm_tones(42, 170)]
    xs = [torch.from_numpy(p).cuda() for p in pcms]
    lm_given = torch.tensor([0.5], dtype=torch.float32, device="cuda")
    clips = [xs[0], xs[1], (xs[2], 128000, 256000, None), (xs[2], 0, n_long, lm_given), xs[3]]
    refs = []
    for c in clips:
        if isinstance(c, tuple):
            pcm, b, e, lm = c
            refs.append(enc.logmel(pcm, b, e, lm))
        else:
            refs.append(enc.logmel(c))
    torch.cuda.synchronize()
    for call in range(2):  # two calls in a row share the static scratch
        mels, mx = binding.logmel_static(clips)
        torch.cuda.synchronize()
        assert len(mels) == len(clips)
        for i, ((ref_mel, ref_mx), got) in enumerate(zip(refs, mels)):
            assert got.shape == ref_mel.shape, (call, i)
            np.testing.assert_allclose(got.cpu().numpy(), ref_mel.cpu().numpy(), rtol=0, atol=MEL_ATOL)
            assert abs(float(mx[i].item()) - float(ref_mx.item())) <= MEL_ATOL, (call, i)
    assert float(mx[3].item()) == 0.5  # the caller's maximum is used as given
    enc.close()


def test_static_logmel_rejects_too_many_clips():
    x = torch.zeros(16000, dtype=torch.float32, device="cuda")
    with pytest.raises(binding.MossEncError) as e:
        binding.logmel_static([x] * (binding.STATIC_MAX_CLIPS + 1))
    assert e.value.status == 2


def test_static_logmel_refuses_a_capturing_stream():
    # Each call copies its clip descriptors from host memory that lives only
    # for the call, so it must not be recorded into a CUDA graph: under
    # capture it returns INVALID_ARG and enqueues nothing.
    x = torch.from_numpy(synth.pcm_tones(43, 16000)).cuda()
    binding.logmel_static([x])  # the first call on the device sets up the scratch
    torch.cuda.synchronize()
    s = torch.cuda.Stream()
    g = torch.cuda.CUDAGraph()
    status = None
    y = torch.zeros(4, device="cuda")
    with torch.cuda.graph(g, stream=s):
        try:
            binding.logmel_static([x], stream=s)
        except binding.MossEncError as e:
            status = e.status
        y.add_(1.0)  # the graph holds one ordinary kernel
    assert status == 1
    g.replay()
    torch.cuda.synchronize()
    assert float(y[0].item()) == 1.0
