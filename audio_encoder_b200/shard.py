"""One long clip encoded by several GPUs, each taking a contiguous range of
its 800-frame chunks (the attention windows).

Chunks are independent from the log-mel to the adapter; the one coupling is
the clip-wide log-mel maximum that sets the Whisper floor (page "Ossicle-4B",
"Long Audio": a piece's log-mel equals the whole clip's).  So each rank
takes the maximum over its own frames (moss_enc_range_log_max), the ranks
max-reduce that one float (the only collective), and each rank encodes its
range against the common maximum.  The rows of rank r are rows
row_offset(r) .. of the whole-clip encode, bit for bit.
"""
from __future__ import annotations

CHUNK_SAMPLES = 128000  # one 800-frame chunk = 8 s of 16 kHz audio


def chunk_ranges(n_samples: int, world: int):
    """Contiguous chunk-aligned sample ranges [(begin, end)] for `world`
    ranks, as even as whole chunks allow (earlier ranks take the extra
    chunk); ranks past the clip's chunk count get empty ranges at its end."""
    if world < 1:
        raise ValueError("world must be >= 1")
    n_chunks = -(-n_samples // CHUNK_SAMPLES) if n_samples > 0 else 0
    base, extra = divmod(n_chunks, world)
    out, c = [], 0
    for r in range(world):
        k = base + (1 if r < extra else 0)
        b = min(c * CHUNK_SAMPLES, n_samples)
        e = min((c + k) * CHUNK_SAMPLES, n_samples)
        out.append((b, e))
        c += k
    return out


def row_offset(n_samples: int, world: int, rank: int) -> int:
    """First whole-clip output row of `rank`'s range."""
    from . import binding
    b, _ = chunk_ranges(n_samples, world)[rank]
    return binding.range_tokens(n_samples, 0, b) if b > 0 else 0


def encode_range(enc, pcm, rank: int, world: int, max_reduce, out=None):
    """Encode this rank's range of the clip `pcm` (device fp32 [n]).

    max_reduce(t) replaces the device float tensor t ([1]) in place by the
    maximum over ranks (e.g. torch.distributed.all_reduce with op MAX);
    every rank calls it exactly once.  Returns (rows, first_row)."""
    import torch
    n = pcm.numel()
    b, e = chunk_ranges(n, world)[rank]
    if e > b:
        m = enc.range_log_max(pcm, b, e)
    else:  # no frames here: the identity of the max
        m = torch.full((1,), float("-inf"), dtype=torch.float32, device=pcm.device)
    max_reduce(m)
    first = row_offset(n, world, rank)
    if e == b:
        return torch.empty((0, 2048), dtype=torch.float32, device=pcm.device), first
    rows, _ = enc.forward([(pcm, b, e, m)], out=out)
    return rows, first
