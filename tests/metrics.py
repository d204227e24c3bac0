"""Comparison metrics shared by the parity tests."""
import numpy as np

# Tolerances of the workload statement: mel within 1e-4 absolute; rows with
# per-row cosine >= 0.999 and max |err| <= 3e-2 * rms of the reference row.
MEL_ATOL = 1e-4
ROW_COS = 0.999
ROW_MAXERR_RMS = 3e-2


def row_metrics(got, ref):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    dot = (got * ref).sum(1)
    cos = dot / (np.linalg.norm(got, axis=1) * np.linalg.norm(ref, axis=1) + 1e-30)
    rms = np.sqrt((ref ** 2).mean(1))
    maxerr = np.abs(got - ref).max(1)
    return cos, maxerr / (rms + 1e-30)


def assert_rows_close(got, ref, what=""):
    if np.asarray(ref).shape[0] == 0:
        assert np.asarray(got).shape == np.asarray(ref).shape
        return
    cos, rel = row_metrics(got, ref)
    bad = (cos < ROW_COS) | (rel > ROW_MAXERR_RMS)
    assert not bad.any(), (f"{what}: {bad.sum()} of {len(cos)} rows out of tolerance; "
                           f"min cos {cos.min():.6f}, max err/rms {rel.max():.4f} (row {int(rel.argmax())})")
    return cos.min(), rel.max()
