"""Writes tiny_oracle_rows.json from the CPU oracle alone (no CUDA path).

Run from the repository root:  python tests/golden/make_golden.py
The file pins the oracle's own output on the 1 s / 4-layer workload so that
an accidental change to its arithmetic shows up as a failing test.
"""
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import oracle  # noqa: E402
from audio_encoder_b200 import synth  # noqa: E402


def main():
    m = oracle.Model(synth.make_weights(4, 1234), 4)
    out = m.encode(synth.pcm_tones(0, 16000))
    data = {
        "_about": "oracle rows for the 1 s tones clip (seed 0), 4 layers, weight seed 1234",
        "rows_first8": np.round(out[:, :8].astype(np.float64), 7).tolist(),
        "row_norms": np.round(np.linalg.norm(out, axis=1).astype(np.float64), 6).tolist(),
    }
    with open(os.path.join(os.path.dirname(os.path.abspath(__file__)), "tiny_oracle_rows.json"), "w") as f:
        json.dump(data, f, indent=1)


if __name__ == "__main__":
    main()
