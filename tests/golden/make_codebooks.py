"""Writes the codebook fixtures used by the parity tests.

Calls only oracle/ (k-means on seeded standard normals, as the pages build
the codebook: "NSNQuant ..." technical summary, Metodologia 3; README "Codebook
tuning" for the --abs variant).  Run from the repository root:
    python tests/golden/make_codebooks.py
"""
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

from oracle.codebook_oracle import build_codebook  # noqa: E402

SPECS = {
    "codebook_1bit.txt": dict(seed=0x4E534E01, abs_mode=False),
    "codebook_2bit.txt": dict(seed=0x4E534E02, abs_mode=True),
}
N_SAMPLES, N_CODES, DIM, ITERS = 65536, 256, 8, 25

if __name__ == "__main__":
    for name, spec in SPECS.items():
        cb = build_codebook(spec["seed"], N_SAMPLES, N_CODES, DIM, spec["abs_mode"], ITERS)
        header = (f"oracle k-means codebook: seed={spec['seed']:#x} abs_mode={spec['abs_mode']} "
                  f"n_samples={N_SAMPLES} n_codes={N_CODES} dim={DIM} iters={ITERS}; "
                  f"written by tests/golden/make_codebooks.py")
        np.savetxt(os.path.join(HERE, name), cb, fmt="%.17g", header=header)
        print(name, cb.shape)
