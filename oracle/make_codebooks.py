"""Train the joint 2D Lloyd-Max codebooks and write them as shipped tables.

Usage: python -m oracle.make_codebooks [N ...]

Writes ``vector_codebook_codec_b200/codebooks/qamw_lloyd_N{N}.npy`` (float32
[N, 2], centroids in trained order) and ``manifest.json`` (seed, sample count,
iterations, convergence, train distortion, polar split and its distortion).
The codebook is a constant of the method: the QAM-W page trains one 2D
Lloyd-Max codebook on a synthetic unit circular Gaussian and reuses it for
every matrix ("QAM-W: Joint 2D Codebook Quantization for LLM Weights ...",
Methodology (4) and Significance and Claims). Training here is the oracle's
plain Lloyd iteration (``oracle.lloyd.train_codebook``); this script calls
nothing outside ``oracle/``.
"""
from __future__ import annotations

import json
import os
import sys
import time

import numpy as np

from oracle import lloyd

OUT_DIR = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                       "vector_codebook_codec_b200", "codebooks")
DEFAULT_N = (4, 16, 128, 256, 1024, 2048)
SEED = 12345
MAX_ITER = 4000


def samples_for(N: int) -> int:
    """Training-set size: at least 1024 samples per centroid (fewer per cell
    overfits the sample set: the held-out distortion of a 256-per-cell
    N=1024 codebook came out 6.5% above its training distortion)."""
    return max(1024 * N, 1 << 18)


def main(argv):
    Ns = [int(a) for a in argv] or list(DEFAULT_N)
    os.makedirs(OUT_DIR, exist_ok=True)
    man_path = os.path.join(OUT_DIR, "manifest.json")
    manifest = json.load(open(man_path)) if os.path.exists(man_path) else {}
    for N in Ns:
        t0 = time.time()
        r = lloyd.train_codebook(N, seed=SEED + N, T=samples_for(N), max_iter=MAX_ITER)
        C32 = r["C"].astype(np.float32)
        np.save(os.path.join(OUT_DIR, f"qamw_lloyd_N{N}.npy"), C32)
        pol = r["polar"]
        manifest[str(N)] = {
            "file": f"qamw_lloyd_N{N}.npy", "N": N, "seed": SEED + N, "T": r["T"],
            "iterations": r["iters"], "converged": bool(r["converged"]),
            "train_distortion": lloyd.distortion(r["samples"], r["C"], r["idx"]),
            "polar_amp_levels": int(pol.amps.size), "polar_sectors": int(pol.P),
            "polar_train_distortion": pol.distortion(r["samples"]),
            "seconds": round(time.time() - t0, 1),
        }
        print(json.dumps(manifest[str(N)]), flush=True)
        with open(man_path, "w") as f:
            json.dump(manifest, f, indent=1, sort_keys=True)


if __name__ == "__main__":
    main(sys.argv[1:])
