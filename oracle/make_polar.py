"""Write the polar baseline codes (amplitude levels and reconstruction points).

Usage: python -m oracle.make_polar [N ...]

For every shipped codebook size N, the polar code of "Joint 2D vs. Polar"
("QAM-W: Joint 2D Codebook Quantization for LLM Weights ...", Results) is the
best power-of-two split N = A * P found when the joint codebook was trained
(``manifest.json``: ``polar_amp_levels``, ``polar_sectors``), with the A
amplitude levels of the 1D Lloyd-Max quantizer of the same training samples'
radii. Writes ``qamw_polar_N{N}_amps.npy`` (float64 [A], ascending) and
``qamw_polar_N{N}_points.npy`` (float32 [N, 2], ``PolarCode.points()`` order)
beside the codebooks and adds both to the manifest. Calls nothing outside
``oracle/``.
"""
from __future__ import annotations

import json
import os
import sys

import numpy as np

from oracle import lloyd
from oracle.make_codebooks import OUT_DIR, SEED, samples_for


def main(argv):
    man_path = os.path.join(OUT_DIR, "manifest.json")
    manifest = json.load(open(man_path))
    Ns = [int(a) for a in argv] or sorted(int(k) for k in manifest)
    for N in Ns:
        e = manifest[str(N)]
        A, P = int(e["polar_amp_levels"]), int(e["polar_sectors"])
        x = lloyd.gaussian_samples(samples_for(N), SEED + N)
        amps = lloyd.lloyd_1d(np.hypot(x[:, 0], x[:, 1]), A)
        code = lloyd.PolarCode(amps, P)
        np.save(os.path.join(OUT_DIR, f"qamw_polar_N{N}_amps.npy"), code.amps.astype(np.float64))
        np.save(os.path.join(OUT_DIR, f"qamw_polar_N{N}_points.npy"), code.points().astype(np.float32))
        e["polar_amps_file"] = f"qamw_polar_N{N}_amps.npy"
        e["polar_points_file"] = f"qamw_polar_N{N}_points.npy"
        e["polar_train_distortion"] = code.distortion(x)
        e.pop("polar_train_distortion_check", None)
        print(N, A, P, e["polar_train_distortion"], flush=True)
    with open(man_path, "w") as f:
        json.dump(manifest, f, indent=1, sort_keys=True)


if __name__ == "__main__":
    main(sys.argv[1:])
