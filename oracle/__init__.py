"""CPU oracle for the QAM-W weight codec -- TEST INFRASTRUCTURE ONLY.

This package is a plain, slow, fp64 restatement of what the QAM-W codec
computes, written from the method description on the QAM-W page
("QAM-W: Joint 2D Codebook Quantization for LLM Weights via Hadamard Rotation
and Activation-Aware Scaling", gist.science/paper/2605.26339, Technical
Summary, section "Methodology: The QAM-W Codec"). It exists to check the CUDA
library, never to stand in for it: only ``tests/``, ``__graft_entry__.smoke()``
and the ``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import
it. It shares no code, table or helper with ``vector_codebook_codec_b200``.

Module map:
  codec      -- sign mask, Sylvester Hadamard, channel scaling, row norms,
                rotation, sigma calibration, pair normalisation, brute-force
                nearest centroid (with tie gaps), bit packing, decode.
  lloyd      -- joint 2D Lloyd-Max codebook training on unit circular Gaussian
                samples, and the polar amplitude/phase baseline code.
  make_codebooks -- script that trains and writes the shipped codebook tables.

Pins: every function is checked in ``tests/test_oracle_*.py`` against facts
fixed by mathematics or by the pages (isometry, Hadamard identities, published
SplitMix64 outputs, Lloyd closed forms, Zador/Shannon bounds, joint <= polar,
the trace identity, exact rational brute force, known bit patterns). The
whole-pipeline composition beyond those pins is "parity unpinned": the pages
print no worked numeric example.
"""
from . import codec, lloyd  # noqa: F401
