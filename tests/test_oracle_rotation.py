"""Pins of the oracle's sign mask and sign-masked block Hadamard rotation.

QAM-W page, Methodology (2) Deterministic Rotation: the rotation is an exact
isometry in real arithmetic. The mask generator is pinned to published
SplitMix64 outputs; the Hadamard matrix to an independent definition.
"""
import math
import os

import numpy as np
import pytest

from oracle import codec

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden_splitmix():
    vals = []
    for line in open(os.path.join(GOLDEN, "splitmix64_seed0.txt")):
        line = line.strip()
        if line and not line.startswith("#"):
            vals.append(int(line, 16))
    return vals


def test_splitmix64_published_outputs():
    ref = _golden_splitmix()
    got = [int(v) for v in codec.splitmix64(0, len(ref))]
    assert got == ref


def test_sign_mask_from_published_outputs():
    ref = _golden_splitmix()
    d = codec.sign_mask(0, len(ref))
    assert list(d) == [-1.0 if (v >> 63) else 1.0 for v in ref]


def test_sign_mask_is_balanced_and_seed_dependent():
    d0 = codec.sign_mask(0, 1 << 16)
    d1 = codec.sign_mask(1, 1 << 16)
    assert abs(d0.mean()) < 0.02 and abs(d1.mean()) < 0.02
    assert np.mean(d0 != d1) > 0.45


def _hadamard_popcount(b):
    p = np.arange(b)
    return np.array([[(-1.0) ** bin(int(i) & int(j)).count("1") for j in p] for i in p])


@pytest.mark.parametrize("b", [1, 2, 4, 8, 16, 64, 128])
def test_sylvester_matches_popcount_definition(b):
    assert np.array_equal(codec.hadamard(b), _hadamard_popcount(b))


@pytest.mark.parametrize("b", [2, 4, 32, 256, 1024])
def test_hadamard_orthogonal(b):
    H = codec.hadamard(b)
    assert np.array_equal(H @ H.T, b * np.eye(b))
    assert np.all(H[0] == 1) and np.all(H[:, 0] == 1)


def test_block_size_two_is_h2():
    U = np.array([[0.3, -1.1, 2.0, 0.5]])
    d = codec.sign_mask(7, 4)
    Y = codec.rotate_fwd(U, d, 2)
    v = U[0] * d
    ref = np.array([v[0] + v[1], v[0] - v[1], v[2] + v[3], v[2] - v[3]]) / math.sqrt(2)
    assert np.allclose(Y[0], ref, rtol=0, atol=1e-15)


@pytest.mark.parametrize("b", [2, 4, 8, 16, 32, 64, 128, 256])
def test_rotation_isometry_and_inverse(b):
    rng = np.random.default_rng(b)
    K = 4 * b if b <= 64 else 2 * b
    U = rng.standard_normal((9, K))
    d = codec.sign_mask(123 + b, K)
    Y = codec.rotate_fwd(U, d, b)
    assert np.allclose(np.linalg.norm(Y, axis=1), np.linalg.norm(U, axis=1), rtol=1e-13)
    U2 = codec.rotate_inv(Y, d, b)
    assert np.max(np.abs(U2 - U)) < 1e-12
    # the explicit operator, built column by column, is orthogonal to 1e-6 in fp32
    E = np.eye(K)
    R = codec.rotate_fwd(E, d, b).T           # R[:, j] = R e_j
    Ri = codec.rotate_inv(E, d, b).T
    assert np.max(np.abs(Ri.astype(np.float32) @ R.astype(np.float32) - np.eye(K))) <= 1e-6
    assert np.max(np.abs(Ri @ R - np.eye(K))) < 1e-13


def test_rotation_is_block_local():
    b, K = 8, 32
    d = codec.sign_mask(5, K)
    e = np.zeros((1, K))
    e[0, 11] = 1.0                       # column 11 lives in block 1 (columns 8..15)
    Y = codec.rotate_fwd(e, d, b)[0]
    nz = np.nonzero(Y)[0]
    assert nz.min() == 8 and nz.max() == 15
    assert np.allclose(np.abs(Y[8:16]), 1 / math.sqrt(b))
