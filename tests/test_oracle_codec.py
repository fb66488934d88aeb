"""Pins of the oracle's codec steps: scaling, norms, sigma, search, packing, decode.

Each test checks the oracle against something other than itself: exact
rational arithmetic, hand-derived bit patterns, closed forms, invariants of
the method ("QAM-W: Joint 2D Codebook Quantization for LLM Weights ...",
Methodology (1)-(6) and the trace identity of its bound chain), or the
distortion the pages' composite bound predicts.
"""
import math
import os
from fractions import Fraction

import numpy as np
import pytest

from oracle import codec, lloyd
from shipped import load_codebook

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden_pack():
    rows = [l.strip() for l in open(os.path.join(GOLDEN, "pack_b11.txt")) if l.strip() and not l.startswith("#")]
    idx = [int(t) for t in rows[0].split()]
    words = [int(t, 16) for t in rows[1].split()]
    return idx, words


# ---------------------------------------------------------------- packing

def test_pack_hand_derived_b11():
    idx, words = _golden_pack()
    got = codec.pack_indices(np.array([idx]), 11)
    assert [int(w) for w in got[0]] == words
    assert codec.words_per_row(12, 11) == 3


@pytest.mark.parametrize("bits", [1, 3, 7, 8, 10, 11, 13, 16])
def test_pack_roundtrip_and_layout(bits):
    rng = np.random.default_rng(bits)
    P = 77
    idx = rng.integers(0, 1 << bits, size=(5, P))
    w = codec.pack_indices(idx, bits)
    assert w.shape == (5, (P * bits + 31) // 32) and w.dtype == np.uint32
    assert np.array_equal(codec.unpack_indices(w, P, bits), idx)
    # bit t of the stream is bit (t % 32) of word t // 32, LSB-first per index
    for k in (0, 1, P - 1):
        for j in range(bits):
            t = k * bits + j
            assert ((int(w[2, t // 32]) >> (t % 32)) & 1) == ((int(idx[2, k]) >> j) & 1)
    # padding bits past the last index are zero
    tail = P * bits
    if tail % 32:
        assert int(w[0, -1]) >> (tail % 32) == 0


# ---------------------------------------------------------------- scaling / norms

def test_channel_scale_closed_forms():
    r = np.array([0.25, 1.0, 3.0, 7.5], dtype=np.float32)
    assert np.array_equal(codec.channel_scale(r, 0.0, 4), np.ones(4, np.float32))
    assert np.array_equal(codec.channel_scale(r, 1.0, 4), r)
    assert np.array_equal(codec.channel_scale(r, 0.5, 4), np.sqrt(r.astype(np.float64)).astype(np.float32))
    assert np.array_equal(codec.channel_scale(None, 0.5, 4), np.ones(4, np.float32))
    with pytest.raises(ValueError):
        codec.channel_scale(np.array([1.0, -1.0], np.float32), 0.5, 2)


def test_row_norm_is_norm_of_scaled_row():
    W = np.array([[3.0, 4.0, 0.0, 0.0], [0.0, 0.0, 0.0, 0.0]], dtype=np.float32)
    s = np.array([1.0, 1.0, 2.0, 2.0], dtype=np.float32)
    r = codec.row_norms(codec.scaled_rows(W, s))
    assert r.dtype == np.float32 and r[0] == 5.0 and r[1] == 0.0
    W[0, 2] = 1.0   # scaled by 2 -> contributes 4
    assert codec.row_norms(codec.scaled_rows(W, s))[0] == np.float32(math.sqrt(29.0))


def test_unit_rows_are_unit():
    rng = np.random.default_rng(0)
    W = rng.standard_normal((6, 64)).astype(np.float32)
    s = codec.channel_scale(np.exp(rng.standard_normal(64)).astype(np.float32), 0.5, 64)
    Wp = codec.scaled_rows(W, s)
    U = codec.unit_rows(Wp, codec.row_norms(Wp))
    assert np.allclose(np.linalg.norm(U, axis=1), 1.0, rtol=1e-7)


# ---------------------------------------------------------------- sigma

def test_sigma_rayleigh_estimator_on_gaussian_rows():
    """Gaussian rows: rotated unit-row coordinates ~ N(0, 1/K), so the Rayleigh
    mean estimator gives sigma_k ~ 1/sqrt(K) for every pair position."""
    rng = np.random.default_rng(1)
    M, K = 4000, 64
    W = rng.standard_normal((M, K)).astype(np.float32)
    sig = codec.calibrate_sigma(W, None, 0.0, 16, 3)
    assert sig.shape == (K // 2,) and sig.dtype == np.float32
    assert np.allclose(sig, 1 / math.sqrt(K), rtol=0.04)


def test_sigma_zero_column_is_one_and_scale_invariant():
    rng = np.random.default_rng(2)
    W = rng.standard_normal((50, 16)).astype(np.float32)
    sig = codec.calibrate_sigma(W, None, 0.0, 16, 0)
    sig2 = codec.calibrate_sigma(W * np.float32(8.0), None, 0.0, 16, 0)  # rows normalised away
    assert np.array_equal(sig, sig2)
    Z = np.zeros((5, 8), np.float32)
    assert np.array_equal(codec.calibrate_sigma(Z, None, 0.0, 4, 0), np.ones(4, np.float32))


def test_sigma_hand_computed_tiny():
    """One row, b = 2, s = 1: y = H2 (d*u)/sqrt(2); sigma = sqrt(2/pi)*|z| exactly."""
    W = np.array([[3.0, 4.0]], dtype=np.float32)
    sig = codec.calibrate_sigma(W, None, 0.0, 2, 0)
    # the rotation is an isometry and the row is normalised: |z| = 1
    assert sig[0] == np.float32(math.sqrt(2 / math.pi))


# ---------------------------------------------------------------- search

def test_nearest_centroid_exact_rational():
    rng = np.random.default_rng(3)
    for trial in range(30):
        N = int(rng.integers(1, 16))
        C = (rng.integers(-8, 9, size=(N, 2)) / 4.0).astype(np.float32)   # dyadic -> exact ties possible
        X = (rng.integers(-12, 13, size=(6, 2)) / 8.0).astype(np.float32)
        idx, gap = codec.nearest_centroid(X, C)
        for p in range(X.shape[0]):
            d = [(Fraction(float(X[p, 0])) - Fraction(float(c[0]))) ** 2 +
                 (Fraction(float(X[p, 1])) - Fraction(float(c[1]))) ** 2 for c in C]
            m = min(d)
            assert idx[p] == d.index(m)                     # lowest index among exact minimisers
            if d.count(m) > 1:
                assert gap[p] == 0.0


def test_nearest_centroid_gap_definition():
    C = np.array([[0, 0], [1, 0], [0, 2]], dtype=np.float32)
    idx, gap = codec.nearest_centroid(np.array([[0.25, 0.0]], np.float32), C)
    assert idx[0] == 0 and gap[0] == pytest.approx((0.5625 - 0.0625) / 0.5625)


# ---------------------------------------------------------------- whole codec

def _roundtrip_codebook_matrix():
    rng = np.random.default_rng(4)
    M, K, b = 3, 8, 4
    W = rng.standard_normal((M, K)).astype(np.float32)
    act = np.exp(rng.standard_normal(K)).astype(np.float32)
    return W, act, b


def test_roundtrip_exact_when_codebook_holds_the_points():
    """If the codebook contains every normalised pair, decode returns W up to
    the fp32 rounding of x: this ties encode and decode to the same mask,
    rotation, sigma, scaling and pair order."""
    W, act, b = _roundtrip_codebook_matrix()
    M, K = W.shape
    alpha, seed = 0.5, 99
    sig = codec.calibrate_sigma(W, act, alpha, b, seed)
    s, r, Y = codec.rotated_rows(W, act, alpha, b, seed)
    X = codec.normalised_pairs(Y, sig).reshape(-1, 2)
    C = X.copy()                                            # M*K/2 = 12 centroids
    enc = codec.encode(W, act, alpha, b, seed, sig, C, 4)
    assert np.array_equal(enc["idx"].ravel(), np.arange(C.shape[0]))
    What = codec.decode(enc["packed"], enc["r"], sig, act, alpha, K, b, seed, C, 4)
    assert np.max(np.abs(What - W) / np.max(np.abs(W), axis=1, keepdims=True)) < 1e-6


@pytest.mark.parametrize("seed", [0, 1, 2, 3, 5, 8])
def test_whole_codec_hand_computed_two_columns(seed):
    """QAM-W page, Methodology (1)-(6) on one row of two columns, worked by
    hand: W = (3, 4), s = 1, b = 2, a QPSK codebook (+-1, +-1). r = 5 and
    u = (0.6, 0.8); y = H_2 (d u) / sqrt 2 is a unit vector, so with one row
    sigma = sqrt(2/pi) |y| = sqrt(2/pi) and x = y sqrt(pi/2); the nearest
    centroid is the sign pattern of x; the decode gives
    w_hat = r d (H_2 sigma c) / sqrt 2. The sign mask d comes from the
    generator pinned to its published outputs (test_oracle_rotation)."""
    W = np.array([[3.0, 4.0]], dtype=np.float32)
    C = np.array([[1, 1], [-1, 1], [-1, -1], [1, -1]], dtype=np.float32)
    d = codec.sign_mask(seed, 2)
    y0 = (d[0] * 0.6 + d[1] * 0.8) / math.sqrt(2.0)
    y1 = (d[0] * 0.6 - d[1] * 0.8) / math.sqrt(2.0)
    sig_hand = math.sqrt(2.0 / math.pi)
    sig = codec.calibrate_sigma(W, None, 0.0, 2, seed)
    assert sig[0] == np.float32(sig_hand)
    x = np.array([y0, y1]) / float(np.float32(sig_hand))
    c_hand = (1.0 if x[0] > 0 else -1.0, 1.0 if x[1] > 0 else -1.0)
    idx_hand = {(1, 1): 0, (-1, 1): 1, (-1, -1): 2, (1, -1): 3}[c_hand]
    enc = codec.encode(W, None, 0.0, 2, seed, sig, C, 2)
    assert float(enc["r"][0]) == 5.0
    assert np.allclose(enc["x"].reshape(-1), x, rtol=1e-6, atol=0)
    assert int(enc["idx"].reshape(-1)[0]) == idx_hand
    sg = float(sig[0])
    yh0, yh1 = sg * c_hand[0], sg * c_hand[1]
    w_hand = [5.0 * d[0] * (yh0 + yh1) / math.sqrt(2.0), 5.0 * d[1] * (yh0 - yh1) / math.sqrt(2.0)]
    What = codec.decode(enc["packed"], enc["r"], sig, None, 0.0, 2, 2, seed, C, 2)
    assert np.allclose(What.reshape(-1), w_hand, rtol=1e-12, atol=1e-12)


def test_end_to_end_distortion_matches_codebook_distortion():
    """u unit, K/2 pairs with sigma^2 ~ 1/K: E|u - u_hat|^2 ~ D_B / 2."""
    rng = np.random.default_rng(5)
    M, K, b, N = 512, 1024, 128, 256
    W = rng.standard_normal((M, K)).astype(np.float32)
    C = load_codebook(N)
    sig = codec.calibrate_sigma(W, None, 0.0, b, 11)
    enc = codec.encode(W, None, 0.0, b, 11, sig, C, 8)
    What = codec.decode(enc["packed"], enc["r"], sig, None, 0.0, K, b, 11, C, 8)
    U = W / np.linalg.norm(W.astype(np.float64), axis=1, keepdims=True)
    Uh = What / enc["r"].astype(np.float64)[:, None]
    e = np.mean(np.sum((U - Uh) ** 2, axis=1))
    D_B = lloyd.distortion(lloyd.gaussian_samples(1 << 19, 5), C.astype(np.float64))
    assert 0.85 * D_B / 2 <= e <= 1.15 * D_B / 2


def test_trace_identity_and_activation_weighting():
    """||X dW^T||_F^2 = Tr(dW X^T X dW^T) (the bound chain's trace identity), and
    with alpha > 0 the codec error weighted by the activation second moment is
    lower than with alpha = 0 for the same rate (the reason for step (5))."""
    rng = np.random.default_rng(6)
    M, K, b, N = 64, 256, 64, 256
    act = np.exp(rng.standard_normal(K) * 1.0).astype(np.float32)
    W = (rng.standard_normal((M, K)) * 0.02).astype(np.float32)
    X = rng.standard_normal((1024, K)) * act[None, :].astype(np.float64)
    C = load_codebook(N)
    weighted = {}
    for alpha in (0.0, 0.5):
        sig = codec.calibrate_sigma(W, act, alpha, b, 3)
        enc = codec.encode(W, act, alpha, b, 3, sig, C, 8)
        dW = codec.decode(enc["packed"], enc["r"], sig, act, alpha, K, b, 3, C, 8) - W
        lhs = np.linalg.norm(X @ dW.T) ** 2
        rhs = np.trace(dW @ (X.T @ X) @ dW.T)
        assert abs(lhs - rhs) <= 1e-10 * abs(lhs)
        weighted[alpha] = float(np.sum((act.astype(np.float64) ** 2)[None, :] * dW ** 2))
    assert weighted[0.5] < weighted[0.0]


def test_zero_row_codes_nearest_to_origin_and_decodes_to_zero():
    C = load_codebook(16)
    W = np.zeros((2, 8), np.float32)
    W[1] = np.arange(8)
    sig = codec.calibrate_sigma(W, None, 0.0, 4, 1)
    enc = codec.encode(W, None, 0.0, 4, 1, sig, C, 4)
    assert enc["r"][0] == 0
    i0 = int(np.argmin(np.sum(C.astype(np.float64) ** 2, axis=1)))
    assert np.all(enc["idx"][0] == i0)
    What = codec.decode(enc["packed"], enc["r"], sig, None, 0.0, 8, 4, 1, C, 4)
    assert np.all(What[0] == 0.0)


@pytest.mark.parametrize("N", [2, 9, 16, 256, 2048])
def test_kd_nearest_equals_brute_force(N):
    """oracle.codec.nearest_centroid_kd gives the brute-force search's index
    and gap bit for bit: Gaussian points, far points, points on centroids,
    exact midpoints between centroid pairs (ties, lowest index wins), zeros."""
    C = load_codebook(N) if N in (16, 256, 2048) else \
        np.random.default_rng(N).standard_normal((N, 2)).astype(np.float32)
    rng = np.random.default_rng(7 + N)
    mids = ((C[rng.integers(0, N, 3000)].astype(np.float64) + C[rng.integers(0, N, 3000)]) / 2).astype(np.float32)
    X = np.concatenate([rng.standard_normal((50000, 2)).astype(np.float32),
                        (rng.standard_normal((2000, 2)) * 40).astype(np.float32),
                        C[rng.integers(0, N, 2000)], mids, np.zeros((10, 2), np.float32),
                        np.array([[np.inf, 0.0], [np.nan, 1.0]], np.float32)])
    with np.errstate(invalid="ignore"):
        i1, g1 = codec.nearest_centroid(X, C)
        i2, g2 = codec.nearest_centroid_kd(X, C, chunk=4096)
    assert np.array_equal(i1, i2)
    assert np.array_equal(g1, g2, equal_nan=True)
    # a symmetric codebook: many exact ties between mirrored centroids
    Cs = np.array([[1, 0], [-1, 0], [0, 1], [0, -1], [2, 2], [-2, -2], [2, -2], [-2, 2], [3, 0], [0, 3],
                   [-3, 0], [0, -3]], np.float32)
    Xs = np.concatenate([np.zeros((4, 2), np.float32), rng.integers(-3, 4, (4000, 2)).astype(np.float32) / 2])
    i1, g1 = codec.nearest_centroid(Xs, Cs)
    i2, g2 = codec.nearest_centroid_kd(Xs, Cs, k=4)
    assert np.array_equal(i1, i2) and np.array_equal(g1, g2)
