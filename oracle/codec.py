"""QAM-W codec oracle: plain fp64 numpy, one function per step of the method.

Source: "QAM-W: Joint 2D Codebook Quantization for LLM Weights via Hadamard
Rotation and Activation-Aware Scaling" (gist.science/paper/2605.26339),
Technical Summary, "Methodology: The QAM-W Codec". Its list names six steps;
citations below say "Methodology (n) <title>":
  (1) Separation of Scale and Direction   (2) Deterministic Rotation
  (3) Pairing and Calibration             (4) Joint 2D Quantization
  (5) Activation-Aware Scaling            (6) Decoding
Step (5) says the scaling is applied *before* quantization, so the execution
order used here is (5) -> (1) -> (2) -> (3) -> (4), then (6) reverses it.

Readings where the page leaves a step open (each also stated at its function):
  * s_j is r_j**alpha with proportionality constant 1, rounded once to fp32
    from an fp64 pow; W is multiplied by s before encoding and divided by s
    after decoding.
  * The stored row norm is the norm of the scaled row w' = w*s, rounded to
    fp32; u = w'/r uses that stored fp32 value.
  * The sign mask is d_j = -1 when bit 63 of the (j+1)-th SplitMix64 output
    for the seed is set (one mask per matrix, shared by all rows); the page
    names no generator.
  * Rotation per block of b columns: y = H_b (d * u) / sqrt(b), H_b the
    Sylvester (natural-order) Hadamard matrix; inverse u = d * (H_b y)/sqrt(b).
  * "unit circular Gaussian" is N(0, I_2); sigma_k is the Rayleigh mean
    estimator sqrt(2/pi) * mean_i |z_ik|, rounded to fp32; sigma_k = 0 -> 1.
  * x_k = RN32(z_k / sigma_k); nearest centroid by exact squared Euclidean
    distance, lowest index on ties.
  * Indices are packed LSB-first into little-endian uint32 words, B bits per
    index, every row starting on a fresh word.
All rounding to fp32 is round-to-nearest-even (numpy casts).
"""
from __future__ import annotations

import math

import numpy as np

GAMMA = np.uint64(0x9E3779B97F4A7C15)
SQRT_2_OVER_PI = math.sqrt(2.0 / math.pi)


def rn32(x) -> np.ndarray:
    """Round fp64 values to the nearest fp32 (ties to even)."""
    return np.asarray(x, dtype=np.float64).astype(np.float32)


# ---------------------------------------------------------------------------
# sign mask and Hadamard matrix -- Methodology (2) Deterministic Rotation
# ---------------------------------------------------------------------------

def splitmix64(seed: int, n: int) -> np.ndarray:
    """First ``n`` outputs of SplitMix64 seeded with ``seed`` (uint64 array).

    SplitMix64 (Steele, Lea & Flood, "Fast splittable pseudorandom number
    generators", OOPSLA 2014): the j-th output (j = 1, 2, ...) is the mix
    function applied to the state seed + j*0x9E3779B97F4A7C15 (mod 2^64):
    z ^= z>>30; z *= 0xBF58476D1CE4E5B9; z ^= z>>27; z *= 0x94D049BB133111EB;
    z ^= z>>31.
    """
    j = np.arange(1, n + 1, dtype=np.uint64)
    with np.errstate(over="ignore"):
        z = np.uint64(seed) + j * GAMMA
        z = (z ^ (z >> np.uint64(30))) * np.uint64(0xBF58476D1CE4E5B9)
        z = (z ^ (z >> np.uint64(27))) * np.uint64(0x94D049BB133111EB)
        z = z ^ (z >> np.uint64(31))
    return z


def sign_mask(seed: int, K: int) -> np.ndarray:
    """d_j in {+1, -1} (float64 [K]); -1 where bit 63 of output j+1 is set."""
    top = splitmix64(seed, K) >> np.uint64(63)
    return np.where(top == 1, -1.0, 1.0)


def hadamard(b: int) -> np.ndarray:
    """Sylvester Hadamard matrix H_b (float64 [b, b]), b a power of two.

    Built by the doubling rule H_1 = [1], H_2n = [[H_n, H_n], [H_n, -H_n]].
    """
    if b < 1 or b & (b - 1):
        raise ValueError("block size must be a power of two")
    H = np.ones((1, 1))
    while H.shape[0] < b:
        H = np.block([[H, H], [H, -H]])
    return H


def rotate_fwd(U: np.ndarray, d: np.ndarray, b: int) -> np.ndarray:
    """y = R_fwd u per row: each block of b columns -> H_b (d * u) / sqrt(b).

    Methodology (2): the sign-masked block-Hadamard rotation, an isometry in
    exact arithmetic. Naive O(b^2) matrix product per block.
    """
    M, K = U.shape
    H = hadamard(b)
    V = (U * d[None, :]).reshape(M, K // b, b)
    return (V @ H.T).reshape(M, K) / math.sqrt(b)


def rotate_inv(Y: np.ndarray, d: np.ndarray, b: int) -> np.ndarray:
    """u = R_inv y per row: each block -> d * (H_b y) / sqrt(b) (H_b H_b = b I)."""
    M, K = Y.shape
    H = hadamard(b)
    V = (Y.reshape(M, K // b, b) @ H.T).reshape(M, K) / math.sqrt(b)
    return V * d[None, :]


# ---------------------------------------------------------------------------
# scaling and norms -- Methodology (5) and (1)
# ---------------------------------------------------------------------------

def channel_scale(act_rms, alpha: float, K: int) -> np.ndarray:
    """s_j = RN32(r_j ** alpha) with the power taken in fp64 (float32 [K]).

    Methodology (5) Activation-Aware Scaling: s_j proportional to r_j^alpha,
    r_j the RMS of input channel j; the constant is taken as 1 (it cancels
    between encode and decode). ``act_rms=None`` means s = 1.
    """
    if act_rms is None:
        return np.ones(K, dtype=np.float32)
    r = np.asarray(act_rms, dtype=np.float32).astype(np.float64)
    if r.shape != (K,) or not np.all(np.isfinite(r)) or np.any(r <= 0):
        raise ValueError("act_rms must be K finite positive values")
    return rn32(np.power(r, float(np.float32(alpha))))


def scaled_rows(W: np.ndarray, s: np.ndarray) -> np.ndarray:
    """w'_ij = w_ij * s_j, exact in fp64 (both factors are fp32 values)."""
    return np.asarray(W, dtype=np.float64) * np.asarray(s, dtype=np.float64)[None, :]


def row_norms(Wp: np.ndarray) -> np.ndarray:
    """r_i = RN32(||w'_i||_2) -- Methodology (1), recorded as metadata (float32 [M])."""
    return rn32(np.sqrt(np.sum(Wp * Wp, axis=1)))


def unit_rows(Wp: np.ndarray, r: np.ndarray) -> np.ndarray:
    """u_i = w'_i / r_i using the stored fp32 r_i; a zero row stays zero."""
    r64 = np.asarray(r, dtype=np.float64)
    safe = np.where(r64 > 0, r64, 1.0)
    U = Wp / safe[:, None]
    U[r64 == 0] = 0.0
    return U


def rotated_rows(W, act_rms, alpha, block, seed):
    """Steps (5), (1), (2): returns (s, r, Y) with Y the rotated unit rows (fp64)."""
    W = np.asarray(W)
    M, K = W.shape
    s = channel_scale(act_rms, alpha, K)
    Wp = scaled_rows(W, s)
    r = row_norms(Wp)
    Y = rotate_fwd(unit_rows(Wp, r), sign_mask(seed, K), block)
    return s, r, Y


# ---------------------------------------------------------------------------
# pairing and calibration -- Methodology (3)
# ---------------------------------------------------------------------------

def pairs(Y: np.ndarray) -> np.ndarray:
    """z_k = (y_2k, y_2k+1) for k = 0..K/2-1 -> array [M, K/2, 2]."""
    M, K = Y.shape
    return Y.reshape(M, K // 2, 2)


def calibrate_sigma(W, act_rms, alpha, block, seed) -> np.ndarray:
    """sigma_k = RN32(sqrt(2/pi) * mean_i |z_ik|) (float32 [K/2]).

    Methodology (3): each pair is scaled by sigma_k estimated from the mean
    amplitude of the pairs under a circular Gaussian model. For z ~ N(0, s^2 I_2)
    the amplitude is Rayleigh with mean s*sqrt(pi/2), hence the sqrt(2/pi)
    factor, which maps the pairs onto the unit circular Gaussian of step (4).
    A pair position that is zero in every row gets sigma = 1.
    """
    _, _, Y = rotated_rows(W, act_rms, alpha, block, seed)
    return sigma_from_rotated(Y)


def sigma_from_rotated(Y: np.ndarray) -> np.ndarray:
    """The estimate of :func:`calibrate_sigma` from the rotated unit rows Y
    (fp64 [M, K]): sigma_k = RN32(sqrt(2/pi) * mean_i |z_ik|), 0 -> 1."""
    Z = pairs(Y)
    amp = np.sqrt(Z[..., 0] ** 2 + Z[..., 1] ** 2)
    sig = rn32(SQRT_2_OVER_PI * (np.sum(amp, axis=0) / Z.shape[0]))
    sig[sig == 0] = np.float32(1.0)
    return sig


def normalised_pairs(Y: np.ndarray, sigma: np.ndarray) -> np.ndarray:
    """x_k = RN32(z_k / sigma_k) using the stored fp32 sigma (float32 [M, K/2, 2])."""
    Z = pairs(Y)
    return rn32(Z / np.asarray(sigma, dtype=np.float64)[None, :, None])


# ---------------------------------------------------------------------------
# joint 2D quantization -- Methodology (4)
# ---------------------------------------------------------------------------

def nearest_centroid(X: np.ndarray, C: np.ndarray, chunk: int = 1 << 14):
    """Brute-force nearest centroid over all N centroids.

    Methodology (4): each normalised pair maps to the nearest centroid of one
    2D codebook. Distances are squared Euclidean, evaluated in fp64 on the
    fp32 inputs; ties go to the lowest index (numpy argmin). Returns
    (idx int64 [...], gap float64 [...]) where gap = (d2 - d1) / d2 is the
    relative gap between the best and second-best distances (0 for an exact
    tie; 1 when the pair sits on its centroid; inf-free).
    """
    X = np.asarray(X, dtype=np.float32)
    C = np.asarray(C, dtype=np.float32).astype(np.float64)
    shape = X.shape[:-1]
    flat = X.reshape(-1, 2).astype(np.float64)
    idx = np.empty(flat.shape[0], dtype=np.int64)
    gap = np.empty(flat.shape[0], dtype=np.float64)
    for a in range(0, flat.shape[0], chunk):
        x = flat[a:a + chunk]
        d = (x[:, 0:1] - C[None, :, 0]) ** 2 + (x[:, 1:2] - C[None, :, 1]) ** 2
        i = np.argmin(d, axis=1)
        rows = np.arange(x.shape[0])
        d1 = d[rows, i]
        if C.shape[0] > 1:
            d[rows, i] = np.inf
            d2 = np.min(d, axis=1)
            with np.errstate(invalid="ignore", divide="ignore"):
                g = np.where(d2 > 0, (d2 - d1) / d2, 0.0)
        else:
            g = np.ones_like(d1)
        idx[a:a + chunk] = i
        gap[a:a + chunk] = g
    return idx.reshape(shape), gap.reshape(shape)


def nearest_centroid_kd(X: np.ndarray, C: np.ndarray, k: int = 4, chunk: int = 1 << 18):
    """:func:`nearest_centroid` for large inputs: the same (idx, gap), bit for bit.

    A k-d tree over the centroids (``scipy.spatial.cKDTree``, an exact
    Euclidean k-nearest query used as a library primitive) proposes each
    point's k nearest centroids. Their squared distances are recomputed with
    the fp64 direct-difference formula of :func:`nearest_centroid`; the least
    one (lowest index among equal distances) and the second least give idx and
    gap. A centroid the tree did not propose is at least as far as the k-th
    proposed one, so the answer is exact whenever the second-least recomputed
    distance lies clearly (1e-9 relative) below the k-th; any other point, and
    any non-finite one, is resolved by :func:`nearest_centroid`. Chunks of
    points run on a thread pool (the tree query and numpy release the GIL).
    """
    import os
    from concurrent.futures import ThreadPoolExecutor
    from scipy.spatial import cKDTree
    X = np.asarray(X, dtype=np.float32)
    C64 = np.asarray(C, dtype=np.float32).astype(np.float64)
    N = C64.shape[0]
    if N <= k + 1:
        return nearest_centroid(X, C)
    shape = X.shape[:-1]
    flat = X.reshape(-1, 2)
    n = flat.shape[0]
    idx = np.empty(n, dtype=np.int64)
    gap = np.empty(n, dtype=np.float64)
    tree = cKDTree(C64)

    def run(a):
        x = flat[a:a + chunk].astype(np.float64)
        finite = np.all(np.isfinite(x), axis=1)
        _, cand = tree.query(np.where(finite[:, None], x, 0.0), k=k)
        d = (x[:, 0:1] - C64[cand, 0]) ** 2 + (x[:, 1:2] - C64[cand, 1]) ** 2
        d1 = d.min(axis=1)
        first = np.where(d == d1[:, None], cand, N).min(axis=1)          # lowest index at the least distance
        d_rest = np.where(cand == first[:, None], np.inf, d)
        d2 = d_rest.min(axis=1)
        dk = d.max(axis=1)
        with np.errstate(invalid="ignore", divide="ignore"):
            g = np.where(d2 > 0, (d2 - d1) / d2, 0.0)
        ok = finite & (d2 < dk * (1.0 - 1e-9))
        if not np.all(ok):
            bad = np.nonzero(~ok)[0]
            bi, bg = nearest_centroid(flat[a + bad], C)
            first[bad] = bi
            g[bad] = bg
        idx[a:a + x.shape[0]] = first
        gap[a:a + x.shape[0]] = g

    with ThreadPoolExecutor(max_workers=os.cpu_count() or 1) as ex:
        list(ex.map(run, range(0, n, chunk)))
    return idx.reshape(shape), gap.reshape(shape)


# ---------------------------------------------------------------------------
# bit packing (the packed index stream that decode "unpacks")
# ---------------------------------------------------------------------------

def words_per_row(K: int, bits: int) -> int:
    return ((K // 2) * bits + 31) // 32


def pack_indices(idx: np.ndarray, bits: int) -> np.ndarray:
    """Pack [M, P] indices, ``bits`` each, LSB-first into uint32 [M, W].

    Bit t of a row's stream is bit (t mod 32) of word t // 32; index k occupies
    stream bits k*bits .. k*bits+bits-1, least significant bit first.
    """
    idx = np.asarray(idx, dtype=np.int64)
    M, P = idx.shape
    if np.any(idx < 0) or np.any(idx >= (1 << bits)):
        raise ValueError("index out of range for the bit width")
    W = (P * bits + 31) // 32
    bitarr = ((idx[:, :, None] >> np.arange(bits)[None, None, :]) & 1).reshape(M, P * bits)
    padded = np.zeros((M, W * 32), dtype=np.uint64)
    padded[:, :P * bits] = bitarr
    words = (padded.reshape(M, W, 32) << np.arange(32, dtype=np.uint64)).sum(axis=2)
    return words.astype(np.uint32)


def unpack_indices(words: np.ndarray, P: int, bits: int) -> np.ndarray:
    """Inverse of :func:`pack_indices`: uint32 [M, W] -> int64 [M, P]."""
    words = np.asarray(words, dtype=np.uint32).astype(np.uint64)
    M, W = words.shape
    bitarr = ((words[:, :, None] >> np.arange(32, dtype=np.uint64)) & np.uint64(1)).reshape(M, W * 32)
    b = bitarr[:, :P * bits].reshape(M, P, bits).astype(np.int64)
    return (b << np.arange(bits)[None, None, :]).sum(axis=2)


# ---------------------------------------------------------------------------
# whole codec
# ---------------------------------------------------------------------------

def encode(W, act_rms, alpha, block, seed, sigma, C, bits):
    """Encode W [M, K] -> dict(packed, r, idx, gap, x, s).

    Steps (5) scale, (1) norm + normalise, (2) rotate, (3) pair and divide by
    the given sigma, (4) nearest centroid, then pack.
    """
    C = np.asarray(C, dtype=np.float32)
    if C.shape[0] > (1 << bits):
        raise ValueError("codebook larger than 2**bits")
    s, r, Y = rotated_rows(W, act_rms, alpha, block, seed)
    X = normalised_pairs(Y, sigma)
    idx, gap = nearest_centroid(X, C)
    return {"packed": pack_indices(idx, bits), "r": r, "idx": idx, "gap": gap, "x": X, "s": s}


def decode(packed, r, sigma, act_rms, alpha, K, block, seed, C, bits) -> np.ndarray:
    """Methodology (6) Decoding, in fp64 -> W_hat [M, K] (float64).

    Unpack indices, look up centroids, rescale by sigma_k, apply the inverse
    rotation, multiply by the stored row norm, then undo the channel scaling
    (divide by s_j).
    """
    idx = unpack_indices(packed, K // 2, bits)
    return decode_indices(idx, r, sigma, act_rms, alpha, K, block, seed, C)


def decode_indices(idx, r, sigma, act_rms, alpha, K, block, seed, C) -> np.ndarray:
    """Decode from unpacked indices (same arithmetic as :func:`decode`)."""
    s = channel_scale(act_rms, alpha, K)
    return decode_with_scale(idx, r, sigma, s, K, block, seed, C)


def decode_with_scale(idx, r, sigma, s, K, block, seed, C) -> np.ndarray:
    """Methodology (6) given the stored channel scale s_j (fp32 [K], or None = 1).

    w_hat = r * R_inv(sigma (.) C[idx]) / s, in fp64 (float64 [M, K]).
    """
    C = np.asarray(C, dtype=np.float32).astype(np.float64)
    idx = np.asarray(idx, dtype=np.int64)
    if np.any(idx < 0) or np.any(idx >= C.shape[0]):
        raise ValueError("index beyond codebook")
    M = idx.shape[0]
    Yh = (C[idx] * np.asarray(sigma, dtype=np.float32).astype(np.float64)[None, :, None]).reshape(M, K)
    Uh = rotate_inv(Yh, sign_mask(seed, K), block)
    s64 = np.ones(K) if s is None else np.asarray(s, dtype=np.float32).astype(np.float64)
    return Uh * np.asarray(r, dtype=np.float32).astype(np.float64)[:, None] / s64[None, :]


def encode_polar(W, act_rms, alpha, block, seed, sigma, amps, P, bits):
    """The polar baseline codec of "Joint 2D vs. Polar" (QAM-W page, Results):
    steps (5), (1), (2), (3) as in :func:`encode`, then each normalised pair is
    quantized by amplitude (nearest of the levels ``amps``) and phase (P
    uniform sectors) independently; the index is a*P + p (the order of
    ``PolarCode.points()``). Returns dict(packed, r, idx, margin, x, s)."""
    from oracle.lloyd import PolarCode
    code = PolarCode(np.asarray(amps, dtype=np.float64), P)
    s, r, Y = rotated_rows(W, act_rms, alpha, block, seed)
    X = normalised_pairs(Y, sigma)
    M, Pp = X.shape[0], X.shape[1]
    idx, margin = code.indices(X.reshape(-1, 2).astype(np.float64))
    idx = idx.reshape(M, Pp)
    return {"packed": pack_indices(idx, bits), "r": r, "idx": idx, "margin": margin.reshape(M, Pp), "x": X, "s": s}
