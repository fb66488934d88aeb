"""Joint 2D Lloyd-Max codebook and the polar amplitude/phase baseline (oracle).

Source: "QAM-W: Joint 2D Codebook Quantization for LLM Weights via Hadamard
Rotation and Activation-Aware Scaling" (gist.science/paper/2605.26339):
  * Methodology (4) Joint 2D Quantization -- one 2D Lloyd-Max codebook trained
    on the unit circular Gaussian, instead of quantizing amplitude and phase
    independently (polar coding);
  * Significance and Claims -- the codebook is trained on a synthetic unit
    circular Gaussian, not per checkpoint;
  * Results, "Joint 2D vs. Polar" -- QAM-W-polar is the baseline at equal rate.

Readings (the page gives no sample count, start point, stopping rule or
empty-cell rule, and does not define the polar code beyond its name):
  * samples are N(0, I_2) draws from a seeded PCG64 generator;
  * Lloyd starts from the reconstruction points of the best polar code of the
    same size and alternates nearest assignment / centroid update until no
    assignment changes or ``max_iter`` is reached; an empty cell keeps its
    centroid;
  * the polar code with N = A*P points quantizes the amplitude with a 1D
    Lloyd-Max quantizer of A levels (trained on the sample amplitudes) and the
    phase uniformly into P sectors centred at 2*pi*(p+1/2)/P, independently;
    among the power-of-two splits A*P = N the one with least 2D MSE is kept.

The assignment step uses ``scipy.spatial.cKDTree`` (an exact Euclidean
nearest-neighbour query) as a library primitive; tests re-check assignments
against brute force.
"""
from __future__ import annotations

import math

import numpy as np
from scipy.spatial import cKDTree


def gaussian_samples(T: int, seed: int) -> np.ndarray:
    """T samples of the unit circular Gaussian N(0, I_2), float64 [T, 2]."""
    g = np.random.Generator(np.random.PCG64(int(seed)))
    return g.standard_normal((T, 2))


def assign(samples: np.ndarray, C: np.ndarray) -> np.ndarray:
    """Index of the nearest centroid for every sample (Euclidean)."""
    _, i = cKDTree(np.asarray(C, dtype=np.float64)).query(samples, k=1, workers=-1)
    return i.astype(np.int64)


def distortion(samples: np.ndarray, C: np.ndarray, idx: np.ndarray | None = None) -> float:
    """Mean squared error per 2D sample, E|x - C[idx(x)]|^2 (nearest if idx is None)."""
    C = np.asarray(C, dtype=np.float64)
    if idx is None:
        idx = assign(samples, C)
    e = samples - C[idx]
    return float(np.mean(np.sum(e * e, axis=1)))


def centroid_update(samples, idx, C):
    """Each centroid moves to the mean of its cell; empty cells keep their centroid."""
    N = C.shape[0]
    cnt = np.bincount(idx, minlength=N).astype(np.float64)
    sx = np.bincount(idx, weights=samples[:, 0], minlength=N)
    sy = np.bincount(idx, weights=samples[:, 1], minlength=N)
    out = C.copy()
    nz = cnt > 0
    out[nz, 0] = sx[nz] / cnt[nz]
    out[nz, 1] = sy[nz] / cnt[nz]
    return out


def lloyd(samples: np.ndarray, init: np.ndarray, max_iter: int = 500):
    """Lloyd iterations from ``init``. Returns (C, idx, iterations, converged).

    On return ``idx`` is the nearest assignment to the *returned* C when
    converged (no assignment changed, so C is the mean of every cell).
    """
    C = np.asarray(init, dtype=np.float64).copy()
    idx = assign(samples, C)
    for it in range(1, max_iter + 1):
        C = centroid_update(samples, idx, C)
        new = assign(samples, C)
        if np.array_equal(new, idx):
            return C, new, it, True
        idx = new
    return C, idx, max_iter, False


# ---------------------------------------------------------------------------
# polar baseline
# ---------------------------------------------------------------------------

def lloyd_1d(values: np.ndarray, levels: int, max_iter: int = 1_000_000) -> np.ndarray:
    """1D Lloyd-Max quantizer levels for ``values`` (ascending).

    Lloyd-Max conditions: every level is the mean of its cell, and the cells
    meet at the midpoints between consecutive levels (a value on a midpoint
    belongs to the lower cell). Starting from the ``levels`` quantiles of the
    values, the two conditions are applied in turn until the partition of the
    (sorted) values no longer changes; the levels are then the exact means of
    their cells. A cell that empties keeps its level. The values are sorted
    once, so each cell is a contiguous range and its sum a difference of
    prefix sums.
    """
    v = np.sort(np.asarray(values, dtype=np.float64))
    S = np.concatenate([[0.0], np.cumsum(v)])
    q = np.quantile(v, (np.arange(levels) + 0.5) / levels)
    bounds = None
    for _ in range(max_iter):
        edges = (q[1:] + q[:-1]) / 2
        # cell i holds the values in (edges[i-1], edges[i]]
        b = np.concatenate([[0], np.searchsorted(v, edges, side="right"), [v.size]])
        if bounds is not None and np.array_equal(b, bounds):
            break
        bounds = b
        cnt = b[1:] - b[:-1]
        s = S[b[1:]] - S[b[:-1]]
        q = np.where(cnt > 0, s / np.maximum(cnt, 1), q)
    return np.sort(q)


class PolarCode:
    """Independent amplitude (A Lloyd levels) x phase (P uniform sectors) code."""

    def __init__(self, amps: np.ndarray, P: int):
        self.amps = np.sort(np.asarray(amps, dtype=np.float64))
        self.P = int(P)

    @property
    def N(self) -> int:
        return self.amps.size * self.P

    def points(self) -> np.ndarray:
        """All A*P reconstruction points a * exp(i theta_p), amplitude-major order."""
        th = 2 * math.pi * (np.arange(self.P) + 0.5) / self.P
        a = self.amps[:, None]
        return np.stack([(a * np.cos(th)[None, :]).ravel(), (a * np.sin(th)[None, :]).ravel()], axis=1)

    def quantize(self, x: np.ndarray) -> np.ndarray:
        """Reconstruction of each sample: nearest amplitude level and nearest sector centre."""
        rad = np.hypot(x[:, 0], x[:, 1])
        ang = np.mod(np.arctan2(x[:, 1], x[:, 0]), 2 * math.pi)
        if self.amps.size > 1:
            edges = (self.amps[1:] + self.amps[:-1]) / 2
            ai = np.searchsorted(edges, rad)
        else:
            ai = np.zeros(rad.shape, dtype=np.int64)
        pi_ = np.floor(ang / (2 * math.pi / self.P)).astype(np.int64) % self.P
        th = 2 * math.pi * (pi_ + 0.5) / self.P
        a = self.amps[ai]
        return np.stack([a * np.cos(th), a * np.sin(th)], axis=1)

    def distortion(self, x: np.ndarray) -> float:
        e = x - self.quantize(x)
        return float(np.mean(np.sum(e * e, axis=1)))

    def indices(self, x: np.ndarray):
        """Index a * P + p of each sample's reconstruction point in ``points()``
        order (a: nearest amplitude level, p: phase sector), and the sample's
        margin: its distance to the nearest decision boundary, relative for the
        amplitude (|rad - edge| / rad) and in sector widths for the phase."""
        x = np.asarray(x, dtype=np.float64)
        rad = np.hypot(x[:, 0], x[:, 1])
        ang = np.mod(np.arctan2(x[:, 1], x[:, 0]), 2 * math.pi)
        w = 2 * math.pi / self.P
        if self.amps.size > 1:
            edges = (self.amps[1:] + self.amps[:-1]) / 2
            ai = np.searchsorted(edges, rad)
            lo = np.abs(rad - edges[np.maximum(ai - 1, 0)])       # the edges on either side of rad
            hi = np.abs(edges[np.minimum(ai, edges.size - 1)] - rad)
            near = np.minimum(lo, hi) / np.maximum(rad, 1e-300)
        else:
            ai = np.zeros(rad.shape, dtype=np.int64)
            near = np.full(rad.shape, np.inf)
        f = ang / w
        pi_ = np.floor(f).astype(np.int64) % self.P
        sec = np.abs(f - np.round(f)) if self.P > 1 else np.full(rad.shape, np.inf)
        return ai * self.P + pi_, np.minimum(near, sec)


def best_polar(samples: np.ndarray, N: int) -> PolarCode:
    """Best power-of-two split N = A*P (least MSE on ``samples``)."""
    if N & (N - 1):
        raise ValueError("polar split needs N a power of two")
    rad = np.hypot(samples[:, 0], samples[:, 1])
    best, best_d = None, math.inf
    A = 1
    while A <= N:
        P = N // A
        code = PolarCode(lloyd_1d(rad, A), P)
        d = code.distortion(samples)
        if d < best_d:
            best, best_d = code, d
        A *= 2
    return best


def train_codebook(N: int, seed: int = 12345, T: int | None = None, max_iter: int = 500):
    """Train the joint 2D codebook of N centroids. Returns dict with C (fp64), info."""
    if T is None:
        T = max(256 * N, 1 << 18)
    x = gaussian_samples(T, seed)
    if N & (N - 1) == 0:
        polar = best_polar(x, N)
        init = polar.points()
    else:
        polar = None
        init = x[:N].copy()
    C, idx, iters, conv = lloyd(x, init, max_iter=max_iter)
    return {"C": C, "idx": idx, "iters": iters, "converged": conv, "T": T, "seed": seed,
            "polar": polar, "samples": x}
