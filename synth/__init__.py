"""Seeded synthetic inputs shared by the oracle side and the CUDA side.

This module only draws random numbers (weights, activation RMS vectors,
random index streams) with the shapes and distributions of the codec's
workloads. It holds none of the codec's arithmetic: no scaling, no rotation,
no norms, no codebook, no packing. Both the oracle (``oracle/``) and the
CUDA path read identical bytes from here.

Workload shapes stand in for the layers of the models that the QAM-W page
evaluates (TinyLlama-1.1B, Llama/Mistral-7B and a 13B model; "QAM-W: Joint 2D
Codebook Quantization for LLM Weights ...", Technical Summary, Results). No
checkpoint is used: weights are Gaussian or Student-t draws, optionally with a
few outlier columns, and activation RMS values are lognormal.

Every array is generated in float32 from ``numpy.random.Generator(PCG64(seed))``;
bf16 matrices are the float32 draws rounded to bf16 with round-to-nearest-even
(``torch`` CPU conversion). ``float32`` copies of bf16 matrices hold exactly the
bf16 values, so the oracle sees the same numbers as the GPU.
"""
from __future__ import annotations

from dataclasses import dataclass, field
import math

import numpy as np

__all__ = [
    "MatrixSpec", "Workload", "make_matrix", "make_act_rms", "make_indices",
    "make_row_norms", "make_sigma", "make_activations", "to_bf16", "tiny", "llama7b_attn", "mlp_runs",
    "stack_1p1b", "decode_sweep_13b", "rate_variant", "gaussian_points", "WORKLOADS",
]


def _rng(seed: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(int(seed)))


def to_bf16(w32: np.ndarray):
    """Round a float32 array to bf16 (RNE). Returns (torch.bfloat16 tensor, float32 copy)."""
    import torch
    t = torch.from_numpy(np.ascontiguousarray(w32, dtype=np.float32)).to(torch.bfloat16)
    return t, t.to(torch.float32).numpy()


@dataclass(frozen=True)
class MatrixSpec:
    """One synthetic weight matrix W [M x K] and its codec parameters."""
    name: str
    M: int
    K: int
    dtype: str              # "f32" or "bf16"
    dist: str               # "normal" or "t4"
    std: float              # target standard deviation of the entries
    outlier_frac: float     # fraction of columns scaled by outlier_scale
    outlier_scale: float
    act_sigma: float        # act RMS ~ lognormal(0, act_sigma)
    alpha: float
    block: int
    N: int                  # centroids
    bits: int               # bits per pair index
    seed: int
    act_seed: int | None = None   # act vector seed (layers share one per distinct input)


def make_matrix(spec: MatrixSpec) -> np.ndarray:
    """float32 draws [M, K] for ``spec`` (not yet rounded to bf16)."""
    g = _rng(spec.seed)
    M, K = spec.M, spec.K
    if spec.dist == "normal":
        w = g.standard_normal((M, K), dtype=np.float32) * np.float32(spec.std)
    elif spec.dist == "t4":
        # Student-t with 4 degrees of freedom: Z / sqrt(chi2_4 / 4); variance 2.
        z = g.standard_normal((M, K), dtype=np.float32)
        chi = np.zeros((M, K), dtype=np.float32)
        for _ in range(4):
            n = g.standard_normal((M, K), dtype=np.float32)
            chi += n * n
        w = z / np.sqrt(chi / np.float32(4.0)) * np.float32(spec.std / math.sqrt(2.0))
    else:
        raise ValueError(spec.dist)
    n_out = int(round(spec.outlier_frac * K))
    if n_out > 0:
        cols = g.choice(K, size=n_out, replace=False)
        w[:, cols] *= np.float32(spec.outlier_scale)
    return w.astype(np.float32)


def make_act_rms(K: int, sigma: float, seed: int) -> np.ndarray:
    """Per-input-channel activation RMS, lognormal(0, sigma), float32 [K]."""
    g = _rng(seed + 7919)
    return np.exp(g.standard_normal(K) * sigma).astype(np.float32)


def make_indices(M: int, P: int, N: int, seed: int) -> np.ndarray:
    """Uniform random centroid indices in [0, N), int64 [M, P] (decode inputs)."""
    return _rng(seed).integers(0, N, size=(M, P), dtype=np.int64)


def make_row_norms(M: int, seed: int) -> np.ndarray:
    """Positive float32 row norms ~ 0.02*sqrt(K)-sized, for decode-only inputs."""
    return (np.exp(_rng(seed + 1).standard_normal(M) * 0.25) * 1.0).astype(np.float32)


def make_activations(T: int, K: int, seed: int) -> np.ndarray:
    """Activations for the fused decode + matmul, N(0, 1) float32 [T, K] (rounded
    to bf16 by the caller where the kernel reads bf16)."""
    return _rng(seed + 11).standard_normal((T, K), dtype=np.float32)


def gaussian_points(T: int, seed: int) -> np.ndarray:
    """T draws of the unit circular Gaussian N(0, I_2), float64 [T, 2] (PCG64
    standard normals, row-major): the training samples of a 2D codebook."""
    return _rng(seed).standard_normal((T, 2))


def make_sigma(P: int, seed: int) -> np.ndarray:
    """Positive float32 per-pair scales, for decode-only inputs."""
    return (np.exp(_rng(seed + 2).standard_normal(P) * 0.3) * 0.02).astype(np.float32)


@dataclass
class Workload:
    name: str
    specs: list = field(default_factory=list)
    ops: tuple = ("calibrate", "encode", "decode")


def _spec(name, M, K, *, dtype="bf16", dist="normal", std=0.02, out=0.0, out_scale=1.0,
          act_sigma=1.0, alpha=0.5, block=128, N=2048, bits=11, seed=0, act_seed=None):
    return MatrixSpec(name, M, K, dtype, dist, std, out, out_scale, act_sigma, alpha,
                      block, N, bits, seed, act_seed)


def tiny() -> Workload:
    """256 x 512 fp32, N(0, 0.02^2), seed 0; act RMS lognormal(0, 0.5); alpha 0.5;
    block 64; 256 centroids (8 bits per pair)."""
    return Workload("tiny_256x512_f32_b64_N256", [
        _spec("tiny", 256, 512, dtype="f32", act_sigma=0.5, block=64, N=256, bits=8, seed=0)])


def llama7b_attn() -> Workload:
    """4096 x 4096 bf16, N(0, 0.02^2) with 0.5% of columns x20; act RMS
    lognormal(0, 1); alpha 0.5; block 128; 2048 centroids (11 bits per pair)."""
    return Workload("llama7b_attn_4096x4096_bf16_b128_N2048", [
        _spec("attn", 4096, 4096, out=0.005, out_scale=20.0, seed=2000)])


def mlp_runs() -> Workload:
    """11008 x 4096 and 4096 x 11008 bf16 Student-t(4) scaled to std 0.02; act RMS
    lognormal(0, 1.5); alpha in {0.25, 0.5, 0.75}; block {128, 256}; N {1024, 2048}."""
    specs = []
    for mid, (M, K) in enumerate([(11008, 4096), (4096, 11008)]):
        for alpha in (0.25, 0.5, 0.75):
            for block in (128, 256):
                for N, bits in ((1024, 10), (2048, 11)):
                    specs.append(_spec(f"mlp{mid}_a{alpha}_b{block}_N{N}", M, K, dist="t4",
                                       act_sigma=1.5, alpha=alpha, block=block, N=N, bits=bits,
                                       seed=3000 + mid, act_seed=3000 + mid))
    return Workload("mlp_11008x4096_t4", specs)


_STACK_SHAPES = (("q", 2048, 2048, 0), ("k", 256, 2048, 0), ("v", 256, 2048, 0),
                 ("o", 2048, 2048, 1), ("gate", 5632, 2048, 2), ("up", 5632, 2048, 2),
                 ("down", 2048, 5632, 3))


def stack_1p1b(layers: int = 22) -> Workload:
    """22 layers of q/o 2048x2048, k/v 256x2048, gate/up 5632x2048, down 2048x5632
    bf16, N(0, 0.02^2) + 0.5% outlier columns; one act RMS vector per distinct
    layer input (q/k/v share, gate/up share); block 128; 2048 centroids."""
    specs = []
    for layer in range(layers):
        for mid, (nm, M, K, inp) in enumerate(_STACK_SHAPES):
            specs.append(_spec(f"L{layer}.{nm}", M, K, out=0.005, out_scale=20.0,
                               seed=4000 + 10 * layer + mid, act_seed=4000 + 10 * layer + 7 + inp))
    return Workload("stack_1p1b_22L_bf16_b128_N2048", specs)


def decode_sweep_13b() -> Workload:
    """5120x5120, 13824x5120, 5120x13824 bf16, N(0, 0.02^2), act RMS lognormal(0, 1),
    alpha 0.5, block 128, 2048 centroids; decode-only."""
    return Workload("decode_13b_sweep_bf16_b128_N2048", [
        _spec("13b.attn", 5120, 5120, seed=5000),
        _spec("13b.up", 13824, 5120, seed=5001),
        _spec("13b.down", 5120, 13824, seed=5002)], ops=("decode",))


def rate_variant(bits: int) -> Workload:
    """The lower-rate codecs on the 4096 x 4096 projection (same matrix recipe):
    3.5 bits/weight (128 centroids, 7 bits per pair) and 4 bits/weight (256
    centroids, 8 bits per pair)."""
    N = 1 << bits
    return Workload(f"llama7b_attn_4096x4096_bf16_b128_N{N}", [
        _spec("attn", 4096, 4096, out=0.005, out_scale=20.0, N=N, bits=bits, seed=2000)])


WORKLOADS = {"tiny": tiny, "llama7b_attn": llama7b_attn, "mlp": mlp_runs,
             "stack_1p1b": stack_1p1b, "decode_13b": decode_sweep_13b,
             "rate35": lambda: rate_variant(7), "rate4": lambda: rate_variant(8)}


def act_for(spec: MatrixSpec) -> np.ndarray:
    seed = spec.seed if spec.act_seed is None else spec.act_seed
    return make_act_rms(spec.K, spec.act_sigma, seed)
