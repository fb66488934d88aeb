"""Helpers for the GPU parity tests: run the CUDA path through the C ABI and
the oracle on the same seeded inputs, and compare.

Parity rules (the codec's own tolerances):
  * sigma_k, r_i, s_j: bit-exact (fp64 sums rounded once to fp32 on both sides);
  * indices: bit-exact, except where the oracle's exact relative gap between
    the two best centroid distances is below 1e-6 (such cases are counted);
  * decode fp32: max_ij |w_gpu - w_ora| / max_j |w_ora,i| <= 1e-5 (row-scaled);
  * decode bf16: within one bf16 ulp of RN_bf16(w_ora), or the bf16 rounding of a
    value within the fp32 tolerance (elements far below their row's scale).
"""
from __future__ import annotations

import numpy as np
import torch

import vector_codebook_codec_b200 as qamw
from oracle import codec

TIE_GAP = 1e-6
DECODE_TOL = 1e-5


def to_gpu_matrix(w32: np.ndarray, dtype: str):
    """Device copy of a float32 draw; for bf16 also returns the exact fp32 values."""
    if dtype == "bf16":
        t = torch.from_numpy(np.ascontiguousarray(w32)).to(torch.bfloat16)
        return t.cuda(), t.float().numpy()
    return torch.from_numpy(np.ascontiguousarray(w32)).cuda(), w32


def gpu_codec(Wd, act, alpha, block, seed, C, bits, sigma=None, search="brute"):
    """calibrate (unless sigma given) + encode on the GPU; returns numpy results.
    search: "brute" (no table) or "pruned" (the codebook's search table)."""
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    act_d = None if act is None else torch.from_numpy(act).cuda()
    if sigma is None:
        sig_d = qamw.calibrate_sigma(Wd, act_d, alpha, block, seed, status=status)
    else:
        sig_d = torch.from_numpy(sigma).cuda()
    Cd = torch.from_numpy(np.ascontiguousarray(C, dtype=np.float32)).cuda()
    table = qamw.build_search_table(Cd) if search == "pruned" else None
    enc = qamw.encode(Wd, act_d, alpha, block, seed, sig_d, Cd, bits, status=status, search_table=table)
    torch.cuda.synchronize()
    return {
        "sigma": sig_d.cpu().numpy(), "r": enc.row_norm.cpu().numpy(), "s": enc.col_scale.cpu().numpy(),
        "packed": enc.packed.cpu().numpy().view(np.uint32), "status": int(status.item()), "enc": enc, "Cd": Cd,
    }


# Index-parity records of this session: one dict per compared encoding
# (printed at the end of the run by conftest.py, and written as JSON to the
# file named by QAMW_PARITY_REPORT if that variable is set).
PARITY_RECORDS: list = []


def index_parity(gpu_packed, ora_idx, ora_gap, bits):
    """(hard mismatches, near-tie mismatches) between GPU packed rows and oracle indices."""
    P = ora_idx.shape[1]
    g = codec.unpack_indices(gpu_packed, P, bits)
    diff = g != ora_idx
    near = diff & (ora_gap < TIE_GAP)
    return int(np.sum(diff & ~near)), int(np.sum(near))


def record_parity(name, ora_gap, hard, near, scope="all pairs"):
    """Keeps the counts of one index comparison: pairs compared, pairs whose two
    best centroid distances are within the 1e-6 relative gap, and the hard and
    near-tie mismatches."""
    rec = {"case": name, "scope": scope, "pairs": int(ora_gap.size),
           "near_tie_pairs": int(np.sum(ora_gap < TIE_GAP)), "hard_mismatches": int(hard),
           "near_tie_mismatches": int(near)}
    PARITY_RECORDS.append(rec)
    return rec


def row_scaled_error(gpu: np.ndarray, ora: np.ndarray) -> float:
    scale = np.max(np.abs(ora), axis=1, keepdims=True)
    scale[scale == 0] = 1.0
    return float(np.max(np.abs(gpu.astype(np.float64) - ora) / scale))


def bf16_ulp_ok(gpu_bf16: torch.Tensor, ora: np.ndarray, tol: float = DECODE_TOL) -> bool:
    """bf16 decode check: every output is within one bf16 ulp of RN_bf16(oracle),
    or -- for elements far below their row's scale, where the fp32 rounding
    noise of the inverse rotation (bounded by ``tol`` x row max, the fp32 decode
    tolerance) exceeds a bf16 ulp of the element itself -- it is the bf16
    rounding of a value within that fp32 tolerance of the oracle."""
    ref = torch.from_numpy(ora).to(torch.float32).to(torch.bfloat16).to(torch.float64).numpy()
    got = gpu_bf16.to(torch.float64).cpu().numpy()

    def ulp(x):
        tiny = 2.0 ** -126
        return np.where(x >= tiny, 2.0 ** (np.floor(np.log2(np.maximum(x, tiny))) - 7), 2.0 ** -133)

    near = np.abs(got - ref) <= ulp(np.maximum(np.abs(ref), np.abs(got)))
    rowmax = np.max(np.abs(ora), axis=1, keepdims=True)
    within = np.abs(got - ora) <= ulp(np.abs(got)) / 2 + tol * rowmax
    return bool(np.all(near | within))


def oracle_encode_rows(W32, act, alpha, block, seed, sigma, C, rows):
    """Oracle indices and gaps for selected rows, with a given sigma (rows are independent)."""
    s, r, Y = codec.rotated_rows(W32[rows], act, alpha, block, seed)
    X = codec.normalised_pairs(Y, sigma)
    idx, gap = codec.nearest_centroid(X, C)
    return idx, gap, r, s
