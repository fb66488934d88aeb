"""vector_codebook_codec_b200 -- Python binding of libqamw.so, the sm_100a QAM-W codec.

The library implements the row-parallel encode and decode of QAM-W ("QAM-W:
Joint 2D Codebook Quantization for LLM Weights via Hadamard Rotation and
Activation-Aware Scaling", Technical Summary, "Methodology: The QAM-W Codec").
Every step of the codec runs in the CUDA kernels of ``libqamw.so``; this module
only marshals arguments: it checks tensor devices, dtypes and shapes, passes raw
device pointers and the current CUDA stream through the C ABI declared in
``include/qamw.h``, and raises on a non-zero status. PyTorch provides device
memory and streams only. There is no CPU fallback: if the library is missing
or was built for another GPU the calls raise.

Functions with the C names (``qamw_calibrate_sigma``, ``qamw_encode``,
``qamw_decode``, ...) take raw pointers exactly like the C ABI; the
lower-case helpers (``calibrate_sigma``, ``encode``, ``decode``) take torch
tensors.
"""
from __future__ import annotations

import ctypes
import json
import os
from dataclasses import dataclass

import numpy as np

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libqamw.so")
CODEBOOK_DIR = os.path.join(_PKG, "codebooks")

QAMW_F32, QAMW_BF16 = 0, 1
QAMW_OK, QAMW_EINVAL, QAMW_ENULL, QAMW_EUNSUPPORTED, QAMW_ECUDA, QAMW_EWORKSPACE = range(6)
STATUS_BAD_INDEX, STATUS_NONFINITE_NORM, STATUS_BAD_ACT_RMS, STATUS_NONFINITE_INPUT, STATUS_TIMEOUT = 1, 2, 4, 8, 16

_c_i64, _c_i32, _c_u64, _c_f32, _c_sz, _c_p = (ctypes.c_int64, ctypes.c_int32, ctypes.c_uint64,
                                               ctypes.c_float, ctypes.c_size_t, ctypes.c_void_p)

# name -> (restype, argtypes); mirrors include/qamw.h
_SIGNATURES = {
    "qamw_words_per_row": (_c_i64, [_c_i64, _c_i32]),
    "qamw_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "qamw_last_error": (ctypes.c_char_p, []),
    "qamw_version": (ctypes.c_char_p, []),
    "qamw_channel_scale": (ctypes.c_int, [_c_p, _c_f32, _c_i64, _c_p, _c_p, _c_p]),
    "qamw_calibrate_workspace_bytes": (_c_sz, [_c_i64, _c_i64]),
    "qamw_calibrate_sigma": (ctypes.c_int, [_c_p, ctypes.c_int, _c_i64, _c_i64, _c_i64, _c_p, _c_f32, _c_i32,
                                            _c_u64, _c_p, _c_p, _c_sz, _c_p, _c_p]),
    "qamw_encode": (ctypes.c_int, [_c_p, ctypes.c_int, _c_i64, _c_i64, _c_i64, _c_p, _c_f32, _c_i32, _c_u64,
                                   _c_p, _c_p, _c_i32, _c_i32, _c_p, _c_p, _c_p, _c_p, _c_p, _c_p]),
    "qamw_calibrate_encode": (ctypes.c_int, [_c_p, ctypes.c_int, _c_i64, _c_i64, _c_i64, _c_p, _c_f32, _c_i32,
                                             _c_u64, _c_p, _c_i32, _c_i32, _c_p, _c_p, _c_p, _c_p, _c_p, _c_p,
                                             _c_sz, _c_p, _c_p]),
    "qamw_decode": (ctypes.c_int, [_c_p, _c_p, _c_p, _c_p, _c_i64, _c_i64, _c_i32, _c_u64, _c_p, _c_i32,
                                   _c_i32, _c_p, ctypes.c_int, _c_i64, _c_p, _c_p]),
    "qamw_rotate_rows": (ctypes.c_int, [_c_p, _c_p, _c_i64, _c_i64, _c_i32, _c_u64, _c_i32, _c_p]),
    "qamw_search_cells": (ctypes.c_int, [_c_p, _c_i64, _c_p, _c_p, _c_p]),
    "qamw_decode_matmul": (ctypes.c_int, [_c_p, _c_p, _c_p, _c_p, _c_i64, _c_i64, _c_i32, _c_u64, _c_p, _c_i32,
                                          _c_i32, _c_p, _c_i64, _c_i64, _c_p, _c_i64, _c_p, _c_sz, _c_p, _c_p]),
    "qamw_decode_matmul_workspace_bytes": (_c_sz, [_c_i64, _c_i64, _c_i64]),
    "qamw_encode_prepared": (ctypes.c_int, [_c_p, ctypes.c_int, _c_i64, _c_i64, _c_i64, _c_p, _c_p, _c_i32, _c_u64,
                                            _c_p, _c_p, _c_i32, _c_i32, _c_p, _c_p, _c_p, _c_p]),
    "qamw_search_table_bytes": (_c_sz, [_c_i32]),
    "qamw_build_search_table": (ctypes.c_int, [_c_p, _c_i32, _c_p, _c_sz, _c_p]),
    "qamw_calibrate_sigma_noalloc": (ctypes.c_int, [_c_p, ctypes.c_int, _c_i64, _c_i64, _c_i64, _c_p, _c_f32,
                                                    _c_i32, _c_u64, _c_p, _c_p, _c_p]),
    "qamw_encode_polar": (ctypes.c_int, [_c_p, ctypes.c_int, _c_i64, _c_i64, _c_i64, _c_p, _c_f32, _c_i32, _c_u64,
                                         _c_p, _c_p, _c_i32, _c_i32, _c_i32, _c_p, _c_p, _c_p, _c_p, _c_p]),
    "qamw_selftest_wait_timeout": (ctypes.c_int, [ctypes.c_uint32, _c_p, _c_p]),
    "qamw_calibrate_partial_sums": (ctypes.c_int, [_c_p, ctypes.c_int, _c_i64, _c_i64, _c_i64, _c_p, _c_f32,
                                                   _c_i32, _c_u64, _c_p, _c_p, _c_sz, _c_p, _c_p]),
    "qamw_sigma_from_partial_sums": (ctypes.c_int, [_c_p, _c_i32, _c_i64, _c_i64, _c_p, _c_p]),
    "qamw_lloyd_workspace_bytes": (_c_sz, [_c_i64, _c_i32]),
    "qamw_lloyd_assign": (ctypes.c_int, [_c_p, _c_i64, _c_p, _c_i32, _c_p, _c_p, _c_p]),
    "qamw_lloyd_update": (ctypes.c_int, [_c_p, _c_i64, _c_p, _c_i32, _c_p, _c_p, _c_sz, _c_p]),
    "qamw_lloyd_train": (ctypes.c_int, [_c_p, _c_i64, _c_p, _c_i32, _c_i32, _c_p, _c_p, _c_sz, _c_p, _c_p, _c_p]),
}

_lib = None


class QamwError(RuntimeError):
    """A libqamw call returned a non-zero status."""

    def __init__(self, fn: str, code: int, msg: str):
        super().__init__(f"{fn} failed with status {code}: {msg}")
        self.code = code


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libqamw.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise ImportError(f"libqamw.so not found at {path}; build it with "
                          f"`python -m vector_codebook_codec_b200.build`")
    lib = ctypes.CDLL(path)
    for name, (res, args) in _SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def _check(fn: str, rc: int):
    if rc != QAMW_OK:
        lib = load_library()
        raise QamwError(fn, rc, lib.qamw_last_error().decode() or lib.qamw_status_string(rc).decode())


def _raw(name):
    def call(*args):
        return getattr(load_library(), name)(*args)
    call.__name__ = name
    call.__doc__ = f"Raw C-ABI call {name} (see include/qamw.h)."
    return call


# Raw C-ABI entry points under their C names.
qamw_words_per_row = _raw("qamw_words_per_row")
qamw_status_string = _raw("qamw_status_string")
qamw_last_error = _raw("qamw_last_error")
qamw_version = _raw("qamw_version")
qamw_channel_scale = _raw("qamw_channel_scale")
qamw_calibrate_workspace_bytes = _raw("qamw_calibrate_workspace_bytes")
qamw_calibrate_sigma = _raw("qamw_calibrate_sigma")
qamw_encode = _raw("qamw_encode")
qamw_calibrate_encode = _raw("qamw_calibrate_encode")
qamw_decode = _raw("qamw_decode")
qamw_rotate_rows = _raw("qamw_rotate_rows")
qamw_encode_polar = _raw("qamw_encode_polar")
qamw_selftest_wait_timeout = _raw("qamw_selftest_wait_timeout")
qamw_calibrate_partial_sums = _raw("qamw_calibrate_partial_sums")
qamw_sigma_from_partial_sums = _raw("qamw_sigma_from_partial_sums")
qamw_lloyd_workspace_bytes = _raw("qamw_lloyd_workspace_bytes")
qamw_lloyd_assign = _raw("qamw_lloyd_assign")
qamw_lloyd_update = _raw("qamw_lloyd_update")
qamw_lloyd_train = _raw("qamw_lloyd_train")
qamw_calibrate_sigma_noalloc = _raw("qamw_calibrate_sigma_noalloc")
qamw_search_table_bytes = _raw("qamw_search_table_bytes")
qamw_build_search_table = _raw("qamw_build_search_table")
qamw_encode_prepared = _raw("qamw_encode_prepared")
qamw_search_cells = _raw("qamw_search_cells")
qamw_decode_matmul = _raw("qamw_decode_matmul")
qamw_decode_matmul_workspace_bytes = _raw("qamw_decode_matmul_workspace_bytes")


# ---------------------------------------------------------------------------
# torch-tensor helpers (argument marshalling only)
# ---------------------------------------------------------------------------

def _torch():
    import torch
    return torch


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream_ptr(stream=None):
    torch = _torch()
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _need_cuda(name, t, dtype=None, ndim=None):
    if t is None:
        return
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must have dtype {dtype}, got {t.dtype}")
    if ndim is not None and t.dim() != ndim:
        raise ValueError(f"{name} must be {ndim}-D")


def _wdtype(W):
    torch = _torch()
    if W.dtype == torch.bfloat16:
        return QAMW_BF16
    if W.dtype == torch.float32:
        return QAMW_F32
    raise ValueError("W must be bfloat16 or float32")


def _ld(W):
    if W.stride(1) != 1:
        raise ValueError("W must be row-major with unit column stride")
    return W.stride(0) if W.shape[0] > 1 else W.shape[1]


def words_per_row(K: int, bits: int) -> int:
    return int(load_library().qamw_words_per_row(K, bits))


def load_codebook(N: int):
    """The shipped joint 2D Lloyd-Max codebook with N centroids (float32 numpy [N, 2])."""
    path = os.path.join(CODEBOOK_DIR, f"qamw_lloyd_N{N}.npy")
    if not os.path.exists(path):
        raise FileNotFoundError(f"no shipped codebook with N={N} ({path})")
    return np.load(path).astype(np.float32)


def load_polar(N: int) -> dict:
    """The shipped polar baseline code of N = A * P points: ``amps`` (float64
    [A], ascending), ``P``, and ``points`` (float32 [N, 2], index order)."""
    import numpy as np
    e = codebook_manifest()[str(N)]
    return {"amps": np.load(os.path.join(CODEBOOK_DIR, e["polar_amps_file"])), "P": int(e["polar_sectors"]),
            "points": np.load(os.path.join(CODEBOOK_DIR, e["polar_points_file"]))}


def codebook_manifest() -> dict:
    with open(os.path.join(CODEBOOK_DIR, "manifest.json")) as f:
        return json.load(f)


def channel_scale(act_rms, alpha: float, K: int, status=None, stream=None):
    torch = _torch()
    _need_cuda("act_rms", act_rms, torch.float32, 1)
    s = torch.empty(K, dtype=torch.float32, device="cuda" if act_rms is None else act_rms.device)
    _check("qamw_channel_scale", load_library().qamw_channel_scale(
        _ptr(act_rms), float(alpha), K, _ptr(s), _ptr(status), _stream_ptr(stream)))
    return s


def calibrate_sigma(W, act_rms, alpha: float, block: int, seed: int, status=None, workspace=None,
                    stream=None, out=None):
    """sigma_k for every pair position of W (float32 [K/2]); see qamw_calibrate_sigma."""
    torch = _torch()
    _need_cuda("W", W, ndim=2)
    _need_cuda("act_rms", act_rms, torch.float32, 1)
    M, K = W.shape
    lib = load_library()
    need = int(lib.qamw_calibrate_workspace_bytes(M, K))
    if workspace is None or workspace.numel() < need:
        workspace = torch.empty(need, dtype=torch.uint8, device=W.device)
    sigma = torch.empty(K // 2, dtype=torch.float32, device=W.device) if out is None else out
    _check("qamw_calibrate_sigma", lib.qamw_calibrate_sigma(
        _ptr(W), _wdtype(W), M, K, _ld(W), _ptr(act_rms), float(alpha), block, seed & (2**64 - 1),
        _ptr(sigma), _ptr(workspace), workspace.numel(), _ptr(status), _stream_ptr(stream)))
    return sigma


def calibrate_partial_sums(W, act_rms, alpha: float, block: int, seed: int, status=None, workspace=None,
                           stream=None, out=None):
    """fp64 [K/2] sums of |z_ik| over W's rows (one shard of a row-split matrix)."""
    torch = _torch()
    _need_cuda("W", W, ndim=2)
    _need_cuda("act_rms", act_rms, torch.float32, 1)
    M, K = W.shape
    lib = load_library()
    need = int(lib.qamw_calibrate_workspace_bytes(M, K))
    if workspace is None or workspace.numel() < need:
        workspace = torch.empty(need, dtype=torch.uint8, device=W.device)
    sums = torch.empty(K // 2, dtype=torch.float64, device=W.device) if out is None else out
    _check("qamw_calibrate_partial_sums", lib.qamw_calibrate_partial_sums(
        _ptr(W), _wdtype(W), M, K, _ld(W), _ptr(act_rms), float(alpha), block, seed & (2**64 - 1),
        _ptr(sums), _ptr(workspace), workspace.numel(), _ptr(status), _stream_ptr(stream)))
    return sums


def sigma_from_partial_sums(sums, M_total: int, stream=None, out=None):
    """sigma [P] from the shards' sums (float64 [R][P], shard order)."""
    torch = _torch()
    _need_cuda("sums", sums, torch.float64, 2)
    sums = sums.contiguous()
    R, P = sums.shape
    sigma = torch.empty(P, dtype=torch.float32, device=sums.device) if out is None else out
    _check("qamw_sigma_from_partial_sums", load_library().qamw_sigma_from_partial_sums(
        _ptr(sums), R, P, int(M_total), _ptr(sigma), _stream_ptr(stream)))
    return sigma


def gather_partial_sums(sums, group=None):
    """All-gathers every rank's [P] sums into a [world, P] tensor in rank order
    (one collective: NCCL over NVLink between GPUs, or gloo on CPU)."""
    torch = _torch()
    import torch.distributed as dist
    world = dist.get_world_size(group)
    flat = torch.empty(world * sums.numel(), dtype=sums.dtype, device=sums.device)
    dist.all_gather_into_tensor(flat, sums.contiguous().view(-1), group=group)
    return flat.view(world, sums.numel())


def calibrate_sigma_sharded(W_shard, act_rms, alpha: float, block: int, seed: int, M_total: int, group=None,
                            status=None, stream=None):
    """sigma of a matrix whose rows are split across the ranks of ``group``:
    each rank passes its rows; every rank gets the same sigma."""
    sums = calibrate_partial_sums(W_shard, act_rms, alpha, block, seed, status=status, stream=stream)
    return sigma_from_partial_sums(gather_partial_sums(sums, group), M_total, stream=stream)


@dataclass
class Encoded:
    """An encoded matrix: the stored artefacts the decode needs."""
    packed: object      # uint32 stored as torch.int32 [M, words_per_row]
    row_norm: object    # float32 [M]
    col_scale: object   # float32 [K]  (s_j)
    sigma: object       # float32 [K/2]
    M: int
    K: int
    block: int
    seed: int
    N: int
    bits: int


def build_search_table(codebook, stream=None):
    """Search table for the exact pruned search (uint8 CUDA tensor); build once per codebook."""
    torch = _torch()
    _need_cuda("codebook", codebook, torch.float32, 2)
    N = codebook.shape[0]
    lib = load_library()
    nbytes = int(lib.qamw_search_table_bytes(N))
    if nbytes == 0:
        raise ValueError(f"no search table for N={N}")
    table = torch.empty(nbytes, dtype=torch.uint8, device=codebook.device)
    _check("qamw_build_search_table", lib.qamw_build_search_table(
        _ptr(codebook.contiguous()), N, _ptr(table), nbytes, _stream_ptr(stream)))
    return table


def encode(W, act_rms, alpha: float, block: int, seed: int, sigma, codebook, bits: int,
           status=None, stream=None, out=None, search_table=None) -> Encoded:
    """Encode W with the given sigma and codebook (float32 CUDA tensor [N, 2]).

    ``search_table`` (from :func:`build_search_table`) selects the exact pruned
    search; without it every pair is compared with all N centroids."""
    torch = _torch()
    _need_cuda("W", W, ndim=2)
    _need_cuda("act_rms", act_rms, torch.float32, 1)
    _need_cuda("sigma", sigma, torch.float32, 1)
    _need_cuda("codebook", codebook, torch.float32, 2)
    M, K = W.shape
    N = codebook.shape[0]
    wpr = words_per_row(K, bits)
    if wpr < 0:
        raise ValueError("invalid K / bits")
    if out is None:
        packed = torch.empty((M, wpr), dtype=torch.int32, device=W.device)
        r = torch.empty(M, dtype=torch.float32, device=W.device)
        s = torch.empty(K, dtype=torch.float32, device=W.device)
    else:
        packed, r, s = out
    _check("qamw_encode", load_library().qamw_encode(
        _ptr(W), _wdtype(W), M, K, _ld(W), _ptr(act_rms), float(alpha), block, seed & (2**64 - 1),
        _ptr(sigma), _ptr(codebook.contiguous()), N, bits, _ptr(search_table), _ptr(packed), _ptr(r), _ptr(s),
        _ptr(status), _stream_ptr(stream)))
    return Encoded(packed, r, s, sigma, M, K, block, seed, N, bits)


def encode_prepared(W, col_scale, row_norm, block: int, seed: int, sigma, codebook, bits: int,
                    status=None, stream=None, out=None, search_table=None) -> Encoded:
    """Encode W given its channel scales s_j and row norms r_i (qamw_encode_prepared):
    the encode kernel alone. ``out`` = packed words preallocated, or None."""
    torch = _torch()
    _need_cuda("W", W, ndim=2)
    _need_cuda("col_scale", col_scale, torch.float32, 1)
    _need_cuda("row_norm", row_norm, torch.float32, 1)
    _need_cuda("sigma", sigma, torch.float32, 1)
    _need_cuda("codebook", codebook, torch.float32, 2)
    M, K = W.shape
    N = codebook.shape[0]
    wpr = words_per_row(K, bits)
    if wpr < 0:
        raise ValueError("invalid K / bits")
    packed = torch.empty((M, wpr), dtype=torch.int32, device=W.device) if out is None else out
    _check("qamw_encode_prepared", load_library().qamw_encode_prepared(
        _ptr(W), _wdtype(W), M, K, _ld(W), _ptr(col_scale), _ptr(row_norm), block, seed & (2**64 - 1),
        _ptr(sigma), _ptr(codebook.contiguous()), N, bits, _ptr(search_table), _ptr(packed), _ptr(status),
        _stream_ptr(stream)))
    return Encoded(packed, row_norm, col_scale, sigma, M, K, block, seed, N, bits)


def calibrate_encode(W, act_rms, alpha: float, block: int, seed: int, codebook, bits: int,
                     status=None, stream=None, out=None, search_table=None, workspace=None) -> Encoded:
    """:func:`calibrate_sigma` then :func:`encode` in one call (qamw_calibrate_encode):
    s_j and r_i are computed once; the result equals the two calls' bit for bit.
    ``out`` = (packed, row_norm, col_scale, sigma) preallocated, or None."""
    torch = _torch()
    _need_cuda("W", W, ndim=2)
    _need_cuda("act_rms", act_rms, torch.float32, 1)
    _need_cuda("codebook", codebook, torch.float32, 2)
    M, K = W.shape
    N = codebook.shape[0]
    wpr = words_per_row(K, bits)
    if wpr < 0:
        raise ValueError("invalid K / bits")
    lib = load_library()
    need = int(lib.qamw_calibrate_workspace_bytes(M, K))
    if workspace is None or workspace.numel() < need:
        workspace = torch.empty(need, dtype=torch.uint8, device=W.device)
    if out is None:
        packed = torch.empty((M, wpr), dtype=torch.int32, device=W.device)
        r = torch.empty(M, dtype=torch.float32, device=W.device)
        s = torch.empty(K, dtype=torch.float32, device=W.device)
        sigma = torch.empty(K // 2, dtype=torch.float32, device=W.device)
    else:
        packed, r, s, sigma = out
    _check("qamw_calibrate_encode", lib.qamw_calibrate_encode(
        _ptr(W), _wdtype(W), M, K, _ld(W), _ptr(act_rms), float(alpha), block, seed & (2**64 - 1),
        _ptr(codebook.contiguous()), N, bits, _ptr(search_table), _ptr(sigma), _ptr(packed), _ptr(r), _ptr(s),
        _ptr(workspace), workspace.numel(), _ptr(status), _stream_ptr(stream)))
    return Encoded(packed, r, s, sigma, M, K, block, seed, N, bits)


def encode_polar(W, act_rms, alpha: float, block: int, seed: int, sigma, amps, P: int, bits: int,
                 status=None, stream=None, out=None) -> Encoded:
    """Encode W with the polar baseline code (amps: float64 CUDA tensor [A], P
    sectors); decode the result with :func:`decode` and the code's points."""
    torch = _torch()
    _need_cuda("W", W, ndim=2)
    _need_cuda("act_rms", act_rms, torch.float32, 1)
    _need_cuda("sigma", sigma, torch.float32, 1)
    _need_cuda("amps", amps, torch.float64, 1)
    M, K = W.shape
    A = amps.shape[0]
    wpr = words_per_row(K, bits)
    if wpr < 0:
        raise ValueError("invalid K / bits")
    if out is None:
        packed = torch.empty((M, wpr), dtype=torch.int32, device=W.device)
        r = torch.empty(M, dtype=torch.float32, device=W.device)
        s = torch.empty(K, dtype=torch.float32, device=W.device)
    else:
        packed, r, s = out
    _check("qamw_encode_polar", load_library().qamw_encode_polar(
        _ptr(W), _wdtype(W), M, K, _ld(W), _ptr(act_rms), float(alpha), block, seed & (2**64 - 1),
        _ptr(sigma), _ptr(amps.contiguous()), A, int(P), bits, _ptr(packed), _ptr(r), _ptr(s), _ptr(status),
        _stream_ptr(stream)))
    return Encoded(packed, r, s, sigma, M, K, block, seed, A * int(P), bits)


def decode(enc: Encoded, codebook, out_dtype=None, status=None, stream=None, out=None):
    """Decode an :class:`Encoded` matrix to bf16 (default) or fp32 [M, K]."""
    torch = _torch()
    out_dtype = torch.bfloat16 if out_dtype is None else out_dtype
    ot = QAMW_BF16 if out_dtype == torch.bfloat16 else QAMW_F32
    if out is None:
        out = torch.empty((enc.M, enc.K), dtype=out_dtype, device=enc.packed.device)
    _check("qamw_decode", load_library().qamw_decode(
        _ptr(enc.packed), _ptr(enc.row_norm), _ptr(enc.sigma), _ptr(enc.col_scale), enc.M, enc.K,
        enc.block, enc.seed & (2**64 - 1), _ptr(codebook.contiguous()), codebook.shape[0], enc.bits,
        _ptr(out), ot, _ld(out), _ptr(status), _stream_ptr(stream)))
    return out


def decode_matmul_workspace_bytes(M: int, K: int, T: int) -> int:
    return int(load_library().qamw_decode_matmul_workspace_bytes(M, K, T))


def decode_matmul(enc: Encoded, codebook, X, status=None, stream=None, out=None, workspace=None):
    """Y = X @ decode(enc)^T with the decode fused into the tensor-core matmul
    (qamw_decode_matmul); X is a bf16 CUDA tensor [T, K], Y float32 [T, M].
    ``workspace`` (a CUDA uint8 tensor of decode_matmul_workspace_bytes(M, K, T)
    bytes) is allocated here when not given."""
    torch = _torch()
    _need_cuda("codebook", codebook, torch.float32, 2)
    _need_cuda("X", X, torch.bfloat16, 2)
    if X.shape[1] != enc.K:
        raise ValueError("X must have K columns")
    T = X.shape[0]
    Y = torch.empty((T, enc.M), dtype=torch.float32, device=X.device) if out is None else out
    nws = decode_matmul_workspace_bytes(enc.M, enc.K, T)
    if workspace is None:
        workspace = torch.empty(nws, dtype=torch.uint8, device=X.device)
    _check("qamw_decode_matmul", load_library().qamw_decode_matmul(
        _ptr(enc.packed), _ptr(enc.row_norm), _ptr(enc.sigma), _ptr(enc.col_scale), enc.M, enc.K, enc.block,
        enc.seed & (2**64 - 1), _ptr(codebook.contiguous()), codebook.shape[0], enc.bits, _ptr(X), T, _ld(X),
        _ptr(Y), _ld(Y), _ptr(workspace), workspace.numel() * workspace.element_size(), _ptr(status),
        _stream_ptr(stream)))
    return Y


def rotate_rows(U, block: int, seed: int, inverse: bool = False, stream=None):
    """The rotation alone on float64 rows (test hook of the encode's fp64 rotation)."""
    torch = _torch()
    _need_cuda("U", U, torch.float64, 2)
    U = U.contiguous()
    Y = torch.empty_like(U)
    M, K = U.shape
    _check("qamw_rotate_rows", load_library().qamw_rotate_rows(
        _ptr(U), _ptr(Y), M, K, block, seed & (2**64 - 1), 1 if inverse else 0, _stream_ptr(stream)))
    return Y


def search_cells(x, table, stream=None):
    """The encode's grid cell of each pair of x (float32 CUDA tensor [n, 2]) for
    a search table (int32 tensor [n]; -1 outside the grid). Test hook."""
    torch = _torch()
    _need_cuda("x", x, torch.float32, 2)
    x = x.contiguous()
    out = torch.empty(x.shape[0], dtype=torch.int32, device=x.device)
    _check("qamw_search_cells", load_library().qamw_search_cells(
        _ptr(x), x.shape[0], _ptr(table), _ptr(out), _stream_ptr(stream)))
    return out


# ---------------------------------------------------------------------------
# Lloyd training of the 2D codebook (qamw_lloyd_*)
# ---------------------------------------------------------------------------

def _lloyd_inputs(points, centroids):
    torch = _torch()
    _need_cuda("points", points, torch.float64, 2)
    _need_cuda("centroids", centroids, torch.float64, 2)
    if points.shape[1] != 2 or centroids.shape[1] != 2:
        raise ValueError("points and centroids must be [.][2]")
    return points.contiguous(), centroids.contiguous()


def _lloyd_workspace(lib, T, N, device):
    torch = _torch()
    need = int(lib.qamw_lloyd_workspace_bytes(T, N))
    return torch.empty(need, dtype=torch.uint8, device=device), need


def lloyd_assign(points, centroids, idx=None, changed=None, stream=None):
    """Nearest centroid (fp64, lowest index on ties) of every point; int32 [T]."""
    torch = _torch()
    points, centroids = _lloyd_inputs(points, centroids)
    T, N = points.shape[0], centroids.shape[0]
    if idx is None:
        idx = torch.full((T,), -1, dtype=torch.int32, device=points.device)
    _check("qamw_lloyd_assign", load_library().qamw_lloyd_assign(
        _ptr(points), T, _ptr(centroids), N, _ptr(idx), _ptr(changed), _stream_ptr(stream)))
    return idx


def lloyd_update(points, idx, centroids, stream=None):
    """Moves the centroids (fp64 [N][2] CUDA tensor, in place) to the means of their points."""
    points, c = _lloyd_inputs(points, centroids)
    if c.data_ptr() != centroids.data_ptr():
        raise ValueError("centroids must be contiguous (updated in place)")
    lib = load_library()
    ws, need = _lloyd_workspace(lib, points.shape[0], c.shape[0], points.device)
    _check("qamw_lloyd_update", lib.qamw_lloyd_update(
        _ptr(points), points.shape[0], _ptr(idx), c.shape[0], _ptr(c), _ptr(ws), need, _stream_ptr(stream)))
    return centroids


def lloyd_train(points, init, max_iter: int = 500, stream=None):
    """Lloyd iterations from ``init`` (fp64 [N][2]) on ``points`` (fp64 [T][2]).
    Returns (centroids, idx, iterations, converged); see qamw_lloyd_train."""
    torch = _torch()
    points, init = _lloyd_inputs(points, init)
    C = init.clone()
    T, N = points.shape[0], C.shape[0]
    idx = torch.empty(T, dtype=torch.int32, device=points.device)
    lib = load_library()
    ws, need = _lloyd_workspace(lib, T, N, points.device)
    it, conv = ctypes.c_int32(0), ctypes.c_int32(0)
    _check("qamw_lloyd_train", lib.qamw_lloyd_train(
        _ptr(points), T, _ptr(C), N, int(max_iter), _ptr(idx), _ptr(ws), need, ctypes.byref(it),
        ctypes.byref(conv), _stream_ptr(stream)))
    return C, idx, int(it.value), bool(conv.value)


# ---------------------------------------------------------------------------
# the encoded artefact on disk
# ---------------------------------------------------------------------------

ENCODED_FORMAT = "qamw-encoded"
ENCODED_VERSION = 1


def save_encoded(path: str, enc: Encoded, codebook) -> None:
    """Writes an encoded matrix and its codebook to ``path`` (numpy .npz): the
    packed words, r_i, s_j, sigma_k, the codebook, and block, seed, N, bits,
    M, K, with a format name and version. Everything qamw_decode needs."""
    import numpy as np

    def host(t):
        return t.detach().cpu().numpy() if hasattr(t, "detach") else np.asarray(t)

    np.savez(path, format=np.array(ENCODED_FORMAT), version=np.array(ENCODED_VERSION, dtype=np.int32),
             packed=host(enc.packed).view(np.uint32), row_norm=host(enc.row_norm).astype(np.float32),
             col_scale=host(enc.col_scale).astype(np.float32), sigma=host(enc.sigma).astype(np.float32),
             codebook=host(codebook).astype(np.float32),
             shape=np.array([enc.M, enc.K, enc.block, enc.N, enc.bits], dtype=np.int64),
             seed=np.array(enc.seed, dtype=np.uint64))


def load_encoded(path: str, device="cuda"):
    """Reads a file written by :func:`save_encoded`; returns (Encoded, codebook)
    as tensors on ``device``. Raises ValueError on another format or version."""
    import numpy as np
    torch = _torch()
    with np.load(path, allow_pickle=False) as z:
        if str(z["format"]) != ENCODED_FORMAT:
            raise ValueError(f"{path}: not a {ENCODED_FORMAT} file")
        if int(z["version"]) != ENCODED_VERSION:
            raise ValueError(f"{path}: format version {int(z['version'])}, expected {ENCODED_VERSION}")
        M, K, block, N, bits = (int(v) for v in z["shape"])
        seed = int(z["seed"])
        if words_per_row(K, bits) != z["packed"].shape[1] or z["packed"].shape[0] != M:
            raise ValueError(f"{path}: packed words do not match M, K, bits")

        def dev(a):
            return torch.from_numpy(np.ascontiguousarray(a)).to(device)

        enc = Encoded(dev(z["packed"].view(np.int32)), dev(z["row_norm"]), dev(z["col_scale"]), dev(z["sigma"]),
                      M, K, block, seed, N, bits)
        return enc, dev(z["codebook"])
