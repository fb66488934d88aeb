"""The no-allocation calibration entry point, checked against the workspace one.

qamw_calibrate_sigma_noalloc serves callers that cannot allocate device
memory: an inference engine whose memory pool is frozen after start-up, a
plug-in whose host framework owns all device memory, or a latency-critical
path that must not call cudaMalloc (it may synchronize the device). It runs
the calibration on a scratch area built into the library instead of a caller
workspace. These tests call it through the C ABI and require the same sigma
as qamw_calibrate_sigma -- bit for bit, the tolerance used for sigma
everywhere (both paths sum |z| in fp64 in the same fixed order and round once)
-- on consecutive calls that share, and overwrite, that one area.

This file is collected last on purpose: if it fails, a run that stops at the
first failure has already run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

import synth
from vector_codebook_codec_b200 import QAMW_BF16, QAMW_F32, QAMW_OK, QAMW_EUNSUPPORTED

pytestmark = pytest.mark.gpu


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _inputs(spec):
    w32 = synth.make_matrix(spec)
    if spec.dtype == "bf16":
        W = torch.from_numpy(w32).to(torch.bfloat16).cuda()
        wt = QAMW_BF16
    else:
        W = torch.from_numpy(w32).cuda()
        wt = QAMW_F32
    act = torch.from_numpy(synth.act_for(spec)).cuda()
    return W, wt, act


def _sigma_noalloc(lib, spec, W, wt, act):
    M, K = W.shape
    sig = torch.full((K // 2,), float("nan"), dtype=torch.float32, device="cuda")
    rc = lib.qamw_calibrate_sigma_noalloc(_p(W), wt, M, K, W.stride(0), _p(act), spec.alpha, spec.block,
                                          spec.seed, _p(sig), None, _stream())
    assert rc == QAMW_OK, lib.qamw_last_error()
    return sig


def _sigma_workspace(lib, spec, W, wt, act):
    M, K = W.shape
    need = lib.qamw_calibrate_workspace_bytes(M, K)
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    sig = torch.full((K // 2,), float("nan"), dtype=torch.float32, device="cuda")
    rc = lib.qamw_calibrate_sigma(_p(W), wt, M, K, W.stride(0), _p(act), spec.alpha, spec.block, spec.seed,
                                  _p(sig), _p(ws), need, None, _stream())
    assert rc == QAMW_OK, lib.qamw_last_error()
    return sig


def test_noalloc_matches_workspace_version_on_consecutive_calls(lib):
    big = synth.llama7b_attn().specs[0]      # 4096 x 4096 bf16: a third of the area
    small = synth.tiny().specs[0]            # 256 x 512 fp32: reuses the stale area
    for spec in (big, small, big):
        W, wt, act = _inputs(spec)
        got = _sigma_noalloc(lib, spec, W, wt, act)
        ref = _sigma_workspace(lib, spec, W, wt, act)
        torch.cuda.synchronize()
        g, r = got.cpu().numpy(), ref.cpu().numpy()
        assert np.all(np.isfinite(g))
        assert np.array_equal(g.view(np.uint32), r.view(np.uint32))


def test_noalloc_rejects_shapes_beyond_its_area(lib):
    M, K = 8192, 8192                         # needs ~10 MiB of scratch
    assert lib.qamw_calibrate_workspace_bytes(M, K) > 8 << 20
    W = torch.zeros((M, K), dtype=torch.bfloat16, device="cuda")
    sig = torch.full((K // 2,), float("nan"), dtype=torch.float32, device="cuda")
    rc = lib.qamw_calibrate_sigma_noalloc(_p(W), QAMW_BF16, M, K, K, None, 0.5, 128, 1, _p(sig), None, _stream())
    assert rc == QAMW_EUNSUPPORTED
    assert b"built-in area" in lib.qamw_last_error()
    torch.cuda.synchronize()
    assert torch.isnan(sig).all()             # nothing was launched


def test_noalloc_limit_is_the_workspace_size_rule(lib):
    """The documented rule: align256(4K) + align256(4M) + align256(ceil(M/28) * K/2 * 8)."""
    def need(M, K):
        a = lambda v: (v + 255) // 256 * 256
        return a(4 * K) + a(4 * M) + a(-(-M // 28) * (K // 2) * 8)
    for M, K in [(1, 2), (1, 1 << 21), (27, 4096), (28, 4096), (4096, 4096), (11008, 4096), (5, 10)]:
        assert lib.qamw_calibrate_workspace_bytes(M, K) == need(M, K)
    assert need(1, 1 << 21) > 8 << 20 and need(4096, 4096) <= 8 << 20
