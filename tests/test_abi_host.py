"""Host-only checks of the C ABI: the library loads, exports every function
``include/qamw.h`` declares, and rejects bad arguments on the host with the
documented status code before touching the GPU (these calls never reach a
CUDA API, so they run without a device)."""
import ctypes
import os
import re
import subprocess

import pytest

from vector_codebook_codec_b200 import (LIB_PATH, QAMW_EINVAL, QAMW_ENULL, QAMW_EUNSUPPORTED,
                                        QAMW_EWORKSPACE, QAMW_OK)

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "qamw.h")
FAKE = ctypes.c_void_p(0x10000)   # never dereferenced: validation fails first


def _declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(qamw_\w+)\s*\(", text)))


def test_header_declares_the_codec_entry_points():
    names = _declared_functions()
    for n in ("qamw_calibrate_sigma", "qamw_encode", "qamw_decode", "qamw_words_per_row",
              "qamw_calibrate_workspace_bytes", "qamw_status_string", "qamw_last_error"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", LIB_PATH], capture_output=True, text=True).stdout
    exported = set(re.findall(r"\bT (qamw_\w+)$", out, flags=re.M))
    missing = [n for n in _declared_functions() if n not in exported]
    assert not missing, missing
    for n in _declared_functions():
        getattr(lib, n)


def test_words_per_row(lib):
    assert lib.qamw_words_per_row(4096, 11) == 704
    assert lib.qamw_words_per_row(11008, 10) == 1720
    assert lib.qamw_words_per_row(13824, 11) == 2376
    assert lib.qamw_words_per_row(512, 8) == 64
    assert lib.qamw_words_per_row(12, 11) == 3
    assert lib.qamw_words_per_row(3, 8) == -1
    assert lib.qamw_words_per_row(8, 0) == -1
    assert lib.qamw_words_per_row(8, 17) == -1


def test_status_strings(lib):
    for code in range(6):
        assert lib.qamw_status_string(code)
    assert lib.qamw_status_string(99) == b"unknown status"


def test_calibrate_workspace_bytes(lib):
    """The layout the header states: s [K] and r [M] in fp32, then the fp64
    partial sums [ceil(M/28)][K/2], each section rounded up to 256 bytes."""
    def a256(n):
        return (n + 255) // 256 * 256
    for M, K in ((4096, 4096), (1, 2), (29, 1000), (11008, 4096), (4096, 11008)):
        groups = (M + 27) // 28
        assert lib.qamw_calibrate_workspace_bytes(M, K) == a256(4 * K) + a256(4 * M) + a256(groups * (K // 2) * 8)
    assert lib.qamw_calibrate_workspace_bytes(0, 8) == 0
    assert lib.qamw_calibrate_workspace_bytes(8, 1) == 0


def _enc(lib, **kw):
    a = dict(W=FAKE, wt=1, M=8, K=256, ldw=256, act=None, alpha=0.5, block=128, seed=1, sigma=FAKE,
             cb=FAKE, N=256, bits=8, table=None, packed=FAKE, r=FAKE, s=FAKE, status=None, stream=None)
    a.update(kw)
    return lib.qamw_encode(a["W"], a["wt"], a["M"], a["K"], a["ldw"], a["act"], a["alpha"], a["block"],
                           a["seed"], a["sigma"], a["cb"], a["N"], a["bits"], a["table"], a["packed"], a["r"],
                           a["s"], a["status"], a["stream"])


def _dec(lib, **kw):
    a = dict(packed=FAKE, r=FAKE, sigma=FAKE, s=None, M=8, K=256, block=128, seed=1, cb=FAKE, N=256,
             bits=8, out=FAKE, ot=1, ldo=256, status=None, stream=None)
    a.update(kw)
    return lib.qamw_decode(a["packed"], a["r"], a["sigma"], a["s"], a["M"], a["K"], a["block"], a["seed"],
                           a["cb"], a["N"], a["bits"], a["out"], a["ot"], a["ldo"], a["status"], a["stream"])


def _cal(lib, **kw):
    a = dict(W=FAKE, wt=1, M=8, K=256, ldw=256, act=None, alpha=0.5, block=128, seed=1, sigma=FAKE,
             ws=FAKE, wsb=1 << 30, status=None, stream=None)
    a.update(kw)
    return lib.qamw_calibrate_sigma(a["W"], a["wt"], a["M"], a["K"], a["ldw"], a["act"], a["alpha"],
                                    a["block"], a["seed"], a["sigma"], a["ws"], a["wsb"], a["status"],
                                    a["stream"])


@pytest.mark.parametrize("kw,code", [
    (dict(W=None), QAMW_ENULL), (dict(sigma=None), QAMW_ENULL), (dict(cb=None), QAMW_ENULL),
    (dict(packed=None), QAMW_ENULL), (dict(r=None), QAMW_ENULL), (dict(s=None), QAMW_ENULL),
    (dict(K=255, ldw=255), QAMW_EINVAL), (dict(K=192, ldw=192), QAMW_EINVAL),
    (dict(block=96), QAMW_EINVAL), (dict(block=1), QAMW_EINVAL), (dict(block=2048, K=2048, ldw=2048), QAMW_EUNSUPPORTED),
    (dict(M=0), QAMW_EINVAL), (dict(ldw=128), QAMW_EINVAL), (dict(bits=0), QAMW_EINVAL),
    (dict(bits=17), QAMW_EINVAL), (dict(N=257), QAMW_EINVAL), (dict(N=0), QAMW_EINVAL),
    (dict(N=16384, bits=16), QAMW_EUNSUPPORTED), (dict(alpha=float("nan")), QAMW_EINVAL),
    (dict(alpha=float("inf")), QAMW_EINVAL), (dict(wt=7), QAMW_EINVAL),
    (dict(table=ctypes.c_void_p(0x10008)), QAMW_EINVAL),
])
def test_encode_rejects_on_host(lib, kw, code):
    assert _enc(lib, **kw) == code
    assert lib.qamw_last_error()


@pytest.mark.parametrize("kw,code", [
    (dict(packed=None), QAMW_ENULL), (dict(r=None), QAMW_ENULL), (dict(sigma=None), QAMW_ENULL),
    (dict(cb=None), QAMW_ENULL), (dict(out=None), QAMW_ENULL), (dict(K=7), QAMW_EINVAL),
    (dict(block=3), QAMW_EINVAL), (dict(ldo=100), QAMW_EINVAL), (dict(N=300), QAMW_EINVAL),
    (dict(ot=5), QAMW_EINVAL), (dict(bits=20, N=4), QAMW_EINVAL),
])
def test_decode_rejects_on_host(lib, kw, code):
    assert _dec(lib, **kw) == code


@pytest.mark.parametrize("kw,code", [
    (dict(W=None), QAMW_ENULL), (dict(sigma=None), QAMW_ENULL), (dict(ws=None), QAMW_EWORKSPACE),
    (dict(wsb=16), QAMW_EWORKSPACE), (dict(ws=ctypes.c_void_p(0x10010)), QAMW_EINVAL),
    (dict(K=100, ldw=100), QAMW_EINVAL), (dict(alpha=float("nan")), QAMW_EINVAL), (dict(ldw=3), QAMW_EINVAL),
])
def test_calibrate_rejects_on_host(lib, kw, code):
    assert _cal(lib, **kw) == code


def _cal_enc(lib, **kw):
    a = dict(W=FAKE, wt=1, M=8, K=256, ldw=256, act=None, alpha=0.5, block=128, seed=1, cb=FAKE, N=256,
             bits=8, table=None, sigma=FAKE, packed=FAKE, r=FAKE, s=FAKE, ws=FAKE, wsb=1 << 30, status=None,
             stream=None)
    a.update(kw)
    return lib.qamw_calibrate_encode(a["W"], a["wt"], a["M"], a["K"], a["ldw"], a["act"], a["alpha"],
                                     a["block"], a["seed"], a["cb"], a["N"], a["bits"], a["table"], a["sigma"],
                                     a["packed"], a["r"], a["s"], a["ws"], a["wsb"], a["status"], a["stream"])


@pytest.mark.parametrize("kw,code", [
    (dict(W=None), QAMW_ENULL), (dict(cb=None), QAMW_ENULL), (dict(sigma=None), QAMW_ENULL),
    (dict(packed=None), QAMW_ENULL), (dict(r=None), QAMW_ENULL), (dict(s=None), QAMW_ENULL),
    (dict(ws=None), QAMW_EWORKSPACE), (dict(wsb=16), QAMW_EWORKSPACE),
    (dict(ws=ctypes.c_void_p(0x10010)), QAMW_EINVAL), (dict(K=255, ldw=255), QAMW_EINVAL),
    (dict(block=96), QAMW_EINVAL), (dict(M=0), QAMW_EINVAL), (dict(ldw=128), QAMW_EINVAL),
    (dict(N=257), QAMW_EINVAL), (dict(bits=17), QAMW_EINVAL), (dict(alpha=float("nan")), QAMW_EINVAL),
    (dict(wt=7), QAMW_EINVAL), (dict(table=ctypes.c_void_p(0x10008)), QAMW_EINVAL),
    (dict(block=2048, K=2048, ldw=2048), QAMW_EUNSUPPORTED),
])
def test_calibrate_encode_rejects_on_host(lib, kw, code):
    assert _cal_enc(lib, **kw) == code
    assert lib.qamw_last_error()


def test_rotate_and_scale_reject_on_host(lib):
    assert lib.qamw_rotate_rows(None, FAKE, 2, 8, 4, 0, 0, None) == QAMW_ENULL
    assert lib.qamw_rotate_rows(FAKE, FAKE, 2, 12, 8, 0, 0, None) == QAMW_EINVAL
    assert lib.qamw_channel_scale(None, 0.5, 8, None, None, None) == QAMW_ENULL
    assert lib.qamw_channel_scale(None, float("nan"), 8, FAKE, None, None) == QAMW_EINVAL


def test_error_message_cleared_on_next_rejection(lib):
    assert _enc(lib, W=None) == QAMW_ENULL
    first = lib.qamw_last_error()
    assert _enc(lib, K=255, ldw=255) == QAMW_EINVAL
    assert lib.qamw_last_error() != first and b"K" in lib.qamw_last_error()
    assert QAMW_OK == 0


def test_lloyd_entry_points_reject_on_host(lib):
    ws = 1 << 30
    assert lib.qamw_lloyd_workspace_bytes(0, 16) == 0
    assert lib.qamw_lloyd_workspace_bytes(1000, 16) >= 3 * 8 * 16 + 8
    assert lib.qamw_lloyd_assign(None, 10, FAKE, 4, FAKE, None, None) == QAMW_ENULL
    assert lib.qamw_lloyd_assign(FAKE, 10, FAKE, 4, None, None, None) == QAMW_ENULL
    assert lib.qamw_lloyd_assign(FAKE, 0, FAKE, 4, FAKE, None, None) == QAMW_EINVAL
    assert lib.qamw_lloyd_assign(FAKE, 10, FAKE, 0, FAKE, None, None) == QAMW_EINVAL
    assert lib.qamw_lloyd_assign(FAKE, 10, FAKE, 8193, FAKE, None, None) == QAMW_EINVAL
    assert lib.qamw_lloyd_assign(ctypes.c_void_p(0x10008), 10, FAKE, 4, FAKE, None, None) == QAMW_EINVAL
    assert lib.qamw_lloyd_update(FAKE, 10, FAKE, 4, FAKE, None, ws, None) == QAMW_EWORKSPACE
    assert lib.qamw_lloyd_update(FAKE, 10, FAKE, 4, FAKE, FAKE, 8, None) == QAMW_EWORKSPACE
    assert lib.qamw_lloyd_update(FAKE, 10, None, 4, FAKE, FAKE, ws, None) == QAMW_ENULL
    assert lib.qamw_lloyd_update(FAKE, 10, FAKE, 4, FAKE, ctypes.c_void_p(0x10010), ws, None) == QAMW_EINVAL
    it, conv = ctypes.c_int32(-5), ctypes.c_int32(-5)
    assert lib.qamw_lloyd_train(FAKE, 10, FAKE, 4, -1, FAKE, FAKE, ws, ctypes.byref(it), ctypes.byref(conv),
                                None) == QAMW_EINVAL
    assert lib.qamw_lloyd_train(FAKE, 10, FAKE, 4, 5, None, FAKE, ws, None, None, None) == QAMW_ENULL
    assert it.value == -5 and conv.value == -5   # untouched on a rejected call


def test_encode_polar_rejects_on_host(lib):
    def call(**kw):
        a = dict(W=FAKE, wt=1, M=8, K=256, ldw=256, act=None, alpha=0.5, block=128, seed=1, sigma=FAKE,
                 amps=FAKE, A=8, P=32, bits=8, packed=FAKE, r=FAKE, s=FAKE)
        a.update(kw)
        return lib.qamw_encode_polar(a["W"], a["wt"], a["M"], a["K"], a["ldw"], a["act"], a["alpha"], a["block"],
                                     a["seed"], a["sigma"], a["amps"], a["A"], a["P"], a["bits"], a["packed"],
                                     a["r"], a["s"], None, None)
    assert call(amps=None) == QAMW_ENULL
    assert call(A=0) == QAMW_EINVAL
    assert call(P=0) == QAMW_EINVAL
    assert call(A=16, P=32) == QAMW_EINVAL          # 512 points > 2^8
    assert call(amps=ctypes.c_void_p(0x10004)) == QAMW_EINVAL
    assert call(block=1024, K=1024, ldw=1024) == QAMW_EUNSUPPORTED


def test_selftest_rejects_on_host(lib):
    assert lib.qamw_selftest_wait_timeout(5, None, None) == QAMW_ENULL
    assert lib.qamw_selftest_wait_timeout(0, FAKE, None) == QAMW_EINVAL
    assert lib.qamw_selftest_wait_timeout((1 << 20) + 1, FAKE, None) == QAMW_EINVAL


def test_sharded_calibration_rejects_on_host(lib):
    assert lib.qamw_sigma_from_partial_sums(None, 1, 8, 8, FAKE, None) == QAMW_ENULL
    assert lib.qamw_sigma_from_partial_sums(FAKE, 0, 8, 8, FAKE, None) == QAMW_EINVAL
    assert lib.qamw_sigma_from_partial_sums(FAKE, 1, 8, 0, FAKE, None) == QAMW_EINVAL
    assert lib.qamw_calibrate_partial_sums(FAKE, 1, 8, 256, 256, None, 0.5, 128, 1, None, FAKE, 1 << 30, None,
                                           None) == QAMW_ENULL
    assert lib.qamw_calibrate_partial_sums(FAKE, 1, 8, 256, 256, None, 0.5, 128, 1, FAKE, None, 0, None,
                                           None) == QAMW_EWORKSPACE


def test_encode_prepared_rejects_on_host(lib):
    def call(**kw):
        a = dict(W=FAKE, wt=1, M=8, K=256, ldw=256, s=FAKE, r=FAKE, block=128, seed=1, sigma=FAKE, cb=FAKE,
                 N=256, bits=8, table=None, packed=FAKE, status=None, stream=None)
        a.update(kw)
        return lib.qamw_encode_prepared(a["W"], a["wt"], a["M"], a["K"], a["ldw"], a["s"], a["r"], a["block"],
                                        a["seed"], a["sigma"], a["cb"], a["N"], a["bits"], a["table"],
                                        a["packed"], a["status"], a["stream"])
    for kw in (dict(W=None), dict(s=None), dict(r=None), dict(sigma=None), dict(cb=None), dict(packed=None)):
        assert call(**kw) == QAMW_ENULL
    for kw in (dict(K=255, ldw=255), dict(block=96), dict(ldw=128), dict(bits=0), dict(N=257), dict(wt=7),
               dict(table=ctypes.c_void_p(0x10008))):
        assert call(**kw) == QAMW_EINVAL
    assert call(N=16384, bits=16) == QAMW_EUNSUPPORTED


def test_decode_matmul_rejects_on_host(lib):
    ws = lib.qamw_decode_matmul_workspace_bytes(128, 256, 16)
    assert ws >= 16 * 256 * 2 + 16 * 4 and ws % 256 == 0
    assert lib.qamw_decode_matmul_workspace_bytes(128, 256, 0) == 0
    assert lib.qamw_decode_matmul_workspace_bytes(0, 256, 16) == 0
    assert lib.qamw_decode_matmul_workspace_bytes(128, 256, (1 << 24) + 1) == 0

    def call(**kw):
        a = dict(packed=FAKE, r=FAKE, sigma=FAKE, s=None, M=128, K=256, block=128, seed=1, cb=FAKE, N=2048,
                 bits=11, X=FAKE, T=16, ldx=256, Y=FAKE, ldy=128, ws=FAKE, nws=ws, status=None, stream=None)
        a.update(kw)
        return lib.qamw_decode_matmul(a["packed"], a["r"], a["sigma"], a["s"], a["M"], a["K"], a["block"],
                                      a["seed"], a["cb"], a["N"], a["bits"], a["X"], a["T"], a["ldx"], a["Y"],
                                      a["ldy"], a["ws"], a["nws"], a["status"], a["stream"])
    for kw in (dict(packed=None), dict(r=None), dict(sigma=None), dict(cb=None), dict(X=None), dict(Y=None),
               dict(ws=None)):
        assert call(**kw) == QAMW_ENULL
    for kw in (dict(T=0), dict(T=(1 << 24) + 1), dict(ldx=255), dict(ldy=127), dict(X=ctypes.c_void_p(0x10008)), dict(ldx=260),
               dict(packed=ctypes.c_void_p(0x10004)), dict(sigma=ctypes.c_void_p(0x10008)),
               dict(ws=ctypes.c_void_p(0x10080)), dict(nws=ws - 1),
               dict(block=96), dict(N=2049)):
        assert call(**kw) == QAMW_EINVAL
    assert call(K=384 - 128 + 64, ldx=384) == QAMW_EINVAL               # K = 320: not a multiple of the block
    assert call(K=192, block=64, ldx=192) == QAMW_EUNSUPPORTED          # K not a multiple of 128
    big = lib.qamw_decode_matmul_workspace_bytes(128, 32768 + 128, 16)
    assert call(K=32768 + 128, ldx=32768 + 128, nws=big) == QAMW_EUNSUPPORTED
