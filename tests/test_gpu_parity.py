"""GPU parity of libqamw (through the C ABI) against the oracle on small and
ragged shapes: every block size, bit widths 1..16, row counts that leave
partial warps and tasks, zero / one-hot / extreme rows, status bits."""
import math

import numpy as np
import pytest
import torch

import synth
import vector_codebook_codec_b200 as qamw
from oracle import codec
from parity_utils import (DECODE_TOL, bf16_ulp_ok, gpu_codec, index_parity, oracle_encode_rows,
                          row_scaled_error, to_gpu_matrix)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built(lib):
    return lib


def _codebook(N):
    return qamw.load_codebook(N)


# ------------------------------------------------------------------ rotation

@pytest.mark.parametrize("b", [2, 4, 8, 16, 32, 64, 128, 256, 512, 1024])
@pytest.mark.parametrize("inverse", [False, True])
def test_rotation_matches_oracle(b, inverse):
    rng = np.random.default_rng(b)
    M, K = 5, max(2 * b, 1088 if b <= 64 else 2 * b)
    K -= K % b
    U = rng.standard_normal((M, K))
    Y = qamw.rotate_rows(torch.from_numpy(U).cuda(), b, 77, inverse).cpu().numpy()
    d = codec.sign_mask(77, K)
    ref = codec.rotate_inv(U, d, b) if inverse else codec.rotate_fwd(U, d, b)
    assert np.max(np.abs(Y - ref)) <= 1e-13 * np.max(np.abs(ref))


# ------------------------------------------------------------------ scaling

def test_channel_scale_bitexact():
    rng = np.random.default_rng(0)
    act = np.exp(rng.standard_normal(5000) * 1.5).astype(np.float32)
    for alpha in (0.0, 0.25, 0.5, 0.75, 1.0, -0.3):
        got = qamw.channel_scale(torch.from_numpy(act).cuda(), alpha, act.size).cpu().numpy()
        assert np.array_equal(got, codec.channel_scale(act, alpha, act.size))


def test_channel_scale_bad_act_sets_status():
    act = torch.tensor([1.0, 0.0, -2.0, float("nan"), 4.0], device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    s = qamw.channel_scale(act, 0.5, 5, status=st).cpu().numpy()
    assert st.item() & qamw.STATUS_BAD_ACT_RMS
    assert s[0] == 1.0 and s[4] == 2.0 and np.all(s[1:4] == 1.0)


# ------------------------------------------------------------------ encode pipeline

ENC_CASES = [
    # M, K, block, N, bits, dtype, alpha
    (256, 512, 64, 256, 8, "f32", 0.5),     # the small configuration's shape
    (33, 1024, 128, 2048, 11, "bf16", 0.5),
    (3, 256, 256, 1024, 10, "bf16", 0.25),
    (1, 2048, 1024, 128, 7, "f32", 0.75),
    (17, 1536, 512, 16, 4, "bf16", 0.5),    # K not a multiple of 1024: ragged unit
    (9, 96, 32, 16, 5, "f32", 0.5),         # K < 1024, lanes past K
    (5, 24, 8, 4, 2, "f32", 0.0),           # b < 32: lanes hold several blocks
    (7, 10, 2, 4, 3, "bf16", 0.5),          # b = 2, K not a multiple of 32
    (40, 4096, 128, 2048, 12, "bf16", 0.5), # bits > log2 N
]


@pytest.mark.parametrize("search", ["brute", "pruned"])
@pytest.mark.parametrize("M,K,b,N,bits,dtype,alpha", ENC_CASES)
def test_encode_pipeline_parity(M, K, b, N, bits, dtype, alpha, search):
    rng = np.random.default_rng(M * 7 + K)
    w32 = (rng.standard_normal((M, K)) * 0.02).astype(np.float32)
    act = np.exp(rng.standard_normal(K) * 1.0).astype(np.float32)
    Wd, W = to_gpu_matrix(w32, dtype)
    C = _codebook(N)
    seed = 1000 + M
    g = gpu_codec(Wd, act, alpha, b, seed, C, bits, search=search)
    sig = codec.calibrate_sigma(W, act, alpha, b, seed)
    assert np.array_equal(g["sigma"], sig)
    assert g["status"] == 0
    enc = codec.encode(W, act, alpha, b, seed, sig, C, bits)
    assert np.array_equal(g["s"], enc["s"])
    assert np.array_equal(g["r"], enc["r"])
    hard, near = index_parity(g["packed"], enc["idx"], enc["gap"], bits)
    assert hard == 0, f"{hard} index mismatches with gap >= 1e-6 ({near} near ties)"
    # when no index differs the packed words are identical, padding included
    if near == 0:
        assert np.array_equal(g["packed"], enc["packed"])


def test_encode_special_rows():
    """Zero rows, one-hot rows, constant rows and rows at fp32 extremes."""
    M, K, b, N, bits = 8, 256, 128, 256, 8
    W = np.zeros((M, K), np.float32)
    W[1, 5] = 1.0
    W[2, :] = 0.25
    W[3, ::2] = -3.0e38 / 4096
    W[4, 7] = 1e-30
    W[5, :] = np.linspace(-1, 1, K, dtype=np.float32)
    W[6, 100] = -7.0
    W[6, 200] = 2.0 ** -126
    W[7] = np.random.default_rng(1).standard_normal(K).astype(np.float32) * 1e-20
    C = _codebook(N)
    Wd = torch.from_numpy(W).cuda()
    g = gpu_codec(Wd, None, 0.0, b, 5, C, bits, search="pruned")
    sig = codec.calibrate_sigma(W, None, 0.0, b, 5)
    assert np.array_equal(g["sigma"], sig)
    enc = codec.encode(W, None, 0.0, b, 5, sig, C, bits)
    assert np.array_equal(g["r"], enc["r"])
    hard, _ = index_parity(g["packed"], enc["idx"], enc["gap"], bits)
    assert hard == 0
    assert g["status"] == 0


def test_encode_nonfinite_sets_status():
    W = np.ones((4, 128), np.float32)
    W[2, 3] = np.nan
    Wd = torch.from_numpy(W).cuda()
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    sig = torch.ones(64, device="cuda")
    Cd = torch.from_numpy(_codebook(16)).cuda()
    qamw.encode(Wd, None, 0.0, 128, 0, sig, Cd, 4, status=st)
    torch.cuda.synchronize()
    assert st.item() & (qamw.STATUS_NONFINITE_NORM | qamw.STATUS_NONFINITE_INPUT)


def test_encode_is_deterministic():
    rng = np.random.default_rng(9)
    Wd, W = to_gpu_matrix((rng.standard_normal((300, 2048)) * 0.02).astype(np.float32), "bf16")
    act = np.exp(rng.standard_normal(2048)).astype(np.float32)
    C = _codebook(2048)
    a = gpu_codec(Wd, act, 0.5, 128, 3, C, 11)
    b = gpu_codec(Wd, act, 0.5, 128, 3, C, 11)
    assert np.array_equal(a["sigma"], b["sigma"]) and np.array_equal(a["packed"], b["packed"])


def test_strided_input_rows():
    rng = np.random.default_rng(10)
    full = torch.from_numpy((rng.standard_normal((20, 1100)) * 0.02).astype(np.float32)).to(torch.bfloat16).cuda()
    Wd = full[:, :1024]                       # ld = 1100 (not 16-byte aligned rows)
    W = Wd.float().cpu().numpy()
    C = _codebook(256)
    g = gpu_codec(Wd, None, 0.0, 64, 4, C, 8)
    sig = codec.calibrate_sigma(W, None, 0.0, 64, 4)
    assert np.array_equal(g["sigma"], sig)
    enc = codec.encode(W, None, 0.0, 64, 4, sig, C, 8)
    assert index_parity(g["packed"], enc["idx"], enc["gap"], 8)[0] == 0


# ------------------------------------------------------------------ decode

DEC_CASES = [
    # M, K, block, N, bits
    (33, 4096, 128, 2048, 11), (64, 1024, 64, 256, 8), (32, 2048, 256, 1024, 10),
    (17, 2048, 512, 2048, 11), (9, 2048, 1024, 128, 7), (5, 384, 128, 4096, 12),
    (3, 96, 32, 16, 4), (2, 10, 2, 2, 1), (31, 640, 128, 65536 // 8, 16), (4, 24, 8, 32, 5),
    (1, 256, 256, 512, 9), (70, 1152, 64, 64, 6), (35, 3072, 128, 1024, 13),
]


@pytest.mark.parametrize("M,K,b,N,bits", DEC_CASES)
@pytest.mark.parametrize("out", ["f32", "bf16"])
def test_decode_parity_random_streams(M, K, b, N, bits, out):
    seed = M * 31 + K
    idx = synth.make_indices(M, K // 2, N, seed)
    r = synth.make_row_norms(M, seed)
    sig = synth.make_sigma(K // 2, seed)
    s = synth.make_act_rms(K, 0.5, seed)          # any positive stored channel scale
    rng = np.random.default_rng(seed)
    C = (rng.standard_normal((N, 2)) * 1.3).astype(np.float32)
    packed = codec.pack_indices(idx, bits)
    ref = codec.decode_with_scale(idx, r, sig, s, K, b, seed, C)
    enc = qamw.Encoded(torch.from_numpy(packed.view(np.int32)).cuda(), torch.from_numpy(r).cuda(),
                       torch.from_numpy(s).cuda(), torch.from_numpy(sig).cuda(), M, K, b, seed, N, bits)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    dt = torch.float32 if out == "f32" else torch.bfloat16
    got = qamw.decode(enc, torch.from_numpy(C).cuda(), out_dtype=dt, status=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    if out == "f32":
        assert row_scaled_error(got.cpu().numpy(), ref) <= DECODE_TOL
    else:
        assert bf16_ulp_ok(got, ref)


def test_decode_strided_output_and_null_scale():
    M, K, b, N, bits = 10, 512, 128, 256, 8
    idx = synth.make_indices(M, K // 2, N, 3)
    r = synth.make_row_norms(M, 3)
    sig = synth.make_sigma(K // 2, 3)
    C = qamw.load_codebook(N)
    packed = codec.pack_indices(idx, bits)
    ref = codec.decode_with_scale(idx, r, sig, None, K, b, 3, C)
    enc = qamw.Encoded(torch.from_numpy(packed.view(np.int32)).cuda(), torch.from_numpy(r).cuda(), None,
                       torch.from_numpy(sig).cuda(), M, K, b, 3, N, bits)
    big = torch.zeros((M, K + 3), dtype=torch.float32, device="cuda")
    qamw.decode(enc, torch.from_numpy(C).cuda(), out_dtype=torch.float32, out=big[:, 1:K + 1])
    torch.cuda.synchronize()
    got = big.cpu().numpy()
    assert row_scaled_error(got[:, 1:K + 1], ref) <= DECODE_TOL
    assert np.all(got[:, 0] == 0) and np.all(got[:, K + 1:] == 0)


def test_decode_bad_index_and_norm_status():
    M, K, b, N, bits = 4, 256, 128, 100, 8
    idx = synth.make_indices(M, K // 2, N, 5)
    idx[2, 17] = 200                                    # >= N
    r = synth.make_row_norms(M, 5)
    r[3] = np.inf
    sig = synth.make_sigma(K // 2, 5)
    C = np.random.default_rng(5).standard_normal((N, 2)).astype(np.float32)
    enc = qamw.Encoded(torch.from_numpy(codec.pack_indices(idx, bits).view(np.int32)).cuda(),
                       torch.from_numpy(r).cuda(), None, torch.from_numpy(sig).cuda(), M, K, b, 1, N, bits)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    got = qamw.decode(enc, torch.from_numpy(C).cuda(), out_dtype=torch.float32, status=st).cpu().numpy()
    assert st.item() & qamw.STATUS_BAD_INDEX and st.item() & qamw.STATUS_NONFINITE_NORM
    idx0 = idx.copy()
    idx0[2, 17] = 0                                      # decoded as centroid 0
    ref = codec.decode_with_scale(idx0[:3], r[:3], sig, None, K, b, 1, C)
    assert row_scaled_error(got[:3], ref) <= DECODE_TOL


def test_roundtrip_small_configuration():
    """The 256x512 fp32 configuration end to end: GPU calibrate, encode, decode."""
    spec = synth.tiny().specs[0]
    w32 = synth.make_matrix(spec)
    act = synth.act_for(spec)
    Wd, W = to_gpu_matrix(w32, spec.dtype)
    C = _codebook(spec.N)
    g = gpu_codec(Wd, act, spec.alpha, spec.block, spec.seed, C, spec.bits)
    sig = codec.calibrate_sigma(W, act, spec.alpha, spec.block, spec.seed)
    assert np.array_equal(g["sigma"], sig)
    enc = codec.encode(W, act, spec.alpha, spec.block, spec.seed, sig, C, spec.bits)
    hard, near = index_parity(g["packed"], enc["idx"], enc["gap"], spec.bits)
    assert hard == 0
    # decode the oracle's packed stream on the GPU (r, s, sigma are bit-equal)
    ora_enc = qamw.Encoded(torch.from_numpy(enc["packed"].view(np.int32)).cuda(), g["enc"].row_norm,
                           g["enc"].col_scale, g["enc"].sigma, spec.M, spec.K, spec.block, spec.seed,
                           spec.N, spec.bits)
    out = qamw.decode(ora_enc, g["Cd"], out_dtype=torch.float32).cpu().numpy()
    ref = codec.decode(enc["packed"], enc["r"], sig, act, spec.alpha, spec.K, spec.block, spec.seed, C,
                       spec.bits)
    assert row_scaled_error(out, ref) <= DECODE_TOL
