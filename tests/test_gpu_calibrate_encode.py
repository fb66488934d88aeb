"""qamw_calibrate_encode (calibration then encode in one call, s_j and r_i
computed once) against the two separate calls and against the oracle.

The fused call runs the same kernels on the same inputs, so every output must
equal the separate calls' bit for bit; the oracle check then ties the fused
path itself to Methodology (3)-(4): sigma bit-exact, indices exact up to
counted near-ties."""
import numpy as np
import pytest
import torch

import synth
import vector_codebook_codec_b200 as qamw
from oracle import codec
from parity_utils import index_parity, oracle_encode_rows, to_gpu_matrix

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built(lib):
    return lib


def _same_bits(x, y):
    return x.shape == y.shape and torch.equal(x.view(torch.int32), y.view(torch.int32))


def _separate(Wd, act_d, alpha, block, seed, Cd, bits, table):
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    sigma = qamw.calibrate_sigma(Wd, act_d, alpha, block, seed, status=st)
    enc = qamw.encode(Wd, act_d, alpha, block, seed, sigma, Cd, bits, status=st, search_table=table)
    torch.cuda.synchronize()
    return enc, int(st.item())


def _fused(Wd, act_d, alpha, block, seed, Cd, bits, table):
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    enc = qamw.calibrate_encode(Wd, act_d, alpha, block, seed, Cd, bits, status=st, search_table=table)
    torch.cuda.synchronize()
    return enc, int(st.item())


CASES = [
    # (M, K, dtype, block, N, bits, alpha, search)
    (256, 512, "f32", 64, 256, 8, 0.5, "brute"),          # the tiny workload's shape
    (61, 1088, "bf16", 64, 2048, 11, 0.5, "pruned"),      # ragged row tile, 17 blocks, a partial 512-column chunk
    (100, 2048, "bf16", 128, 2048, 11, 0.25, "pruned"),
    (33, 2048, "bf16", 256, 1024, 10, 0.75, "brute"),
    (9, 2048, "f32", 1024, 256, 8, 0.5, "brute"),         # the 1024-column calibration and brute-force encode
    (40, 1536, "bf16", 512, 16, 4, 0.5, "pruned"),
]


@pytest.mark.parametrize("M,K,dt,block,N,bits,alpha,search", CASES)
def test_fused_equals_separate_calls_bitwise(M, K, dt, block, N, bits, alpha, search):
    rng = np.random.default_rng(M * 7 + K)
    W32 = (rng.standard_normal((M, K)) * 0.02).astype(np.float32)
    W32[:, rng.choice(K, size=max(1, K // 200), replace=False)] *= 20.0
    W32[M // 2] = 0.0                                                  # a zero row codes x = 0
    act = np.exp(rng.standard_normal(K)).astype(np.float32)
    Wd, _ = to_gpu_matrix(W32, dt)
    act_d = torch.from_numpy(act).cuda()
    Cd = torch.from_numpy(qamw.load_codebook(N)).cuda()
    table = qamw.build_search_table(Cd) if search == "pruned" else None
    a, sa = _separate(Wd, act_d, alpha, block, 5, Cd, bits, table)
    b, sb = _fused(Wd, act_d, alpha, block, 5, Cd, bits, table)
    assert sa == sb == 0
    for x, y in ((a.sigma, b.sigma), (a.row_norm, b.row_norm), (a.col_scale, b.col_scale), (a.packed, b.packed)):
        assert _same_bits(x, y)
    # the encode kernel alone, given the scales and norms the encode wrote
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    c = qamw.encode_prepared(Wd, a.col_scale, a.row_norm, block, 5, a.sigma, Cd, bits, status=st,
                             search_table=table)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    assert _same_bits(a.packed, c.packed)


def test_fused_matches_the_oracle_on_the_tiny_workload():
    spec = synth.tiny().specs[0]
    W = synth.make_matrix(spec)
    act = synth.act_for(spec)
    N, bits = spec.N, spec.bits
    C = qamw.load_codebook(N)
    Wd, W32 = to_gpu_matrix(W, "f32")
    enc, st = _fused(Wd, torch.from_numpy(act).cuda(), spec.alpha, spec.block, spec.seed,
                     torch.from_numpy(C).cuda(), bits, None)
    assert st == 0
    sigma = codec.calibrate_sigma(W32, act, spec.alpha, spec.block, spec.seed)
    assert np.array_equal(enc.sigma.cpu().numpy(), sigma)
    rows = np.arange(spec.M)
    idx, gap, r, s = oracle_encode_rows(W32, act, spec.alpha, spec.block, spec.seed, sigma, C, rows)
    assert np.array_equal(enc.row_norm.cpu().numpy(), r)
    assert np.array_equal(enc.col_scale.cpu().numpy(), s)
    hard, _near = index_parity(enc.packed.cpu().numpy().view(np.uint32), idx, gap, bits)
    assert hard == 0


def test_fused_reports_bad_input_like_the_separate_calls():
    rng = np.random.default_rng(3)
    W32 = (rng.standard_normal((30, 512)) * 0.02).astype(np.float32)
    W32[7, 3] = np.inf
    act = np.exp(rng.standard_normal(512)).astype(np.float32)
    act[11] = -1.0                                                     # not > 0: status bit, s = 1
    Wd, _ = to_gpu_matrix(W32, "f32")
    act_d = torch.from_numpy(act).cuda()
    Cd = torch.from_numpy(qamw.load_codebook(256)).cuda()
    a, sa = _separate(Wd, act_d, 0.5, 64, 9, Cd, 8, None)
    b, sb = _fused(Wd, act_d, 0.5, 64, 9, Cd, 8, None)
    assert sa == sb and sb & qamw.STATUS_BAD_ACT_RMS and sb & qamw.STATUS_NONFINITE_NORM
    for x, y in ((a.sigma, b.sigma), (a.row_norm, b.row_norm), (a.col_scale, b.col_scale), (a.packed, b.packed)):
        assert _same_bits(x, y)
    # the encode kernel alone reports the non-finite row norm it is given
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    c = qamw.encode_prepared(Wd, a.col_scale, a.row_norm, 64, 9, a.sigma, Cd, 8, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) & qamw.STATUS_NONFINITE_INPUT
    assert _same_bits(a.packed, c.packed)
