"""The fused decode + matmul (qamw_decode_matmul) against the oracle.

QAM-W page, Methodology (6) Decoding and "Significance and Claims". The
expected value is the oracle's decode (oracle.codec.decode_with_scale, fp64)
multiplied with the exact bf16 activations in fp64: Y_ref = X W_hat^T.

The kernel applies the decode's linear steps to the activations instead
(a_t = sigma (.) H_b (d (.) x_t / s) / sqrt(b), fp32, then fp16 with a
power-of-two factor per token) and multiplies them with the fp16 centroids
on the tensor cores (fp32 accumulation), then scales by r_m. Derived bound,
element by element, with c_mi = C[idx(m, i/2)][i % 2] and a the exact
(fp64) rotated activations:
  S = r_m sum_i |a_ti c_mi|                      two fp16 roundings per product: 2^-11 each,
                                                 and the fp32 roundings of a (2^-24 each);
                                                 fp32 accumulation of K products: K 2^-22 (generous);
  Q = r_m sum_i sigma_i |c_mi| sum_{j in block(i)} |x_tj / s_j| / sqrt(b)
                                                 the fp32 butterflies (log2 b + 2 roundings <= 2^-19 / 2^-24);
  fp16 subnormals: a below 2^-14 of the token's scale rounds to 2^-25 of it
  (2^e_t <= 2^-12 max|a_t|), a centroid below 2^-14 to 2^-25 absolute;
  the final products by r_m and 2^e_t: 2^-23 |Y|.
  |Y - Y_ref| <= (2^-10 + 2^-18 + K 2^-22) S + 2^-19 Q
                 + r_m (2^-36 max|a_t| sum_i |c_mi| + 2^-24 sum_i |a_ti|) + 2^-22 |Y_ref|.
Besides the bound, the error must be well below that of the pages' own
pipeline, which rounds every decoded weight to bf16 (2^-8) before the
matmul: its RMS is checked to be under half of it."""
import numpy as np
import pytest
import torch

import synth
import vector_codebook_codec_b200 as qamw
from oracle import codec

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built(lib):
    return lib


def _codebook(N, seed):
    if N == 8192:   # no shipped codebook of this size: any fp32 point set decodes the same way
        return synth.gaussian_points(N, seed).astype(np.float32)
    return qamw.load_codebook(N)


def _case(M, K, T, block, N, bits, seed, with_scale=True):
    idx = synth.make_indices(M, K // 2, N, seed)
    r = synth.make_row_norms(M, seed)
    sig = synth.make_sigma(K // 2, seed)
    s = synth.make_act_rms(K, 0.5, seed) if with_scale else None
    C = _codebook(N, seed)
    X32 = synth.make_activations(T, K, seed)
    if T >= 3:   # a zero token, a very large and a very small one (the per-token power of two)
        X32[0] = 0.0
        X32[1] *= 1.0e4
        X32[2] *= 1.0e-4
    Xb = torch.from_numpy(X32).to(torch.bfloat16)
    packed = codec.pack_indices(idx, bits)
    enc = qamw.Encoded(torch.from_numpy(packed.view(np.int32)).cuda(), torch.from_numpy(r).cuda(),
                       None if s is None else torch.from_numpy(s).cuda(), torch.from_numpy(sig).cuda(),
                       M, K, block, seed, N, bits)
    return enc, torch.from_numpy(C).cuda(), Xb, idx, r, sig, s, C


def _bound(X64, idx, r, sig, s, C, K, block, seed, rows):
    """The derived bound for the outputs of `rows` (every token)."""
    d = codec.sign_mask(seed, K)
    s64 = np.ones(K) if s is None else s.astype(np.float64)
    sig64 = np.repeat(sig.astype(np.float64), 2)                       # sigma of column i = sigma_{i/2}
    A = codec.rotate_fwd(X64 / s64[None, :], d, block) * sig64[None, :]  # exact a_t (fp64)
    T = X64.shape[0]
    blk = (np.abs(X64 / s64[None, :]).reshape(T, K // block, block).sum(axis=2) / np.sqrt(block))
    Qcol = np.repeat(blk, block, axis=1) * sig64[None, :]
    Cm = np.abs(C.astype(np.float64)[idx[rows]].reshape(len(rows), K))   # |c_mi|
    rr = r[rows].astype(np.float64)[None, :]
    S = (np.abs(A) @ Cm.T) * rr
    Q = (Qcol @ Cm.T) * rr
    amax = np.abs(A).max(axis=1)[:, None]
    small = rr * (2.0 ** -36 * amax * Cm.sum(axis=1)[None, :] + 2.0 ** -24 * np.abs(A).sum(axis=1)[:, None])
    return (2.0 ** -10 + 2.0 ** -18 + K * 2.0 ** -22) * S + 2.0 ** -19 * Q + small


def _check(M, K, T, block, N, bits, seed, with_scale=True):
    enc, Cd, Xb, idx, r, sig, s, C = _case(M, K, T, block, N, bits, seed, with_scale)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    Y = qamw.decode_matmul(enc, Cd, Xb.cuda(), status=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    Y = Y.cpu().numpy().astype(np.float64)
    Wh = codec.decode_with_scale(idx, r, sig, s, K, block, seed, C)              # fp64 [M, K]
    X64 = Xb.to(torch.float64).numpy()
    ref = X64 @ Wh.T
    bound = _bound(X64, idx, r, sig, s, C, K, block, seed, np.arange(M)) + 2.0 ** -22 * np.abs(ref) + 1e-30
    err = np.abs(Y - ref)
    assert np.all(err <= bound), float(np.max(err / bound))
    # the pages' pipeline: every decoded weight rounded to bf16, exact product
    Wb = torch.from_numpy(Wh).to(torch.bfloat16).to(torch.float64).numpy()
    err_bf16 = X64 @ Wb.T - ref
    live = np.abs(X64).sum(axis=1) > 0
    assert np.sqrt(np.mean(err[live] ** 2)) <= 0.5 * np.sqrt(np.mean(err_bf16[live] ** 2))
    if T >= 3:
        assert np.all(Y[0] == 0.0)
    return Y


@pytest.mark.parametrize("M,K,T,block,N,bits", [
    (128, 128, 16, 128, 2048, 11),      # one tile, one chunk; 88-byte rows: words by cp.async
    (256, 512, 40, 128, 2048, 11),      # two row tiles, four chunks (TMA words), a partial token tile (40 of 48)
    (256, 1024, 100, 128, 2048, 11),    # a 112-token tile: one MMA warp, two accumulators of 128 columns
    (200, 256, 1, 64, 256, 8),          # ragged rows (TMA zero fill), one token, b = 64
    (200, 384, 5, 128, 2048, 11),       # ragged rows with the cp.async words (3 x 88-byte chunks per row)
    (128, 384, 256, 32, 1024, 10),      # a full 256-token tile, b = 32
    (384, 1024, 300, 128, 2048, 11),    # two token tiles
    (128, 256, 8, 2, 16, 4),            # b = 2, a 16-centroid codebook, the run-time code size
    (128, 1024, 16, 1024, 256, 8),      # b = 1024: butterflies through shared memory
    (256, 1024, 24, 512, 2048, 11),     # b = 512: all shuffle stages
    (128, 256, 16, 128, 8192, 13),      # 8192 centroids (32 KB of fp16 pairs)
])
def test_fused_decode_matmul_matches_the_oracle(M, K, T, block, N, bits):
    _check(M, K, T, block, N, bits, seed=M + K + T)


def test_fused_decode_matmul_many_tokens():
    """600 tokens: the activation kernel runs one CTA per token (from 512 on)
    and the output has three 256-token tiles, the last one ragged."""
    _check(256, 512, 600, 128, 2048, 11, seed=21)


def test_fused_decode_matmul_single_row_and_strided_operands():
    """M = 1 (one row tile, 127 rows past M) and activations / outputs with
    leading dimensions larger than K / M."""
    M, K, T = 1, 256, 5
    enc, Cd, Xb, idx, r, sig, s, C = _case(M, K, T, 128, 2048, 11, seed=31)
    Xpad = torch.zeros((T, K + 64), dtype=torch.bfloat16)
    Xpad[:, :K] = Xb
    Xs = Xpad.cuda()[:, :K]                       # ldx = K + 64
    Ypad = torch.full((T, M + 7), -7.0, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    qamw.decode_matmul(enc, Cd, Xs, status=st, out=Ypad[:, :M])
    torch.cuda.synchronize()
    assert st.item() == 0
    assert torch.all(Ypad[:, M:] == -7.0)          # nothing written past M
    Y = Ypad[:, :M].cpu().numpy().astype(np.float64)
    Wh = codec.decode_with_scale(idx, r, sig, s, K, 128, 31, C)
    X64 = Xb.to(torch.float64).numpy()
    ref = X64 @ Wh.T
    bound = _bound(X64, idx, r, sig, s, C, K, 128, 31, np.arange(M)) + 2.0 ** -22 * np.abs(ref) + 1e-30
    assert np.all(np.abs(Y - ref) <= bound)


def test_fused_decode_matmul_without_channel_scale():
    _check(256, 512, 16, 128, 2048, 11, seed=3, with_scale=False)


def test_fused_decode_matmul_13b_shape_sampled_rows():
    """5120 x 5120 at 1 and 48 tokens: the oracle bound on every output of 48
    sampled rows, and every output against the unfused path (qamw_decode to
    bf16, then a float32-accumulated matmul on the GPU) within the sum of the
    two paths' bounds."""
    M = K = 5120
    for T in (1, 48):
        enc, Cd, Xb, idx, r, sig, s, C = _case(M, K, T, 128, 2048, 11, seed=77 + T)
        Y = qamw.decode_matmul(enc, Cd, Xb.cuda()).cpu().numpy().astype(np.float64)
        Wbd = qamw.decode(enc, Cd, out_dtype=torch.bfloat16)
        Yu = (Xb.cuda().float() @ Wbd.float().T).cpu().numpy().astype(np.float64)
        X64 = Xb.to(torch.float64).numpy()
        rows = np.random.default_rng(T).choice(M, 48, replace=False)
        Wh = codec.decode_with_scale(idx[rows], r[rows], sig, s, K, 128, 77 + T, C)
        ref = X64 @ Wh.T
        bound = _bound(X64, idx, r, sig, s, C, K, 128, 77 + T, rows) + 2.0 ** -22 * np.abs(ref)
        assert np.all(np.abs(Y[:, rows] - ref) <= bound)
        for r0 in range(0, M, 1024):
            rs = np.arange(r0, min(M, r0 + 1024))
            bf = _bound(X64, idx, r, sig, s, C, K, 128, 77 + T, rs)
            Wb = Wbd[r0:r0 + len(rs)].float().cpu().numpy().astype(np.float64)
            bu = (2.0 ** -8 + K * 2.0 ** -22) * (np.abs(X64) @ np.abs(Wb).T) * (1 + 2.0 ** -7)
            assert np.all(np.abs(Y[:, rs] - Yu[:, rs]) <= bf + bu + 2.0 ** -21 * np.abs(Yu[:, rs]) + 1e-30)


def test_fused_decode_matmul_reports_bad_indices():
    M, K, T = 128, 256, 16
    enc, Cd, Xb, idx, r, sig, s, C = _case(M, K, T, 128, 256, 11, seed=5)   # 11-bit fields, 256 centroids
    bad = idx.copy()
    bad[3, 7] = 2000
    enc.packed.copy_(torch.from_numpy(codec.pack_indices(bad, 11).view(np.int32)).cuda())
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    qamw.decode_matmul(enc, Cd, Xb.cuda(), status=st)
    torch.cuda.synchronize()
    assert st.item() & qamw.STATUS_BAD_INDEX


def test_fused_decode_matmul_reuses_a_caller_workspace():
    """The same call with a caller-owned workspace (and again, reused) gives
    the same bits as with one allocated by the binding."""
    enc, Cd, Xb, *_ = _case(256, 512, 33, 128, 2048, 11, seed=9)
    X = Xb.cuda()
    Y0 = qamw.decode_matmul(enc, Cd, X)
    ws = torch.empty(qamw.decode_matmul_workspace_bytes(256, 512, 33), dtype=torch.uint8, device="cuda")
    Y1 = qamw.decode_matmul(enc, Cd, X, workspace=ws)
    Y2 = qamw.decode_matmul(enc, Cd, X, workspace=ws)
    assert torch.equal(Y0, Y1) and torch.equal(Y1, Y2)


def test_fused_decode_matmul_codebook_at_a_4_byte_offset():
    """A codebook that starts 4 bytes past an 8-byte boundary: the kernel fills
    its table with 4-byte loads instead of the 8-byte ones (same values)."""
    M, K, T, block, N, bits, seed = 256, 512, 16, 128, 2048, 11, 27
    enc, Cd, Xb, *_ = _case(M, K, T, block, N, bits, seed)
    buf = torch.zeros(2 * N + 1, dtype=torch.float32, device="cuda")
    buf[1:] = Cd.reshape(-1)
    C_off = buf[1:].view(N, 2)
    assert C_off.data_ptr() % 8 == 4
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    Y_aligned = qamw.decode_matmul(enc, Cd, Xb.cuda(), status=st)
    Y_off = qamw.decode_matmul(enc, C_off, Xb.cuda(), status=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    assert torch.equal(Y_aligned, Y_off)
