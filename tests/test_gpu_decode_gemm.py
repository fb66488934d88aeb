"""The fused decode + matmul (qamw_decode_matmul) against the oracle.

QAM-W page, Methodology (6) Decoding and "Significance and Claims": the
decoded weights are rounded to BF16 and multiplied with the activations. The
oracle decodes in fp64 (oracle.codec.decode_with_scale); the reference is
X @ W_hat^T in fp64 with X the exact bf16 activations. The kernel rounds each
weight to bf16 (at most one bf16 unit in the last place, 2^-7 relative, from
the exact value: its fp32 decode is within a fraction of a bf16 ulp of the
oracle's) and accumulates in fp32, so for every output
  |Y - Y_ref| <= (2^-7 + K 2^-23) * sum_k |X[t][k]| |W_hat[m][k]|
                 + 1e-5 * max_k |W_hat[m][k]| * sum_k |X[t][k]|
(the last term: the fp32 decode's own error, at most 1e-5 of its row's
largest weight, which a weight far below that scale does not bound
relatively), which is the bound the tests apply element by element. They also compare with
the unfused path (qamw_decode to bf16, then a float32-accumulated matmul of the
same bf16 values), which may differ only by the accumulation order and by the
rare weight whose fp32 decode rounds to the neighbouring bf16 value."""
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


def _case(M, K, T, block, N, bits, seed):
    idx = synth.make_indices(M, K // 2, N, seed)
    r = synth.make_row_norms(M, seed)
    sig = synth.make_sigma(K // 2, seed)
    s = synth.make_act_rms(K, 0.5, seed)
    C = qamw.load_codebook(N)
    X32 = synth.make_activations(T, K, seed)
    Xb = torch.from_numpy(X32).to(torch.bfloat16)
    packed = codec.pack_indices(idx, bits)
    enc = qamw.Encoded(torch.from_numpy(packed.view(np.int32)).cuda(), torch.from_numpy(r).cuda(),
                       torch.from_numpy(s).cuda(), torch.from_numpy(sig).cuda(), M, K, block, seed, N, bits)
    return enc, torch.from_numpy(C).cuda(), Xb, idx, r, sig, s, C


def _check(M, K, T, block, N, bits, seed):
    enc, Cd, Xb, idx, r, sig, s, C = _case(M, K, T, block, N, bits, seed)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    Y = qamw.decode_matmul(enc, Cd, Xb.cuda(), status=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    Wh = codec.decode_with_scale(idx, r, sig, s, K, block, seed, C)              # fp64 [M, K]
    X64 = Xb.to(torch.float64).numpy()
    ref = X64 @ Wh.T
    rowtol = 1e-5 * np.abs(X64).sum(axis=1)[:, None] * np.abs(Wh).max(axis=1)[None, :]
    bound = (2.0 ** -7 + K * 2.0 ** -23) * (np.abs(X64) @ np.abs(Wh).T) + rowtol + 1e-30
    err = np.abs(Y.cpu().numpy().astype(np.float64) - ref)
    assert np.all(err <= bound), float(np.max(err / bound))
    # the unfused path: decode to bf16, then a float32-accumulated matmul
    Wb = qamw.decode(enc, Cd, out_dtype=torch.bfloat16)
    Yu = (Xb.cuda().float() @ Wb.float().T)
    torch.cuda.synchronize()
    du = np.abs(Y.cpu().numpy().astype(np.float64) - Yu.cpu().numpy())
    scale = np.abs(X64) @ np.abs(Wh).T
    assert np.all(du <= (2.0 ** -7 + K * 2.0 ** -22) * scale + rowtol + 1e-30)
    assert np.median(du / np.maximum(scale, 1e-30)) < 1e-6
    return Y


@pytest.mark.parametrize("M,K,T,block,N,bits", [
    (128, 128, 16, 128, 2048, 11),      # one tile, one chunk
    (256, 512, 40, 128, 2048, 11),      # two row tiles, four chunks, a partial token tile (40 of 48)
    (200, 256, 1, 64, 256, 8),          # ragged rows, one token, b = 64
    (128, 384, 256, 32, 1024, 10),      # a full 256-token tile, b = 32
    (384, 1024, 300, 128, 2048, 11),    # two token tiles (256 + 44)
    (128, 256, 8, 2, 16, 4),            # b = 2, a 16-centroid codebook
])
def test_fused_decode_matmul_matches_the_oracle(M, K, T, block, N, bits):
    _check(M, K, T, block, N, bits, seed=M + K + T)


def test_fused_decode_matmul_13b_shape_sampled_rows():
    """5120 x 5120 at 1 and 48 tokens: every output against the unfused path,
    and the oracle bound on every output of 32 sampled rows."""
    M = K = 5120
    for T in (1, 48):
        enc, Cd, Xb, idx, r, sig, s, C = _case(M, K, T, 128, 2048, 11, seed=77 + T)
        Y = qamw.decode_matmul(enc, Cd, Xb.cuda()).cpu().numpy().astype(np.float64)
        Wb = qamw.decode(enc, Cd, out_dtype=torch.bfloat16)
        Yu = (Xb.cuda().float() @ Wb.float().T).cpu().numpy()
        X64 = Xb.to(torch.float64).numpy()
        rows = np.random.default_rng(T).choice(M, 32, replace=False)
        Wh = codec.decode_with_scale(idx[rows], r[rows], sig, s, K, 128, 77 + T, C)
        ref = X64 @ Wh.T
        scale = np.abs(X64) @ np.abs(Wh).T
        rowtol = 1e-5 * np.abs(X64).sum(axis=1)[:, None] * np.abs(Wh).max(axis=1)[None, :]
        assert np.all(np.abs(Y[:, rows] - ref) <= (2.0 ** -7 + K * 2.0 ** -23) * scale + rowtol)
        # all rows against the unfused path (bf16 decode, fp32 matmul)
        sc_all = np.abs(X64) @ np.abs(Wb.float().cpu().numpy().astype(np.float64)).T
        assert np.all(np.abs(Y - Yu) <= (2.0 ** -7 + K * 2.0 ** -22) * sc_all + 1e-30)


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
