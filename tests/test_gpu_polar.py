"""The polar baseline codec on the GPU (qamw_encode_polar + qamw_decode with
the polar points) against the oracle's encode_polar: indices bit-exact except
where a pair lies within 1e-12 of a decision boundary (the two sides take the
amplitude / phase decisions in fp64 with different hypot / atan2 routines),
and the joint codec's lower error at equal rate."""
import numpy as np
import pytest
import torch

import synth
import vector_codebook_codec_b200 as qamw
from oracle import codec
from parity_utils import DECODE_TOL, bf16_ulp_ok, row_scaled_error, to_gpu_matrix

pytestmark = pytest.mark.gpu
MARGIN = 1e-12


@pytest.fixture(scope="module", autouse=True)
def _built(lib):
    return lib


def _gpu_polar(Wd, act, alpha, b, seed, N, bits, sig=None):
    pol = qamw.load_polar(N)
    actd = None if act is None else torch.from_numpy(act).cuda()
    if sig is None:
        sig = qamw.calibrate_sigma(Wd, actd, alpha, b, seed)
    amps = torch.from_numpy(pol["amps"]).cuda()
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    enc = qamw.encode_polar(Wd, actd, alpha, b, seed, sig, amps, pol["P"], bits, status=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    return enc, sig, pol


def _index_check(enc, idx_o, margin, bits):
    P = idx_o.shape[1]
    g = codec.unpack_indices(enc.packed.cpu().numpy().view(np.uint32), P, bits)
    diff = g != idx_o
    assert np.all(margin[diff] < MARGIN), int(np.sum(diff & (margin >= MARGIN)))
    return int(np.sum(diff))


CASES = [
    # M, K, block, N, bits, dtype
    (64, 1024, 128, 2048, 11, "bf16"),
    (33, 512, 64, 256, 8, "f32"),
    (17, 1536, 512, 16, 4, "bf16"),
    (9, 96, 32, 4, 2, "f32"),
]


@pytest.mark.parametrize("M,K,b,N,bits,dtype", CASES)
def test_polar_encode_matches_oracle(M, K, b, N, bits, dtype):
    rng = np.random.default_rng(M + K + N)
    w32 = (rng.standard_normal((M, K)) * 0.02).astype(np.float32)
    act = np.exp(rng.standard_normal(K)).astype(np.float32)
    Wd, W = to_gpu_matrix(w32, dtype)
    enc, sig, pol = _gpu_polar(Wd, act, 0.5, b, 11, N, bits)
    sig_o = codec.calibrate_sigma(W, act, 0.5, b, 11)
    assert np.array_equal(sig.cpu().numpy(), sig_o)
    o = codec.encode_polar(W, act, 0.5, b, 11, sig_o, pol["amps"], pol["P"], bits)
    assert np.array_equal(enc.row_norm.cpu().numpy(), o["r"])
    _index_check(enc, o["idx"], o["margin"], bits)
    # the decode of the polar stream is the joint decode with the polar points
    Cd = torch.from_numpy(pol["points"]).cuda()
    out32 = qamw.decode(enc, Cd, out_dtype=torch.float32).cpu().numpy()
    ref = codec.decode_with_scale(o["idx"], o["r"], sig_o, o["s"], K, b, 11, pol["points"])
    g_idx = codec.unpack_indices(enc.packed.cpu().numpy().view(np.uint32), K // 2, bits)
    if np.array_equal(g_idx, o["idx"]):
        assert row_scaled_error(out32, ref) <= DECODE_TOL


def test_polar_rejects_block_1024():
    W = torch.zeros((2, 1024), dtype=torch.float32, device="cuda")
    with pytest.raises(qamw.QamwError):
        _gpu_polar(W, None, 0.0, 1024, 1, 16, 4, sig=torch.ones(512, device="cuda"))


def test_full_size_joint_beats_polar_at_equal_rate():
    """4096 x 4096 projection at 2048 points (5.5 bits/weight): sampled-row index
    parity with the oracle, and the joint codec's whole-matrix error below the
    polar codec's (the page's "Joint 2D vs. Polar" comparison)."""
    spec = synth.llama7b_attn().specs[0]
    w32 = synth.make_matrix(spec)
    act = synth.act_for(spec)
    Wd, W = to_gpu_matrix(w32, spec.dtype)
    enc, sig, pol = _gpu_polar(Wd, act, spec.alpha, spec.block, spec.seed, spec.N, spec.bits)
    rows = np.array([0, 1, 2047, spec.M - 1])
    o = codec.encode_polar(W[rows], act, spec.alpha, spec.block, spec.seed, sig.cpu().numpy(), pol["amps"],
                           pol["P"], spec.bits)
    g = codec.unpack_indices(enc.packed.cpu().numpy().view(np.uint32)[rows], spec.K // 2, spec.bits)
    assert np.all(o["margin"][g != o["idx"]] < MARGIN)
    C = torch.from_numpy(qamw.load_codebook(spec.N)).cuda()
    table = qamw.build_search_table(C)
    actd = torch.from_numpy(act).cuda()
    joint = qamw.encode(Wd, actd, spec.alpha, spec.block, spec.seed, sig, C, spec.bits, search_table=table)
    wj = qamw.decode(joint, C, out_dtype=torch.float32)
    wp = qamw.decode(enc, torch.from_numpy(pol["points"]).cuda(), out_dtype=torch.float32)
    Wf = Wd.float()
    ej = torch.sum((wj - Wf) ** 2).item()
    ep = torch.sum((wp - Wf) ** 2).item()
    assert ej < ep
