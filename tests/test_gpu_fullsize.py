"""GPU parity at the workloads' full sizes, in the launch configuration the
benchmark uses (the same C-ABI calls on whole matrices).

sigma, row norms and channel scales are compared in full (the oracle's fp64
rotation of a whole matrix takes seconds); indices on sampled rows (always
rows 0 and M-1), since the oracle's brute-force search is slow; decode on
seeded random index streams, in full or on sampled rows (rows are
independent)."""
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


def _sample_rows(M, n, seed):
    rng = np.random.default_rng(seed)
    rows = set([0, M - 1]) | set(rng.choice(M, size=min(n, M), replace=False).tolist())
    return np.array(sorted(rows))


def _check_encode(spec, n_rows=12):
    w32 = synth.make_matrix(spec)
    act = synth.act_for(spec)
    Wd, W = to_gpu_matrix(w32, spec.dtype)
    C = qamw.load_codebook(spec.N)
    g = gpu_codec(Wd, act, spec.alpha, spec.block, spec.seed, C, spec.bits, search="pruned")
    assert g["status"] == 0
    sig = codec.calibrate_sigma(W, act, spec.alpha, spec.block, spec.seed)
    n_sig = int(np.sum(g["sigma"] != sig))
    assert n_sig == 0, f"{n_sig} sigma values differ"
    s = codec.channel_scale(act, spec.alpha, spec.K)
    assert np.array_equal(g["s"], s)
    r = codec.row_norms(codec.scaled_rows(W, s))
    assert np.array_equal(g["r"], r)
    rows = _sample_rows(spec.M, n_rows, spec.seed)
    idx, gap, _, _ = oracle_encode_rows(W, act, spec.alpha, spec.block, spec.seed, sig, C, rows)
    hard, near = index_parity(g["packed"][rows], idx, gap, spec.bits)
    assert hard == 0, f"{hard} index mismatches ({near} near ties)"
    return g, W, sig, C


def test_llama7b_attention_projection():
    spec = synth.llama7b_attn().specs[0]
    g, W, sig, C = _check_encode(spec, n_rows=14)
    # decode of the GPU encoding vs the oracle decode of the same indices is not
    # used (inputs never come from the CUDA path); decode parity below runs on
    # seeded random streams at this shape.
    _check_decode_random(spec.M, spec.K, spec.block, spec.N, spec.bits, spec.seed, rows=None)


@pytest.mark.parametrize("which", [0, 9, 19])
def test_mlp_projection_runs(which):
    spec = synth.mlp_runs().specs[which]
    _check_encode(spec, n_rows=6)


@pytest.mark.parametrize("bits", [7, 8])
def test_rate_variants_on_the_projection(bits):
    """QAM-W at 3.5 and 4 bits per weight (128 and 256 centroids) on the 4096x4096
    projection: encode through the pruned search, and the bf16 decode path of
    7- and 8-bit words."""
    spec = synth.rate_variant(bits).specs[0]
    _check_encode(spec, n_rows=10)
    _check_decode_random(spec.M, spec.K, spec.block, spec.N, spec.bits, spec.seed, rows=_sample_rows(spec.M, 8, 1))


def test_stack_layer0():
    for spec in synth.stack_1p1b(1).specs:
        _check_encode(spec, n_rows=4)


def _check_decode_random(M, K, b, N, bits, seed, rows):
    idx = synth.make_indices(M, K // 2, N, seed)
    r = synth.make_row_norms(M, seed)
    sig = synth.make_sigma(K // 2, seed)
    s = synth.make_act_rms(K, 0.5, seed)
    C = qamw.load_codebook(N)
    packed = codec.pack_indices(idx, bits)
    enc = qamw.Encoded(torch.from_numpy(packed.view(np.int32)).cuda(), torch.from_numpy(r).cuda(),
                       torch.from_numpy(s).cuda(), torch.from_numpy(sig).cuda(), M, K, b, seed, N, bits)
    Cd = torch.from_numpy(C).cuda()
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    out32 = qamw.decode(enc, Cd, out_dtype=torch.float32, status=st)
    out16 = qamw.decode(enc, Cd, out_dtype=torch.bfloat16, status=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    sel = np.arange(M) if rows is None else rows
    ref = codec.decode_with_scale(idx[sel], r[sel], sig, s, K, b, seed, C)
    assert row_scaled_error(out32.cpu().numpy()[sel], ref) <= DECODE_TOL
    assert bf16_ulp_ok(out16[torch.from_numpy(sel).cuda()], ref)


@pytest.mark.parametrize("which", [0, 1, 2])
def test_decode_13b_sweep(which):
    spec = synth.decode_sweep_13b().specs[which]
    rows = _sample_rows(spec.M, 64, spec.seed)
    _check_decode_random(spec.M, spec.K, spec.block, spec.N, spec.bits, spec.seed, rows)
