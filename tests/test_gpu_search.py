"""The exact pruned nearest-centroid search (search table + encode).

The table must list, for every grid cell, each centroid that can be nearest
to a point of the cell; with it, qamw_encode must return bit-identical packed
streams to the brute-force search (and so the same parity with the oracle)."""
import numpy as np
import pytest
import torch

import synth
import vector_codebook_codec_b200 as qamw
from oracle import codec
from parity_utils import gpu_codec, index_parity, oracle_encode_rows, to_gpu_matrix

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built(lib):
    return lib


HEADER_BYTES = 48


def _read_table(table):
    raw = table.cpu().numpy()
    hdr = raw[:HEADER_BYTES].view(np.int32)
    magic, N, G, total, valid, cap = (int(hdr[0]) & 0xFFFFFFFF, int(hdr[1]), int(hdr[2]), int(hdr[3]),
                                      int(hdr[4]), int(hdr[5]))
    a, UL, inv, L = raw[24:40].view(np.float32)
    offsets = raw[HEADER_BYTES:HEADER_BYTES + 4 * (G * G + 1)].view(np.uint32).astype(np.int64)
    cand = raw[HEADER_BYTES + 4 * (G * G + 1):].view(np.uint16)[:total].astype(np.int64)
    return dict(magic=magic, N=N, G=G, total=total, valid=valid, capacity=cap, a=np.float32(a),
                UL=np.float32(UL), inv=np.float32(inv), L=float(L), offsets=offsets, cand=cand)


def _cell_coord(x, t):
    """The encode's fp32 cell coordinate: (x / (a + |x|) + UL) * inv_cw."""
    x = x.astype(np.float32)
    u = (x / (t["a"] + np.abs(x))).astype(np.float32)
    return ((u + t["UL"]).astype(np.float32) * t["inv"]).astype(np.float32)


@pytest.mark.parametrize("N", [4, 16, 128, 256, 1024, 2048])
def test_table_lists_the_nearest_centroid_of_every_point(N):
    C = qamw.load_codebook(N)
    t = _read_table(qamw.build_search_table(torch.from_numpy(C).cuda()))
    assert t["valid"] == 1 and t["N"] == N
    G, L, off, cand = t["G"], t["L"], t["offsets"], t["cand"]
    assert L > np.abs(C).max()
    assert off[0] == 0 and off[-1] == t["total"] and np.all(np.diff(off) >= 1)
    for k in range(G * G):
        lst = cand[off[k]:off[k + 1]]
        assert np.all(np.diff(lst) > 0) and lst.max() < N
    # random points: a Gaussian cloud, a uniform spread over [-L, L]^2, and
    # points within 1e-4 cells of a cell edge (edges mapped back to x)
    rng = np.random.default_rng(N)
    a, UL, inv = float(t["a"]), float(t["UL"]), float(t["inv"])
    edge_u = rng.integers(0, G + 1, size=(100000, 2)) / inv - UL
    edge_u = edge_u + rng.uniform(-1e-4, 1e-4, size=edge_u.shape) / inv
    edge_u = np.clip(edge_u, -0.999, 0.999)
    edge_x = a * edge_u / (1.0 - np.abs(edge_u))
    pts = np.concatenate([rng.standard_normal((100000, 2)), rng.uniform(-L, L, size=(100000, 2)),
                          edge_x]).astype(np.float32)
    fx, fy = _cell_coord(pts[:, 0], t), _cell_coord(pts[:, 1], t)
    inside = (fx >= 0) & (fx < G) & (fy >= 0) & (fy < G)
    assert inside.mean() > 0.9
    cell = fy[inside].astype(np.int64) * G + fx[inside].astype(np.int64)
    idx, _ = codec.nearest_centroid(pts[inside], C)
    for c, i in zip(cell, idx):
        assert i in cand[off[c]:off[c + 1]]


CASES = [
    # M, K, block, N, bits, dtype
    (64, 4096, 128, 2048, 11, "bf16"),
    (40, 1024, 64, 256, 8, "f32"),
    (33, 2048, 256, 1024, 10, "bf16"),
    (9, 96, 32, 16, 4, "f32"),
    (5, 24, 8, 4, 2, "f32"),
    (17, 1536, 512, 128, 7, "bf16"),
    (6, 2048, 1024, 256, 8, "bf16"),     # b = 1024: the table is not used (brute-force kernel)
    (300, 1000, 8, 1024, 10, "bf16"),    # K not a multiple of 16: a lane partly past K
    (20, 1004, 4, 256, 8, "bf16"),       # rows not 16-byte aligned: scalar loads
]


@pytest.mark.parametrize("M,K,b,N,bits,dtype", CASES)
def test_pruned_equals_brute_force(M, K, b, N, bits, dtype):
    rng = np.random.default_rng(M + K)
    w32 = (rng.standard_normal((M, K)) * 0.02).astype(np.float32)
    w32[1, :] *= 50.0                            # a loud row
    w32[2, ::7] = 0.5                            # structured row: large normalised pairs
    act = np.exp(rng.standard_normal(K)).astype(np.float32)
    Wd, W = to_gpu_matrix(w32, dtype)
    C = qamw.load_codebook(N)
    Cd = torch.from_numpy(C).cuda()
    actd = torch.from_numpy(act).cuda()
    sig = qamw.calibrate_sigma(Wd, actd, 0.5, b, 7)
    table = qamw.build_search_table(Cd)
    e_brute = qamw.encode(Wd, actd, 0.5, b, 7, sig, Cd, bits)
    e_pruned = qamw.encode(Wd, actd, 0.5, b, 7, sig, Cd, bits, search_table=table)
    torch.cuda.synchronize()
    assert torch.equal(e_brute.packed, e_pruned.packed)
    # and against the oracle
    sig_o = codec.calibrate_sigma(W, act, 0.5, b, 7)
    enc = codec.encode(W, act, 0.5, b, 7, sig_o, C, bits)
    hard, _ = index_parity(e_pruned.packed.cpu().numpy().view(np.uint32), enc["idx"], enc["gap"], bits)
    assert hard == 0


def test_pruned_outside_grid_points():
    """sigma far too small makes |x| huge: every pair leaves the grid and takes
    the brute-force path; results must still equal the brute-force encode."""
    rng = np.random.default_rng(3)
    W = torch.from_numpy((rng.standard_normal((8, 256)) * 0.02).astype(np.float32)).cuda()
    C = torch.from_numpy(qamw.load_codebook(256)).cuda()
    sig = torch.full((128,), 1e-4, device="cuda")
    table = qamw.build_search_table(C)
    a = qamw.encode(W, None, 0.0, 64, 1, sig, C, 8)
    b = qamw.encode(W, None, 0.0, 64, 1, sig, C, 8, search_table=table)
    torch.cuda.synchronize()
    assert torch.equal(a.packed, b.packed)


def test_pruned_full_size_projection_matches_oracle():
    spec = synth.llama7b_attn().specs[0]
    w32 = synth.make_matrix(spec)
    act = synth.act_for(spec)
    Wd, W = to_gpu_matrix(w32, spec.dtype)
    C = qamw.load_codebook(spec.N)
    Cd = torch.from_numpy(C).cuda()
    actd = torch.from_numpy(act).cuda()
    sig = qamw.calibrate_sigma(Wd, actd, spec.alpha, spec.block, spec.seed)
    table = qamw.build_search_table(Cd)
    e_brute = qamw.encode(Wd, actd, spec.alpha, spec.block, spec.seed, sig, Cd, spec.bits)
    e_pruned = qamw.encode(Wd, actd, spec.alpha, spec.block, spec.seed, sig, Cd, spec.bits, search_table=table)
    torch.cuda.synchronize()
    assert torch.equal(e_brute.packed, e_pruned.packed)
    sig_o = codec.calibrate_sigma(W, act, spec.alpha, spec.block, spec.seed)
    rows = np.array([0, 1, 2047, spec.M - 1])
    idx, gap, _, _ = oracle_encode_rows(W, act, spec.alpha, spec.block, spec.seed, sig_o, C, rows)
    hard, _ = index_parity(e_pruned.packed.cpu().numpy().view(np.uint32)[rows], idx, gap, spec.bits)
    assert hard == 0


def test_lists_are_pruned_subsets_of_the_first_test():
    """The second (corner-dominance) test only removes centroids: every cell's
    list is inside the first-test list (recomputed here in numpy with a
    slightly larger slack, so fp64 contraction differences cannot matter), and
    on the shipped N = 2048 codebook it removes at least a fifth of the
    entries (about a third in practice)."""
    N = 2048
    C = qamw.load_codebook(N).astype(np.float64)
    t = _read_table(qamw.build_search_table(torch.from_numpy(C.astype(np.float32)).cuda()))
    G, off, cand = t["G"], t["offsets"], t["cand"]
    a, UL, inv = float(t["a"]), float(t["UL"]), float(t["inv"])
    cw = 1.0 / inv
    k = np.arange(G)
    lo_u, hi_u = k * cw - UL - 1e-3 * cw, (k + 1) * cw - UL + 1e-3 * cw
    lo, hi = a * lo_u / (1 - np.abs(lo_u)), a * hi_u / (1 - np.abs(hi_u))
    lo, hi = lo - 1e-12 * np.abs(lo), hi + 1e-12 * np.abs(hi)
    cx, cy = C[:, 0], C[:, 1]
    ax = np.maximum(np.abs(cx[None] - lo[:, None]), np.abs(cx[None] - hi[:, None]))      # [G, N]
    ay = np.maximum(np.abs(cy[None] - lo[:, None]), np.abs(cy[None] - hi[:, None]))
    bx = np.maximum(0, np.maximum(lo[:, None] - cx[None], cx[None] - hi[:, None]))
    by = np.maximum(0, np.maximum(lo[:, None] - cy[None], cy[None] - hi[:, None]))
    first_total = 0
    for iy in range(G):
        bound = (ax ** 2 + ay[iy][None] ** 2).min(axis=1) * (1 + 2e-5)                   # [G]
        inside = (bx ** 2 + by[iy][None] ** 2) <= bound[:, None]                           # [G, N]
        first_total += int(inside.sum())
        for ix in range(G):
            c = iy * G + ix
            lst = cand[off[c]:off[c + 1]]
            assert np.all(inside[ix, lst]), (ix, iy)
    assert t["total"] <= 0.8 * first_total, (t["total"], first_total)
