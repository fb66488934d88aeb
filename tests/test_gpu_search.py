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


IMAGE_OFFSET = 64


def _read_table(table):
    """Header fields and every cell's list (offsets/cand, concatenated in cell
    order) decoded from the table's records and overflow lists."""
    raw = table.cpu().numpy()
    hdr = raw[:48].view(np.int32)
    magic, N, G, total, valid, cap = (int(hdr[0]) & 0xFFFFFFFF, int(hdr[1]), int(hdr[2]), int(hdr[3]),
                                      int(hdr[4]), int(hdr[5]))
    a, UL, inv, L = raw[24:40].view(np.float32)
    rec = raw[IMAGE_OFFSET:IMAGE_OFFSET + 8 * G * G].view(np.uint64)
    ovf = raw[IMAGE_OFFSET + 8 * G * G:].view(np.uint16).astype(np.int64)
    e = np.stack([(rec >> np.uint64(16 * f)) & np.uint64(0xFFFF) for f in range(3)], axis=1).astype(np.int64)
    meta = (rec >> np.uint64(48)).astype(np.int64)
    n = meta & 3
    lists = []
    for c in range(G * G):
        if n[c] > 0:
            lists.append(e[c, :n[c]])
        else:
            o = meta[c] >> 2
            lists.append(np.concatenate([e[c], ovf[o + 1:o + 1 + ovf[o]]]))
    lens = np.array([x.size for x in lists], dtype=np.int64)
    offsets = np.concatenate([[0], np.cumsum(lens)])
    cand = np.concatenate(lists)
    return dict(magic=magic, N=N, G=G, total=total, valid=valid, capacity=cap, a=np.float32(a),
                UL=np.float32(UL), inv=np.float32(inv), L=float(L), offsets=offsets, cand=cand, records=rec,
                n_inline=n)


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
    assert off[0] == 0 and np.all(np.diff(off) >= 1) and t["total"] <= t["capacity"]
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


def test_pruned_full_size_projection_equals_brute_force():
    """Whole 4096x4096 projection: pruned and brute-force packed streams are
    identical (test_gpu_fullsize compares every pair with the oracle)."""
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


@pytest.mark.parametrize("N", [16, 128, 256, 1024, 2048])
def test_cells_the_encode_computes_list_the_nearest_centroid(N):
    """The encode's own cell arithmetic (qamw_search_cells runs its device
    function): for points on and within 1e-4 cells of every kind of cell edge,
    the cell the encode looks in lists the oracle's nearest centroid; and that
    cell is the exact cell (fp64) or, within 1e-3 cells of an edge, a
    neighbour whose enlarged bounds contain the point."""
    C = qamw.load_codebook(N)
    Cd = torch.from_numpy(C).cuda()
    table = qamw.build_search_table(Cd)
    t = _read_table(table)
    G, off, cand = t["G"], t["offsets"], t["cand"]
    assert G % 2 == 1
    a, UL, inv = float(t["a"]), float(t["UL"]), float(t["inv"])
    rng = np.random.default_rng(1000 + N)
    n = 200000
    k = rng.integers(0, G + 1, size=(n, 2)).astype(np.float64)
    jitter = np.where(rng.random((n, 2)) < 0.2, 0.0, rng.uniform(-1e-4, 1e-4, size=(n, 2)))
    u = np.clip((k + jitter) / inv - UL, -0.9999, 0.9999)
    pts = (a * u / (1.0 - np.abs(u))).astype(np.float32)
    pts = np.concatenate([pts, rng.standard_normal((n, 2)).astype(np.float32)])
    cells = qamw.search_cells(torch.from_numpy(pts).cuda(), table).cpu().numpy().astype(np.int64)
    inside = cells >= 0
    assert inside.mean() > 0.9
    # exact (fp64) cell coordinates; the encode's must agree up to 1e-3 cells
    p64 = pts.astype(np.float64)
    f = (p64 / (a + np.abs(p64)) + UL) * inv
    cx, cy = cells % G, cells // G
    for c, ff in ((cx, f[:, 0]), (cy, f[:, 1])):
        sel = inside
        assert np.all((ff[sel] >= c[sel] - 1e-3) & (ff[sel] <= c[sel] + 1 + 1e-3))
    idx, _ = codec.nearest_centroid_kd(pts[inside], C)
    for c, i in zip(cells[inside], idx):
        assert i in cand[off[c]:off[c + 1]]
    # points beyond the grid, huge and non-finite ones are off the grid
    far = np.array([[t["L"] * 1.01, 0], [0, -t["L"] * 1.01], [1e38, 0], [3e38, -3e38], [np.nan, 0],
                    [np.inf, 1]], np.float32)
    assert np.all(qamw.search_cells(torch.from_numpy(far).cuda(), table).cpu().numpy() == -1)


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
    assert off[-1] <= 0.8 * first_total, (off[-1], first_total)


def test_records_hold_short_lists_inline():
    """The table layout: a list of one to three entries sits in its cell's
    record (unused fields repeat the first entry); longer lists keep their
    first three entries inline and the rest, counted, in the overflow array,
    which holds nothing else."""
    C = qamw.load_codebook(2048)
    t = _read_table(qamw.build_search_table(torch.from_numpy(C).cuda()))
    n, rec = t["n_inline"], t["records"]
    off, cand = t["offsets"], t["cand"]
    lens = np.diff(off)
    assert np.array_equal(np.where(n > 0, n, 0), np.where(lens <= 3, lens, 0))
    e0 = (rec & np.uint64(0xFFFF)).astype(np.int64)
    for f in (1, 2):
        ef = ((rec >> np.uint64(16 * f)) & np.uint64(0xFFFF)).astype(np.int64)
        short = (lens >= 1) & (lens <= f)
        assert np.array_equal(ef[short], e0[short])
    long_ = lens > 3
    assert t["total"] == int(np.sum(lens[long_] - 3 + 1))
    # most pairs of the unit circular Gaussian fall in cells of at most three entries
    G, a, UL, inv = t["G"], float(t["a"]), float(t["UL"]), float(t["inv"])
    x = np.random.default_rng(5).standard_normal((200000, 2))
    f = np.floor((x / (a + np.abs(x)) + UL) * inv).astype(np.int64)
    assert np.mean(lens[f[:, 1] * G + f[:, 0]] <= 3) > 0.9
