"""Lloyd training of the 2D codebook on the GPU (qamw_lloyd_*) against the
oracle's Lloyd iteration (oracle/lloyd.py): exact nearest assignment, cell
means, the same stopping rule, on the same seeded samples."""
import numpy as np
import pytest
import torch

import vector_codebook_codec_b200 as qamw
import synth
from oracle import lloyd

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built(lib):
    return lib


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float64)).cuda()


def _gap_ok(points, C, gpu_idx, ora_idx):
    """Indices differ only where the two nearest centroids are equidistant to
    within fp64 rounding (relative 1e-12)."""
    diff = np.nonzero(gpu_idx != ora_idx)[0]
    for t in diff:
        d = np.sum((C - points[t]) ** 2, axis=1)
        a, b = d[gpu_idx[t]], d[ora_idx[t]]
        assert abs(a - b) <= 1e-12 * max(a, b), (t, a, b)
    return len(diff)


@pytest.mark.parametrize("N", [4, 256, 2048])
def test_assign_is_the_exact_nearest_centroid(N):
    x = synth.gaussian_points(60000, seed=N)
    x[:50] *= 40.0                                   # far-out points
    C = qamw.load_codebook(N).astype(np.float64)
    g = qamw.lloyd_assign(_dev(x), _dev(C)).cpu().numpy()
    o = lloyd.assign(x, C)
    assert _gap_ok(x, C, g, o) == 0


def test_assign_ties_take_the_lowest_index():
    C = np.array([[1.0, 0.0], [1.0, 0.0], [-1.0, 0.0], [0.0, 3.0]])
    x = np.array([[2.0, 0.0], [0.0, 0.0], [0.0, 1.5], [-5.0, 0.0]])
    g = qamw.lloyd_assign(_dev(x), _dev(C)).cpu().numpy()
    # (0,0) is at distance 1 from centroids 0, 1, 2: lowest index 0; (0,1.5) is at
    # distance sqrt(3.25) from 0, 1, 2 and 1.5 from 3
    assert g.tolist() == [0, 0, 3, 2]


def test_assign_counts_changes():
    x = synth.gaussian_points(10000, seed=3)
    C = qamw.load_codebook(16).astype(np.float64)
    idx = torch.zeros(10000, dtype=torch.int32, device="cuda")
    changed = torch.zeros(1, dtype=torch.int64, device="cuda")
    qamw.lloyd_assign(_dev(x), _dev(C), idx=idx, changed=changed)
    o = lloyd.assign(x, C)
    assert int(changed.item()) == int(np.sum(o != 0))
    changed.zero_()
    qamw.lloyd_assign(_dev(x), _dev(C), idx=idx, changed=changed)
    assert int(changed.item()) == 0


def test_update_is_the_cell_mean_and_empty_cells_stay():
    x = synth.gaussian_points(50000, seed=5)
    C = qamw.load_codebook(256).astype(np.float64).copy()
    C[17] = [100.0, -100.0]                          # no sample is nearest: keeps its place
    idx = lloyd.assign(x, C)
    assert not np.any(idx == 17)
    Cg = _dev(C)
    qamw.lloyd_update(_dev(x), torch.from_numpy(idx.astype(np.int32)).cuda(), Cg)
    got = Cg.cpu().numpy()
    ref = lloyd.centroid_update(x, idx, C)
    assert np.array_equal(got[17], C[17])
    assert np.max(np.abs(got - ref)) <= 1e-13


def test_update_is_deterministic():
    x = synth.gaussian_points(300000, seed=6)
    C = qamw.load_codebook(1024).astype(np.float64)
    idx = torch.from_numpy(lloyd.assign(x, C).astype(np.int32)).cuda()
    a, b = _dev(C), _dev(C)
    qamw.lloyd_update(_dev(x), idx, a)
    qamw.lloyd_update(_dev(x), idx, b)
    assert torch.equal(a, b)


def test_train_matches_the_oracle_to_convergence():
    x = synth.gaussian_points(20000, seed=7)
    init = lloyd.best_polar(x, 16).points()
    Co, io, it_o, conv_o = lloyd.lloyd(x, init, max_iter=300)
    Cg, ig, it_g, conv_g = qamw.lloyd_train(_dev(x), _dev(init), max_iter=300)
    assert conv_o and conv_g and it_g == it_o
    assert np.max(np.abs(Cg.cpu().numpy() - Co)) <= 1e-12
    assert np.array_equal(ig.cpu().numpy(), io)


def test_train_stops_at_max_iter():
    x = synth.gaussian_points(1 << 16, seed=8)
    init = lloyd.best_polar(x, 256).points()
    Co, io, it_o, conv_o = lloyd.lloyd(x, init, max_iter=12)
    Cg, ig, it_g, conv_g = qamw.lloyd_train(_dev(x), _dev(init), max_iter=12)
    assert not conv_o and not conv_g and it_o == it_g == 12
    assert np.max(np.abs(Cg.cpu().numpy() - Co)) <= 1e-11
    _gap_ok(x, Co, ig.cpu().numpy(), io)


@pytest.mark.parametrize("N", [16, 256])
def test_retraining_gives_a_lloyd_fixed_point_as_good_as_the_shipped_codebook(N):
    """Re-train with the recipe of the shipped codebook (same samples and start):
    the result is a fixed point of Lloyd's map (centroid and Voronoi conditions
    checked by the oracle) whose distortion equals the shipped codebook's.
    (N = 2048 passes the same checks; its oracle-side start, the best polar code
    of 2^21 samples, takes minutes of CPU, so it is not part of the suite.)"""
    T = max(1024 * N, 1 << 18)
    x = synth.gaussian_points(T, seed=12345 + N)
    init = lloyd.best_polar(x, N).points()
    Cg, ig, it, conv = qamw.lloyd_train(_dev(x), _dev(init), max_iter=4000)
    assert conv
    C = Cg.cpu().numpy()
    idx = lloyd.assign(x, C)
    assert np.array_equal(idx, ig.cpu().numpy())                          # Voronoi condition
    assert np.max(np.abs(lloyd.centroid_update(x, idx, C) - C)) <= 1e-12   # centroid condition
    shipped = qamw.load_codebook(N).astype(np.float64)
    d_gpu, d_ship = lloyd.distortion(x, C), lloyd.distortion(x, shipped)
    assert abs(d_gpu - d_ship) <= 1e-6 * d_ship
