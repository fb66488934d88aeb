"""Pins of the oracle's polar baseline code (oracle/lloyd.py PolarCode,
oracle/codec.py encode_polar): the index function against the reconstruction
the code defines, its decision margins on constructed boundary points, and
the shipped polar codes against the figures recorded when they were trained."""
import math

import numpy as np
import pytest

import synth
import vector_codebook_codec_b200 as qamw
from oracle import codec, lloyd


@pytest.mark.parametrize("N", [16, 256, 2048])
def test_indices_name_the_points_the_quantizer_returns(N):
    pol = qamw.load_polar(N)
    code = lloyd.PolarCode(pol["amps"], pol["P"])
    x = synth.gaussian_points(20000, seed=N)
    idx, _ = code.indices(x)
    assert idx.min() >= 0 and idx.max() < code.N
    assert np.array_equal(code.points()[idx], code.quantize(x))


def test_margins_vanish_on_decision_boundaries():
    code = lloyd.PolarCode(np.array([0.5, 1.5, 2.5]), 8)
    w = 2 * math.pi / 8
    # on the amplitude edge 1.0, away from sector edges
    on_edge = np.array([[math.cos(0.5 * w), math.sin(0.5 * w)]])
    _, m = code.indices(on_edge)
    assert m[0] < 1e-15
    # on the sector edge at angle 3w, radius between edges
    on_sector = np.array([[1.3 * math.cos(3 * w), 1.3 * math.sin(3 * w)]])
    _, m = code.indices(on_sector)
    assert m[0] < 1e-12
    # a point in the middle of cell (amplitude 1, sector 2)
    mid = np.array([[1.5 * math.cos(2.5 * w), 1.5 * math.sin(2.5 * w)]])
    i, m = code.indices(mid)
    assert i[0] == 1 * 8 + 2 and m[0] > 0.3


@pytest.mark.parametrize("N", [4, 16, 128, 256])
def test_shipped_polar_codes_reproduce_their_training_distortion(N):
    e = qamw.codebook_manifest()[str(N)]
    pol = qamw.load_polar(N)
    assert pol["amps"].size == e["polar_amp_levels"] and pol["P"] == e["polar_sectors"]
    assert np.all(np.diff(pol["amps"]) > 0)
    x = lloyd.gaussian_samples(e["T"], e["seed"])
    d = lloyd.PolarCode(pol["amps"], pol["P"]).distortion(x)
    assert abs(d - e["polar_train_distortion"]) <= 1e-12 * d


def test_encode_polar_indices_and_joint_beats_polar():
    spec = synth.tiny().specs[0]
    W = synth.make_matrix(spec)
    act = synth.act_for(spec)
    sig = codec.calibrate_sigma(W, act, spec.alpha, spec.block, spec.seed)
    pol = qamw.load_polar(256)
    enc = codec.encode_polar(W, act, spec.alpha, spec.block, spec.seed, sig, pol["amps"], pol["P"], 8)
    assert enc["idx"].shape == (spec.M, spec.K // 2) and enc["idx"].max() < 256
    assert np.array_equal(codec.unpack_indices(enc["packed"], spec.K // 2, 8), enc["idx"])
    # reconstruct both codecs and compare the error (joint at most the polar one)
    C = qamw.load_codebook(256)
    joint = codec.encode(W, act, spec.alpha, spec.block, spec.seed, sig, C, 8)
    wj = codec.decode_with_scale(joint["idx"], joint["r"], sig, joint["s"], spec.K, spec.block, spec.seed, C)
    wp = codec.decode_with_scale(enc["idx"], enc["r"], sig, enc["s"], spec.K, spec.block, spec.seed,
                                 pol["points"])
    ej = np.sum((wj - W) ** 2)
    ep = np.sum((wp - W) ** 2)
    assert ej < ep
