"""The encoded artefact on disk (save_encoded / load_encoded): a lossless,
versioned round trip of everything the decode needs (CPU tensors; no GPU)."""
import numpy as np
import pytest
import torch

import synth
import vector_codebook_codec_b200 as qamw
from oracle import codec


def _encoded():
    spec = synth.tiny().specs[0]
    W = synth.make_matrix(spec)[:16]
    act = synth.act_for(spec)
    sig = codec.calibrate_sigma(W, act, spec.alpha, spec.block, spec.seed)
    C = qamw.load_codebook(spec.N)
    e = codec.encode(W, act, spec.alpha, spec.block, spec.seed, sig, C, spec.bits)
    enc = qamw.Encoded(torch.from_numpy(e["packed"].view(np.int32)), torch.from_numpy(e["r"]),
                       torch.from_numpy(e["s"]), torch.from_numpy(sig), 16, spec.K, spec.block,
                       spec.seed, spec.N, spec.bits)
    return enc, C, e, sig, spec


def test_round_trip_is_lossless(tmp_path):
    enc, C, e, sig, spec = _encoded()
    path = str(tmp_path / "m.npz")
    qamw.save_encoded(path, enc, torch.from_numpy(C))
    got, Cg = qamw.load_encoded(path, device="cpu")
    assert (got.M, got.K, got.block, got.seed, got.N, got.bits) == (16, spec.K, spec.block, spec.seed, spec.N,
                                                                    spec.bits)
    for a, b in ((got.packed, enc.packed), (got.row_norm, enc.row_norm), (got.col_scale, enc.col_scale),
                 (got.sigma, enc.sigma)):
        assert torch.equal(a, b)
    assert np.array_equal(Cg.numpy(), C)
    # the loaded artefact decodes (oracle) to the same matrix
    idx = codec.unpack_indices(got.packed.numpy().view(np.uint32), spec.K // 2, spec.bits)
    assert np.array_equal(idx, e["idx"])


def test_other_formats_and_versions_are_rejected(tmp_path):
    enc, C, *_ = _encoded()
    path = str(tmp_path / "m.npz")
    qamw.save_encoded(path, enc, torch.from_numpy(C))
    z = dict(np.load(path))
    z["version"] = np.array(99, dtype=np.int32)
    np.savez(str(tmp_path / "v.npz"), **z)
    with pytest.raises(ValueError, match="version"):
        qamw.load_encoded(str(tmp_path / "v.npz"), device="cpu")
    z["version"] = np.array(1, dtype=np.int32)
    z["format"] = np.array("something-else")
    np.savez(str(tmp_path / "f.npz"), **z)
    with pytest.raises(ValueError, match="not a"):
        qamw.load_encoded(str(tmp_path / "f.npz"), device="cpu")
