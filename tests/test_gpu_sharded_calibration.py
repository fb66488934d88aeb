"""Row-sharded calibration on one GPU: shards' fp64 sums (qamw_calibrate_partial_sums)
combined in shard order (qamw_sigma_from_partial_sums) give the oracle's sigma of
the whole matrix; one shard gives qamw_calibrate_sigma's sigma bit for bit."""
import numpy as np
import pytest
import torch

import synth
import vector_codebook_codec_b200 as qamw
from oracle import codec
from parity_utils import to_gpu_matrix

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("dtype,b,bounds", [("bf16", 128, [0, 1000, 1001, 2048]), ("f32", 64, [0, 77, 300])])
def test_shards_combine_to_the_whole_matrix_sigma(lib, dtype, b, bounds):
    rng = np.random.default_rng(len(bounds))
    M, K = bounds[-1], 1024
    w32 = (rng.standard_normal((M, K)) * 0.02).astype(np.float32)
    act = np.exp(rng.standard_normal(K)).astype(np.float32)
    Wd, W = to_gpu_matrix(w32, dtype)
    actd = torch.from_numpy(act).cuda()
    sums = torch.stack([qamw.calibrate_partial_sums(Wd[lo:hi], actd, 0.5, b, 9)
                        for lo, hi in zip(bounds[:-1], bounds[1:])])
    sig = qamw.sigma_from_partial_sums(sums, M).cpu().numpy()
    assert np.array_equal(sig, codec.calibrate_sigma(W, act, 0.5, b, 9))
    one = qamw.sigma_from_partial_sums(qamw.calibrate_partial_sums(Wd, actd, 0.5, b, 9)[None], M)
    assert torch.equal(one, qamw.calibrate_sigma(Wd, actd, 0.5, b, 9))
