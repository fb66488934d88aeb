"""The codec's calls under CUDA-graph capture: calibrate + encode (pruned
search) + decode captured once and replayed give the eager results bit for
bit, so a caller can run the whole step as one graph launch. The first calls
(which cache the device's SM count and driver entry points) run before the
capture."""
import numpy as np
import pytest
import torch

import synth
import vector_codebook_codec_b200 as qamw

pytestmark = pytest.mark.gpu


def test_capture_and_replay_equal_eager(lib):
    spec = synth.llama7b_attn().specs[0]
    M, K = 1024, spec.K
    Wt, _ = synth.to_bf16(synth.make_matrix(spec)[:M])
    W = Wt.cuda()
    act = torch.from_numpy(synth.act_for(spec)).cuda()
    C = torch.from_numpy(qamw.load_codebook(spec.N)).cuda()
    table = qamw.build_search_table(C)
    wpr = qamw.words_per_row(K, spec.bits)
    ws = torch.empty(int(lib.qamw_calibrate_workspace_bytes(M, K)), dtype=torch.uint8, device="cuda")
    sigma = torch.empty(K // 2, device="cuda")
    packed = torch.empty((M, wpr), dtype=torch.int32, device="cuda")
    r = torch.empty(M, device="cuda")
    s = torch.empty(K, device="cuda")
    out = torch.empty((M, K), dtype=torch.bfloat16, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")

    def step(stream=None):
        sg = qamw.calibrate_sigma(W, act, spec.alpha, spec.block, spec.seed, status=status, workspace=ws,
                                  out=sigma, stream=stream)
        enc = qamw.encode(W, act, spec.alpha, spec.block, spec.seed, sg, C, spec.bits, status=status,
                          out=(packed, r, s), search_table=table, stream=stream)
        qamw.decode(enc, C, out_dtype=torch.bfloat16, status=status, out=out, stream=stream)

    step()                                            # eager, also warms the caches
    torch.cuda.synchronize()
    ref = [t.clone() for t in (sigma, packed, r, s, out)]
    for t in (sigma, packed, r, s, out):
        t.zero_()
    side = torch.cuda.Stream()
    g = torch.cuda.CUDAGraph()
    torch.cuda.synchronize()
    with torch.cuda.graph(g, stream=side):
        step(stream=side)
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    assert status.item() == 0
    for a, b in zip(ref, (sigma, packed, r, s, out)):
        assert torch.equal(a, b)
