"""Failure detection without a GPU fault: a bounded wait that runs out sets
QAMW_STATUS_TIMEOUT in the status word and the context stays usable."""
import numpy as np
import pytest
import torch

import synth
import vector_codebook_codec_b200 as qamw

pytestmark = pytest.mark.gpu


def test_a_wait_that_runs_out_reports_timeout_and_the_context_survives(lib):
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    rc = lib.qamw_selftest_wait_timeout(1000, qamw._ptr(st), qamw._stream_ptr())
    assert rc == qamw.QAMW_OK
    torch.cuda.synchronize()
    assert st.item() & qamw.STATUS_TIMEOUT
    # the context is usable: a decode right after runs and sets no status
    M, K, N, bits = 32, 256, 256, 8
    idx = synth.make_indices(M, K // 2, N, 1)
    from oracle import codec
    packed = torch.from_numpy(codec.pack_indices(idx, bits).view(np.int32)).cuda()
    enc = qamw.Encoded(packed, torch.ones(M, device="cuda"), torch.ones(K, device="cuda"),
                       torch.ones(K // 2, device="cuda"), M, K, 64, 3, N, bits)
    st2 = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = qamw.decode(enc, torch.from_numpy(qamw.load_codebook(N)).cuda(), out_dtype=torch.bfloat16, status=st2)
    torch.cuda.synchronize()
    assert st2.item() == 0 and torch.isfinite(out.float()).all()
