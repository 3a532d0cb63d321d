"""Failure detection on the GPU without a fault: a bounded pipeline wait that
nothing satisfies ends with BSA_ERR_TIMEOUT in the status word after its short
limit, and the CUDA context stays usable for real work afterwards."""
import time

import numpy as np
import pytest
import torch

from block_sparse_attention_tokens_b200 import binding as B

pytestmark = pytest.mark.gpu


def test_stuck_wait_reports_timeout_and_context_survives():
    t0 = time.perf_counter()
    status = B.bsa_wait_selftest(20_000_000)          # 20 ms limit
    elapsed = time.perf_counter() - t0
    assert status == 5, B.bsa_status_string(status)   # BSA_ERR_TIMEOUT
    assert elapsed < 5.0
    # the context still runs kernels: a tiny attention call succeeds afterwards
    q = torch.randn(1, 256, 1, 64).to(torch.bfloat16).cuda()
    rp = torch.tensor([0, 2, 4], dtype=torch.int32).cuda()
    ci = torch.tensor([0, 1, 0, 1], dtype=torch.int32).cuda()
    o, lse, ws = B.bsa_attn_fwd(q, q, q, rp, ci, 128, 128, 1)
    torch.cuda.synchronize()
    assert B.bsa_read_status(ws) == 0
    assert torch.isfinite(o.float()).all()


def test_selftest_rejects_bad_limits():
    with pytest.raises(B.BsaError):
        B.bsa_wait_selftest(0)
