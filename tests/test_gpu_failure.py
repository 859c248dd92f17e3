"""Failure detection on the GPU without a fault: a bounded pipeline wait that
nothing will complete gives up at its limit, the kernel records
MISA_DEVERR_TIMEOUT in the error word and returns, and the context keeps
working for the next call."""
import time

import pytest
import torch

import sparse_attention_token_misa_b200 as misa
from sparse_attention_token_misa_b200 import _native as nat

pytestmark = pytest.mark.gpu


def test_bounded_wait_times_out_and_context_survives():
    ws = misa.alloc_workspace(256)
    t0 = time.time()
    nat.selftest_wait_timeout(ws)
    bits = misa.error_query(ws)               # synchronises
    elapsed = time.time() - t0
    assert bits & nat.DEVERR_TIMEOUT
    assert int(ws[4:8].view(torch.int32).item()) == 0   # the wait reported failure
    assert 1.0 < elapsed < 60.0                          # the wait's limit is about two seconds
    # the context is still usable: an ordinary call runs and is right
    misa.error_reset(ws)
    s = torch.randn(3, 5000, device="cuda")
    idx = misa.topk(s, 16, workspace=ws)
    torch.cuda.synchronize()
    assert misa.error_query(ws) == 0
    ref = torch.topk(s, 16, dim=1).indices.sort(dim=1).values.to(torch.int32)
    assert torch.equal(idx, ref)
