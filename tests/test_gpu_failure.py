"""Failure detection on the GPU without a fault: a bounded device wait that
nothing completes runs out, the kernel raises the device status word and
returns, the host reads MEDUSA_ERR_TIMEOUT, and the context stays usable."""
import time

import pytest
import torch

from medusa_head_speculative_02_b200 import _lib as L
from medusa_head_speculative_02_b200 import api

pytestmark = pytest.mark.gpu


def test_bounded_wait_runs_out_and_reports_timeout():
    torch.cuda.synchronize()
    assert api.device_status(clear=True) == L.OK
    t0 = time.perf_counter()
    api.selftest_wait_timeout(50)
    torch.cuda.synchronize()
    dt = time.perf_counter() - t0
    assert api.device_status(clear=False) == L.ERR_TIMEOUT
    assert api.device_status(clear=True) == L.ERR_TIMEOUT   # read, then cleared
    assert api.device_status(clear=False) == L.OK
    assert 0.045 <= dt < 1.5                                  # gave up after ~50 ms


def test_context_usable_after_timeout():
    api.selftest_wait_timeout(10)
    torch.cuda.synchronize()
    assert api.device_status(clear=True) == L.ERR_TIMEOUT
    # a library call still runs and matches its plain definition afterwards
    g = torch.Generator().manual_seed(3)
    x = torch.randn(4, 1000, generator=g).cuda()   # fp32: no ties
    idx, val = api.medusa_topk(x, 5)
    ref = torch.topk(x.cpu(), 5, dim=1)
    assert torch.equal(idx.cpu().long(), ref.indices)
    assert api.device_status(clear=True) == L.OK


def test_limit_out_of_range_is_rejected():
    for bad in (0, -5, 2001):
        with pytest.raises(Exception):
            api.selftest_wait_timeout(bad)
