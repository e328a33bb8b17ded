"""The bounded waits give up instead of hanging (GPU only): a wait on a
barrier that nothing completes runs out after its budget, the kernel returns
its status, and the context stays usable."""
import time

import pytest
import torch

import moe_expert_routing_token_b200 as moe
from moe_expert_routing_token_b200 import inputs

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def test_wait_runs_out_and_reports():
    status = torch.full((2,), -1, dtype=torch.int32, device=DEV)
    t0 = time.perf_counter()
    st = moe.lib().moe_selftest_bounded_wait(2_000_000, status.data_ptr(),
                                             torch.cuda.current_stream().cuda_stream)  # 2 ms budget
    torch.cuda.synchronize()
    elapsed = time.perf_counter() - t0
    assert st == 0
    ran_out, waited_us = status.tolist()
    assert ran_out == 1
    assert 2000 <= waited_us < 200_000
    assert elapsed < 5.0
    # the context is still usable: a routing call works and trips no watchdog
    d = inputs.make("biased", 2048)
    before = moe.watchdog_trips()
    w, ids = moe.biased_grouped_topk(d["logits"].to(DEV), d["bias"].to(DEV), 8, True, 8, 4, 2.5)
    torch.cuda.synchronize()
    assert moe.watchdog_trips() == before
    assert int(ids.min()) >= 0 and int(ids.max()) < 256


def test_budget_is_validated():
    status = torch.zeros(2, dtype=torch.int32, device=DEV)
    assert moe.lib().moe_selftest_bounded_wait(0, status.data_ptr(), None) == 1
    assert moe.lib().moe_selftest_bounded_wait(2_000_000_000, status.data_ptr(), None) == 1
