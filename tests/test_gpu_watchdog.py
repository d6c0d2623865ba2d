"""The kernels' failure handling on a GPU, without a fault or a hang.

fa_watchdog_selftest() runs the library's bounded mbarrier wait with a short
limit on a barrier that nothing arrives on.  The wait must give up, record a
timeout in the device error flag and mark its CTA aborted; a second waiter in
the same CTA must leave on that mark long before its own 4 s limit.  The
context stays usable: a forward and backward pass afterwards still match the
oracle.
"""
import time

import numpy as np
import pytest
import torch

from flashattention_bf16_fwd_b200.stats import normwise_rel_err
from flashattention_bf16_fwd_b200.workloads import WORKLOADS, make_inputs
from oracle import attention_bwd, attention_fwd

pytestmark = pytest.mark.gpu

FA_ERR_TIMEOUT = -8


def test_bounded_wait_times_out_and_the_context_survives():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from flashattention_bf16_fwd_b200 import fa

    assert fa.fa_check_device_error() == 0
    t0 = time.perf_counter()
    assert fa.fa_watchdog_selftest(2000) == 0          # 2 ms limit
    assert fa.fa_check_device_error() == FA_ERR_TIMEOUT
    elapsed = time.perf_counter() - t0
    # the second waiter left on the abort mark, not on its own 4 s limit
    assert elapsed < 1.0, elapsed
    assert fa.fa_check_device_error() == 0             # reading the flag cleared it

    x = make_inputs(WORKLOADS["tiny"], seed=4)
    dev = torch.device("cuda")
    q, k, v, do = (x[n].to(dev) for n in ("q", "k", "v", "do"))
    o, lse = fa.attention_fwd(q, k, v, causal=True, scale=x["scale"], fix_mode=1)
    dq, dk, dv = fa.attention_bwd(q, k, v, o, lse, do, causal=True, scale=x["scale"])
    torch.cuda.synchronize()
    assert fa.fa_check_device_error() == 0
    o_ref, _ = attention_fwd(x["q"], x["k"], x["v"], True, x["scale"])
    assert np.abs(o.float().cpu().numpy() - o_ref).max() <= 2e-2
    refs = attention_bwd(x["q"], x["k"], x["v"], x["do"], True, x["scale"])
    for g, r in zip((dq, dk, dv), refs):
        assert normwise_rel_err(g.float().cpu().numpy(), r) <= 5e-2
