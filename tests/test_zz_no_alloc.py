"""fa_bwd_noalloc (the backward for callers that cannot allocate device
memory) against fa_bwd on the same inputs, through the C ABI.

The file name sorts last so that it also runs after every other GPU test in
one process; it passes on its own in a fresh process as well.  Two calls in a
row on the same shape: the fixed scratch array keeps the first call's
contents, so a second call that failed to clear its accumulator would show
the first call's dQ in its own (an error of order 100%).  dK and dV do not
depend on the scratch and must match fa_bwd bit for bit.  dQ is summed with
reduce-adds in an order that varies from run to run, so after its rounding to
bf16 a few elements land one bf16 step apart; it is held to the gradient
tolerance of the parity tests (normwise 5e-2).  A d = 128 call follows to
cover the other kernel instantiation.  Last, once every kernel has run (so
that loading their code has already claimed its memory), a call on a shape
not seen before must leave the device's free memory exactly where it was:
the call allocates nothing.
"""
import pytest
import torch

from flashattention_bf16_fwd_b200.stats import normwise_rel_err
from flashattention_bf16_fwd_b200.workloads import Workload, make_inputs

pytestmark = pytest.mark.gpu

GRAD_RTOL = 5e-2


def test_noalloc_matches_fa_bwd_on_calls_in_a_row():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from flashattention_bf16_fwd_b200 import fa

    dev = torch.device("cuda")
    cases = [(Workload("noalloc", 2, 3, 1000, 64, causal=True), 1),
             (Workload("noalloc", 2, 3, 1000, 64, causal=True), 2),
             (Workload("noalloc", 1, 4, 777, 128, causal=False), 3)]
    for w, seed in cases:
        x = make_inputs(w, seed=seed)
        q, k, v, do = (x[n].to(dev) for n in ("q", "k", "v", "do"))
        o, lse = fa.attention_fwd(q, k, v, causal=w.causal, scale=w.scale, fix_mode=1)
        ref = fa.attention_bwd(q, k, v, o, lse, do, causal=w.causal, scale=w.scale)
        # NaN-filled outputs: every element must be written
        got = [torch.full_like(q, float("nan")) for _ in range(3)]
        assert fa.fa_bwd_noalloc(q, k, v, o, lse, do, *got, w.causal, w.scale) == 0
        torch.cuda.synchronize()
        assert fa.fa_check_device_error() == 0
        dq, dk, dv = got
        assert torch.equal(dk, ref[1]) and torch.equal(dv, ref[2]), (w, seed)
        err = normwise_rel_err(dq.float().cpu().numpy(), ref[0].float().cpu().numpy())
        assert err <= GRAD_RTOL, (w, seed, err)
    # a new shape after every kernel has been loaded: no device memory changes hands
    w = Workload("noalloc", 1, 2, 513, 64, causal=True)
    x = make_inputs(w, seed=4)
    q, k, v, do = (x[n].to(dev) for n in ("q", "k", "v", "do"))
    o, lse = fa.attention_fwd(q, k, v, causal=w.causal, scale=w.scale, fix_mode=1)
    got = [torch.empty_like(q) for _ in range(3)]
    torch.cuda.synchronize()
    free_before, _ = torch.cuda.mem_get_info()
    assert fa.fa_bwd_noalloc(q, k, v, o, lse, do, *got, w.causal, w.scale) == 0
    torch.cuda.synchronize()
    free_after, _ = torch.cuda.mem_get_info()
    assert fa.fa_check_device_error() == 0
    assert free_after == free_before, (free_before, free_after)
