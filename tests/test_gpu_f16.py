"""The FP16 variant (fa_fwd_ex / fa_bwd_ex with FP16 tensors) against the FP64 oracle.

Inputs are drawn in float32 and cast once to fp16, so they use fp16's full
11-bit significand.  The exact oracle and the tolerances of the bf16 parity
suite apply unchanged; the emulating oracle with fp16 P_bar checks the
rounding point and the fix (maxima at 1 - 2^-11).
"""
import numpy as np
import pytest
import torch

from flashattention_bf16_fwd_b200.stats import lse_rel_err, normwise_rel_err
from flashattention_bf16_fwd_b200.workloads import WORKLOADS, make_inputs
from oracle import attention_bwd, attention_fwd, attention_fwd_bf16p

pytestmark = pytest.mark.gpu

O_ATOL, LSE_RTOL, GRAD_RTOL = 2e-2, 1e-3, 5e-2


@pytest.fixture(scope="module")
def fa():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from flashattention_bf16_fwd_b200 import fa as binding
    return binding


def run(fa, q, k, v, do, causal, scale, fix_mode, bwd=True):
    dev = torch.device("cuda")
    qd, kd, vd = (t.to(dev) for t in (q, k, v))
    B, H, N, d = q.shape
    o = torch.empty_like(qd)
    lse = torch.empty(B, H, N, dtype=torch.float32, device=dev)
    assert fa.fa_fwd_ex(qd, kd, vd, o, lse, causal, scale, fix_mode) == 0
    out = {"o": o, "lse": lse}
    if bwd:
        dod = do.to(dev)
        dq, dk, dv = torch.empty_like(qd), torch.empty_like(kd), torch.empty_like(vd)
        ws = torch.empty(fa.fa_bwd_workspace_size(B, H, N, d), dtype=torch.uint8, device=dev)
        assert fa.fa_bwd_ex(qd, kd, vd, o, lse, dod, dq, dk, dv, ws, causal, scale) == 0
        out.update(dq=dq, dk=dk, dv=dv)
    torch.cuda.synchronize()
    assert fa.fa_check_device_error() == 0
    return {n: t.float().cpu().numpy() for n, t in out.items()}


SHAPES = [(1, 2, 127, 64, 1), (1, 2, 1000, 64, 1), (1, 1, 200, 128, 1), (1, 2, 384, 128, 0)]


@pytest.mark.parametrize("B,H,N,d,causal", SHAPES, ids=[f"B{b}H{h}N{n}d{d}{'c' if c else 'f'}" for b, h, n, d, c in SHAPES])
@pytest.mark.parametrize("fix_mode", [0, 1])
def test_f16_parity(fa, B, H, N, d, causal, fix_mode):
    g = torch.Generator().manual_seed(N + d)
    q, k, v, do = (torch.randn(B, H, N, d, generator=g).half() for _ in range(4))
    scale = d ** -0.5
    r = run(fa, q, k, v, do, bool(causal), scale, fix_mode)
    o_ref, lse_ref = attention_fwd(q, k, v, bool(causal), scale)
    assert np.abs(r["o"] - o_ref).max() <= O_ATOL
    assert lse_rel_err(r["lse"], lse_ref) <= LSE_RTOL
    for name, ref in zip(("dq", "dk", "dv"), attention_bwd(q, k, v, do, bool(causal), scale)):
        err = normwise_rel_err(r[name], ref)
        assert err <= GRAD_RTOL, (name, err)


def test_f16_fix_on_repeated_maxima(fa):
    x = make_inputs(WORKLOADS["tiny"], seed=0)   # bf16 values, exact in fp16
    q, k, v, do = (x[n].half() for n in ("q", "k", "v", "do"))
    r1 = run(fa, q, k, v, do, True, x["scale"], 1, bwd=False)
    r0 = run(fa, q, k, v, do, True, x["scale"], 0, bwd=False)
    oe, le = attention_fwd_bf16p(q, k, v, True, x["scale"], 1, fmt="fp16")
    assert np.abs(r1["o"] - oe).max() <= O_ATOL
    assert lse_rel_err(r1["lse"], le) <= LSE_RTOL
    # the fix changes O only on some rows (those whose maximum repeats)
    changed = np.any(r1["o"] != r0["o"], axis=-1)
    assert 0 < changed.sum() < changed.size
