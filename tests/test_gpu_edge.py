"""Degenerate inputs on the GPU, against the FP64 oracle and against the
values the definition fixes exactly.

* Q = 0: every visible score is equal, so every row is one big tie (counted
  across key tiles), O is the mean of the visible V rows and LSE = ln(#visible).
* V = 0 and dO = 0: outputs and gradients that the definition makes exactly 0.
* Large scores (|S| up to a few hundred): most P underflow to 0.
* A tiny scale: nearly uniform attention.
"""
import math

import numpy as np
import pytest
import torch

from flashattention_bf16_fwd_b200.stats import lse_rel_err, normwise_rel_err
from flashattention_bf16_fwd_b200.workloads import Workload, make_inputs
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
    o, lse, ties = fa.attention_fwd(qd, kd, vd, causal=causal, scale=scale, fix_mode=fix_mode, ties=True)
    out = {"o": o, "lse": lse, "ties": ties}
    if bwd:
        out.update(zip(("dq", "dk", "dv"), fa.attention_bwd(qd, kd, vd, o, lse, do.to(dev), causal=causal,
                                                            scale=scale)))
    torch.cuda.synchronize()
    assert fa.fa_check_device_error() == 0
    return {n: (t.cpu().numpy() if t.dtype == torch.int32 else t.float().cpu().numpy()) for n, t in out.items()}


CASES = [(1000, 64, True), (1000, 128, True), (300, 64, False)]


@pytest.mark.parametrize("N,d,causal", CASES, ids=[f"N{n}d{d}{'c' if c else 'f'}" for n, d, c in CASES])
@pytest.mark.parametrize("fix_mode", [0, 1])
def test_all_scores_equal(fa, N, d, causal, fix_mode):
    x = make_inputs(Workload("eq", 1, 2, N, d, causal=causal), seed=N + d)
    q = torch.zeros_like(x["q"])
    g = run(fa, q, x["k"], x["v"], x["do"], causal, x["scale"], fix_mode)
    n_vis = np.arange(1, N + 1) if causal else np.full(N, N)
    # every visible key ties with the maximum, across all key tiles
    assert np.array_equal(g["ties"][0] & ((1 << 29) - 1), np.broadcast_to(n_vis, (2, N)))
    fired = (g["ties"][0] >> 30) & 1
    assert np.array_equal(fired, np.broadcast_to(n_vis >= 2, (2, N)).astype(fired.dtype))
    # LSE = ln(#visible) exactly up to fp32 rounding, O = mean of the visible V
    assert np.abs(g["lse"][0] - np.log(n_vis)).max() <= 1e-5 * np.log(N) + 1e-6
    v = x["v"].double().numpy()[0]
    mean = np.cumsum(v, axis=1) / n_vis[None, :, None] if causal else np.broadcast_to(v.mean(axis=1, keepdims=True), v.shape)
    assert np.abs(g["o"][0] - mean).max() <= O_ATOL
    oe, _ = attention_fwd_bf16p(q, x["k"], x["v"], causal, x["scale"], fix_mode)
    assert np.abs(g["o"] - oe).max() <= O_ATOL
    for name, ref in zip(("dq", "dk", "dv"), attention_bwd(q, x["k"], x["v"], x["do"], causal, x["scale"])):
        assert np.isfinite(g[name]).all()
        if name == "dv":
            assert normwise_rel_err(g[name], ref) <= GRAD_RTOL
        else:   # dK = scale dS^T Q = 0 exactly; dQ is a genuine gradient
            if name == "dk":
                assert np.all(g[name] == 0.0)
            else:
                assert normwise_rel_err(g[name], ref) <= GRAD_RTOL


def test_zero_values_and_zero_output_gradient(fa):
    x = make_inputs(Workload("z", 1, 2, 777, 64), seed=4)
    # V = 0: O = 0, D = 0, dP = 0, so dS = 0 and dQ = dK = 0 exactly; dV = P^T dO
    v0 = torch.zeros_like(x["v"])
    g = run(fa, x["q"], x["k"], v0, x["do"], True, x["scale"], 1)
    assert np.all(g["o"] == 0.0) and np.all(g["dq"] == 0.0) and np.all(g["dk"] == 0.0)
    _, lse_ref = attention_fwd(x["q"], x["k"], v0, True, x["scale"])
    assert lse_rel_err(g["lse"], lse_ref) <= LSE_RTOL
    _, _, dv_ref = attention_bwd(x["q"], x["k"], v0, x["do"], True, x["scale"])
    assert normwise_rel_err(g["dv"], dv_ref) <= GRAD_RTOL
    # dO = 0: every gradient is exactly 0
    g = run(fa, x["q"], x["k"], x["v"], torch.zeros_like(x["do"]), True, x["scale"], 1)
    assert np.all(g["dq"] == 0.0) and np.all(g["dk"] == 0.0) and np.all(g["dv"] == 0.0)


def test_large_scores(fa):
    """Q and K scaled by 6 (|S| up to a few hundred): most exponentials
    underflow to 0, nothing overflows, and O and LSE match the oracle.  The
    seed leaves every row's two largest scores at least 0.04 apart, far above
    the FP32 error of S, so the kernel and the oracle agree on every maximum."""
    w = Workload("peak", 1, 2, 700, 64)
    x = make_inputs(w, seed=0)
    q, k = ((x[n].float() * 6).to(torch.bfloat16) for n in ("q", "k"))
    g = run(fa, q, k, x["v"], x["do"], True, w.scale, 1)
    o_ref, lse_ref = attention_fwd(q, k, x["v"], True, w.scale)
    assert np.isfinite(g["o"]).all() and np.isfinite(g["lse"]).all()
    assert np.abs(g["o"] - o_ref).max() <= O_ATOL
    assert lse_rel_err(g["lse"], lse_ref) <= LSE_RTOL
    for name in ("dq", "dk", "dv"):
        assert np.isfinite(g[name]).all()
    _, _, dv_ref = attention_bwd(q, k, x["v"], x["do"], True, w.scale)
    assert normwise_rel_err(g["dv"], dv_ref) <= GRAD_RTOL


def test_tiny_scale(fa):
    """scale = 1e-3: nearly uniform attention, full gradients against the oracle."""
    x = make_inputs(Workload("flat", 1, 2, 500, 128), seed=6)
    g = run(fa, x["q"], x["k"], x["v"], x["do"], True, 1e-3, 1)
    o_ref, lse_ref = attention_fwd(x["q"], x["k"], x["v"], True, 1e-3)
    assert np.abs(g["o"] - o_ref).max() <= O_ATOL
    assert lse_rel_err(g["lse"], lse_ref) <= LSE_RTOL
    assert abs(float(g["lse"][0, 0, 499]) - math.log(500)) < 1e-2
    for name, ref in zip(("dq", "dk", "dv"), attention_bwd(x["q"], x["k"], x["v"], x["do"], True, 1e-3)):
        assert normwise_rel_err(g[name], ref) <= GRAD_RTOL, name


REPEAT_CASES = [(2, 3, 777, 64, True), (1, 4, 1000, 64, True), (3, 2, 129, 64, True), (2, 2, 700, 128, True),
                (1, 3, 333, 64, False)]


@pytest.mark.parametrize("B,H,N,d,causal", REPEAT_CASES,
                         ids=[f"B{b}H{h}N{n}d{d}{'c' if c else 'f'}" for b, h, n, d, c in REPEAT_CASES])
def test_forward_repeats_bit_for_bit(fa, B, H, N, d, causal):
    """The forward is deterministic: 40 back-to-back calls give the same O,
    LSE and tie record, bit for bit, and no bounded wait expires.  At d = 64
    the two softmax warpgroups run independent MMA chains that share the K/V
    stages and the Q buffers; a release that raced ahead of the other chain
    would let a stage be refilled while still in use, and show here as a
    changed output or an expired wait.  The shapes include items with a
    single query tile and odd tails."""
    x = make_inputs(Workload("rep", B, H, N, d, causal=causal), seed=N + d + B)
    dev = torch.device("cuda")
    q, k, v = (x[n].to(dev) for n in ("q", "k", "v"))
    o0, l0, t0 = fa.attention_fwd(q, k, v, causal=causal, scale=x["scale"], fix_mode=1, ties=True)
    outs = []
    for _ in range(40):
        outs.append(fa.attention_fwd(q, k, v, causal=causal, scale=x["scale"], fix_mode=1, ties=True))
    torch.cuda.synchronize()
    assert fa.fa_check_device_error() == 0
    for o, l, t in outs:
        assert torch.equal(o, o0) and torch.equal(l, l0) and torch.equal(t, t0)
    # the production instantiation (no records) as well
    p0 = fa.attention_fwd(q, k, v, causal=causal, scale=x["scale"], fix_mode=1)
    for _ in range(40):
        o, l = fa.attention_fwd(q, k, v, causal=causal, scale=x["scale"], fix_mode=1)
        assert torch.equal(o, p0[0]) and torch.equal(l, p0[1])
    torch.cuda.synchronize()
    assert fa.fa_check_device_error() == 0
    assert torch.equal(p0[0], o0) and torch.equal(p0[1], l0)


SPLIT_CASES = [(2, 3, 777, 64, True), (1, 4, 1000, 64, True), (2, 2, 700, 128, True), (1, 3, 333, 64, False)]


@pytest.mark.parametrize("B,H,N,d,causal", SPLIT_CASES,
                         ids=[f"B{b}H{h}N{n}d{d}{'c' if c else 'f'}" for b, h, n, d, c in SPLIT_CASES])
def test_backward_one_call_matches_three_calls(fa, B, H, N, d, causal):
    """fa_bwd launches the main kernel right after the preprocess and lets it
    load Q, K, V, dO and LSE and start its first MMAs before the preprocess
    has finished (only D and the zeroed dQ accumulator come from it); the
    three calls one by one make every thread of the main kernel wait.  Both
    give the same dK and dV bit for bit (each is summed in one CTA in a fixed
    order) and the same dQ up to the order of the FP32 reduce-adds, repeated
    20 times so that a read of D or of the accumulator ahead of the
    preprocess would show (the workspace holds NaN before each call)."""
    x = make_inputs(Workload("split", B, H, N, d, causal=causal), seed=N + d + 7 * B)
    dev = torch.device("cuda")
    q, k, v, do = (x[n].to(dev) for n in ("q", "k", "v", "do"))
    o, lse = fa.attention_fwd(q, k, v, causal=causal, scale=x["scale"], fix_mode=1)
    ws = torch.empty(fa.fa_bwd_workspace_size(B, H, N, d), dtype=torch.uint8, device=dev)
    dq3, dk3, dv3 = (torch.empty_like(q) for _ in range(3))
    for call, rc in (("pre", fa.fa_bwd_preprocess(o, do, ws)),
                     ("main", fa.fa_bwd_main(q, k, v, lse, do, dk3, dv3, ws, causal, x["scale"])),
                     ("finish", fa.fa_bwd_finish(dq3, ws, x["scale"]))):
        assert rc == 0, call
    torch.cuda.synchronize()
    assert fa.fa_check_device_error() == 0
    for _ in range(20):
        dq1, dk1, dv1 = (torch.empty_like(q) for _ in range(3))
        ws.fill_(0xFF)                                 # NaN in D and in the accumulator until the preprocess runs
        assert fa.fa_bwd(q, k, v, o, lse, do, dq1, dk1, dv1, ws, causal, x["scale"]) == 0
        torch.cuda.synchronize()
        assert fa.fa_check_device_error() == 0
        assert torch.equal(dk1, dk3) and torch.equal(dv1, dv3)
        # dQ: FP32 sums in a varying order, then one rounding to bf16
        diff = (dq1.float() - dq3.float()).abs()
        assert float(diff.max()) <= 2 ** -7 * float(dq3.float().abs().max()) + 1e-6
