"""Grouped-query attention on the GPU against the FP64 oracle.

H query heads share Hkv key/value heads (MQA when Hkv = 1); the oracle runs
the plain definition with K and V repeated over each group and sums the
gradients of a shared head over its group.  Same tolerances as the parity
suite.
"""
import numpy as np
import pytest
import torch

from flashattention_bf16_fwd_b200.stats import lse_rel_err, normwise_rel_err
from oracle import attention_bwd, attention_fwd, gqa_expand, gqa_reduce

pytestmark = pytest.mark.gpu

O_ATOL, LSE_RTOL, GRAD_RTOL = 2e-2, 1e-3, 5e-2


@pytest.fixture(scope="module")
def fa():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from flashattention_bf16_fwd_b200 import fa as binding
    return binding


def draw(B, H, Hkv, N, d, seed):
    g = torch.Generator().manual_seed(seed)
    q, do = (torch.randn(B, H, N, d, generator=g).to(torch.bfloat16) for _ in range(2))
    k, v = (torch.randn(B, Hkv, N, d, generator=g).to(torch.bfloat16) for _ in range(2))
    return q, k, v, do


CASES = [(1, 4, 2, 300, 64, True), (2, 8, 1, 256, 128, True), (1, 6, 3, 384, 64, False),
         (1, 16, 2, 1024, 64, True)]


@pytest.mark.parametrize("B,H,Hkv,N,d,causal", CASES,
                         ids=[f"B{b}H{h}kv{k}N{n}d{d}{'c' if c else 'f'}" for b, h, k, n, d, c in CASES])
def test_gqa_parity(fa, B, H, Hkv, N, d, causal):
    q, k, v, do = draw(B, H, Hkv, N, d, seed=N + H)
    scale = d ** -0.5
    dev = torch.device("cuda")
    qd, kd, vd, dod = (t.to(dev) for t in (q, k, v, do))
    o = torch.empty_like(qd)
    lse = torch.empty(B, H, N, dtype=torch.float32, device=dev)
    assert fa.fa_fwd_ex(qd, kd, vd, o, lse, causal, scale, 1) == 0
    dq, dk, dv = torch.empty_like(qd), torch.empty_like(kd), torch.empty_like(vd)
    ws = torch.empty(fa.fa_bwd_workspace_size(B, H, N, d), dtype=torch.uint8, device=dev)
    assert fa.fa_bwd_ex(qd, kd, vd, o, lse, dod, dq, dk, dv, ws, causal, scale) == 0
    torch.cuda.synchronize()
    assert fa.fa_check_device_error() == 0

    g = H // Hkv
    ke, ve = gqa_expand(k, g), gqa_expand(v, g)
    o_ref, lse_ref = attention_fwd(q, ke, ve, causal, scale)
    assert np.abs(o.float().cpu().numpy() - o_ref).max() <= O_ATOL
    assert lse_rel_err(lse.cpu().numpy(), lse_ref) <= LSE_RTOL
    dq_ref, dk_rep, dv_rep = attention_bwd(q, ke, ve, do, causal, scale)
    refs = {"dq": dq_ref, "dk": gqa_reduce(dk_rep, g), "dv": gqa_reduce(dv_rep, g)}
    for name, t in (("dq", dq), ("dk", dk), ("dv", dv)):
        err = normwise_rel_err(t.float().cpu().numpy(), refs[name])
        assert err <= GRAD_RTOL, (name, err)


def test_gqa_with_one_group_per_head_is_plain_attention(fa):
    """Hkv == H through fa_fwd_ex / fa_bwd_ex runs the same arithmetic as
    fa_fwd / fa_bwd, bit for bit (dQ up to the order of its reduce-adds)."""
    B, H, N, d = 1, 3, 333, 64
    q, k, v, do = (t.cuda() for t in draw(B, H, H, N, d, seed=5))
    o1, l1 = torch.empty_like(q), torch.empty(B, H, N, dtype=torch.float32, device="cuda")
    assert fa.fa_fwd(q, k, v, o1, l1, True, 0.125, 1) == 0
    o2, l2 = fa.attention_fwd(q, k, v, causal=True, scale=0.125, fix_mode=1)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
    dq1, dk1, dv1 = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ws = torch.empty(fa.fa_bwd_workspace_size(B, H, N, d), dtype=torch.uint8, device="cuda")
    assert fa.fa_bwd(q, k, v, o1, l1, do, dq1, dk1, dv1, ws, True, 0.125) == 0
    dq2, dk2, dv2 = fa.attention_bwd(q, k, v, o1, l1, do, causal=True, scale=0.125)
    torch.cuda.synchronize()
    assert torch.equal(dk1, dk2) and torch.equal(dv1, dv2)
    assert normwise_rel_err(dq1.float().cpu().numpy(), dq2.float().cpu().numpy().astype(np.float64)) < 2.0 ** -8


def test_gqa_at_a_size_that_takes_the_pair_schedule(fa):
    """B=6, H=32 query heads over Hkv=8 key/value heads, N=1024, d=64, causal.
    The backward's heads in flight (48 key/value heads, each with its group's
    Q, dO and FP32 dQ rows: 2 MiB) exceed the 64 MiB the host allows for the
    L2, so the backward runs the head-major pair schedule (key tiles t and
    n_kv-1-t of one head, each over the four query heads of its group).  Two
    sampled key/value heads, with their query heads, against the oracle."""
    B, H, Hkv, N, d = 6, 32, 8, 1024, 64
    g = H // Hkv
    q, k, v, do = draw(B, H, Hkv, N, d, seed=77)
    scale = d ** -0.5
    dev = torch.device("cuda")
    qd, kd, vd, dod = (t.to(dev) for t in (q, k, v, do))
    o = torch.empty_like(qd)
    lse = torch.empty(B, H, N, dtype=torch.float32, device=dev)
    assert fa.fa_fwd_ex(qd, kd, vd, o, lse, True, scale, 1) == 0
    dq, dk, dv = torch.empty_like(qd), torch.empty_like(kd), torch.empty_like(vd)
    ws = torch.empty(fa.fa_bwd_workspace_size(B, H, N, d), dtype=torch.uint8, device=dev)
    assert fa.fa_bwd_ex(qd, kd, vd, o, lse, dod, dq, dk, dv, ws, True, scale) == 0
    torch.cuda.synchronize()
    assert fa.fa_check_device_error() == 0
    for b, hk in ((0, 0), (5, 7)):
        hq = slice(hk * g, (hk + 1) * g)
        qs, dos = q[b:b + 1, hq], do[b:b + 1, hq]
        ks, vs = k[b:b + 1, hk:hk + 1], v[b:b + 1, hk:hk + 1]
        ke, ve = gqa_expand(ks, g), gqa_expand(vs, g)
        o_ref, lse_ref = attention_fwd(qs, ke, ve, True, scale)
        assert np.abs(o[b:b + 1, hq].float().cpu().numpy() - o_ref).max() <= O_ATOL
        assert lse_rel_err(lse[b:b + 1, hq].cpu().numpy(), lse_ref) <= LSE_RTOL
        dq_ref, dk_rep, dv_rep = attention_bwd(qs, ke, ve, dos, True, scale)
        refs = {"dq": (dq[b:b + 1, hq], dq_ref), "dk": (dk[b:b + 1, hk:hk + 1], gqa_reduce(dk_rep, g)),
                "dv": (dv[b:b + 1, hk:hk + 1], gqa_reduce(dv_rep, g))}
        for name, (got, ref) in refs.items():
            err = normwise_rel_err(got.float().cpu().numpy(), ref)
            assert err <= GRAD_RTOL, (b, hk, name, err)
    for t in (o, lse, dq, dk, dv):
        assert torch.isfinite(t).all()
