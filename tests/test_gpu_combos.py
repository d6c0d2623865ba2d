"""Combinations through the general entry points (fa_fwd_ex / fa_bwd_ex, via
attention_fwd / attention_bwd): fp16 with the fix variants (fix_mode 2-5),
fp16 with grouped-query heads, and fa_fwd_debug's agreement with fa_fwd_ex.

Same tolerances as the parity suite: the exact FP64 oracle applies to every
mode; the emulating oracle with fp16 P_bar (one shift per row) checks each
mode's rounding point, and fix_mode 5's near-tie test is made in fp16
(P >= 1 - 2^-12 rounds to 1).
"""
import numpy as np
import pytest
import torch

from flashattention_bf16_fwd_b200.stats import bias_stats, lse_rel_err, normwise_rel_err
from flashattention_bf16_fwd_b200.workloads import WORKLOADS, make_inputs
from oracle import (attention_bwd, attention_fwd, attention_fwd_bf16p, gqa_expand, gqa_reduce, near_tie_counts,
                    tie_counts)

pytestmark = pytest.mark.gpu

O_ATOL, LSE_RTOL, GRAD_RTOL = 2e-2, 1e-3, 5e-2


@pytest.fixture(scope="module")
def fa():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from flashattention_bf16_fwd_b200 import fa as binding
    return binding


def fwd(fa, q, k, v, causal, scale, fix_mode):
    dev = torch.device("cuda")
    o, lse, ties = fa.attention_fwd(q.to(dev), k.to(dev), v.to(dev), causal=causal, scale=scale,
                                    fix_mode=fix_mode, ties=True)
    torch.cuda.synchronize()
    assert fa.fa_check_device_error() == 0
    return o.float().cpu().numpy(), lse.cpu().numpy(), ties.cpu().numpy()


def half_inputs(structure, seed, **shape):
    """The tiny workload's structured inputs (bf16 values, exact in fp16) as fp16."""
    x = make_inputs(WORKLOADS["tiny"].with_shape(structure=structure, **shape), seed=seed, with_grad=False)
    return x["q"].half(), x["k"].half(), x["v"].half(), x["scale"]


SHAPES = [(1, 2, 1000, 64, 1), (1, 2, 384, 128, 0)]


@pytest.mark.parametrize("B,H,N,d,causal", SHAPES, ids=[f"B{b}H{h}N{n}d{d}{'c' if c else 'f'}" for b, h, n, d, c in SHAPES])
@pytest.mark.parametrize("fix_mode", [2, 3, 4, 5])
def test_f16_variant_parity(fa, B, H, N, d, causal, fix_mode):
    g = torch.Generator().manual_seed(N + d + fix_mode)
    q, k, v = (torch.randn(B, H, N, d, generator=g).half() for _ in range(3))
    scale = d ** -0.5
    o, lse, _ = fwd(fa, q, k, v, bool(causal), scale, fix_mode)
    o_ref, lse_ref = attention_fwd(q, k, v, bool(causal), scale)
    assert np.isfinite(o).all() and np.isfinite(lse).all()
    assert np.abs(o - o_ref).max() <= O_ATOL
    assert lse_rel_err(lse, lse_ref) <= LSE_RTOL


@pytest.mark.parametrize("fix_mode", [2, 3, 4])
def test_f16_variant_on_repeated_maxima(fa, fix_mode):
    q, k, v, scale = half_inputs("argmax_dup", 0)
    o, lse, ties = fwd(fa, q, k, v, True, scale, fix_mode)
    oe, le = attention_fwd_bf16p(q, k, v, True, scale, fix_mode, fmt="fp16")
    assert np.abs(o - oe).max() <= O_ATOL
    assert lse_rel_err(lse, le) <= LSE_RTOL
    o0, lse0, ties0 = fwd(fa, q, k, v, True, scale, 0)
    # the detector does not depend on the mode (bit 29, the final shift raised, does)
    assert np.array_equal(ties & ~(1 << 29), ties0 & ~(1 << 29))
    assert not np.any(ties0 & (1 << 29))             # fix_mode 0 never raises the shift
    if fix_mode in (2, 3):                             # the raised rows are those whose final maximum repeats
        assert np.array_equal((ties >> 29) & 1, ((ties & ((1 << 29) - 1)) >= 2).astype(ties.dtype))
    fired = ((ties >> 30) & 1) == 1
    assert fired.sum() > 10
    assert np.array_equal(lse[~fired], lse0[~fired])
    if fix_mode != 4:                                  # mode 4 changes every row's denominator
        assert np.array_equal(o[~fired], o0[~fired])
    if fix_mode == 3:                                  # maxima off the fp16 grid: O moves on fired rows
        assert np.any(o[fired] != o0[fired])


def test_f16_near_tie_detector(fa):
    """fix_mode 5 with fp16 P_bar: the detector fires where the oracle counts
    two or more entries whose P rounds to fp16 1.0 (one key tile, so the
    kernel's per-tile count is the row's), and rows left alone run fix_mode
    0's arithmetic."""
    q, k, v, scale = half_inputs("argmax_near", 0)
    o5, lse5, t5 = fwd(fa, q, k, v, True, scale, 5)
    o0, lse0, _ = fwd(fa, q, k, v, True, scale, 0)
    near = near_tie_counts(q, k, True, scale, fmt="fp16") >= 2
    assert near.sum() > 40
    fired = ((t5 >> 30) & 1) == 1
    assert np.mean(fired == near) >= 0.99
    assert np.array_equal(o5[~fired], o0[~fired]) and np.array_equal(lse5[~fired], lse0[~fired])
    oe, le = attention_fwd_bf16p(q, k, v, True, scale, 5, fmt="fp16")
    assert np.abs(o5 - oe).max() <= O_ATOL
    assert lse_rel_err(lse5, le) <= LSE_RTOL
    o_ref, _ = attention_fwd(q, k, v, True, scale)
    assert np.abs(o5 - o_ref).max() <= O_ATOL


def test_f16_self_normalised_output_of_ones(fa):
    q, k, v, scale = half_inputs("argmax_dup", 2, H=4, N=700)
    o4, _, _ = fwd(fa, q, k, torch.ones_like(v), True, scale, 4)
    assert np.abs(o4 - 1.0).max() <= 2.0 ** -11          # one fp16 step below 1 at most
    assert np.mean(o4 == 1.0) > 0.99



def test_f16_bias_sweep_over_fix_modes(fa):
    """The bias statistics of every mode with fp16 P_bar on the repeated-max
    rows of the long-structured input (printed).  As in bf16, fix_mode 1 must
    show no sign-coherent error (|z| < 3 for both statistics)."""
    w = WORKLOADS["long"].with_shape(B=2, H=8, N=2048)
    x = make_inputs(w, seed=1, with_grad=False)
    q, k, v = (x[n].half() for n in ("q", "k", "v"))
    o_ref, _ = attention_fwd(q, k, v, True, w.scale)
    rep = tie_counts(q, k, True) >= 2
    assert rep.sum() > 1000
    rows = {}
    for mode in range(6):
        o, _, _ = fwd(fa, q, k, v, True, w.scale, mode)
        rows[mode] = s = bias_stats(o, o_ref, rep)
        print(f"fp16 fix_mode {mode}: z_mean {s['z_mean']:+.2f}  z_aligned {s['z_aligned']:+.2f}  "
              f"aligned_mean/mean|O| {s['aligned_mean'] / s['mean_abs_ref']:+.3e}")
    assert abs(rows[1]["z_mean"]) < 3 and abs(rows[1]["z_aligned"]) < 3

GQA_CASES = [(1, 4, 2, 300, 64, True, 1), (2, 8, 1, 256, 128, True, 5), (1, 6, 3, 384, 64, False, 3)]


@pytest.mark.parametrize("B,H,Hkv,N,d,causal,fix_mode", GQA_CASES,
                         ids=[f"B{b}H{h}kv{k}N{n}d{d}{'c' if c else 'f'}fix{m}" for b, h, k, n, d, c, m in GQA_CASES])
def test_f16_gqa_parity(fa, B, H, Hkv, N, d, causal, fix_mode):
    g = torch.Generator().manual_seed(N + H)
    q, do = (torch.randn(B, H, N, d, generator=g).half() for _ in range(2))
    k, v = (torch.randn(B, Hkv, N, d, generator=g).half() for _ in range(2))
    scale = d ** -0.5
    dev = torch.device("cuda")
    qd, kd, vd, dod = (t.to(dev) for t in (q, k, v, do))
    o, lse = fa.attention_fwd(qd, kd, vd, causal=causal, scale=scale, fix_mode=fix_mode)
    dq, dk, dv = fa.attention_bwd(qd, kd, vd, o, lse, dod, causal=causal, scale=scale)
    torch.cuda.synchronize()
    assert fa.fa_check_device_error() == 0
    assert o.dtype == dq.dtype == dk.dtype == torch.float16 and dk.shape == k.shape
    grp = H // Hkv
    ke, ve = gqa_expand(k, grp), gqa_expand(v, grp)
    o_ref, lse_ref = attention_fwd(q, ke, ve, causal, scale)
    assert np.abs(o.float().cpu().numpy() - o_ref).max() <= O_ATOL
    assert lse_rel_err(lse.cpu().numpy(), lse_ref) <= LSE_RTOL
    dq_ref, dk_rep, dv_rep = attention_bwd(q, ke, ve, do, causal, scale)
    refs = {"dq": dq_ref, "dk": gqa_reduce(dk_rep, grp), "dv": gqa_reduce(dv_rep, grp)}
    for name, t in (("dq", dq), ("dk", dk), ("dv", dv)):
        err = normwise_rel_err(t.float().cpu().numpy(), refs[name])
        assert err <= GRAD_RTOL, (name, err)


def test_debug_call_matches_plain_forward(fa):
    """fa_fwd_debug runs the kernel fa_fwd_ex runs, with the records switched
    on: O and LSE bit for bit, in both element formats and every fix_mode."""
    dev = torch.device("cuda")
    g = torch.Generator().manual_seed(9)
    B, H, N, d = 1, 2, 333, 64
    for dtype in (torch.bfloat16, torch.float16):
        q, k, v = (torch.randn(B, H, N, d, generator=g).to(dtype).to(dev) for _ in range(3))
        for fix_mode in range(6):
            o1, lse1 = fa.attention_fwd(q, k, v, causal=True, scale=0.125, fix_mode=fix_mode)
            o2, lse2, ties, hits = fa.attention_fwd(q, k, v, causal=True, scale=0.125, fix_mode=fix_mode,
                                                    ties=True, one_hit=True)
            torch.cuda.synchronize()
            assert fa.fa_check_device_error() == 0
            assert torch.equal(o1, o2) and torch.equal(lse1, lse2), (dtype, fix_mode)
            # every row has a maximum; N(0,1) scores repeat only by coincidence
            assert bool(((ties & fa.TIE_COUNT_MASK) >= 1).all()) and bool((hits >= 0).all())
