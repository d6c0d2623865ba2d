"""Pins for the FP64 oracle: it is checked against things other than itself.

The pages print no worked example, so the oracle is pinned by
* brute force: scalar Python loops of the attention definition on tiny inputs
  ("Is Flash Attention Stable?", the standard-attention definition it measures
  FlashAttention against);
* closed forms: equal scores give the (prefix) mean of V, one key gives V_0,
  a dominant score gives that key's value row;
* invariants: rows of P sum to one (V = 1 gives O = 1), key permutation
  equivariance, causal locality, shift invariance of the exact result;
* finite differences of the brute-force forward for the backward pass;
* torch's CPU float32 -> bf16 cast for the bf16 rounding;
* the fix's defining property ("Why Low-Precision Transformer Training Fails",
  mechanism 2): on repeated-max rows every P_bar, the maxima included, is
  strictly below 1 (exactly 1 - 2^-8 at the maxima); without it they are 1;
* the fix variants: the maxima land on 0.5 (fix_mode 2) and on exp(-1/16),
  0.9375 after rounding (fix_mode 3); the self-normalised mode (4) gives O = 1
  exactly for V = 1, which the unrounded denominator does not; LSE is the
  unrounded log-sum-exp in every mode;
* grouped-query attention: scalar loops with the explicit head mapping, and
  central finite differences for the gradients of a shared K/V head;
* fp16 rounding against torch's fp16 cast, and the fix with fp16 P_bar
  (maxima at 1 - 2^-11);
* the near-tie detector (fix_mode 5): counts against scalar loops with
  math.exp and torch's bf16 cast on inputs with near ties but no exact ones,
  and every P_bar below 1 on the rows it raises.

A mutation suite then plants plausible mistakes in a copy of the oracle's
source and checks that each one trips at least one pin.
"""
import math
import os
import types

import numpy as np
import pytest
import torch

from oracle import attention64 as ORACLE

ORACLE_SRC = os.path.join(os.path.dirname(ORACLE.__file__), "attention64.py")


# ----------------------------------------------------------------------------
# independent scalar references (pure Python loops, tiny inputs only)
# ----------------------------------------------------------------------------

def brute_fwd(q, k, v, causal, scale):
    """Scalar attention of one head: lists in, lists out."""
    n, d, dv = len(q), len(q[0]), len(v[0])
    out, lse = [], []
    for i in range(n):
        keys = range(i + 1) if causal else range(n)
        s = [scale * sum(q[i][t] * k[j][t] for t in range(d)) for j in keys]
        mx = max(s)
        e = [math.exp(x - mx) for x in s]
        z = sum(e)
        out.append([sum(e[a] * v[j][c] for a, j in enumerate(keys)) / z for c in range(dv)])
        lse.append(mx + math.log(z))
    return out, lse


def brute_ties(q, k, causal):
    n, d = len(q), len(q[0])
    res = []
    for i in range(n):
        keys = range(i + 1) if causal else range(n)
        s = [sum(q[i][t] * k[j][t] for t in range(d)) for j in keys]
        res.append(sum(1 for x in s if x == max(s)))
    return res


def _rand(rng, *shape, scale=1.0):
    return scale * rng.standard_normal(shape)


# ----------------------------------------------------------------------------
# pin suites: each takes an oracle module and returns the names of failed pins
# ----------------------------------------------------------------------------

def fwd_pins(M):
    failed = []
    rng = np.random.default_rng(1)
    # P1 brute force, causal and not, odd sizes
    ok = True
    for causal in (True, False):
        q, k, v = _rand(rng, 1, 2, 5, 3), _rand(rng, 1, 2, 5, 3), _rand(rng, 1, 2, 5, 4)
        o, lse = M.attention_fwd(q, k, v, causal, 0.7)
        for h in range(2):
            bo, bl = brute_fwd(q[0, h].tolist(), k[0, h].tolist(), v[0, h].tolist(), causal, 0.7)
            ok &= np.allclose(o[0, h], bo, rtol=0, atol=1e-12)
            ok &= np.allclose(lse[0, h], bl, rtol=0, atol=1e-12)
    if not ok:
        failed.append("brute_force")
    # P2 equal scores: Q = 0 -> prefix mean of V and LSE = log(#visible)
    n = 9
    q = np.zeros((1, 1, n, 4))
    k, v = _rand(rng, 1, 1, n, 4), _rand(rng, 1, 1, n, 3)
    o, lse = M.attention_fwd(q, k, v, True, 0.5)
    pref = np.cumsum(v[0, 0], axis=0) / np.arange(1, n + 1)[:, None]
    if not (np.allclose(o[0, 0], pref, atol=1e-13) and np.allclose(lse[0, 0], np.log(np.arange(1, n + 1)), atol=1e-13)):
        failed.append("equal_scores")
    o, lse = M.attention_fwd(q, k, v, False, 0.5)
    if not (np.allclose(o[0, 0], v[0, 0].mean(0), atol=1e-13) and np.allclose(lse[0, 0], math.log(n), atol=1e-13)):
        failed.append("equal_scores_full")
    # P3 a single key: O = V_0, LSE = scale * q.k
    q, k, v = _rand(rng, 1, 1, 1, 5), _rand(rng, 1, 1, 1, 5), _rand(rng, 1, 1, 1, 5)
    o, lse = M.attention_fwd(q, k, v, True, 0.3)
    if not (np.allclose(o, v, atol=1e-14) and abs(lse[0, 0, 0] - 0.3 * float(q[0, 0, 0] @ k[0, 0, 0])) < 1e-13):
        failed.append("single_key")
    # P4 rows of P sum to one: V = 1 gives O = 1
    q, k = _rand(rng, 2, 1, 7, 3, scale=3), _rand(rng, 2, 1, 7, 3, scale=3)
    o, _ = M.attention_fwd(q, k, np.ones((2, 1, 7, 2)), True, 1.0)
    if not np.allclose(o, 1.0, atol=1e-13):
        failed.append("rows_sum_to_one")
    # P5 key permutation equivariance (non-causal): permute K and V rows together
    q, k, v = _rand(rng, 1, 1, 6, 3), _rand(rng, 1, 1, 6, 3), _rand(rng, 1, 1, 6, 3)
    perm = rng.permutation(6)
    o1, l1 = M.attention_fwd(q, k, v, False, 0.9)
    o2, l2 = M.attention_fwd(q, k[:, :, perm], v[:, :, perm], False, 0.9)
    if not (np.allclose(o1, o2, atol=1e-13) and np.allclose(l1, l2, atol=1e-13)):
        failed.append("permutation")
    # P6 causal locality: rows <= i0 ignore keys/values beyond i0
    q, k, v = _rand(rng, 1, 1, 8, 3), _rand(rng, 1, 1, 8, 3), _rand(rng, 1, 1, 8, 3)
    k2, v2 = k.copy(), v.copy()
    k2[:, :, 5:] += 10.0
    v2[:, :, 5:] -= 3.0
    o1, l1 = M.attention_fwd(q, k, v, True, 1.0)
    o2, l2 = M.attention_fwd(q, k2, v2, True, 1.0)
    if not (np.array_equal(o1[:, :, :5], o2[:, :, :5]) and np.array_equal(l1[:, :, :5], l2[:, :, :5])
            and not np.allclose(o1[:, :, 5:], o2[:, :, 5:])):
        failed.append("causal_locality")
    # P7 a dominant score: S_ij* = G above every other score pulls O_i to V_j*
    n, G = 6, 30.0
    k = _rand(rng, 1, 1, n, 4, scale=1e-3)
    q = np.zeros((1, 1, n, 4))
    q[0, 0, :, 0] = G
    k[0, 0, 2, 0] = 1.0
    v = _rand(rng, 1, 1, n, 3)
    o, _ = M.attention_fwd(q, k, v, False, 1.0)
    bound = (n - 1) * math.exp(-(G - 2 * G * 1e-3 * 4)) * 2 * np.abs(v).max()
    if not np.all(np.abs(o[0, 0] - v[0, 0, 2]) <= bound):
        failed.append("dominant_score")
    return failed


def bwd_pins(M):
    """Central finite differences of the brute-force forward, L = sum(dO * O)."""
    failed = []
    rng = np.random.default_rng(2)
    for causal in (True, False):
        q, k, v = _rand(rng, 1, 1, 4, 3), _rand(rng, 1, 1, 4, 3), _rand(rng, 1, 1, 4, 2)
        do = _rand(rng, 1, 1, 4, 2)
        scale = 0.8
        dq, dk, dv = M.attention_bwd(q, k, v, do, causal, scale)

        def loss(qq, kk, vv):
            o, _ = brute_fwd(qq[0, 0].tolist(), kk[0, 0].tolist(), vv[0, 0].tolist(), causal, scale)
            return float(np.sum(np.asarray(o) * do[0, 0]))

        h = 1e-6
        for name, x, g in (("dq", q, dq), ("dk", k, dk), ("dv", v, dv)):
            fd = np.zeros_like(x)
            for idx in np.ndindex(*x.shape):
                xp, xm = x.copy(), x.copy()
                xp[idx] += h
                xm[idx] -= h
                args_p = {"dq": (xp, k, v), "dk": (q, xp, v), "dv": (q, k, xp)}[name]
                args_m = {"dq": (xm, k, v), "dk": (q, xm, v), "dv": (q, k, xm)}[name]
                fd[idx] = (loss(*args_p) - loss(*args_m)) / (2 * h)
            if not np.allclose(g, fd, rtol=1e-6, atol=1e-8):
                failed.append(f"fd_{name}_{'causal' if causal else 'full'}")
    return failed


def bf16_pins(M):
    failed = []
    rng = np.random.default_rng(3)
    x = np.concatenate([
        rng.standard_normal(20000).astype(np.float32),
        (rng.standard_normal(20000) * 1e-38).astype(np.float32),   # subnormal range of bf16
        (rng.standard_normal(5000) * 1e37).astype(np.float32),
        np.exp(rng.uniform(-30, 0, 20000)).astype(np.float32),      # the range of softmax weights
    ])
    edges = np.array([0.0, -0.0, 1.0, 1 + 2 ** -8, 1 + 3 * 2 ** -8, 1 - 2 ** -9, 1 - 3 * 2 ** -9,
                      0.99609375, 2.0 ** -126, 2.0 ** -133, 2.0 ** -134, 3 * 2.0 ** -135, 2.0 ** -149,
                      3.3895313892515355e38, 3.3961e38, 3.4e38, np.inf, -np.inf], dtype=np.float32)
    x = np.concatenate([x, edges, -edges])
    ref = torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy()
    got = M.bf16_round(x.astype(np.float64))
    same = (got == ref) | (np.isnan(got) & np.isnan(ref))
    signs = np.signbit(got) == np.signbit(ref)
    if not (same.all() and signs.all()):
        failed.append("torch_cast")
    nan = M.bf16_round(np.array([np.nan]))
    if not np.isnan(nan).all():
        failed.append("nan")
    return failed


def fp16_pins(M):
    """fp16 rounding against torch's float32 -> float16 cast, and the fix's
    property with fp16 P_bar: the maxima of repeated-max rows land on
    1 - 2^-11, the largest fp16 value below 1."""
    failed = []
    rng = np.random.default_rng(13)
    x = np.concatenate([
        rng.standard_normal(20000).astype(np.float32),
        (rng.standard_normal(20000) * 1e-6).astype(np.float32),     # fp16 subnormals
        (rng.standard_normal(5000) * 3e4).astype(np.float32),
        np.exp(rng.uniform(-20, 0, 20000)).astype(np.float32),
    ])
    edges = np.array([0.0, -0.0, 1.0, 1 - 2 ** -12, 1 - 3 * 2 ** -12, 1 - 2 ** -11, 2.0 ** -14, 2.0 ** -24,
                      2.0 ** -25, 3 * 2.0 ** -26, 65504.0, 65519.0, 65520.0, 7e4, np.inf], dtype=np.float32)
    x = np.concatenate([x, edges, -edges])
    ref = torch.from_numpy(x).to(torch.float16).to(torch.float64).numpy()
    got = M.fp16_round(x.astype(np.float64))
    if not (np.all((got == ref) | (np.isnan(got) & np.isnan(ref))) and np.all(np.signbit(got) == np.signbit(ref))):
        failed.append("fp16_torch_cast")
    q, k, v = _tie_inputs(rng)
    ties = np.stack([np.asarray(brute_ties(q[0, h].tolist(), k[0, h].tolist(), True)) for h in range(2)])
    _, _, p1 = M.attention_fwd_bf16p(q, k, v, True, 0.5, 1, return_pbar=True, fmt="fp16")
    _, _, p0 = M.attention_fwd_bf16p(q, k, v, True, 0.5, 0, return_pbar=True, fmt="fp16")
    ok = True
    for h in range(2):
        for i in range(q.shape[2]):
            r1, r0 = p1[0, h, i, : i + 1], p0[0, h, i, : i + 1]
            if ties[h, i] >= 2:
                ok &= r1.max() == 1.0 - 2.0 ** -11 and np.sum(r1 == 1.0 - 2.0 ** -11) == ties[h, i]
            else:
                ok &= np.array_equal(r1, r0) and r0.max() == 1.0
            # P_bar is on the fp16 grid (torch's cast, not the oracle's)
            ok &= np.array_equal(torch.from_numpy(r1).to(torch.float16).double().numpy(), r1)
    if not ok:
        failed.append("fp16_fix_property")
    # the variants with fp16 P_bar: where the maxima of a repeated-max row land,
    # unrounded and after the fp16 rounding.  exp(-1/16) = 0.9394130..., and
    # 2^11 times that is 1923.918..., so fp16 rounds it to 1924 / 2048.
    for fix, top, top16 in ((2, 0.5, 0.5), (3, float(np.exp(-1.0 / 16.0)), 1924.0 / 2048.0)):
        _, _, pu = M.attention_fwd_bf16p(q, k, v, True, 0.5, fix, round_p=False, return_pbar=True, fmt="fp16")
        _, _, pr = M.attention_fwd_bf16p(q, k, v, True, 0.5, fix, return_pbar=True, fmt="fp16")
        ok = True
        for h in range(2):
            for i in range(q.shape[2]):
                ru, rr = pu[0, h, i, : i + 1], pr[0, h, i, : i + 1]
                if ties[h, i] >= 2:
                    ok &= abs(ru.max() - top) <= 1e-15 and np.sum(np.abs(ru - top) <= 1e-15) == ties[h, i]
                    ok &= rr.max() == top16
                else:
                    ok &= ru.max() == 1.0 and rr.max() == 1.0
        if not ok:
            failed.append(f"fp16_variant_maxima_fix{fix}")
    # self-normalised with fp16 P_bar: V = 1 gives O = 1 exactly
    o4, _ = M.attention_fwd_bf16p(q, k, np.ones_like(v), True, 0.5, 4, fmt="fp16")
    if not np.allclose(o4, 1.0, atol=1e-14, rtol=0):
        failed.append("fp16_self_normalised_ones")
    # LSE stays the unrounded log-sum-exp of the definition in every mode
    _, lse_exact = M.attention_fwd(q, k, v, True, 0.5)
    for fix in range(6):
        _, le = M.attention_fwd_bf16p(q, k, v, True, 0.5, fix, fmt="fp16")
        if not np.allclose(le, lse_exact, atol=1e-13, rtol=0):
            failed.append(f"fp16_lse_unrounded_fix{fix}")
    # near ties in fp16: every query is (2, 0), key 2 is key 0 moved by a gap
    # g in its first coordinate, so from row 2 on the maximum is key 2 and key
    # 0 trails it by g in S.  Head 0: g = 1e-4, P = exp(-g) rounds to 1 in fp16
    # and in bf16.  Head 1: g = 1e-3, P rounds to 1 in bf16 (>= 1 - 2^-9) but
    # not in fp16 (< 1 - 2^-12).  Counts by brute force (math.exp, torch's
    # casts), then fix_mode 5's property with fp16 P_bar.
    n = 7
    qn = np.zeros((1, 2, n, 2))
    qn[..., 0] = 2.0
    kn = np.zeros((1, 2, n, 2))
    kn[0, :, 0] = (1.0, 0.0)
    kn[0, :, 1] = (0.0, 1.0)
    kn[0, :, 3:] = (0.5, 0.0)
    kn[0, 0, 2] = (1.0 + 1e-4, 0.0)
    kn[0, 1, 2] = (1.0 + 1e-3, 0.0)
    vn = rng.standard_normal((1, 2, n, 3))
    sc = 0.5
    brute16 = np.zeros((1, 2, n), dtype=np.int64)
    brute_bf = np.zeros((1, 2, n), dtype=np.int64)
    exact = np.zeros((1, 2, n), dtype=np.int64)
    for h in range(2):
        for i in range(n):
            row = [sc * sum(qn[0, h, i, c] * kn[0, h, j, c] for c in range(qn.shape[3])) for j in range(i + 1)]
            mx = max(row)
            pr = torch.tensor([math.exp(r - mx) for r in row], dtype=torch.float64).float()
            brute16[0, h, i] = int((pr.to(torch.float16).float() == 1.0).sum())
            brute_bf[0, h, i] = int((pr.to(torch.bfloat16).float() == 1.0).sum())
            exact[0, h, i] = sum(r == mx for r in row)
    if not np.array_equal(M.near_tie_counts(qn, kn, True, sc, fmt="fp16"), brute16):
        failed.append("fp16_near_tie_counts")
    if not (np.any((brute16 >= 2) & (exact < 2)) and np.any(brute16 != brute_bf)):
        failed.append("fp16_near_tie_fixture")
    _, _, p5 = M.attention_fwd_bf16p(qn, kn, vn, True, sc, 5, return_pbar=True, fmt="fp16")
    _, _, p0 = M.attention_fwd_bf16p(qn, kn, vn, True, sc, 0, return_pbar=True, fmt="fp16")
    ok = True
    for h in range(2):
        for i in range(n):
            r5, r0 = p5[0, h, i, : i + 1], p0[0, h, i, : i + 1]
            if brute16[0, h, i] >= 2:
                ok &= bool(np.all(r5 < 1.0)) and np.sum(r0 == 1.0) == brute16[0, h, i]
            else:
                ok &= np.array_equal(r5, r0)
    if not ok:
        failed.append("fp16_near_tie_fix_property")
    return failed


def _tie_inputs(rng, n=8, d=3):
    """Small integer-valued inputs with duplicated keys: exact ties by construction."""
    q = rng.integers(-2, 3, size=(1, 2, n, d)).astype(np.float64)
    k = rng.integers(-2, 3, size=(1, 2, n, d)).astype(np.float64)
    v = rng.standard_normal((1, 2, n, 4))
    k[0, 0, 5] = k[0, 0, 1]
    k[0, 1, 6] = k[0, 1, 0]
    return q, k, v


def emulation_pins(M):
    failed = []
    rng = np.random.default_rng(4)
    # E1 without rounding the emulation is the exact definition, whatever the fix does
    q, k, v = _rand(rng, 1, 2, 9, 4), _rand(rng, 1, 2, 9, 4), _rand(rng, 1, 2, 9, 4)
    k[0, 0, 7] = k[0, 0, 2]
    o, lse = M.attention_fwd(q, k, v, True, 0.6)
    for fix in (0, 1, 2, 3, 4):
        oe, le = M.attention_fwd_bf16p(q, k, v, True, 0.6, fix, round_p=False)
        if not (np.allclose(oe, o, atol=1e-13) and np.allclose(le, lse, atol=1e-13)):
            failed.append(f"unrounded_equals_exact_fix{fix}")
    # E2 the fix's defining property on repeated-max rows
    q, k, v = _tie_inputs(rng)
    ties = np.asarray(brute_ties(q[0, 0].tolist(), k[0, 0].tolist(), True))
    ties1 = np.asarray(brute_ties(q[0, 1].tolist(), k[0, 1].tolist(), True))
    all_ties = np.stack([ties, ties1])
    _, _, p0 = M.attention_fwd_bf16p(q, k, v, True, 0.5, 0, return_pbar=True)
    _, _, p1 = M.attention_fwd_bf16p(q, k, v, True, 0.5, 1, return_pbar=True)
    rep = all_ties >= 2
    if not rep.any():
        failed.append("no_repeated_rows_in_fixture")
    ok = True
    for h in range(2):
        for i in range(q.shape[2]):
            row0, row1 = p0[0, h, i, : i + 1], p1[0, h, i, : i + 1]
            if rep[h, i]:
                ok &= row0.max() == 1.0 and np.sum(row0 == 1.0) == all_ties[h, i]
                ok &= row1.max() == 1.0 - 2.0 ** -8 and np.all(row1 < 1.0)
                ok &= np.sum(row1 == 1.0 - 2.0 ** -8) == all_ties[h, i]
            else:
                ok &= np.array_equal(row0, row1) and row0.max() == 1.0
    if not ok:
        failed.append("fix_property")
    # E3 rounding P to bf16 moves O by at most 2^-8 * max|V| (unit roundoff of bf16)
    q, k, v = _rand(rng, 2, 2, 16, 8), _rand(rng, 2, 2, 16, 8), _rand(rng, 2, 2, 16, 8)
    o, lse = M.attention_fwd(q, k, v, True, 0.35)
    for fix in (0, 1):
        oe, le = M.attention_fwd_bf16p(q, k, v, True, 0.35, fix)
        bound = 2.0 ** -8 * np.abs(v).max(axis=2, keepdims=True)
        if not (np.all(np.abs(oe - o) <= bound) and np.allclose(le, lse, atol=1e-13)):
            failed.append(f"rounding_bound_fix{fix}")
        if np.abs(oe - o).max() < 1e-6:
            failed.append(f"rounding_not_applied_fix{fix}")
    # P_bar lies on the bf16 grid (checked with torch's cast, not the oracle's)
    _, _, pb = M.attention_fwd_bf16p(q, k, v, True, 0.35, 1, return_pbar=True)
    pb32 = pb.astype(np.float32)
    if not (np.array_equal(pb32.astype(np.float64), pb) and
            np.array_equal(torch.from_numpy(pb32).to(torch.bfloat16).float().numpy(), pb32)):
        failed.append("pbar_off_bf16_grid")
    # E5 the variants of the fix: where each puts the maxima of a repeated-max
    # row (unrounded, and after the bf16 rounding), and the self-normalised mode
    q, k, v = _tie_inputs(rng)
    ties = np.stack([np.asarray(brute_ties(q[0, h].tolist(), k[0, h].tolist(), True)) for h in range(2)])
    for fix, top, top_bf16 in ((2, 0.5, 0.5), (3, float(np.exp(-1.0 / 16.0)), 0.9375)):
        _, _, pu = M.attention_fwd_bf16p(q, k, v, True, 0.5, fix, round_p=False, return_pbar=True)
        _, _, pr = M.attention_fwd_bf16p(q, k, v, True, 0.5, fix, return_pbar=True)
        ok = True
        for h in range(2):
            for i in range(q.shape[2]):
                ru, rr = pu[0, h, i, : i + 1], pr[0, h, i, : i + 1]
                if ties[h, i] >= 2:
                    ok &= abs(ru.max() - top) <= 1e-15 and np.sum(np.abs(ru - top) <= 1e-15) == ties[h, i]
                    ok &= rr.max() == top_bf16 and np.all(ru < 1.0)
                else:
                    ok &= ru.max() == 1.0
        if not ok:
            failed.append(f"variant_maxima_fix{fix}")
    # self-normalised: V = 1 gives O = 1 exactly, which the unrounded
    # denominator does not; LSE stays the unrounded log-sum-exp in every mode
    ones = np.ones_like(v)
    o4, _ = M.attention_fwd_bf16p(q, k, ones, True, 0.5, 4)
    o0, _ = M.attention_fwd_bf16p(q, k, ones, True, 0.5, 0)
    if not (np.allclose(o4, 1.0, atol=1e-14, rtol=0) and not np.allclose(o0, 1.0, atol=1e-6, rtol=0)):
        failed.append("self_normalised_ones")
    _, lse_exact = M.attention_fwd(q, k, v, True, 0.5)
    for fix in (0, 1, 2, 3, 4):
        _, le = M.attention_fwd_bf16p(q, k, v, True, 0.5, fix)
        if not np.allclose(le, lse_exact, atol=1e-13, rtol=0):
            failed.append(f"lse_unrounded_fix{fix}")
    # E6 near ties: brute-force count (math.exp, torch's bf16 cast) and the
    # defining property of fix_mode 5 on the rows it raises
    from flashattention_bf16_fwd_b200.workloads import WORKLOADS as _W, make_inputs as _mk
    x = _mk(_W["tiny"].with_shape(H=2, N=24, d=8, structure="argmax_near", frac=0.5), seed=7, with_grad=False)
    qn, kn, vn = (x[n].double().numpy() for n in ("q", "k", "v"))
    sc = x["scale"]
    brute = np.zeros((1, 2, 24), dtype=np.int64)
    exact_rep = np.zeros((1, 2, 24), dtype=bool)
    for h in range(2):
        for i in range(24):
            row = [sc * sum(qn[0, h, i, c] * kn[0, h, j, c] for c in range(8)) for j in range(i + 1)]
            mx = max(row)
            pr = torch.tensor([math.exp(r - mx) for r in row], dtype=torch.float64)
            brute[0, h, i] = int((pr.float().to(torch.bfloat16).float() == 1.0).sum())
            exact_rep[0, h, i] = sum(r == mx for r in row) >= 2
    near = M.near_tie_counts(qn, kn, True, sc)
    if not np.array_equal(near, brute):
        failed.append("near_tie_counts")
    if not np.any((brute >= 2) & ~exact_rep):
        failed.append("no_near_only_rows_in_fixture")
    _, _, p5 = M.attention_fwd_bf16p(qn, kn, vn, True, sc, 5, return_pbar=True)
    _, _, p0 = M.attention_fwd_bf16p(qn, kn, vn, True, sc, 0, return_pbar=True)
    ok = True
    for h in range(2):
        for i in range(24):
            r5, r0 = p5[0, h, i, : i + 1], p0[0, h, i, : i + 1]
            if brute[0, h, i] >= 2:
                ok &= bool(np.all(r5 < 1.0)) and np.sum(r0 == 1.0) == brute[0, h, i]
            else:
                ok &= np.array_equal(r5, r0)
    if not ok:
        failed.append("near_tie_fix_property")
    # E4 exact tie counts against brute force
    q, k, v = _tie_inputs(rng)
    for causal in (True, False):
        got = M.tie_counts(q, k, causal)
        exp = np.stack([brute_ties(q[0, h].tolist(), k[0, h].tolist(), causal) for h in range(2)])
        if not np.array_equal(got[0], exp):
            failed.append(f"tie_counts_{'causal' if causal else 'full'}")
    return failed


def gqa_pins(M):
    """Grouped-query attention: scalar loops with the explicit head mapping
    (query head h reads key/value head h // group), and the gradient of a
    shared head against central finite differences of those loops."""
    failed = []
    rng = np.random.default_rng(11)
    B, Hq, Hkv, N, d = 1, 4, 2, 5, 3
    g = Hq // Hkv
    q, k, v = _rand(rng, B, Hq, N, d), _rand(rng, B, Hkv, N, d), _rand(rng, B, Hkv, N, d)
    do = _rand(rng, B, Hq, N, d)
    sc = 0.7

    def brute_o(qq, kk, vv):
        out = np.zeros((B, Hq, N, d))
        for h in range(Hq):
            hk = h // g
            for i in range(N):
                s = [sc * sum(qq[0, h, i, c] * kk[0, hk, j, c] for c in range(d)) for j in range(i + 1)]
                mx = max(s)
                e = [math.exp(x - mx) for x in s]
                tot = sum(e)
                for c in range(d):
                    out[0, h, i, c] = sum(e[j] * vv[0, hk, j, c] for j in range(i + 1)) / tot
        return out

    o, _ = M.attention_fwd(q, M.gqa_expand(k, g), M.gqa_expand(v, g), True, sc)
    if not np.allclose(o, brute_o(q, k, v), atol=1e-13):
        failed.append("gqa_forward")
    _, dk_rep, dv_rep = M.attention_bwd(q, M.gqa_expand(k, g), M.gqa_expand(v, g), do, True, sc)
    dk, dv = M.gqa_reduce(dk_rep, g), M.gqa_reduce(dv_rep, g)
    eps = 1e-6
    for name, arr, grad in (("k", k, dk), ("v", v, dv)):
        num = np.zeros_like(arr)
        for idx in np.ndindex(arr.shape):
            a1, a2 = arr.copy(), arr.copy()
            a1[idx] += eps
            a2[idx] -= eps
            kk1, vv1 = (a1, v) if name == "k" else (k, a1)
            kk2, vv2 = (a2, v) if name == "k" else (k, a2)
            num[idx] = (np.sum(do * brute_o(q, kk1, vv1)) - np.sum(do * brute_o(q, kk2, vv2))) / (2 * eps)
        if not np.allclose(grad, num, rtol=1e-6, atol=1e-8):
            failed.append(f"gqa_d{name}")
    if not np.array_equal(M.gqa_reduce(M.gqa_expand(k, g), g), g * np.asarray(k, np.float64)):
        failed.append("gqa_expand_reduce")
    return failed


# ----------------------------------------------------------------------------
# the oracle passes every pin
# ----------------------------------------------------------------------------

def test_forward_pins():
    assert fwd_pins(ORACLE) == []


def test_backward_pins_finite_differences():
    assert bwd_pins(ORACLE) == []


def test_bf16_rounding_matches_torch_cast():
    assert bf16_pins(ORACLE) == []


def test_emulation_and_fix_pins():
    assert emulation_pins(ORACLE) == []


def test_gqa_pins():
    assert gqa_pins(ORACLE) == []


def test_fp16_pins():
    assert fp16_pins(ORACLE) == []


def test_delta_constant():
    # the shift maps a maximum to exactly the largest bf16 value below 1
    assert ORACLE.bf16_round(np.exp(-ORACLE.DELTA_NAT)) == 0.99609375
    assert ORACLE.bf16_round(2.0 ** -ORACLE.DELTA_LOG2) == 0.99609375
    assert abs(ORACLE.DELTA_NAT - ORACLE.DELTA_LOG2 * math.log(2)) < 1e-16


def test_hand_worked_example():
    """tests/golden/handworked_2x2.txt: two keys whose scores differ by ln 3."""
    path = os.path.join(os.path.dirname(__file__), "golden", "handworked_2x2.txt")
    vals = {}
    for line in open(path):
        line = line.split("#", 1)[0].strip()
        if line:
            key, rhs = line.split("=", 1)
            vals[key.strip()] = np.array([float(eval(t, {"ln": math.log, "sqrt": math.sqrt}))
                                          for t in rhs.split()])
    q = vals["q"].reshape(1, 1, 1, 2)
    k = vals["k"].reshape(1, 1, 2, 2)
    v = vals["v"].reshape(1, 1, 2, 2)
    # one query against two keys, non-causal
    o, lse = ORACLE.attention_fwd(np.repeat(q, 2, axis=2), k, v, False, float(vals["scale"][0]))
    assert np.allclose(o[0, 0, 0], vals["o"], atol=1e-15)
    assert abs(lse[0, 0, 0] - vals["lse"][0]) < 1e-15


# ----------------------------------------------------------------------------
# planted mistakes: each must trip at least one pin
# ----------------------------------------------------------------------------

MUTATIONS = [
    ("fwd_drops_scale", "s = scale * (q[b, h] @ k[b, h].T)\n        s = np.where(vis, s, -np.inf)\n        m = s.max(axis=1, keepdims=True)\n        e = np.exp(s - m)\n        l = e",
     "s = (q[b, h] @ k[b, h].T)\n        s = np.where(vis, s, -np.inf)\n        m = s.max(axis=1, keepdims=True)\n        e = np.exp(s - m)\n        l = e"),
    ("fwd_wrong_operand", "o[b, h] = p @ v[b, h]\n        lse", "o[b, h] = p @ k[b, h][:, : v.shape[-1]]\n        lse"),
    ("mask_off_by_one", "np.tril(np.ones((n, n), dtype=bool))", "np.tril(np.ones((n, n), dtype=bool), k=1)"),
    ("lse_drops_max", "lse[b, h] = m[:, 0] + np.log(l[:, 0])", "lse[b, h] = np.log(l[:, 0])"),
    ("dv_not_transposed", "dv[b, h] = p.T @ do[b, h]", "dv[b, h] = p @ do[b, h]"),
    ("ds_drops_D", "ds = p * (dp - D)", "ds = p * dp"),
    ("ds_wrong_sign", "ds = p * (dp - D)", "ds = p * (D - dp)"),
    ("dk_not_transposed", "dk[b, h] = scale * (ds.T @ q[b, h])", "dk[b, h] = scale * (ds @ q[b, h])"),
    ("dq_drops_scale", "dq[b, h] = scale * (ds @ k[b, h])", "dq[b, h] = (ds @ k[b, h])"),
    ("bf16_one_bit_short", "q_exp = np.maximum(e, -125) - 8", "q_exp = np.maximum(e, -125) - 7"),
    ("bf16_truncates", "q_exp = np.maximum(e, -125) - 8\n    r = np.ldexp(np.rint(np.ldexp(xf, -q_exp)), q_exp)",
     "q_exp = np.maximum(e, -125) - 8\n    r = np.ldexp(np.trunc(np.ldexp(xf, -q_exp)), q_exp)"),
    ("bf16_no_subnormals", "q_exp = np.maximum(e, -125) - 8", "q_exp = e - 8"),
    ("fix_on_every_row", "* (ties >= 2)", "* (ties >= 1)"),
    ("fix_wrong_delta", "DELTA_NAT = -np.log(1.0 - 2.0 ** -8)", "DELTA_NAT = -np.log(1.0 - 2.0 ** -6)"),
    ("emulation_skips_rounding", "pbar = round_fn(p) if round_p else p", "pbar = p"),
    ("ties_ignore_mask", "s = np.where(vis, q[b, h] @ k[b, h].T, -np.inf)\n        out[b, h]", "s = q[b, h] @ k[b, h].T\n        out[b, h]"),
    ("variant_shift_in_log2", "1: DELTA_NAT, 2: float(np.log(2.0))", "1: DELTA_NAT, 2: 1.0"),
    ("variant_off_grid_value", "3: 1.0 / 16.0, 4: 0.0, 5: DELTA_NAT}", "3: 1.0 / 8.0, 4: 0.0, 5: DELTA_NAT}"),
    ("self_normalised_unrounded_den", "den = pbar.sum(axis=1, keepdims=True) if", "den = l if"),
    ("near_ties_count_exact_ties", "ties = np.sum(round_fn(np.exp(s - m)) == 1.0, axis=1, keepdims=True)",
     "ties = np.sum(raw == raw.max(axis=1, keepdims=True), axis=1, keepdims=True)"),
    ("near_tie_no_shift", "4: 0.0, 5: DELTA_NAT}", "4: 0.0, 5: 0.0}"),
    ("near_tie_threshold_off", "out[b, h] = np.sum(round_fn(p) == 1.0, axis=1)", "out[b, h] = np.sum(p == 1.0, axis=1)"),
    ("gqa_expand_wrong_axis", "return np.repeat(_f64(x), group, axis=1)", "return np.tile(_f64(x), (1, group, 1, 1))"),
    ("gqa_reduce_mean", "return x.reshape(B, H // group, group, N, d).sum(axis=2)",
     "return x.reshape(B, H // group, group, N, d).mean(axis=2)"),
    ("fp16_one_bit_short", "q_exp = np.maximum(e, -13) - 11", "q_exp = np.maximum(e, -13) - 10"),
    ("fp16_no_subnormals", "q_exp = np.maximum(e, -13) - 11", "q_exp = e - 11"),
    ("fp16_fix_bf16_delta", "shifts = FIX_SHIFT_NAT if fmt == \"bf16\" else FIX_SHIFT_NAT_FP16",
     "shifts = FIX_SHIFT_NAT"),
    ("fp16_variant_shift_in_log2", "1: DELTA16_NAT, 2: float(np.log(2.0))", "1: DELTA16_NAT, 2: 1.0"),
    ("fp16_variant_off_grid_value", "3: 1.0 / 16.0, 4: 0.0, 5: DELTA16_NAT}", "3: 1.0 / 8.0, 4: 0.0, 5: DELTA16_NAT}"),
    ("fp16_near_tie_no_shift", "4: 0.0, 5: DELTA16_NAT}", "4: 0.0, 5: 0.0}"),
    ("fp16_near_tie_rounds_in_bf16", "round_fn = {\"bf16\": bf16_round, \"fp16\": fp16_round}[fmt]",
     "round_fn = bf16_round"),
    ("self_normalised_lse_from_pbar", "lse[b, h] = shift[:, 0] + np.log(l[:, 0])",
     "lse[b, h] = shift[:, 0] + np.log(den[:, 0])"),
]


def _mutant(old, new):
    src = open(ORACLE_SRC).read()
    assert src.count(old) == 1, f"mutation anchor not unique: {old!r}"
    mod = types.ModuleType("oracle_mutant")
    exec(compile(src.replace(old, new), "oracle_mutant", "exec"), mod.__dict__)
    return mod


@pytest.mark.parametrize("name,old,new", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_planted_mistake_is_caught(name, old, new):
    M = _mutant(old, new)
    failed = []
    for suite in (fwd_pins, bf16_pins, emulation_pins, bwd_pins, gqa_pins, fp16_pins):
        try:
            failed += suite(M)
        except Exception as exc:  # a mutant that cannot even run fails its pins
            failed.append(f"{suite.__name__}: {type(exc).__name__}")
        if failed:
            break
    assert failed, f"mutation {name} passed every pin"
