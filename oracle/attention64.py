"""FP64 CPU oracle for BF16 attention with the repeated-max fix.

TEST INFRASTRUCTURE ONLY.  Only the tests, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this module.  The product path (the
CUDA library and its Python binding) never calls it, and it shares no code with
that path: plain NumPy, whole N x N matrices, one (batch, head) pair at a time.

What it computes, and where each step is stated:

* Standard attention, the "baseline attention" of "Is Flash Attention Stable?"
  (chibakuma.com; sections "Flash Attention: from academic breakthrough to
  industry standard" and "What did Meta's study find?"):
  S = scale * Q K^T, P = softmax(S) per row, O = P V.  Computed here in FP64
  instead of FP32.  Causal masking (key j visible to query i iff j <= i) is the
  plain reading for decoder training (GPT-2 and Llama 2 on the pages).
* The log-sum-exp LSE_i = log sum_j exp(S_ij), the per-row statistic the
  recomputing backward pass needs (yicaiai article, abstract and section 5.1).
* The backward pass, written out from the chain rule of the definition above:
  dV = P^T dO, dP = dO V^T, D_i = sum_k dO_ik O_ik, dS = P * (dP - D),
  dQ = scale dS K, dK = scale dS^T Q (the gradients d loss/dQ, d loss/dK named
  in the yicaiai article, section 4.3).
* The safe-softmax shift and the BF16 rounding point of the unnormalised
  output ("Why Low-Precision Transformer Training Fails", admirer.cn summary,
  "mechanism 2"): P_bar = bf16(exp(S - m)), O = (P_bar V) / l.
* The fix (same section): per row, detect whether the maximum of S occurs more
  than once; if so raise the shift m so that every exponent, the ones at the
  maximum included, is strictly below 1.  Reading taken here (the pages leave
  the amount open): m' = m + delta with delta = -ln(1 - 2^-8), so the maxima
  map to exactly 1 - 2^-8 = 0.99609375, the largest bf16 value below 1.
* Variants of the fix, to measure which choices remove the bias (the pages
  leave the amount of the shift open and trace the bias to P_bar = 1 in the
  unnormalised output, same section): fix_mode 2 raises the shift by ln 2
  (maxima -> 0.5, on the bf16 grid), fix_mode 3 by 1/16 (maxima ->
  exp(-1/16) = 0.93941, off the grid: P_bar = 0.9375 there), and fix_mode 4
  keeps the plain shift but divides by the sum of the rounded P_bar instead of
  the unrounded P (a self-normalised output).  LSE is the unrounded
  log-sum-exp in every mode.
* The same in FP16 (the pages treat FP16 and BF16 together as the
  low-precision formats of the instability: yicaiai article, abstract):
  P_bar rounded to fp16, and the fix maps the maxima to 1 - 2^-11, the
  largest fp16 value below 1.  The variants carry over: fix_mode 2, 3 and 4
  as above, fix_mode 5 with the near-tie test made in fp16 (P rounds to 1 in
  fp16 when P >= 1 - 2^-12).
* Grouped-query attention (GQA/MQA head layouts, the Llama 2 family the
  chibakuma.com page names): H_q query heads share H_kv key/value heads,
  query head h reading key/value head h // (H_q / H_kv).  The forward is the
  definition above with K and V repeated over each group; the gradients of a
  shared K or V head are the sums over its group.
* A near-tie detector (fix_mode 5), after the same section's statement that
  the bias comes from probabilities of exactly 1: the shift is raised by
  delta when at least two entries of the row have P_bar == 1 under the plain
  shift (their P rounds to 1 in bf16), not only when S ties exactly.

Parity pins for every function live in tests/test_oracle_pins.py (brute force,
closed forms, invariants, finite differences, torch's bf16 cast).
"""
from __future__ import annotations

import numpy as np

__all__ = [
    "DELTA_LOG2", "DELTA_NAT", "DELTA16_NAT", "fp16_round", "FIX_SHIFT_NAT", "FIX_SHIFT_NAT_FP16", "SELF_NORMALISED_MODES", "NEAR_TIE_MODES", "bf16_round", "scores", "attention_fwd",
    "attention_bwd", "attention_fwd_bf16p", "tie_counts", "near_tie_counts", "gqa_expand", "gqa_reduce",
]

# Shift added to m on repeated-max rows, in log2 units and in natural-log units.
DELTA_LOG2 = -np.log2(1.0 - 2.0 ** -8)
DELTA_NAT = -np.log(1.0 - 2.0 ** -8)

# Shift (natural-log units) added on repeated-max rows for each fix_mode, and
# the modes whose output is normalised by the sum of the rounded P_bar.
FIX_SHIFT_NAT = {0: 0.0, 1: DELTA_NAT, 2: float(np.log(2.0)), 3: 1.0 / 16.0, 4: 0.0, 5: DELTA_NAT}
NEAR_TIE_MODES = (5,)
SELF_NORMALISED_MODES = (4,)

_BF16_MAX = (2.0 - 2.0 ** -7) * 2.0 ** 127
_FP16_MAX = (2.0 - 2.0 ** -10) * 2.0 ** 15

# The fix's shift for fp16 P_bar (natural-log units): maxima -> 1 - 2^-11.
DELTA16_NAT = -np.log(1.0 - 2.0 ** -11)

# FIX_SHIFT_NAT for fp16 P_bar: modes 1 and 5 land the maxima on 1 - 2^-11,
# the largest fp16 value below 1; modes 2, 3 and 4 do not depend on the format.
FIX_SHIFT_NAT_FP16 = {0: 0.0, 1: DELTA16_NAT, 2: float(np.log(2.0)), 3: 1.0 / 16.0, 4: 0.0, 5: DELTA16_NAT}


def bf16_round(x) -> np.ndarray:
    """Round to the nearest bf16 value, ties to even, returned as float64.

    bf16 keeps 8 significant bits and the float32 exponent range: the quantum
    of a normal value in [2^(e-1), 2^e) is 2^(e-8); below 2^-126 the quantum
    is fixed at 2^-133 (subnormals).  Results beyond the largest finite bf16
    value become infinities; NaN stays NaN; the sign of zero is kept.
    """
    x = np.asarray(x, dtype=np.float64)
    out = x.copy()
    fin = np.isfinite(x) & (x != 0.0)
    xf = x[fin]
    _, e = np.frexp(xf)
    q_exp = np.maximum(e, -125) - 8
    r = np.ldexp(np.rint(np.ldexp(xf, -q_exp)), q_exp)
    r = np.where(np.abs(r) > _BF16_MAX, np.copysign(np.inf, xf), r)
    # keep the sign of values that round to zero
    r = np.where(r == 0.0, np.copysign(0.0, xf), r)
    out[fin] = r
    return out


def fp16_round(x) -> np.ndarray:
    """Round to the nearest IEEE binary16 value, ties to even, returned as float64.

    fp16 keeps 11 significant bits: the quantum of a normal value in
    [2^(e-1), 2^e) is 2^(e-11); below 2^-14 the quantum is fixed at 2^-24
    (subnormals).  Results beyond 65504 become infinities; NaN stays NaN; the
    sign of zero is kept.
    """
    x = np.asarray(x, dtype=np.float64)
    out = x.copy()
    fin = np.isfinite(x) & (x != 0.0)
    xf = x[fin]
    _, e = np.frexp(xf)
    q_exp = np.maximum(e, -13) - 11
    r = np.ldexp(np.rint(np.ldexp(xf, -q_exp)), q_exp)
    r = np.where(np.abs(r) > _FP16_MAX, np.copysign(np.inf, xf), r)
    r = np.where(r == 0.0, np.copysign(0.0, xf), r)
    out[fin] = r
    return out


def _f64(a) -> np.ndarray:
    if hasattr(a, "detach"):
        a = a.detach().to("cpu").double().numpy()
    return np.asarray(a, dtype=np.float64)


def _mask(n: int, causal: bool) -> np.ndarray:
    """True where key j is visible to query i."""
    if not causal:
        return np.ones((n, n), dtype=bool)
    return np.tril(np.ones((n, n), dtype=bool))


def scores(q, k) -> np.ndarray:
    """Raw dot products Q K^T of one head, float64 [N, N] (no scale, no mask)."""
    return _f64(q) @ _f64(k).T


def _heads(*arrays):
    """Iterate over (b, h) for arrays shaped [B, H, N, d] (or [B, H, N])."""
    B, H = arrays[0].shape[:2]
    for b in range(B):
        for h in range(H):
            yield b, h


def attention_fwd(q, k, v, causal: bool, scale: float):
    """Exact attention: O [B,H,N,d] and LSE [B,H,N] (natural log), float64."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, H, N, d = q.shape
    o = np.empty((B, H, N, v.shape[-1]))
    lse = np.empty((B, H, N))
    vis = _mask(N, causal)
    for b, h in _heads(q):
        s = scale * (q[b, h] @ k[b, h].T)
        s = np.where(vis, s, -np.inf)
        m = s.max(axis=1, keepdims=True)
        e = np.exp(s - m)
        l = e.sum(axis=1, keepdims=True)
        p = e / l
        o[b, h] = p @ v[b, h]
        lse[b, h] = m[:, 0] + np.log(l[:, 0])
    return o, lse


def attention_bwd(q, k, v, do, causal: bool, scale: float):
    """Exact gradients (dQ, dK, dV) of sum(dO * O) for O = attention(Q, K, V)."""
    q, k, v, do = _f64(q), _f64(k), _f64(v), _f64(do)
    B, H, N, d = q.shape
    dq, dk, dv = np.empty_like(q), np.empty_like(k), np.empty_like(v)
    vis = _mask(N, causal)
    for b, h in _heads(q):
        s = scale * (q[b, h] @ k[b, h].T)
        s = np.where(vis, s, -np.inf)
        m = s.max(axis=1, keepdims=True)
        e = np.exp(s - m)
        p = e / e.sum(axis=1, keepdims=True)
        o = p @ v[b, h]
        dv[b, h] = p.T @ do[b, h]
        dp = do[b, h] @ v[b, h].T
        D = np.sum(do[b, h] * o, axis=1, keepdims=True)
        ds = p * (dp - D)
        dq[b, h] = scale * (ds @ k[b, h])
        dk[b, h] = scale * (ds.T @ q[b, h])
    return dq, dk, dv


def tie_counts(q, k, causal: bool) -> np.ndarray:
    """Per row, how many visible keys reach the row maximum of S exactly (int64 [B,H,N])."""
    q, k = _f64(q), _f64(k)
    B, H, N, _ = q.shape
    out = np.empty((B, H, N), dtype=np.int64)
    vis = _mask(N, causal)
    for b, h in _heads(q):
        s = np.where(vis, q[b, h] @ k[b, h].T, -np.inf)
        out[b, h] = np.sum(s == s.max(axis=1, keepdims=True), axis=1)
    return out


def gqa_expand(x, group: int) -> np.ndarray:
    """[B, H_kv, N, d] -> [B, H_kv * group, N, d]: each head repeated for its group."""
    return np.repeat(_f64(x), group, axis=1)


def gqa_reduce(x, group: int) -> np.ndarray:
    """[B, H_kv * group, N, d] -> [B, H_kv, N, d]: the sum over each group."""
    x = _f64(x)
    B, H, N, d = x.shape
    return x.reshape(B, H // group, group, N, d).sum(axis=2)


def near_tie_counts(q, k, causal: bool, scale: float, fmt: str = "bf16") -> np.ndarray:
    """#{j visible : round(exp(scale * (S_ij - max_j S_ij))) == 1} per row, the
    rounding being to bf16 (default) or to fp16 (fmt = "fp16")."""
    round_fn = {"bf16": bf16_round, "fp16": fp16_round}[fmt]
    q, k = _f64(q), _f64(k)
    B, H, N, _ = q.shape
    out = np.zeros((B, H, N), dtype=np.int64)
    vis = _mask(N, causal)
    for b, h in _heads(q):
        s = np.where(vis, scale * (q[b, h] @ k[b, h].T), -np.inf)
        p = np.exp(s - s.max(axis=1, keepdims=True))
        out[b, h] = np.sum(round_fn(p) == 1.0, axis=1)
    return out


def attention_fwd_bf16p(q, k, v, causal: bool, scale: float, fix_mode: int,
                        round_p: bool = True, return_pbar: bool = False, fmt: str = "bf16"):
    """Attention with the safe-softmax shift, BF16-rounded P_bar and the fix.

    Per row i (one shift for the whole row):
      m_i    = max_j S_ij over visible keys,
      c_i    = #{j : S_ij == m_i}  (exact ties of the raw dot products),
      m'_i   = m_i + FIX_SHIFT_NAT[fix_mode] if c_i >= 2, else m_i
               (fix_mode 5 counts c_i as the entries with bf16(exp(S_ij - m_i)) == 1),
      P_ij   = exp(S_ij - m'_i),          l_i = sum_j P_ij (unrounded),
      P_bar  = bf16(P) if round_p else P,
      O_i    = (sum_j P_bar_ij V_j) / l_i   (fix_mode 4: / sum_j P_bar_ij),
      LSE_i  = m'_i + log l_i.
    fix_mode 0 leaves the shift at the maximum, so repeated maxima give
    P_bar == 1 exactly; fix_mode 1 maps them to 1 - 2^-8, fix_mode 2 to 0.5,
    fix_mode 3 to exp(-1/16); fix_mode 4 keeps them at 1 and self-normalises;
    fix_mode 5 is fix_mode 1 triggered by near ties.
    fmt = "fp16" rounds P_bar to fp16 instead; fix_mode 1 and 5 then map the
    maxima to 1 - 2^-11 (FIX_SHIFT_NAT_FP16), and fix_mode 5 counts the
    entries whose P rounds to 1 in fp16.
    """
    if fix_mode not in FIX_SHIFT_NAT:
        raise ValueError("fix_mode must be 0, 1, 2, 3, 4 or 5")
    if fmt not in ("bf16", "fp16"):
        raise ValueError("fmt must be bf16 or fp16")
    round_fn = bf16_round if fmt == "bf16" else fp16_round
    shifts = FIX_SHIFT_NAT if fmt == "bf16" else FIX_SHIFT_NAT_FP16
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, H, N, d = q.shape
    o = np.empty((B, H, N, v.shape[-1]))
    lse = np.empty((B, H, N))
    pbars = np.empty((B, H, N, N)) if return_pbar else None
    vis = _mask(N, causal)
    for b, h in _heads(q):
        raw = np.where(vis, q[b, h] @ k[b, h].T, -np.inf)
        s = scale * raw
        m = s.max(axis=1, keepdims=True)
        if fix_mode in NEAR_TIE_MODES:
            ties = np.sum(round_fn(np.exp(s - m)) == 1.0, axis=1, keepdims=True)
        else:
            ties = np.sum(raw == raw.max(axis=1, keepdims=True), axis=1, keepdims=True)
        shift = m + shifts[fix_mode] * (ties >= 2)
        p = np.exp(s - shift)
        l = p.sum(axis=1, keepdims=True)
        pbar = round_fn(p) if round_p else p
        den = pbar.sum(axis=1, keepdims=True) if fix_mode in SELF_NORMALISED_MODES else l
        o[b, h] = (pbar @ v[b, h]) / den
        lse[b, h] = shift[:, 0] + np.log(l[:, 0])
        if return_pbar:
            pbars[b, h] = pbar
    if return_pbar:
        return o, lse, pbars
    return o, lse
