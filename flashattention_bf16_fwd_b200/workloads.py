"""Seeded synthetic inputs for the attention workloads.

This module only draws random numbers and arranges them into the shapes and
structures of the workloads studied on the source pages; it holds none of the
attention arithmetic.  Both the CUDA path (through the tests and the bench) and
the FP64 oracle consume what it returns.

Workloads (all causal, bf16, ``scale = 1/sqrt(d)``):

* ``tiny``    B=1,  H=2,  N=128,  d=64  - N(0,1); a quarter of the query rows get
  their best key copied to a second visible position, so that the row maximum
  of S repeats ("Why Low-Precision Transformer Training Fails", mechanism 2:
  the fix targets rows whose maximum of S appears more than once).
  ``structure="argmax_near"`` moves one element of each copy by one bf16 step,
  against the row's query, so the copy scores just below the maximum: a near
  tie whose probability still rounds to 1 (same page: P_bar exactly 1).
* ``gpt2s``   B=8,  H=12, N=1024, d=64  - N(0,1) for Q, K, V, dO (GPT-2 small
  attention, the training runs of the same page's experiments section).
* ``gpt2m``   B=8,  H=16, N=1024, d=64  - rank-4 keys K = U W plus an attention
  sink: key 0 scaled by 4 and copied to position 1, so sink rows carry an exact
  repeated maximum (same page: attention sinks and multiple maxima).
* ``long``    B=64, H=12, N=2048, d=64  - N(0,1); 10 % of key positions j' are
  overwritten with an earlier key K[j], j < j' (sequence x batch = 131072, the
  critical size quoted by the yicaiai article, section 3.3).
* ``llama7b`` B=2,  H=32, N=4096, d=128 - N(0,1) (Llama 2 7B attention shape,
  "Is Flash Attention Stable?" numeric-deviation study).

Every array is drawn in float32 with ``numpy.random.default_rng(seed)`` and
cast once to bf16 (round to nearest even).  Both sides then use those exact
bf16 values.
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np
import torch

__all__ = ["Workload", "WORKLOADS", "make_inputs", "workload_flops", "visible_pairs"]


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    N: int
    d: int
    causal: bool = True
    structure: str = "normal"       # normal | argmax_dup | argmax_near | lowrank_sink | key_dup
    frac: float = 0.0               # fraction of rows / keys touched by the structure
    rank: int = 4                   # rank of the keys for lowrank_sink
    sink_scale: float = 4.0         # sink key multiplier for lowrank_sink

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    def with_shape(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


WORKLOADS = {
    "tiny": Workload("tiny", 1, 2, 128, 64, structure="argmax_dup", frac=0.25),
    "gpt2s": Workload("gpt2s", 8, 12, 1024, 64),
    "gpt2m": Workload("gpt2m", 8, 16, 1024, 64, structure="lowrank_sink"),
    "long": Workload("long", 64, 12, 2048, 64, structure="key_dup", frac=0.10),
    "llama7b": Workload("llama7b", 2, 32, 4096, 128),
}


def visible_pairs(B: int, H: int, N: int, causal: bool) -> int:
    """Number of (query, key) pairs that enter the softmax."""
    per_head = N * (N + 1) // 2 if causal else N * N
    return B * H * per_head


def workload_flops(B: int, H: int, N: int, d: int, causal: bool) -> dict:
    """Algorithmic FLOPs: 2 contractions forward, 5 backward, 2*d FLOPs each per pair."""
    p = visible_pairs(B, H, N, causal)
    return {"fwd": 4.0 * d * p, "bwd": 10.0 * d * p, "total": 14.0 * d * p}


def _to_bf16(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)


def _argmax_dup(rng, q16: torch.Tensor, k16: torch.Tensor, frac: float, causal: bool,
                near: bool = False) -> torch.Tensor:
    """Copy each chosen row's best visible key into a second visible position.

    Rows are visited in increasing order and always see the keys as modified so
    far.  Row 0 of a causal head sees one key only and is never chosen.  With
    ``near`` the copy's element at the query's smallest nonzero component moves
    by one bf16 step in the direction that lowers the copy's score.
    """
    B, H, N, _ = q16.shape
    k = k16.clone()
    qf = q16.to(torch.float64)
    for b in range(B):
        for h in range(H):
            first = 1 if causal else 0
            n_pick = int(round(frac * N))
            rows = np.sort(rng.choice(np.arange(first, N), size=min(n_pick, N - first), replace=False))
            for i in rows:
                hi = i + 1 if causal else N
                scores = k[b, h, :hi].to(torch.float64) @ qf[b, h, i]
                j_star = int(torch.argmax(scores))
                others = [j for j in range(hi) if j != j_star]
                j_dst = int(rng.choice(others))
                k[b, h, j_dst] = k[b, h, j_star]
                if near:
                    qi = q16[b, h, i].to(torch.float64)
                    ki = k[b, h, j_dst].to(torch.float64)
                    ok = (qi != 0) & (ki != 0)
                    if not bool(ok.any()):
                        continue
                    mag = torch.where(ok, qi.abs(), torch.full_like(qi, float("inf")))
                    c = int(torch.argmin(mag))
                    # bf16 is sign-magnitude: +1 on the bit pattern grows |k_c|,
                    # -1 shrinks it; take the step that lowers q_c * k_c
                    bits = k[b, h, j_dst, c:c + 1].view(torch.int16)
                    bits += 1 if bool(qi[c] * ki[c] < 0) else -1
    return k


def make_inputs(w: Workload, seed: int = 0, with_grad: bool = True) -> dict:
    """Draw Q, K, V (and dO) for workload ``w`` as CPU bf16 tensors [B, H, N, d]."""
    rng = np.random.default_rng(seed)
    shape = (w.B, w.H, w.N, w.d)
    q = _to_bf16(rng.standard_normal(shape, dtype=np.float32))
    if w.structure == "lowrank_sink":
        u = rng.standard_normal((w.B, w.H, w.N, w.rank), dtype=np.float32)
        wm = rng.standard_normal((w.B, w.H, w.rank, w.d), dtype=np.float32)
        kf = np.matmul(u, wm)
        kf[:, :, 0, :] *= w.sink_scale
        k = _to_bf16(kf)
        if w.N > 1:
            k[:, :, 1, :] = k[:, :, 0, :]
    else:
        k = _to_bf16(rng.standard_normal(shape, dtype=np.float32))
    v = _to_bf16(rng.standard_normal(shape, dtype=np.float32))
    if w.structure in ("argmax_dup", "argmax_near"):
        k = _argmax_dup(rng, q, k, w.frac, w.causal, near=(w.structure == "argmax_near"))
    elif w.structure == "key_dup":
        n_dup = int(round(w.frac * w.N))
        for b in range(w.B):
            for h in range(w.H):
                dst = rng.choice(np.arange(1, w.N), size=min(n_dup, w.N - 1), replace=False)
                src = np.array([rng.integers(0, j) for j in dst], dtype=np.int64)
                k[b, h, torch.from_numpy(dst)] = k[b, h, torch.from_numpy(src)]
    out = {"q": q, "k": k, "v": v, "scale": w.scale, "causal": w.causal}
    if with_grad:
        out["do"] = _to_bf16(rng.standard_normal(shape, dtype=np.float32))
    return out
