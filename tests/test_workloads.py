"""Host-side checks of the seeded input generators (no GPU)."""
import numpy as np
import torch

from flashattention_bf16_fwd_b200.workloads import WORKLOADS, make_inputs, workload_flops
from oracle import near_tie_counts, tie_counts


def test_deterministic_by_seed():
    w = WORKLOADS["tiny"]
    a, b, c = make_inputs(w, seed=0), make_inputs(w, seed=0), make_inputs(w, seed=1)
    for name in ("q", "k", "v", "do"):
        assert a[name].dtype == torch.bfloat16 and a[name].shape == (1, 2, 128, 64)
        assert torch.equal(a[name], b[name])
        assert not torch.equal(a[name], c[name])


def test_tiny_has_repeated_maxima():
    w = WORKLOADS["tiny"]
    x = make_inputs(w, seed=0)
    ties = tie_counts(x["q"], x["k"], True)
    frac = float(np.mean(ties >= 2))
    # a quarter of the rows are constructed to tie; later copies may undo a few
    assert 0.12 <= frac <= 0.40, frac


def test_sink_and_key_dup_structures_tie():
    gm = WORKLOADS["gpt2m"].with_shape(B=1, H=2, N=256)
    x = make_inputs(gm, seed=0, with_grad=False)
    assert torch.equal(x["k"][:, :, 0], x["k"][:, :, 1])
    assert np.mean(tie_counts(x["q"], x["k"], True) >= 2) > 0.05
    lg = WORKLOADS["long"].with_shape(B=1, H=2, N=512)
    x = make_inputs(lg, seed=0, with_grad=False)
    assert np.mean(tie_counts(x["q"], x["k"], True) >= 2) > 0.01



def test_argmax_near_has_near_ties_and_no_exact_ties():
    """The near-tie structure: every constructed copy scores one bf16 step of
    one key element below the maximum, so no row ties exactly, and a large
    share of rows has two or more P that round to 1 (bf16).  Rounding to 1 in
    fp16 (P >= 1 - 2^-12) implies it in bf16 (P >= 1 - 2^-9), so the fp16
    near-tie rows are a subset of the bf16 ones."""
    for seed in (0, 3):
        x = make_inputs(WORKLOADS["tiny"].with_shape(structure="argmax_near"), seed=seed, with_grad=False)
        assert not np.any(tie_counts(x["q"], x["k"], True) >= 2)
        near = near_tie_counts(x["q"], x["k"], True, x["scale"]) >= 2
        near16 = near_tie_counts(x["q"].half(), x["k"].half(), True, x["scale"], fmt="fp16") >= 2
        assert near.mean() > 0.25 and near16.mean() > 0.15, (near.mean(), near16.mean())
        assert not np.any(near16 & ~near)

def test_flop_convention():
    f = workload_flops(8, 12, 1024, 64, True)
    assert abs(f["total"] - 45.14e9) / 45.14e9 < 1e-3
    f = workload_flops(2, 32, 4096, 128, True)
    assert abs(f["total"] - 962.3e9) / 962.3e9 < 1e-3
