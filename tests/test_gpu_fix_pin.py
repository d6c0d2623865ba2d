"""The fix itself, pinned on the GPU.

"Why Low-Precision Transformer Training Fails" (admirer.cn summary,
mechanism 2) defines the fix by one property: on a row whose maximum of S
occurs more than once, the shift is raised so that every exponent, the ones
at the maxima included, is strictly below 1.  Two checks of the kernel's own
arithmetic, through fa_fwd_debug and fa_fwd_ex:

1. The P_bar == 1 record (one_hit).  Among the entries the kernel rounded for
   the P_bar V product under the row's final shift, it counts those that are
   exactly 1.0.  A row whose final shift is raised must have none; a row with
   the plain shift has at least its maximum.  On rows that see one key tile
   (N <= 128) the kernel's shift is the row's, so the count must equal the
   emulating oracle's count of P_bar == 1.

2. Where the maxima land.  Moving the maxima from 1 to 1 - 2^-8 (or to any
   other value) changes how every other entry of the row rounds to bf16, so O
   changes in a large share of its bf16 values.  On one-tile rows the kernel
   must match the emulating oracle of its own fix_mode bit for bit except for
   rare rounding flips, and must miss, in a large share of values, the oracle
   with another mode or with a wrong shift planted in it (maxima at
   1 - 2^-6 in bf16, 1 - 2^-9 in fp16: also on the grid, also below 1).
"""
import contextlib

import numpy as np
import pytest
import torch

import oracle.attention64 as oracle_mod
from flashattention_bf16_fwd_b200.workloads import WORKLOADS, make_inputs
from oracle import attention_fwd_bf16p, bf16_round, fp16_round, tie_counts

pytestmark = pytest.mark.gpu

RAISED = 1 << 29
COUNT = (1 << 29) - 1

# share of O's values on repeated-max rows that may differ from the emulating
# oracle of the same mode (rounding flips of the FP32 path), and the share by
# which another shift must differ
SAME_MAX_MISMATCH = 0.03
OTHER_MIN_MISMATCH = 0.20


@pytest.fixture(scope="module")
def fa():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from flashattention_bf16_fwd_b200 import fa as binding
    return binding


def gpu_debug(fa, x, fix_mode, dtype):
    dev = torch.device("cuda")
    q, k, v = (x[n].to(dtype).to(dev) for n in ("q", "k", "v"))
    o, lse, ties, hits = fa.attention_fwd(q, k, v, causal=x["causal"], scale=x["scale"], fix_mode=fix_mode,
                                          ties=True, one_hit=True)
    torch.cuda.synchronize()
    assert fa.fa_check_device_error() == 0
    return o.float().cpu().numpy(), ties.cpu().numpy(), hits.cpu().numpy()


def emulate(x, fix_mode, fmt, planted_shift=None):
    """The oracle's bf16/fp16 P_bar emulation; optionally with a wrong shift
    planted for fix_mode (a mistake in the oracle, on the CPU, to show the
    comparison has the power to see it)."""
    table = oracle_mod.FIX_SHIFT_NAT if fmt == "bf16" else oracle_mod.FIX_SHIFT_NAT_FP16
    dtype = torch.bfloat16 if fmt == "bf16" else torch.float16
    with planted(table, fix_mode, planted_shift):
        return attention_fwd_bf16p(x["q"].to(dtype), x["k"].to(dtype), x["v"].to(dtype), x["causal"], x["scale"],
                                   fix_mode, fmt=fmt, return_pbar=True)


@contextlib.contextmanager
def planted(table, key, value):
    if value is None:
        yield
        return
    saved = table[key]
    table[key] = value
    try:
        yield
    finally:
        table[key] = saved


FMTS = {"bf16": torch.bfloat16, "fp16": torch.float16}
CASES = [  # (workload, shape overrides, fix modes)
    ("tiny", {}, (0, 1, 2, 3)),
    ("tiny", {"structure": "argmax_near"}, (0, 5)),
    ("long", {"B": 1, "H": 4, "N": 1024}, (0, 1, 2, 3)),
    ("gpt2m", {"B": 1, "H": 2, "N": 512}, (0, 1, 2, 3)),
]


@pytest.mark.parametrize("fmt", sorted(FMTS))
@pytest.mark.parametrize("case", range(len(CASES)),
                         ids=[f"{n}-{o.get('structure', 'std')}" for n, o, _ in CASES])
def test_one_hit_record(fa, fmt, case):
    name, shape, modes = CASES[case]
    w = WORKLOADS[name].with_shape(**shape)
    x = make_inputs(w, seed=3, with_grad=False)
    single = np.broadcast_to(np.arange(w.N) < 128, (w.B, w.H, w.N))   # rows that see one key tile
    for fix_mode in modes:
        _, ties, hits = gpu_debug(fa, x, fix_mode, FMTS[fmt])
        raised = (ties & RAISED) != 0
        count = ties & COUNT
        # no exponent reaches 1 under a raised shift; the plain shift puts its
        # maximum on exactly 1
        assert np.all(hits[raised] == 0), (fix_mode, int(hits[raised].max()))
        assert np.all(hits[~raised] >= 1), fix_mode
        if fix_mode in (0, 4):
            assert not raised.any()
            rep = count >= 2
            assert rep.sum() > 0 or shape.get("structure") == "argmax_near"
            # every copy of the final maximum lands on 1 without the fix
            assert np.all(hits[rep] >= count[rep])
        elif fix_mode in (1, 2, 3):
            assert raised.sum() > 0
            assert np.array_equal(raised, count >= 2)
        else:
            assert raised.sum() > 0
        # one key tile: the kernel's shift is the row's shift, so its count is
        # the oracle's count of P_bar == 1 for the same mode and format
        _, _, pbar = emulate(x, fix_mode, fmt)
        ref = np.sum(pbar == 1.0, axis=-1)
        agree = hits[single] == ref[single]
        assert np.mean(agree) >= 0.995, (fix_mode, np.mean(agree))
        assert np.all(ref[single & raised] == 0)


def mismatch(o_gpu, o_emul, fmt, rows):
    rnd = bf16_round if fmt == "bf16" else fp16_round
    return float(np.mean((o_gpu != rnd(o_emul))[rows]))


@pytest.mark.parametrize("fmt", sorted(FMTS))
@pytest.mark.parametrize("fix_mode", [0, 1, 3])
def test_maxima_land_on_the_fix_value(fa, fmt, fix_mode):
    w = WORKLOADS["tiny"].with_shape(B=2, H=4)          # N = 128: one key tile per row
    x = make_inputs(w, seed=7, with_grad=False)
    rep = tie_counts(x["q"], x["k"], True) >= 2
    assert rep.sum() > 300
    o, ties, _ = gpu_debug(fa, x, fix_mode, FMTS[fmt])
    own, _, _ = emulate(x, fix_mode, fmt)
    same = mismatch(o, own, fmt, rep)
    assert same <= SAME_MAX_MISMATCH, (fix_mode, same)
    # the other modes' maxima, and a wrong shift planted in the oracle
    wrong = -np.log(1.0 - (2.0 ** -6 if fmt == "bf16" else 2.0 ** -9))
    others = [(m, None) for m in (0, 1, 3) if m != fix_mode] + [(1, wrong)]
    for m, shift in others:
        alt, _, _ = emulate(x, m, fmt, planted_shift=shift)
        diff = mismatch(o, alt, fmt, rep)
        assert diff >= OTHER_MIN_MISMATCH, (fix_mode, m, shift, diff, same)
    # rows without a repeated maximum are the same in every mode
    assert mismatch(o, own, fmt, ~rep) <= SAME_MAX_MISMATCH


# Bias on repeated-max rows (the error the fix targets), measured on O before
# its rounding to bf16: on attention-sink rows O sits just inside midpoints of
# the bf16 grid (two equal weights on two bf16 rows of V, shrunk slightly by
# the other keys), so the output's own rounding shrinks magnitudes even for
# the exactly computed O.  That error is the same in every mode; the fp32
# output isolates the error of the P_bar V path.
BIAS_INPUTS = [("gpt2m", {}), ("long", {"B": 32, "H": 12, "N": 2048})]


def test_bias_on_repeated_maxima(fa):
    """Pass for fix_mode 1: the mean error and the magnitude-aligned mean error
    over repeated-max rows are bounded, |mean| + 3 SE <= 2^-14 mean|O| (1/32 of
    bf16's half step 2^-9): the sign-coherent error the fix targets stays far
    below what a bf16 output could show, with 3-sigma confidence at any sample
    size.  Power: fix_mode 3 puts the maxima off the bf16 grid (P_bar 0.9375
    where l holds 0.9394) and must be seen outside the same bound, shrinking
    |O|.  fix_mode 0 is measured and printed beside them, with the paired
    difference of the two modes on the same rows.  (A bare |z| < 3 would not
    do: over a few hundred thousand rows every mode, the self-normalised one
    included, shows a common FP32 shrink of about 1e-6 mean|O|.)"""
    from flashattention_bf16_fwd_b200.stats import bias_stats
    from oracle import attention_fwd

    dev = torch.device("cuda")
    sel = {m: {"f32": [], "bf16": []} for m in (0, 1, 3)}
    ref_rows, ctrl = [], {m: [] for m in (0, 1, 3)}
    ctrl_ref = []
    for name, shape in BIAS_INPUTS:
        w = WORKLOADS[name].with_shape(**shape)
        x = make_inputs(w, seed=11, with_grad=False)
        o_ref, _ = attention_fwd(x["q"], x["k"], x["v"], True, w.scale)
        rep = tie_counts(x["q"], x["k"], True) >= 2
        ref_rows.append(o_ref[rep])
        ctrl_ref.append(o_ref[~rep][:20000])
        q, k, v = (x[n].to(dev) for n in ("q", "k", "v"))
        for m in sel:
            o, _, of = fa.attention_fwd(q, k, v, causal=True, scale=w.scale, fix_mode=m, o_f32=True)
            torch.cuda.synchronize()
            assert fa.fa_check_device_error() == 0
            # the returned O is the round-to-nearest-even of the FP32 output
            assert torch.equal(o, of.to(torch.bfloat16))
            of, o = of.cpu().numpy().astype(np.float64), o.float().cpu().numpy()
            sel[m]["f32"].append(of[rep])
            sel[m]["bf16"].append(o[rep])
            ctrl[m].append(of[~rep][:20000])
        del q, k, v
    ref = np.concatenate(ref_rows)
    rows = np.ones(ref.shape[0], bool)
    assert ref.shape[0] >= 100_000
    stats = {}
    for m in sel:
        for kind in ("f32", "bf16"):
            stats[(m, kind)] = bias_stats(np.concatenate(sel[m][kind]), ref, rows)
        cr = np.concatenate(ctrl_ref)
        stats[(m, "control_f32")] = bias_stats(np.concatenate(ctrl[m]), cr, np.ones(cr.shape[0], bool))
    a0 = np.mean(np.sign(ref) * (np.concatenate(sel[0]["f32"]) - ref), axis=-1)
    a1 = np.mean(np.sign(ref) * (np.concatenate(sel[1]["f32"]) - ref), axis=-1)
    dpair = a0 - a1
    print(f"bias paired aligned fix_mode 0 - 1: {dpair.mean() / np.abs(ref).mean():+.2e} mean|O|, "
          f"z {dpair.mean() / (dpair.std(ddof=1) / np.sqrt(dpair.size)):+.2f}")
    for key, s in stats.items():
        print(f"bias fix_mode {key[0]} {key[1]}: rows {s['rows']} z_mean {s['z_mean']:+.2f} "
              f"z_aligned {s['z_aligned']:+.2f} aligned/mean|O| {s['aligned_mean'] / s['mean_abs_ref']:+.2e}")
    bound = 2.0 ** -14

    def within(st):
        m = st["mean_abs_ref"]
        return (abs(st["mean"]) + 3 * st["se_mean"] <= bound * m and
                abs(st["aligned_mean"]) + 3 * st["se_aligned"] <= bound * m)

    assert within(stats[(1, "f32")]), stats[(1, "f32")]
    assert within(stats[(1, "control_f32")]), stats[(1, "control_f32")]
    s3 = stats[(3, "f32")]
    assert s3["aligned_mean"] + 3 * s3["se_aligned"] < -bound * s3["mean_abs_ref"], s3
