"""FP64 CPU oracle for the BF16 FlashAttention path (test infrastructure only).

Only tests/, ``__graft_entry__.smoke()`` and the CPU-baseline leg of bench.py
may import this package.  The CUDA path never calls it and shares no code with
it.  Every function is pinned by tests/test_oracle_pins.py.
"""
from .attention64 import (  # noqa: F401
    DELTA_LOG2, DELTA_NAT, DELTA16_NAT, fp16_round, FIX_SHIFT_NAT, FIX_SHIFT_NAT_FP16, NEAR_TIE_MODES, SELF_NORMALISED_MODES, bf16_round, scores,
    attention_fwd, attention_bwd, attention_fwd_bf16p, tie_counts, near_tie_counts, gqa_expand, gqa_reduce,
)
