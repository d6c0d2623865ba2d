"""The C-ABI library loads, exports every declared symbol, and validates its
arguments on the host (no GPU, no launch).  Invalid calls return their error
code before any CUDA call; a valid call without an sm_100 device returns
FA_ERR_DEVICE (there is no CPU fallback)."""
import ctypes
import os
import re

import pytest
import torch

from flashattention_bf16_fwd_b200 import build as fa_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "fa_b200.h")

FA_OK, FA_ERR_NULL, FA_ERR_SHAPE, FA_ERR_HEADDIM, FA_ERR_ALIGN = 0, -1, -2, -3, -4
FA_ERR_FIXMODE, FA_ERR_WORKSPACE, FA_ERR_LAUNCH, FA_ERR_TIMEOUT, FA_ERR_ARG, FA_ERR_DEVICE = -5, -6, -7, -8, -9, -10
FA_ERR_BUILD = -12


@pytest.fixture(scope="module")
def fa():
    fa_build.build()
    from flashattention_bf16_fwd_b200 import fa as binding
    return binding


def declared_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"FA_API\s+[\w\s\*]+?\b(fa_\w+)\s*\(", text)))


def test_header_declares_the_boundary():
    assert declared_symbols() == sorted(["fa_fwd", "fa_fwd_ex", "fa_bwd_ex", "fa_fwd_debug", "fa_bwd_workspace_size",
                                         "fa_bwd", "fa_bwd_preprocess", "fa_bwd_main", "fa_bwd_finish",
                                         "fa_bwd_noalloc", "fa_watchdog_selftest", "fa_status_string",
                                         "fa_check_device_error"])


def test_library_exports_every_declared_symbol(fa):
    so = ctypes.CDLL(fa.LIB_PATH)
    for name in declared_symbols():
        assert hasattr(so, name), name
    assert sorted(fa.EXPORTED) == declared_symbols()


def test_status_strings(fa):
    for code in range(0, -13, -1):
        s = fa.fa_status_string(code)
        assert s and s != "unknown status"
    assert fa.fa_status_string(-99) == "unknown status"


def test_workspace_size(fa):
    B, H, N, d = 2, 3, 1000, 64
    rows = B * H * N
    exp = -(-rows * d * 4 // 256) * 256 + -(-rows * 4 // 256) * 256
    assert fa.fa_bwd_workspace_size(B, H, N, d) == exp
    assert fa.fa_bwd_workspace_size(1, 1, 1, 96) == 0
    assert fa.fa_bwd_workspace_size(0, 1, 1, 64) == 0


A = 0x10000          # fake, 16-byte aligned device addresses: never dereferenced.  Calls with
                     # them either fail an argument check before any launch, or sit in the
                     # test that is skipped when a GPU is present.
MIS = 0x10008


def fwd(fa, q=A, k=A, v=A, o=A, lse=A, B=1, H=1, N=128, d=64, causal=1, scale=0.125, fix=1):
    return fa.lib.fa_fwd(q, k, v, o, lse, B, H, N, d, causal, scale, fix, None)


def test_fwd_argument_errors(fa):
    assert fwd(fa, q=None) == FA_ERR_NULL
    assert fwd(fa, lse=None) == FA_ERR_NULL
    assert fwd(fa, d=96) == FA_ERR_HEADDIM
    assert fwd(fa, d=256) == FA_ERR_HEADDIM
    assert fwd(fa, N=0) == FA_ERR_SHAPE
    assert fwd(fa, B=0) == FA_ERR_SHAPE
    assert fwd(fa, B=1 << 14, H=1 << 10, N=1 << 10, d=64) == FA_ERR_SHAPE
    # the bound is B*H*N*d < 2^31: 32768 heads of 1024 x 64 is exactly 2^31
    assert fwd(fa, H=32768, N=1024, d=64) == FA_ERR_SHAPE
    assert fa.fa_bwd_workspace_size(1, 32768, 1024, 64) == 0
    assert fa.fa_bwd_workspace_size(1, 32767, 1024, 64) == 32767 * 1024 * (64 + 1) * 4
    assert fwd(fa, causal=2) == FA_ERR_ARG
    assert fwd(fa, scale=0.0) == FA_ERR_ARG
    assert fwd(fa, scale=float("nan")) == FA_ERR_ARG
    assert fwd(fa, scale=float("inf")) == FA_ERR_ARG
    assert fwd(fa, k=MIS) == FA_ERR_ALIGN
    assert fwd(fa, o=MIS) == FA_ERR_ALIGN
    assert fwd(fa, fix=6) == FA_ERR_FIXMODE
    assert fwd(fa, fix=-1) == FA_ERR_FIXMODE
    # fa_fwd_debug needs at least one of its two records
    assert fa.lib.fa_fwd_debug(A, A, A, A, A, None, None, None, 1, 1, 1, 128, 64, 1, 0.125, 1, 0, None) == FA_ERR_NULL
    assert fa.lib.fa_fwd_debug(A, A, A, A, A, A, None, None, 1, 1, 1, 128, 64, 1, 0.125, 6, 0, None) == FA_ERR_FIXMODE
    assert fa.lib.fa_fwd_debug(A, A, A, A, A, None, A, None, 1, 4, 3, 128, 64, 1, 0.125, 1, 0, None) == FA_ERR_SHAPE
    assert fa.lib.fa_fwd_debug(A, A, A, A, A, None, None, MIS, 1, 1, 1, 128, 64, 1, 0.125, 1, 0, None) == FA_ERR_ALIGN
    assert fa.lib.fa_fwd_debug(A, A, A, A, A, None, A, None, 1, 1, 1, 128, 64, 1, 0.125, 1, 2, None) == FA_ERR_ARG


def test_bwd_argument_errors(fa):
    ws = fa.fa_bwd_workspace_size(1, 1, 128, 64)

    def bwd(dq=A, ws_ptr=A, ws_bytes=ws, d=64, N=128):
        return fa.lib.fa_bwd(A, A, A, A, A, A, dq, A, A, ws_ptr, ws_bytes, 1, 1, N, d, 1, 0.125, None)

    assert bwd(dq=None) == FA_ERR_NULL
    assert bwd(d=80) == FA_ERR_HEADDIM
    assert bwd(dq=MIS) == FA_ERR_ALIGN
    assert bwd(ws_ptr=None) == FA_ERR_WORKSPACE
    assert bwd(ws_ptr=MIS) == FA_ERR_WORKSPACE
    assert bwd(ws_bytes=ws - 1) == FA_ERR_WORKSPACE
    assert fa.lib.fa_bwd_preprocess(A, None, A, ws, 1, 1, 128, 64, None) == FA_ERR_NULL
    assert fa.lib.fa_bwd_preprocess(A, A, A, ws - 16, 1, 1, 128, 64, None) == FA_ERR_WORKSPACE
    assert fa.lib.fa_bwd_main(A, A, A, A, A, A, MIS, A, ws, 1, 1, 128, 64, 1, 0.125, None) == FA_ERR_ALIGN
    assert fa.lib.fa_bwd_main(A, A, A, A, A, A, A, A, ws, 1, 1, 128, 64, 3, 0.125, None) == FA_ERR_ARG
    assert fa.lib.fa_bwd_finish(A, A, ws, 1, 1, 128, 32, 0.125, None) == FA_ERR_HEADDIM
    assert fa.lib.fa_bwd_finish(A, A, ws, 1, 1, 128, 64, -1.0, None) == FA_ERR_ARG


FA_ERR_SCRATCH_LIMIT = -11


def test_general_entry_point_argument_errors(fa):
    fx = lambda **kw: fa.lib.fa_fwd_ex(*[kw.get(n, dflt) for n, dflt in (
        ("q", A), ("k", A), ("v", A), ("o", A), ("lse", A), ("B", 1), ("H", 4), ("Hkv", 2),
        ("N", 128), ("d", 64), ("causal", 1), ("scale", 0.125), ("fix", 1), ("elem", 0), ("stream", None))])
    assert fx(elem=2) == FA_ERR_ARG
    assert fx(elem=-1) == FA_ERR_ARG
    assert fx(fix=6) == FA_ERR_FIXMODE
    assert fx(Hkv=3) == FA_ERR_SHAPE
    assert fx(v=None) == FA_ERR_NULL
    assert fx(o=MIS, elem=1) == FA_ERR_ALIGN
    # grouped heads: Hkv must divide H and not exceed it
    assert fx(Hkv=0) == FA_ERR_SHAPE
    assert fx(Hkv=8) == FA_ERR_SHAPE
    assert fx(d=96, elem=1) == FA_ERR_HEADDIM
    assert fx(lse=None, elem=1) == FA_ERR_NULL
    ws = fa.fa_bwd_workspace_size(1, 4, 128, 64)
    bx = lambda **kw: fa.lib.fa_bwd_ex(*[kw.get(n, dflt) for n, dflt in (
        ("q", A), ("k", A), ("v", A), ("o", A), ("lse", A), ("do", A), ("dq", A), ("dk", A), ("dv", A),
        ("ws", A), ("wsz", ws), ("B", 1), ("H", 4), ("Hkv", 2), ("N", 128), ("d", 64), ("causal", 1),
        ("scale", 0.125), ("elem", 1), ("stream", None))])
    assert bx(elem=3) == FA_ERR_ARG
    assert bx(wsz=ws - 1) == FA_ERR_WORKSPACE
    assert bx(Hkv=8) == FA_ERR_SHAPE
    assert bx(d=96) == FA_ERR_HEADDIM
    assert bx(Hkv=3) == FA_ERR_SHAPE
    assert bx(dk=MIS) == FA_ERR_ALIGN
    assert bx(dk=None) == FA_ERR_NULL
    assert bx(dq=MIS, elem=0) == FA_ERR_ALIGN


def test_binding_checks_shapes_and_dtypes(fa):
    q = torch.zeros(1, 4, 128, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError):                   # k with a head count that does not divide H
        fa.attention_fwd(q, torch.zeros(1, 3, 128, 64, dtype=torch.bfloat16), torch.zeros(1, 3, 128, 64, dtype=torch.bfloat16))
    with pytest.raises(ValueError):                   # mixed element formats
        fa.attention_fwd(q, q.half(), q)
    with pytest.raises(ValueError):                   # not contiguous
        fa.attention_fwd(q.transpose(2, 3).contiguous().transpose(2, 3), q, q)
    with pytest.raises(ValueError):                   # float32 is not a supported format
        fa.attention_fwd(q.float(), q.float(), q.float())


def test_bwd_noalloc_argument_errors(fa):
    def nb(dq=A, N=128, d=64, H=1):
        return fa.lib.fa_bwd_noalloc(A, A, A, A, A, A, dq, A, A, 1, H, N, d, 1, 0.125, None)

    assert nb(dq=None) == FA_ERR_NULL
    assert nb(d=96) == FA_ERR_HEADDIM
    assert nb(dq=MIS) == FA_ERR_ALIGN
    # the fixed 32 MiB scratch holds 129055 rows at d = 64 and 65027 at d = 128
    assert nb(N=129056, d=64) == FA_ERR_SCRATCH_LIMIT
    assert nb(N=65028, d=128) == FA_ERR_SCRATCH_LIMIT
    assert nb(N=4096, H=32, d=128) == FA_ERR_SCRATCH_LIMIT
    assert fa.fa_bwd_workspace_size(1, 1, 129055, 64) <= 32 << 20 < fa.fa_bwd_workspace_size(1, 1, 129056, 64)
    assert fa.fa_bwd_workspace_size(1, 1, 65027, 128) <= 32 << 20 < fa.fa_bwd_workspace_size(1, 1, 65028, 128)


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-GPU behaviour")
def test_valid_call_without_gpu_reports_device_error(fa):
    assert fwd(fa) == FA_ERR_DEVICE
    ws = fa.fa_bwd_workspace_size(1, 1, 128, 64)
    assert fa.lib.fa_bwd(A, A, A, A, A, A, A, A, A, A, ws, 1, 1, 128, 64, 1, 0.125, None) == FA_ERR_DEVICE
    assert fa.lib.fa_bwd_noalloc(A, A, A, A, A, A, A, A, A, 1, 1, 128, 64, 1, 0.125, None) == FA_ERR_DEVICE
    assert fa.lib.fa_watchdog_selftest(1000, None) == FA_ERR_DEVICE
    # arguments that pass every check; with a GPU these would launch
    assert fwd(fa, H=32767, N=1024, d=64) == FA_ERR_DEVICE            # one head below the 2^31 bound
    assert fa.lib.fa_fwd_ex(A, A, A, A, A, 1, 1, 1, 128, 64, 1, 0.125, 5, 1, None) == FA_ERR_DEVICE
    assert fa.lib.fa_fwd_ex(A, A, A, A, A, 1, 4, 2, 128, 64, 1, 0.125, 1, 0, None) == FA_ERR_DEVICE
    assert fa.lib.fa_fwd_ex(A, A, A, A, A, 1, 4, 2, 128, 64, 1, 0.125, 5, 1, None) == FA_ERR_DEVICE
    assert fa.lib.fa_fwd_debug(A, A, A, A, A, A, A, A, 1, 4, 2, 128, 64, 1, 0.125, 1, 0, None) == FA_ERR_DEVICE
    ws4 = fa.fa_bwd_workspace_size(1, 4, 128, 64)
    assert fa.lib.fa_bwd_ex(A, A, A, A, A, A, A, A, A, A, ws4, 1, 4, 2, 128, 64, 1, 0.125, 1, None) == FA_ERR_DEVICE


def test_watchdog_selftest_argument_errors(fa):
    assert fa.lib.fa_watchdog_selftest(0, None) == FA_ERR_ARG
    assert fa.lib.fa_watchdog_selftest(1000001, None) == FA_ERR_ARG


def test_binding_rejects_cpu_tensors(fa):
    q = torch.zeros(1, 1, 128, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        fa.attention_fwd(q, q, q)
