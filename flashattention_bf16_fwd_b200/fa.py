"""Thin ctypes binding of libfa_b200.so (include/fa_b200.h).

Argument marshalling only: every step of attention runs in the library's CUDA
kernels.  Tensors are torch tensors on a CUDA device (torch provides memory
and streams); there is no CPU path.  Importing this module loads the library
and raises if it has not been built.
"""
from __future__ import annotations

import ctypes
import os

import torch

__all__ = [
    "FAError", "LIB_PATH", "lib", "fa_fwd", "fa_bwd", "fa_fwd_ex", "fa_bwd_ex", "fa_fwd_debug", "FA_ELEM_BF16",
    "FA_ELEM_F16", "fa_bwd_workspace_size", "fa_bwd_preprocess", "fa_bwd_main", "fa_bwd_finish", "fa_bwd_noalloc",
    "fa_watchdog_selftest", "fa_status_string", "fa_check_device_error", "EXPORTED", "attention_fwd",
    "attention_bwd", "TIE_COUNT_MASK", "TIE_RAISED_BIT", "TIE_FIRED_BIT",
]

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libfa_b200.so")

FA_OK = 0
FA_ELEM_BF16, FA_ELEM_F16 = 0, 1
# fa_fwd_debug's tie record: the count, the final shift raised, the detector fired
TIE_COUNT_MASK, TIE_RAISED_BIT, TIE_FIRED_BIT = (1 << 29) - 1, 1 << 29, 1 << 30
EXPORTED = ("fa_fwd", "fa_fwd_ex", "fa_bwd_ex", "fa_fwd_debug", "fa_bwd_workspace_size", "fa_bwd",
            "fa_bwd_preprocess", "fa_bwd_main", "fa_bwd_finish", "fa_bwd_noalloc", "fa_watchdog_selftest",
            "fa_status_string", "fa_check_device_error")


class FAError(RuntimeError):
    def __init__(self, call: str, status: int):
        self.status = status
        super().__init__(f"{call} failed: {status} ({fa_status_string(status)})")


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with `python -m flashattention_bf16_fwd_b200.build` "
            "(there is no CPU fallback)")
    so = ctypes.CDLL(LIB_PATH)
    vp, i, f, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
    so.fa_fwd.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, f, i, vp]
    so.fa_fwd.restype = i
    so.fa_fwd_ex.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, i, f, i, i, vp]
    so.fa_fwd_ex.restype = i
    so.fa_bwd_ex.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, i, i, i, i, i, i, f, i, vp]
    so.fa_bwd_ex.restype = i
    so.fa_fwd_debug.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, f, i, i, vp]
    so.fa_fwd_debug.restype = i
    so.fa_bwd_workspace_size.argtypes = [i, i, i, i]
    so.fa_bwd_workspace_size.restype = sz
    so.fa_bwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, i, i, i, i, i, f, vp]
    so.fa_bwd.restype = i
    so.fa_bwd_preprocess.argtypes = [vp, vp, vp, sz, i, i, i, i, vp]
    so.fa_bwd_preprocess.restype = i
    so.fa_bwd_main.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, sz, i, i, i, i, i, f, vp]
    so.fa_bwd_main.restype = i
    so.fa_bwd_finish.argtypes = [vp, vp, sz, i, i, i, i, f, vp]
    so.fa_bwd_finish.restype = i
    so.fa_bwd_noalloc.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, f, vp]
    so.fa_bwd_noalloc.restype = i
    so.fa_watchdog_selftest.argtypes = [ctypes.c_uint, vp]
    so.fa_watchdog_selftest.restype = i
    so.fa_status_string.argtypes = [i]
    so.fa_status_string.restype = ctypes.c_char_p
    so.fa_check_device_error.argtypes = [vp]
    so.fa_check_device_error.restype = i
    return so


lib = _load()


def _ptr(t) -> int | None:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    if not t.is_cuda:
        raise ValueError("tensors must live on a CUDA device (the library has no CPU path)")
    return t.data_ptr()


def _stream(stream) -> int | None:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _shape(q):
    if q.dim() != 4:
        raise ValueError("expected [B, H, N, d] tensors")
    return tuple(int(x) for x in q.shape)


def fa_status_string(status: int) -> str:
    return lib.fa_status_string(int(status)).decode()


def fa_fwd(q, k, v, o, lse, causal: bool, scale: float, fix_mode: int, stream=None) -> int:
    B, H, N, d = _shape(q)
    return lib.fa_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, H, N, d, int(causal), float(scale),
                      int(fix_mode), _stream(stream))


def _elem(t) -> int:
    if t.dtype == torch.bfloat16:
        return FA_ELEM_BF16
    if t.dtype == torch.float16:
        return FA_ELEM_F16
    raise ValueError(f"tensors must be bfloat16 or float16, not {t.dtype}")


def fa_fwd_ex(q, k, v, o, lse, causal: bool, scale: float, fix_mode: int, stream=None) -> int:
    """The general forward: element format from q's dtype, Hkv from k's head count."""
    B, H, N, d = _shape(q)
    return lib.fa_fwd_ex(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, H, int(k.shape[1]), N, d, int(causal),
                         float(scale), int(fix_mode), _elem(q), _stream(stream))


def fa_fwd_debug(q, k, v, o, lse, ties, one_hit, o_f32, causal: bool, scale: float, fix_mode: int,
                 stream=None) -> int:
    """fa_fwd_ex plus the per-row tie record, the P_bar == 1 count and O before
    its final rounding (each may be None, not all)."""
    B, H, N, d = _shape(q)
    return lib.fa_fwd_debug(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(ties), _ptr(one_hit), _ptr(o_f32),
                            B, H, int(k.shape[1]), N, d, int(causal), float(scale), int(fix_mode), _elem(q),
                            _stream(stream))


def fa_bwd_ex(q, k, v, o, lse, do, dq, dk, dv, workspace, causal: bool, scale: float, stream=None) -> int:
    """The general backward: element format from q's dtype, Hkv from k's head count."""
    B, H, N, d = _shape(q)
    return lib.fa_bwd_ex(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(do), _ptr(dq), _ptr(dk), _ptr(dv),
                         _ptr(workspace), _nbytes(workspace), B, H, int(k.shape[1]), N, d, int(causal),
                         float(scale), _elem(q), _stream(stream))


def fa_bwd_workspace_size(B: int, H: int, N: int, d: int) -> int:
    return int(lib.fa_bwd_workspace_size(B, H, N, d))


def fa_bwd(q, k, v, o, lse, do, dq, dk, dv, workspace, causal: bool, scale: float, stream=None) -> int:
    B, H, N, d = _shape(q)
    nbytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    return lib.fa_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(do), _ptr(dq), _ptr(dk), _ptr(dv),
                      _ptr(workspace), nbytes, B, H, N, d, int(causal), float(scale), _stream(stream))


def _nbytes(t) -> int:
    return t.numel() * t.element_size() if t is not None else 0


def fa_bwd_preprocess(o, do, workspace, stream=None) -> int:
    B, H, N, d = _shape(o)
    return lib.fa_bwd_preprocess(_ptr(o), _ptr(do), _ptr(workspace), _nbytes(workspace), B, H, N, d,
                                 _stream(stream))


def fa_bwd_main(q, k, v, lse, do, dk, dv, workspace, causal: bool, scale: float, stream=None) -> int:
    B, H, N, d = _shape(q)
    return lib.fa_bwd_main(_ptr(q), _ptr(k), _ptr(v), _ptr(lse), _ptr(do), _ptr(dk), _ptr(dv), _ptr(workspace),
                           _nbytes(workspace), B, H, N, d, int(causal), float(scale), _stream(stream))


def fa_bwd_finish(dq, workspace, scale: float, stream=None) -> int:
    B, H, N, d = _shape(dq)
    return lib.fa_bwd_finish(_ptr(dq), _ptr(workspace), _nbytes(workspace), B, H, N, d, float(scale),
                             _stream(stream))


def fa_bwd_noalloc(q, k, v, o, lse, do, dq, dk, dv, causal: bool, scale: float, stream=None) -> int:
    B, H, N, d = _shape(q)
    return lib.fa_bwd_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(do), _ptr(dq), _ptr(dk),
                              _ptr(dv), B, H, N, d, int(causal), float(scale), _stream(stream))


def fa_watchdog_selftest(timeout_us: int, stream=None) -> int:
    return lib.fa_watchdog_selftest(int(timeout_us), _stream(stream))


def fa_check_device_error(stream=None) -> int:
    return lib.fa_check_device_error(_stream(stream))


def _check(call: str, status: int):
    if status != FA_OK:
        raise FAError(call, status)


def _validate(q, k, v, like_q=()):
    """Shapes, dtypes, devices and contiguity the C ABI assumes but cannot see:
    q and like_q [B,H,N,d]; k, v [B,Hkv,N,d] with Hkv dividing H; one dtype."""
    B, H, N, d = _shape(q)
    if k.dim() != 4 or k.shape[0] != B or tuple(k.shape[2:]) != (N, d) or v.shape != k.shape:
        raise ValueError(f"k and v must be [B, Hkv, N, d] = [{B}, Hkv, {N}, {d}], got {tuple(k.shape)}, "
                         f"{tuple(v.shape)}")
    if H % int(k.shape[1]) != 0:
        raise ValueError(f"the {k.shape[1]} key/value heads must divide the {H} query heads")
    for t in like_q:
        if t.shape != q.shape:
            raise ValueError(f"expected a {tuple(q.shape)} tensor, got {tuple(t.shape)}")
    for t in (q, k, v) + tuple(like_q):
        if t.dtype != q.dtype or t.device != q.device or not t.is_contiguous():
            raise ValueError("q, k, v, o and do must share one dtype and device and be contiguous")


def attention_fwd(q, k, v, causal: bool = True, scale: float | None = None, fix_mode: int = 1,
                  stream=None, ties: bool = False, one_hit: bool = False, o_f32: bool = False):
    """Allocate O and LSE and run the forward; returns (o, lse), followed, in
    this order and only when asked for, by the per-row tie record (``ties``),
    the P_bar == 1 count (``one_hit``) and O before its final rounding
    (``o_f32``), all from fa_fwd_debug.  bf16 or fp16 tensors (from q's dtype);
    k and v may have fewer heads than q (grouped-query attention)."""
    _validate(q, k, v)
    B, H, N, d = _shape(q)
    scale = d ** -0.5 if scale is None else scale
    o = torch.empty_like(q)
    lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    t = torch.empty((B, H, N), dtype=torch.int32, device=q.device) if ties else None
    h = torch.empty((B, H, N), dtype=torch.int32, device=q.device) if one_hit else None
    of = torch.empty((B, H, N, d), dtype=torch.float32, device=q.device) if o_f32 else None
    if ties or one_hit or o_f32:
        _check("fa_fwd_debug", fa_fwd_debug(q, k, v, o, lse, t, h, of, causal, scale, fix_mode, stream))
    else:
        _check("fa_fwd_ex", fa_fwd_ex(q, k, v, o, lse, causal, scale, fix_mode, stream))
    return (o, lse) + tuple(x for x, want in ((t, ties), (h, one_hit), (of, o_f32)) if want)


def attention_bwd(q, k, v, o, lse, do, causal: bool = True, scale: float | None = None, stream=None,
                  workspace=None):
    """Allocate dQ, dK, dV (and the workspace unless given) and run the
    backward.  Formats and head layout as in attention_fwd."""
    _validate(q, k, v, (o, do))
    B, H, N, d = _shape(q)
    if lse.shape != (B, H, N) or lse.dtype != torch.float32 or not lse.is_contiguous():
        raise ValueError("lse must be a contiguous float32 [B, H, N] tensor")
    scale = d ** -0.5 if scale is None else scale
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    if workspace is None:
        workspace = torch.empty(fa_bwd_workspace_size(B, H, N, d), dtype=torch.uint8, device=q.device)
    _check("fa_bwd_ex", fa_bwd_ex(q, k, v, o, lse, do, dq, dk, dv, workspace, causal, scale, stream))
    return dq, dk, dv
