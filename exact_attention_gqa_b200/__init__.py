"""Exact grouped-query attention forward for B200 (sm_100a).

The computation runs in hand-written CUDA kernels behind the C ABI of
``include/gqa_attn.h`` (``libgqa_attn.so``).  This module marshals torch
tensors into that ABI: it checks dtypes, devices and layouts, allocates the
outputs (and the split-KV workspace) with torch, passes raw pointers and the
current CUDA stream, and raises on a non-zero status.  There is no fallback:
without the built library or a CUDA tensor every call raises.

    out, lse = gqa_attn(q, k, v, causal=True)

Layouts follow FlashAttention's ``flash_attn_func`` ([batch, seq, heads, dim]):
q [B, Sq, Hq, D], k/v [B, Sk, Hkv, D] -> out [B, Sq, Hq, D], lse [B, Hq, Sq];
packed variable length: q [total, Hq, D], k/v [total, Hkv, D], cu_seqlens
int32 [B + 1] -> out [total, Hq, D], lse [Hq, total].
"""
from __future__ import annotations

import ctypes
import math

from . import _capi
from ._capi import GqaError, STATUS, STATUS_CODE, strerror

__all__ = ["gqa_attn", "gqa_attn_host", "gqa_attn_kvcache", "gqa_attn_blocksparse",
           "gqa_attn_backward",
           "gqa_attn_fwd", "gqa_attn_fwd_f32", "gqa_attn_plan",
           "gqa_attn_workspace_bytes", "gqa_attn_set_workspace", "gqa_attn_get_device_error",
           "GqaError", "STATUS", "STATUS_CODE", "strerror", "library_path",
           "gqa_attn_blocksparse_varlen", "gqa_attn_blocksparse_varlen_plan",
           "SparseVarlenPlan", "gqa_attn_fp8"]

KERNEL_NAMES = {0: "none", 1: "prefill_sm100", 2: "decode_splitkv", 3: "zero_fill"}


def library_path() -> str:
    return str(_capi.LIB_PATH)


def _stream_handle(torch, device):
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else None


# ------------------------------------------------------------------ raw C-ABI calls
def gqa_attn_fwd(q_ptr, k_ptr, v_ptr, out_ptr, lse_ptr, B, Hq, Hkv, Sq, Sk, D, scale, causal,
                 num_splits, pack_gqa, cu_seqlens_ptr, stream) -> int:
    """Direct call of the C entry point (pointers as ints or c_void_p); returns the status."""
    return _capi.load().gqa_attn_fwd(q_ptr, k_ptr, v_ptr, out_ptr, lse_ptr, B, Hq, Hkv, Sq, Sk,
                                     D, scale, causal, num_splits, pack_gqa, cu_seqlens_ptr,
                                     stream)


def gqa_attn_fwd_f32(q_ptr, k_ptr, v_ptr, out_ptr, lse_ptr, B, Hq, Hkv, Sq, Sk, D, scale, causal,
                     num_splits, pack_gqa, cu_seqlens_ptr, stream) -> int:
    return _capi.load().gqa_attn_fwd_f32(q_ptr, k_ptr, v_ptr, out_ptr, lse_ptr, B, Hq, Hkv, Sq,
                                         Sk, D, scale, causal, num_splits, pack_gqa,
                                         cu_seqlens_ptr, stream)


def gqa_attn_workspace_bytes(B, Hq, Sq, D, num_splits) -> int:
    return int(_capi.load().gqa_attn_workspace_bytes(B, Hq, Sq, D, num_splits))


def gqa_attn_set_workspace(ptr, nbytes) -> int:
    return _capi.load().gqa_attn_set_workspace(ptr, nbytes)


def gqa_attn_plan(B, Hq, Hkv, Sq, Sk, D, scale=None, causal=False, num_splits=1, pack_gqa=-1,
                  varlen=False):
    """(status, kernel name, effective num_splits, effective pack_gqa)."""
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    kern, spl, pk = ctypes.c_int(0), ctypes.c_int(0), ctypes.c_int(0)
    rc = _capi.load().gqa_attn_plan(B, Hq, Hkv, Sq, Sk, D, scale, int(bool(causal)), num_splits,
                                    pack_gqa, int(bool(varlen)), ctypes.byref(kern),
                                    ctypes.byref(spl), ctypes.byref(pk))
    return rc, KERNEL_NAMES.get(kern.value, kern.value), spl.value, pk.value


def gqa_attn_get_device_error(stream=None) -> int:
    code = ctypes.c_int(0)
    rc = _capi.load().gqa_attn_get_device_error(ctypes.byref(code), stream)
    if rc != 0:
        raise GqaError("gqa_attn_get_device_error", rc)
    return code.value


# ------------------------------------------------------------------ torch front end
_ws = {}  # device index -> torch buffer registered as the split-KV workspace
_ws_retired = []  # buffers replaced by a larger one, kept alive for in-flight kernels


def _workspace(torch, device, nbytes):
    if nbytes == 0:
        return
    idx = device.index if device.index is not None else torch.cuda.current_device()
    buf = _ws.get(idx)
    if buf is None or buf.numel() < nbytes:
        # grow geometrically; a replaced buffer stays alive (a kernel on another stream
        # may still read it), which keeps at most about twice the largest size
        old = 0 if buf is None else buf.numel()
        if buf is not None:
            _ws_retired.append(buf)
        buf = torch.empty(max(nbytes, 2 * old, 1 << 20), dtype=torch.uint8, device=device)
        _ws[idx] = buf
    with torch.cuda.device(device):  # the registration belongs to this device
        rc = gqa_attn_set_workspace(ctypes.c_void_p(buf.data_ptr()), buf.numel())
    if rc != 0:
        raise GqaError("gqa_attn_set_workspace", rc)


def gqa_attn(q, k, v, *, causal: bool = False, scale: float | None = None,
             num_splits: int = 1, pack_gqa: int = -1, cu_seqlens=None, max_seqlen=None,
             window: int = 0, out=None, lse=None):
    """Exact attention forward with grouped-query heads on the current CUDA stream.

    Returns (out, lse).  bf16 inputs run the sm_100a kernels, fp32 inputs the fp32
    path.  ``scale`` defaults to 1/sqrt(D) (FlashAttention's softmax_scale=None).
    ``window`` > 0 (bf16, causal) limits each query to its `window` most recent keys
    (gqa_attn_fwd_window).
    """
    import torch

    if not (q.is_cuda and k.is_cuda and v.is_cuda):
        raise ValueError("gqa_attn needs CUDA tensors (there is no CPU path)")
    if not (q.dtype == k.dtype == v.dtype) or q.dtype not in (torch.bfloat16, torch.float32):
        raise ValueError("q, k, v must all be bf16 or all fp32")
    for name, t in (("q", q), ("k", k), ("v", v)):
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
    varlen = cu_seqlens is not None
    if varlen:
        if q.dim() != 3 or k.dim() != 3 or v.shape != k.shape:
            raise ValueError("packed inputs are q [total, Hq, D], k/v [total, Hkv, D]")
        total, Hq, D = q.shape
        Hkv = k.shape[1]
        if k.shape[0] != total:
            raise ValueError("q and k/v must hold the same packed rows")
        cu = cu_seqlens
        if not cu.is_cuda or cu.dtype != torch.int32:
            raise ValueError("cu_seqlens must be a CUDA int32 tensor")
        B = cu.numel() - 1
        if max_seqlen is None:
            max_seqlen = int((cu[1:] - cu[:-1]).max().item()) if B > 0 else 0
        Sq, Sk = int(max_seqlen), int(total)
        lse_shape = (Hq, total)
    else:
        if q.dim() != 4 or k.dim() != 4 or v.shape != k.shape:
            raise ValueError("dense inputs are q [B, Sq, Hq, D], k/v [B, Sk, Hkv, D]")
        B, Sq, Hq, D = q.shape
        _, Sk, Hkv, _ = k.shape
        cu = None
        lse_shape = (B, Hq, Sq)
    scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty(lse_shape, dtype=torch.float32, device=q.device)
    if window:
        if not causal or window < 1 or q.dtype != torch.bfloat16 or num_splits not in (0, 1):
            raise ValueError("a sliding window needs causal=True, window >= 1, bf16 inputs "
                             "and no split count")
        with torch.cuda.device(q.device):
            rc = _capi.load().gqa_attn_fwd_window(
                _ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, Hq, Hkv, Sq, Sk, D, scale,
                int(window), pack_gqa, _ptr(cu), _stream_handle(torch, q.device))
        if rc != 0:
            raise GqaError("gqa_attn_fwd_window", rc)
        return out, lse
    with torch.cuda.device(q.device):  # the library works on the current device
        _call(torch, q, k, v, out, lse, B, Hq, Hkv, Sq, Sk, D, scale, causal, num_splits,
              pack_gqa, varlen, cu)
    return out, lse


def _call(torch, q, k, v, out, lse, B, Hq, Hkv, Sq, Sk, D, scale, causal, num_splits, pack_gqa,
          varlen, cu):
    stream = _stream_handle(torch, q.device)
    if q.dtype == torch.bfloat16:
        rc, _, splits, _ = gqa_attn_plan(B, Hq, Hkv, Sq, Sk, D, scale, causal, num_splits,
                                         pack_gqa, varlen)
        if rc == 0 and splits > 1:
            _workspace(torch, q.device, gqa_attn_workspace_bytes(B, Hq, Sq, D, splits))
        rc = gqa_attn_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, Hq, Hkv, Sq, Sk,
                          D, scale, int(bool(causal)), num_splits, pack_gqa, _ptr(cu), stream)
        if rc != 0:
            raise GqaError("gqa_attn_fwd", rc)
    else:
        rc = gqa_attn_fwd_f32(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, Hq, Hkv, Sq,
                              Sk, D, scale, int(bool(causal)), num_splits, pack_gqa, _ptr(cu),
                              stream)
        if rc != 0:
            raise GqaError("gqa_attn_fwd_f32", rc)


def gqa_attn_fp8(q8, k8, v8, *, q_scale: float, k_scale: float, v_scale: float,
                 causal: bool = False, scale: float | None = None, cu_seqlens=None,
                 max_seqlen: int | None = None, out=None, lse=None):
    """Prefill on e4m3 codes (gqa_attn_fwd_fp8): q8 [B, Sq, Hq, 128], k8/v8 [B, Sk, Hkv,
    128] as torch.float8_e4m3fn or uint8 on the GPU (or packed [total, H, 128] with
    cu_seqlens and max_seqlen); element = value(code) * its tensor's scale.  Returns
    (out bf16 like q8, lse)."""
    import torch

    for name, t in (("q8", q8), ("k8", k8), ("v8", v8)):
        if not t.is_cuda:
            raise ValueError(f"{name} must be a CUDA tensor (there is no CPU path)")
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
        if t.dtype not in (torch.uint8, torch.float8_e4m3fn):
            raise ValueError(f"{name} must hold e4m3 codes (uint8 or float8_e4m3fn)")
    varlen = cu_seqlens is not None
    if varlen:
        if q8.dim() != 3 or k8.dim() != 3 or v8.shape != k8.shape or max_seqlen is None:
            raise ValueError("packed q8 [total, Hq, D], k8/v8 [total, Hkv, D], max_seqlen")
        total, Hq, D = q8.shape
        Hkv = k8.shape[1]
        B, Sq, Sk = cu_seqlens.numel() - 1, int(max_seqlen), total
        lse_shape = (Hq, total)
    else:
        if q8.dim() != 4 or k8.dim() != 4 or v8.shape != k8.shape:
            raise ValueError("q8 [B, Sq, Hq, D], k8/v8 [B, Sk, Hkv, D]")
        B, Sq, Hq, D = q8.shape
        _, Sk, Hkv, _ = k8.shape
        lse_shape = (B, Hq, Sq)
    scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
    out = torch.empty(q8.shape, dtype=torch.bfloat16, device=q8.device) if out is None else out
    lse = torch.empty(lse_shape, dtype=torch.float32, device=q8.device) if lse is None else lse
    lib = _capi.load()
    with torch.cuda.device(q8.device):
        rc = lib.gqa_attn_fwd_fp8(_ptr(q8), _ptr(k8), _ptr(v8), _ptr(out), _ptr(lse), B, Hq,
                                  Hkv, Sq, Sk, D, scale, float(q_scale), float(k_scale),
                                  float(v_scale), int(bool(causal)),
                                  _ptr(cu_seqlens) if varlen else None,
                                  _stream_handle(torch, q8.device))
    if rc != 0:
        raise GqaError("gqa_attn_fwd_fp8", rc)
    return out, lse


class SparseVarlenPlan:
    """Device metadata of one packed block-sparse problem: each sequence's first
    pattern row (blk_off) and, when balanced, the tile order with its grid."""

    def __init__(self, blk_off, order, n_order: int, grid: int, rows: int):
        self.blk_off, self.order, self.n_order, self.grid, self.rows = \
            blk_off, order, n_order, grid, rows


def gqa_attn_blocksparse_varlen_plan(cu_seqlens, blk_row_ptr, *, Hq: int, Hkv: int,
                                     max_seqlen: int, device, balance: bool = True):
    """Build a SparseVarlenPlan with the library's host schedule
    (gqa_attn_sparse_varlen_schedule): cu_seqlens and blk_row_ptr are read on the host
    once, the plan's arrays live on `device`."""
    import numpy as np
    import torch

    lib = _capi.load()
    cu_h = np.ascontiguousarray(torch.as_tensor(cu_seqlens).cpu().numpy(), dtype=np.int32)
    rp_h = np.ascontiguousarray(torch.as_tensor(blk_row_ptr).cpu().numpy(), dtype=np.int32)
    B = cu_h.size - 1
    off_h = np.zeros(B + 1, dtype=np.int32)
    n_order, grid = ctypes.c_int(0), ctypes.c_int(0)
    sms = torch.cuda.get_device_properties(device).multi_processor_count
    args = (cu_h.ctypes.data, rp_h.ctypes.data, B, int(Hq), int(Hkv), int(max_seqlen), sms,
            off_h.ctypes.data)
    rc = lib.gqa_attn_sparse_varlen_schedule(*args, None, 0, ctypes.byref(n_order),
                                             ctypes.byref(grid))
    if rc not in (0, STATUS_CODE["GQA_ERR_WORKSPACE"]):
        raise GqaError("gqa_attn_sparse_varlen_schedule", rc)
    order_h = np.zeros(max(n_order.value, 1), dtype=np.int32)
    rc = lib.gqa_attn_sparse_varlen_schedule(*args, order_h.ctypes.data, order_h.size,
                                             ctypes.byref(n_order), ctypes.byref(grid))
    if rc != 0:
        raise GqaError("gqa_attn_sparse_varlen_schedule", rc)
    if int(off_h[-1]) + 1 != rp_h.size:
        raise ValueError(f"blk_row_ptr must hold {int(off_h[-1]) + 1} entries (one row per "
                         "128-position block of each sequence, plus one)")
    order = torch.from_numpy(order_h).to(device) if balance else None
    return SparseVarlenPlan(torch.from_numpy(off_h).to(device), order,
                            n_order.value if balance else 0, grid.value if balance else 0,
                            int(off_h[-1]))


def gqa_attn_blocksparse_varlen(q, k, v, cu_seqlens, blk_row_ptr, blk_col, *,
                                max_seqlen: int, plan=None, balance: bool = True,
                                causal: bool = False, scale: float | None = None, out=None,
                                lse=None):
    """Block-sparse attention over packed sequences with minimum padding
    (gqa_attn_fwd_blocksparse_varlen).

    q [total, Hq, D], k/v [total, Hkv, D] bf16 on the GPU (Hq / Hkv >= 2 dividing 128);
    cu_seqlens int32 [B + 1] on the GPU; blk_row_ptr / blk_col int32 on the GPU: one
    pattern row per 128-position block of each sequence in order, col entries counting
    the sequence's own key blocks.  `plan` (gqa_attn_blocksparse_varlen_plan) is built
    here when not given; balance=True orders the tiles by the library's host schedule
    (longest first onto the least loaded CTA); causal=True also masks keys after each
    query within the listed blocks.  Returns (out, lse [Hq, total])."""
    import torch

    for name, t in (("q", q), ("k", k), ("v", v), ("cu_seqlens", cu_seqlens),
                    ("blk_row_ptr", blk_row_ptr), ("blk_col", blk_col)):
        if not t.is_cuda:
            raise ValueError(f"{name} must be a CUDA tensor (there is no CPU path)")
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
    if not (q.dtype == k.dtype == v.dtype == torch.bfloat16):
        raise ValueError("q, k, v must be bf16")
    if q.dim() != 3 or k.dim() != 3 or v.shape != k.shape or k.shape[0] != q.shape[0]:
        raise ValueError("q [total, Hq, D], k/v [total, Hkv, D]")
    for name, t in (("cu_seqlens", cu_seqlens), ("blk_row_ptr", blk_row_ptr),
                    ("blk_col", blk_col)):
        if t.dtype != torch.int32:
            raise ValueError(f"{name} must be int32")
    total, Hq, D = q.shape
    Hkv = k.shape[1]
    B = cu_seqlens.numel() - 1
    if plan is None:
        plan = gqa_attn_blocksparse_varlen_plan(cu_seqlens, blk_row_ptr, Hq=Hq, Hkv=Hkv,
                                                max_seqlen=max_seqlen, device=q.device,
                                                balance=balance)
    if plan.rows + 1 != blk_row_ptr.numel():
        raise ValueError("the plan was built for another pattern")
    scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
    out = torch.empty_like(q) if out is None else out
    lse = torch.empty(Hq, total, dtype=torch.float32, device=q.device) if lse is None else lse
    lib = _capi.load()
    with torch.cuda.device(q.device):
        rc = lib.gqa_attn_fwd_blocksparse_varlen(
            _ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), _ptr(cu_seqlens),
            _ptr(plan.blk_off), B, Hq, Hkv, int(max_seqlen), total, D, scale,
            int(bool(causal)), _ptr(blk_row_ptr), _ptr(blk_col), None if plan.order is None else _ptr(plan.order),
            plan.n_order, plan.grid, _stream_handle(torch, q.device))
    if rc != 0:
        raise GqaError("gqa_attn_fwd_blocksparse_varlen", rc)
    return out, lse


def gqa_attn_backward(q, k, v, out, lse, dout, *, causal: bool = False,
                      scale: float | None = None, dq=None, dk=None, dv=None):
    """dQ, dK, dV of gqa_attn's dense forward for the gradient dout (gqa_attn_bwd).

    q, out, dout [B, Sq, Hq, D], k/v [B, Sk, Hkv, D] bf16 on the GPU; lse [B, Hq, Sq] as
    gqa_attn returned it for the same inputs, causal and scale.  Returns (dq, dk, dv).
    """
    import torch

    if q.dim() != 4 or k.dim() != 4 or v.shape != k.shape or out.shape != q.shape \
            or dout.shape != q.shape:
        raise ValueError("q/out/dout [B, Sq, Hq, D], k/v [B, Sk, Hkv, D]")
    B, Sq, Hq, D = q.shape
    _, Sk, Hkv, _ = k.shape
    if k.shape[0] != B or k.shape[3] != D:
        raise ValueError("k/v must match q in batch and head dimension")
    if tuple(lse.shape) != (B, Hq, Sq):
        raise ValueError(f"lse must be [B, Hq, Sq] = {(B, Hq, Sq)}, got {tuple(lse.shape)}")
    if not (q.dtype == k.dtype == v.dtype == out.dtype == dout.dtype == torch.bfloat16):
        raise ValueError("q, k, v, out, dout must be bf16")
    if lse.dtype != torch.float32:
        raise ValueError("lse must be fp32")
    for name, g, like in (("dq", dq, q), ("dk", dk, k), ("dv", dv, v)):
        if g is not None and (g.shape != like.shape or g.dtype != like.dtype
                              or g.device != like.device or not g.is_contiguous()):
            raise ValueError(f"{name} must be a contiguous bf16 tensor shaped like its input, "
                             "on the same device")
    for name, t in (("q", q), ("k", k), ("v", v), ("out", out), ("lse", lse), ("dout", dout)):
        if not t.is_cuda:
            raise ValueError(f"{name} must be a CUDA tensor (there is no CPU path)")
        if t.device != q.device:
            raise ValueError(f"{name} must be on q's device")
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
    scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    lib = _capi.load()
    with torch.cuda.device(q.device):
        _workspace(torch, q.device, lib.gqa_attn_bwd_workspace_bytes(B, Hq, Sq))
        rc = lib.gqa_attn_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), _ptr(dout),
                              _ptr(dq), _ptr(dk), _ptr(dv), B, Hq, Hkv, Sq, Sk, D, scale,
                              int(bool(causal)), _stream_handle(torch, q.device))
    if rc != 0:
        raise GqaError("gqa_attn_bwd", rc)
    return dq, dk, dv


def gqa_attn_blocksparse(q, k, v, blk_row_ptr, blk_col, *, causal: bool = False,
                         scale: float | None = None, out=None, lse=None):
    """Attention restricted to a block pattern (gqa_attn_fwd_blocksparse), optionally
    also causal.

    q [B, Sq, Hq, D], k/v [B, Sk, Hkv, D] bf16 (Hq / Hkv >= 2 and dividing 128);
    blk_row_ptr int32 [ceil(Sq / 128) + 1] and blk_col int32 [nnz] on the GPU: the
    128-key blocks each 128-position query block attends to.  Returns (out, lse).
    """
    import torch

    for name, t in (("q", q), ("k", k), ("v", v), ("blk_row_ptr", blk_row_ptr),
                    ("blk_col", blk_col)):
        if not t.is_cuda:
            raise ValueError(f"{name} must be a CUDA tensor (there is no CPU path)")
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
    if not (q.dtype == k.dtype == v.dtype == torch.bfloat16):
        raise ValueError("q, k, v must be bf16")
    if blk_row_ptr.dtype != torch.int32 or blk_col.dtype != torch.int32:
        raise ValueError("the block pattern is int32")
    if q.dim() != 4 or k.dim() != 4 or v.shape != k.shape:
        raise ValueError("dense inputs are q [B, Sq, Hq, D], k/v [B, Sk, Hkv, D]")
    B, Sq, Hq, D = q.shape
    _, Sk, Hkv, _ = k.shape
    if blk_row_ptr.numel() != -(-Sq // 128) + 1:
        raise ValueError("blk_row_ptr must have ceil(Sq / 128) + 1 entries")
    scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, Hq, Sq), dtype=torch.float32, device=q.device)
    col = blk_col if blk_col.numel() else torch.zeros(1, dtype=torch.int32, device=q.device)
    with torch.cuda.device(q.device):
        rc = _capi.load().gqa_attn_fwd_blocksparse(
            _ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, Hq, Hkv, Sq, Sk, D, scale,
            int(bool(causal)), _ptr(blk_row_ptr), _ptr(col), _stream_handle(torch, q.device))
    if rc != 0:
        raise GqaError("gqa_attn_fwd_blocksparse", rc)
    return out, lse


def gqa_attn_kvcache(q, k_cache, v_cache, *, seqlens_k=None, max_seqlen_k=None,
                     block_table=None, window: int = 0, scale: float | None = None,
                     num_splits: int = 0, pack_gqa: int = -1, k_scale: float | None = None,
                     v_scale: float | None = None, out=None, lse=None):
    """One decode step against a KV cache (gqa_attn_decode_kvcache / _paged / _fp8).

    q [B, 1, Hq, D] bf16.  Dense cache: k_cache/v_cache [B, Sk, Hkv, D].  Paged
    cache (block_table given, int32 [B, max_pages]): k_cache/v_cache [num_pages,
    page_size, Hkv, D].  seqlens_k: int32 [B] keys per sequence (required when
    paged); max_seqlen_k: a host upper bound of it (read from the tensor when not
    given, which synchronises).  window > 0 keeps the last `window` keys.
    An e4m3 cache (torch.float8_e4m3fn or uint8 codes) needs k_scale and v_scale: the
    stored value is code * scale.  Returns (out [B, 1, Hq, D], lse [B, Hq, 1]).
    """
    import torch

    paged = block_table is not None
    tensors = [("q", q), ("k_cache", k_cache), ("v_cache", v_cache)]
    if seqlens_k is not None:
        tensors.append(("seqlens_k", seqlens_k))
    if paged:
        tensors.append(("block_table", block_table))
    for name, t in tensors:
        if not t.is_cuda:
            raise ValueError(f"{name} must be a CUDA tensor (there is no CPU path)")
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
    fp8_types = (torch.uint8, getattr(torch, "float8_e4m3fn", torch.uint8))
    fp8 = k_cache.dtype in fp8_types
    if q.dtype != torch.bfloat16:
        raise ValueError("q must be bf16")
    if fp8:
        if v_cache.dtype not in fp8_types:
            raise ValueError("k_cache and v_cache must both be e4m3 (or both bf16)")
        if k_scale is None or v_scale is None:
            raise ValueError("an e4m3 cache needs k_scale and v_scale")
    elif not (k_cache.dtype == v_cache.dtype == torch.bfloat16):
        raise ValueError("k_cache, v_cache must be bf16 or e4m3")
    if q.dim() != 4 or q.shape[1] != 1 or k_cache.dim() != 4 or v_cache.shape != k_cache.shape:
        raise ValueError("q is [B, 1, Hq, D]; k_cache/v_cache are 4-D and alike")
    B, _, Hq, D = q.shape
    Hkv = k_cache.shape[2]
    for name, t in (("seqlens_k", seqlens_k), ("block_table", block_table)):
        if t is not None and t.dtype != torch.int32:
            raise ValueError(f"{name} must be int32")
    if seqlens_k is not None and seqlens_k.shape != (B,):
        raise ValueError("seqlens_k must be [B]")
    if paged:
        if seqlens_k is None:
            raise ValueError("a paged cache needs seqlens_k")
        if block_table.dim() != 2 or block_table.shape[0] != B:
            raise ValueError("block_table must be [B, max_pages]")
        num_pages, page_size = k_cache.shape[0], k_cache.shape[1]
        max_pages = block_table.shape[1]
        cap = max_pages * page_size
    else:
        cap = k_cache.shape[1]
        if k_cache.shape[0] != B:
            raise ValueError("a dense cache is [B, Sk, Hkv, D]")
    if seqlens_k is not None and max_seqlen_k is None:
        max_seqlen_k = int(seqlens_k.max().item()) if B > 0 else 0
    keys = int(max_seqlen_k) if seqlens_k is not None else cap
    if window > 0:
        keys = min(keys, int(window) + 64)
    scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, Hq, 1), dtype=torch.float32, device=q.device)
    with torch.cuda.device(q.device):
        stream = _stream_handle(torch, q.device)
        rc, _, splits, _ = gqa_attn_plan(B, Hq, Hkv, 1, keys, D, scale, False, num_splits,
                                         pack_gqa, False)
        if fp8 and num_splits == 0:
            splits = 64  # the e4m3 path picks its own count, at most 64
        if rc == 0 and splits > 1:
            _workspace(torch, q.device, gqa_attn_workspace_bytes(B, Hq, 1, D, splits))
        msl = int(max_seqlen_k) if seqlens_k is not None else 0
        if fp8:
            rc = _capi.load().gqa_attn_decode_fp8(
                _ptr(q), _ptr(k_cache), _ptr(v_cache), float(k_scale), float(v_scale),
                _ptr(block_table), _ptr(seqlens_k), _ptr(out), _ptr(lse), B, Hq, Hkv, D,
                0 if paged else cap, num_pages if paged else 0, page_size if paged else 0,
                max_pages if paged else 0, msl if (paged or seqlens_k is not None) else cap,
                scale, int(window), num_splits, pack_gqa, stream)
            name = "gqa_attn_decode_fp8"
        elif paged:
            rc = _capi.load().gqa_attn_decode_paged(
                _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_table), _ptr(seqlens_k),
                _ptr(out), _ptr(lse), B, Hq, Hkv, D, num_pages, page_size, max_pages, msl,
                scale, int(window), num_splits, pack_gqa, stream)
            name = "gqa_attn_decode_paged"
        else:
            rc = _capi.load().gqa_attn_decode_kvcache(
                _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(seqlens_k), _ptr(out), _ptr(lse), B,
                Hq, Hkv, cap, D, msl, scale, int(window), num_splits, pack_gqa, stream)
            name = "gqa_attn_decode_kvcache"
    if rc != 0:
        raise GqaError(name, rc)
    return out, lse


def gqa_attn_host(q_h, k_h, v_h, out_h, lse_h, q_d, k_d, v_d, out_d, lse_d, *,
                  causal: bool = False, scale: float | None = None, num_splits: int = 1,
                  pack_gqa: int = -1, chunks: int = 0, cu_seqlens=None, max_seqlen=None):
    """Attention on host-resident tensors with the transfers overlapped (gqa_attn_fwd_host).

    q_h, k_h, v_h, out_h, lse_h: CPU tensors (pinned for overlap) in the dense layouts of
    ``gqa_attn``; q_d ... lse_d: CUDA tensors of the same shapes used as the staging area.
    Enqueued on the current stream of q_d's device; out_h and lse_h are complete once
    that stream has been synchronised.
    """
    import torch

    if cu_seqlens is not None:
        return _gqa_attn_host_varlen(torch, q_h, k_h, v_h, out_h, lse_h, q_d, k_d, v_d, out_d,
                                     lse_d, causal, scale, pack_gqa, chunks, cu_seqlens,
                                     max_seqlen)
    B, Sq, Hq, D = q_d.shape
    _, Sk, Hkv, _ = k_d.shape
    for h, d in ((q_h, q_d), (k_h, k_d), (v_h, v_d), (out_h, out_d), (lse_h, lse_d)):
        if h.device.type != "cpu" or d.device != q_d.device or h.shape != d.shape or \
                h.dtype != d.dtype or not h.is_contiguous() or not d.is_contiguous():
            raise ValueError("host tensors on the CPU and device tensors on one GPU, "
                             "same shapes and dtypes, contiguous")
    if q_d.dtype != torch.bfloat16:
        raise ValueError("gqa_attn_host takes bf16 q, k, v")
    scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
    with torch.cuda.device(q_d.device):
        n = chunks if chunks > 0 else 8
        per = -(-B // max(1, min(n, B))) if B else 0
        need = 0
        for b in {per, B - (-(-B // per) - 1) * per} if per else ():
            rc, _, splits, _ = gqa_attn_plan(b, Hq, Hkv, Sq, Sk, D, scale, causal, num_splits,
                                             pack_gqa, False)
            if rc == 0 and splits > 1:
                need = max(need, gqa_attn_workspace_bytes(b, Hq, Sq, D, splits))
        _workspace(torch, q_d.device, need)
        stream = _stream_handle(torch, q_d.device)
        rc = _capi.load().gqa_attn_fwd_host(
            _ptr(q_h), _ptr(k_h), _ptr(v_h), _ptr(out_h), _ptr(lse_h), _ptr(q_d), _ptr(k_d),
            _ptr(v_d), _ptr(out_d), _ptr(lse_d), B, Hq, Hkv, Sq, Sk, D, scale,
            int(bool(causal)), num_splits, pack_gqa, chunks, stream)
    if rc != 0:
        raise GqaError("gqa_attn_fwd_host", rc)


def _gqa_attn_host_varlen(torch, q_h, k_h, v_h, out_h, lse_h, q_d, k_d, v_d, out_d, lse_d, causal,
                          scale, pack_gqa, chunks, cu_seqlens, max_seqlen):
    """Packed variable-length form; cu_seqlens = (host int32 [B+1], device int32 [B+1])."""
    cu_h, cu_d = cu_seqlens
    total, Hq, D = q_d.shape
    Hkv = k_d.shape[1]
    B = cu_h.numel() - 1
    for h, d in ((q_h, q_d), (k_h, k_d), (v_h, v_d), (out_h, out_d), (lse_h, lse_d)):
        if h.device.type != "cpu" or d.device != q_d.device or h.shape != d.shape or \
                h.dtype != d.dtype or not h.is_contiguous() or not d.is_contiguous():
            raise ValueError("host tensors on the CPU and device tensors on one GPU, "
                             "same shapes and dtypes, contiguous")
    if cu_h.device.type != "cpu" or cu_h.dtype != torch.int32 or cu_d.dtype != torch.int32 or \
            cu_d.device != q_d.device or cu_d.numel() != B + 1:
        raise ValueError("cu_seqlens = (host int32 [B+1], device int32 [B+1])")
    cu_h = cu_h.contiguous()
    if max_seqlen is None:
        max_seqlen = int((cu_h[1:] - cu_h[:-1]).max()) if B > 0 else 0
    scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
    with torch.cuda.device(q_d.device):
        stream = _stream_handle(torch, q_d.device)
        rc = _capi.load().gqa_attn_fwd_host_varlen(
            _ptr(q_h), _ptr(k_h), _ptr(v_h), _ptr(out_h), _ptr(lse_h), _ptr(q_d), _ptr(k_d),
            _ptr(v_d), _ptr(out_d), _ptr(lse_d), _ptr(cu_h), _ptr(cu_d), B, Hq, Hkv,
            int(max_seqlen), total, D, scale, int(bool(causal)), pack_gqa, chunks, stream)
    if rc != 0:
        raise GqaError("gqa_attn_fwd_host_varlen", rc)
