"""Float64 CPU oracle for grouped-query exact attention.

TEST INFRASTRUCTURE ONLY: the test suite, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package.  The CUDA library and
its Python binding never do, and they share no code with it.

The arithmetic lives in ``oracle.c`` (plain C, float64, OpenMP over rows); this
module only compiles it on first use and marshals numpy arrays.  Each entry point
states the passage of the pages it follows in the C source:

* ``attention``        -- the plain definition S = scale*QK^T, P = softmax(S),
                          O = PV, L = m + ln l (FlashAttention-2 summary page,
                          standard-attention and normalisation paragraphs), with the
                          causal mask of that page's masking paragraph and the
                          grouping of the Ultralytics GQA glossary, "How GQA works".
* ``attention_rows``   -- the same, for a list of (b, h, i) rows only.
* ``attention_keyrange`` / ``combine`` -- split-KV partials and their
                          log-sum-exp weighted combine.
* ``attention_tiled``  -- the per-step normalised (form 1) and deferred
                          normalisation (form 2) online-softmax forms.
* ``attention_backward`` -- dQ, dK, dV for a given dO (FA-2 page, backward pass).
* ``attention_blocksparse_varlen`` -- the block pattern over packed sequences, each
                          padded only to whole blocks (Raptor-T's minimum padding).
* ``attention_blocksparse`` -- attention restricted to a (query block, key block)
                          pattern (Raptor-T abstract: BigBird's block-sparse attention).
* ``attention_e4m3``   -- the forward on e4m3 Q, K, V codes with one scale per tensor
                          (the batch-size guide's FP8 precision lever).
* ``decode_kvcache``   -- one decode query per sequence against a dense or paged
                          KV cache with per-sequence lengths and a sliding window
                          (Ultralytics GQA glossary, KV-cache and related-techniques
                          sections).

Every function takes float32 numpy arrays (bf16 and fp32 values widen exactly)
and returns float64 arrays.
"""
from __future__ import annotations

import ctypes
import os
import pathlib
import subprocess

import numpy as np

_HERE = pathlib.Path(__file__).resolve().parent
_SRC = _HERE / "oracle.c"
_LIB_PATH = _HERE / "liboracle.so"
_lib = None

FLAWS = {
    "none": 0,
    "strided_heads": 1,
    "drop_diagonal": 2,
    "top_left_causal": 3,
    "no_scale": 4,
    "lse_no_max": 5,
    "fa1_no_rescale": 6,
    "swap_kv": 7,
    "pages_contiguous": 8,
    "window_short": 9,
    "e4m3_bias": 10,
    "sparse_row": 11,
    "bwd_no_d": 12,
    "e4m3_no_vscale": 13,
    "sparse_maxpad": 14,
}


def build(force: bool = False) -> pathlib.Path:
    """Compile oracle.c into liboracle.so next to it (gcc, -O2, OpenMP)."""
    if force or not _LIB_PATH.exists() or _LIB_PATH.stat().st_mtime < _SRC.stat().st_mtime:
        tmp = _LIB_PATH.with_suffix(f".so.tmp{os.getpid()}")
        cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared", str(_SRC),
               "-o", str(tmp), "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(str(_LIB_PATH))
        P = ctypes.c_void_p
        I = ctypes.c_int
        Dbl = ctypes.c_double
        lib.oracle_attention.argtypes = [P, P, P, P, P, I, I, I, I, I, I, Dbl, I, P, I]
        lib.oracle_attention_rows.argtypes = [P, P, P, I, I, I, I, I, I, Dbl, I, P, I, P, P,
                                              P, I]
        lib.oracle_attention_window.argtypes = [P, P, P, P, P, I, I, I, I, I, I, Dbl, I, P, I]
        lib.oracle_attention_rows_window.argtypes = [P, P, P, I, I, I, I, I, I, Dbl, I, I, P, I,
                                                     P, P, P, I]
        lib.oracle_attention_keyrange.argtypes = [P, P, P, P, P, I, I, I, I, I, I, Dbl, I, I,
                                                  I, I]
        lib.oracle_combine.argtypes = [I, I, P, P, P, P]
        lib.oracle_combine.restype = None
        lib.oracle_attention_tiled.argtypes = [P, P, P, P, P, I, I, I, I, I, I, Dbl, I, I, I,
                                               I]
        lib.oracle_decode_kvcache.argtypes = [P, P, P, P, P, P, P, I, I, I, I, I, I, I, I, I,
                                              Dbl, I]
        lib.oracle_decode_kvcache.restype = I
        lib.oracle_decode_kvcache_e4m3.argtypes = [P, P, P, Dbl, Dbl, P, P, P, P, I, I, I, I, I,
                                                   I, I, I, I, Dbl, I]
        lib.oracle_decode_kvcache_e4m3.restype = I
        lib.oracle_attention_e4m3.argtypes = [P, P, P, Dbl, Dbl, Dbl, P, P, I, I, I, I, I, I,
                                              Dbl, I, P, I]
        lib.oracle_attention_e4m3.restype = I
        lib.oracle_attention_blocksparse_varlen.argtypes = [P, P, P, P, P, P, I, I, I, I, Dbl,
                                                            I, P, P, I, I]
        lib.oracle_attention_blocksparse_varlen.restype = I
        lib.oracle_attention_blocksparse.argtypes = [P, P, P, P, P, I, I, I, I, I, I, Dbl, I, P,
                                                     P, I, I]
        lib.oracle_attention_blocksparse.restype = I
        lib.oracle_attention_backward.argtypes = [P, P, P, P, P, P, P, I, I, I, I, I, I, Dbl, I,
                                                  I]
        lib.oracle_attention_backward.restype = I
        lib.oracle_e4m3_table.argtypes = [P]
        lib.oracle_e4m3_table.restype = None
        lib.oracle_set_flaw.argtypes = [I]
        lib.oracle_set_flaw.restype = None
        lib.oracle_get_flaw.restype = I
        lib.oracle_max_threads.restype = I
        for name in ("oracle_attention", "oracle_attention_rows", "oracle_attention_keyrange",
                     "oracle_attention_tiled", "oracle_attention_window",
                     "oracle_attention_rows_window"):
            getattr(lib, name).restype = I
        _lib = lib
    return _lib


def _f32(a) -> np.ndarray:
    if hasattr(a, "detach"):  # torch tensor: widen bf16/fp16 exactly to float32
        a = a.detach().to("cpu").float().numpy()
    return np.ascontiguousarray(a, dtype=np.float32)


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _dims(q, k, cu):
    """(B, Hq, Hkv, Sq, Sk, D) from dense [B,S,H,D] or packed [total,H,D] arrays."""
    if cu is None:
        if q.ndim != 4 or k.ndim != 4:
            raise ValueError("dense inputs are [B, S, H, D]")
        B, Sq, Hq, D = q.shape
        _, Sk, Hkv, _ = k.shape
    else:
        if q.ndim != 3 or k.ndim != 3:
            raise ValueError("packed inputs are [total, H, D]")
        B = len(cu) - 1
        _, Hq, D = q.shape
        _, Hkv, _ = k.shape
        Sq = Sk = int(np.max(np.diff(cu))) if B > 0 else 0
    return B, Hq, Hkv, Sq, Sk, D


def max_threads() -> int:
    return int(_load().oracle_max_threads())


def set_flaw(name: str) -> None:
    """Plant one deliberate mistake (pin-strength tests only); 'none' clears it."""
    _load().oracle_set_flaw(FLAWS[name])


def attention(q, k, v, *, scale: float, causal: bool, cu_seqlens=None, window: int = 0,
              threads: int = 0):
    """Full forward.  Returns (O float64 like q, L float64 [B,Hq,Sq] or [Hq,total]).
    window > 0 (causal only): each query sees its `window` most recent keys."""
    q, k, v = _f32(q), _f32(k), _f32(v)
    cu = None if cu_seqlens is None else np.ascontiguousarray(cu_seqlens, dtype=np.int32)
    B, Hq, Hkv, Sq, Sk, D = _dims(q, k, cu)
    o = np.zeros(q.shape, dtype=np.float64)
    lse = np.zeros((Hq, q.shape[0]) if cu is not None else (B, Hq, Sq), dtype=np.float64)
    if window:
        if not causal or window < 1:
            raise ValueError("a sliding window needs causal=True and window >= 1")
        rc = _load().oracle_attention_window(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B,
                                             Hq, Hkv, Sq, Sk, D, float(scale), int(window),
                                             None if cu is None else _ptr(cu), int(threads))
    else:
        rc = _load().oracle_attention(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, Hq,
                                      Hkv, Sq, Sk, D, float(scale), int(bool(causal)),
                                      None if cu is None else _ptr(cu), int(threads))
    if rc != 0:
        raise ValueError("oracle_attention: bad arguments")
    return o, lse


def attention_rows(q, k, v, rows, *, scale: float, causal: bool, cu_seqlens=None,
                   window: int = 0, threads: int = 0):
    """O and L for selected rows; rows is an int array [n, 3] of (b, h, i)."""
    q, k, v = _f32(q), _f32(k), _f32(v)
    cu = None if cu_seqlens is None else np.ascontiguousarray(cu_seqlens, dtype=np.int32)
    B, Hq, Hkv, Sq, Sk, D = _dims(q, k, cu)
    rows = np.ascontiguousarray(rows, dtype=np.int32).reshape(-1, 3)
    n = rows.shape[0]
    o = np.zeros((n, D), dtype=np.float64)
    lse = np.zeros((n,), dtype=np.float64)
    rc = _load().oracle_attention_rows_window(_ptr(q), _ptr(k), _ptr(v), B, Hq, Hkv, Sq, Sk,
                                              D, float(scale), int(bool(causal)), int(window),
                                              None if cu is None else _ptr(cu), n, _ptr(rows),
                                              _ptr(o), _ptr(lse), int(threads))
    if rc != 0:
        raise ValueError("oracle_attention_rows: bad arguments")
    return o, lse


def attention_keyrange(q, k, v, j0: int, j1: int, *, scale: float, causal: bool,
                       threads: int = 0):
    """Split-KV partial over keys [j0, j1) of a dense problem: (O_s, L_s)."""
    q, k, v = _f32(q), _f32(k), _f32(v)
    B, Hq, Hkv, Sq, Sk, D = _dims(q, k, None)
    o = np.zeros(q.shape, dtype=np.float64)
    lse = np.zeros((B, Hq, Sq), dtype=np.float64)
    rc = _load().oracle_attention_keyrange(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B,
                                           Hq, Hkv, Sq, Sk, D, float(scale),
                                           int(bool(causal)), int(j0), int(j1), int(threads))
    if rc != 0:
        raise ValueError("oracle_attention_keyrange: bad arguments")
    return o, lse


def combine(Os, Ls):
    """Log-sum-exp combine of one row's partials: Os [n, D], Ls [n] -> (O [D], L)."""
    Os = np.ascontiguousarray(Os, dtype=np.float64)
    Ls = np.ascontiguousarray(Ls, dtype=np.float64)
    n, D = Os.shape
    O = np.zeros((D,), dtype=np.float64)
    L = np.zeros((1,), dtype=np.float64)
    _load().oracle_combine(n, D, _ptr(Os), _ptr(Ls), _ptr(O), _ptr(L))
    return O, float(L[0])


def attention_tiled(q, k, v, *, scale: float, causal: bool, Bm: int, Bn: int, form: int):
    """Online-softmax forward in float64 with Bm x Bn blocks (form 1 or 2)."""
    q, k, v = _f32(q), _f32(k), _f32(v)
    B, Hq, Hkv, Sq, Sk, D = _dims(q, k, None)
    o = np.zeros(q.shape, dtype=np.float64)
    lse = np.zeros((B, Hq, Sq), dtype=np.float64)
    rc = _load().oracle_attention_tiled(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, Hq,
                                        Hkv, Sq, Sk, D, float(scale), int(bool(causal)),
                                        int(Bm), int(Bn), int(form))
    if rc != 0:
        raise ValueError("oracle_attention_tiled: bad arguments")
    return o, lse


def e4m3_table() -> np.ndarray:
    """Values of the 256 e4m3 codes (float64; NaN for 0x7f and 0xff)."""
    out = np.zeros(256, dtype=np.float64)
    _load().oracle_e4m3_table(_ptr(out))
    return out


def _codes(a):
    if hasattr(a, "detach"):  # torch uint8 or float8_e4m3fn: the raw bytes
        import torch
        a = a.detach().to("cpu")
        if a.dtype != torch.uint8:
            a = a.view(torch.uint8)
        a = a.numpy()
    return np.ascontiguousarray(a, dtype=np.uint8)


def attention_e4m3(q8, k8, v8, *, q_scale: float, k_scale: float, v_scale: float,
                   scale: float, causal: bool, cu_seqlens=None, threads: int = 0):
    """Forward on e4m3 codes (uint8 or float8_e4m3fn; element = value(code) * scale of
    its tensor), layouts as ``attention``.  Returns (O float64 like q, L float64)."""
    q, k, v = _codes(q8), _codes(k8), _codes(v8)
    cu = None if cu_seqlens is None else np.ascontiguousarray(cu_seqlens, dtype=np.int32)
    B, Hq, Hkv, Sq, Sk, D = _dims(q, k, cu)
    if v.shape != k.shape:
        raise ValueError("v must have the shape of k")
    o = np.zeros(q.shape, dtype=np.float64)
    lse = np.zeros((Hq, q.shape[0]) if cu is not None else (B, Hq, Sq), dtype=np.float64)
    rc = _load().oracle_attention_e4m3(_ptr(q), _ptr(k), _ptr(v), float(q_scale),
                                       float(k_scale), float(v_scale), _ptr(o), _ptr(lse), B,
                                       Hq, Hkv, Sq, Sk, D, float(scale), int(bool(causal)),
                                       None if cu is None else _ptr(cu), int(threads))
    if rc != 0:
        raise ValueError("oracle_attention_e4m3: bad arguments or a NaN code")
    return o, lse


def decode_kvcache(q, k_cache, v_cache, *, scale: float, seqlens_k=None, block_table=None,
                   window: int = 0, k_scale=None, v_scale=None, threads: int = 0):
    """Decode against a KV cache.  q [B, 1, Hq, D] or [B, Hq, D]; dense k/v_cache
    [B, Sk, Hkv, D] or paged [num_pages, page_size, Hkv, D] with block_table
    [B, max_pages].  With k_scale/v_scale the caches are e4m3 codes (uint8 or
    float8_e4m3fn) whose values are code * scale.  Returns (O float64 [B, Hq, D],
    L float64 [B, Hq])."""
    fp8 = k_scale is not None
    q = _f32(q)
    if fp8:
        k, v = _codes(k_cache), _codes(v_cache)
    else:
        k, v = _f32(k_cache), _f32(v_cache)
    B, Hq, D = q.shape[0], q.shape[-2], q.shape[-1]
    Hkv = k.shape[2]
    sl = None if seqlens_k is None else np.ascontiguousarray(_np_int(seqlens_k), dtype=np.int32)
    bt = None if block_table is None else np.ascontiguousarray(_np_int(block_table),
                                                                dtype=np.int32)
    if bt is None:
        Sk, page_size, max_pages, num_pages = k.shape[1], 0, 0, 0
    else:
        Sk, page_size, max_pages, num_pages = 0, k.shape[1], bt.shape[1], k.shape[0]
    o = np.zeros((B, Hq, D), dtype=np.float64)
    lse = np.zeros((B, Hq), dtype=np.float64)
    args = (None if bt is None else _ptr(bt), None if sl is None else _ptr(sl), _ptr(o),
            _ptr(lse), B, Hq, Hkv, D, Sk, page_size, max_pages, num_pages, int(window),
            float(scale), int(threads))
    if fp8:
        rc = _load().oracle_decode_kvcache_e4m3(_ptr(q), _ptr(k), _ptr(v), float(k_scale),
                                                float(v_scale), *args)
    else:
        rc = _load().oracle_decode_kvcache(_ptr(q), _ptr(k), _ptr(v), *args)
    if rc != 0:
        raise ValueError("oracle_decode_kvcache: bad arguments")
    return o, lse


def _np_int(a):
    if hasattr(a, "detach"):
        a = a.detach().to("cpu").numpy()
    return a


def attention_blocksparse(q, k, v, row_ptr, col, *, scale: float, blk: int = 128,
                          causal: bool = False, threads: int = 0):
    """Dense-layout attention restricted to a block pattern (CSR rows of key blocks per
    query block of blk positions), optionally also causal (bottom-right aligned).
    Returns (O float64 like q, L float64 [B,Hq,Sq])."""
    q, k, v = _f32(q), _f32(k), _f32(v)
    B, Hq, Hkv, Sq, Sk, D = _dims(q, k, None)
    rp = np.ascontiguousarray(_np_int(row_ptr), dtype=np.int32)
    cl = np.ascontiguousarray(_np_int(col), dtype=np.int32)
    if cl.size == 0:
        cl = np.zeros(1, dtype=np.int32)
    o = np.zeros(q.shape, dtype=np.float64)
    lse = np.zeros((B, Hq, Sq), dtype=np.float64)
    rc = _load().oracle_attention_blocksparse(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B,
                                              Hq, Hkv, Sq, Sk, D, float(scale),
                                              int(bool(causal)), _ptr(rp), _ptr(cl), int(blk),
                                              int(threads))
    if rc != 0:
        raise ValueError("oracle_attention_blocksparse: bad arguments")
    return o, lse


def attention_blocksparse_varlen(q, k, v, cu_seqlens, row_ptr, col, *, scale: float,
                                 blk: int = 128, causal: bool = False, threads: int = 0):
    """Packed sequences ([total, H, D]), each with its own block pattern: the pattern's
    rows are the query blocks of sequence 0, then of sequence 1, ... (ceil(n_b / blk)
    each), col entries are key blocks of the same sequence.  Returns (O float64 like q,
    L float64 [Hq, total])."""
    q, k, v = _f32(q), _f32(k), _f32(v)
    cu = np.ascontiguousarray(_np_int(cu_seqlens), dtype=np.int32)
    B, Hq, Hkv, _, _, D = _dims(q, k, cu)
    rp = np.ascontiguousarray(_np_int(row_ptr), dtype=np.int32)
    cl = np.ascontiguousarray(_np_int(col), dtype=np.int32)
    if cl.size == 0:
        cl = np.zeros(1, dtype=np.int32)
    n_rows = int(sum(-(-(int(cu[b + 1]) - int(cu[b])) // blk) for b in range(B)))
    if rp.size != n_rows + 1:
        raise ValueError(f"row_ptr must hold {n_rows + 1} entries (one row per block)")
    o = np.zeros(q.shape, dtype=np.float64)
    lse = np.zeros((Hq, q.shape[0]), dtype=np.float64)
    rc = _load().oracle_attention_blocksparse_varlen(_ptr(q), _ptr(k), _ptr(v), _ptr(o),
                                                     _ptr(lse), _ptr(cu), B, Hq, Hkv, D,
                                                     float(scale), int(bool(causal)), _ptr(rp),
                                                     _ptr(cl), int(blk), int(threads))
    if rc != 0:
        raise ValueError("oracle_attention_blocksparse_varlen: bad arguments")
    return o, lse


def attention_backward(q, k, v, dout, *, scale: float, causal: bool, threads: int = 0):
    """Gradients (dQ like q, dK and dV like k; float64) of the forward for a given dO."""
    q, k, v, do = _f32(q), _f32(k), _f32(v), _f32(dout)
    B, Hq, Hkv, Sq, Sk, D = _dims(q, k, None)
    dq = np.zeros(q.shape, dtype=np.float64)
    dk = np.zeros(k.shape, dtype=np.float64)
    dv = np.zeros(k.shape, dtype=np.float64)
    rc = _load().oracle_attention_backward(_ptr(q), _ptr(k), _ptr(v), _ptr(do), _ptr(dq),
                                           _ptr(dk), _ptr(dv), B, Hq, Hkv, Sq, Sk, D,
                                           float(scale), int(bool(causal)), int(threads))
    if rc != 0:
        raise ValueError("oracle_attention_backward: bad arguments")
    return dq, dk, dv
