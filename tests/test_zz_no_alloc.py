"""The allocation-free split-KV decode entry point, called through the C ABI.

gqa_attn_decode_noalloc serves callers that cannot get device memory when they
run attention (a plugin handed only its input and output buffers, a loop that
may not pay for cudaMalloc): its split-KV partials live in a scratch array built
into the library instead of a registered workspace.  These checks compare it
with the regular entry point (gqa_attn_fwd with a registered workspace) on two
calls in a row, within the parity tolerance the other GPU tests use.  This file
is collected last so that a run stopping at its first failure has already run
everything else; it also passes alone in a fresh process.
"""
import ctypes
import math

import numpy as np
import pytest
import torch

import oracle
from exact_attention_gqa_b200 import STATUS, _capi, build, gqa_attn, gqa_attn_get_device_error, \
    gqa_attn_plan
from parity import BF16_MAX_ABS, BF16_MAX_LSE, compare

pytestmark = pytest.mark.gpu

SCRATCH_BYTES = 4 << 20  # GQA_NOALLOC_SCRATCH_BYTES in include/gqa_attn.h


def noalloc_fn():
    build.build()
    lib = _capi.load()
    fn = lib.gqa_attn_decode_noalloc
    P, I, F = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
    fn.argtypes = [P, P, P, P, P, I, I, I, I, I, F, I, I, P]
    fn.restype = I
    return fn


def call_noalloc(fn, q, k, v, splits, pack=-1):
    B, _, Hq, D = q.shape
    Sk, Hkv = k.shape[1], k.shape[2]
    out = torch.empty_like(q)
    lse = torch.empty(B, Hq, 1, dtype=torch.float32, device=q.device)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    rc = fn(ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(k.data_ptr()),
            ctypes.c_void_p(v.data_ptr()), ctypes.c_void_p(out.data_ptr()),
            ctypes.c_void_p(lse.data_ptr()), B, Hq, Hkv, Sk, D, 1.0 / math.sqrt(D), splits, pack,
            stream)
    return rc, out, lse


def draw(B, Hq, Hkv, Sk, D, seed):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(B, 1, Hq, D, generator=g).to(torch.bfloat16).cuda()
    k = torch.randn(B, Sk, Hkv, D, generator=g).to(torch.bfloat16).cuda()
    v = torch.randn(B, Sk, Hkv, D, generator=g).to(torch.bfloat16).cuda()
    return q, k, v


@pytest.mark.parametrize("D,splits,pack", [(128, 4, 1), (64, 8, 0), (128, 0, -1)])
def test_noalloc_decode_matches_workspace_path_twice(D, splits, pack):
    fn = noalloc_fn()
    # two calls in a row with different inputs: the second must not see the first's partials
    for call, seed in enumerate((101, 202)):
        q, k, v = draw(3, 32, 8, 2000 + 37 * call, D, seed + D)
        rc, out, lse = call_noalloc(fn, q, k, v, splits, pack)
        assert STATUS[rc] == "GQA_OK"
        ref_out, ref_lse = gqa_attn(q, k, v, num_splits=splits, pack_gqa=pack)
        torch.cuda.synchronize()
        d_out = (out.float() - ref_out.float()).abs().max().item()
        d_lse = (lse - ref_lse).abs().max().item()
        assert d_out <= BF16_MAX_ABS and d_lse <= BF16_MAX_LSE, (call, d_out, d_lse)
        # and both meet the bar against the float64 oracle
        compare(out, lse, *oracle.attention(q.cpu(), k.cpu(), v.cpu(), scale=1 / math.sqrt(D),
                                            causal=False))
    assert gqa_attn_get_device_error() == 0


def test_noalloc_rejects_partials_beyond_the_scratch():
    fn = noalloc_fn()
    B, Hq, D, splits = 64, 32, 128, 8      # 64*32*8*129*4 bytes > 4 MiB
    assert B * Hq * splits * (D + 1) * 4 > SCRATCH_BYTES
    q, k, v = draw(B, Hq, 8, 600, D, 7)
    rc, out, lse = call_noalloc(fn, q, k, v, splits)
    assert STATUS[rc] == "GQA_ERR_WORKSPACE"
    # automatic splits: on a 148-SM part the planner's count (at most one CTA per SM)
    # always fits the scratch, so the library's step-down loop is only a guard for parts
    # with more SMs; this checks the planned count the call actually runs with
    q1, k1, v1 = draw(1, Hq, 8, 8192, D, 8)
    rc_plan, _, n_auto, _ = gqa_attn_plan(1, Hq, 8, 1, 8192, D, num_splits=0, pack_gqa=1)
    assert STATUS[rc_plan] == "GQA_OK" and n_auto > 1
    assert Hq * n_auto * (D + 1) * 4 <= SCRATCH_BYTES
    rc, out, lse = call_noalloc(fn, q1, k1, v1, 0)
    assert STATUS[rc] == "GQA_OK"
    torch.cuda.synchronize()
    compare(out, lse, *oracle.attention(q1.cpu(), k1.cpu(), v1.cpu(),
                                        scale=1 / math.sqrt(D), causal=False))
