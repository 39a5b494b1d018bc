"""GPU parity of the backward pass (gqa_attn_bwd) against the float64 oracle's
gradients on the same seeded inputs, with lse and O from the library's own forward."""
import math

import numpy as np
import pytest
import torch

import oracle
from exact_attention_gqa_b200 import build, gqa_attn, gqa_attn_backward, \
    gqa_attn_get_device_error
from parity import bf16_backward_model, compare_grad

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    yield
    torch.cuda.synchronize()
    assert gqa_attn_get_device_error() == 0


def inputs(B, Hq, Hkv, Sq, Sk, D, seed):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(B, Sq, Hq, D, generator=g).bfloat16()
    k = torch.randn(B, Sk, Hkv, D, generator=g).bfloat16()
    v = torch.randn(B, Sk, Hkv, D, generator=g).bfloat16()
    do = torch.randn(B, Sq, Hq, D, generator=g).bfloat16()
    return q, k, v, do


def run_bwd(q, k, v, do, causal):
    qd, kd, vd, dod = (t.to(DEV) for t in (q, k, v, do))
    out, lse = gqa_attn(qd, kd, vd, causal=causal)
    grads = gqa_attn_backward(qd, kd, vd, out, lse, dod, causal=causal)
    torch.cuda.synchronize()
    return grads


@pytest.mark.parametrize("B,Hq,Hkv,Sq,Sk,D,causal", [
    (2, 8, 2, 300, 300, 128, True),    # GQA, causal, ragged tail
    (1, 8, 2, 200, 333, 64, False),
    (1, 4, 1, 257, 513, 128, True),    # MQA, Sq < Sk (bottom-right)
    (2, 4, 4, 130, 130, 64, True),     # MHA
    (1, 16, 2, 100, 700, 128, False),  # G = 8
    (1, 6, 2, 90, 90, 64, True),       # G = 3
    (3, 8, 2, 1, 500, 128, False),     # a single query row
])
def test_backward_matches_oracle(B, Hq, Hkv, Sq, Sk, D, causal):
    q, k, v, do = inputs(B, Hq, Hkv, Sq, Sk, D, seed=B + Sq + Sk + D)
    grads = run_bwd(q, k, v, do, causal)
    ref = oracle.attention_backward(q, k, v, do, scale=1 / math.sqrt(D), causal=causal)
    model = bf16_backward_model(q, k, v, do, 1 / math.sqrt(D), causal)
    for g, r, m in zip(grads, ref, model):
        compare_grad(g, r, m)


def test_backward_is_bitwise_reproducible():
    q, k, v, do = inputs(2, 8, 2, 400, 400, 128, seed=9)
    a = run_bwd(q, k, v, do, True)
    b = run_bwd(q, k, v, do, True)
    for x, y in zip(a, b):
        assert torch.equal(x, y)


def test_queries_without_keys_get_zero_gradient():
    # causal with Sq > Sk: the first Sq - Sk queries see no key
    q, k, v, do = inputs(1, 4, 2, 200, 80, 64, seed=11)
    dq, dk, dv = run_bwd(q, k, v, do, True)
    assert torch.all(dq[:, :120] == 0)
    ref = oracle.attention_backward(q, k, v, do, scale=0.125, causal=True)
    for g, r in zip((dq, dk, dv), ref):
        compare_grad(g, r)


@pytest.mark.parametrize("D", [64, 128])
def test_query_blocks_without_any_key(D):
    # causal with Sq - Sk >= 128: whole 128-query blocks see no key (their dQ launch
    # streams nothing and writes zeros); the later rows are checked against the oracle
    q, k, v, do = inputs(1, 4, 2, 400, 100, D, seed=13 + D)
    dq, dk, dv = run_bwd(q, k, v, do, True)
    assert torch.all(dq[:, :300] == 0)
    ref = oracle.attention_backward(q, k, v, do, scale=1 / math.sqrt(D), causal=True)
    model = bf16_backward_model(q, k, v, do, 1 / math.sqrt(D), True)
    for g, r, m in zip((dq, dk, dv), ref, model):
        compare_grad(g, r, m)


@pytest.mark.parametrize("B,Hq,Hkv,Sq,Sk,D,causal", [
    (1, 16, 2, 520, 390, 64, True),    # G = 8, several key and query blocks, Sq > Sk
    (2, 2, 2, 129, 1100, 128, True),   # MHA, one row past a block, long keys
    (1, 4, 1, 700, 65, 128, False),    # one key past a 64-key block
])
def test_backward_multiblock_shapes(B, Hq, Hkv, Sq, Sk, D, causal):
    q, k, v, do = inputs(B, Hq, Hkv, Sq, Sk, D, seed=B * 7 + Sq + Sk)
    grads = run_bwd(q, k, v, do, causal)
    ref = oracle.attention_backward(q, k, v, do, scale=1 / math.sqrt(D), causal=causal)
    model = bf16_backward_model(q, k, v, do, 1 / math.sqrt(D), causal)
    for g, r, m in zip(grads, ref, model):
        compare_grad(g, r, m)


def test_no_keys_gives_zero_dq():
    q, k, v, do = inputs(2, 4, 2, 50, 0, 64, seed=12)
    qd, dod = q.to(DEV), do.to(DEV)
    kd, vd = k.to(DEV), v.to(DEV)
    out = torch.zeros_like(qd)
    lse = torch.full((2, 4, 50), float("-inf"), device=DEV)
    dq, dk, dv = gqa_attn_backward(qd, kd, vd, out, lse, dod)
    torch.cuda.synchronize()
    assert torch.all(dq == 0) and dk.numel() == 0


def test_full_llama_backward_slice():
    """The benchmark's backward workload (B=4, Hq=32, Hkv=8, S=8192, D=128, causal) on
    the GPU; batch element 3, K/V head 5 (its 4 query heads) checked against the oracle."""
    import workloads as W
    w = W.LLAMA
    q, k, v = W.make_qkv(w)
    do = W.make_dout(w)
    dq, dk, dv = run_bwd(q, k, v, do, True)
    for t in (dq, dk, dv):
        assert torch.isfinite(t.float()).all()
    b, c = 3, 5
    hs = slice(c * w.G, (c + 1) * w.G)
    ref = oracle.attention_backward(q[b:b + 1, :, hs], k[b:b + 1, :, c:c + 1],
                                    v[b:b + 1, :, c:c + 1], do[b:b + 1, :, hs], scale=w.scale,
                                    causal=True)
    compare_grad(dq[b:b + 1, :, hs], ref[0])
    compare_grad(dk[b:b + 1, :, c:c + 1], ref[1])
    compare_grad(dv[b:b + 1, :, c:c + 1], ref[2])
