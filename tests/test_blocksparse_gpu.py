"""GPU parity of the block-sparse prefill (gqa_attn_fwd_blocksparse) against the
float64 oracle: seeded patterns with ragged sequence tails, empty query blocks,
the full pattern (equal to the dense kernel), and the BigBird-style workload."""
import math

import numpy as np
import pytest
import torch

import oracle
from exact_attention_gqa_b200 import build, gqa_attn, gqa_attn_blocksparse, \
    gqa_attn_get_device_error
from parity import compare

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    yield
    torch.cuda.synchronize()
    assert gqa_attn_get_device_error() == 0


def rand_qkv(B, Hq, Hkv, Sq, Sk, D, seed):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(B, Sq, Hq, D, generator=g).bfloat16()
    k = torch.randn(B, Sk, Hkv, D, generator=g).bfloat16()
    v = torch.randn(B, Sk, Hkv, D, generator=g).bfloat16()
    return q, k, v


def pattern(n_q, n_k, seed, density=0.3, empty=()):
    rng = np.random.default_rng(seed)
    rows = []
    for r in range(n_q):
        cols = [] if r in empty else sorted(set(np.flatnonzero(rng.random(n_k) < density)
                                                .tolist()) | {min(r, n_k - 1)})
        rows.append(cols)
    rp = np.zeros(n_q + 1, dtype=np.int32)
    rp[1:] = np.cumsum([len(c) for c in rows])
    col = np.array([c for cs in rows for c in cs], dtype=np.int32)
    return torch.from_numpy(rp), torch.from_numpy(col)


@pytest.mark.parametrize("B,Hq,Hkv,Sq,Sk,D", [
    (2, 8, 2, 700, 900, 128),    # G = 4, ragged tails on both sides
    (1, 16, 2, 1000, 640, 64),   # G = 8, D = 64
    (2, 4, 2, 513, 513, 128),    # G = 2: one CTA tile = one query block
    (1, 32, 1, 300, 1100, 64),   # MQA, G = 32
])
def test_blocksparse_matches_oracle(B, Hq, Hkv, Sq, Sk, D):
    q, k, v = rand_qkv(B, Hq, Hkv, Sq, Sk, D, seed=Sq + Sk + D)
    n_q, n_k = -(-Sq // 128), -(-Sk // 128)
    rp, col = pattern(n_q, n_k, seed=Sq, empty=(1,))
    out, lse = gqa_attn_blocksparse(q.to(DEV), k.to(DEV), v.to(DEV), rp.to(DEV), col.to(DEV))
    torch.cuda.synchronize()
    ref = oracle.attention_blocksparse(q, k, v, rp, col, scale=1 / math.sqrt(D), blk=128)
    compare(out, lse, *ref)


def test_full_pattern_equals_the_dense_kernel():
    q, k, v = rand_qkv(2, 16, 4, 600, 777, 128, seed=3)
    n_q, n_k = -(-600 // 128), -(-777 // 128)
    rp = torch.arange(n_q + 1, dtype=torch.int32) * n_k
    col = torch.arange(n_k, dtype=torch.int32).repeat(n_q)
    qd, kd, vd = q.to(DEV), k.to(DEV), v.to(DEV)
    out, lse = gqa_attn_blocksparse(qd, kd, vd, rp.to(DEV), col.to(DEV))
    ref_o, ref_l = gqa_attn(qd, kd, vd, causal=False, pack_gqa=1)
    torch.cuda.synchronize()
    assert torch.equal(out, ref_o) and torch.equal(lse, ref_l)


def test_unsorted_rows_and_an_out_of_range_block():
    q, k, v = rand_qkv(1, 8, 2, 256, 384, 64, seed=5)
    rp = torch.tensor([0, 2, 4], dtype=torch.int32)
    col = torch.tensor([2, 0, 1, 2], dtype=torch.int32)  # row 0 in descending order
    out, lse = gqa_attn_blocksparse(q.to(DEV), k.to(DEV), v.to(DEV), rp.to(DEV), col.to(DEV))
    torch.cuda.synchronize()
    compare(out, lse, *oracle.attention_blocksparse(q, k, v, rp, col, scale=0.125, blk=128))
    bad = torch.tensor([0, 7, 1, 2], dtype=torch.int32)  # block 7 of 3
    gqa_attn_blocksparse(q.to(DEV), k.to(DEV), v.to(DEV), rp.to(DEV), bad.to(DEV))
    torch.cuda.synchronize()
    assert gqa_attn_get_device_error() == 2


def test_full_bigbird_workload():
    """The benchmark's block-sparse workload (B=4, Hq=32, Hkv=8, S=8192, D=128, BigBird-
    style pattern over 128-blocks), whole, on the GPU; two (batch element, KV head)
    groups of heads checked against the oracle."""
    import workloads as W
    w = W.BIGBIRD
    q, k, v = W.make_qkv(w)
    rp, col = W.bigbird_pattern(w)
    out, lse = gqa_attn_blocksparse(q.to(DEV), k.to(DEV), v.to(DEV), rp.to(DEV), col.to(DEV))
    torch.cuda.synchronize()
    assert torch.isfinite(out.float()).all() and torch.isfinite(lse).all()
    for b, c in ((0, 0), (3, 7)):
        hs = slice(c * w.G, (c + 1) * w.G)
        ref = oracle.attention_blocksparse(q[b:b + 1, :, hs], k[b:b + 1, :, c:c + 1],
                                           v[b:b + 1, :, c:c + 1], rp, col, scale=w.scale,
                                           blk=128)
        compare(out[b:b + 1, :, hs], lse[b:b + 1, hs], *ref)


# ------------------------------------------------------------------ causal patterns
@pytest.mark.parametrize("B,Hq,Hkv,Sq,Sk,D", [
    (2, 8, 2, 700, 700, 128),    # blocks above the diagonal in the pattern: fully masked
    (1, 16, 2, 500, 900, 64),    # Sq < Sk: the diagonal is shifted (bottom-right)
    (1, 8, 4, 640, 300, 128),    # Sq > Sk: the first rows see no key at all
])
def test_causal_blocksparse_matches_oracle(B, Hq, Hkv, Sq, Sk, D):
    q, k, v = rand_qkv(B, Hq, Hkv, Sq, Sk, D, seed=Sq + 3 * Sk + D)
    n_q, n_k = -(-Sq // 128), -(-Sk // 128)
    rp, col = pattern(n_q, n_k, seed=Sq + 1, density=0.5, empty=(2,))
    out, lse = gqa_attn_blocksparse(q.to(DEV), k.to(DEV), v.to(DEV), rp.to(DEV), col.to(DEV),
                                    causal=True)
    torch.cuda.synchronize()
    ref = oracle.attention_blocksparse(q, k, v, rp, col, scale=1 / math.sqrt(D), blk=128,
                                       causal=True)
    compare(out, lse, *ref)


def test_causal_full_pattern_equals_the_causal_dense_kernel():
    q, k, v = rand_qkv(2, 16, 4, 600, 777, 128, seed=13)
    n_q, n_k = -(-600 // 128), -(-777 // 128)
    rp = torch.arange(n_q + 1, dtype=torch.int32) * n_k
    col = torch.arange(n_k, dtype=torch.int32).repeat(n_q)
    qd, kd, vd = q.to(DEV), k.to(DEV), v.to(DEV)
    out, lse = gqa_attn_blocksparse(qd, kd, vd, rp.to(DEV), col.to(DEV), causal=True)
    torch.cuda.synchronize()
    ref = oracle.attention(q, k, v, scale=1 / math.sqrt(128), causal=True)
    compare(out, lse, *ref)
