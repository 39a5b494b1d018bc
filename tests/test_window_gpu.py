"""GPU parity of the causal sliding-window prefill (gqa_attn_fwd_window) against the
float64 oracle: windows smaller than, equal to and larger than a tile or a key block,
Sq != Sk, packed sequences, PackGQA on and off, D = 64 and 128, one decode query, and a
Llama-shaped batch with a 4096-key window checked on sampled rows."""
import math

import numpy as np
import pytest
import torch

import oracle
import workloads as W
from exact_attention_gqa_b200 import build, gqa_attn, gqa_attn_get_device_error
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


@pytest.mark.parametrize("B,Hq,Hkv,Sq,Sk,D,window,pack", [
    (2, 8, 2, 700, 700, 128, 1, 1),      # one key per query: the diagonal
    (2, 8, 2, 700, 700, 128, 3, 1),
    (1, 8, 2, 900, 900, 128, 128, 1),    # exactly one key block
    (1, 8, 2, 900, 900, 128, 129, 1),
    (1, 16, 2, 1000, 1000, 64, 300, 1),  # G = 8, D = 64
    (2, 4, 4, 520, 520, 128, 200, 0),    # MHA, no packing
    (1, 8, 2, 400, 1300, 128, 333, 1),   # Sq < Sk: bottom-right window
    (1, 8, 2, 700, 300, 64, 50, 1),      # Sq > Sk: first rows see nothing
    (1, 32, 8, 777, 777, 128, 500, -1),
])
def test_window_matches_oracle(B, Hq, Hkv, Sq, Sk, D, window, pack):
    q, k, v = rand_qkv(B, Hq, Hkv, Sq, Sk, D, seed=Sq + Sk + window)
    out, lse = gqa_attn(q.to(DEV), k.to(DEV), v.to(DEV), causal=True, window=window,
                        pack_gqa=pack)
    torch.cuda.synchronize()
    compare(out, lse, *oracle.attention(q, k, v, scale=1 / math.sqrt(D), causal=True,
                                        window=window))


def test_window_covering_every_key_equals_causal_attention():
    q, k, v = rand_qkv(2, 8, 2, 300, 300, 128, seed=7)
    qd, kd, vd = q.to(DEV), k.to(DEV), v.to(DEV)
    a = gqa_attn(qd, kd, vd, causal=True, window=300)
    b = gqa_attn(qd, kd, vd, causal=True)
    torch.cuda.synchronize()
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


def test_window_one_query_runs_the_decode_window():
    q, k, v = rand_qkv(3, 32, 8, 1, 5000, 128, seed=9)
    out, lse = gqa_attn(q.to(DEV), k.to(DEV), v.to(DEV), causal=True, window=1000)
    torch.cuda.synchronize()
    compare(out, lse, *oracle.attention(q, k, v, scale=1 / math.sqrt(128), causal=True,
                                        window=1000))


def test_window_varlen_is_per_sequence():
    lens = [300, 0, 1, 129, 1000, 57]
    cu = W.cu_seqlens_of(lens)
    total = int(cu[-1])
    g = torch.Generator().manual_seed(11)
    q = torch.randn(total, 8, 128, generator=g).bfloat16()
    k = torch.randn(total, 2, 128, generator=g).bfloat16()
    v = torch.randn(total, 2, 128, generator=g).bfloat16()
    out, lse = gqa_attn(q.to(DEV), k.to(DEV), v.to(DEV), causal=True, window=150,
                        cu_seqlens=cu.to(DEV), max_seqlen=max(lens))
    torch.cuda.synchronize()
    compare(out, lse, *oracle.attention(q, k, v, scale=1 / math.sqrt(128), causal=True,
                                        cu_seqlens=cu.numpy(), window=150))


def test_window_llama_shape_sampled_rows():
    """The Llama-8B prefill shape (B=4, Hq=32, Hkv=8, S=8192, D=128) with a 4096-key
    window (a Mistral-style sliding window): sampled rows against the oracle."""
    w = W.LLAMA
    q, k, v = W.make_qkv(w)
    out, lse = gqa_attn(q.to(DEV), k.to(DEV), v.to(DEV), causal=True, window=4096)
    torch.cuda.synchronize()
    assert torch.isfinite(out.float()).all() and torch.isfinite(lse).all()
    rng = np.random.default_rng(21)
    rows = {(int(rng.integers(w.B)), int(rng.integers(w.Hq)), int(rng.integers(w.Sq)))
            for _ in range(120)}
    rows |= {(0, 0, 0), (0, 0, 4095), (1, 5, 4096), (2, 9, 4097), (3, 31, 8191)}
    rows = np.array(sorted(rows), dtype=np.int32)
    o_ref, l_ref = oracle.attention_rows(q, k, v, rows, scale=w.scale, causal=True,
                                         window=4096)
    o_gpu = torch.stack([out[b, i, h] for b, h, i in rows])
    l_gpu = torch.stack([lse[b, h, i] for b, h, i in rows])
    compare(o_gpu, l_gpu, o_ref, l_ref)
