"""GPU parity of the e4m3 prefill (gqa_attn_fwd_fp8) against the float64 oracle on the
same seeded codes; the bar for O follows a rounding model of the e4m3 arithmetic."""
import math

import numpy as np
import pytest
import torch

import oracle
from exact_attention_gqa_b200 import build, gqa_attn_fp8, gqa_attn_get_device_error
from parity import compare_e4m3, e4m3_prefill_model

pytestmark = pytest.mark.gpu

DEV = "cuda"
SCALES = dict(q_scale=0.5, k_scale=0.25, v_scale=2.0)


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    yield
    torch.cuda.synchronize()
    assert gqa_attn_get_device_error() == 0


def codes(shape, seed, spread=2.0):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(*shape, generator=g) * spread).to(torch.float8_e4m3fn)


@pytest.mark.parametrize("B,Hq,Hkv,Sq,Sk,causal", [
    (2, 8, 2, 300, 300, True),     # GQA, causal, ragged tail
    (1, 4, 1, 257, 513, True),     # MQA, Sq < Sk (bottom-right)
    (1, 8, 2, 200, 333, False),
    (2, 4, 4, 130, 130, True),     # MHA (no PackGQA)
    (3, 32, 8, 1, 500, False),     # one query row
])
def test_fp8_prefill_matches_oracle(B, Hq, Hkv, Sq, Sk, causal):
    seed = B + Hq + Sq + Sk
    q8, k8, v8 = codes((B, Sq, Hq, 128), seed), codes((B, Sk, Hkv, 128), seed + 1), \
        codes((B, Sk, Hkv, 128), seed + 2)
    scale = 1 / math.sqrt(128)
    out, lse = gqa_attn_fp8(q8.to(DEV), k8.to(DEV), v8.to(DEV), causal=causal, **SCALES)
    torch.cuda.synchronize()
    o_ref, l_ref = oracle.attention_e4m3(q8, k8, v8, scale=scale, causal=causal, **SCALES)
    model = e4m3_prefill_model(q8, k8, v8, SCALES["q_scale"], SCALES["k_scale"],
                               SCALES["v_scale"], scale, causal)
    compare_e4m3(out, lse, o_ref, l_ref, model)


def test_fp8_prefill_varlen_is_per_sequence():
    lens = [130, 0, 257, 64]
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lens)]), dtype=torch.int32)
    total = int(cu[-1])
    q8, k8, v8 = codes((total, 8, 128), 31), codes((total, 2, 128), 32), \
        codes((total, 2, 128), 33)
    out, lse = gqa_attn_fp8(q8.to(DEV), k8.to(DEV), v8.to(DEV), causal=True,
                            cu_seqlens=cu.to(DEV), max_seqlen=max(lens), **SCALES)
    torch.cuda.synchronize()
    for b, n in enumerate(lens):
        if n == 0:
            continue
        sl = slice(int(cu[b]), int(cu[b + 1]))
        o_ref, l_ref = oracle.attention_e4m3(q8[sl][None], k8[sl][None], v8[sl][None],
                                             scale=1 / math.sqrt(128), causal=True, **SCALES)
        model = e4m3_prefill_model(q8[sl][None], k8[sl][None], v8[sl][None],
                                   SCALES["q_scale"], SCALES["k_scale"], SCALES["v_scale"],
                                   1 / math.sqrt(128), True)
        compare_e4m3(out[sl][None], lse[:, sl][None], o_ref, l_ref, model)


def test_fp8_prefill_uint8_codes_equal_float8_codes():
    q8, k8, v8 = codes((1, 200, 8, 128), 41), codes((1, 200, 2, 128), 42), \
        codes((1, 200, 2, 128), 43)
    a = gqa_attn_fp8(q8.to(DEV), k8.to(DEV), v8.to(DEV), causal=True, **SCALES)
    b = gqa_attn_fp8(q8.view(torch.uint8).to(DEV), k8.view(torch.uint8).to(DEV),
                     v8.view(torch.uint8).to(DEV), causal=True, **SCALES)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


def test_full_llama_fp8_workload_prefix_and_suffix_rows():
    """The benchmark's e4m3 workload (Llama shape B=4, Hq=32, Hkv=8, S=8192, causal), whole
    on the GPU.  Causal rows depend only on the keys up to their own position, so the
    first 2048 positions of a (batch, KV head) group are exactly the problem cut to 2048
    positions, and the last 16 positions are the problem of those 16 queries against all
    8192 keys with bottom-right alignment: both are compared with the oracle, for two
    groups."""
    import workloads as W
    w = W.LLAMA_FP8
    sc = W.FP8_PREFILL_SCALE
    q8, k8, v8 = W.make_qkv_e4m3(w)
    out, lse = gqa_attn_fp8(q8.to(DEV), k8.to(DEV), v8.to(DEV), causal=True, q_scale=sc,
                            k_scale=sc, v_scale=sc)
    torch.cuda.synchronize()
    assert torch.isfinite(out.float()).all() and torch.isfinite(lse).all()
    for b, c in ((0, 0), (3, 7)):
        hs = slice(c * w.G, (c + 1) * w.G)
        kc, vc = k8[b:b + 1, :, c:c + 1].contiguous(), v8[b:b + 1, :, c:c + 1].contiguous()
        for rows in (slice(0, 2048), slice(w.Sq - 16, w.Sq)):
            qs = q8[b:b + 1, rows, hs].contiguous()
            ks, vs = (kc, vc) if rows.start > 0 else (kc[:, :2048].contiguous(),
                                                      vc[:, :2048].contiguous())
            o_ref, l_ref = oracle.attention_e4m3(qs, ks, vs, q_scale=sc, k_scale=sc,
                                                 v_scale=sc, scale=w.scale, causal=True)
            model = e4m3_prefill_model(qs, ks, vs, sc, sc, sc, w.scale, True)
            compare_e4m3(out[b:b + 1, rows, hs], lse[b:b + 1, hs, rows], o_ref, l_ref, model)
