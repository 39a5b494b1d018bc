"""GPU parity of the KV-cache decode entry points against the float64 oracle.

gqa_attn_decode_kvcache (dense cache, per-sequence lengths) and
gqa_attn_decode_paged (a pool of fixed-size pages and a block table), both with an
optional sliding window (Ultralytics GQA glossary, "How GQA shrinks the KV cache"
and "GQA and related techniques").  Inputs are seeded; ragged lengths include 0,
block and page multiples; unused block-table entries hold -1 so that reading one
would show as a device error."""
import math

import numpy as np
import pytest
import torch

import oracle
from exact_attention_gqa_b200 import build, gqa_attn_get_device_error, gqa_attn_kvcache
from parity import compare

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    yield
    torch.cuda.synchronize()
    assert gqa_attn_get_device_error() == 0


def make_cache(B, Hq, Hkv, Sk, D, seed):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(B, 1, Hq, D, generator=g).bfloat16()
    k = torch.randn(B, Sk, Hkv, D, generator=g).bfloat16()
    v = torch.randn(B, Sk, Hkv, D, generator=g).bfloat16()
    return q, k, v


def to_pages(k, v, lens, page_size, seed, spare=5):
    """Scatter each sequence's first lens[b] keys into a shuffled pool of pages.
    Table entries past a sequence's last page are -1; unused rows hold noise."""
    B, Sk, Hkv, D = k.shape
    max_pages = -(-Sk // page_size)
    used = [-(-int(n) // page_size) for n in lens]
    num_pages = sum(used) + spare
    g = torch.Generator().manual_seed(seed)
    perm = torch.randperm(num_pages, generator=g)
    kp = (torch.randn(num_pages, page_size, Hkv, D, generator=g) * 3).bfloat16()
    vp = (torch.randn(num_pages, page_size, Hkv, D, generator=g) * 3).bfloat16()
    table = torch.full((B, max_pages), -1, dtype=torch.int32)
    nxt = 0
    for b in range(B):
        for pg in range(used[b]):
            phys = int(perm[nxt])
            nxt += 1
            table[b, pg] = phys
            j0, j1 = pg * page_size, min((pg + 1) * page_size, int(lens[b]))
            kp[phys, : j1 - j0] = k[b, j0:j1]
            vp[phys, : j1 - j0] = v[b, j0:j1]
    return kp, vp, table


def check(out, lse, o_ref, l_ref):
    compare(out[:, 0], lse[:, :, 0], o_ref, l_ref)


LENS = [0, 1, 63, 64, 65, 1500, 2999, 3000]


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("window", [0, 1, 100, 2000])
@pytest.mark.parametrize("splits,pack", [(1, 1), (3, 1), (0, 1), (0, 0)])
def test_dense_cache_with_lengths(D, window, splits, pack):
    B, Hq, Hkv, Sk = len(LENS), 32, 8, 3000
    q, k, v = make_cache(B, Hq, Hkv, Sk, D, seed=D + window + splits)
    lens = torch.tensor(LENS, dtype=torch.int32)
    out, lse = gqa_attn_kvcache(q.to(DEV), k.to(DEV), v.to(DEV), seqlens_k=lens.to(DEV),
                                max_seqlen_k=Sk, window=window, num_splits=splits,
                                pack_gqa=pack)
    torch.cuda.synchronize()
    check(out, lse, *oracle.decode_kvcache(q, k, v, scale=1 / math.sqrt(D), seqlens_k=lens,
                                           window=window))


def test_dense_cache_without_lengths_equals_the_dense_decode():
    from exact_attention_gqa_b200 import gqa_attn
    q, k, v = make_cache(3, 16, 4, 1234, 128, seed=5)
    qd, kd, vd = q.to(DEV), k.to(DEV), v.to(DEV)
    out, lse = gqa_attn_kvcache(qd, kd, vd, num_splits=4)
    ref_o, ref_l = gqa_attn(qd, kd, vd, num_splits=4)
    torch.cuda.synchronize()
    assert torch.equal(out, ref_o) and torch.equal(lse, ref_l)


@pytest.mark.parametrize("page_size", [16, 32, 64, 128, 256])
@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("window,splits", [(0, 1), (0, 0), (300, 4), (17, 0)])
def test_paged_cache(page_size, D, window, splits):
    B, Hq, Hkv, Sk = len(LENS), 16, 4, 3000
    q, k, v = make_cache(B, Hq, Hkv, Sk, D, seed=page_size + D + window)
    kp, vp, table = to_pages(k, v, LENS, page_size, seed=page_size * 3 + D)
    lens = torch.tensor(LENS, dtype=torch.int32)
    out, lse = gqa_attn_kvcache(q.to(DEV), kp.to(DEV), vp.to(DEV), seqlens_k=lens.to(DEV),
                                block_table=table.to(DEV), window=window, num_splits=splits)
    torch.cuda.synchronize()
    ref = oracle.decode_kvcache(q, kp, vp, scale=1 / math.sqrt(D), seqlens_k=lens,
                                block_table=table.clamp(min=0), window=window)
    check(out, lse, *ref)
    # the same logical cache through the dense entry point
    dense = oracle.decode_kvcache(q, k, v, scale=1 / math.sqrt(D), seqlens_k=lens, window=window)
    np.testing.assert_allclose(ref[0], dense[0], rtol=0, atol=1e-12)


def test_paged_sixteen_heads_per_kv_head_many_splits():
    B, Hq, Hkv, Sk, D = 3, 32, 2, 5000, 128
    lens = [5000, 4097, 1]
    q, k, v = make_cache(B, Hq, Hkv, Sk, D, seed=11)
    kp, vp, table = to_pages(k, v, lens, 64, seed=12)
    tl = torch.tensor(lens, dtype=torch.int32)
    out, lse = gqa_attn_kvcache(q.to(DEV), kp.to(DEV), vp.to(DEV), seqlens_k=tl.to(DEV),
                                block_table=table.to(DEV), num_splits=40)
    torch.cuda.synchronize()
    check(out, lse, *oracle.decode_kvcache(q, kp, vp, scale=1 / math.sqrt(D), seqlens_k=tl,
                                           block_table=table.clamp(min=0)))


def test_bad_page_and_length_raise_device_error_without_faulting():
    B, Hq, Hkv, Sk, D = 2, 8, 2, 200, 64
    q, k, v = make_cache(B, Hq, Hkv, Sk, D, seed=21)
    lens = [200, 100]
    kp, vp, table = to_pages(k, v, lens, 64, seed=22)
    table[1, 0] = kp.shape[0] + 3  # a page that is not in the pool
    tl = torch.tensor(lens, dtype=torch.int32)
    out, _ = gqa_attn_kvcache(q.to(DEV), kp.to(DEV), vp.to(DEV), seqlens_k=tl.to(DEV),
                              block_table=table.to(DEV))
    torch.cuda.synchronize()
    assert gqa_attn_get_device_error() == 3
    assert torch.isfinite(out.float()).all()
    # a length past the dense cache's capacity is clamped and reported the same way
    tl2 = torch.tensor([Sk + 5, 3], dtype=torch.int32)
    gqa_attn_kvcache(q.to(DEV), k.to(DEV), v.to(DEV), seqlens_k=tl2.to(DEV), max_seqlen_k=Sk)
    torch.cuda.synchronize()
    assert gqa_attn_get_device_error() == 3
    assert gqa_attn_get_device_error() == 0


def test_full_paged_decode_workload():
    """The benchmark's paged decode (B=16, Sk=32768, shuffled pages of 256 keys, automatic
    splits), whole, on the GPU; three sequences checked against the oracle, also with a
    4096-key window."""
    import workloads as W
    w = W.decode_paged(16)
    table = W.page_table(w).to(DEV)
    kp, vp = W.make_paged_kv(w, table, device=DEV)
    q = W.make_decode_q(w, device=DEV)
    lens = torch.full((w.B,), w.Sk, dtype=torch.int32, device=DEV)
    rng = np.random.default_rng(16)
    bs = sorted({0, w.B - 1, int(rng.integers(w.B))})
    for window in (0, 4096):
        out, lse = gqa_attn_kvcache(q, kp, vp, seqlens_k=lens, max_seqlen_k=w.Sk,
                                    block_table=table, window=window)
        torch.cuda.synchronize()
        assert torch.isfinite(out.float()).all()
        for b in bs:
            idx = table[b].long()
            kb = kp[idx].reshape(1, w.Sk, w.Hkv, w.D).cpu()
            vb = vp[idx].reshape(1, w.Sk, w.Hkv, w.D).cpu()
            ref = oracle.decode_kvcache(q[b:b + 1].cpu(), kb, vb, scale=w.scale, window=window)
            check(out[b:b + 1], lse[b:b + 1], *ref)


# ------------------------------------------------------------------ e4m3 (FP8) cache
def e4m3_cache(B, Sk, Hkv, D, seed, spread=50.0):
    """Finite e4m3 codes of N(0, spread^2) draws (|x| stays far below 448)."""
    g = torch.Generator().manual_seed(seed)
    k = (torch.randn(B, Sk, Hkv, D, generator=g) * spread).to(torch.float8_e4m3fn)
    v = (torch.randn(B, Sk, Hkv, D, generator=g) * spread).to(torch.float8_e4m3fn)
    return k, v


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("window,splits,pack", [(0, 1, 1), (0, 0, 1), (100, 3, 0), (2000, 0, 1)])
def test_fp8_dense_cache(D, window, splits, pack):
    B, Hq, Hkv, Sk = len(LENS), 32, 8, 3000
    q, _, _ = make_cache(B, Hq, Hkv, 1, D, seed=D + window)
    k8, v8 = e4m3_cache(B, Sk, Hkv, D, seed=D + splits)
    ks, vs = 1 / 50, 1 / 40
    lens = torch.tensor(LENS, dtype=torch.int32)
    out, lse = gqa_attn_kvcache(q.to(DEV), k8.to(DEV), v8.to(DEV), seqlens_k=lens.to(DEV),
                                max_seqlen_k=Sk, window=window, num_splits=splits,
                                pack_gqa=pack, k_scale=ks, v_scale=vs)
    torch.cuda.synchronize()
    check(out, lse, *oracle.decode_kvcache(q, k8, v8, scale=1 / math.sqrt(D), seqlens_k=lens,
                                           window=window, k_scale=ks, v_scale=vs))


@pytest.mark.parametrize("page_size", [16, 256])
@pytest.mark.parametrize("D", [64, 128])
def test_fp8_paged_cache_as_uint8_codes(page_size, D):
    B, Hq, Hkv, Sk = len(LENS), 16, 4, 3000
    q, _, _ = make_cache(B, Hq, Hkv, 1, D, seed=page_size + D)
    k8, v8 = e4m3_cache(B, Sk, Hkv, D, seed=page_size * 7 + D)
    ku, vu = k8.view(torch.uint8), v8.view(torch.uint8)
    # pages of codes through the same shuffled table as the bf16 test
    kp, vp, table = to_pages(ku.view(torch.int8).float(), vu.view(torch.int8).float(), LENS,
                             page_size, seed=page_size + 1)
    kp = kp.float().round().to(torch.int8).view(torch.uint8)
    vp = vp.float().round().to(torch.int8).view(torch.uint8)
    lens = torch.tensor(LENS, dtype=torch.int32)
    out, lse = gqa_attn_kvcache(q.to(DEV), kp.to(DEV), vp.to(DEV), seqlens_k=lens.to(DEV),
                                block_table=table.to(DEV), window=300, k_scale=0.02,
                                v_scale=0.03)
    torch.cuda.synchronize()
    ref = oracle.decode_kvcache(q, kp, vp, scale=1 / math.sqrt(D), seqlens_k=lens,
                                block_table=table.clamp(min=0), window=300, k_scale=0.02,
                                v_scale=0.03)
    check(out, lse, *ref)
    dense = oracle.decode_kvcache(q, ku, vu, scale=1 / math.sqrt(D), seqlens_k=lens, window=300,
                                  k_scale=0.02, v_scale=0.03)
    np.testing.assert_allclose(ref[0], dense[0], rtol=0, atol=1e-12)


def test_full_fp8_decode_workload():
    """The benchmark's e4m3 decode (B=16, Sk=32768, automatic splits) on the GPU, three
    sequences checked against the oracle's e4m3 decode."""
    import workloads as W
    w = W.decode_fp8(16)
    q = W.make_decode_q(w, device=DEV)
    k8 = torch.empty(w.B, w.Sk, w.Hkv, w.D, dtype=torch.float8_e4m3fn, device=DEV)
    v8 = torch.empty_like(k8)
    W.fill_decode_kv(w, k8, v8)
    out, lse = gqa_attn_kvcache(q, k8, v8, k_scale=W.FP8_SCALE, v_scale=W.FP8_SCALE)
    torch.cuda.synchronize()
    assert torch.isfinite(out.float()).all()
    rng = np.random.default_rng(8)
    for b in sorted({0, w.B - 1, int(rng.integers(w.B))}):
        ref = oracle.decode_kvcache(q[b:b + 1].cpu(), k8[b:b + 1].cpu(), v8[b:b + 1].cpu(),
                                    scale=w.scale, k_scale=W.FP8_SCALE, v_scale=W.FP8_SCALE)
        check(out[b:b + 1], lse[b:b + 1], *ref)


def nan_like(shape, fp8):
    if fp8:
        return torch.full(shape, 0x7F, dtype=torch.uint8).view(torch.float8_e4m3fn)
    return torch.full(shape, float("nan"), dtype=torch.bfloat16)


@pytest.mark.parametrize("fp8", [False, True])
@pytest.mark.parametrize("page_size", [0, 16, 64])
def test_unwritten_cache_rows_holding_nan_never_reach_the_output(fp8, page_size):
    """Rows a sequence does not own (past its length, in its last page or in the dense
    cache's spare capacity) hold NaN: their weight is 0, and nothing of them may show."""
    B, Hq, Hkv, Sk, D = 4, 16, 4, 700, 128
    lens = [700, 1, 300, 65]
    q, k, v = make_cache(B, Hq, Hkv, Sk, D, seed=31 + page_size)
    if fp8:
        k, v = e4m3_cache(B, Sk, Hkv, D, seed=32 + page_size)
    for b, n in enumerate(lens):
        k[b, n:] = nan_like(k[b, n:].shape, fp8)
        v[b, n:] = nan_like(v[b, n:].shape, fp8)
    kw = dict(k_scale=0.02, v_scale=0.02) if fp8 else {}
    tl = torch.tensor(lens, dtype=torch.int32)
    if page_size == 0:
        kc, vc, table = k, v, None
    else:
        per = -(-Sk // page_size)
        used = [-(-n // page_size) for n in lens]
        kc = nan_like((sum(used) + 3, page_size, Hkv, D), fp8)
        vc = nan_like((sum(used) + 3, page_size, Hkv, D), fp8)
        table = torch.full((B, per), -1, dtype=torch.int32)
        perm = torch.randperm(kc.shape[0], generator=torch.Generator().manual_seed(5))
        nxt = 0
        for b, n in enumerate(lens):
            for pg in range(used[b]):
                phys = int(perm[nxt])
                nxt += 1
                table[b, pg] = phys
                j1 = min((pg + 1) * page_size, n)
                kc[phys, : j1 - pg * page_size] = k[b, pg * page_size:j1]
                vc[phys, : j1 - pg * page_size] = v[b, pg * page_size:j1]
    out, lse = gqa_attn_kvcache(q.to(DEV), kc.to(DEV), vc.to(DEV), seqlens_k=tl.to(DEV),
                                max_seqlen_k=Sk,
                                block_table=None if table is None else table.to(DEV), **kw)
    torch.cuda.synchronize()
    assert torch.isfinite(out.float()).all()
    check(out, lse, *oracle.decode_kvcache(q, k, v, scale=1 / math.sqrt(D), seqlens_k=tl, **kw))
