"""GPU parity: the CUDA path (through the C ABI) against the float64 oracle on the
same seeded inputs.  Element-wise at sizes that span several tiles and a ragged
tail; sampled rows at the full workload sizes, launched as the benchmark does."""
import math

import numpy as np
import pytest
import torch

import oracle
import workloads as W
from exact_attention_gqa_b200 import (build, gqa_attn, gqa_attn_get_device_error, gqa_attn_host,
                                    gqa_attn_plan)
from parity import compare

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    yield
    torch.cuda.synchronize()
    assert gqa_attn_get_device_error() == 0


def rand_qkv(B, Hq, Hkv, Sq, Sk, D, seed, dtype=torch.bfloat16, q_mult=1.0):
    g = torch.Generator().manual_seed(seed)
    q = (torch.randn(B, Sq, Hq, D, generator=g).to(dtype) * q_mult).to(dtype)
    k = torch.randn(B, Sk, Hkv, D, generator=g).to(dtype)
    v = torch.randn(B, Sk, Hkv, D, generator=g).to(dtype)
    return q, k, v


def run(q, k, v, **kw):
    out, lse = gqa_attn(q.to(DEV), k.to(DEV), v.to(DEV), **kw)
    torch.cuda.synchronize()
    return out, lse


# ------------------------------------------------------------------ prefill, element-wise
PREFILL = [
    # B, Hq, Hkv, Sq,  Sk,  D,  causal, pack
    (2, 8, 2, 300, 300, 128, True, 1),
    (2, 8, 2, 300, 300, 128, True, 0),
    (2, 8, 2, 300, 333, 64, False, 1),
    (2, 8, 2, 300, 333, 64, False, 0),
    (1, 4, 1, 257, 513, 128, True, -1),   # MQA, Sq < Sk (bottom-right mask)
    (1, 4, 4, 130, 130, 64, True, -1),    # MHA (G = 1)
    (1, 6, 2, 200, 150, 128, True, 1),    # G = 3 (no packing possible), Sq > Sk
    (3, 16, 2, 700, 700, 128, True, 1),   # G = 8
    (1, 32, 8, 129, 129, 128, False, 1),
    (2, 16, 1, 64, 1000, 64, True, 1),    # G = 16, long keys, short queries
    (1, 8, 2, 2, 777, 128, True, 1),      # two query rows
    (1, 32, 1, 200, 200, 128, True, 1),   # MQA, G = 32: 4 positions per packed sub-tile
    (2, 8, 2, 3, 20000, 64, True, 1),     # 3 queries against 20000 keys (bottom-right)
    (1, 64, 8, 257, 257, 64, False, 1),   # G = 8 at D = 64, ragged tail
    (3, 12, 4, 190, 190, 64, True, 0),    # G = 3 without packing, causal, D = 64
]


@pytest.mark.parametrize("B,Hq,Hkv,Sq,Sk,D,causal,pack", PREFILL)
def test_prefill_matches_oracle(B, Hq, Hkv, Sq, Sk, D, causal, pack):
    q, k, v = rand_qkv(B, Hq, Hkv, Sq, Sk, D, seed=B * 1000 + Sq + Sk + D)
    scale = 1.0 / math.sqrt(D)
    out, lse = run(q, k, v, causal=causal, pack_gqa=pack)
    o_ref, l_ref = oracle.attention(q, k, v, scale=scale, causal=causal)
    compare(out, lse, o_ref, l_ref)


def test_prefill_large_logits():
    q, k, v = rand_qkv(2, 8, 2, 384, 384, 128, seed=7, q_mult=4.0)
    out, lse = run(q, k, v, causal=True)
    compare(out, lse, *oracle.attention(q, k, v, scale=1 / math.sqrt(128), causal=True))


def rising_qkv(B, Hq, Hkv, Sq, Sk, D, seed, step_log2=10.0):
    """Scores that rise block by block: every 128-key block's row max exceeds the
    previous block's by about `step_log2` in log2 units, so the online softmax must
    rescale its running output at every block (FlashAttention-2 summary page, online
    softmax: earlier partial results are rescaled when the running max grows)."""
    q, k, v = rand_qkv(B, Hq, Hkv, Sq, Sk, D, seed)
    scale = 1.0 / math.sqrt(D)
    step = step_log2 / (scale * 8.0 * math.log2(math.e))
    q[..., 0] = 8.0
    k[..., 0] = (torch.arange(Sk) // 128).to(torch.float32).mul(step).view(1, Sk, 1).to(k.dtype)
    return q, k, v


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("pack", [1, 0])
def test_prefill_rescales_at_every_block(D, causal, pack):
    q, k, v = rising_qkv(2, 8, 2, 520, 1100, D, seed=31 + D)
    out, lse = run(q, k, v, causal=causal, pack_gqa=pack)
    compare(out, lse, *oracle.attention(q, k, v, scale=1 / math.sqrt(D), causal=causal))


@pytest.mark.parametrize("splits", [1, 3, 0])
def test_decode_rescales_at_every_block(splits):
    q, k, v = rising_qkv(3, 32, 8, 1, 4000, 128, seed=77)
    out, lse = run(q, k, v, causal=False, num_splits=splits)
    compare(out, lse, *oracle.attention(q, k, v, scale=1 / math.sqrt(128), causal=False))


@pytest.mark.parametrize("D", [64, 128])
def test_decode_at_the_split_limit(D):
    """256 splits of one 64-key block each: the most partials the combine takes."""
    q, k, v = rand_qkv(1, 8, 2, 1, 256 * 64, D, seed=91 + D)
    rc, kern, splits, pack = gqa_attn_plan(1, 8, 2, 1, 256 * 64, D, num_splits=256)
    assert kern == "decode_splitkv" and splits == 256
    out, lse = run(q, k, v, causal=False, num_splits=256)
    compare(out, lse, *oracle.attention(q, k, v, scale=1 / math.sqrt(D), causal=False))


@pytest.mark.parametrize("splits", [2, 0])
def test_decode_sixteen_heads_per_kv_head(splits):
    """G = 16 packed in one CTA, D = 64, with and without splits."""
    q, k, v = rand_qkv(2, 32, 2, 1, 3000, 64, seed=93)
    out, lse = run(q, k, v, causal=False, num_splits=splits, pack_gqa=1)
    compare(out, lse, *oracle.attention(q, k, v, scale=1 / math.sqrt(64), causal=False))


@pytest.mark.parametrize("B,Hq,Hkv,Sq,Sk,D,causal,splits,chunks", [
    (5, 8, 2, 300, 300, 64, False, 1, 3),     # ragged chunks (2, 2, 1 batch elements)
    (4, 16, 4, 257, 513, 128, True, 1, 0),    # default chunking, Sq < Sk
    (6, 32, 8, 1, 3000, 128, False, 4, 4),    # decode, explicit splits per chunk
    (3, 8, 2, 64, 0, 64, True, 1, 2),         # no keys: zeros and -inf come back
    # fewer batch elements than chunks: ranges of query positions, keys copied as the
    # causal prefix grows (or all at once without the mask)
    (1, 8, 2, 2000, 2000, 128, True, 1, 0),   # 8 ranges of 256 positions, ragged last
    (2, 16, 4, 1100, 1500, 64, True, 1, 6),   # Sq < Sk: the prefix is shifted
    (3, 8, 8, 700, 900, 128, False, 1, 0),    # non-causal, MHA (no packing)
    (1, 32, 8, 4096, 4096, 128, True, 1, 64), # 16 ranges
    (2, 8, 2, 800, 600, 64, True, 1, 8),      # causal Sq > Sk: whole batch elements
])
def test_host_pipeline_equals_device_path(B, Hq, Hkv, Sq, Sk, D, causal, splits, chunks):
    """gqa_attn_fwd_host (inputs and outputs in pinned host memory, chunked and
    overlapped) gives exactly the device path's results."""
    q, k, v = rand_qkv(B, Hq, Hkv, Sq, Sk, D, seed=B * 7 + Sk + D)
    ref_o, ref_l = run(q, k, v, causal=causal, num_splits=splits)
    pin = lambda t: t.contiguous().pin_memory()
    qh, kh, vh = pin(q), pin(k), pin(v)
    oh = torch.empty_like(qh).pin_memory()
    lh = torch.empty(B, Hq, Sq, dtype=torch.float32).pin_memory()
    qd, kd, vd = torch.empty_like(q, device=DEV), torch.empty_like(k, device=DEV), \
        torch.empty_like(v, device=DEV)
    od, ld = torch.empty_like(qd), torch.empty(B, Hq, Sq, dtype=torch.float32, device=DEV)
    gqa_attn_host(qh, kh, vh, oh, lh, qd, kd, vd, od, ld, causal=causal, num_splits=splits,
                  chunks=chunks)
    torch.cuda.synchronize()
    assert torch.equal(oh, ref_o.cpu()) and torch.equal(lh, ref_l.cpu())
    compare(oh, lh, *oracle.attention(q, k, v, scale=1 / math.sqrt(D), causal=causal))


def test_host_pipeline_decode_auto_splits_per_chunk():
    """Chunks of 3, 3 and 1 batch elements pick different automatic split counts; the
    workspace covers the largest and every chunk meets the bar."""
    B, Hq, Hkv, Sk, D = 7, 32, 8, 5000, 128
    q, k, v = rand_qkv(B, Hq, Hkv, 1, Sk, D, seed=501)
    pin = lambda t: t.contiguous().pin_memory()
    qh, kh, vh = pin(q), pin(k), pin(v)
    oh = torch.empty_like(qh).pin_memory()
    lh = torch.empty(B, Hq, 1, dtype=torch.float32).pin_memory()
    qd, kd, vd = q.to(DEV), k.to(DEV), v.to(DEV)
    od, ld = torch.empty_like(qd), torch.empty(B, Hq, 1, dtype=torch.float32, device=DEV)
    splits = {gqa_attn_plan(b, Hq, Hkv, 1, Sk, D, num_splits=0)[2] for b in (3, 1)}
    assert len(splits) == 2
    gqa_attn_host(qh, kh, vh, oh, lh, qd, kd, vd, od, ld, num_splits=0, chunks=3)
    torch.cuda.synchronize()
    compare(oh, lh, *oracle.attention(q, k, v, scale=1 / math.sqrt(D), causal=False))


@pytest.mark.parametrize("chunks", [0, 3, 64])
def test_host_pipeline_varlen_equals_device_path(chunks):
    """gqa_attn_fwd_host_varlen: chunks of whole sequences, exactly the device path."""
    lengths = [300, 1, 0, 129, 700, 64, 513, 2]
    Hq, Hkv, D = 16, 4, 128
    cu = torch.tensor([0] + list(np.cumsum(lengths)), dtype=torch.int32)
    total = int(cu[-1])
    g = torch.Generator().manual_seed(606 + chunks)
    q = torch.randn(total, Hq, D, generator=g).to(torch.bfloat16)
    k = torch.randn(total, Hkv, D, generator=g).to(torch.bfloat16)
    v = torch.randn(total, Hkv, D, generator=g).to(torch.bfloat16)
    cu_d = cu.to(DEV)
    ref_o, ref_l = gqa_attn(q.to(DEV), k.to(DEV), v.to(DEV), causal=True, cu_seqlens=cu_d,
                            max_seqlen=max(lengths))
    torch.cuda.synchronize()
    pin = lambda t: t.contiguous().pin_memory()
    qh, kh, vh = pin(q), pin(k), pin(v)
    oh = torch.empty_like(qh).pin_memory()
    lh = torch.empty(Hq, total, dtype=torch.float32).pin_memory()
    qd, kd, vd = torch.empty_like(q, device=DEV), torch.empty_like(k, device=DEV), \
        torch.empty_like(v, device=DEV)
    od, ld = torch.empty_like(qd), torch.empty(Hq, total, dtype=torch.float32, device=DEV)
    gqa_attn_host(qh, kh, vh, oh, lh, qd, kd, vd, od, ld, causal=True, chunks=chunks,
                  cu_seqlens=(cu, cu_d), max_seqlen=max(lengths))
    torch.cuda.synchronize()
    assert torch.equal(oh, ref_o.cpu()) and torch.equal(lh, ref_l.cpu())


def test_pack_on_and_off_agree():
    q, k, v = rand_qkv(2, 16, 4, 333, 333, 128, seed=11)
    a, la = run(q, k, v, causal=True, pack_gqa=1)
    b, lb = run(q, k, v, causal=True, pack_gqa=0)
    o_ref, l_ref = oracle.attention(q, k, v, scale=1 / math.sqrt(128), causal=True)
    compare(a, la, o_ref, l_ref)
    compare(b, lb, o_ref, l_ref)
    # same key blocks in the same order: the two layouts give the same numbers
    assert torch.equal(a, b) and torch.equal(la, lb)


def test_gqa_equals_repeat_interleaved_mha_on_gpu():
    q, k, v = rand_qkv(1, 8, 2, 200, 200, 64, seed=13)
    a, la = run(q, k, v, causal=True, pack_gqa=0)
    b, lb = run(q, k.repeat_interleave(4, dim=2), v.repeat_interleave(4, dim=2), causal=True,
                pack_gqa=0)
    assert torch.equal(a, b) and torch.equal(la, lb)


# ------------------------------------------------------------------ decode (split-KV)
@pytest.mark.parametrize("splits", [1, 2, 4, 8, 0])
@pytest.mark.parametrize("pack", [1, 0])
def test_decode_matches_oracle(splits, pack):
    q, k, v = rand_qkv(3, 32, 8, 1, 1000, 128, seed=17)
    out, lse = run(q, k, v, causal=True, num_splits=splits, pack_gqa=pack)
    compare(out, lse, *oracle.attention(q, k, v, scale=1 / math.sqrt(128), causal=True))


@pytest.mark.parametrize("B,Hq,Hkv,Sk,D,splits", [
    (2, 8, 1, 4097, 64, 8),     # MQA, G = 8, D = 64
    (1, 48, 2, 300, 128, 3),    # G = 24: two head chunks per KV head
    (2, 4, 4, 65, 64, 2),       # MHA, one key past a block
    (1, 8, 2, 1, 128, 1),       # a single key
])
def test_decode_shapes(B, Hq, Hkv, Sk, D, splits):
    q, k, v = rand_qkv(B, Hq, Hkv, 1, Sk, D, seed=19 + Sk)
    out, lse = run(q, k, v, num_splits=splits)
    compare(out, lse, *oracle.attention(q, k, v, scale=1 / math.sqrt(D), causal=False))


# ------------------------------------------------------------------ variable length
@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("pack,D", [(1, 128), (0, 128), (1, 64)])
def test_varlen_matches_oracle(causal, pack, D):
    lengths = [5, 0, 300, 1, 129, 128, 257]
    cu = W.cu_seqlens_of(lengths)
    total = int(cu[-1])
    g = torch.Generator().manual_seed(23)
    q = torch.randn(total, 8, D, generator=g).to(torch.bfloat16)
    k = torch.randn(total, 2, D, generator=g).to(torch.bfloat16)
    v = torch.randn(total, 2, D, generator=g).to(torch.bfloat16)
    out, lse = gqa_attn(q.to(DEV), k.to(DEV), v.to(DEV), causal=causal, pack_gqa=pack,
                        cu_seqlens=cu.to(DEV), max_seqlen=max(lengths))
    torch.cuda.synchronize()
    compare(out, lse, *oracle.attention(q, k, v, scale=1 / math.sqrt(D), causal=causal,
                                        cu_seqlens=cu.numpy()))


# ------------------------------------------------------------------ edge cases
def test_no_keys_gives_zero_and_minus_inf():
    q, k, v = rand_qkv(2, 8, 2, 5, 0, 64, seed=29)
    out, lse = run(q, k, v)
    assert torch.all(out == 0) and torch.all(torch.isneginf(lse))


def test_empty_batch_is_a_noop():
    q, k, v = rand_qkv(0, 8, 2, 5, 5, 64, seed=31)
    out, lse = run(q, k, v)
    assert out.shape == (0, 5, 8, 64)


def test_writes_stay_inside_the_outputs():
    q, k, v = rand_qkv(1, 8, 2, 130, 130, 128, seed=37)
    n_out, n_lse = q.numel(), 8 * 130
    out_buf = torch.full((n_out + 4096,), 7.0, dtype=torch.bfloat16, device=DEV)
    lse_buf = torch.full((n_lse + 1024,), 7.0, dtype=torch.float32, device=DEV)
    out = out_buf[:n_out].view(q.shape)
    lse = lse_buf[:n_lse].view(1, 8, 130)
    gqa_attn(q.to(DEV), k.to(DEV), v.to(DEV), causal=True, out=out, lse=lse)
    torch.cuda.synchronize()
    assert torch.all(out_buf[n_out:] == 7.0) and torch.all(lse_buf[n_lse:] == 7.0)
    compare(out, lse, *oracle.attention(q, k, v, scale=1 / math.sqrt(128), causal=True))


def test_run_to_run_bitwise_determinism():
    q, k, v = rand_qkv(2, 16, 4, 500, 500, 128, seed=41)
    a = run(q, k, v, causal=True)
    b = run(q, k, v, causal=True)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


# ------------------------------------------------------------------ fp32 path
def test_fp32_glossary_example():
    q, k, v = W.make_qkv(W.TINY)
    out, lse = run(q, k, v, causal=True)
    o_ref, l_ref = oracle.attention(q, k, v, scale=W.TINY.scale, causal=True)
    compare(out, lse, o_ref, l_ref, f32=True)
    out2, lse2 = run(q, k.repeat_interleave(4, dim=2), v.repeat_interleave(4, dim=2), causal=True)
    assert torch.allclose(out, out2, atol=1e-6)
    assert torch.equal(out, out2)


@pytest.mark.parametrize("B,Hq,Hkv,Sq,Sk,D,causal", [
    (2, 6, 3, 37, 50, 40, True), (1, 4, 1, 70, 33, 96, True), (1, 2, 2, 1, 9, 256, False)])
def test_fp32_shapes(B, Hq, Hkv, Sq, Sk, D, causal):
    q, k, v = rand_qkv(B, Hq, Hkv, Sq, Sk, D, seed=43 + D, dtype=torch.float32)
    out, lse = run(q, k, v, causal=causal)
    compare(out, lse, *oracle.attention(q, k, v, scale=1 / math.sqrt(D), causal=causal), f32=True)


def test_fp32_varlen():
    lengths = [3, 0, 40, 17]
    cu = W.cu_seqlens_of(lengths)
    g = torch.Generator().manual_seed(47)
    total = int(cu[-1])
    q = torch.randn(total, 4, 64, generator=g)
    k = torch.randn(total, 2, 64, generator=g)
    v = torch.randn(total, 2, 64, generator=g)
    out, lse = gqa_attn(q.to(DEV), k.to(DEV), v.to(DEV), causal=True, cu_seqlens=cu.to(DEV),
                        max_seqlen=40)
    torch.cuda.synchronize()
    compare(out, lse, *oracle.attention(q, k, v, scale=1 / 8, causal=True, cu_seqlens=cu.numpy()),
            f32=True)


# ------------------------------------------------------------------ full workload sizes
def sample_rows(rng, B, Hq, Sq, n, extra=()):
    rows = {(int(rng.integers(B)), int(rng.integers(Hq)), int(rng.integers(Sq))) for _ in range(n)}
    rows |= set(extra)
    return np.array(sorted(rows), dtype=np.int32)


def check_rows(out, lse, q, k, v, rows, scale, causal, cu=None):
    o_ref, l_ref = oracle.attention_rows(q, k, v, rows, scale=scale, causal=causal,
                                         cu_seqlens=cu)
    if cu is None:
        o_gpu = torch.stack([out[b, i, h] for b, h, i in rows])
        l_gpu = torch.stack([lse[b, h, i] for b, h, i in rows])
    else:
        o_gpu = torch.stack([out[cu[b] + i, h] for b, h, i in rows])
        l_gpu = torch.stack([lse[h, cu[b] + i] for b, h, i in rows])
    return compare(o_gpu, l_gpu, o_ref, l_ref)


@pytest.mark.parametrize("pack", [1, 0])
def test_full_encoder_workload(pack):
    w = W.ENCODER
    q, k, v = W.make_qkv(w)
    out, lse = run(q, k, v, causal=w.causal, pack_gqa=pack)
    assert torch.isfinite(out).all() and torch.isfinite(lse).all()
    rng = np.random.default_rng(1)
    edges = [(0, 0, 0), (w.B - 1, w.Hq - 1, w.Sq - 1), (3, 5, 127), (3, 5, 128), (7, 47, 255)]
    check_rows(out, lse, q, k, v, sample_rows(rng, w.B, w.Hq, w.Sq, 200, edges), w.scale,
               w.causal)


@pytest.mark.parametrize("w", [W.LLAMA, W.LLAMA_STRESS], ids=lambda w: w.name)
def test_full_llama_prefill_workload(w):
    q, k, v = W.make_qkv(w)
    out, lse = run(q, k, v, causal=w.causal)
    assert torch.isfinite(out).all() and torch.isfinite(lse).all()
    rng = np.random.default_rng(2)
    edges = [(0, 0, 0), (0, 0, 1), (3, 31, 8191), (1, 7, 63), (1, 7, 64), (2, 9, 4095),
             (2, 9, 4096)]
    check_rows(out, lse, q, k, v, sample_rows(rng, w.B, w.Hq, w.Sq, 150, edges), w.scale,
               w.causal)


@pytest.mark.parametrize("B", W.DECODE_BATCHES)
def test_full_decode_workload(B):
    """Every batch size of the decode sweep (B up to 256: a 34 GB cache, drawn on the
    device one element at a time) at every split count the sweep times, the automatic
    count (0) included, with and without PackGQA; sampled batch elements {0, B - 1, one
    at random} are compared element-wise with the oracle on that element's cache."""
    w = W.decode(B)
    q = W.make_decode_q(w, device=DEV)
    k = torch.empty(B, w.Sk, w.Hkv, w.D, dtype=torch.bfloat16, device=DEV)
    v = torch.empty_like(k)
    W.fill_decode_kv(w, k, v)
    rng = np.random.default_rng(B)
    bs = sorted({0, B - 1, int(rng.integers(B))})
    # the oracle's result for an element does not depend on the split count or packing
    refs = {b: oracle.attention(q[b:b + 1].cpu(), k[b:b + 1].cpu(), v[b:b + 1].cpu(),
                                scale=w.scale, causal=False) for b in bs}
    for splits in W.DECODE_SPLITS + (0,):
        for pack in (1, 0):
            out, lse = gqa_attn(q, k, v, num_splits=splits, pack_gqa=pack)
            torch.cuda.synchronize()
            for b in bs:
                compare(out[b:b + 1], lse[b:b + 1], *refs[b])
    del k, v
    torch.cuda.empty_cache()


def test_full_varlen_workload():
    w = W.VARLEN
    lengths = W.varlen_lengths(w)
    q, k, v, cu = W.make_varlen(w, lengths=lengths)
    out, lse = gqa_attn(q.to(DEV), k.to(DEV), v.to(DEV), causal=True, cu_seqlens=cu.to(DEV),
                        max_seqlen=int(lengths.max()))
    torch.cuda.synchronize()
    assert torch.isfinite(out).all() and torch.isfinite(lse).all()
    rng = np.random.default_rng(5)
    rows = set()
    for _ in range(200):
        b = int(rng.integers(len(lengths)))
        rows.add((b, int(rng.integers(w.Hq)), int(rng.integers(int(lengths[b])))))
    for b in (0, len(lengths) - 1):
        rows.add((b, 0, 0))
        rows.add((b, w.Hq - 1, int(lengths[b]) - 1))
    rows = np.array(sorted(rows), dtype=np.int32)
    check_rows(out, lse, q, k, v, rows, w.scale, True, cu=cu.numpy())
