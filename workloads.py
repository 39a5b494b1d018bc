"""Seeded synthetic inputs for grouped-query attention, and work accounting.

This module is shared by the tests, the benchmark and the smoke check.  It holds
no attention arithmetic: it only draws inputs and counts bytes and flops.

Recipe (the same for every workload):
* a ``torch.Generator`` on the target device, seeded with the workload's seed;
* q, k, v drawn in that order with ``randn`` in the logical [B, H, S, D] order of
  the Ultralytics GQA glossary example (``torch.manual_seed(0)`` then
  ``randn(1, 8, 16, 64)``, ``randn(1, 2, 16, 64)`` twice), in float32;
* cast to the workload dtype (bf16 rounds to nearest even);
* a "stress" variant multiplies q by 4 after the cast (exact in bf16);
* permuted to the library layout [B, S, H, D] (contiguous), as FlashAttention's
  ``flash_attn_func`` expects (StructBERT/FlashAttention page, section 2.2).

Variable-length batches draw their lengths with ``randint(lo, hi + 1, (n,))`` from
their own seed, then q, k, v for the packed [total, H, D] tensors.

Decode KV caches too large to draw on the host are drawn on the device, one
batch element at a time, each from its own seed ``seed * 1_000_003 + b``, so any
element can be redrawn alone.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    Hq: int
    Hkv: int
    Sq: int
    Sk: int
    D: int
    dtype: str          # "f32" or "bf16"
    causal: bool
    seed: int
    q_mult: float = 1.0  # 4.0 for the large-logit stress variant
    pack_gqa: int = 1
    num_splits: int = 1
    varlen: dict = field(default_factory=dict)  # {"n": 32, "lo": 128, "hi": 8192}
    page_size: int = 0  # > 0: decode against a paged KV cache of pages of this many keys
    kv_fp8: bool = False  # decode against an e4m3 KV cache (scale FP8_SCALE)
    qkv_fp8: bool = False  # prefill on e4m3 Q, K, V (scale FP8_PREFILL_SCALE each)
    block_sparse: dict = field(default_factory=dict)  # {"window": 3, "global": 2, "random": 3}
    backward: bool = False  # time the backward pass (dQ, dK, dV) of this forward
    window: int = 0  # > 0: causal attention within a sliding window of this many keys

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.D)

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    @property
    def torch_dtype(self):
        return torch.float32 if self.dtype == "f32" else torch.bfloat16


# The five workloads of the headline measurement; sizes as the pages' examples.
TINY = Workload("tiny_gqa_causal", B=1, Hq=8, Hkv=2, Sq=16, Sk=16, D=64, dtype="f32",
                causal=True, seed=0)
ENCODER = Workload("encoder_b64_h48kv12_s512_d64", B=64, Hq=48, Hkv=12, Sq=512, Sk=512,
                   D=64, dtype="bf16", causal=False, seed=1)
LLAMA = Workload("llama8b_prefill_b4_s8192_causal", B=4, Hq=32, Hkv=8, Sq=8192, Sk=8192,
                 D=128, dtype="bf16", causal=True, seed=2)
# the backward of the Llama prefill shape (and one batch element of it, for profiles)
LLAMA_BWD = Workload("llama8b_backward_b4_s8192_causal", B=4, Hq=32, Hkv=8, Sq=8192, Sk=8192,
                     D=128, dtype="bf16", causal=True, seed=2, backward=True)
LLAMA_BWD_B1 = Workload("llama8b_backward_b1_s8192_causal", B=1, Hq=32, Hkv=8, Sq=8192, Sk=8192,
                     D=128, dtype="bf16", causal=True, seed=2, backward=True)
# the Llama prefill's inputs as e4m3 codes (value / FP8_PREFILL_SCALE, rounded)
LLAMA_FP8 = Workload("llama8b_prefill_fp8_b4_s8192_causal", B=4, Hq=32, Hkv=8, Sq=8192,
                     Sk=8192, D=128, dtype="bf16", causal=True, seed=2, qkv_fp8=True)
FP8_PREFILL_SCALE = 1.0 / 16.0
# the Llama prefill shape with a 4096-key sliding window (Ultralytics GQA glossary, "GQA
# and related techniques": sliding-window attention, paired there with GQA in Mistral 7B)
LLAMA_WINDOW = Workload("llama8b_prefill_b4_s8192_window4096", B=4, Hq=32, Hkv=8, Sq=8192,
                        Sk=8192, D=128, dtype="bf16", causal=True, seed=2, window=4096)
LLAMA_STRESS = Workload("llama8b_prefill_b4_s8192_causal_qx4", B=4, Hq=32, Hkv=8, Sq=8192,
                        Sk=8192, D=128, dtype="bf16", causal=True, seed=3, q_mult=4.0)
DECODE_BATCHES = (1, 16, 64, 128, 256)
DECODE_SPLITS = (1, 2, 4, 8)


def decode(B: int, num_splits: int = 1, pack_gqa: int = 1) -> Workload:
    return Workload(f"decode_b{B}_sk32768_n{num_splits}_pack{pack_gqa}", B=B, Hq=32, Hkv=8,
                    Sq=1, Sk=32768, D=128, dtype="bf16", causal=False, seed=4,
                    pack_gqa=pack_gqa, num_splits=num_splits)


def decode_paged(B: int, page_size: int = 256) -> Workload:
    """The decode workload with its cache stored in shuffled pages (PagedAttention,
    Ultralytics GQA glossary, "GQA and related techniques")."""
    return Workload(f"decode_paged_b{B}_sk32768_p{page_size}", B=B, Hq=32, Hkv=8, Sq=1,
                    Sk=32768, D=128, dtype="bf16", causal=False, seed=4, pack_gqa=1,
                    num_splits=0, page_size=page_size)


FP8_SCALE = 1.0 / 32.0  # e4m3 cache: the bf16 values times 32, rounded to e4m3


def decode_fp8(B: int) -> Workload:
    """The decode workload with its cache in 8 bits (FP8 for decode bandwidth, GQA
    batch-size guide, hardware adaptation section)."""
    return Workload(f"decode_fp8_b{B}_sk32768", B=B, Hq=32, Hkv=8, Sq=1, Sk=32768, D=128,
                    dtype="bf16", causal=False, seed=4, pack_gqa=1, num_splits=0, kv_fp8=True)


BIGBIRD = Workload("bigbird_b4_s8192_blk128", B=4, Hq=32, Hkv=8, Sq=8192, Sk=8192, D=128,
                   dtype="bf16", causal=False, seed=6,
                   block_sparse={"window": 3, "global": 2, "random": 3})


def bigbird_pattern(w: Workload):
    """BigBird-style block pattern over 128-position blocks (Raptor-T abstract: several
    patterns combined): a window of `window` blocks around the diagonal, `global` blocks
    every row attends to and whose rows attend to everything, and `random` more blocks
    per row drawn from a seeded generator.  Returns CSR (row_ptr, col) int32 tensors."""
    blk = 128
    n_q, n_k = -(-w.Sq // blk), -(-w.Sk // blk)
    bs = w.block_sparse
    g = _gen("cpu", w.seed + 101)
    rows = []
    for r in range(n_q):
        if r < bs["global"]:
            rows.append(list(range(n_k)))
            continue
        cols = set(range(min(bs["global"], n_k)))
        half = bs["window"] // 2
        cols |= {c for c in range(r - half, r + half + 1) if 0 <= c < n_k}
        rnd = torch.randperm(n_k, generator=g)[: bs["random"]].tolist()
        cols |= set(rnd)
        rows.append(sorted(cols))
    row_ptr = torch.zeros(n_q + 1, dtype=torch.int32)
    row_ptr[1:] = torch.cumsum(torch.tensor([len(c) for c in rows]), 0)
    col = torch.tensor([c for cs in rows for c in cs], dtype=torch.int32)
    return row_ptr, col


def bigbird_pattern_varlen(lengths, block_sparse: dict, seed: int, blk: int = 128):
    """Per-sequence BigBird-style patterns for packed sequences with minimum padding:
    sequence b has ceil(n_b / blk) query and key blocks, its rows follow those of the
    earlier sequences, its col entries count its own key blocks.  The pattern of each
    sequence is built as in bigbird_pattern (window, global, seeded random blocks)."""
    g = _gen("cpu", seed)
    rows = []
    for n in [int(x) for x in lengths]:
        nb = -(-n // blk)
        for r in range(nb):
            if r < block_sparse["global"]:
                rows.append(list(range(nb)))
                continue
            cols = set(range(min(block_sparse["global"], nb)))
            half = block_sparse["window"] // 2
            cols |= {c for c in range(r - half, r + half + 1) if 0 <= c < nb}
            cols |= set(torch.randperm(nb, generator=g)[: block_sparse["random"]].tolist())
            rows.append(sorted(cols))
    row_ptr = torch.zeros(len(rows) + 1, dtype=torch.int32)
    if rows:
        row_ptr[1:] = torch.cumsum(torch.tensor([len(c) for c in rows]), 0)
    col = torch.tensor([c for cs in rows for c in cs], dtype=torch.int32)
    return row_ptr, col


def blocksparse_varlen_flops(lengths, row_ptr, col, Hq: int, D: int, blk: int = 128) -> int:
    """4*D flops per visible (query, key) pair per head over packed sequences."""
    rp, cl = row_ptr.tolist(), col.tolist()
    pairs, r = 0, 0
    for n in [int(x) for x in lengths]:
        for qb in range(-(-n // blk)):
            rows_in = min(blk, n - qb * blk)
            pairs += rows_in * sum(min(blk, n - c * blk) for c in cl[rp[r]:rp[r + 1]])
            r += 1
    return 4 * D * pairs * Hq


def blocksparse_flops(w: Workload, row_ptr, col) -> int:
    """4*D flops per visible (query, key) pair per head under the block pattern."""
    blk = 128
    pairs = 0
    rp = row_ptr.tolist()
    cl = col.tolist()
    for r in range(len(rp) - 1):
        rows_in = min(blk, w.Sq - r * blk)
        keys = sum(min(blk, w.Sk - c * blk) for c in cl[rp[r]:rp[r + 1]])
        pairs += rows_in * keys
    return 4 * w.D * pairs * w.B * w.Hq


VARLEN = Workload("varlen32_len128to8192_causal", B=32, Hq=32, Hkv=8, Sq=0, Sk=0, D=128,
                  dtype="bf16", causal=True, seed=5,
                  varlen={"n": 32, "lo": 128, "hi": 8192})
# the same 32 lengths (seed 5), non-causal, a BigBird-style pattern per sequence
BIGBIRD_VARLEN = Workload("bigbird_varlen32_len128to8192_blk128", B=32, Hq=32, Hkv=8, Sq=0,
                          Sk=0, D=128, dtype="bf16", causal=False, seed=5,
                          varlen={"n": 32, "lo": 128, "hi": 8192},
                          block_sparse={"window": 3, "global": 2, "random": 3})


def _gen(device, seed: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def make_qkv(w: Workload, device="cpu", *, B=None, Sq=None, Sk=None):
    """Dense q [B,Sq,Hq,D], k/v [B,Sk,Hkv,D] for workload w (shape overrides allowed)."""
    B = w.B if B is None else B
    Sq = w.Sq if Sq is None else Sq
    Sk = w.Sk if Sk is None else Sk
    g = _gen(device, w.seed)
    q = torch.randn(B, w.Hq, Sq, w.D, generator=g, device=device)
    k = torch.randn(B, w.Hkv, Sk, w.D, generator=g, device=device)
    v = torch.randn(B, w.Hkv, Sk, w.D, generator=g, device=device)
    q, k, v = (t.to(w.torch_dtype) for t in (q, k, v))
    if w.q_mult != 1.0:
        q = q * w.q_mult
    return tuple(t.transpose(1, 2).contiguous() for t in (q, k, v))


def make_qkv_e4m3(w: Workload, device="cpu", **kw):
    """make_qkv's values as e4m3 codes: value / FP8_PREFILL_SCALE rounded (nearest
    even) by torch's float8_e4m3fn cast."""
    q, k, v = make_qkv(w, device=device, **kw)
    return tuple((t.float() / FP8_PREFILL_SCALE).to(torch.float8_e4m3fn) for t in (q, k, v))


def make_dout(w: Workload, device="cpu"):
    """The output gradient dO [B, Sq, Hq, D] for the backward pass (seeded N(0, 1))."""
    g = _gen(device, w.seed + 500)
    d = torch.randn(w.B, w.Hq, w.Sq, w.D, generator=g, device=device).to(w.torch_dtype)
    return d.transpose(1, 2).contiguous()


def varlen_lengths(w: Workload, n=None, lo=None, hi=None) -> torch.Tensor:
    n = w.varlen["n"] if n is None else n
    lo = w.varlen["lo"] if lo is None else lo
    hi = w.varlen["hi"] if hi is None else hi
    g = _gen("cpu", w.seed)
    return torch.randint(lo, hi + 1, (n,), generator=g, dtype=torch.int64)


def cu_seqlens_of(lengths) -> torch.Tensor:
    lengths = torch.as_tensor(lengths, dtype=torch.int64)
    cu = torch.zeros(len(lengths) + 1, dtype=torch.int64)
    cu[1:] = torch.cumsum(lengths, 0)
    return cu.to(torch.int32)


def make_varlen(w: Workload, device="cpu", lengths=None):
    """Packed q [total,Hq,D], k/v [total,Hkv,D] and int32 cu_seqlens (host)."""
    if lengths is None:
        lengths = varlen_lengths(w)
    cu = cu_seqlens_of(lengths)
    total = int(cu[-1])
    g = _gen(device, w.seed + 1000)
    q = torch.randn(total, w.Hq, w.D, generator=g, device=device).to(w.torch_dtype)
    k = torch.randn(total, w.Hkv, w.D, generator=g, device=device).to(w.torch_dtype)
    v = torch.randn(total, w.Hkv, w.D, generator=g, device=device).to(w.torch_dtype)
    if w.q_mult != 1.0:
        q = q * w.q_mult
    return q, k, v, cu


def make_decode_q(w: Workload, device="cpu"):
    g = _gen(device, w.seed)
    q = torch.randn(w.B, w.Hq, 1, w.D, generator=g, device=device).to(w.torch_dtype)
    return q.transpose(1, 2).contiguous()


def make_decode_kv_one(w: Workload, b: int, device="cpu"):
    """K and V [Sk, Hkv, D] of batch element b, from its own seed."""
    g = _gen(device, w.seed * 1_000_003 + b)
    k = torch.randn(w.Hkv, w.Sk, w.D, generator=g, device=device).to(w.torch_dtype)
    v = torch.randn(w.Hkv, w.Sk, w.D, generator=g, device=device).to(w.torch_dtype)
    return k.transpose(0, 1).contiguous(), v.transpose(0, 1).contiguous()


def fill_decode_kv(w: Workload, k_out: torch.Tensor, v_out: torch.Tensor) -> None:
    """Fill preallocated k/v [B,Sk,Hkv,D] element by element (on their device).  An
    e4m3 (float8_e4m3fn) destination gets the values divided by FP8_SCALE, rounded."""
    for b in range(k_out.shape[0]):
        kb, vb = make_decode_kv_one(w, b, device=k_out.device)
        if k_out.dtype != kb.dtype:
            kb, vb = (t.float() / FP8_SCALE for t in (kb, vb))
        k_out[b].copy_(kb)
        v_out[b].copy_(vb)


def page_table(w: Workload) -> torch.Tensor:
    """Block table int32 [B, Sk / page_size]: a seeded shuffle of the page pool, so
    consecutive keys of a sequence sit in scattered pages."""
    per = w.Sk // w.page_size
    g = _gen("cpu", w.seed + 7)
    return torch.randperm(w.B * per, generator=g).to(torch.int32).reshape(w.B, per)


def make_paged_kv(w: Workload, table: torch.Tensor, device="cpu"):
    """Page pools k/v [B * Sk / page_size, page_size, Hkv, D] holding batch element
    b's cache (the same values as the dense decode workload) in pages table[b]."""
    per = w.Sk // w.page_size
    shape = (w.B * per, w.page_size, w.Hkv, w.D)
    kp = torch.empty(shape, dtype=w.torch_dtype, device=device)
    vp = torch.empty(shape, dtype=w.torch_dtype, device=device)
    idx = table.to(device=device, dtype=torch.int64)
    for b in range(w.B):
        kb, vb = make_decode_kv_one(w, b, device=device)
        kp[idx[b]] = kb.view(per, w.page_size, w.Hkv, w.D)
        vp[idx[b]] = vb.view(per, w.page_size, w.Hkv, w.D)
    return kp, vp


# ----------------------------------------------------------------------------------
# Work accounting (the benchmark's denominators)

def causal_pairs(Sq: int, Sk: int) -> int:
    """Number of visible (i, j) pairs under the bottom-right causal mask j <= i + Sk - Sq."""
    off = Sk - Sq
    return sum(min(max(i + off + 1, 0), Sk) for i in range(Sq))


def attention_flops(B: int, Hq: int, Sq: int, Sk: int, D: int, causal: bool,
                    window: int = 0) -> int:
    """4*D flops per visible (query, key) pair per head: 2*D for QK^T, 2*D for PV.  With a
    window, query i sees keys (i + Sk - Sq - window, i + Sk - Sq] that exist."""
    if window > 0:
        # row i: keys max(0, t - window + 1) .. t with t = i + Sk - Sq (none when t < 0)
        pairs = sum(max(0, min(i + Sk - Sq + 1, window)) for i in range(Sq))
    else:
        pairs = causal_pairs(Sq, Sk) if causal else Sq * Sk
    return 4 * D * pairs * B * Hq


def varlen_flops(lengths, Hq: int, D: int, causal: bool) -> int:
    return sum(attention_flops(1, Hq, int(L), int(L), D, causal) for L in lengths)


def kv_values_per_token(Hkv: int, D: int, layers: int = 1) -> int:
    """Cached key and value elements per token: 2 * Hkv * D per layer."""
    return 2 * Hkv * D * layers


def kv_cache_bytes(batch: int, seq: int, Hkv: int, D: int, bytes_per_elt: int = 2,
                   layers: int = 1) -> int:
    """KV memory = 2 x batch x seq x head_dim x kv_heads (x bytes x layers)."""
    return 2 * batch * seq * D * Hkv * bytes_per_elt * layers


def decode_bytes(B: int, Hq: int, Hkv: int, Sk: int, D: int, elt: int = 2,
                 kv_elt: int | None = None) -> int:
    """Algorithmic HBM bytes of one decode step: K and V once (kv_elt bytes each, default
    elt), q and O (elt), L (fp32)."""
    kv_elt = elt if kv_elt is None else kv_elt
    return kv_cache_bytes(B, Sk, Hkv, D, kv_elt) + 2 * B * Hq * D * elt + 4 * B * Hq


def prefill_min_bytes(B: int, Hq: int, Hkv: int, Sq: int, Sk: int, D: int, elt: int = 2):
    """q, k, v read once, O written once (elt bytes), L written (fp32)."""
    return elt * D * (2 * B * Sq * Hq + 2 * B * Sk * Hkv) + 4 * B * Hq * Sq
