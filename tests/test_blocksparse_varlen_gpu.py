"""GPU parity of block-sparse attention over packed sequences with minimum padding
(gqa_attn_fwd_blocksparse_varlen) against the float64 oracle on the same seeded inputs."""
import math

import numpy as np
import pytest
import torch

import oracle
import workloads as W
from exact_attention_gqa_b200 import build, gqa_attn_blocksparse_varlen, \
    gqa_attn_get_device_error
from parity import compare

pytestmark = pytest.mark.gpu

DEV = "cuda"
PATTERN = {"window": 3, "global": 1, "random": 2}


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    yield
    torch.cuda.synchronize()
    assert gqa_attn_get_device_error() == 0


def packed(lens, Hq, Hkv, D, seed):
    g = torch.Generator().manual_seed(seed)
    total = int(sum(lens))
    q = torch.randn(total, Hq, D, generator=g).bfloat16()
    k = torch.randn(total, Hkv, D, generator=g).bfloat16()
    v = torch.randn(total, Hkv, D, generator=g).bfloat16()
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lens)]), dtype=torch.int32)
    return q, k, v, cu


def run(q, k, v, cu, rp, cl, lens, balance=True):
    out, lse = gqa_attn_blocksparse_varlen(q.to(DEV), k.to(DEV), v.to(DEV), cu.to(DEV),
                                           rp.to(DEV), cl.to(DEV), max_seqlen=max(lens),
                                           balance=balance)
    torch.cuda.synchronize()
    return out, lse


@pytest.mark.parametrize("lens,Hq,Hkv,D", [
    ([300, 0, 128, 1000, 17, 513], 8, 2, 128),   # empty, one-block, ragged sequences
    ([129, 256, 700], 8, 4, 64),                  # G = 2
    ([1, 127, 128, 255, 400], 16, 2, 128),        # G = 8, the smallest sequences
])
def test_blocksparse_varlen_matches_oracle(lens, Hq, Hkv, D):
    q, k, v, cu = packed(lens, Hq, Hkv, D, seed=sum(lens) + D)
    rp, cl = W.bigbird_pattern_varlen(lens, PATTERN, seed=len(lens))
    out, lse = run(q, k, v, cu, rp, cl, lens)
    o_ref, l_ref = oracle.attention_blocksparse_varlen(q, k, v, cu, rp, cl,
                                                       scale=1 / math.sqrt(D))
    compare(out, lse, o_ref, l_ref)


def test_balanced_order_changes_nothing():
    lens = [1000, 60, 2048, 333]
    q, k, v, cu = packed(lens, 8, 2, 128, seed=5)
    rp, cl = W.bigbird_pattern_varlen(lens, PATTERN, seed=6)
    a = run(q, k, v, cu, rp, cl, lens, balance=True)
    b = run(q, k, v, cu, rp, cl, lens, balance=False)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


def test_full_size_varlen_bigbird_sampled():
    """The benchmark's shape: 32 sequences of 128..8192 positions, Hq=32, Hkv=8, D=128,
    the BigBird-style pattern per sequence; sampled rows checked against the oracle."""
    w = W.BIGBIRD_VARLEN
    lens = W.varlen_lengths(w).tolist()
    q, k, v, cu = W.make_varlen(w, lengths=lens)
    rp, cl = W.bigbird_pattern_varlen(lens, w.block_sparse, seed=w.seed + 101)
    out, lse = run(q, k, v, cu, rp, cl, lens)
    assert torch.isfinite(out.float()).all()
    # three sequences (shortest, middle, longest): every row and head against the oracle
    for b in (int(np.argmin(lens)), len(lens) // 2, int(np.argmax(lens))):
        sl = slice(int(cu[b]), int(cu[b + 1]))
        nb = -(-lens[b] // 128)
        r0 = int(sum(-(-n // 128) for n in lens[:b]))
        sub_rp = rp[r0:r0 + nb + 1] - rp[r0]
        sub_cl = cl[int(rp[r0]):int(rp[r0 + nb])]
        o_ref, l_ref = oracle.attention_blocksparse(q[sl][None], k[sl][None], v[sl][None],
                                                    sub_rp, sub_cl, scale=w.scale)
        compare(out[sl][None], lse[:, sl][None], o_ref, l_ref)


@pytest.mark.parametrize("lens,Hq,Hkv,D", [
    ([300, 0, 128, 1000, 17, 513], 8, 2, 128),
    ([129, 256, 700], 8, 4, 64),
])
def test_causal_blocksparse_varlen_matches_oracle(lens, Hq, Hkv, D):
    q, k, v, cu = packed(lens, Hq, Hkv, D, seed=sum(lens) + D + 1)
    rp, cl = W.bigbird_pattern_varlen(lens, PATTERN, seed=len(lens) + 1)
    out, lse = gqa_attn_blocksparse_varlen(q.to(DEV), k.to(DEV), v.to(DEV), cu.to(DEV),
                                           rp.to(DEV), cl.to(DEV), max_seqlen=max(lens),
                                           causal=True)
    torch.cuda.synchronize()
    o_ref, l_ref = oracle.attention_blocksparse_varlen(q, k, v, cu, rp, cl,
                                                       scale=1 / math.sqrt(D), causal=True)
    compare(out, lse, o_ref, l_ref)
