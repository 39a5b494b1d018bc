"""Pins of the float64 oracle against what the pages and the mathematics fix.

None of these tests reruns the oracle's own formula: each compares it with a
printed example of the pages, a library routine (torch's float64 SDPA, logsumexp),
a 50-digit brute force, a closed form or an invariant.  The last test plants
plausible mistakes in the oracle and checks that at least one pin catches each.
"""
import json
import math
import os

import mpmath
import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
import workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def rnd(shape, seed, scale=1.0):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(*shape, generator=g) * scale).numpy().astype(np.float32)


def bshd_to_bhsd64(a):
    return torch.from_numpy(np.ascontiguousarray(a)).double().transpose(1, 2)


def sdpa_ref(q, k, v, scale, causal, bottom_right=False):
    """torch float64 SDPA on [B,S,H,D] numpy inputs; returns O [B,S,H,D] and L [B,H,S]."""
    qt, kt, vt = bshd_to_bhsd64(q), bshd_to_bhsd64(k), bshd_to_bhsd64(v)
    G = qt.shape[1] // kt.shape[1]
    mask = None
    is_causal = causal
    if causal and bottom_right:
        Sq, Sk = qt.shape[2], kt.shape[2]
        mask = torch.ones(Sq, Sk, dtype=torch.bool).tril(diagonal=Sk - Sq)
        is_causal = False
    o = F.scaled_dot_product_attention(qt, kt, vt, attn_mask=mask, is_causal=is_causal,
                                       scale=scale, enable_gqa=True)
    kf = kt.repeat_interleave(G, dim=1)
    s = scale * qt @ kf.transpose(-1, -2)
    if causal:
        Sq, Sk = s.shape[-2:]
        vis = torch.ones(Sq, Sk, dtype=torch.bool)
        vis = vis.tril(diagonal=Sk - Sq) if bottom_right else vis.tril()
        s = s.masked_fill(~vis, float("-inf"))
    lse = torch.logsumexp(s, dim=-1)
    return o.transpose(1, 2).numpy(), lse.numpy()


# ---------------------------------------------------------------------------------
# The page's worked example

def test_glossary_example_gqa_equals_repeat_interleaved_mha():
    gold = json.load(open(os.path.join(GOLDEN, "gqa_glossary_example.json")))
    w = W.TINY
    assert [w.B, w.Hq, w.Sq, w.D] == gold["q_shape_bhsd"]
    assert [w.B, w.Hkv, w.Sk, w.D] == gold["kv_shape_bhsd"]
    q, k, v = W.make_qkv(w)
    # the recipe reproduces the page's draws: torch.manual_seed(0) then randn in order
    torch.manual_seed(gold["seed"])
    q_page = torch.randn(*gold["q_shape_bhsd"])
    k_page = torch.randn(*gold["kv_shape_bhsd"])
    assert torch.equal(q.transpose(1, 2), q_page)
    assert torch.equal(k.transpose(1, 2), k_page)
    scale = 1.0 / math.sqrt(64)
    o, lse = oracle.attention(q, k, v, scale=scale, causal=gold["causal"])
    assert list(o.transpose(0, 2, 1, 3).shape) == gold["printed_output_shape"]
    G = gold["group"]
    o_mha, lse_mha = oracle.attention(q, k.repeat_interleave(G, dim=2),
                                      v.repeat_interleave(G, dim=2), scale=scale,
                                      causal=gold["causal"])
    # same arithmetic on the same operands: identical, hence allclose(atol=1e-6) True
    assert np.array_equal(o, o_mha) and np.array_equal(lse, lse_mha)
    assert np.allclose(o, o_mha, atol=gold["printed_allclose_atol"]) == \
        gold["printed_same_as_copied_heads"]
    assert W.kv_values_per_token(w.Hkv, w.D) == \
        gold["printed_cached_values_per_token_per_layer_gqa"]
    assert W.kv_values_per_token(w.Hq, w.D) == \
        gold["printed_cached_values_per_token_per_layer_mha"]
    # and the page's own library call agrees with the oracle in float64
    o_ref, lse_ref = sdpa_ref(q.numpy(), k.numpy(), v.numpy(), scale, True)
    assert np.max(np.abs(o - o_ref)) < 1e-13
    assert np.max(np.abs(lse - lse_ref)) < 1e-13


def test_kv_cache_arithmetic_of_the_pages():
    gold = json.load(open(os.path.join(GOLDEN, "kv_cache_arithmetic.json")))
    ll = gold["llama31_8b"]
    per_tok = W.kv_cache_bytes(1, 1, ll["kv_heads"], ll["head_dim"], ll["bytes_per_value"],
                               ll["layers"])
    assert per_tok == ll["bytes_per_token_gqa"] == 128 * 1024
    assert W.kv_cache_bytes(1, 131072, ll["kv_heads"], ll["head_dim"], 2, ll["layers"]) == \
        ll["bytes_at_131072_tokens_gqa"] == 16 * 2**30
    assert W.kv_cache_bytes(1, 1, ll["q_heads"], ll["head_dim"], 2, ll["layers"]) == \
        ll["bytes_per_token_mha"]
    assert W.kv_cache_bytes(1, 131072, ll["q_heads"], ll["head_dim"], 2, ll["layers"]) == \
        ll["bytes_at_131072_tokens_mha"]
    g = gold["grouping_48_12"]
    red = 1 - W.kv_cache_bytes(1, 1, g["kv_heads"], 64) / W.kv_cache_bytes(1, 1, g["q_heads"], 64)
    assert round(100 * red) == g["reduction_percent"]


def test_flop_accounting_counts_visible_pairs():
    for Sq, Sk in [(1, 7), (5, 5), (4, 9), (9, 4), (16, 16)]:
        brute = sum(1 for i in range(Sq) for j in range(Sk) if j <= i + Sk - Sq)
        assert W.causal_pairs(Sq, Sk) == brute
    assert W.causal_pairs(8192, 8192) == 8192 * 8193 // 2
    assert W.attention_flops(2, 3, 5, 7, 8, False) == 4 * 8 * 5 * 7 * 2 * 3
    # sliding window: the pairs the oracle's window mask keeps, counted one by one
    for Sq, Sk, win in [(9, 9, 1), (9, 9, 4), (6, 11, 3), (11, 6, 2), (16, 16, 40)]:
        brute = int(band_mask(Sq, Sk, win).sum())
        assert W.attention_flops(1, 1, Sq, Sk, 1, True, window=win) == 4 * brute
    assert W.attention_flops(1, 1, 64, 64, 1, True, window=64) == \
        W.attention_flops(1, 1, 64, 64, 1, True)


# ---------------------------------------------------------------------------------
# Library routine: torch float64 scaled_dot_product_attention(enable_gqa=True)

@pytest.mark.parametrize("B,Hq,Hkv,Sq,Sk,D,causal", [
    (2, 8, 2, 33, 33, 16, True),
    (2, 8, 2, 33, 33, 16, False),
    (1, 6, 3, 17, 40, 8, False),
    (1, 4, 1, 12, 12, 32, True),     # MQA limit (one group)
    (1, 4, 4, 12, 12, 32, True),     # MHA limit (G = 1)
    (3, 12, 4, 20, 31, 24, True),    # Sq < Sk, bottom-right mask given explicitly
    (1, 4, 2, 25, 9, 8, True),       # Sq > Sk: leading rows see no key
])
def test_matches_torch_sdpa_float64(B, Hq, Hkv, Sq, Sk, D, causal):
    q = rnd((B, Sq, Hq, D), 11)
    k = rnd((B, Sk, Hkv, D), 12)
    v = rnd((B, Sk, Hkv, D), 13)
    scale = 0.37
    o, lse = oracle.attention(q, k, v, scale=scale, causal=causal)
    bottom_right = causal and Sq != Sk
    o_ref, lse_ref = sdpa_ref(q, k, v, scale, causal, bottom_right=bottom_right)
    if causal and Sq > Sk:
        dead = Sq - Sk  # rows with no visible key: O = 0, L = -inf (SDPA gives NaN)
        assert np.all(o[:, :dead] == 0) and np.all(np.isneginf(lse[:, :, :dead]))
        o, o_ref = o[:, dead:], o_ref[:, dead:]
        lse, lse_ref = lse[:, :, dead:], lse_ref[:, :, dead:]
    assert np.max(np.abs(o - o_ref)) < 1e-12
    assert np.max(np.abs(lse - lse_ref)) < 1e-12


def test_decode_row_sees_every_key():
    """Sq = 1 under the bottom-right causal reading equals the unmasked result."""
    q = rnd((3, 1, 8, 16), 21)
    k = rnd((3, 50, 2, 16), 22)
    v = rnd((3, 50, 2, 16), 23)
    a = oracle.attention(q, k, v, scale=0.25, causal=True)
    b = oracle.attention(q, k, v, scale=0.25, causal=False)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])
    o_ref, lse_ref = sdpa_ref(q, k, v, 0.25, False)
    assert np.max(np.abs(a[0] - o_ref)) < 1e-12


# ---------------------------------------------------------------------------------
# Softmax properties, read through V = identity (then O = P)

@pytest.mark.parametrize("causal,Sq,Sk", [(False, 9, 9), (True, 9, 9), (True, 5, 11)])
def test_probabilities_are_a_distribution(causal, Sq, Sk):
    Hq, Hkv = 4, 2
    q = rnd((1, Sq, Hq, Sk), 31, 2.0)
    k = rnd((1, Sk, Hkv, Sk), 32, 2.0)
    eye = np.broadcast_to(np.eye(Sk, dtype=np.float32)[:, None, :], (Sk, Hkv, Sk))
    v = np.ascontiguousarray(eye[None])
    P, _ = oracle.attention(q, k, v, scale=0.5, causal=causal)  # [1, Sq, Hq, Sk] == P
    assert np.all(P >= 0)
    assert np.max(np.abs(P.sum(-1) - 1.0)) < 1e-12
    if causal:
        for i in range(Sq):
            hidden = np.arange(Sk) > i + Sk - Sq
            assert np.all(P[0, i, :, hidden] == 0.0)
            assert np.all(P[0, i, :, ~hidden] > 0.0)


# ---------------------------------------------------------------------------------
# Exact values: 50-digit brute force of the definition on tiny problems

def brute_force(q, k, v, scale, causal):
    mpmath.mp.dps = 50
    B, Sq, Hq, D = q.shape
    _, Sk, Hkv, _ = k.shape
    G = Hq // Hkv
    O = np.zeros(q.shape)
    L = np.zeros((B, Hq, Sq))
    for b in range(B):
        for h in range(Hq):
            c = h // G
            for i in range(Sq):
                vis = [j for j in range(Sk) if not causal or j <= i + Sk - Sq]
                s = [mpmath.mpf(scale) * mpmath.fsum(mpmath.mpf(float(q[b, i, h, d])) *
                                                     mpmath.mpf(float(k[b, j, c, d]))
                                                     for d in range(D)) for j in vis]
                e = [mpmath.exp(x) for x in s]
                z = mpmath.fsum(e)
                for d in range(D):
                    O[b, i, h, d] = float(mpmath.fsum(e[t] * mpmath.mpf(float(v[b, j, c, d]))
                                                      for t, j in enumerate(vis)) / z)
                L[b, h, i] = float(mpmath.log(z))
    return O, L


@pytest.mark.parametrize("causal,Sq,Sk", [(True, 4, 4), (False, 3, 5), (True, 2, 6)])
def test_brute_force_50_digits(causal, Sq, Sk):
    q = rnd((2, Sq, 4, 3), 41, 3.0)  # large logits: exercises the max shift
    k = rnd((2, Sk, 2, 3), 42, 3.0)
    v = rnd((2, Sk, 2, 3), 43)
    o, lse = oracle.attention(q, k, v, scale=1.3, causal=causal)
    o_bf, lse_bf = brute_force(q, k, v, 1.3, causal)
    assert np.max(np.abs(o - o_bf)) < 1e-13
    assert np.max(np.abs(lse - lse_bf)) < 1e-13


# ---------------------------------------------------------------------------------
# Closed forms

def test_single_key_returns_its_value():
    q = rnd((2, 3, 4, 8), 51)
    k = rnd((2, 1, 2, 8), 52)
    v = rnd((2, 1, 2, 8), 53)
    o, lse = oracle.attention(q, k, v, scale=0.7, causal=False)
    for h in range(4):
        np.testing.assert_array_equal(o[:, :, h, :], np.broadcast_to(v[:, 0:1, h // 2, :], (2, 3, 8)))
        expect = 0.7 * np.einsum("bid,bd->bi", q[:, :, h, :].astype(np.float64),
                                 k[:, 0, h // 2, :].astype(np.float64))
        assert np.max(np.abs(lse[:, h, :] - expect)) < 1e-12


def test_equal_keys_average_the_visible_values():
    Sq = Sk = 7
    q = rnd((1, Sq, 2, 5), 61)
    k1 = rnd((1, 1, 1, 5), 62)
    k = np.ascontiguousarray(np.repeat(k1, Sk, axis=1))
    v = rnd((1, Sk, 1, 5), 63)
    o, lse = oracle.attention(q, k, v, scale=0.9, causal=True)
    for i in range(Sq):
        mean = v[0, : i + 1, 0, :].astype(np.float64).mean(0)
        for h in range(2):
            assert np.max(np.abs(o[0, i, h] - mean)) < 1e-13
            s0 = 0.9 * float(np.dot(q[0, i, h].astype(np.float64), k1[0, 0, 0].astype(np.float64)))
            assert abs(lse[0, h, i] - (s0 + math.log(i + 1))) < 1e-12


def test_zero_query_gives_uniform_average_and_log_count():
    q = np.zeros((1, 6, 2, 4), np.float32)
    k = rnd((1, 6, 1, 4), 71)
    v = rnd((1, 6, 1, 4), 72)
    o, lse = oracle.attention(q, k, v, scale=0.5, causal=True)
    for i in range(6):
        assert np.max(np.abs(o[0, i, 0] - v[0, : i + 1, 0].astype(np.float64).mean(0))) < 1e-14
        assert abs(lse[0, 0, i] - math.log(i + 1)) < 1e-14
    # causal row 0 attends to key 0 only
    np.testing.assert_array_equal(o[0, 0, 1], v[0, 0, 0].astype(np.float64))


# ---------------------------------------------------------------------------------
# Invariants

def test_key_permutation_invariance_when_unmasked():
    q = rnd((2, 5, 4, 8), 81)
    k = rnd((2, 13, 2, 8), 82)
    v = rnd((2, 13, 2, 8), 83)
    perm = np.random.default_rng(0).permutation(13)
    a = oracle.attention(q, k, v, scale=0.3, causal=False)
    b = oracle.attention(q, np.ascontiguousarray(k[:, perm]), np.ascontiguousarray(v[:, perm]),
                         scale=0.3, causal=False)
    assert np.max(np.abs(a[0] - b[0])) < 1e-13 and np.max(np.abs(a[1] - b[1])) < 1e-13


def test_key_shift_leaves_probabilities_and_shifts_lse():
    """k_j -> k_j + u adds scale*q_i.u to every logit of row i."""
    # dyadic values with few bits, so that k + u is exact in float32
    q = np.round(rnd((1, 6, 2, 4), 91) * 8) / 8
    k = np.round(rnd((1, 6, 1, 4), 92) * 8) / 8
    v = rnd((1, 6, 1, 4), 93)
    u = np.array([0.5, -0.25, 1.0, 0.125], np.float32)
    a = oracle.attention(q, k, v, scale=0.5, causal=True)
    b = oracle.attention(q, np.ascontiguousarray(k + u), v, scale=0.5, causal=True)
    assert np.max(np.abs(a[0] - b[0])) < 1e-12
    shift = 0.5 * np.einsum("ihd,d->hi", q[0].astype(np.float64), u.astype(np.float64))
    assert np.max(np.abs(b[1][0] - a[1][0] - shift)) < 1e-12


def test_value_linearity_and_scale_folding():
    q = rnd((1, 7, 4, 8), 101)
    k = rnd((1, 9, 2, 8), 102)
    v1 = rnd((1, 9, 2, 8), 103)
    v2 = rnd((1, 9, 2, 8), 104)
    o1, _ = oracle.attention(q, k, v1, scale=0.4, causal=True)
    o2, _ = oracle.attention(q, k, v2, scale=0.4, causal=True)
    o12, _ = oracle.attention(q, k, np.ascontiguousarray(v1.astype(np.float64) + v2).astype(np.float32),
                              scale=0.4, causal=True)
    assert np.max(np.abs(o12 - (o1 + o2))) < 1e-6  # v1 + v2 rounds to float32
    a = oracle.attention(q, k, v1, scale=0.5, causal=True)
    b = oracle.attention(np.ascontiguousarray(q * 2), k, v1, scale=0.25, causal=True)
    assert np.max(np.abs(a[0] - b[0])) < 1e-13 and np.max(np.abs(a[1] - b[1])) < 1e-13


def test_varlen_equals_per_sequence_problems():
    lengths = [5, 1, 12, 7]
    cu = W.cu_seqlens_of(lengths).numpy()
    total = int(cu[-1])
    q = rnd((total, 8, 16), 111)
    k = rnd((total, 2, 16), 112)
    v = rnd((total, 2, 16), 113)
    o, lse = oracle.attention(q, k, v, scale=0.25, causal=True, cu_seqlens=cu)
    assert lse.shape == (8, total)
    for b, L in enumerate(lengths):
        s0 = cu[b]
        ob, lb = oracle.attention(q[None, s0:s0 + L], k[None, s0:s0 + L], v[None, s0:s0 + L],
                                  scale=0.25, causal=True)
        np.testing.assert_array_equal(o[s0:s0 + L], ob[0])
        np.testing.assert_array_equal(lse[:, s0:s0 + L], lb[0])


def test_rows_entry_point_matches_full():
    q = rnd((2, 10, 8, 16), 121)
    k = rnd((2, 14, 2, 16), 122)
    v = rnd((2, 14, 2, 16), 123)
    o, lse = oracle.attention(q, k, v, scale=0.25, causal=True)
    rows = np.array([[0, 0, 0], [1, 7, 9], [0, 3, 4], [1, 2, 0]])
    orow, lrow = oracle.attention_rows(q, k, v, rows, scale=0.25, causal=True)
    for r, (b, h, i) in enumerate(rows):
        np.testing.assert_array_equal(orow[r], o[b, i, h])
        assert lrow[r] == lse[b, h, i]


# ---------------------------------------------------------------------------------
# Online softmax: "exactly identical, no approximation"

@pytest.mark.parametrize("Bm,Bn", [(1, 1), (3, 3), (16, 64), (64, 16), (7, 5)])
@pytest.mark.parametrize("form", [1, 2])
@pytest.mark.parametrize("causal,Sq,Sk", [(True, 37, 37), (False, 20, 45), (True, 9, 40)])
def test_tiled_forms_equal_full_matrix(Bm, Bn, form, causal, Sq, Sk):
    q = rnd((1, Sq, 4, 8), 131, 3.0)  # large logits so the running max moves
    k = rnd((1, Sk, 2, 8), 132, 3.0)
    v = rnd((1, Sk, 2, 8), 133)
    full = oracle.attention(q, k, v, scale=0.5, causal=causal)
    tiled = oracle.attention_tiled(q, k, v, scale=0.5, causal=causal, Bm=Bm, Bn=Bn, form=form)
    assert np.max(np.abs(full[0] - tiled[0])) < 1e-12
    assert np.max(np.abs(full[1] - tiled[1])) < 1e-12


# ---------------------------------------------------------------------------------
# Split-KV: contiguous ranges of whole key blocks, log-sum-exp combine

def split_ranges(Sk, n, Bn):
    nblk = -(-Sk // Bn)
    n = min(n, nblk)
    per = -(-nblk // n)
    return [(min(s * per * Bn, Sk), min((s + 1) * per * Bn, Sk)) for s in range(n)]


@pytest.mark.parametrize("n", [1, 2, 4, 8, 1000])
@pytest.mark.parametrize("causal,Sq,Sk", [(False, 1, 300), (True, 1, 300), (True, 24, 24)])
def test_split_combine_equals_full(n, causal, Sq, Sk):
    q = rnd((2, Sq, 4, 8), 141, 2.0)
    k = rnd((2, Sk, 2, 8), 142, 2.0)
    v = rnd((2, Sk, 2, 8), 143)
    Bn = 16
    o, lse = oracle.attention(q, k, v, scale=0.5, causal=causal)
    parts = [oracle.attention_keyrange(q, k, v, a, b, scale=0.5, causal=causal)
             for a, b in split_ranges(Sk, n, Bn)]
    for bb in range(2):
        for h in range(4):
            for i in range(Sq):
                Os = np.stack([p[0][bb, i, h] for p in parts])
                Ls = np.array([p[1][bb, h, i] for p in parts])
                O, L = oracle.combine(Os, Ls)
                assert np.max(np.abs(O - o[bb, i, h])) < 1e-12
                assert abs(L - lse[bb, h, i]) < 1e-12


def test_combine_of_empty_partials():
    O, L = oracle.combine(np.zeros((3, 4)), np.full(3, -np.inf))
    assert np.all(O == 0) and L == -np.inf
    O, L = oracle.combine(np.array([[1.0, 2.0], [9.0, 9.0]]), np.array([0.5, -np.inf]))
    np.testing.assert_array_equal(O, [1.0, 2.0])
    assert L == 0.5


# ---------------------------------------------------------------------------------
# KV-cache decode: per-sequence lengths, paged storage, sliding window (Ultralytics
# GQA glossary, "How GQA shrinks the KV cache" and "GQA and related techniques")

def scatter_to_pages(k, v, page_size, seed, spare=3):
    """Dense caches [B, Sk, Hkv, D] -> a shuffled pool of pages and its block table.
    Rows no sequence owns hold unrelated values, so a wrong row shows."""
    B, Sk, Hkv, D = k.shape
    max_pages = -(-Sk // page_size)
    num_pages = B * max_pages + spare
    rng = np.random.default_rng(seed)
    table = rng.permutation(num_pages)[: B * max_pages].reshape(B, max_pages).astype(np.int32)
    kp = rnd((num_pages, page_size, Hkv, D), seed + 1, 3.0)
    vp = rnd((num_pages, page_size, Hkv, D), seed + 2, 3.0)
    for b in range(B):
        for pg in range(max_pages):
            j0, j1 = pg * page_size, min((pg + 1) * page_size, Sk)
            kp[table[b, pg], : j1 - j0] = k[b, j0:j1]
            vp[table[b, pg], : j1 - j0] = v[b, j0:j1]
    return kp, vp, table


def kv_sdpa(q, k, v, lens, window, scale):
    """torch float64 SDPA over each sequence's visible keys, cut from the dense cache."""
    B, _, Hq, D = q.shape
    O = np.zeros((B, Hq, D))
    L = np.zeros((B, Hq))
    for b in range(B):
        j1 = int(lens[b])
        j0 = max(0, j1 - window) if window > 0 else 0
        if j1 <= j0:
            L[b] = -np.inf
            continue
        o, l = sdpa_ref(q[b:b + 1], k[b:b + 1, j0:j1], v[b:b + 1, j0:j1], scale, False)
        O[b] = o[0, 0]
        L[b] = l[0, :, 0]
    return O, L


def assert_kv_close(O, L, Or, Lr):
    np.testing.assert_allclose(O, Or, rtol=0, atol=1e-12)
    assert np.array_equal(np.isneginf(L), np.isneginf(Lr))
    fin = np.isfinite(Lr)
    np.testing.assert_allclose(L[fin], Lr[fin], rtol=0, atol=1e-12)


@pytest.mark.parametrize("window", [0, 1, 7, 64, 1000])
def test_kvcache_lengths_and_window_match_sdpa_on_slices(window):
    B, Hq, Hkv, Sk, D = 5, 8, 2, 90, 32
    q, k, v = rnd((B, 1, Hq, D), 40), rnd((B, Sk, Hkv, D), 41), rnd((B, Sk, Hkv, D), 42)
    lens = np.array([0, 1, 37, 89, 90], dtype=np.int32)
    O, L = oracle.decode_kvcache(q, k, v, scale=0.2, seqlens_k=lens, window=window)
    assert_kv_close(O, L, *kv_sdpa(q, k, v, lens, window, 0.2))


def test_kvcache_without_lengths_reads_the_whole_cache():
    B, Hq, Hkv, Sk, D = 2, 6, 3, 21, 8
    q, k, v = rnd((B, 1, Hq, D), 50), rnd((B, Sk, Hkv, D), 51), rnd((B, Sk, Hkv, D), 52)
    O, L = oracle.decode_kvcache(q, k, v, scale=0.3)
    assert_kv_close(O, L, *kv_sdpa(q, k, v, np.full(B, Sk), 0, 0.3))


@pytest.mark.parametrize("page_size,window", [(1, 0), (3, 5), (16, 0), (16, 20), (64, 0)])
def test_kvcache_paged_matches_sdpa(page_size, window):
    B, Hq, Hkv, Sk, D = 4, 8, 4, 75, 16
    q, k, v = rnd((B, 1, Hq, D), 60), rnd((B, Sk, Hkv, D), 61), rnd((B, Sk, Hkv, D), 62)
    lens = np.array([75, 0, 17, 64], dtype=np.int32)
    kp, vp, table = scatter_to_pages(k, v, page_size, 63)
    O, L = oracle.decode_kvcache(q, kp, vp, scale=0.25, seqlens_k=lens, block_table=table,
                                 window=window)
    assert_kv_close(O, L, *kv_sdpa(q, k, v, lens, window, 0.25))


def test_kvcache_window_of_one_returns_the_newest_value():
    # a single visible key: its value comes out unchanged and L is its logit
    B, Hq, Hkv, Sk, D = 3, 4, 2, 12, 8
    q, k, v = rnd((B, 1, Hq, D), 70), rnd((B, Sk, Hkv, D), 71), rnd((B, Sk, Hkv, D), 72)
    lens = np.array([12, 5, 1], dtype=np.int32)
    O, L = oracle.decode_kvcache(q, k, v, scale=0.5, seqlens_k=lens, window=1)
    for b in range(B):
        for h in range(Hq):
            c = h // (Hq // Hkv)
            j = lens[b] - 1
            np.testing.assert_array_equal(O[b, h], v[b, j, c].astype(np.float64))
            expect = 0.5 * float(np.dot(q[b, 0, h].astype(np.float64), k[b, j, c].astype(np.float64)))
            assert abs(L[b, h] - expect) < 1e-12


def test_kvcache_rejects_bad_lengths_and_pages():
    q, k, v = rnd((1, 1, 2, 4), 80), rnd((1, 8, 1, 4), 81), rnd((1, 8, 1, 4), 82)
    with pytest.raises(ValueError):
        oracle.decode_kvcache(q, k, v, scale=1.0, seqlens_k=np.array([9], np.int32))
    with pytest.raises(ValueError):
        # 12 keys in pages of 8 use both table entries; page 5 is not in the pool of 1
        oracle.decode_kvcache(q, k, v, scale=1.0, seqlens_k=np.array([12], np.int32),
                              block_table=np.array([[0, 5]], np.int32))


def test_e4m3_table_matches_torch_float8():
    # every code: torch's float8_e4m3fn decoding (a library routine) is the reference
    t = oracle.e4m3_table()
    ref = torch.arange(256, dtype=torch.int32).to(torch.uint8).view(torch.float8_e4m3fn)
    ref = ref.double().numpy()
    assert np.array_equal(np.isnan(t), np.isnan(ref))
    np.testing.assert_array_equal(t[~np.isnan(t)], ref[~np.isnan(ref)])
    assert t[0x7E] == 448.0 and t[0x01] == 2.0 ** -9 and t[0x38] == 1.0


def e4m3_codes(shape, seed, spread=1.0):
    """Random finite e4m3 codes (torch rounds normal draws to the format)."""
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(*shape, generator=g) * spread
    return x.to(torch.float8_e4m3fn).view(torch.uint8)


def decoded(codes, scale):
    return codes.view(torch.float8_e4m3fn).double().numpy() * scale


@pytest.mark.parametrize("window", [0, 9])
def test_kvcache_e4m3_matches_sdpa_on_decoded_values(window):
    B, Hq, Hkv, Sk, D = 3, 8, 2, 70, 16
    q = rnd((B, 1, Hq, D), 90)
    k8, v8 = e4m3_codes((B, Sk, Hkv, D), 91, 40.0), e4m3_codes((B, Sk, Hkv, D), 92, 40.0)
    ks, vs = 0.03125, 0.0217
    lens = np.array([70, 33, 0], dtype=np.int32)
    O, L = oracle.decode_kvcache(q, k8, v8, scale=0.25, seqlens_k=lens, window=window,
                                 k_scale=ks, v_scale=vs)
    assert_kv_close(O, L, *kv_sdpa(q, decoded(k8, ks), decoded(v8, vs), lens, window, 0.25))


def test_kvcache_e4m3_paged_matches_sdpa():
    B, Hq, Hkv, Sk, D = 2, 4, 1, 48, 8
    q = rnd((B, 1, Hq, D), 93)
    k8, v8 = e4m3_codes((B, Sk, Hkv, D), 94, 8.0), e4m3_codes((B, Sk, Hkv, D), 95, 8.0)
    lens = np.array([48, 20], dtype=np.int32)
    kp, vp, table = scatter_to_pages(k8.numpy().astype(np.float32),
                                     v8.numpy().astype(np.float32), 16, 96)
    # owned rows hold the codes exactly; the noise in unowned rows becomes small codes
    kp = np.ascontiguousarray(np.clip(np.abs(kp), 0, 255)).astype(np.uint8)
    vp = np.ascontiguousarray(np.clip(np.abs(vp), 0, 255)).astype(np.uint8)
    O, L = oracle.decode_kvcache(q, kp, vp, scale=0.5, seqlens_k=lens, block_table=table,
                                 k_scale=0.1, v_scale=0.2)
    assert_kv_close(O, L, *kv_sdpa(q, decoded(k8, 0.1), decoded(v8, 0.2), lens, 0, 0.5))


# ---------------------------------------------------------------------------------
# Block-sparse attention (Raptor-T abstract: BigBird's block pattern)

# ---------------------------------------------------------------------------------
# Prefill sliding window (causal): query i sees keys (i + Sk - Sq - W, i + Sk - Sq]

def band_mask(Sq, Sk, window):
    i = np.arange(Sq)[:, None] + (Sk - Sq)
    j = np.arange(Sk)[None, :]
    return (j <= i) & (j > i - window)


@pytest.mark.parametrize("Sq,Sk,window", [(40, 40, 1), (40, 40, 7), (33, 70, 16), (50, 20, 5),
                                          (25, 25, 25), (25, 25, 400)])
def test_window_prefill_matches_sdpa_with_the_band_mask(Sq, Sk, window):
    B, Hq, Hkv, D = 2, 6, 2, 16
    q, k, v = rnd((B, Sq, Hq, D), 300 + Sq, 2.0), rnd((B, Sk, Hkv, D), 301 + Sk, 2.0), \
        rnd((B, Sk, Hkv, D), 302)
    O, L = oracle.attention(q, k, v, scale=0.3, causal=True, window=window)
    Or, Lr = masked_sdpa(q, k, v, 0.3, band_mask(Sq, Sk, window))
    np.testing.assert_allclose(O, Or, rtol=0, atol=1e-12)
    assert np.array_equal(np.isneginf(L), np.isneginf(Lr))
    fin = np.isfinite(Lr)
    np.testing.assert_allclose(L[fin], Lr[fin], rtol=0, atol=1e-12)


def test_window_of_one_returns_the_diagonal_value():
    # one visible key per row: its value unchanged, L its logit (closed form)
    B, Hq, Hkv, Sq, Sk, D = 2, 4, 2, 9, 13, 8
    q, k, v = rnd((B, Sq, Hq, D), 310), rnd((B, Sk, Hkv, D), 311), rnd((B, Sk, Hkv, D), 312)
    O, L = oracle.attention(q, k, v, scale=0.7, causal=True, window=1)
    for b in range(B):
        for h in range(Hq):
            c = h // (Hq // Hkv)
            for i in range(Sq):
                j = i + Sk - Sq
                np.testing.assert_array_equal(O[b, i, h], v[b, j, c].astype(np.float64))
                expect = 0.7 * float(np.dot(q[b, i, h].astype(np.float64),
                                            k[b, j, c].astype(np.float64)))
                assert abs(L[b, h, i] - expect) < 1e-12


def test_window_covering_every_key_is_causal_attention():
    B, Hq, Hkv, Sq, Sk, D = 2, 8, 2, 30, 45, 16
    q, k, v = rnd((B, Sq, Hq, D), 320), rnd((B, Sk, Hkv, D), 321), rnd((B, Sk, Hkv, D), 322)
    O, L = oracle.attention(q, k, v, scale=0.25, causal=True, window=Sk)
    Or, Lr = sdpa_ref(q, k, v, 0.25, True, bottom_right=True)
    np.testing.assert_allclose(O, Or, rtol=0, atol=1e-12)
    np.testing.assert_allclose(L, Lr, rtol=0, atol=1e-12)


@pytest.mark.parametrize("window", [1, 6, 31])
def test_window_last_row_equals_the_decode_window(window):
    # the newest query of a windowed prefill (Sq = Sk) is the decode step with that window
    B, Hq, Hkv, S, D = 3, 8, 4, 31, 16
    q, k, v = rnd((B, S, Hq, D), 330), rnd((B, S, Hkv, D), 331), rnd((B, S, Hkv, D), 332)
    O, L = oracle.attention(q, k, v, scale=0.4, causal=True, window=window)
    Od, Ld = oracle.decode_kvcache(np.ascontiguousarray(q[:, -1:]), k, v, scale=0.4,
                                   window=window)
    np.testing.assert_allclose(O[:, -1], Od, rtol=0, atol=1e-13)
    np.testing.assert_allclose(L[:, :, -1], Ld, rtol=0, atol=1e-13)


def brute_force_window(q, k, v, scale, window):
    mpmath.mp.dps = 50
    B, Sq, Hq, D = q.shape
    _, Sk, Hkv, _ = k.shape
    O = np.zeros(q.shape)
    L = np.zeros((B, Hq, Sq))
    for b in range(B):
        for h in range(Hq):
            c = h // (Hq // Hkv)
            for i in range(Sq):
                top = i + Sk - Sq
                vis = [j for j in range(Sk) if top - window < j <= top]
                if not vis:
                    L[b, h, i] = -np.inf
                    continue
                e = [mpmath.exp(mpmath.mpf(scale) * mpmath.fsum(
                    mpmath.mpf(float(q[b, i, h, d])) * mpmath.mpf(float(k[b, j, c, d]))
                    for d in range(D))) for j in vis]
                z = mpmath.fsum(e)
                for d in range(D):
                    O[b, i, h, d] = float(mpmath.fsum(e[t] * mpmath.mpf(float(v[b, j, c, d]))
                                                      for t, j in enumerate(vis)) / z)
                L[b, h, i] = float(mpmath.log(z))
    return O, L


def test_window_brute_force_50_digits():
    q, k, v = rnd((1, 6, 4, 3), 340, 3.0), rnd((1, 8, 2, 3), 341, 3.0), rnd((1, 8, 2, 3), 342)
    O, L = oracle.attention(q, k, v, scale=1.1, causal=True, window=3)
    Ob, Lb = brute_force_window(q, k, v, 1.1, 3)
    assert np.max(np.abs(O - Ob)) < 1e-13
    assert np.max(np.abs(L - Lb)) < 1e-13


def test_window_varlen_and_rows_agree_with_the_dense_form():
    lens = [9, 0, 23, 1, 40]
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    total, Hq, Hkv, D = int(cu[-1]), 4, 2, 8
    q, k, v = rnd((total, Hq, D), 350), rnd((total, Hkv, D), 351), rnd((total, Hkv, D), 352)
    O, L = oracle.attention(q, k, v, scale=0.5, causal=True, cu_seqlens=cu, window=6)
    for b, n in enumerate(lens):
        if n == 0:
            continue
        sl = slice(int(cu[b]), int(cu[b + 1]))
        Ob, Lb = oracle.attention(q[sl][None], k[sl][None], v[sl][None], scale=0.5,
                                  causal=True, window=6)
        np.testing.assert_array_equal(O[sl], Ob[0])
        np.testing.assert_array_equal(L[:, sl], Lb[0])
    rows = np.array([[2, 1, 22], [4, 3, 0], [0, 0, 8], [4, 2, 39]], dtype=np.int32)
    Or, Lr = oracle.attention_rows(q, k, v, rows, scale=0.5, causal=True, cu_seqlens=cu,
                                   window=6)
    for r, (b, h, i) in enumerate(rows):
        np.testing.assert_array_equal(Or[r], O[cu[b] + i, h])
        assert Lr[r] == L[h, cu[b] + i]


def test_window_needs_causal():
    q, k, v = rnd((1, 4, 2, 8), 360), rnd((1, 4, 1, 8), 361), rnd((1, 4, 1, 8), 362)
    with pytest.raises(ValueError):
        oracle.attention(q, k, v, scale=0.5, causal=False, window=2)


def random_pattern(n_q, n_k, seed, density=0.35, empty_rows=()):
    rng = np.random.default_rng(seed)
    rows = []
    for r in range(n_q):
        cols = [] if r in empty_rows else sorted(set(
            np.flatnonzero(rng.random(n_k) < density).tolist()) | {min(r, n_k - 1)})
        rows.append(cols)
    row_ptr = np.zeros(n_q + 1, dtype=np.int32)
    row_ptr[1:] = np.cumsum([len(c) for c in rows])
    col = np.array([c for cols in rows for c in cols], dtype=np.int32)
    return row_ptr, col


def expand_pattern(row_ptr, col, Sq, Sk, blk):
    mask = np.zeros((Sq, Sk), dtype=bool)
    for r in range(len(row_ptr) - 1):
        for c in col[row_ptr[r]:row_ptr[r + 1]]:
            mask[r * blk:(r + 1) * blk, c * blk:(c + 1) * blk] = True
    return mask


def masked_sdpa(q, k, v, scale, mask):
    """torch float64 SDPA with a boolean element mask, and logsumexp; rows without a
    visible key are O = 0, L = -inf."""
    qt, kt, vt = bshd_to_bhsd64(q), bshd_to_bhsd64(k), bshd_to_bhsd64(v)
    G = qt.shape[1] // kt.shape[1]
    kf, vf = kt.repeat_interleave(G, dim=1), vt.repeat_interleave(G, dim=1)
    m = torch.from_numpy(mask)
    s = (scale * qt @ kf.transpose(-1, -2)).masked_fill(~m, float("-inf"))
    lse = torch.logsumexp(s, dim=-1)
    dead = ~m.any(dim=-1)
    live = torch.from_numpy(np.where(mask.any(axis=1))[0])
    o = torch.zeros_like(qt)
    if live.numel():
        o[:, :, live] = F.scaled_dot_product_attention(qt[:, :, live], kf, vf,
                                                       attn_mask=m[live], scale=scale)
    lse[..., dead] = float("-inf")
    return o.transpose(1, 2).numpy(), lse.numpy()


@pytest.mark.parametrize("Sq,Sk,blk,seed", [(300, 333, 128, 1), (96, 80, 16, 2), (64, 200, 8, 3)])
def test_blocksparse_matches_sdpa_with_the_expanded_mask(Sq, Sk, blk, seed):
    B, Hq, Hkv, D = 2, 8, 2, 16
    q, k, v = rnd((B, Sq, Hq, D), seed), rnd((B, Sk, Hkv, D), seed + 10), \
        rnd((B, Sk, Hkv, D), seed + 20)
    n_q, n_k = -(-Sq // blk), -(-Sk // blk)
    row_ptr, col = random_pattern(n_q, n_k, seed, empty_rows=(1,))
    O, L = oracle.attention_blocksparse(q, k, v, row_ptr, col, scale=0.3, blk=blk)
    Or, Lr = masked_sdpa(q, k, v, 0.3, expand_pattern(row_ptr, col, Sq, Sk, blk))
    np.testing.assert_allclose(O, Or, rtol=0, atol=1e-12)
    assert np.array_equal(np.isneginf(L), np.isneginf(Lr))
    fin = np.isfinite(Lr)
    np.testing.assert_allclose(L[fin], Lr[fin], rtol=0, atol=1e-12)
    assert np.all(O[:, blk:2 * blk] == 0)  # the empty query block


def test_blocksparse_with_every_block_is_dense_attention():
    B, Hq, Hkv, Sq, Sk, D = 1, 4, 2, 70, 90, 8
    q, k, v = rnd((B, Sq, Hq, D), 30), rnd((B, Sk, Hkv, D), 31), rnd((B, Sk, Hkv, D), 32)
    n_q, n_k = -(-Sq // 16), -(-Sk // 16)
    row_ptr = np.arange(n_q + 1, dtype=np.int32) * n_k
    col = np.tile(np.arange(n_k, dtype=np.int32), n_q)
    O, L = oracle.attention_blocksparse(q, k, v, row_ptr, col, scale=0.5, blk=16)
    Or, Lr = sdpa_ref(q, k, v, 0.5, False)
    np.testing.assert_allclose(O, Or, rtol=0, atol=1e-12)
    np.testing.assert_allclose(L, Lr, rtol=0, atol=1e-12)


@pytest.mark.parametrize("Sq,Sk,blk,seed", [(300, 300, 128, 4), (96, 120, 16, 5), (70, 40, 8, 6)])
def test_causal_blocksparse_matches_sdpa_with_pattern_and_causal_mask(Sq, Sk, blk, seed):
    B, Hq, Hkv, D = 2, 8, 2, 16
    q, k, v = rnd((B, Sq, Hq, D), seed), rnd((B, Sk, Hkv, D), seed + 10), \
        rnd((B, Sk, Hkv, D), seed + 20)
    n_q, n_k = -(-Sq // blk), -(-Sk // blk)
    row_ptr, col = random_pattern(n_q, n_k, seed, density=0.5)
    O, L = oracle.attention_blocksparse(q, k, v, row_ptr, col, scale=0.3, blk=blk, causal=True)
    mask = expand_pattern(row_ptr, col, Sq, Sk, blk) & band_mask(Sq, Sk, Sk + Sq)
    Or, Lr = masked_sdpa(q, k, v, 0.3, mask)
    np.testing.assert_allclose(O, Or, rtol=0, atol=1e-12)
    assert np.array_equal(np.isneginf(L), np.isneginf(Lr))
    fin = np.isfinite(Lr)
    np.testing.assert_allclose(L[fin], Lr[fin], rtol=0, atol=1e-12)


def test_causal_blocksparse_with_every_block_is_causal_attention():
    B, Hq, Hkv, Sq, Sk, D = 1, 4, 2, 70, 90, 8
    q, k, v = rnd((B, Sq, Hq, D), 33), rnd((B, Sk, Hkv, D), 34), rnd((B, Sk, Hkv, D), 35)
    n_q, n_k = -(-Sq // 16), -(-Sk // 16)
    row_ptr = np.arange(n_q + 1, dtype=np.int32) * n_k
    col = np.tile(np.arange(n_k, dtype=np.int32), n_q)
    O, L = oracle.attention_blocksparse(q, k, v, row_ptr, col, scale=0.5, blk=16, causal=True)
    Or, Lr = sdpa_ref(q, k, v, 0.5, True, bottom_right=True)
    np.testing.assert_allclose(O, Or, rtol=0, atol=1e-12)
    np.testing.assert_allclose(L, Lr, rtol=0, atol=1e-12)


def test_blocksparse_rejects_bad_patterns():
    q, k, v = rnd((1, 20, 2, 4), 40), rnd((1, 20, 1, 4), 41), rnd((1, 20, 1, 4), 42)
    with pytest.raises(ValueError):  # key block 3 does not exist for 20 keys in blocks of 8
        oracle.attention_blocksparse(q, k, v, np.array([0, 1, 1, 1], np.int32),
                                     np.array([3], np.int32), scale=1.0, blk=8)
    with pytest.raises(ValueError):  # row pointers must not decrease
        oracle.attention_blocksparse(q, k, v, np.array([0, 2, 1, 2], np.int32),
                                     np.array([0, 1], np.int32), scale=1.0, blk=8)


# ---------------------------------------------------------------------------------
# Block-sparse over packed sequences with minimum padding (Raptor-T abstract)

VARLEN_LENS = [50, 0, 130, 17, 260, 33]


def varlen_sparse_case(blk, seed):
    cu = np.concatenate([[0], np.cumsum(VARLEN_LENS)]).astype(np.int32)
    total, Hq, Hkv, D = int(cu[-1]), 4, 2, 16
    q, k, v = rnd((total, Hq, D), seed), rnd((total, Hkv, D), seed + 1), \
        rnd((total, Hkv, D), seed + 2)
    rp, cl = W.bigbird_pattern_varlen(VARLEN_LENS, {"window": 3, "global": 1, "random": 2},
                                      seed=seed + 3, blk=blk)
    return cu, q, k, v, rp.numpy(), cl.numpy()


@pytest.mark.parametrize("blk,seed", [(16, 90), (32, 95)])
def test_blocksparse_varlen_matches_sdpa_per_sequence(blk, seed):
    cu, q, k, v, rp, cl = varlen_sparse_case(blk, seed)
    O, L = oracle.attention_blocksparse_varlen(q, k, v, cu, rp, cl, scale=0.3, blk=blk)
    row0 = 0  # first pattern row of the sequence: its blocks follow the earlier ones'
    for b, n in enumerate(VARLEN_LENS):
        nb = -(-n // blk)
        sl = slice(cu[b], cu[b + 1])
        if n:
            sub_rp = rp[row0:row0 + nb + 1] - rp[row0]
            sub_cl = cl[rp[row0]:rp[row0 + nb]]
            mask = expand_pattern(sub_rp, sub_cl, n, n, blk)
            Or, Lr = masked_sdpa(q[sl][None], k[sl][None], v[sl][None], 0.3, mask)
            np.testing.assert_allclose(O[sl], Or[0], rtol=0, atol=1e-12)
            Lb = L[:, sl]
            assert np.array_equal(np.isneginf(Lb), np.isneginf(Lr[0]))
            fin = np.isfinite(Lr[0])
            np.testing.assert_allclose(Lb[fin], Lr[0][fin], rtol=0, atol=1e-12)
        row0 += nb


def test_blocksparse_varlen_equals_the_dense_form_per_sequence():
    blk = 16
    cu, q, k, v, rp, cl = varlen_sparse_case(blk, 97)
    O, L = oracle.attention_blocksparse_varlen(q, k, v, cu, rp, cl, scale=0.25, blk=blk)
    row0 = 0
    for b, n in enumerate(VARLEN_LENS):
        nb = -(-n // blk)
        if n:
            sl = slice(cu[b], cu[b + 1])
            sub_rp = rp[row0:row0 + nb + 1] - rp[row0]
            Od, Ld = oracle.attention_blocksparse(q[sl][None], k[sl][None], v[sl][None], sub_rp,
                                                  cl[rp[row0]:rp[row0 + nb]], scale=0.25,
                                                  blk=blk)
            np.testing.assert_allclose(O[sl], Od[0], rtol=0, atol=1e-13)
            np.testing.assert_allclose(L[:, sl], Ld[0], rtol=0, atol=1e-13)
        row0 += nb


def test_causal_blocksparse_varlen_equals_the_causal_dense_form_per_sequence():
    blk = 16
    lens = [37, 0, 64, 5, 90]
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    total, Hq, Hkv, D = int(cu[-1]), 4, 2, 8
    q, k, v = rnd((total, Hq, D), 370), rnd((total, Hkv, D), 371), rnd((total, Hkv, D), 372)
    rps, cols, r0 = [np.zeros(1, dtype=np.int32)], [], 0
    parts = []
    for b, n in enumerate(lens):
        nb = -(-n // blk)
        rp, cl = random_pattern(nb, nb, 380 + b, density=0.6) if nb else \
            (np.zeros(1, dtype=np.int32), np.zeros(0, dtype=np.int32))
        parts.append((rp, cl))
        rps.append(rp[1:] + r0)
        cols.append(cl)
        r0 += int(rp[-1])
    row_ptr = np.concatenate(rps).astype(np.int32)
    col = np.concatenate(cols).astype(np.int32)
    O, L = oracle.attention_blocksparse_varlen(q, k, v, cu, row_ptr, col, scale=0.4, blk=blk,
                                               causal=True)
    for b, n in enumerate(lens):
        if n == 0:
            continue
        sl = slice(int(cu[b]), int(cu[b + 1]))
        rp, cl = parts[b]
        Ob, Lb = oracle.attention_blocksparse(q[sl][None], k[sl][None], v[sl][None], rp, cl,
                                              scale=0.4, blk=blk, causal=True)
        np.testing.assert_array_equal(O[sl], Ob[0])
        np.testing.assert_array_equal(L[:, sl], Lb[0])


def test_blocksparse_varlen_rejects_blocks_of_other_sequences():
    blk = 16
    cu, q, k, v, rp, cl = varlen_sparse_case(blk, 99)
    bad = cl.copy()
    bad[0] = 4  # sequence 0 (50 positions) has key blocks 0..3 only
    with pytest.raises(ValueError):
        oracle.attention_blocksparse_varlen(q, k, v, cu, rp, bad, scale=0.3, blk=blk)
    with pytest.raises(ValueError):  # one row per block of every sequence
        oracle.attention_blocksparse_varlen(q, k, v, cu, rp[:-1], cl, scale=0.3, blk=blk)


# ---------------------------------------------------------------------------------
# Backward (FA-2 page: dK, dV per K/V block, dQ shared; GQA: dK, dV summed over heads)

def autograd_ref(q, k, v, do, scale, causal):
    """torch float64 autograd through scaled_dot_product_attention (enable_gqa), with
    the forward's bottom-right causal mask; returns dq, dk, dv in [B, S, H, D]."""
    qt, kt, vt = (bshd_to_bhsd64(a).clone().requires_grad_(True) for a in (q, k, v))
    mask = None
    if causal:
        Sq, Sk = qt.shape[2], kt.shape[2]
        mask = torch.ones(Sq, Sk, dtype=torch.bool).tril(diagonal=Sk - Sq)
    o = F.scaled_dot_product_attention(qt, kt, vt, attn_mask=mask, scale=scale,
                                       enable_gqa=True)
    o.backward(bshd_to_bhsd64(do))
    return tuple(t.grad.transpose(1, 2).numpy() for t in (qt, kt, vt))


@pytest.mark.parametrize("B,Hq,Hkv,Sq,Sk,D,causal", [
    (2, 8, 2, 33, 33, 16, True),     # GQA, causal, Sq = Sk
    (1, 6, 2, 20, 45, 8, True),      # Sq < Sk, bottom-right
    (2, 4, 1, 17, 29, 16, False),    # MQA
    (1, 3, 3, 12, 12, 32, False),    # MHA
])
def test_backward_matches_torch_autograd_float64(B, Hq, Hkv, Sq, Sk, D, causal):
    seed = B * 100 + Sq + Sk
    q, k, v = rnd((B, Sq, Hq, D), seed), rnd((B, Sk, Hkv, D), seed + 1), \
        rnd((B, Sk, Hkv, D), seed + 2)
    do = rnd((B, Sq, Hq, D), seed + 3)
    got = oracle.attention_backward(q, k, v, do, scale=0.4, causal=causal)
    for g, r in zip(got, autograd_ref(q, k, v, do, 0.4, causal)):
        np.testing.assert_allclose(g, r, rtol=0, atol=1e-11)


def test_backward_matches_finite_differences_of_the_forward():
    # d/dx of sum(O * dO) by central differences of the (separately pinned) forward
    B, Hq, Hkv, Sq, Sk, D = 1, 2, 1, 4, 5, 3
    q, k, v = rnd((B, Sq, Hq, D), 60), rnd((B, Sk, Hkv, D), 61), rnd((B, Sk, Hkv, D), 62)
    do = rnd((B, Sq, Hq, D), 63)
    dq, dk, dv = oracle.attention_backward(q, k, v, do, scale=0.7, causal=True)

    def loss(q_, k_, v_):
        o, _ = oracle.attention(q_, k_, v_, scale=0.7, causal=True)
        return float(np.sum(o * do.astype(np.float64)))

    h = 2.0 ** -8  # exact in float32 next to values of order 1
    for arr, grad, which in ((q, dq, 0), (k, dk, 1), (v, dv, 2)):
        for idx in np.ndindex(arr.shape):
            plus, minus = arr.copy(), arr.copy()
            plus[idx] += h
            minus[idx] -= h
            args_p = [q, k, v]
            args_m = [q, k, v]
            args_p[which], args_m[which] = plus, minus
            num = (loss(*args_p) - loss(*args_m)) / (float(plus[idx]) - float(minus[idx]))
            assert abs(num - grad[idx]) < 2e-4, (which, idx, num, grad[idx])


# ---------------------------------------------------------------------------------
# e4m3 prefill (the batch-size guide's FP8 lever): element = value(code) * tensor scale

def e4m3_tensors(shape, seed, spread=3.0):
    """float8_e4m3fn tensors from seeded normal draws (torch rounds to the format)."""
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(*shape, generator=g) * spread).to(torch.float8_e4m3fn)


@pytest.mark.parametrize("B,Hq,Hkv,Sq,Sk,D,causal", [
    (2, 8, 2, 33, 33, 16, True),    # GQA, causal
    (1, 6, 2, 20, 45, 8, True),     # Sq < Sk, bottom-right
    (2, 4, 1, 17, 29, 16, False),   # MQA
])
def test_e4m3_prefill_matches_sdpa_on_torch_decoded_values(B, Hq, Hkv, Sq, Sk, D, causal):
    q8, k8, v8 = e4m3_tensors((B, Sq, Hq, D), 80), e4m3_tensors((B, Sk, Hkv, D), 81), \
        e4m3_tensors((B, Sk, Hkv, D), 82)
    qs, ks, vs, scale = 0.75, 0.125, 3.0, 0.3
    o, lse = oracle.attention_e4m3(q8, k8, v8, q_scale=qs, k_scale=ks, v_scale=vs,
                                   scale=scale, causal=causal)
    dec = [(t.to(torch.float64) * sc).numpy() for t, sc in ((q8, qs), (k8, ks), (v8, vs))]
    o_ref, lse_ref = sdpa_ref(*dec, scale, causal, bottom_right=causal and Sq != Sk)
    assert np.max(np.abs(o - o_ref)) < 1e-11 * max(1.0, np.abs(o_ref).max())
    assert np.max(np.abs(lse - lse_ref)) < 1e-11 * max(1.0, np.abs(lse_ref).max())


def test_e4m3_prefill_varlen_is_per_sequence():
    lens = [5, 0, 17, 9]
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    q8, k8, v8 = e4m3_tensors((cu[-1], 4, 16), 83), e4m3_tensors((cu[-1], 2, 16), 84), \
        e4m3_tensors((cu[-1], 2, 16), 85)
    o, lse = oracle.attention_e4m3(q8, k8, v8, q_scale=0.5, k_scale=2.0, v_scale=0.25,
                                   scale=0.2, causal=True, cu_seqlens=cu)
    for b, n in enumerate(lens):
        if n == 0:
            continue
        sl = slice(cu[b], cu[b + 1])
        ob, lb = oracle.attention_e4m3(q8[sl][None], k8[sl][None], v8[sl][None], q_scale=0.5,
                                       k_scale=2.0, v_scale=0.25, scale=0.2, causal=True)
        assert np.array_equal(o[sl], ob[0]) and np.array_equal(lse[:, sl], lb[0])


def test_e4m3_prefill_rejects_nan_codes():
    q8 = e4m3_tensors((1, 4, 2, 8), 86)
    k8 = e4m3_tensors((1, 4, 1, 8), 87)
    bad = k8.view(torch.uint8).clone()
    bad[0, 2, 0, 3] = 0x7F
    with pytest.raises(ValueError):
        oracle.attention_e4m3(q8, bad, k8, q_scale=1, k_scale=1, v_scale=1, scale=0.3,
                              causal=False)


def test_bf16_backward_model_tracks_the_oracle():
    # the tolerance model of the backward's bf16 arithmetic: close to the exact
    # gradients (its error is rounding, a fraction of a percent), but not equal to them
    from parity import bf16_backward_model
    q, k, v = rnd((1, 40, 4, 16), 70), rnd((1, 50, 2, 16), 71), rnd((1, 50, 2, 16), 72)
    do = rnd((1, 40, 4, 16), 73)
    tq, tk, tv, tdo = (torch.from_numpy(a).bfloat16() for a in (q, k, v, do))
    exact = oracle.attention_backward(tq, tk, tv, tdo, scale=0.25, causal=True)
    model = bf16_backward_model(tq, tk, tv, tdo, 0.25, True)
    for m, r in zip(model, exact):
        err = np.abs(m - r)
        assert 0 < err.max() <= 1e-2 * max(1.0, np.abs(r).max())
        assert err.mean() <= 2e-3 * max(1.0, np.abs(r).mean())


def test_e4m3_prefill_model_tracks_the_oracle():
    # the tolerance model of the e4m3 prefill: P rounded to e4m3 costs a few percent of
    # O, not more; without that rounding (p kept exact) it equals the oracle
    from parity import e4m3_prefill_model
    q8, k8, v8 = e4m3_tensors((1, 64, 4, 128), 110), e4m3_tensors((1, 80, 2, 128), 111), \
        e4m3_tensors((1, 80, 2, 128), 112)
    o, _ = oracle.attention_e4m3(q8, k8, v8, q_scale=0.5, k_scale=0.25, v_scale=2.0,
                                 scale=0.088, causal=True)
    m = e4m3_prefill_model(q8, k8, v8, 0.5, 0.25, 2.0, 0.088, True)
    err = np.abs(m - o)
    assert 0 < err.mean() <= 0.05 * np.abs(o).mean()
    assert err.max() <= 0.1 * np.abs(o).max()


# ---------------------------------------------------------------------------------
# Pin strength: every planted mistake is caught by at least one pin above

PIN_BATTERY = [
    lambda: test_glossary_example_gqa_equals_repeat_interleaved_mha(),
    lambda: test_matches_torch_sdpa_float64(2, 8, 2, 33, 33, 16, True),
    lambda: test_matches_torch_sdpa_float64(3, 12, 4, 20, 31, 24, True),
    lambda: test_decode_row_sees_every_key(),
    lambda: test_brute_force_50_digits(True, 4, 4),
    lambda: test_tiled_forms_equal_full_matrix(7, 5, 1, True, 37, 37),
    lambda: test_equal_keys_average_the_visible_values(),
    lambda: test_kvcache_lengths_and_window_match_sdpa_on_slices(7),
    lambda: test_kvcache_paged_matches_sdpa(16, 0),
    lambda: test_e4m3_table_matches_torch_float8(),
    lambda: test_blocksparse_matches_sdpa_with_the_expanded_mask(96, 80, 16, 2),
    lambda: test_backward_matches_torch_autograd_float64(2, 8, 2, 33, 33, 16, True),
    lambda: test_e4m3_prefill_matches_sdpa_on_torch_decoded_values(2, 8, 2, 33, 33, 16, True),
    lambda: test_blocksparse_varlen_matches_sdpa_per_sequence(16, 90),
    lambda: test_window_prefill_matches_sdpa_with_the_band_mask(33, 70, 16),
    lambda: test_causal_blocksparse_matches_sdpa_with_pattern_and_causal_mask(96, 120, 16, 5),
]


def battery_passes():
    for pin in PIN_BATTERY:
        try:
            pin()
        except AssertionError:
            return False
    return True


@pytest.mark.parametrize("flaw", [f for f in oracle.FLAWS if f != "none"])
def test_each_planted_mistake_is_caught(flaw):
    try:
        oracle.set_flaw(flaw)
        assert not battery_passes(), f"planted mistake '{flaw}' slipped through every pin"
    finally:
        oracle.set_flaw("none")
    assert battery_passes()
