"""Host-side checks of the C ABI: the library loads, exports every declared
symbol, and rejects bad arguments with the documented status codes before it
touches a GPU.  No compute call is made here."""
import ctypes
import os
import re

import pytest

import exact_attention_gqa_b200 as G
from exact_attention_gqa_b200 import _capi, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "gqa_attn.h")


@pytest.fixture(scope="module")
def lib():
    build.build()
    return _capi.load()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(gqa_attn_\w+)\s*\(", text)))


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert set(names) == set(_capi.EXPORTS)
    for n in names:
        assert hasattr(lib, n), n


def test_library_needs_no_driver_to_load():
    out = os.popen(f"ldd {_capi.LIB_PATH}").read()
    assert "libcuda.so" not in out and "libcudart.so" not in out


def test_status_codes_match_header(lib):
    text = open(HEADER).read()
    for name, val in re.findall(r"(GQA_(?:OK|ERR_\w+))\s*=\s*(-?\d+)", text):
        assert G.STATUS[int(val)] == name
        assert lib.gqa_attn_strerror(int(val)) != b"unknown status"


FAKE = ctypes.c_void_p(0x1000)  # never dereferenced: every case fails argument checks first


def call(lib, *, q=FAKE, k=FAKE, v=FAKE, out=FAKE, lse=FAKE, B=1, Hq=8, Hkv=2, Sq=16, Sk=16,
         D=64, scale=0.125, causal=1, splits=1, pack=-1, cu=None, f32=False):
    fn = lib.gqa_attn_fwd_f32 if f32 else lib.gqa_attn_fwd
    return fn(q, k, v, out, lse, B, Hq, Hkv, Sq, Sk, D, scale, causal, splits, pack, cu, None)


@pytest.mark.parametrize("kw,code", [
    (dict(q=None), "GQA_ERR_NULL"),
    (dict(lse=None), "GQA_ERR_NULL"),
    (dict(k=None), "GQA_ERR_NULL"),
    (dict(v=None, cu=FAKE), "GQA_ERR_NULL"),          # packed rows are always read
    (dict(Hq=6, Hkv=4), "GQA_ERR_SHAPE"),
    (dict(B=-1), "GQA_ERR_SHAPE"),
    (dict(Sk=-3), "GQA_ERR_SHAPE"),
    (dict(Hkv=0), "GQA_ERR_SHAPE"),
    (dict(D=96), "GQA_ERR_HEADDIM"),
    (dict(D=256), "GQA_ERR_HEADDIM"),
    (dict(D=300, f32=True), "GQA_ERR_HEADDIM"),
    (dict(scale=0.0), "GQA_ERR_SCALE"),
    (dict(scale=float("nan")), "GQA_ERR_SCALE"),
    (dict(scale=float("inf")), "GQA_ERR_SCALE"),
    (dict(splits=-1), "GQA_ERR_SPLITS"),
    (dict(splits=257, Sq=1), "GQA_ERR_SPLITS"),
    (dict(splits=4), "GQA_ERR_SPLITS"),                   # split-KV needs Sq == 1
    (dict(splits=2, Sq=1, f32=True), "GQA_ERR_SPLITS"),
    (dict(pack=2), "GQA_ERR_UNSUPPORTED"),
    (dict(q=ctypes.c_void_p(0x1008)), "GQA_ERR_ALIGN"),
    (dict(lse=ctypes.c_void_p(0x1002)), "GQA_ERR_ALIGN"),
])
def test_argument_errors(lib, kw, code):
    assert G.STATUS[call(lib, **kw)] == code


def test_empty_problems_are_successful_noops(lib):
    assert call(lib, B=0, q=None, k=None, v=None, out=None, lse=None) == 0
    assert call(lib, Sq=0, q=None, k=None, v=None, out=None, lse=None) == 0
    assert call(lib, B=0, f32=True, q=None, k=None, v=None, out=None, lse=None) == 0
    # packed batch with no rows at all
    assert call(lib, Sk=0, Sq=5, cu=FAKE, q=None, k=None, v=None, out=None, lse=None) == 0


def test_workspace_accounting(lib):
    assert lib.gqa_attn_workspace_bytes(4, 32, 1, 128, 1) == 0
    n = lib.gqa_attn_workspace_bytes(4, 32, 1, 128, 8)
    rows = 4 * 32 * 8
    assert n >= rows * 128 * 4 + rows * 4
    assert lib.gqa_attn_set_workspace(ctypes.c_void_p(0x1004), 64) == G.STATUS_CODE["GQA_ERR_ALIGN"]
    assert lib.gqa_attn_set_workspace(None, 0) == 0


def test_plan_choices(lib):
    # prefill: PackGQA when the group divides the 128-row tile
    rc, kern, splits, pack = G.gqa_attn_plan(4, 32, 8, 8192, 8192, 128, causal=True)
    assert (kern, splits, pack) == ("prefill_sm100", 1, 1)
    rc, kern, splits, pack = G.gqa_attn_plan(1, 6, 2, 100, 100, 64, pack_gqa=1)
    assert kern == "prefill_sm100" and pack == 0        # G = 3 cannot pack a 128-row tile
    rc, kern, splits, pack = G.gqa_attn_plan(1, 32, 8, 1, 32768, 128, num_splits=8)
    assert (kern, splits, pack) == ("decode_splitkv", 8, 1)
    rc, kern, splits, pack = G.gqa_attn_plan(1, 32, 8, 1, 100, 128, num_splits=8)
    assert kern == "decode_splitkv" and splits == 2     # clamped to the 64-key blocks
    rc, kern, splits, pack = G.gqa_attn_plan(1, 32, 8, 1, 32768, 128, num_splits=0)
    assert kern == "decode_splitkv" and 1 < splits <= 64
    rc, kern, splits, pack = G.gqa_attn_plan(2, 8, 2, 5, 0, 64)
    assert kern == "zero_fill"
    rc, kern, splits, pack = G.gqa_attn_plan(0, 8, 2, 5, 7, 64)
    assert kern == "none"


def test_python_front_end_refuses_cpu_tensors():
    import torch
    q = torch.zeros(1, 4, 2, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="CUDA"):
        G.gqa_attn(q, q[:, :, :1].contiguous(), q[:, :, :1].contiguous())


def test_host_pipeline_argument_errors(lib):
    """gqa_attn_fwd_host validates before it touches a device."""
    fn = lib.gqa_attn_fwd_host
    P = ctypes.c_void_p
    h = P(0x1000)
    args = [h] * 10 + [2, 8, 2, 16, 16, 64, 0.125, 0, 1, -1]
    assert fn(*args, 65, None) == G.STATUS_CODE["GQA_ERR_SHAPE"]     # chunks > 64
    assert fn(*args, -1, None) == G.STATUS_CODE["GQA_ERR_SHAPE"]     # chunks < 0
    bad = [None] + [h] * 9 + [2, 8, 2, 16, 16, 64, 0.125, 0, 1, -1]
    assert fn(*bad, 2, None) == G.STATUS_CODE["GQA_ERR_NULL"]
    wrong_d = [h] * 10 + [2, 8, 2, 16, 16, 96, 0.125, 0, 1, -1]
    assert fn(*wrong_d, 2, None) == G.STATUS_CODE["GQA_ERR_HEADDIM"]
    empty = [None] * 10 + [0, 8, 2, 16, 16, 64, 0.125, 0, 1, -1]
    assert fn(*empty, 2, None) == 0                                  # nothing to do


def test_host_pipeline_varlen_checks_offsets(lib):
    """gqa_attn_fwd_host_varlen rejects host offsets that do not describe the rows."""
    fn = lib.gqa_attn_fwd_host_varlen
    P = ctypes.c_void_p
    h = P(0x1000)

    def call(cu, B, max_len, total, chunks=2):
        arr = (ctypes.c_int * len(cu))(*cu)
        return fn(*([h] * 10), ctypes.cast(arr, P), h, B, 8, 2, max_len, total, 64, 0.125, 1,
                  -1, chunks, None)

    assert call([1, 5, 9], 2, 8, 9) == G.STATUS_CODE["GQA_ERR_SHAPE"]      # cu[0] != 0
    assert call([0, 5, 8], 2, 8, 9) == G.STATUS_CODE["GQA_ERR_SHAPE"]      # cu[B] != total
    assert call([0, 6, 5], 2, 8, 5) == G.STATUS_CODE["GQA_ERR_SHAPE"]      # decreasing
    assert call([0, 6, 9], 2, 5, 9) == G.STATUS_CODE["GQA_ERR_SHAPE"]      # longer than max
    assert call([0, 5, 9], 2, 8, 9, chunks=65) == G.STATUS_CODE["GQA_ERR_SHAPE"]


def kv_call(lib, *, q=FAKE, k=FAKE, v=FAKE, sl=None, out=FAKE, lse=FAKE, B=2, Hq=8, Hkv=2,
            Sk=100, D=64, msl=0, scale=0.125, window=0, splits=0, pack=-1):
    return lib.gqa_attn_decode_kvcache(q, k, v, sl, out, lse, B, Hq, Hkv, Sk, D, msl, scale,
                                       window, splits, pack, None)


def paged_call(lib, *, q=FAKE, k=FAKE, v=FAKE, bt=FAKE, sl=FAKE, out=FAKE, lse=FAKE, B=2, Hq=8,
               Hkv=2, D=64, num_pages=10, page_size=64, max_pages=4, msl=100, scale=0.125,
               window=0, splits=0, pack=-1):
    return lib.gqa_attn_decode_paged(q, k, v, bt, sl, out, lse, B, Hq, Hkv, D, num_pages,
                                     page_size, max_pages, msl, scale, window, splits, pack, None)


@pytest.mark.parametrize("kw,code", [
    (dict(q=None), "GQA_ERR_NULL"),
    (dict(k=None), "GQA_ERR_NULL"),
    (dict(window=-1), "GQA_ERR_SHAPE"),
    (dict(sl=FAKE, msl=101), "GQA_ERR_SHAPE"),        # bound above the capacity
    (dict(B=70000, Sk=40000), "GQA_ERR_SHAPE"),       # rows past 32-bit TMA coordinates
    (dict(Hq=6, Hkv=4), "GQA_ERR_SHAPE"),
    (dict(D=96), "GQA_ERR_HEADDIM"),
    (dict(scale=0.0), "GQA_ERR_SCALE"),
    (dict(splits=257), "GQA_ERR_SPLITS"),
    (dict(pack=2), "GQA_ERR_UNSUPPORTED"),
    (dict(q=ctypes.c_void_p(0x1008)), "GQA_ERR_ALIGN"),
    (dict(sl=ctypes.c_void_p(0x1002), msl=10), "GQA_ERR_ALIGN"),
])
def test_kvcache_argument_errors(lib, kw, code):
    assert G.STATUS[kv_call(lib, **kw)] == code


@pytest.mark.parametrize("kw,code", [
    (dict(bt=None), "GQA_ERR_NULL"),
    (dict(sl=None), "GQA_ERR_NULL"),
    (dict(page_size=48), "GQA_ERR_SHAPE"),            # not a power of two
    (dict(page_size=8), "GQA_ERR_SHAPE"),             # below 16
    (dict(num_pages=0), "GQA_ERR_SHAPE"),
    (dict(max_pages=0), "GQA_ERR_SHAPE"),
    (dict(msl=257), "GQA_ERR_SHAPE"),                 # past max_pages * page_size
    (dict(num_pages=1 << 22, page_size=1024), "GQA_ERR_SHAPE"),
    (dict(window=-5), "GQA_ERR_SHAPE"),
    (dict(D=32), "GQA_ERR_HEADDIM"),
    (dict(bt=ctypes.c_void_p(0x1002)), "GQA_ERR_ALIGN"),
])
def test_paged_argument_errors(lib, kw, code):
    assert G.STATUS[paged_call(lib, **kw)] == code


def test_kvcache_empty_batch_is_a_noop(lib):
    assert kv_call(lib, B=0, q=None, k=None, v=None, out=None, lse=None) == 0
    assert paged_call(lib, B=0, q=None, k=None, v=None, out=None, lse=None) == 0


def fp8_call(lib, *, q=FAKE, k=FAKE, v=FAKE, ks=0.5, vs=0.5, bt=None, sl=None, out=FAKE,
             lse=FAKE, B=2, Hq=8, Hkv=2, D=128, Sk=64, num_pages=0, page_size=0, max_pages=0,
             msl=0, scale=0.125, window=0, splits=0, pack=-1):
    return lib.gqa_attn_decode_fp8(q, k, v, ks, vs, bt, sl, out, lse, B, Hq, Hkv, D, Sk,
                                   num_pages, page_size, max_pages, msl, scale, window, splits,
                                   pack, None)


@pytest.mark.parametrize("kw,code", [
    (dict(ks=0.0), "GQA_ERR_SCALE"),
    (dict(vs=-1.0), "GQA_ERR_SCALE"),
    (dict(ks=float("nan")), "GQA_ERR_SCALE"),
    (dict(vs=float("inf")), "GQA_ERR_SCALE"),
    (dict(k=None), "GQA_ERR_NULL"),
    (dict(D=96), "GQA_ERR_HEADDIM"),
    (dict(window=-1), "GQA_ERR_SHAPE"),
    (dict(sl=FAKE, msl=65), "GQA_ERR_SHAPE"),
    (dict(bt=FAKE, sl=FAKE, num_pages=4, page_size=24, max_pages=2, msl=10), "GQA_ERR_SHAPE"),
    (dict(bt=FAKE, sl=None, num_pages=4, page_size=64, max_pages=2, msl=10), "GQA_ERR_NULL"),
    (dict(v=ctypes.c_void_p(0x1004)), "GQA_ERR_ALIGN"),
])
def test_fp8_argument_errors(lib, kw, code):
    assert G.STATUS[fp8_call(lib, **kw)] == code


def test_fp8_empty_batch_is_a_noop(lib):
    assert fp8_call(lib, B=0, q=None, k=None, v=None, out=None, lse=None) == 0


def sparse_call(lib, *, q=FAKE, k=FAKE, v=FAKE, out=FAKE, lse=FAKE, B=1, Hq=8, Hkv=2, Sq=256,
                Sk=256, D=128, scale=0.125, causal=0, rp=FAKE, col=FAKE):
    return lib.gqa_attn_fwd_blocksparse(q, k, v, out, lse, B, Hq, Hkv, Sq, Sk, D, scale,
                                        causal, rp, col, None)


@pytest.mark.parametrize("kw,code", [
    (dict(Hq=8, Hkv=8), "GQA_ERR_UNSUPPORTED"),     # G = 1: a tile spans two query blocks
    (dict(Hq=6, Hkv=2), "GQA_ERR_UNSUPPORTED"),     # G = 3 does not divide 128
    (dict(rp=None), "GQA_ERR_NULL"),
    (dict(col=None), "GQA_ERR_NULL"),
    (dict(q=None), "GQA_ERR_NULL"),
    (dict(D=96), "GQA_ERR_HEADDIM"),
    (dict(scale=-1.0), "GQA_ERR_SCALE"),
    (dict(Hq=6, Hkv=4), "GQA_ERR_SHAPE"),
    (dict(col=ctypes.c_void_p(0x1002)), "GQA_ERR_ALIGN"),
])
def test_blocksparse_argument_errors(lib, kw, code):
    assert G.STATUS[sparse_call(lib, **kw)] == code


def test_blocksparse_empty_batch_is_a_noop(lib):
    assert sparse_call(lib, B=0, q=None, k=None, v=None, out=None, lse=None) == 0
    assert sparse_call(lib, B=0, causal=1, q=None, k=None, v=None, out=None, lse=None) == 0


# ---------------------------------------------------------------- sliding window
def window_call(lib, *, q=FAKE, k=FAKE, v=FAKE, out=FAKE, lse=FAKE, B=1, Hq=8, Hkv=2, Sq=256,
                Sk=256, D=128, scale=0.125, window=64, pack=-1, cu=None):
    return lib.gqa_attn_fwd_window(q, k, v, out, lse, B, Hq, Hkv, Sq, Sk, D, scale, window,
                                   pack, cu, None)


@pytest.mark.parametrize("kw,code", [
    (dict(window=0), "GQA_ERR_SHAPE"),
    (dict(window=-3), "GQA_ERR_SHAPE"),
    (dict(Hq=6, Hkv=4), "GQA_ERR_SHAPE"),
    (dict(D=96), "GQA_ERR_HEADDIM"),
    (dict(scale=0.0), "GQA_ERR_SCALE"),
    (dict(pack=2), "GQA_ERR_UNSUPPORTED"),
    (dict(q=None), "GQA_ERR_NULL"),
    (dict(k=None), "GQA_ERR_NULL"),
    (dict(out=ctypes.c_void_p(0x1008)), "GQA_ERR_ALIGN"),
])
def test_window_argument_errors(lib, kw, code):
    assert G.STATUS[window_call(lib, **kw)] == code


def test_window_empty_problems_are_noops(lib):
    assert window_call(lib, B=0, q=None, k=None, v=None, out=None, lse=None) == 0
    assert window_call(lib, Sq=0, q=None, k=None, v=None, out=None, lse=None) == 0


# ---------------------------------------------------------------------------- backward
def bwd_call(lib, *, q=FAKE, k=FAKE, v=FAKE, out=FAKE, lse=FAKE, dout=FAKE, dq=FAKE, dk=FAKE,
             dv=FAKE, B=1, Hq=8, Hkv=2, Sq=256, Sk=256, D=128, scale=0.125, causal=1):
    return lib.gqa_attn_bwd(q, k, v, out, lse, dout, dq, dk, dv, B, Hq, Hkv, Sq, Sk, D, scale,
                            causal, None)


@pytest.mark.parametrize("kw,code", [
    (dict(D=96), "GQA_ERR_HEADDIM"),
    (dict(scale=-1.0), "GQA_ERR_SCALE"),
    (dict(Hq=6, Hkv=4), "GQA_ERR_SHAPE"),
    (dict(Sq=-1), "GQA_ERR_SHAPE"),
    (dict(q=None), "GQA_ERR_NULL"),
    (dict(lse=None), "GQA_ERR_NULL"),
    (dict(dout=None), "GQA_ERR_NULL"),
    (dict(dk=None), "GQA_ERR_NULL"),
    (dict(dv=ctypes.c_void_p(0x1008)), "GQA_ERR_ALIGN"),
    (dict(lse=ctypes.c_void_p(0x1002)), "GQA_ERR_ALIGN"),
])
def test_backward_argument_errors(lib, kw, code):
    assert G.STATUS[bwd_call(lib, **kw)] == code


def test_backward_empty_problems_are_noops(lib):
    assert bwd_call(lib, B=0, q=None, k=None, v=None, out=None, lse=None, dout=None, dq=None,
                    dk=None, dv=None) == 0
    assert bwd_call(lib, Sq=0, Sk=0, q=None, k=None, v=None, out=None, lse=None, dout=None,
                    dq=None, dk=None, dv=None) == 0


def test_backward_workspace_bytes(lib):
    # one fp32 D_i per (batch, query head, row), rounded up to 256 bytes
    assert lib.gqa_attn_bwd_workspace_bytes(2, 3, 5) == 256
    assert lib.gqa_attn_bwd_workspace_bytes(4, 32, 8192) == 4 * 32 * 8192 * 4
    assert lib.gqa_attn_bwd_workspace_bytes(0, 32, 8192) == 0


def test_backward_front_end_checks_shapes_first():
    import torch
    q = torch.zeros(1, 16, 4, 64, dtype=torch.bfloat16)
    k = torch.zeros(1, 20, 2, 64, dtype=torch.bfloat16)
    lse = torch.zeros(1, 4, 16)
    with pytest.raises(ValueError, match="lse must be"):
        G.gqa_attn_backward(q, k, k, q, lse[:, :, :8], q)
    with pytest.raises(ValueError, match="dk must be"):
        G.gqa_attn_backward(q, k, k, q, lse, q, dk=torch.zeros(1, 20, 2, 32, dtype=torch.bfloat16))
    with pytest.raises(ValueError, match="k/v must match"):
        G.gqa_attn_backward(q, k[..., :32], k[..., :32], q, lse, q)
    with pytest.raises(ValueError, match="CUDA tensor"):
        G.gqa_attn_backward(q, k, k, q, lse, q)


# ---------------------------------------------------------------- varlen block-sparse
def schedule(lib, lens, rows_per_block, Hq=8, Hkv=2, grid=148):
    """Run the host schedule; rows_per_block(b, r) gives the row length of block r of
    sequence b.  Returns (status, blk_off, order, g)."""
    import numpy as np
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    nblk = [-(-n // 128) for n in lens]
    rp = [0]
    for b, nb in enumerate(nblk):
        for r in range(nb):
            rp.append(rp[-1] + rows_per_block(b, r))
    rp = np.array(rp, dtype=np.int32)
    off = np.zeros(len(lens) + 1, dtype=np.int32)
    n, g = ctypes.c_int(0), ctypes.c_int(0)
    args = (cu.ctypes.data, rp.ctypes.data, len(lens), Hq, Hkv, max(lens), grid, off.ctypes.data)
    rc = lib.gqa_attn_sparse_varlen_schedule(*args, None, 0, ctypes.byref(n), ctypes.byref(g))
    if rc not in (0, G.STATUS_CODE["GQA_ERR_WORKSPACE"]):
        return rc, None, None, None
    order = np.zeros(max(n.value, 1), dtype=np.int32)
    rc = lib.gqa_attn_sparse_varlen_schedule(*args, order.ctypes.data, order.size,
                                             ctypes.byref(n), ctypes.byref(g))
    return rc, off, order[:n.value], g.value


def test_schedule_lists_every_tile_once_with_minimum_padding(lib):
    import numpy as np
    lens = [300, 0, 128, 1000, 17, 4096]
    Hq, Hkv = 8, 2
    rc, off, order, g = schedule(lib, lens, lambda b, r: 1 + (b + r) % 5, Hq, Hkv)
    assert rc == 0
    assert off.tolist() == [0, 3, 3, 4, 12, 13, 45]  # ceil(n / 128) rows per sequence
    sub = 128 // (Hq // Hkv)
    n_mblk = -(-max(lens) // (2 * sub))
    want = sorted((b * Hkv + h) * n_mblk + m for b, n in enumerate(lens)
                  for m in range(-(-n // (2 * sub))) for h in range(Hkv))
    assert sorted(order[order >= 0].tolist()) == want
    assert len(order) % g == 0 and g == min(148, len(want))


def test_schedule_balances_the_cost(lib):
    import numpy as np
    lens = [8192, 128, 4000, 2000, 640] * 4
    Hq, Hkv, grid = 8, 2, 16
    cost_of = lambda b, r: 40 if r < 2 else 6  # global rows are long, the rest short
    rc, off, order, g = schedule(lib, lens, cost_of, Hq, Hkv, grid)
    assert rc == 0 and g == grid
    sub = 128 // (Hq // Hkv)
    n_mblk = -(-max(lens) // (2 * sub))
    loads = np.zeros(g)
    for idx, u in enumerate(order.tolist()):
        if u < 0:
            continue
        m = u % n_mblk
        b = (u // n_mblk) // Hkv
        p0 = m * 2 * sub
        subs = 1 + (p0 + sub < lens[b])
        loads[idx % g] += cost_of(b, p0 // 128) * subs + 1
    # longest-first onto the least loaded CTA: no CTA exceeds another by more than the
    # largest single tile
    assert loads.max() - loads.min() <= 40 * 2 + 1


def test_schedule_argument_errors(lib):
    rc, *_ = schedule(lib, [100, 50], lambda b, r: 1, Hq=8, Hkv=8)  # G = 1
    assert G.STATUS[rc] == "GQA_ERR_UNSUPPORTED"
    import numpy as np
    cu = np.array([0, 300], dtype=np.int32)
    rp = np.array([0, 1, 2, 3], dtype=np.int32)
    off = np.zeros(2, dtype=np.int32)
    n, g = ctypes.c_int(0), ctypes.c_int(0)
    rc = lib.gqa_attn_sparse_varlen_schedule(cu.ctypes.data, rp.ctypes.data, 1, 8, 2, 200, 148,
                                             off.ctypes.data, None, 0, ctypes.byref(n),
                                             ctypes.byref(g))
    assert G.STATUS[rc] == "GQA_ERR_SHAPE"  # a sequence longer than max_seqlen


def test_blocksparse_varlen_argument_errors(lib):
    def call(**kw):
        a = dict(q=FAKE, k=FAKE, v=FAKE, out=FAKE, lse=FAKE, cu=FAKE, off=FAKE, B=2, Hq=8,
                 Hkv=2, S=256, total=300, D=128, scale=0.125, rp=FAKE, col=FAKE, order=None,
                 n_order=0, grid=0)
        a.update(kw)
        return G.STATUS[lib.gqa_attn_fwd_blocksparse_varlen(
            a["q"], a["k"], a["v"], a["out"], a["lse"], a["cu"], a["off"], a["B"], a["Hq"],
            a["Hkv"], a["S"], a["total"], a["D"], a["scale"], 0, a["rp"], a["col"], a["order"],
            a["n_order"], a["grid"], None)]
    assert call(Hq=8, Hkv=8) == "GQA_ERR_UNSUPPORTED"
    assert call(off=None) == "GQA_ERR_NULL"
    assert call(D=96) == "GQA_ERR_HEADDIM"
    assert call(order=FAKE, n_order=10, grid=3) == "GQA_ERR_SHAPE"
    assert call(cu=ctypes.c_void_p(0x1002)) == "GQA_ERR_ALIGN"
    assert call(B=0) == "GQA_OK"


# ---------------------------------------------------------------- e4m3 prefill
def fp8_prefill_call(lib, *, q=FAKE, k=FAKE, v=FAKE, out=FAKE, lse=FAKE, B=1, Hq=8, Hkv=2, Sq=256,
             Sk=256, D=128, scale=0.125, qs=1.0, ks=1.0, vs=1.0, causal=1, cu=None):
    return lib.gqa_attn_fwd_fp8(q, k, v, out, lse, B, Hq, Hkv, Sq, Sk, D, scale, qs, ks, vs,
                                causal, cu, None)


@pytest.mark.parametrize("kw,code", [
    (dict(D=64), "GQA_ERR_HEADDIM"),
    (dict(qs=0.0), "GQA_ERR_SCALE"),
    (dict(vs=float("inf")), "GQA_ERR_SCALE"),
    (dict(scale=-1.0), "GQA_ERR_SCALE"),
    (dict(Hq=6, Hkv=4), "GQA_ERR_SHAPE"),
    (dict(q=None), "GQA_ERR_NULL"),
    (dict(v=None), "GQA_ERR_NULL"),
    (dict(k=ctypes.c_void_p(0x1004)), "GQA_ERR_ALIGN"),
])
def test_fp8_prefill_argument_errors(lib, kw, code):
    assert G.STATUS[fp8_prefill_call(lib, **kw)] == code


def test_fp8_prefill_empty_problems_are_noops(lib):
    assert fp8_prefill_call(lib, B=0, q=None, k=None, v=None, out=None, lse=None) == 0
    assert fp8_prefill_call(lib, Sq=0, q=None, k=None, v=None, out=None, lse=None) == 0
