// Host side of the C ABI declared in include/gqa_attn.h: argument checks, the
// choice of kernel and knobs, TMA descriptor encoding and the launches.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstring>
#include <algorithm>
#include <mutex>
#include <queue>
#include <vector>

#include "gqa_attn.h"
#include "sm100_ptx.cuh"
#include "prefill_sm100.cuh"
#include "decode.cuh"
#include "simt_f32.cuh"

namespace {

using gqa::DecodeCfg;
using gqa::DecodeParams;
using gqa::F32Params;
using gqa::PrefillCfg;
using gqa::PrefillParams;

constexpr float kLog2e = 1.4426950408889634f;
constexpr int kMaxSplits = 256;
static_assert(kMaxSplits <= gqa::kCombineMaxSplits, "combine weights table too small");

enum Kernel { kNone = 0, kPrefill = 1, kDecode = 2, kZeroFill = 3 };

struct Workspace {
    void* ptr = nullptr;
    size_t bytes = 0;
};
Workspace g_ws[64];  // one registered split-KV workspace per device
std::mutex g_mu;

// ---------------------------------------------------------------------------- device
struct DeviceInfo {
    int ok = 0;       // 1 when the device is sm_100
    int sms = 0;
    int attrs_set = 0;  // bit mask of kernels whose shared-memory limit is raised here
};
DeviceInfo g_dev[64];

int device_info(DeviceInfo** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return GQA_ERR_CUDA;
    DeviceInfo& d = g_dev[dev];
    if (d.sms == 0) {
        int major = 0, minor = 0, sms = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return GQA_ERR_CUDA;
        d.ok = (major == 10 && minor == 0);
        d.sms = sms;
    }
    *out = &d;
    return d.ok ? GQA_OK : GQA_ERR_UNSUPPORTED;
}

// Raise a kernel's dynamic shared-memory limit once per device (the setting belongs to
// the device's context, so a process that drives several GPUs needs it on each).
template <typename Kernel>
int ensure_smem_limit(Kernel kernel, int bit, int bytes) {
    DeviceInfo* d = nullptr;
    const int rc = device_info(&d);
    if (rc != GQA_OK) return rc;
    if (d->attrs_set & bit) return GQA_OK;
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) !=
        cudaSuccess)
        return GQA_ERR_CUDA;
    d->attrs_set |= bit;
    return GQA_OK;
}

// ---------------------------------------------------------------------------- TMA
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

// 3-D bf16 view [rows, heads, D] with a {64, box_h, box_rows} box, 128-byte swizzle.
bool make_map(CUtensorMap* m, const void* base, long long rows, int heads, int D, int box_h,
              int box_rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[3] = {cuuint64_t(D), cuuint64_t(heads), cuuint64_t(rows)};
    cuuint64_t strides[2] = {cuuint64_t(D) * 2, cuuint64_t(heads) * D * 2};
    cuuint32_t box[3] = {64u, cuuint32_t(box_h), cuuint32_t(box_rows)};
    cuuint32_t estr[3] = {1u, 1u, 1u};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
              estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 8-bit [rows, heads, D] view (e4m3 K/V): boxes of {D bytes, 1 head, box_rows}, no swizzle
bool make_map_u8(CUtensorMap* m, const void* base, long long rows, int heads, int D,
                 int box_rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[3] = {cuuint64_t(D), cuuint64_t(heads), cuuint64_t(rows)};
    cuuint64_t strides[2] = {cuuint64_t(D), cuuint64_t(heads) * D};
    cuuint32_t box[3] = {cuuint32_t(D), 1u, cuuint32_t(box_rows)};
    cuuint32_t estr[3] = {1u, 1u, 1u};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides, box,
              estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 8-bit [rows, heads, D] view with 128-byte swizzle: boxes of {128 bytes, box_h,
// box_rows} (e4m3 Q, K, V of the prefill; D = 128 is one swizzle atom)
bool make_map_u8_sw128(CUtensorMap* m, const void* base, long long rows, int heads, int D,
                       int box_h, int box_rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[3] = {cuuint64_t(D), cuuint64_t(heads), cuuint64_t(rows)};
    cuuint64_t strides[2] = {cuuint64_t(D), cuuint64_t(heads) * D};
    cuuint32_t box[3] = {128u, cuuint32_t(box_h), cuuint32_t(box_rows)};
    cuuint32_t estr[3] = {1u, 1u, 1u};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides, box,
              estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// ---------------------------------------------------------------------------- plan
struct Plan {
    int kernel = kNone;
    int splits = 1;
    int pack = 0;
    int decode_rows = 1;
    int decode_units = 1;
    int blocks_per_split = 0;
};

int check_shape(int B, int Hq, int Hkv, int Sq, int Sk, int D, float scale, int num_splits,
                int pack_gqa, bool varlen, bool is_f32) {
    if (B < 0 || Sq < 0 || Sk < 0 || Hq <= 0 || Hkv <= 0) return GQA_ERR_SHAPE;
    if (Hq % Hkv != 0) return GQA_ERR_SHAPE;
    if (is_f32) {
        if (D < 1 || D > 256) return GQA_ERR_HEADDIM;
    } else if (D != 64 && D != 128) {
        return GQA_ERR_HEADDIM;
    }
    if (!(std::isfinite(scale) && scale > 0.f)) return GQA_ERR_SCALE;
    if (pack_gqa < -1 || pack_gqa > 1) return GQA_ERR_UNSUPPORTED;
    if (num_splits < 0 || num_splits > kMaxSplits) return GQA_ERR_SPLITS;
    if (num_splits > 1 && (is_f32 || varlen || Sq != 1)) return GQA_ERR_SPLITS;
    // index ranges: rows * heads * D must stay addressable with 32-bit row indices
    const long long rows_q = varlen ? 0 : (long long)B * Sq;
    const long long rows_k = varlen ? 0 : (long long)B * Sk;
    if (rows_q > INT32_MAX || rows_k > INT32_MAX) return GQA_ERR_SHAPE;
    return GQA_OK;
}

// Split count of the e4m3 decode for `units` CTAs' worth of (batch, head unit) work of
// `nblk` 64-key blocks each over `slots` resident CTAs: the n in [1, min(64, nblk / 4)]
// minimising ceil(units * pieces / slots) * (ceil(nblk / n) + 3).
int fp8_decode_splits(long long units, int nblk, long long slots) {
    const int n_max = std::max(1, std::min(64, nblk / 4));
    int best_n = 1;
    long long best = -1;
    for (int n = 1; n <= n_max; ++n) {
        const long long bps = (nblk + n - 1) / n;
        const long long pieces = (nblk + bps - 1) / bps;
        const long long waves = (units * pieces + slots - 1) / slots;
        const long long cost = waves * (bps + 3);
        if (best < 0 || cost < best) {
            best = cost;
            best_n = n;
        }
    }
    return best_n;
}

void make_plan(Plan* pl, int B, int Hq, int Hkv, int Sq, int Sk, int num_splits, int pack_gqa,
               bool varlen, int sms) {
    const int G = Hq / Hkv;
    *pl = Plan();
    if (B == 0 || Sq == 0) return;
    if (!varlen && Sk == 0) {
        pl->kernel = kZeroFill;
        return;
    }
    if (!varlen && Sq == 1) {
        pl->kernel = kDecode;
        pl->pack = (pack_gqa < 0) ? (G > 1 ? 1 : 0) : pack_gqa;
        pl->decode_rows = pl->pack ? (G < 16 ? G : 16) : 1;
        pl->decode_units = (G + pl->decode_rows - 1) / pl->decode_rows;
        const int nblk = (Sk + DecodeCfg<128>::BN - 1) / DecodeCfg<128>::BN;
        int n = num_splits;
        if (n == 0) {
            // As many splits as keep every CTA on an SM of its own (one CTA per SM
            // already streams at the HBM rate; a partial second wave only adds a
            // tail), with splits of at least four 64-key blocks.
            const long long ctas = (long long)B * Hkv * pl->decode_units;
            const long long want = sms / ctas;
            n = int(want < 1 ? 1 : (want > 64 ? 64 : want));
            const int max_by_len = nblk / 4 > 0 ? nblk / 4 : 1;
            if (n > max_by_len) n = max_by_len;
        }
        if (n > nblk) n = nblk;
        if (n < 1) n = 1;
        pl->blocks_per_split = (nblk + n - 1) / n;
        n = (nblk + pl->blocks_per_split - 1) / pl->blocks_per_split;  // drop empty splits
        pl->splits = n;
        return;
    }
    pl->kernel = kPrefill;
    pl->splits = 1;
    const bool can_pack = G > 1 && (128 % G == 0);
    pl->pack = (pack_gqa < 0) ? (can_pack ? 1 : 0) : (pack_gqa == 1 && can_pack ? 1 : 0);
}

size_t ws_bytes(int B, int Hq, int Sq, int D, int n) {
    if (n <= 1) return 0;
    const size_t rows = size_t(B) * Hq * Sq * n;
    const size_t o = rows * D * 4;
    return ((o + 255) / 256) * 256 + rows * 4;
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

template <int HD, bool FP8 = false>
int launch_prefill(const void* q, const void* k, const void* v, void* out, float* lse, int B,
                   int Hq, int Hkv, int Sq, int Sk, float scale, int causal, int pack,
                   const int* cu, int sms, cudaStream_t stream,
                   const int* blk_row_ptr = nullptr, const int* blk_col = nullptr,
                   const int* blk_off = nullptr, const int* tile_order = nullptr,
                   int n_order = 0, int order_grid = 0, float qk_scale = 1.f,
                   float o_scale = 1.f, int window = 0, int lse_ld = 0) {
    using C = PrefillCfg<HD, FP8>;
    if constexpr (!FP8) {
        const int rc = ensure_smem_limit(gqa::prefill_fwd_sm100<HD>, HD == 64 ? 1 : 2,
                                         C::SMEM_BYTES);
        if (rc != GQA_OK) return rc;
    }
    const int G = Hq / Hkv;
    PrefillParams p;
    p.out = static_cast<__nv_bfloat16*>(out);
    p.lse = lse;
    p.cu_seqlens = cu;
    p.B = B;
    p.Hq = Hq;
    p.Hkv = Hkv;
    p.Sq = Sq;
    p.Sk = Sk;
    p.G = G;
    p.pack = pack;
    p.sub_pos = pack ? 128 / G : 128;
    p.n_mblk = (Sq + 2 * p.sub_pos - 1) / (2 * p.sub_pos);
    p.n_hu = pack ? Hkv : Hq;
    const long long units = (long long)p.n_mblk * B * p.n_hu;
    if (units > INT32_MAX) return GQA_ERR_SHAPE;
    p.n_units = int(units);
    p.causal = causal ? 1 : 0;
    // dense non-causal: a (batch, head unit)'s position tiles back to back so its K/V
    // stay in L2; causal and packed batches: longest tiles first
    p.kv_major = (!causal && !cu) ? 1 : 0;
    {
        // about 32 MB of K and V per group of (batch, head unit) pairs (an L2 share);
        // without packing, G consecutive head units read the same KV head
        const long long kv_per_head = (long long)(cu ? Sq : Sk) * HD * 2 * 2;
        long long hg = (32LL << 20) / (kv_per_head > 0 ? kv_per_head : 1);
        if (!pack) hg *= G;
        const long long per_m = (long long)B * p.n_hu;
        if (hg < 1) hg = 1;
        if (hg > per_m) hg = per_m;
        p.hu_group = int(hg);
    }
    p.scale_log2 = scale * qk_scale * kLog2e;  // e4m3: the Q and K code units folded in
    p.o_scale = o_scale;
    p.blk_row_ptr = blk_row_ptr;
    p.blk_col = blk_col;
    p.n_kblk = (Sk + C::BN - 1) / C::BN;
    p.blk_off = blk_off;
    p.tile_order = tile_order;
    if (tile_order) p.n_units = n_order;  // the balanced order lists every step
    p.window = window;
    p.lse_ld = lse_ld > 0 ? lse_ld : Sq;
    // Row extents of the 3-D views: exactly the rows the caller allocated
    // (packed variable length: Sk carries the packed row count).
    const long long rows_q = cu ? (long long)Sk : (long long)B * Sq;
    const long long rows_k = cu ? (long long)Sk : (long long)B * Sk;
    p.total_rows = cu ? Sk : 0;
    CUtensorMap tq, tk, tv, to;
    // the output leaves through the same box shape as Q arrives in (one sub-tile)
    bool maps_ok;
    if constexpr (FP8)
        maps_ok = make_map_u8_sw128(&tq, q, rows_q, Hq, HD, pack ? G : 1, pack ? 128 / G : 128) &&
                  make_map_u8_sw128(&tk, k, rows_k, Hkv, HD, 1, C::BN) &&
                  make_map_u8_sw128(&tv, v, rows_k, Hkv, HD, 1, C::BN);
    else
        maps_ok = make_map(&tq, q, rows_q, Hq, HD, pack ? G : 1, pack ? 128 / G : 128) &&
                  make_map(&tk, k, rows_k, Hkv, HD, 1, C::BN) &&
                  make_map(&tv, v, rows_k, Hkv, HD, 1, C::BN);
    if (!maps_ok || !make_map(&to, out, rows_q, Hq, HD, pack ? G : 1, pack ? 128 / G : 128))
        return GQA_ERR_CUDA;
    const int grid = tile_order ? order_grid : (p.n_units < sms ? p.n_units : sms);
    if constexpr (FP8) {
        const int rc = ensure_smem_limit(gqa::prefill_fwd_sm100<HD, false, true>, 65536,
                                         C::SMEM_BYTES);
        if (rc != GQA_OK) return rc;
        gqa::prefill_fwd_sm100<HD, false, true><<<grid, C::THREADS, C::SMEM_BYTES, stream>>>(
            tq, tk, tv, to, p);
        return cudaGetLastError() == cudaSuccess ? GQA_OK : GQA_ERR_CUDA;
    }
    if (window > 0) {
        const int rc = ensure_smem_limit(gqa::prefill_fwd_sm100<HD, false, false, true>,
                                         HD == 64 ? 1 << 17 : 1 << 18, C::SMEM_BYTES);
        if (rc != GQA_OK) return rc;
        gqa::prefill_fwd_sm100<HD, false, false, true>
            <<<grid, C::THREADS, C::SMEM_BYTES, stream>>>(tq, tk, tv, to, p);
        return cudaGetLastError() == cudaSuccess ? GQA_OK : GQA_ERR_CUDA;
    }
    if (blk_row_ptr) {
        const int rc = ensure_smem_limit(gqa::prefill_fwd_sm100<HD, true>, HD == 64 ? 1024 : 2048,
                                         C::SMEM_BYTES);
        if (rc != GQA_OK) return rc;
        gqa::prefill_fwd_sm100<HD, true><<<grid, C::THREADS, C::SMEM_BYTES, stream>>>(tq, tk, tv,
                                                                                     to, p);
    } else {
        gqa::prefill_fwd_sm100<HD><<<grid, C::THREADS, C::SMEM_BYTES, stream>>>(tq, tk, tv, to, p);
    }
    return cudaGetLastError() == cudaSuccess ? GQA_OK : GQA_ERR_CUDA;
}

// The combine runs as a programmatic dependent launch of the split kernel: its CTAs
// are scheduled while the split kernel drains and wait in griddep_wait() for its
// completion, which removes the launch gap between the two kernels.
template <int HD>
int launch_combine(const float* part_o, const float* part_l, __nv_bfloat16* out, float* lse,
                   int rows_bh, int n, cudaStream_t stream) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(rows_bh);
    cfg.blockDim = dim3(HD);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, gqa::splitkv_combine<HD>, part_o, part_l, out, lse, rows_bh, n) !=
        cudaSuccess)
        return GQA_ERR_CUDA;
    return GQA_OK;
}

// KV-cache forms of a decode launch (decode.cuh); the defaults give the dense cache
struct KvCacheArgs {
    const int* seqlens_k = nullptr;    // [B] keys per sequence, or null: Sk each
    const int* block_table = nullptr;  // [B, max_pages], or null: dense [B, Sk, Hkv, D]
    int max_pages = 0;
    int page_size = 0;
    int num_pages = 0;
    int window = 0;                    // > 0: last `window` keys only
    bool fp8 = false;                  // K and V are e4m3 codes
    float k_scale = 1.f, v_scale = 1.f;  // value of one code unit of K and of V
};

int log2_exact(int x) {
    int l = 0;
    while ((1 << l) < x) ++l;
    return l;
}

template <int HD>
int launch_decode(const void* q, const void* k, const void* v, void* out, float* lse, int B,
                  int Hq, int Hkv, int Sk, float scale, const Plan& pl, cudaStream_t stream,
                  const KvCacheArgs& kv = KvCacheArgs()) {
    using C = DecodeCfg<HD>;
    {
        const int rc = ensure_smem_limit(gqa::decode_split_sm100<HD>, HD == 64 ? 4 : 8,
                                         C::SMEM_BYTES);
        if (rc != GQA_OK) return rc;
    }
    DecodeParams p;
    p.q = static_cast<const __nv_bfloat16*>(q);
    p.out = static_cast<__nv_bfloat16*>(out);
    p.lse = lse;
    p.B = B;
    p.Hq = Hq;
    p.Hkv = Hkv;
    p.Sk = Sk;
    p.G = Hq / Hkv;
    p.rows = pl.decode_rows;
    p.units_per_kv = pl.decode_units;
    p.n_splits = pl.splits;
    p.blocks_per_split = pl.blocks_per_split;
    p.scale_log2 = scale * kLog2e;
    p.part_o = nullptr;
    p.part_l = nullptr;
    p.seqlens_k = kv.seqlens_k;
    p.block_table = kv.block_table;
    p.max_pages = kv.max_pages;
    p.page_shift = kv.block_table ? log2_exact(kv.page_size) : 0;
    p.num_pages = kv.num_pages;
    p.window = kv.window;
    if (kv.fp8) {
        p.scale_log2 = scale * kv.k_scale * kLog2e;  // logits of the decoded keys
        p.v_scale = kv.v_scale;
    }
    if (pl.splits > 1) {
        const size_t need = ws_bytes(B, Hq, 1, HD, pl.splits);
        int dev = 0;
        if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return GQA_ERR_CUDA;
        Workspace ws;
        {
            std::lock_guard<std::mutex> lk(g_mu);
            ws = g_ws[dev];
        }
        if (!ws.ptr || ws.bytes < need) return GQA_ERR_WORKSPACE;
        const size_t o_bytes = size_t(B) * Hq * pl.splits * HD * 4;
        p.part_o = static_cast<float*>(ws.ptr);
        p.part_l = reinterpret_cast<float*>(static_cast<char*>(ws.ptr) +
                                            ((o_bytes + 255) / 256) * 256);
    }
    CUtensorMap tk, tv;
    // dense: B * Sk rows in 64-row boxes; paged: the pool's rows in boxes of one page
    // (at most 64 rows)
    const long long rows = kv.block_table ? (long long)kv.num_pages * kv.page_size
                                          : (long long)B * Sk;
    const int box = kv.block_table ? (kv.page_size < C::BN ? kv.page_size : C::BN) : C::BN;
    const bool maps = kv.fp8 ? (make_map_u8(&tk, k, rows, Hkv, HD, box) &&
                                make_map_u8(&tv, v, rows, Hkv, HD, box))
                             : (make_map(&tk, k, rows, Hkv, HD, 1, box) &&
                                make_map(&tv, v, rows, Hkv, HD, 1, box));
    if (!maps) return GQA_ERR_CUDA;
    dim3 grid(pl.splits, Hkv * pl.decode_units, B);
    // one instantiation per (paged, e4m3) pair; each raises its own shared-memory limit
    auto launch = [&](auto kernel, int bit, int smem) -> int {
        const int rc = ensure_smem_limit(kernel, bit, smem);
        if (rc != GQA_OK) return rc;
        kernel<<<grid, C::THREADS, smem, stream>>>(tk, tv, p);
        return GQA_OK;
    };
    constexpr int SM8 = gqa::DecodeCfg8<HD>::SMEM_BYTES;
    const int sh = HD == 64 ? 0 : 1;
    int rc = GQA_OK;
    if (kv.fp8)
        rc = kv.block_table ? launch(gqa::decode_split_sm100<HD, true, true>, 256 << sh, SM8)
                            : launch(gqa::decode_split_sm100<HD, false, true>, 64 << sh, SM8);
    else if (kv.block_table)
        rc = launch(gqa::decode_split_sm100<HD, true>, 16 << sh, C::SMEM_BYTES);
    else
        gqa::decode_split_sm100<HD><<<grid, C::THREADS, C::SMEM_BYTES, stream>>>(tk, tv, p);
    if (rc != GQA_OK) return rc;
    if (cudaGetLastError() != cudaSuccess) return GQA_ERR_CUDA;
    if (pl.splits > 1) {
        const int rows_bh = B * Hq;
        const int rc = launch_combine<HD>(p.part_o, p.part_l, p.out, lse, rows_bh, pl.splits, stream);
        if (rc != GQA_OK) return rc;
    }
    return GQA_OK;
}

// Decode against a KV cache (dense with per-sequence lengths, or paged), with an
// optional sliding window.  Sk is the dense cache's keys per sequence (its
// capacity); for the paged form the capacity is max_pages * page_size.
int kvcache_common(const void* q, const void* k, const void* v, void* out, float* lse, int B,
                   int Hq, int Hkv, int Sk, int D, int max_seqlen_k, float scale,
                   const KvCacheArgs& kv, int num_splits, int pack_gqa, cudaStream_t stream) {
    const bool paged = kv.block_table != nullptr;
    if (B < 0 || Sk < 0 || max_seqlen_k < 0 || kv.window < 0) return GQA_ERR_SHAPE;
    if (kv.fp8 && !(std::isfinite(kv.k_scale) && kv.k_scale > 0.f &&
                    std::isfinite(kv.v_scale) && kv.v_scale > 0.f))
        return GQA_ERR_SCALE;
    if (paged) {
        if (kv.page_size < 16 || (kv.page_size & (kv.page_size - 1)) != 0 ||
            kv.num_pages < 1 || kv.max_pages < 1 || !kv.seqlens_k)
            return kv.seqlens_k ? GQA_ERR_SHAPE : GQA_ERR_NULL;
        if ((long long)kv.num_pages * kv.page_size > INT32_MAX ||
            (long long)kv.max_pages * kv.page_size > INT32_MAX)
            return GQA_ERR_SHAPE;
        Sk = kv.max_pages * kv.page_size;  // per-sequence capacity
    }
    if (max_seqlen_k > Sk) return GQA_ERR_SHAPE;
    if (!paged && (long long)B * Sk > INT32_MAX) return GQA_ERR_SHAPE;  // 32-bit TMA rows
    // keys one sequence can touch: its length, or the window plus a partial block
    int keys = kv.seqlens_k ? max_seqlen_k : Sk;
    if (kv.window > 0 && keys > kv.window + 64) keys = kv.window + 64;
    int rc = check_shape(B, Hq, Hkv, 1, keys, D, scale, num_splits, pack_gqa, false, false);
    if (rc != GQA_OK) return rc;
    if (B == 0) return GQA_OK;
    if (!q || !out || !lse || (keys > 0 && (!k || !v))) return GQA_ERR_NULL;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16) ||
        !aligned(lse, 4) || !aligned(kv.seqlens_k, 4) || !aligned(kv.block_table, 4))
        return GQA_ERR_ALIGN;
    DeviceInfo* dev = nullptr;
    rc = device_info(&dev);
    if (rc != GQA_OK) return rc;
    Plan pl;
    make_plan(&pl, B, Hq, Hkv, 1, keys, num_splits, pack_gqa, false, dev->sms);
    if (kv.fp8 && num_splits == 0 && pl.kernel == kDecode) {
        // The e4m3 kernel converts every element, so its rate is set by each SM, not by
        // HBM: two CTAs per SM (they fit) measured faster at every batch size, and the
        // split count is the one with the shortest estimated makespan over those slots:
        // whole waves of equal splits, each split costing its 64-key blocks plus about
        // three blocks of pipeline fill and drain (ties: fewer splits).
        const int n = fp8_decode_splits((long long)B * Hkv * pl.decode_units,
                                        (keys + 63) / 64, 2LL * dev->sms);
        make_plan(&pl, B, Hq, Hkv, 1, keys, n, pack_gqa, false, dev->sms);
    }
    if (pl.kernel == kZeroFill) {
        gqa::fill_no_keys<__nv_bfloat16><<<256, 256, 0, stream>>>(
            static_cast<__nv_bfloat16*>(out), (long long)B * Hq * D, lse, (long long)B * Hq);
        return cudaGetLastError() == cudaSuccess ? GQA_OK : GQA_ERR_CUDA;
    }
    if (pl.kernel != kDecode) return GQA_OK;
    return D == 128 ? launch_decode<128>(q, k, v, out, lse, B, Hq, Hkv, Sk, scale, pl, stream, kv)
                    : launch_decode<64>(q, k, v, out, lse, B, Hq, Hkv, Sk, scale, pl, stream, kv);
}

int fwd_common(const void* q, const void* k, const void* v, void* out, float* lse, int B, int Hq,
               int Hkv, int Sq, int Sk, int D, float scale, int causal, int num_splits,
               int pack_gqa, const int* cu, cudaStream_t stream, bool is_f32) {
    const bool varlen = cu != nullptr;
    int rc = check_shape(B, Hq, Hkv, Sq, Sk, D, scale, num_splits, pack_gqa, varlen, is_f32);
    if (rc != GQA_OK) return rc;
    if (B == 0 || Sq == 0 || (varlen && Sk == 0)) return GQA_OK;  // nothing to compute
    // k and v are never read when there are no keys (dense Sk == 0)
    const bool reads_kv = varlen || Sk > 0;
    if (!q || !out || !lse || (reads_kv && (!k || !v))) return GQA_ERR_NULL;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16) ||
        !aligned(lse, 4) || (cu && !aligned(cu, 4)))
        return GQA_ERR_ALIGN;
    DeviceInfo* dev = nullptr;
    rc = device_info(&dev);
    if (rc != GQA_OK) return rc;

    if (is_f32) {
        if (!varlen && Sk == 0) {
            gqa::fill_no_keys<float><<<256, 256, 0, stream>>>(
                static_cast<float*>(out), (long long)B * Sq * Hq * D, lse, (long long)B * Hq * Sq);
            return cudaGetLastError() == cudaSuccess ? GQA_OK : GQA_ERR_CUDA;
        }
        F32Params p;
        p.q = static_cast<const float*>(q);
        p.k = static_cast<const float*>(k);
        p.v = static_cast<const float*>(v);
        p.out = static_cast<float*>(out);
        p.lse = lse;
        p.cu_seqlens = cu;
        p.B = B;
        p.Hq = Hq;
        p.Hkv = Hkv;
        p.Sq = Sq;
        p.Sk = Sk;
        p.D = D;
        p.G = Hq / Hkv;
        p.causal = causal ? 1 : 0;
        p.scale = scale;
        p.total_rows = varlen ? Sk : 0;
        p.n_rows = varlen ? (long long)Sk * Hq : (long long)B * Sq * Hq;
        const long long blocks = (p.n_rows + 3) / 4;
        if (blocks > INT32_MAX) return GQA_ERR_SHAPE;
        gqa::attn_fwd_f32_simt<<<unsigned(blocks), 128, 0, stream>>>(p);
        return cudaGetLastError() == cudaSuccess ? GQA_OK : GQA_ERR_CUDA;
    }

    Plan pl;
    make_plan(&pl, B, Hq, Hkv, Sq, Sk, num_splits, pack_gqa, varlen, dev->sms);
    switch (pl.kernel) {
        case kNone:
            return GQA_OK;
        case kZeroFill:
            gqa::fill_no_keys<__nv_bfloat16><<<256, 256, 0, stream>>>(
                static_cast<__nv_bfloat16*>(out), (long long)B * Sq * Hq * D, lse,
                (long long)B * Hq * Sq);
            return cudaGetLastError() == cudaSuccess ? GQA_OK : GQA_ERR_CUDA;
        case kDecode:
            return D == 128 ? launch_decode<128>(q, k, v, out, lse, B, Hq, Hkv, Sk, scale, pl,
                                                 stream)
                            : launch_decode<64>(q, k, v, out, lse, B, Hq, Hkv, Sk, scale, pl,
                                                stream);
        default:
            return D == 128 ? launch_prefill<128>(q, k, v, out, lse, B, Hq, Hkv, Sq, Sk, scale,
                                                  causal, pl.pack, cu, dev->sms, stream)
                            : launch_prefill<64>(q, k, v, out, lse, B, Hq, Hkv, Sq, Sk, scale,
                                                 causal, pl.pack, cu, dev->sms, stream);
    }
}

// ---------------------------------------------------------------------------- no-alloc decode
// Scratch for the allocation-free split-KV decode entry point below.  It lives in
// the library image itself, so every GPU that loads the library holds these bytes
// until the process exits; the entry point never asks anyone for memory.
static __device__ __align__(256) unsigned char g_noalloc_scratch[GQA_NOALLOC_SCRATCH_BYTES];

struct NoallocScratch {
    void* ptr = nullptr;  // device address of g_noalloc_scratch on this device
};
NoallocScratch g_noalloc[64];
std::mutex g_noalloc_mu;

// Device address of the scratch array for the current device.  Host code cannot
// use the array's name as an address (on the host it names a stand-in object), so
// the address is asked from the runtime once per device, with that device current.
int noalloc_scratch(void** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return GQA_ERR_CUDA;
    std::lock_guard<std::mutex> lk(g_noalloc_mu);
    if (!g_noalloc[dev].ptr) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return GQA_ERR_CUDA;
        g_noalloc[dev].ptr = p;
    }
    *out = g_noalloc[dev].ptr;
    return GQA_OK;
}

template <int HD>
int launch_decode_noalloc(const void* q, const void* k, const void* v, void* out, float* lse,
                          int B, int Hq, int Hkv, int Sk, float scale, const Plan& pl,
                          void* scratch, cudaStream_t stream) {
    using C = DecodeCfg<HD>;
    if (cudaFuncSetAttribute(gqa::decode_split_sm100<HD>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                             C::SMEM_BYTES) != cudaSuccess)
        return GQA_ERR_CUDA;
    DecodeParams p;
    p.q = static_cast<const __nv_bfloat16*>(q);
    p.out = static_cast<__nv_bfloat16*>(out);
    p.lse = lse;
    p.B = B;
    p.Hq = Hq;
    p.Hkv = Hkv;
    p.Sk = Sk;
    p.G = Hq / Hkv;
    p.rows = pl.decode_rows;
    p.units_per_kv = pl.decode_units;
    p.n_splits = pl.splits;
    p.blocks_per_split = pl.blocks_per_split;
    p.scale_log2 = scale * kLog2e;
    p.part_o = nullptr;
    p.part_l = nullptr;
    if (pl.splits > 1) {
        // same partial layout as the registered-workspace path: O parts, then L parts
        const size_t o_bytes = size_t(B) * Hq * pl.splits * HD * 4;
        p.part_o = static_cast<float*>(scratch);
        p.part_l = reinterpret_cast<float*>(static_cast<char*>(scratch) +
                                            ((o_bytes + 255) / 256) * 256);
    }
    CUtensorMap tk, tv;
    const long long rows = (long long)B * Sk;
    if (!make_map(&tk, k, rows, Hkv, HD, 1, C::BN) || !make_map(&tv, v, rows, Hkv, HD, 1, C::BN))
        return GQA_ERR_CUDA;
    dim3 grid(pl.splits, Hkv * pl.decode_units, B);
    gqa::decode_split_sm100<HD><<<grid, C::THREADS, C::SMEM_BYTES, stream>>>(tk, tv, p);
    if (cudaGetLastError() != cudaSuccess) return GQA_ERR_CUDA;
    if (pl.splits > 1) {
        const int rows_bh = B * Hq;
        const int rc = launch_combine<HD>(p.part_o, p.part_l, p.out, lse, rows_bh, pl.splits, stream);
        if (rc != GQA_OK) return rc;
    }
    return GQA_OK;
}

// ---------------------------------------------------------------------------- self-test
// One warp waits, with the kernels' own bounded wait, on an mbarrier that nothing
// will ever complete; the wait gives up after limit_ns, records the timeout in
// the device error word and the kernel returns normally.
__global__ void selftest_wait_timeout(uint64_t limit_ns) {
    __shared__ __align__(8) uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        gqa::mbar_init(&bar, 1);
        abort_flag = 0;
        gqa::fence_mbar_init();
    }
    __syncthreads();
    gqa::mbar_wait_limit(&bar, 0, &abort_flag, limit_ns);
}

}  // namespace

// ---------------------------------------------------------------------------- host pipeline
// gqa_attn_fwd_host: three library-owned streams per device (copy in, compute, copy
// out) and events that chain them chunk by chunk, created on first use and kept.
constexpr int kMaxChunks = 64;
struct Pipe {
    cudaStream_t s_in = nullptr, s_c = nullptr, s_out = nullptr;
    cudaEvent_t start = nullptr, done = nullptr;
    cudaEvent_t in_done[kMaxChunks] = {};
    cudaEvent_t c_done[kMaxChunks] = {};
    bool ready = false;
};
Pipe g_pipe[64];
std::mutex g_pipe_mu;  // held while a call enqueues, so that its waits see its own records

int pipe_for_device(Pipe** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return GQA_ERR_CUDA;
    Pipe& pp = g_pipe[dev];
    if (!pp.ready) {
        const unsigned ef = cudaEventDisableTiming;
        if (cudaStreamCreateWithFlags(&pp.s_in, cudaStreamNonBlocking) != cudaSuccess ||
            cudaStreamCreateWithFlags(&pp.s_c, cudaStreamNonBlocking) != cudaSuccess ||
            cudaStreamCreateWithFlags(&pp.s_out, cudaStreamNonBlocking) != cudaSuccess ||
            cudaEventCreateWithFlags(&pp.start, ef) != cudaSuccess ||
            cudaEventCreateWithFlags(&pp.done, ef) != cudaSuccess)
            return GQA_ERR_CUDA;
        for (int c = 0; c < kMaxChunks; ++c)
            if (cudaEventCreateWithFlags(&pp.in_done[c], ef) != cudaSuccess ||
                cudaEventCreateWithFlags(&pp.c_done[c], ef) != cudaSuccess)
                return GQA_ERR_CUDA;
        pp.ready = true;
    }
    *out = &pp;
    return GQA_OK;
}

extern "C" {

int gqa_attn_fwd(const void* q, const void* k, const void* v, void* out, float* lse, int B,
                 int Hq, int Hkv, int Sq, int Sk, int D, float scale, int causal,
                 int num_splits, int pack_gqa, const int* cu_seqlens, cudaStream_t stream) {
    return fwd_common(q, k, v, out, lse, B, Hq, Hkv, Sq, Sk, D, scale, causal, num_splits,
                      pack_gqa, cu_seqlens, stream, false);
}

int gqa_attn_fwd_window(const void* q, const void* k, const void* v, void* out, float* lse,
                        int B, int Hq, int Hkv, int Sq, int Sk, int D, float scale, int window,
                        int pack_gqa, const int* cu_seqlens, cudaStream_t stream) {
    const bool varlen = cu_seqlens != nullptr;
    int rc = check_shape(B, Hq, Hkv, Sq, Sk, D, scale, 1, pack_gqa, varlen, false);
    if (rc != GQA_OK) return rc;
    if (window < 1) return GQA_ERR_SHAPE;
    // a window that holds every key is plain causal attention
    if (window >= (varlen ? Sq : Sk))
        return fwd_common(q, k, v, out, lse, B, Hq, Hkv, Sq, Sk, D, scale, 1, 1, pack_gqa,
                          cu_seqlens, stream, false);
    if (!varlen && Sq == 1) {
        // one query: the decode kernel's window over a dense cache of Sk keys
        KvCacheArgs kv;
        kv.window = window;
        return kvcache_common(q, k, v, out, lse, B, Hq, Hkv, Sk, D, Sk, scale, kv, 1, pack_gqa,
                              stream);
    }
    if (B == 0 || Sq == 0) return GQA_OK;
    if (!q || !k || !v || !out || !lse) return GQA_ERR_NULL;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16) ||
        !aligned(lse, 4) || (varlen && !aligned(cu_seqlens, 4)))
        return GQA_ERR_ALIGN;
    DeviceInfo* dev = nullptr;
    rc = device_info(&dev);
    if (rc != GQA_OK) return rc;
    Plan pl;
    make_plan(&pl, B, Hq, Hkv, Sq, Sk, 1, pack_gqa, varlen, dev->sms);
    if (pl.kernel == kNone) return GQA_OK;
    return D == 128 ? launch_prefill<128>(q, k, v, out, lse, B, Hq, Hkv, Sq, Sk, scale, 1,
                                          pl.pack, cu_seqlens, dev->sms, stream, nullptr,
                                          nullptr, nullptr, nullptr, 0, 0, 1.f, 1.f, window)
                    : launch_prefill<64>(q, k, v, out, lse, B, Hq, Hkv, Sq, Sk, scale, 1,
                                         pl.pack, cu_seqlens, dev->sms, stream, nullptr,
                                         nullptr, nullptr, nullptr, 0, 0, 1.f, 1.f, window);
}

int gqa_attn_fwd_host(const void* q_h, const void* k_h, const void* v_h, void* out_h,
                      float* lse_h, void* q_d, void* k_d, void* v_d, void* out_d, float* lse_d,
                      int B, int Hq, int Hkv, int Sq, int Sk, int D, float scale, int causal,
                      int num_splits, int pack_gqa, int chunks, cudaStream_t stream) {
    int rc = check_shape(B, Hq, Hkv, Sq, Sk, D, scale, num_splits, pack_gqa, false, false);
    if (rc != GQA_OK) return rc;
    if (chunks < 0 || chunks > kMaxChunks) return GQA_ERR_SHAPE;
    if (B == 0 || Sq == 0) return GQA_OK;
    const bool reads_kv = Sk > 0;
    if (!q_h || !out_h || !lse_h || !q_d || !out_d || !lse_d ||
        (reads_kv && (!k_h || !v_h || !k_d || !v_d)))
        return GQA_ERR_NULL;
    DeviceInfo* dev = nullptr;
    rc = device_info(&dev);
    if (rc != GQA_OK) return rc;
    std::lock_guard<std::mutex> lk(g_pipe_mu);
    Pipe* pp = nullptr;
    rc = pipe_for_device(&pp);
    if (rc != GQA_OK) return rc;
    const int want = chunks == 0 ? 8 : chunks;
    const size_t qb = size_t(Sq) * Hq * D * 2, kb = size_t(Sk) * Hkv * D * 2;
    const size_t lb = size_t(Hq) * Sq * 4;
    auto at = [](const void* base, size_t off) {
        return static_cast<void*>(static_cast<char*>(const_cast<void*>(base)) + off);
    };
    // Fewer batch elements than chunks: a prefill (not a decode step, keys at least as
    // many as queries when causal) is cut into ranges of query positions of each batch
    // element instead.  Queries [s0, s1) see the key prefix [0, e(s1)) (e(s) = s + Sk - Sq
    // when causal, Sk otherwise), so a chunk copies in only the keys the previous
    // chunks of its batch element did not, and runs as a problem of its own with
    // bottom-right alignment: every row computes what the whole launch computes.
    int per_b = B < want ? (want + B - 1) / B : 1;
    if (per_b > kMaxChunks / B) per_b = kMaxChunks / B;
    const bool by_pos = per_b > 1 && Sq >= 512 && Sk > 0 && (!causal || Sq <= Sk);
    if (by_pos && (!aligned(q_d, 16) || !aligned(k_d, 16) || !aligned(v_d, 16) ||
                   !aligned(out_d, 16) || !aligned(lse_d, 4)))
        return GQA_ERR_ALIGN;
    if (cudaEventRecord(pp->start, stream) != cudaSuccess ||
        cudaStreamWaitEvent(pp->s_in, pp->start, 0) != cudaSuccess ||
        cudaStreamWaitEvent(pp->s_c, pp->start, 0) != cudaSuccess ||
        cudaStreamWaitEvent(pp->s_out, pp->start, 0) != cudaSuccess)
        return GQA_ERR_CUDA;
    int status = GQA_OK;
    if (by_pos) {
        int len = (Sq + per_b - 1) / per_b;
        len = (len + 255) / 256 * 256;  // whole 256-row tiles for every group size
        const int cpb = (Sq + len - 1) / len;  // <= per_b, so B * cpb <= kMaxChunks
        const size_t qrow = size_t(Hq) * D * 2, krow = size_t(Hkv) * D * 2;
        for (int b = 0; b < B && status == GQA_OK; ++b) {
            int kdone = 0;  // keys of batch element b already copied in
            for (int j = 0; j < cpb && status == GQA_OK; ++j) {
                const int c = b * cpb + j;
                const int s0 = j * len, s1 = (s0 + len < Sq) ? s0 + len : Sq;
                const int kend = causal ? s1 + (Sk - Sq) : Sk;
                const size_t oq = size_t(b) * qb + size_t(s0) * qrow;
                const size_t okb = size_t(b) * kb;
                const size_t ok = okb + size_t(kdone) * krow;
                const size_t nk = size_t(kend - kdone) * krow;
                if (cudaMemcpyAsync(at(q_d, oq), at(q_h, oq), size_t(s1 - s0) * qrow,
                                    cudaMemcpyHostToDevice, pp->s_in) != cudaSuccess ||
                    (nk && (cudaMemcpyAsync(at(k_d, ok), at(k_h, ok), nk,
                                            cudaMemcpyHostToDevice, pp->s_in) != cudaSuccess ||
                            cudaMemcpyAsync(at(v_d, ok), at(v_h, ok), nk,
                                            cudaMemcpyHostToDevice, pp->s_in) != cudaSuccess)) ||
                    cudaEventRecord(pp->in_done[c], pp->s_in) != cudaSuccess ||
                    cudaStreamWaitEvent(pp->s_c, pp->in_done[c], 0) != cudaSuccess) {
                    status = GQA_ERR_CUDA;
                    break;
                }
                kdone = kend;
                Plan pl;
                make_plan(&pl, 1, Hq, Hkv, s1 - s0, kend, 1, pack_gqa, false, dev->sms);
                float* lse_c = lse_d + size_t(b) * Hq * Sq + s0;
                status = D == 128
                             ? launch_prefill<128>(at(q_d, oq), at(k_d, okb), at(v_d, okb),
                                                   at(out_d, oq), lse_c, 1, Hq, Hkv, s1 - s0,
                                                   kend, scale, causal, pl.pack, nullptr,
                                                   dev->sms, pp->s_c, nullptr, nullptr,
                                                   nullptr, nullptr, 0, 0, 1.f, 1.f, 0, Sq)
                             : launch_prefill<64>(at(q_d, oq), at(k_d, okb), at(v_d, okb),
                                                  at(out_d, oq), lse_c, 1, Hq, Hkv, s1 - s0,
                                                  kend, scale, causal, pl.pack, nullptr,
                                                  dev->sms, pp->s_c, nullptr, nullptr, nullptr,
                                                  nullptr, 0, 0, 1.f, 1.f, 0, Sq);
                if (status != GQA_OK) break;
                // O rows of the range are contiguous; L is Hq rows of s1 - s0 values
                float* lse_hc = lse_h + size_t(b) * Hq * Sq + s0;
                if (cudaEventRecord(pp->c_done[c], pp->s_c) != cudaSuccess ||
                    cudaStreamWaitEvent(pp->s_out, pp->c_done[c], 0) != cudaSuccess ||
                    cudaMemcpyAsync(at(out_h, oq), at(out_d, oq), size_t(s1 - s0) * qrow,
                                    cudaMemcpyDeviceToHost, pp->s_out) != cudaSuccess ||
                    cudaMemcpy2DAsync(lse_hc, size_t(Sq) * 4, lse_c, size_t(Sq) * 4,
                                      size_t(s1 - s0) * 4, Hq, cudaMemcpyDeviceToHost,
                                      pp->s_out) != cudaSuccess)
                    status = GQA_ERR_CUDA;
            }
        }
    }
    // otherwise chunks of whole batch elements: [B, S, H, D] and [B, H, S] are batch-major
    int n = want;
    if (n > B) n = B;
    const int per = (B + n - 1) / n;
    n = by_pos ? 0 : (B + per - 1) / per;
    for (int c = 0; c < n && status == GQA_OK; ++c) {
        const int b0 = c * per, nb = (B - b0 < per) ? B - b0 : per;
        const size_t oq = size_t(b0) * qb, ok = size_t(b0) * kb, ol = size_t(b0) * lb;
        if (cudaMemcpyAsync(at(q_d, oq), at(q_h, oq), nb * qb, cudaMemcpyHostToDevice,
                            pp->s_in) != cudaSuccess ||
            (reads_kv && (cudaMemcpyAsync(at(k_d, ok), at(k_h, ok), nb * kb,
                                          cudaMemcpyHostToDevice, pp->s_in) != cudaSuccess ||
                          cudaMemcpyAsync(at(v_d, ok), at(v_h, ok), nb * kb,
                                          cudaMemcpyHostToDevice, pp->s_in) != cudaSuccess)) ||
            cudaEventRecord(pp->in_done[c], pp->s_in) != cudaSuccess ||
            cudaStreamWaitEvent(pp->s_c, pp->in_done[c], 0) != cudaSuccess) {
            status = GQA_ERR_CUDA;
            break;
        }
        status = fwd_common(at(q_d, oq), reads_kv ? at(k_d, ok) : nullptr,
                            reads_kv ? at(v_d, ok) : nullptr, at(out_d, oq),
                            static_cast<float*>(at(lse_d, ol)), nb, Hq, Hkv, Sq, Sk, D, scale,
                            causal, num_splits, pack_gqa, nullptr, pp->s_c, false);
        if (status != GQA_OK) break;
        if (cudaEventRecord(pp->c_done[c], pp->s_c) != cudaSuccess ||
            cudaStreamWaitEvent(pp->s_out, pp->c_done[c], 0) != cudaSuccess ||
            cudaMemcpyAsync(at(out_h, oq), at(out_d, oq), nb * qb, cudaMemcpyDeviceToHost,
                            pp->s_out) != cudaSuccess ||
            cudaMemcpyAsync(at(lse_h, ol), at(lse_d, ol), nb * lb, cudaMemcpyDeviceToHost,
                            pp->s_out) != cudaSuccess)
            status = GQA_ERR_CUDA;
    }
    // whatever was enqueued (all of it, also after an error) finishes before later
    // work on the caller's stream: join the copy-in and compute streams into copy-out
    cudaEvent_t tail_c = pp->c_done[0];
    if (cudaEventRecord(tail_c, pp->s_c) != cudaSuccess ||
        cudaStreamWaitEvent(pp->s_out, tail_c, 0) != cudaSuccess ||
        cudaEventRecord(pp->in_done[0], pp->s_in) != cudaSuccess ||
        cudaStreamWaitEvent(pp->s_out, pp->in_done[0], 0) != cudaSuccess ||
        cudaEventRecord(pp->done, pp->s_out) != cudaSuccess ||
        cudaStreamWaitEvent(stream, pp->done, 0) != cudaSuccess)
        status = status == GQA_OK ? GQA_ERR_CUDA : status;
    return status;
}

int gqa_attn_fwd_f32(const void* q, const void* k, const void* v, void* out, float* lse, int B,
                     int Hq, int Hkv, int Sq, int Sk, int D, float scale, int causal,
                     int num_splits, int pack_gqa, const int* cu_seqlens, cudaStream_t stream) {
    return fwd_common(q, k, v, out, lse, B, Hq, Hkv, Sq, Sk, D, scale, causal, num_splits,
                      pack_gqa, cu_seqlens, stream, true);
}

size_t gqa_attn_workspace_bytes(int B, int Hq, int Sq, int D, int num_splits) {
    if (B <= 0 || Hq <= 0 || Sq <= 0 || D <= 0 || num_splits <= 1) return 0;
    return ws_bytes(B, Hq, Sq, D, num_splits);
}

int gqa_attn_fwd_host_varlen(const void* q_h, const void* k_h, const void* v_h, void* out_h,
                             float* lse_h, void* q_d, void* k_d, void* v_d, void* out_d,
                             float* lse_d, const int* cu_seqlens_h, const int* cu_seqlens_d,
                             int B, int Hq, int Hkv, int max_seqlen, int total, int D,
                             float scale, int causal, int pack_gqa, int chunks,
                             cudaStream_t stream) {
    int rc = check_shape(B, Hq, Hkv, max_seqlen, total, D, scale, 1, pack_gqa, true, false);
    if (rc != GQA_OK) return rc;
    if (chunks < 0 || chunks > kMaxChunks) return GQA_ERR_SHAPE;
    if (B == 0 || max_seqlen == 0 || total == 0) return GQA_OK;
    if (!cu_seqlens_h || !cu_seqlens_d || !q_h || !k_h || !v_h || !out_h || !lse_h || !q_d ||
        !k_d || !v_d || !out_d || !lse_d)
        return GQA_ERR_NULL;
    // the host offsets must describe the packed rows: 0 = cu[0] <= ... <= cu[B] = total,
    // no sequence longer than max_seqlen
    if (cu_seqlens_h[0] != 0 || cu_seqlens_h[B] != total) return GQA_ERR_SHAPE;
    for (int b = 0; b < B; ++b) {
        const int len = cu_seqlens_h[b + 1] - cu_seqlens_h[b];
        if (len < 0 || len > max_seqlen) return GQA_ERR_SHAPE;
    }
    DeviceInfo* dev = nullptr;
    rc = device_info(&dev);
    if (rc != GQA_OK) return rc;
    std::lock_guard<std::mutex> lk(g_pipe_mu);
    Pipe* pp = nullptr;
    rc = pipe_for_device(&pp);
    if (rc != GQA_OK) return rc;
    const int n_target = chunks == 0 ? 8 : chunks;
    const long long target = ((long long)total + n_target - 1) / n_target;
    const size_t qrow = size_t(Hq) * D * 2, krow = size_t(Hkv) * D * 2;
    auto at = [](const void* base, size_t off) {
        return static_cast<void*>(static_cast<char*>(const_cast<void*>(base)) + off);
    };
    if (cudaEventRecord(pp->start, stream) != cudaSuccess ||
        cudaStreamWaitEvent(pp->s_in, pp->start, 0) != cudaSuccess ||
        cudaStreamWaitEvent(pp->s_c, pp->start, 0) != cudaSuccess ||
        cudaStreamWaitEvent(pp->s_out, pp->start, 0) != cudaSuccess)
        return GQA_ERR_CUDA;
    int status = GQA_OK;
    int s0 = 0, c = 0;
    while (s0 < B && status == GQA_OK) {
        // whole sequences until the chunk holds about total / chunks rows
        int s1 = s0 + 1;
        while (s1 < B && (long long)cu_seqlens_h[s1] - cu_seqlens_h[s0] < target &&
               B - s1 > 0 && c + 1 < kMaxChunks)
            ++s1;
        if (c + 1 == kMaxChunks) s1 = B;  // the last event pair takes the rest
        const int r0 = cu_seqlens_h[s0], r1 = cu_seqlens_h[s1];
        int len_max = 0;
        for (int b = s0; b < s1; ++b)
            len_max = std::max(len_max, cu_seqlens_h[b + 1] - cu_seqlens_h[b]);
        const size_t rows = size_t(r1 - r0);
        if (rows > 0 &&
            (cudaMemcpyAsync(at(q_d, r0 * qrow), at(q_h, r0 * qrow), rows * qrow,
                             cudaMemcpyHostToDevice, pp->s_in) != cudaSuccess ||
             cudaMemcpyAsync(at(k_d, r0 * krow), at(k_h, r0 * krow), rows * krow,
                             cudaMemcpyHostToDevice, pp->s_in) != cudaSuccess ||
             cudaMemcpyAsync(at(v_d, r0 * krow), at(v_h, r0 * krow), rows * krow,
                             cudaMemcpyHostToDevice, pp->s_in) != cudaSuccess)) {
            status = GQA_ERR_CUDA;
            break;
        }
        if (cudaEventRecord(pp->in_done[c], pp->s_in) != cudaSuccess ||
            cudaStreamWaitEvent(pp->s_c, pp->in_done[c], 0) != cudaSuccess) {
            status = GQA_ERR_CUDA;
            break;
        }
        // the chunk's sequences, addressed through the full buffers and the offsets
        if (len_max > 0) {
            status = fwd_common(q_d, k_d, v_d, out_d, lse_d, s1 - s0, Hq, Hkv, len_max, total, D,
                                scale, causal, 1, pack_gqa, cu_seqlens_d + s0, pp->s_c, false);
            if (status != GQA_OK) break;
        }
        if (cudaEventRecord(pp->c_done[c], pp->s_c) != cudaSuccess ||
            cudaStreamWaitEvent(pp->s_out, pp->c_done[c], 0) != cudaSuccess ||
            (rows > 0 &&
             (cudaMemcpyAsync(at(out_h, r0 * qrow), at(out_d, r0 * qrow), rows * qrow,
                              cudaMemcpyDeviceToHost, pp->s_out) != cudaSuccess ||
              cudaMemcpy2DAsync(lse_h + r0, size_t(total) * 4, lse_d + r0, size_t(total) * 4,
                                rows * 4, size_t(Hq), cudaMemcpyDeviceToHost,
                                pp->s_out) != cudaSuccess)))
            status = GQA_ERR_CUDA;
        s0 = s1;
        ++c;
    }
    cudaEvent_t tail_c = pp->c_done[0];
    if (cudaEventRecord(tail_c, pp->s_c) != cudaSuccess ||
        cudaStreamWaitEvent(pp->s_out, tail_c, 0) != cudaSuccess ||
        cudaEventRecord(pp->in_done[0], pp->s_in) != cudaSuccess ||
        cudaStreamWaitEvent(pp->s_out, pp->in_done[0], 0) != cudaSuccess ||
        cudaEventRecord(pp->done, pp->s_out) != cudaSuccess ||
        cudaStreamWaitEvent(stream, pp->done, 0) != cudaSuccess)
        status = status == GQA_OK ? GQA_ERR_CUDA : status;
    return status;
}

int gqa_attn_set_workspace(void* dev_ptr, size_t bytes) {
    if (dev_ptr && !aligned(dev_ptr, 16)) return GQA_ERR_ALIGN;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64)
        return dev_ptr ? GQA_ERR_CUDA : GQA_OK;  // no device: nothing is registered
    std::lock_guard<std::mutex> lk(g_mu);
    g_ws[dev].ptr = bytes ? dev_ptr : nullptr;
    g_ws[dev].bytes = dev_ptr ? bytes : 0;
    return GQA_OK;
}

int gqa_attn_plan(int B, int Hq, int Hkv, int Sq, int Sk, int D, float scale, int causal,
                  int num_splits, int pack_gqa, int varlen, int* kernel, int* splits, int* pack) {
    (void)causal;
    int rc = check_shape(B, Hq, Hkv, Sq, Sk, D, scale, num_splits, pack_gqa, varlen != 0, false);
    if (rc != GQA_OK) return rc;
    DeviceInfo* dev = nullptr;
    rc = device_info(&dev);
    const int sms = (dev && dev->sms > 0) ? dev->sms : 148;
    Plan pl;
    make_plan(&pl, B, Hq, Hkv, Sq, Sk, num_splits, pack_gqa, varlen != 0, sms);
    if (kernel) *kernel = pl.kernel;
    if (splits) *splits = pl.splits;
    if (pack) *pack = pl.pack;
    return rc;
}

int gqa_attn_get_device_error(int* host_code, cudaStream_t stream) {
    if (!host_code) return GQA_ERR_NULL;
    int code = 0;
    if (cudaMemcpyFromSymbolAsync(&code, gqa::g_device_error, sizeof(int), 0,
                                  cudaMemcpyDeviceToHost, stream) != cudaSuccess)
        return GQA_ERR_CUDA;
    if (cudaStreamSynchronize(stream) != cudaSuccess) return GQA_ERR_CUDA;
    const int zero = 0;
    if (cudaMemcpyToSymbolAsync(gqa::g_device_error, &zero, sizeof(int), 0,
                                cudaMemcpyHostToDevice, stream) != cudaSuccess)
        return GQA_ERR_CUDA;
    if (cudaStreamSynchronize(stream) != cudaSuccess) return GQA_ERR_CUDA;
    *host_code = code;
    return GQA_OK;
}

const char* gqa_attn_strerror(int code) {
    switch (code) {
        case GQA_OK: return "success";
        case GQA_ERR_NULL: return "a required pointer is NULL";
        case GQA_ERR_SHAPE: return "invalid shape (negative size, Hq % Hkv != 0, or varlen Sq != Sk)";
        case GQA_ERR_HEADDIM: return "unsupported head dimension";
        case GQA_ERR_ALIGN: return "pointer not aligned (tensors 16 bytes, lse 4 bytes)";
        case GQA_ERR_SPLITS: return "invalid num_splits for this shape";
        case GQA_ERR_WORKSPACE: return "split-KV workspace missing or too small";
        case GQA_ERR_SCALE: return "scale must be finite and positive";
        case GQA_ERR_CUDA: return "CUDA runtime or launch failure";
        case GQA_ERR_UNSUPPORTED: return "unsupported device or pack_gqa value";
        default: return "unknown status";
    }
}


// Split-KV decode that allocates nothing: its partial results go to the library's
// static scratch array instead of a registered workspace.  See gqa_attn.h.
int gqa_attn_decode_noalloc(const void* q, const void* k, const void* v, void* out,
                            float* lse, int B, int Hq, int Hkv, int Sk, int D, float scale,
                            int num_splits, int pack_gqa, cudaStream_t stream) {
    int rc = check_shape(B, Hq, Hkv, 1, Sk, D, scale, num_splits, pack_gqa, false, false);
    if (rc != GQA_OK) return rc;
    if (B == 0) return GQA_OK;
    const bool reads_kv = Sk > 0;
    if (!q || !out || !lse || (reads_kv && (!k || !v))) return GQA_ERR_NULL;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16) ||
        !aligned(lse, 4))
        return GQA_ERR_ALIGN;
    DeviceInfo* dev = nullptr;
    rc = device_info(&dev);
    if (rc != GQA_OK) return rc;
    if (Sk == 0) {
        gqa::fill_no_keys<__nv_bfloat16><<<256, 256, 0, stream>>>(
            static_cast<__nv_bfloat16*>(out), (long long)B * Hq * D, lse, (long long)B * Hq);
        return cudaGetLastError() == cudaSuccess ? GQA_OK : GQA_ERR_CUDA;
    }
    Plan pl;
    make_plan(&pl, B, Hq, Hkv, 1, Sk, num_splits, pack_gqa, false, dev->sms);
    if (num_splits == 0) {
        // automatic choice: the planned count puts at most one CTA on each SM, whose
        // partials (at most SMs x 16 rows) fit the static scratch on a 148-SM part; this
        // step-down is a guard for parts with more SMs (one split needs no scratch)
        while (pl.splits > 1 && ws_bytes(B, Hq, 1, D, pl.splits) > GQA_NOALLOC_SCRATCH_BYTES) {
            Plan smaller;
            make_plan(&smaller, B, Hq, Hkv, 1, Sk, pl.splits - 1, pack_gqa, false, dev->sms);
            pl = smaller;
        }
    }
    if (ws_bytes(B, Hq, 1, D, pl.splits) > GQA_NOALLOC_SCRATCH_BYTES) return GQA_ERR_WORKSPACE;
    void* scratch = nullptr;
    rc = noalloc_scratch(&scratch);
    if (rc != GQA_OK) return rc;
    return D == 128 ? launch_decode_noalloc<128>(q, k, v, out, lse, B, Hq, Hkv, Sk, scale, pl,
                                                 scratch, stream)
                    : launch_decode_noalloc<64>(q, k, v, out, lse, B, Hq, Hkv, Sk, scale, pl,
                                                scratch, stream);
}


int gqa_attn_fwd_blocksparse(const void* q, const void* k, const void* v, void* out, float* lse,
                             int B, int Hq, int Hkv, int Sq, int Sk, int D, float scale,
                             int causal, const int* blk_row_ptr, const int* blk_col,
                             cudaStream_t stream) {
    int rc = check_shape(B, Hq, Hkv, Sq, Sk, D, scale, 1, 1, false, false);
    if (rc != GQA_OK) return rc;
    const int G = Hq / Hkv;
    // a CTA tile (2 x 128 / G positions) must lie inside one 128-position query block
    if (G < 2 || 128 % G != 0) return GQA_ERR_UNSUPPORTED;
    if (B == 0 || Sq == 0) return GQA_OK;
    if (!q || !out || !lse || !blk_row_ptr || !blk_col || (Sk > 0 && (!k || !v)))
        return GQA_ERR_NULL;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16) ||
        !aligned(lse, 4) || !aligned(blk_row_ptr, 4) || !aligned(blk_col, 4))
        return GQA_ERR_ALIGN;
    DeviceInfo* dev = nullptr;
    rc = device_info(&dev);
    if (rc != GQA_OK) return rc;
    if (Sk == 0) {
        gqa::fill_no_keys<__nv_bfloat16><<<256, 256, 0, stream>>>(
            static_cast<__nv_bfloat16*>(out), (long long)B * Sq * Hq * D, lse,
            (long long)B * Hq * Sq);
        return cudaGetLastError() == cudaSuccess ? GQA_OK : GQA_ERR_CUDA;
    }
    const int cz = causal ? 1 : 0;
    return D == 128 ? launch_prefill<128>(q, k, v, out, lse, B, Hq, Hkv, Sq, Sk, scale, cz, 1,
                                          nullptr, dev->sms, stream, blk_row_ptr, blk_col)
                    : launch_prefill<64>(q, k, v, out, lse, B, Hq, Hkv, Sq, Sk, scale, cz, 1,
                                         nullptr, dev->sms, stream, blk_row_ptr, blk_col);
}

int gqa_attn_fwd_fp8(const void* q8, const void* k8, const void* v8, void* out, float* lse,
                     int B, int Hq, int Hkv, int Sq, int Sk, int D, float scale, float q_scale,
                     float k_scale, float v_scale, int causal, const int* cu_seqlens,
                     cudaStream_t stream) {
    const bool varlen = cu_seqlens != nullptr;
    int rc = check_shape(B, Hq, Hkv, Sq, Sk, D, scale, 1, -1, varlen, false);
    if (rc != GQA_OK) return rc;
    if (D != 128) return GQA_ERR_HEADDIM;
    if (!(std::isfinite(q_scale) && q_scale > 0.f && std::isfinite(k_scale) && k_scale > 0.f &&
          std::isfinite(v_scale) && v_scale > 0.f))
        return GQA_ERR_SCALE;
    if (B == 0 || Sq == 0 || (varlen && Sk == 0)) return GQA_OK;
    const bool reads_kv = varlen || Sk > 0;
    if (!q8 || !out || !lse || (reads_kv && (!k8 || !v8))) return GQA_ERR_NULL;
    if (!aligned(q8, 16) || !aligned(k8, 16) || !aligned(v8, 16) || !aligned(out, 16) ||
        !aligned(lse, 4) || (varlen && !aligned(cu_seqlens, 4)))
        return GQA_ERR_ALIGN;
    DeviceInfo* dev = nullptr;
    rc = device_info(&dev);
    if (rc != GQA_OK) return rc;
    if (!varlen && Sk == 0) {
        gqa::fill_no_keys<__nv_bfloat16><<<256, 256, 0, stream>>>(
            static_cast<__nv_bfloat16*>(out), (long long)B * Sq * Hq * D, lse,
            (long long)B * Hq * Sq);
        return cudaGetLastError() == cudaSuccess ? GQA_OK : GQA_ERR_CUDA;
    }
    Plan pl;
    make_plan(&pl, B, Hq, Hkv, Sq, Sk, 1, -1, varlen, dev->sms);
    return launch_prefill<128, true>(q8, k8, v8, out, lse, B, Hq, Hkv, Sq, Sk, scale, causal,
                                     pl.pack, cu_seqlens, dev->sms, stream, nullptr, nullptr,
                                     nullptr, nullptr, 0, 0, q_scale * k_scale, v_scale);
}

int gqa_attn_sparse_varlen_schedule(const int* cu_seqlens, const int* blk_row_ptr, int B,
                                    int Hq, int Hkv, int max_seqlen, int grid, int* blk_off,
                                    int* order, int order_cap, int* n_order, int* order_grid) {
    if (!cu_seqlens || !blk_row_ptr || !blk_off || !n_order || !order_grid || B < 0 ||
        Hq <= 0 || Hkv <= 0 ||
        Hq % Hkv != 0 || max_seqlen < 0 || grid <= 0 || order_cap < 0 || (order_cap && !order))
        return GQA_ERR_NULL;
    const int G = Hq / Hkv;
    if (G < 2 || 128 % G != 0) return GQA_ERR_UNSUPPORTED;
    // minimum padding: sequence b owns ceil(n_b / 128) pattern rows, after the earlier ones
    blk_off[0] = 0;
    for (int b = 0; b < B; ++b) {
        const int n = cu_seqlens[b + 1] - cu_seqlens[b];
        if (n < 0 || n > max_seqlen) return GQA_ERR_SHAPE;
        blk_off[b + 1] = blk_off[b] + (n + 127) / 128;
    }
    // units (b, kv head, m) as the kernel linearises them; cost = key blocks of the row
    // times the sub-tiles that hold positions, plus one block for the tile's fixed work
    const int sub = 128 / G, n_mblk = (max_seqlen + 2 * sub - 1) / (2 * sub);
    struct Unit { long long cost; int u; };
    std::vector<Unit> units;
    for (int b = 0; b < B; ++b) {
        const int n = cu_seqlens[b + 1] - cu_seqlens[b];
        for (int m = 0; m < n_mblk; ++m) {
            const int p0 = m * 2 * sub;
            if (p0 >= n) break;
            const int qb = blk_off[b] + p0 / 128;
            const int row = blk_row_ptr[qb + 1] - blk_row_ptr[qb];
            if (row < 0) return GQA_ERR_SHAPE;
            const int subs = 1 + (p0 + sub < n ? 1 : 0);
            for (int h = 0; h < Hkv; ++h)
                units.push_back({(long long)row * subs + 1, (b * Hkv + h) * n_mblk + m});
        }
    }
    // longest processing time first: each unit goes to the CTA with the least work so far
    std::stable_sort(units.begin(), units.end(),
                     [](const Unit& a, const Unit& c) { return a.cost > c.cost; });
    const int g = (int)std::min<size_t>((size_t)grid, std::max<size_t>(units.size(), 1));
    std::vector<std::vector<int>> lists(g);
    using Load = std::pair<long long, int>;
    std::priority_queue<Load, std::vector<Load>, std::greater<Load>> heap;
    for (int c = 0; c < g; ++c) heap.push({0, c});
    for (const Unit& x : units) {
        Load top = heap.top();
        heap.pop();
        lists[top.second].push_back(x.u);
        heap.push({top.first + x.cost, top.second});
    }
    size_t depth = 0;
    for (const auto& l : lists) depth = std::max(depth, l.size());
    const long long need = (long long)g * (long long)depth;
    if (need > INT32_MAX) return GQA_ERR_SHAPE;
    *n_order = (int)need;
    *order_grid = g;
    if (need > order_cap) return GQA_ERR_WORKSPACE;  // *n_order says how many entries
    // CTA c takes steps c, c + g, c + 2 g, ... of the persistent loop
    for (size_t k = 0; k < depth; ++k)
        for (int c = 0; c < g; ++c)
            order[k * g + c] = k < lists[c].size() ? lists[c][k] : -1;
    return GQA_OK;
}

int gqa_attn_fwd_blocksparse_varlen(const void* q, const void* k, const void* v, void* out,
                                    float* lse, const int* cu_seqlens, const int* blk_off,
                                    int B, int Hq, int Hkv, int max_seqlen, int total, int D,
                                    float scale, int causal, const int* blk_row_ptr,
                                    const int* blk_col,
                                    const int* tile_order, int n_order, int order_grid,
                                    cudaStream_t stream) {
    int rc = check_shape(B, Hq, Hkv, max_seqlen, total, D, scale, 1, 1, true, false);
    if (rc != GQA_OK) return rc;
    const int G = Hq / Hkv;
    if (G < 2 || 128 % G != 0) return GQA_ERR_UNSUPPORTED;
    if (B == 0 || max_seqlen == 0 || total == 0) return GQA_OK;
    if (!q || !k || !v || !out || !lse || !cu_seqlens || !blk_off || !blk_row_ptr || !blk_col)
        return GQA_ERR_NULL;
    if (tile_order && (n_order <= 0 || order_grid <= 0 || n_order % order_grid != 0))
        return GQA_ERR_SHAPE;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16) ||
        !aligned(lse, 4) || !aligned(blk_row_ptr, 4) || !aligned(blk_col, 4) ||
        !aligned(cu_seqlens, 4) || !aligned(blk_off, 4) || !aligned(tile_order, 4))
        return GQA_ERR_ALIGN;
    DeviceInfo* dev = nullptr;
    rc = device_info(&dev);
    if (rc != GQA_OK) return rc;
    return D == 128 ? launch_prefill<128>(q, k, v, out, lse, B, Hq, Hkv, max_seqlen, total,
                                          scale, causal ? 1 : 0, 1, cu_seqlens, dev->sms, stream,
                                          blk_row_ptr, blk_col, blk_off, tile_order, n_order,
                                          order_grid)
                    : launch_prefill<64>(q, k, v, out, lse, B, Hq, Hkv, max_seqlen, total,
                                         scale, causal ? 1 : 0, 1, cu_seqlens, dev->sms, stream,
                                         blk_row_ptr, blk_col, blk_off, tile_order, n_order,
                                         order_grid);
}

int gqa_attn_decode_kvcache(const void* q, const void* k_cache, const void* v_cache,
                            const int* seqlens_k, void* out, float* lse, int B, int Hq, int Hkv,
                            int Sk, int D, int max_seqlen_k, float scale, int window,
                            int num_splits, int pack_gqa, cudaStream_t stream) {
    KvCacheArgs kv;
    kv.seqlens_k = seqlens_k;
    kv.window = window;
    return kvcache_common(q, k_cache, v_cache, out, lse, B, Hq, Hkv, Sk, D,
                          seqlens_k ? max_seqlen_k : Sk, scale, kv, num_splits, pack_gqa, stream);
}

int gqa_attn_decode_paged(const void* q, const void* k_pages, const void* v_pages,
                          const int* block_table, const int* seqlens_k, void* out, float* lse,
                          int B, int Hq, int Hkv, int D, int num_pages, int page_size,
                          int max_pages, int max_seqlen_k, float scale, int window,
                          int num_splits, int pack_gqa, cudaStream_t stream) {
    if (!block_table) return GQA_ERR_NULL;
    KvCacheArgs kv;
    kv.seqlens_k = seqlens_k;
    kv.block_table = block_table;
    kv.max_pages = max_pages;
    kv.page_size = page_size;
    kv.num_pages = num_pages;
    kv.window = window;
    return kvcache_common(q, k_pages, v_pages, out, lse, B, Hq, Hkv, 0, D, max_seqlen_k, scale,
                          kv, num_splits, pack_gqa, stream);
}

int gqa_attn_decode_fp8(const void* q, const void* k8, const void* v8, float k_scale,
                        float v_scale, const int* block_table, const int* seqlens_k, void* out,
                        float* lse, int B, int Hq, int Hkv, int D, int Sk, int num_pages,
                        int page_size, int max_pages, int max_seqlen_k, float scale, int window,
                        int num_splits, int pack_gqa, cudaStream_t stream) {
    KvCacheArgs kv;
    kv.seqlens_k = seqlens_k;
    kv.window = window;
    kv.fp8 = true;
    kv.k_scale = k_scale;
    kv.v_scale = v_scale;
    if (block_table) {
        kv.block_table = block_table;
        kv.max_pages = max_pages;
        kv.page_size = page_size;
        kv.num_pages = num_pages;
        Sk = 0;
    }
    return kvcache_common(q, k8, v8, out, lse, B, Hq, Hkv, Sk, D,
                          (seqlens_k || block_table) ? max_seqlen_k : Sk, scale, kv, num_splits,
                          pack_gqa, stream);
}

int gqa_attn_selftest_timeout(int limit_ms, cudaStream_t stream) {
    if (limit_ms < 1 || limit_ms > 1000) return GQA_ERR_SHAPE;
    DeviceInfo* dev = nullptr;
    const int rc = device_info(&dev);
    if (rc != GQA_OK) return rc;
    selftest_wait_timeout<<<1, 32, 0, stream>>>(uint64_t(limit_ms) * 1000000ull);
    return cudaGetLastError() == cudaSuccess ? GQA_OK : GQA_ERR_CUDA;
}

}  // extern "C"

// The backward pass (its kernels and their host side) is kept in files of its own.
#include "backward_host.cuh"
