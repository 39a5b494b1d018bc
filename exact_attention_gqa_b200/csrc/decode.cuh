// Split-KV decode (one query position against a long KV cache) and the
// log-sum-exp weighted combine of its partial results.
//
// Decode reads every key and value once and does ~4 flops per byte, so it is
// bound by HBM bandwidth.  The kernel therefore streams K/V blocks through a
// TMA + mbarrier ring (one producer warp, four consumer warps), spreads the cache
// over many CTAs (batch x KV-head unit x split), and keeps the arithmetic small
// enough never to limit the stream: per 16 keys a consumer warp issues 16
// ldmatrix and 32 warp-level bf16 MMAs (m16n8k16, fp32 accumulate) for
// S = q K^T and O += P V, with P kept in registers between the two.
//
// The split-KV knob is the num_splits parameter of the GQA batch-size guide
// (parameter table and flash_attn_func example).  Its combine follows from the
// online softmax being exact and associative (FlashAttention-2 summary page,
// streaming softmax and L = m + log l): with per-split normalised O_s and L_s,
// L = M + ln sum_s exp(L_s - M) and O = sum_s exp(L_s - L) O_s.
// Splits are contiguous ranges of whole 64-key blocks.
//
// pack_gqa = 1 puts the query heads of one KV head (up to 16) in the rows of
// one CTA so that K/V are read once per group; pack_gqa = 0 gives every query
// head its own CTA (the group's CTAs then share K/V through L2).
//
// KV-cache forms (Ultralytics GQA glossary, "GQA and related techniques"):
//   - per-sequence cache lengths: sequence b attends to its first seqlens_k[b] keys;
//   - PagedAttention: the cache is a pool of fixed-size pages [num_pages, page_size,
//     Hkv, D] and block_table[b][p] names the page that holds keys
//     [p * page_size, (p + 1) * page_size) of sequence b; a 64-key block is one TMA
//     copy per page it touches (page_size a power of two >= 16);
//   - sliding window: the query, the newest position, sees only the last `window`
//     keys of its sequence (keys j >= L - window of L cached keys).
// With any of these, each sequence splits its own key range into num_splits parts.
//
// FP8 cache (KV8): K and V stored as e4m3 with one scale each per tensor.  The 8-bit
// tiles land by TMA in an unswizzled ring; each consumer warp converts its own 16
// keys of K and V to f16 in a swizzled buffer of its own, frees the stage, and runs
// the f16 form of the same MMAs (q is rounded to f16 once, P is packed as f16).  Every
// e4m3 value is an f16 value, so the conversion is exact; the K scale is folded into
// the softmax scale, O is multiplied by the V scale.  (An integer form of the
// conversion, shifting the byte into f16 bit positions, measured no faster: it frees
// the conversion unit but doubles the instructions per element.)
#pragma once
#include <type_traits>

#include "sm100_ptx.cuh"

namespace gqa {

struct DecodeParams {
    const __nv_bfloat16* q;  // [B, 1, Hq, D]
    __nv_bfloat16* out;      // [B, 1, Hq, D]
    float* lse;              // [B, Hq, 1]
    float* part_o;           // [B, Hq, n, D] fp32 (n > 1)
    float* part_l;           // [B, Hq, n]    fp32 (n > 1)
    int B, Hq, Hkv, Sk, G;
    int rows;                // query heads per CTA (1..16)
    int units_per_kv;        // ceil(G / rows)
    int n_splits;
    int blocks_per_split;    // 64-key blocks per split (whole-cache ranges)
    float scale_log2;
    // KV-cache forms; the defaults give the dense [B, Sk, Hkv, D] cache of Sk keys
    const int* seqlens_k = nullptr;    // [B] keys per sequence (<= its capacity)
    const int* block_table = nullptr;  // [B, max_pages] page of each logical page
    int max_pages = 0;                 // block_table row length
    int page_shift = 0;                // log2(page_size)
    int num_pages = 0;                 // pages in the pool
    int window = 0;                    // > 0: only the last `window` keys
    float v_scale = 1.f;               // e4m3 cache: value of one V code unit
};

template <int HD>
struct DecodeCfg {
    static constexpr int BN = 64;                  // keys per stage
    static constexpr int ATOMS = HD / 64;
    static constexpr int ATOM = BN * 128;          // bytes of one 64-key x 64-dim atom
    static constexpr int TILE = BN * HD * 2;       // bytes of K (or V) per stage
    static constexpr int STAGES = (HD == 128) ? 3 : 6;
    static constexpr int OFF_K = 0;
    static constexpr int OFF_V = STAGES * TILE;
    static constexpr int OFF_BAR = 2 * STAGES * TILE;
    static constexpr int OFF_MISC = OFF_BAR + 2 * STAGES * 8;
    static constexpr int MERGE_BYTES = 4 * 16 * (HD + 3) * 4;  // per-warp partials
    static constexpr int SMEM_BYTES =
        (OFF_MISC + 16 > MERGE_BYTES ? OFF_MISC + 16 : MERGE_BYTES) + 1024;
    static constexpr int THREADS = 160;
};

// e4m3 K/V: 8-bit stages (rows of HD bytes, no swizzle) and per-warp f16 copies of the
// warp's 16 keys in the 128B-swizzled layout the ldmatrix addressing expects
template <int HD>
struct DecodeCfg8 {
    static constexpr int BN = 64;
    static constexpr int TILE = BN * HD;        // bytes of K (or V) per stage
    static constexpr int STAGES = 4;
    static constexpr int WATOM = 16 * 128;      // a warp's 16 keys x 64 dims in f16
    static constexpr int WTILE = 16 * HD * 2;   // a warp's 16 keys, all dims, f16
    static constexpr int OFF_K = 0;
    static constexpr int OFF_V = STAGES * TILE;
    static constexpr int OFF_W = 2 * STAGES * TILE;  // [4 warps][K, V][WTILE]
    static constexpr int OFF_BAR = OFF_W + 4 * 2 * WTILE;
    static constexpr int OFF_MISC = OFF_BAR + 2 * STAGES * 8;
    static constexpr int MERGE_BYTES = 4 * 16 * (HD + 3) * 4;
    static constexpr int SMEM_BYTES =
        (OFF_MISC + 16 > MERGE_BYTES ? OFF_MISC + 16 : MERGE_BYTES) + 1024;
    static constexpr int THREADS = 160;
};

// four e4m3 values (byte i = element i) -> two f16x2 words (elements 0,1 and 2,3)
__device__ __forceinline__ void e4m3x4_to_f16x4(uint32_t x, uint32_t& lo, uint32_t& hi) {
    asm("{\n\t.reg .b16 a, b;\n\tmov.b32 {a, b}, %2;\n\t"
        "cvt.rn.f16x2.e4m3x2 %0, a;\n\tcvt.rn.f16x2.e4m3x2 %1, b;\n\t}"
        : "=r"(lo), "=r"(hi)
        : "r"(x));
}
// lo += float(low f16 of packed), hi += float(high f16): mixed-precision adds
__device__ __forceinline__ void add_f16x2_to_f32(uint32_t packed, float& lo, float& hi) {
    asm("{\n\t.reg .b16 l, h;\n\tmov.b32 {l, h}, %2;\n\t"
        "add.rn.f32.f16 %0, l, %0;\n\tadd.rn.f32.f16 %1, h, %1;\n\t}"
        : "+f"(lo), "+f"(hi)
        : "r"(packed));
}
__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
    uint32_t r;
    asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}
// bf16x2 -> f16x2 (round to nearest; |x| > 65504 becomes inf)
__device__ __forceinline__ uint32_t bf16x2_to_f16x2(uint32_t x) {
    return pack_f16x2(__uint_as_float(x << 16), __uint_as_float(x & 0xffff0000u));
}
__device__ __forceinline__ uint4 ld_shared_v4(uint32_t addr) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "r"(addr));
    return v;
}
__device__ __forceinline__ void st_shared_v4u(uint32_t addr, uint32_t a, uint32_t b, uint32_t c,
                                              uint32_t d) {
    asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c),
                 "r"(d));
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                        uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1,
                                          uint32_t& r2, uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}
// D += A(16x16, row) * B(16x8, col), bf16 inputs, fp32 accumulate
__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                               uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, "
        "{%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
// the same with f16 inputs
__device__ __forceinline__ void mma_f16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                              uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, "
        "{%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
template <bool F16>
__device__ __forceinline__ void mma_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                          uint32_t b1) {
    if constexpr (F16)
        mma_f16_16816(d, a, b0, b1);
    else
        mma_bf16_16816(d, a, b0, b1);
}

// Byte offset of the 16-byte chunk holding dims [8c, 8c+8) of row `row` in a
// 128B-swizzled [rows x 64 dims] atom written by TMA.
__device__ __forceinline__ uint32_t sw128_off(int row, int chunk) {
    return uint32_t(row * 128 + (((chunk & 7) ^ (row & 7)) << 4));
}

// PAGED = true reads K and V through p.block_table; the dense instantiation carries
// none of that code.  KV8 = true: K and V are e4m3 (see the top of the file).
template <int HD, bool PAGED = false, bool KV8 = false>
__global__ void __launch_bounds__(160, 2)
    decode_split_sm100(const __grid_constant__ CUtensorMap tm_k,
                       const __grid_constant__ CUtensorMap tm_v, const DecodeParams p) {
    using C = std::conditional_t<KV8, DecodeCfg8<HD>, DecodeCfg<HD>>;
    constexpr int ST = C::STAGES;
    constexpr int KSTEPS = HD / 16;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bar_full = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
    uint64_t* bar_empty = bar_full + ST;
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC);

    const int split = blockIdx.x;
    const int unit = blockIdx.y;  // kv head * units_per_kv + head chunk
    const int b = blockIdx.z;
    const int kvh = unit / p.units_per_kv;
    const int h0 = kvh * p.G + (unit - kvh * p.units_per_kv) * p.rows;
    const int rows = min(p.rows, kvh * p.G + p.G - h0);
    // this sequence's keys [key_start, len) and this split's 64-key blocks of them
    constexpr bool paged = PAGED;
    int len = p.Sk;
    if (p.seqlens_k) {
        const int cap = paged ? (p.max_pages << p.page_shift) : p.Sk;
        len = __ldg(p.seqlens_k + b);
        if (len < 0 || len > cap) {
            if (threadIdx.x == 0) raise_device_error(kDevBadKvIndex);
            len = min(max(len, 0), cap);
        }
    }
    const int key_start = p.window > 0 ? max(len - p.window, 0) : 0;
    const int kb_first = key_start / C::BN;
    const int kb_end = (len + C::BN - 1) / C::BN;
    const bool per_seq = p.seqlens_k != nullptr || p.window > 0;
    const int bps = per_seq ? (kb_end - kb_first + p.n_splits - 1) / p.n_splits
                            : p.blocks_per_split;
    const int blk0 = kb_first + split * bps;
    const int blk1 = min(blk0 + bps, kb_end);
    const int nblk = max(blk1 - blk0, 0);
    const int key_end = min(blk1 * C::BN, len);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    // the combine kernel (launched as a programmatic dependent) may be scheduled
    // now; it waits for this grid's completion before it reads any partial
    griddep_launch_dependents();
    if (threadIdx.x == 0) {
        for (int s = 0; s < ST; ++s) {
            mbar_init(bar_full + s, 1);
            mbar_init(bar_empty + s, 4);
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();

    // per-warp online-softmax state: rows g = lane/4 and g + 8
    float m_run[2] = {-INFINITY, -INFINITY};
    float l_part[2] = {0.f, 0.f};
    float l_rnd[2] = {0.f, 0.f};
    float o[KSTEPS * 2][4];
#pragma unroll
    for (int t = 0; t < KSTEPS * 2; ++t)
#pragma unroll
        for (int e = 0; e < 4; ++e) o[t][e] = 0.f;

    if (warp == 4) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            tma_prefetch_desc(&tm_k);
            tma_prefetch_desc(&tm_v);
            // paged: the pages of block c + 1 are looked up while block c is issued,
            // so the table read never sits between a free stage and its copies
            const int rows = paged ? min(1 << p.page_shift, C::BN) : C::BN;
            const int* trow = paged ? p.block_table + size_t(b) * p.max_pages : nullptr;
            int pg_cur[4] = {0, 0, 0, 0}, pg_nxt[4] = {0, 0, 0, 0};
            auto lookup = [&](int blk, int (&pg)[4]) {
                const int key0 = blk * C::BN;
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    if (i * rows >= C::BN) break;
                    // rows past the sequence's end are masked: they are read from the
                    // block's first page (key0 < len) rather than from table entries the
                    // sequence may not have filled
                    const int key = (key0 + i * rows < len) ? key0 + i * rows : key0;
                    pg[i] = __ldg(trow + (key >> p.page_shift));
                }
            };
            // copies of rows [r0, r0 + box) of stage s from tensor row z
            auto load_rows = [&](int s, int r0, int z) {
                if constexpr (KV8) {
                    tma_load_3d(smem + C::OFF_K + s * C::TILE + r0 * HD, &tm_k, bar_full + s, 0,
                                kvh, z);
                    tma_load_3d(smem + C::OFF_V + s * C::TILE + r0 * HD, &tm_v, bar_full + s, 0,
                                kvh, z);
                } else {
#pragma unroll
                    for (int a = 0; a < C::ATOMS; ++a) {
                        tma_load_3d(smem + C::OFF_K + s * C::TILE + a * C::ATOM + r0 * 128,
                                    &tm_k, bar_full + s, a * 64, kvh, z);
                        tma_load_3d(smem + C::OFF_V + s * C::TILE + a * C::ATOM + r0 * 128,
                                    &tm_v, bar_full + s, a * 64, kvh, z);
                    }
                }
            };
            if (paged && nblk > 0) lookup(blk0, pg_cur);
            int c = 0;
            for (; c < nblk; ++c) {
                if (paged && c + 1 < nblk) lookup(blk0 + c + 1, pg_nxt);
                const int s = c % ST;
                if (!mbar_wait(bar_empty + s, ((c / ST) & 1) ^ 1, abort_flag)) break;
                mbar_arrive_expect_tx(bar_full + s, 2 * C::TILE);
                const int key0 = (blk0 + c) * C::BN;
                if (!paged) {
                    load_rows(s, 0, b * p.Sk + key0);
                } else {
                    // one copy of min(page_size, 64) rows per page the block touches;
                    // rows land at their key offset, so the 128B swizzle (a function
                    // of the shared-memory address) matches a single 64-row copy
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        if (i * rows >= C::BN) break;
                        const int r0 = i * rows;
                        const int key = (key0 + r0 < len) ? key0 + r0 : key0;
                        int page = pg_cur[i];
                        if (page < 0 || page >= p.num_pages) {
                            raise_device_error(kDevBadKvIndex);
                            page = 0;
                        }
                        load_rows(s, r0,
                                  (page << p.page_shift) + (key & ((1 << p.page_shift) - 1)));
                    }
#pragma unroll
                    for (int i = 0; i < 4; ++i) pg_cur[i] = pg_nxt[i];
                }
            }
            // every issued copy lands before the CTA may reuse or release the memory
            for (int s = 0; s < ST; ++s) {
                const int u = c / ST + (s < c % ST ? 1 : 0);
                if (u > 0) {
                    const uint64_t t0 = globaltimer_ns();
                    while (!mbar_try_wait(bar_full + s, (u - 1) & 1))
                        if (globaltimer_ns() - t0 > kWaitLimitNs) {
                            raise_device_error(kDevWaitTimeout);
                            break;
                        }
                }
            }
        }
    } else {
        // ------------------------------------------------------------ consumers
        const float sl2 = p.scale_log2;
        const int g = lane >> 2;      // row (query head offset) of c0/c1, +8 for c2/c3
        const int qd = (lane & 3) * 2;  // column pair within an 8-wide tile
        // q as the A operand of m16n8k16 (rows >= `rows` are zero)
        uint32_t qa[KSTEPS][4];
        {
            const uint32_t* qrow0 = reinterpret_cast<const uint32_t*>(
                p.q + (size_t(b) * p.Hq + h0 + g) * HD);
            const uint32_t* qrow1 = reinterpret_cast<const uint32_t*>(
                p.q + (size_t(b) * p.Hq + h0 + g + 8) * HD);
            const bool v0 = g < rows, v1 = g + 8 < rows;
#pragma unroll
            for (int kk = 0; kk < KSTEPS; ++kk) {
                qa[kk][0] = v0 ? __ldg(qrow0 + (kk * 16 + qd) / 2) : 0u;
                qa[kk][1] = v1 ? __ldg(qrow1 + (kk * 16 + qd) / 2) : 0u;
                qa[kk][2] = v0 ? __ldg(qrow0 + (kk * 16 + 8 + qd) / 2) : 0u;
                qa[kk][3] = v1 ? __ldg(qrow1 + (kk * 16 + 8 + qd) / 2) : 0u;
                if constexpr (KV8) {
#pragma unroll
                    for (int e = 0; e < 4; ++e) qa[kk][e] = bf16x2_to_f16x2(qa[kk][e]);
                }
            }
        }
        const uint32_t sK0 = smem_u32(smem + C::OFF_K);
        const uint32_t sV0 = smem_u32(smem + C::OFF_V);
        // KV8: this warp's f16 copies of its 16 keys; ldmatrix rows count from the warp's
        // first key there, and an atom (64 dims) holds 16 rows
        uint32_t wK = 0, wV = 0;
        if constexpr (KV8) {
            wK = smem_u32(smem + C::OFF_W + warp * 2 * C::WTILE);
            wV = wK + C::WTILE;
        }
        constexpr int ATOM_B = KV8 ? 16 * 128 : 64 * 128;
        const int row0 = KV8 ? warp * 16 : 0;
        // ldmatrix row addresses: lane provides row (lane & 7) of matrix (lane >> 3)
        const int mat = lane >> 3, mrow = lane & 7;
        // QK: matrices (keys +0/+8) x (dim chunk +0/+1): key = 16w + (mat>>1)*8 + mrow
        const int key_qk = warp * 16 + (mat >> 1) * 8 + mrow;
        const int chunk_qk = mat & 1;
        // PV (trans): matrices (keys +0/+8) x (dim chunk +0/+1): key = 16w + (mat&1)*8 + mrow
        const int key_pv = warp * 16 + (mat & 1) * 8 + mrow;
        const int chunk_pv = mat >> 1;
        for (int c = 0; c < nblk; ++c) {
            const int s = c % ST;
            if (!mbar_wait_warp(bar_full + s, (c / ST) & 1, abort_flag)) break;
            uint32_t sK = sK0 + s * C::TILE;
            uint32_t sV = sV0 + s * C::TILE;
            // keys past the end may be unwritten cache memory (a page's or the dense
            // cache's unused rows): their P is 0, but 0 * NaN would still reach O, so this
            // warp zeroes its own V rows there; the stage is handed back to TMA only after
            // a proxy fence orders these writes before the next copy into it
            bool zeroed = false;
            if constexpr (!KV8) {
                const int r_end = key_end - (blk0 + c) * C::BN - warp * 16;  // rows kept
                if (r_end < 16) {
                    zeroed = true;
                    constexpr int CH = 16 * C::ATOMS * 8;  // 16-byte chunks of 16 rows
                    for (int ci = lane; ci < CH; ci += 32) {
                        const int row = ci / (C::ATOMS * 8);
                        if (row < r_end) continue;
                        const int rest = ci - row * (C::ATOMS * 8);
                        const int a = rest >> 3, q16 = rest & 7;
                        st_shared_v4u(sV + uint32_t(a * C::ATOM + (warp * 16 + row) * 128 +
                                                    q16 * 16),
                                      0u, 0u, 0u, 0u);
                    }
                    __syncwarp();
                }
            }
            if constexpr (KV8) {
                // e4m3 rows of this warp's 16 keys -> f16, 16-byte chunks read in order
                // (conflict-free) and written to the swizzled atoms; then the stage is free
                __syncwarp();  // the previous block's ldmatrix reads of wK / wV are done
                // lane -> one 8-dim chunk: the loads are consecutive 8-byte pieces and
                // each group of 8 lanes stores one 128-byte row of an atom (every bank
                // once), so neither side has bank conflicts
                const int r_keep = key_end - (blk0 + c) * C::BN - warp * 16;  // rows kept
#pragma unroll
                for (int kv = 0; kv < 2; ++kv) {
                    const uint32_t src = (kv ? sV : sK) + uint32_t(warp * 16 * HD);
                    const uint32_t dst = kv ? wV : wK;
#pragma unroll
                    for (int it = 0; it < HD / 16; ++it) {
                        const int ci = it * 32 + lane;       // 8-dim chunk of the warp's rows
                        const int row = ci / (HD / 8);       // key within the warp's 16
                        const int ch = ci - row * (HD / 8);  // f16 chunk index over HD / 8
                        uint32_t x0, x1;
                        asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];"
                                     : "=r"(x0), "=r"(x1)
                                     : "r"(src + uint32_t(ci * 8)));
                        uint32_t h[4];
                        e4m3x4_to_f16x4(x0, h[0], h[1]);
                        e4m3x4_to_f16x4(x1, h[2], h[3]);
                        // keys past the end may be unwritten cache memory: their P is 0,
                        // and 0 * NaN would still reach O, so they become zeros
                        if (row >= r_keep) h[0] = h[1] = h[2] = h[3] = 0u;
                        st_shared_v4u(dst + uint32_t((ch >> 3) * ATOM_B) + sw128_off(row, ch),
                                      h[0], h[1], h[2], h[3]);
                    }
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(bar_empty + s);
                sK = wK;
                sV = wV;
            }
            float sc[2][4];
#pragma unroll
            for (int t = 0; t < 2; ++t)
#pragma unroll
                for (int e = 0; e < 4; ++e) sc[t][e] = 0.f;
#pragma unroll
            for (int kk = 0; kk < KSTEPS; ++kk) {
                const int chunk = kk * 2 + chunk_qk;
                uint32_t b0, b1, b2, b3;
                ldsm_x4(sK + (chunk >> 3) * ATOM_B + sw128_off(key_qk - row0, chunk), b0, b1, b2,
                        b3);
                mma_16816<KV8>(sc[0], qa[kk], b0, b1);
                mma_16816<KV8>(sc[1], qa[kk], b2, b3);
            }
            // mask keys past the end of this split / of the sequence, and keys
            // before the window (only blocks that straddle one of those edges)
            const int kblk = (blk0 + c) * C::BN;
            if (kblk + C::BN > key_end || kblk < key_start) {
                const int kbase = kblk + warp * 16 + qd;
#pragma unroll
                for (int t = 0; t < 2; ++t)
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int key = kbase + t * 8 + (e & 1);
                        if (key >= key_end || key < key_start) sc[t][e] = -INFINITY;
                    }
            }
            // online softmax (rows g and g + 8), quad reduction of the block max
            float alpha[2];
#pragma unroll
            for (int hr = 0; hr < 2; ++hr) {
                float mx = fmaxf(fmaxf(sc[0][2 * hr], sc[0][2 * hr + 1]),
                                 fmaxf(sc[1][2 * hr], sc[1][2 * hr + 1]));
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
                const float mb = mx * sl2;
                alpha[hr] = 1.f;
                if (mb > m_run[hr] + 8.0f) {
                    alpha[hr] = ex2_approx(m_run[hr] - mb);
                    m_run[hr] = mb;
                }
            }
            uint32_t pa[4];
            {
                float pr[2][4];
#pragma unroll
                for (int t = 0; t < 2; ++t)
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int hr = e >> 1;
                        const float mu = (m_run[hr] == -INFINITY) ? 0.f : m_run[hr];
                        pr[t][e] = ex2_approx(fmaf(sc[t][e], sl2, -mu));
                    }
                if constexpr (KV8) {
                    pa[0] = pack_f16x2(pr[0][0], pr[0][1]);
                    pa[1] = pack_f16x2(pr[0][2], pr[0][3]);
                    pa[2] = pack_f16x2(pr[1][0], pr[1][1]);
                    pa[3] = pack_f16x2(pr[1][2], pr[1][3]);
                } else {
                    pa[0] = pack_bf16x2(pr[0][0], pr[0][1]);
                    pa[1] = pack_bf16x2(pr[0][2], pr[0][3]);
                    pa[2] = pack_bf16x2(pr[1][0], pr[1][1]);
                    pa[3] = pack_bf16x2(pr[1][2], pr[1][3]);
                }
                // two row sums: exact p (for L) and the bf16 weights the MMA consumes
                // (for O / l); rows g: pa[0], pa[2]; rows g + 8: pa[1], pa[3]
#pragma unroll
                for (int hr = 0; hr < 2; ++hr)
                    l_part[hr] = l_part[hr] * alpha[hr] + pr[0][2 * hr] + pr[0][2 * hr + 1] +
                                 pr[1][2 * hr] + pr[1][2 * hr + 1];
                if constexpr (KV8) {
                    float a0 = 0.f, a1 = 0.f, b0 = 0.f, b1 = 0.f;
                    add_f16x2_to_f32(pa[0], a0, a1);
                    add_f16x2_to_f32(pa[2], a0, a1);
                    add_f16x2_to_f32(pa[1], b0, b1);
                    add_f16x2_to_f32(pa[3], b0, b1);
                    l_rnd[0] = l_rnd[0] * alpha[0] + (a0 + a1);
                    l_rnd[1] = l_rnd[1] * alpha[1] + (b0 + b1);
                } else {
                    l_rnd[0] = l_rnd[0] * alpha[0] + bf16_lo(pa[0]) + bf16_hi(pa[0]) +
                               bf16_lo(pa[2]) + bf16_hi(pa[2]);
                    l_rnd[1] = l_rnd[1] * alpha[1] + bf16_lo(pa[1]) + bf16_hi(pa[1]) +
                               bf16_lo(pa[3]) + bf16_hi(pa[3]);
                }
            }
            if (alpha[0] != 1.f || alpha[1] != 1.f) {
#pragma unroll
                for (int t = 0; t < KSTEPS * 2; ++t) {
                    o[t][0] *= alpha[0];
                    o[t][1] *= alpha[0];
                    o[t][2] *= alpha[1];
                    o[t][3] *= alpha[1];
                }
            }
#pragma unroll
            for (int nt = 0; nt < KSTEPS; ++nt) {
                const int chunk = nt * 2 + chunk_pv;
                uint32_t b0, b1, b2, b3;
                ldsm_x4_t(sV + (chunk >> 3) * ATOM_B + sw128_off(key_pv - row0, chunk), b0, b1, b2,
                          b3);
                mma_16816<KV8>(o[2 * nt], pa, b0, b1);
                mma_16816<KV8>(o[2 * nt + 1], pa, b2, b3);
            }
            if (zeroed) fence_proxy_async();
            __syncwarp();
            if (!KV8 && lane == 0) mbar_arrive(bar_empty + s);
        }
#pragma unroll
        for (int hr = 0; hr < 2; ++hr) {
            l_part[hr] += __shfl_xor_sync(0xffffffffu, l_part[hr], 1);
            l_part[hr] += __shfl_xor_sync(0xffffffffu, l_part[hr], 2);
            l_rnd[hr] += __shfl_xor_sync(0xffffffffu, l_rnd[hr], 1);
            l_rnd[hr] += __shfl_xor_sync(0xffffffffu, l_rnd[hr], 2);
        }
    }
    __syncthreads();  // every stage consumed, every copy landed: reuse smem for the merge

    // ---------------------------------------------------------------- merge warps
    float* mo = reinterpret_cast<float*>(smem);           // [4][16][HD]
    float* mm = mo + 4 * 16 * HD;                          // [4][16]
    float* ml = mm + 4 * 16;                               // [4][16] exact sums
    float* mr = ml + 4 * 16;                               // [4][16] bf16-weight sums
    if (warp < 4) {
        const int g = lane >> 2, qd = (lane & 3) * 2;
#pragma unroll
        for (int nt = 0; nt < KSTEPS * 2; ++nt) {
            float* r0 = mo + (warp * 16 + g) * HD + nt * 8 + qd;
            float* r1 = mo + (warp * 16 + g + 8) * HD + nt * 8 + qd;
            r0[0] = o[nt][0];
            r0[1] = o[nt][1];
            r1[0] = o[nt][2];
            r1[1] = o[nt][3];
        }
        if ((lane & 3) == 0) {
            mm[warp * 16 + g] = m_run[0];
            mm[warp * 16 + g + 8] = m_run[1];
            ml[warp * 16 + g] = l_part[0];
            ml[warp * 16 + g + 8] = l_part[1];
            mr[warp * 16 + g] = l_rnd[0];
            mr[warp * 16 + g + 8] = l_rnd[1];
        }
    }
    __syncthreads();
    const bool aborted = *abort_flag != 0;
    for (int idx = threadIdx.x; idx < rows * HD; idx += blockDim.x) {
        const int r = idx / HD, d = idx - r * HD;
        if (aborted) {
            // a wait gave up (device error word set): this CTA's rows become empty,
            // O = 0 and L = -inf, so that neither the output nor the combine can pick
            // up what an earlier call left in the output or the partials buffer
            const int h = h0 + r;
            if (p.n_splits == 1) {
                p.out[(size_t(b) * p.Hq + h) * HD + d] = __float2bfloat16_rn(0.f);
                if (d == 0) p.lse[size_t(b) * p.Hq + h] = -INFINITY;
            } else {
                const size_t base = (size_t(b) * p.Hq + h) * p.n_splits + split;
                p.part_o[base * HD + d] = 0.f;
                if (d == 0) p.part_l[base] = -INFINITY;
            }
            continue;
        }
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < 4; ++w) M = fmaxf(M, mm[w * 16 + r]);
        const float Mu = (M == -INFINITY) ? 0.f : M;
        float acc = 0.f, l = 0.f, lr = 0.f;
#pragma unroll
        for (int w = 0; w < 4; ++w) {
            const float f = ex2_approx(mm[w * 16 + r] - Mu);
            acc += f * mo[(w * 16 + r) * HD + d];
            l += f * ml[w * 16 + r];
            lr += f * mr[w * 16 + r];
        }
        const int h = h0 + r;
        const float inv_l = (lr > 0.f) ? (KV8 ? p.v_scale : 1.f) / lr : 0.f;
        const float L = (l > 0.f) ? (Mu + __log2f(l)) * 0.69314718055994531f : -INFINITY;
        if (p.n_splits == 1) {
            p.out[(size_t(b) * p.Hq + h) * HD + d] = __float2bfloat16_rn(acc * inv_l);
            if (d == 0) p.lse[size_t(b) * p.Hq + h] = L;
        } else {
            const size_t base = (size_t(b) * p.Hq + h) * p.n_splits + split;
            p.part_o[base * HD + d] = acc * inv_l;
            if (d == 0) p.part_l[base] = L;
        }
    }
}

// One CTA per (batch, query head), one thread per output dimension:
// L = M + ln sum_s exp(L_s - M) with M = max_s L_s, then O = sum_s exp(L_s - L) O_s.
// The split weights are computed once into shared memory, and the weighted sum
// over splits keeps many independent loads in flight (the partials were just
// written and sit in L2, so the sum is bound by load latency, not bandwidth).
constexpr int kCombineMaxSplits = 256;
template <int HD>
__global__ void __launch_bounds__(HD)
    splitkv_combine(const float* __restrict__ part_o, const float* __restrict__ part_l,
                    __nv_bfloat16* __restrict__ out, float* __restrict__ lse, int rows_bh,
                    int n) {
    constexpr int WARPS = HD / 32;
    __shared__ float wts[kCombineMaxSplits];
    __shared__ float red[WARPS];
    __shared__ float s_stat[2];
    const int w = blockIdx.x;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    griddep_wait();  // the split kernel has finished and its partials are visible
    if (w >= rows_bh) return;
    const float* Ls = part_l + size_t(w) * n;
    float M = -INFINITY;
    for (int s = tid; s < n; s += HD) M = fmaxf(M, Ls[s]);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
    if (lane == 0) red[warp] = M;
    __syncthreads();
    if (tid == 0) {
        float m = red[0];
#pragma unroll
        for (int i = 1; i < WARPS; ++i) m = fmaxf(m, red[i]);
        s_stat[0] = m;
    }
    __syncthreads();
    M = s_stat[0];
    float sum = 0.f;
    if (M != -INFINITY)
        for (int s = tid; s < n; s += HD) sum += (Ls[s] == -INFINITY) ? 0.f : expf(Ls[s] - M);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
    __syncthreads();
    if (lane == 0) red[warp] = sum;
    __syncthreads();
    if (tid == 0) {
        float t = 0.f;
#pragma unroll
        for (int i = 0; i < WARPS; ++i) t += red[i];
        s_stat[1] = (M == -INFINITY) ? -INFINITY : M + logf(t);
    }
    __syncthreads();
    const float L = s_stat[1];
    for (int s = tid; s < n; s += HD)
        wts[s] = (L == -INFINITY || Ls[s] == -INFINITY) ? 0.f : expf(Ls[s] - L);
    __syncthreads();
    const float* os = part_o + size_t(w) * n * HD + tid;
    float acc0 = 0.f, acc1 = 0.f, acc2 = 0.f, acc3 = 0.f;
    int s = 0;
#pragma unroll 4
    for (; s + 4 <= n; s += 4) {
        const float x0 = os[size_t(s) * HD], x1 = os[size_t(s + 1) * HD];
        const float x2 = os[size_t(s + 2) * HD], x3 = os[size_t(s + 3) * HD];
        acc0 += (wts[s] != 0.f) ? wts[s] * x0 : 0.f;
        acc1 += (wts[s + 1] != 0.f) ? wts[s + 1] * x1 : 0.f;
        acc2 += (wts[s + 2] != 0.f) ? wts[s + 2] * x2 : 0.f;
        acc3 += (wts[s + 3] != 0.f) ? wts[s + 3] * x3 : 0.f;
    }
    for (; s < n; ++s) {
        const float x = os[size_t(s) * HD];
        acc0 += (wts[s] != 0.f) ? wts[s] * x : 0.f;
    }
    out[size_t(w) * HD + tid] = __float2bfloat16_rn((acc0 + acc1) + (acc2 + acc3));
    if (tid == 0) lse[w] = L;
}

}  // namespace gqa
