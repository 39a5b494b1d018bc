// Prefill forward of exact grouped-query attention on sm_100a.
//
// What it computes: O = softmax(scale * Q K^T [+ causal mask]) V per query head,
// with the per-row log-sum-exp L written out (FlashAttention-2 summary page:
// tiled online softmax, deferred 1/l normalisation, L = m + log l; causal
// paragraph: blocks above the diagonal skipped, the mask applied only where the
// diagonal crosses a block).  Query head h reads key/value head h / G
// (Ultralytics GQA glossary, "How GQA works").
//
// Work unit ("CTA tile"): 256 query rows that share one key/value head, split
// in two sub-tiles of 128 rows that ping-pong on the tensor core:
//   pack_gqa = 1: rows are (position, head) pairs, 128/G positions x the G query
//                 heads of one KV head per sub-tile, so K/V are streamed once
//                 for the whole group (GQA batch-size guide, PackGQA items 1-3);
//   pack_gqa = 0: rows are 128 consecutive positions of one query head.
// Work units are spread over a persistent grid (sequence-dimension parallelism,
// FlashAttention-2 summary page).  Causal and variable-length batches run the
// longest units first (attention balancing, Raptor-T abstract) within groups of
// (batch, head unit) pairs whose K and V fit a share of L2; dense non-causal
// batches run the position tiles of one (batch, KV head) back to back so that
// its K and V are re-read from L2 rather than HBM.
//
// Roles inside the CTA (320 threads):
//   warps 0-3  softmax for sub-tile 0 (one thread = one row = one TMEM lane)
//   warps 4-7  softmax for sub-tile 1
//   warp 8     tcgen05.mma issuer (one thread), owns the TMEM allocation
//   warp 9     TMA producer (one thread): Q once per tile (double-buffered when it
//              fits, so the next tile's Q lands while this one computes), K/V
//              blocks in a ring
// Tensor memory (512 columns): S0 [0,128) S1 [128,256) O0 [256,256+D)
// O1 [256+D, 256+2D); P_i (bf16 pairs, 64 columns) has its own columns
// [384+64i, 448+64i) when D = 64 and otherwise overwrites the first half of S_i
// after the softmax has read S_i into registers.  The two sub-tiles run their
// softmax independently; the tensor core alternates between them.  At the end of
// a sub-tile the softmax threads normalise O; with D = 64 a sub-tile whose rows
// are all real is staged in shared memory and written by one TMA store.
//
// Block-sparse form (Raptor-T abstract: BigBird computes attention between blocks of
// a fixed size, several patterns combined): blk_row_ptr / blk_col list, per query block
// of 128 positions, the 128-key blocks it attends to; a CTA tile (at most 128 positions,
// PackGQA with G >= 2) lies in one query block and walks that list instead of 0..n-1.
// With causal set, keys past a row's diagonal are masked inside the listed blocks.
//
// Sliding-window form (WINDOW; Ultralytics GQA glossary, "GQA and related techniques":
// sliding-window attention caps the tokens attended to): causal, and query position i
// sees only keys (i + Sk - Sq - window, i + Sk - Sq].  Each sub-tile walks its own
// blocks [jb0, nblk); the K/V stream covers their union, and only blocks that cross the
// window's lower edge or the diagonal are masked element by element.
//
// Online softmax in the log2 domain: s2 = s * scale * log2(e).  The running
// max used for the exponentials is only raised when a block's max exceeds it by
// more than 8 (a factor 256), so O is rescaled rarely; since O and l always
// share the same reference max, O / l and L = m + log l are unchanged.  The
// per-element work uses sm_100's paired fp32 instructions (fma/add .f32x2) and
// three-input max to halve its issue slots.
#pragma once
#include "sm100_ptx.cuh"

namespace gqa {

struct PrefillParams {
    __nv_bfloat16* out;      // [rows, Hq, D]
    float* lse;              // [B, Hq, Sq] or [Hq, total]
    const int* cu_seqlens;   // device int32[B+1] or nullptr
    int B, Hq, Hkv, Sq, Sk;  // varlen: Sq = maximum sequence length, Sk = total_rows
    int total_rows;          // varlen: packed rows of q, k, v (cu_seqlens[B])
    int G;
    int pack;
    int sub_pos;             // positions per 128-row sub-tile: 128 / G (pack) or 128
    int n_mblk;              // CTA tiles along the positions of the longest sequence
    int n_hu;                // head units: Hkv (pack) or Hq
    int n_units;             // n_mblk * B * n_hu
    int causal;
    int kv_major;            // 1: tiles of one (batch, head unit) consecutive (L2 reuse)
    int hu_group;            // kv_major = 0: (batch, head unit) pairs per longest-first pass
    float scale_log2;        // scale * log2(e)
    // block-sparse: CSR rows of 128-key blocks per 128-position query block (nullptr: dense)
    const int* blk_row_ptr = nullptr;  // [ceil(Sq / 128) + 1]
    const int* blk_col = nullptr;      // [nnz], ascending within a row
    int n_kblk = 0;                    // ceil(Sk / 128): key blocks that exist
    // block-sparse over packed sequences (minimum padding): first pattern row of each
    // sequence, [B + 1] (prefix sum of ceil(n_b / 128)); nullptr: one dense pattern
    const int* blk_off = nullptr;
    // optional tile order (attention balancing): entry t is the unit the persistent
    // loop's t-th step takes, as (b * n_hu + hu) * n_mblk + m, or -1 for no tile
    const int* tile_order = nullptr;
    // e4m3 Q/K/V: O = accumulator * o_scale / l (v_scale over P's range shift)
    float o_scale = 1.f;
    // sliding window (causal): keys per query, >= 1 (WINDOW instantiation only)
    int window = 0;
    // dense layout: elements between consecutive (batch, head) rows of lse (Sq, or the
    // full problem's length when a range of positions is computed on its own)
    int lse_ld = 0;
};

template <int HD, bool FP8 = false>
struct PrefillCfg {
    // FP8: Q, K, V are e4m3 (one byte per element); D = 128 only
    static_assert(!FP8 || HD == 128, "e4m3 prefill: D = 128");
    static constexpr int ES = FP8 ? 1 : 2;        // bytes per input element
    static constexpr int BM = 128;                // rows per sub-tile
    static constexpr int BN = 128;                // keys per K/V block
    static constexpr int ATOMS = HD * ES / 128;   // 128-byte swizzle atoms along D
    static constexpr int ATOM_ELEMS = 128 / ES;   // elements of D per atom
    static constexpr int ATOM_Q = BM * 128;       // bytes of one Q atom
    static constexpr int ATOM_KV = BN * 128;      // bytes of one K or V atom
    static constexpr int Q_SUB = BM * HD * ES;    // bytes of one Q sub-tile
    static constexpr int Q_TILE = 2 * Q_SUB;      // both sub-tiles
    static constexpr int KV_TILE = BN * HD * ES;  // bytes of one K or V block
    static constexpr int STAGES = (HD == 128) ? (FP8 ? 4 : 2) : 4;
    static constexpr int Q_STAGES = (HD == 128) ? 1 : 2;
    // MMA K-step: 32 bytes of the reduction dimension (16 bf16 or 32 e4m3 elements)
    static constexpr int KSTEP = 32 / ES;
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_K = OFF_Q + Q_STAGES * Q_TILE;
    static constexpr int OFF_V = OFF_K + STAGES * KV_TILE;
    // D = 64: full sub-tiles of O leave through a shared-memory box and one TMA store
    // (128B-swizzled rows, the same box as Q's); D = 128 has no room and stores rows.
    static constexpr bool EPI_TMA = (HD == 64) && !FP8;
    static constexpr int OFF_O = OFF_V + STAGES * KV_TILE;
    static constexpr int O_SUB = BM * HD * 2;  // bf16 output
    static constexpr int OFF_BAR = OFF_O + (EPI_TMA ? 2 * O_SUB : 0);
    static constexpr int NUM_BARS = 2 * Q_STAGES + 4 * STAGES + 6 + 1 + 4;
    static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
    static constexpr int SMEM_BYTES = OFF_MISC + 64 + 1024;  // + alignment slack
    static constexpr int TMEM_COLS = 512;
    static constexpr int THREADS = 320;
    __device__ static constexpr uint32_t s_col(int i) { return uint32_t(i) * 128u; }
    __device__ static constexpr uint32_t o_col(int i) { return 256u + uint32_t(i) * HD; }
    // P (bf16, 64 columns): its own columns when they fit (D = 64), else over S
    static constexpr bool P_OWN = (HD == 64);
    __device__ static constexpr uint32_t p_col(int i) {
        return P_OWN ? 384u + uint32_t(i) * 64u : s_col(i);
    }
    // e4m3 P: the running max moves when a block's max exceeds it by more than a factor
    // 2, and P carries a factor 2^7 (folded into the exponent), so P <= 256 < 448 (the
    // largest e4m3 value) while small probabilities keep 7 more bits of range
    static constexpr float RESCALE_THRESHOLD = FP8 ? 1.0f : 8.0f;  // log2 units
    static constexpr float P_SHIFT = FP8 ? 7.0f : 0.0f;            // log2 units
};

struct TileInfo {
    int b, hu, m;
    int q_row0, k_row0;   // first row of this sequence in the [rows, H, D] views
    int sq, sk;           // lengths of this sequence
    int p0[2];            // first position of each sub-tile
    int nblk[2];          // K/V blocks each sub-tile visits (0: nothing to compute)
    int valid[2];         // sub-tile holds at least one real query row
    int full_blk[2];      // blocks [0, full_blk) need no mask for any row
    int kb0;              // block-sparse: first entry of this tile's row in blk_col
    int jb0[2];           // sliding window: first block each sub-tile visits (else 0)
    int lo_full[2];       // sliding window: blocks >= lo_full have no key below a row's window
};

template <int BN, bool SPARSE = false, bool WINDOW = false>
__device__ __forceinline__ TileInfo decode_tile(const PrefillParams& p, int t) {
    TileInfo ti;
    bool none = false;
    if constexpr (SPARSE) {
        if (p.tile_order) {  // balanced order: unit index in the (b, hu, m) linearisation
            const int u = __ldg(p.tile_order + t);
            none = u < 0;
            t = none ? 0 : u;
        }
    }
    if (p.kv_major || (SPARSE && p.tile_order)) {
        const int bh = t / p.n_mblk;
        ti.m = t - bh * p.n_mblk;
        ti.b = bh / p.n_hu;
        ti.hu = bh - ti.b * p.n_hu;
    } else {
        // Longest-first within groups of hu_group (batch, head unit) pairs: a group's
        // position tiles run from the last (longest under the causal mask) to the
        // first, then the next group follows.  A group's K and V stay in L2 while
        // its tiles run, and the tiles still end in short ones.
        const int per_m = p.B * p.n_hu;
        const int hg_full = p.hu_group;
        const int n_full = per_m / hg_full;
        const int t_full = n_full * hg_full * p.n_mblk;
        int c, hg, rem;
        if (t < t_full) {
            c = t / (hg_full * p.n_mblk);
            hg = hg_full;
            rem = t - c * hg_full * p.n_mblk;
        } else {
            c = n_full;
            hg = per_m - n_full * hg_full;
            rem = t - t_full;
        }
        ti.m = p.n_mblk - 1 - rem / hg;
        const int r = c * hg_full + (rem - (rem / hg) * hg);
        ti.b = r / p.n_hu;
        ti.hu = r - ti.b * p.n_hu;
    }
    if (p.cu_seqlens) {
        const int a = __ldg(p.cu_seqlens + ti.b), e = __ldg(p.cu_seqlens + ti.b + 1);
        ti.q_row0 = ti.k_row0 = a;
        ti.sq = ti.sk = e - a;
    } else {
        ti.q_row0 = ti.b * p.Sq;
        ti.k_row0 = ti.b * p.Sk;
        ti.sq = p.Sq;
        ti.sk = p.Sk;
    }
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const int p0 = ti.m * 2 * p.sub_pos + i * p.sub_pos;
        ti.p0[i] = p0;
        ti.valid[i] = p0 < ti.sq;
        const int last = min(p0 + p.sub_pos - 1, ti.sq - 1);
        int lim = p.causal ? min(ti.sk, last + ti.sk - ti.sq + 1) : ti.sk;
        ti.nblk[i] = (ti.valid[i] && lim > 0) ? (lim + BN - 1) / BN : 0;
        int first_lim = p.causal ? min(ti.sk, p0 + ti.sk - ti.sq + 1) : ti.sk;
        ti.full_blk[i] = first_lim > 0 ? first_lim / BN : 0;
        ti.jb0[i] = 0;
        ti.lo_full[i] = 0;
        if constexpr (WINDOW) {
            // first visible key of the sub-tile's first and last rows
            const int lo_first = p0 + ti.sk - ti.sq - p.window + 1;
            const int lo_last = last + ti.sk - ti.sq - p.window + 1;
            ti.jb0[i] = (ti.nblk[i] > 0 && lo_first > 0) ? min(lo_first / BN, ti.nblk[i]) : 0;
            ti.lo_full[i] = lo_last > 0 ? (lo_last + BN - 1) / BN : 0;
        }
    }
    ti.kb0 = 0;
    if constexpr (SPARSE) {
        // both sub-tiles lie in query block qb (of this sequence) and share its list of
        // key blocks; packed sequences start at their own first pattern row
        const int qb = ((ti.m * 2 * p.sub_pos) >> 7) + (p.blk_off ? __ldg(p.blk_off + ti.b) : 0);
        // an empty slot of the balanced order is no tile at all: no role may touch the
        // unit it decoded to (the softmax warps key their epilogue on `valid`)
        if (none) ti.valid[0] = ti.valid[1] = 0;
        const bool any = ti.valid[0] || ti.valid[1];
        const int r0 = any ? __ldg(p.blk_row_ptr + qb) : 0;
        const int r1 = any ? __ldg(p.blk_row_ptr + qb + 1) : 0;
        ti.kb0 = r0;
#pragma unroll
        for (int i = 0; i < 2; ++i) ti.nblk[i] = ti.valid[i] ? max(r1 - r0, 0) : 0;
    }
    return ti;
}

// Key block of a tile's j-th step: j itself (dense) or the j-th entry of the tile's
// row of the block pattern; an index past the keys is reported and clamped.
template <bool SPARSE>
__device__ __forceinline__ int sparse_block(const PrefillParams& p, const TileInfo& ti, int j) {
    if constexpr (!SPARSE) return j;
    int kb = __ldg(p.blk_col + ti.kb0 + j);
    if (kb < 0 || kb >= (ti.sk + 127) >> 7) {  // key blocks of this sequence
        raise_device_error(kDevBadTile);
        kb = 0;
    }
    return kb;
}

// Wait that ignores the abort flag (used to drain in-flight copies before exit).
__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity) {
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (globaltimer_ns() - t0 > kWaitLimitNs) {
            raise_device_error(kDevWaitTimeout);
            return;
        }
    }
}

// SPARSE = true walks the block pattern of p.blk_row_ptr / p.blk_col; the dense
// instantiation carries none of that code.
template <int HD, bool SPARSE = false, bool FP8 = false, bool WINDOW = false>
__global__ void __launch_bounds__(320, 1)
    prefill_fwd_sm100(const __grid_constant__ CUtensorMap tm_q,
                      const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v,
                      const __grid_constant__ CUtensorMap tm_o, const PrefillParams p) {
    using C = PrefillCfg<HD, FP8>;
    // e4m3 P is stored chunk by chunk over S (no wait for P.V(j-1) in the block loop)
    static_assert(!(FP8 && C::P_OWN), "e4m3 P overlays S");
    constexpr int BN = C::BN;
    constexpr int ST = C::STAGES;
    constexpr int QS = C::Q_STAGES;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
    uint64_t* bar_q_full = bars;                   // [QS]
    uint64_t* bar_q_empty = bar_q_full + QS;       // [QS]
    uint64_t* bar_k_full = bar_q_empty + QS;       // [ST]
    uint64_t* bar_k_empty = bar_k_full + ST;
    uint64_t* bar_v_full = bar_k_empty + ST;
    uint64_t* bar_v_empty = bar_v_full + ST;
    uint64_t* bar_s_full = bar_v_empty + ST;  // [2]
    uint64_t* bar_p_full = bar_s_full + 2;    // [2]
    uint64_t* bar_o_done = bar_p_full + 2;    // [2] O_i += P_i(j) V_j finished (every block)
    uint64_t* bar_drain = bar_o_done + 2;     // MMA completion before exit
    uint64_t* bar_epi = bar_drain + 1;        // [2] a sub-tile's O rows are in shared memory
    uint64_t* bar_ofree = bar_epi + 2;        // [2] the previous O store has read them
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < QS; ++s) {
            mbar_init(bar_q_full + s, 1);
            mbar_init(bar_q_empty + s, 1);
        }
        for (int s = 0; s < ST; ++s) {
            mbar_init(bar_k_full + s, 1);
            mbar_init(bar_k_empty + s, 1);
            mbar_init(bar_v_full + s, 1);
            mbar_init(bar_v_empty + s, 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(bar_s_full + i, 1);
            mbar_init(bar_p_full + i, 128);
            mbar_init(bar_o_done + i, 1);
        }
        mbar_init(bar_drain, 1);
        for (int i = 0; i < 2; ++i) {
            mbar_init(bar_epi + i, 4);
            mbar_init(bar_ofree + i, 1);
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 8) {
        tmem_alloc(tmem_slot, C::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 9) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            tma_prefetch_desc(&tm_q);
            tma_prefetch_desc(&tm_k);
            tma_prefetch_desc(&tm_v);
            uint8_t* sQ = smem + C::OFF_Q;
            uint8_t* sK = smem + C::OFF_K;
            uint8_t* sV = smem + C::OFF_V;
            int qc = 0, kc = 0, vc = 0;
            for (int t = blockIdx.x; t < p.n_units; t += gridDim.x) {
                const TileInfo ti = decode_tile<BN, SPARSE, WINDOW>(p, t);
                const int n = max(ti.nblk[0], ti.nblk[1]);
                if (n == 0) continue;
                const int qs = qc % QS;
                if (!mbar_wait(bar_q_empty + qs, ((qc / QS) & 1) ^ 1, abort_flag))
                    goto producer_done;
                mbar_arrive_expect_tx(bar_q_full + qs,
                                      uint32_t(((ti.nblk[0] > 0) + (ti.nblk[1] > 0)) * C::Q_SUB));
#pragma unroll
                for (int i = 0; i < 2; ++i) {
                    if (ti.nblk[i] == 0) continue;
                    const int y = p.pack ? ti.hu * p.G : ti.hu;
                    const int z = ti.q_row0 + ti.p0[i];
#pragma unroll
                    for (int a = 0; a < C::ATOMS; ++a)
                        tma_load_3d(sQ + qs * C::Q_TILE + i * C::Q_SUB + a * C::ATOM_Q, &tm_q,
                                    bar_q_full + qs, a * C::ATOM_ELEMS, y, z);
                }
                ++qc;
                const int kvh = p.pack ? ti.hu : ti.hu / p.G;
                // the blocks the sub-tiles visit: [0, n), or with a window the union of
                // their ranges (sub-tile 0 holds the earlier positions)
                const int jmin = WINDOW ? (ti.nblk[0] > 0 ? ti.jb0[0] : ti.jb0[1]) : 0;
                for (int j = jmin; j < n; ++j) {
                    const int z = ti.k_row0 + sparse_block<SPARSE>(p, ti, j) * BN;
                    {
                        const int s = kc % ST;
                        if (!mbar_wait(bar_k_empty + s, ((kc / ST) & 1) ^ 1, abort_flag))
                            goto producer_done;
                        mbar_arrive_expect_tx(bar_k_full + s, C::KV_TILE);
#pragma unroll
                        for (int a = 0; a < C::ATOMS; ++a)
                            tma_load_3d(sK + s * C::KV_TILE + a * C::ATOM_KV, &tm_k,
                                        bar_k_full + s, a * C::ATOM_ELEMS, kvh, z);
                        ++kc;
                    }
                    {
                        const int s = vc % ST;
                        if (!mbar_wait(bar_v_empty + s, ((vc / ST) & 1) ^ 1, abort_flag))
                            goto producer_done;
                        mbar_arrive_expect_tx(bar_v_full + s, C::KV_TILE);
#pragma unroll
                        for (int a = 0; a < C::ATOMS; ++a)
                            tma_load_3d(sV + s * C::KV_TILE + a * C::ATOM_KV, &tm_v,
                                        bar_v_full + s, a * C::ATOM_ELEMS, kvh, z);
                        ++vc;
                    }
                }
            }
        producer_done:
            // Every copy this thread issued has landed before the CTA may exit.
            for (int s = 0; s < QS; ++s) {
                const int uq = qc / QS + (s < qc % QS ? 1 : 0);
                if (uq > 0) drain_wait(bar_q_full + s, (uq - 1) & 1);
            }
            for (int s = 0; s < ST; ++s) {
                const int uk = kc / ST + (s < kc % ST ? 1 : 0);  // loads issued into stage s
                if (uk > 0) drain_wait(bar_k_full + s, (uk - 1) & 1);
                const int uv = vc / ST + (s < vc % ST ? 1 : 0);
                if (uv > 0) drain_wait(bar_v_full + s, (uv - 1) & 1);
            }
        }
    } else if (warp == 8) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc_s =
                FP8 ? idesc_e4m3_f32(128, BN, 0, 0) : idesc_bf16_f32(128, BN, 0, 0);
            constexpr uint32_t idesc_o =
                FP8 ? idesc_e4m3_f32(128, HD, 0, 1) : idesc_bf16_f32(128, HD, 0, 1);
            const uint32_t sQ0 = smem_u32(smem + C::OFF_Q);
            const uint32_t sK = smem_u32(smem + C::OFF_K);
            const uint32_t sV = smem_u32(smem + C::OFF_V);
            int qc = 0, kc = 0, vc = 0;
            uint32_t p_phase[2] = {0, 0};
            // Descriptors are built once and advanced by adding (byte offset >> 4) to
            // the start-address field (no carry: shared addresses stay below 256 KB).
            const uint64_t dq0 = sw128_desc(sQ0, 16, 1024);
            const uint64_t dk0 = sw128_desc(sK, 16, 1024);
            const uint64_t dv0 = sw128_desc(sV, C::ATOM_KV, 1024);
            constexpr int NS = HD / C::KSTEP;   // k-steps of S = Q K^T (32 bytes each)
            constexpr int NPV = BN / C::KSTEP;  // k-steps of O += P V
            auto s_step = [&](uint64_t dq, uint64_t dk, int i, int kk) {
                const uint32_t oq = ((kk >> 2) * C::ATOM_Q + (kk & 3) * 32) >> 4;
                const uint32_t ok = ((kk >> 2) * C::ATOM_KV + (kk & 3) * 32) >> 4;
                if constexpr (FP8)
                    umma_ss_f8(tmem + C::s_col(i), dq + oq, dk + ok, idesc_s, kk > 0 ? 1u : 0u);
                else
                    umma_ss(tmem + C::s_col(i), dq + oq, dk + ok, idesc_s, kk > 0 ? 1u : 0u);
            };
            // P: 32 bytes of keys per k-step are 8 TMEM columns in either precision
            auto pv_step = [&](uint64_t dv, int i, int kk, bool accumulate) {
                const uint64_t b = dv + uint64_t((kk * C::KSTEP * 128) >> 4);
                const uint32_t acc = (accumulate || kk > 0) ? 1u : 0u;
                if constexpr (FP8)
                    umma_ts_f8(tmem + C::o_col(i), tmem + C::p_col(i) + kk * 8, b, idesc_o, acc);
                else
                    umma_ts(tmem + C::o_col(i), tmem + C::p_col(i) + kk * 8, b, idesc_o, acc);
            };
            for (int t = blockIdx.x; t < p.n_units; t += gridDim.x) {
                const TileInfo ti = decode_tile<BN, SPARSE, WINDOW>(p, t);
                const int n = max(ti.nblk[0], ti.nblk[1]);
                if (n == 0) continue;
                const int qs = qc % QS;
                if (!mbar_wait(bar_q_full + qs, (qc / QS) & 1, abort_flag)) goto mma_done;
                ++qc;
                const uint64_t dq = dq0 + uint64_t((qs * C::Q_TILE) >> 4);
                if constexpr (WINDOW) {
                    // sub-tile i visits blocks [jb0[i], nblk[i]); the stream covers their
                    // union [jmin, n), and every streamed block is released (a block in a
                    // gap between the two ranges is waited for and handed back unused)
                    const int jmin = ti.nblk[0] > 0 ? ti.jb0[0] : ti.jb0[1];
                    {
                        const int s = kc % ST;
                        if (!mbar_wait(bar_k_full + s, (kc / ST) & 1, abort_flag)) goto mma_done;
                        tc_fence_after();
                        const uint64_t dk = dk0 + uint64_t((s * C::KV_TILE) >> 4);
#pragma unroll
                        for (int i = 0; i < 2; ++i)
                            if (ti.nblk[i] > jmin && ti.jb0[i] == jmin) {
                                const uint64_t dqi = dq + uint64_t((i * C::Q_SUB) >> 4);
#pragma unroll
                                for (int kk = 0; kk < NS; ++kk) s_step(dqi, dk, i, kk);
                                umma_commit(bar_s_full + i);
                            }
                        umma_commit(bar_k_empty + s);
                        ++kc;
                    }
                    for (int j = jmin; j < n; ++j) {
                        const int sv = vc % ST;
                        if (!mbar_wait(bar_v_full + sv, (vc / ST) & 1, abort_flag)) goto mma_done;
                        tc_fence_after();
                        const uint64_t dv = dv0 + uint64_t((sv * C::KV_TILE) >> 4);
                        int sk_next = -1;
                        uint64_t dk = 0;
                        if (j + 1 < n) {
                            sk_next = kc % ST;
                            if (!mbar_wait(bar_k_full + sk_next, (kc / ST) & 1, abort_flag))
                                goto mma_done;
                            dk = dk0 + uint64_t((sk_next * C::KV_TILE) >> 4);
                        }
#pragma unroll
                        for (int i = 0; i < 2; ++i) {
                            const bool act = ti.jb0[i] <= j && j < ti.nblk[i];
                            const bool nxt = ti.jb0[i] <= j + 1 && j + 1 < ti.nblk[i];
                            if (!act && !nxt) continue;
                            if (act) {
                                if (!mbar_wait(bar_p_full + i, p_phase[i], abort_flag))
                                    goto mma_done;
                                p_phase[i] ^= 1;
                                tc_fence_after();
                            }
                            const uint64_t dqi = dq + uint64_t((i * C::Q_SUB) >> 4);
                            const bool acc = j > ti.jb0[i];
                            if constexpr (C::P_OWN) {
                                if (nxt) {
#pragma unroll
                                    for (int kk = 0; kk < NS; ++kk) s_step(dqi, dk, i, kk);
                                    umma_commit(bar_s_full + i);
                                }
                                if (act) {
#pragma unroll
                                    for (int kk = 0; kk < NPV; ++kk) pv_step(dv, i, kk, acc);
                                    umma_commit(bar_o_done + i);
                                }
                            } else {
                                if (act) {
#pragma unroll
                                    for (int kk = 0; kk < NPV; ++kk) pv_step(dv, i, kk, acc);
                                    if (!nxt) umma_commit(bar_o_done + i);
                                }
                                if (nxt) {
#pragma unroll
                                    for (int kk = 0; kk < NS; ++kk) s_step(dqi, dk, i, kk);
                                    umma_commit(bar_s_full + i);
                                }
                            }
                        }
                        umma_commit(bar_v_empty + sv);
                        ++vc;
                        if (sk_next >= 0) {
                            umma_commit(bar_k_empty + sk_next);
                            ++kc;
                        }
                    }
                } else {
                    {
                        const int s = kc % ST;
                        if (!mbar_wait(bar_k_full + s, (kc / ST) & 1, abort_flag)) goto mma_done;
                        tc_fence_after();
                        const uint64_t dk = dk0 + uint64_t((s * C::KV_TILE) >> 4);
#pragma unroll
                        for (int i = 0; i < 2; ++i)
                            if (ti.nblk[i] > 0) {
                                const uint64_t dqi = dq + uint64_t((i * C::Q_SUB) >> 4);
#pragma unroll
                                for (int kk = 0; kk < NS; ++kk) s_step(dqi, dk, i, kk);
                                umma_commit(bar_s_full + i);
                            }
                        umma_commit(bar_k_empty + s);
                        ++kc;
                    }
                    for (int j = 0; j < n; ++j) {
                        const int sv = vc % ST;
                        if (!mbar_wait(bar_v_full + sv, (vc / ST) & 1, abort_flag)) goto mma_done;
                        tc_fence_after();
                        const uint64_t dv = dv0 + uint64_t((sv * C::KV_TILE) >> 4);
                        int sk_next = -1;
                        uint64_t dk = 0;
#pragma unroll
                        for (int i = 0; i < 2; ++i) {
                            if (j >= ti.nblk[i]) continue;
                            const bool more = j + 1 < ti.nblk[i];
                            if (more && sk_next < 0) {
                                sk_next = kc % ST;
                                if (!mbar_wait(bar_k_full + sk_next, (kc / ST) & 1, abort_flag))
                                    goto mma_done;
                                dk = dk0 + uint64_t((sk_next * C::KV_TILE) >> 4);
                            }
                            if (!mbar_wait(bar_p_full + i, p_phase[i], abort_flag)) goto mma_done;
                            p_phase[i] ^= 1;
                            tc_fence_after();
                            // When P has its own columns (D = 64), S_i(j+1) = Q_i K_{j+1}^T is
                            // issued before O_i += P_i(j) V_j, since the softmax needs it first,
                            // and o_done_i is committed after every P.V: the softmax waits for
                            // it before it writes P_i(j+1) or rescales O_i.  When P overlays S,
                            // every P.V step must come before S(j+1) overwrites those columns;
                            // the commit of S(j+1) then also covers P.V(j) (a commit tracks all
                            // earlier MMAs of this thread), so o_done_i is committed only after
                            // the sub-tile's last P.V, for the epilogue.
                            const uint64_t dqi = dq + uint64_t((i * C::Q_SUB) >> 4);
                            if constexpr (C::P_OWN) {
                                // S(j+1) first: the softmax needs it next, P.V(j) only later
                                if (more) {
#pragma unroll
                                    for (int kk = 0; kk < NS; ++kk) s_step(dqi, dk, i, kk);
                                    umma_commit(bar_s_full + i);
                                }
#pragma unroll
                                for (int kk = 0; kk < NPV; ++kk) pv_step(dv, i, kk, j > 0);
                                umma_commit(bar_o_done + i);
                            } else {
#pragma unroll
                                for (int kk = 0; kk < NPV; ++kk) pv_step(dv, i, kk, j > 0);
                                if (!more) umma_commit(bar_o_done + i);
                                if (more) {
#pragma unroll
                                    for (int kk = 0; kk < NS; ++kk) s_step(dqi, dk, i, kk);
                                    umma_commit(bar_s_full + i);
                                }
                            }
                        }
                        umma_commit(bar_v_empty + sv);
                        ++vc;
                        if (sk_next >= 0) {
                            umma_commit(bar_k_empty + sk_next);
                            ++kc;
                        }
                    }
                }
                umma_commit(bar_q_empty + qs);
            }
        mma_done:
            // Wait until every MMA issued by this thread has completed.
            umma_commit(bar_drain);
            drain_wait(bar_drain, 0);
        }
    } else {
        // ------------------------------------------------------------ softmax warps
        const int i = warp >> 2;                       // sub-tile
        const int r = ((warp & 3) << 5) + lane;        // row within the sub-tile
        const uint32_t lane_base = uint32_t((warp & 3) << 5) << 16;
        const uint32_t tS = tmem + lane_base + C::s_col(i);
        const uint32_t tO = tmem + lane_base + C::o_col(i);
        const uint32_t tP = tmem + lane_base + C::p_col(i);
        const float sl2 = p.scale_log2;
        const uint64_t sl2x2 = f2_pack(sl2, sl2);
        uint32_t s_phase = 0, o_phase = 0;
        uint32_t ec = 0;  // O stores issued through the shared-memory box
        for (int t = blockIdx.x; t < p.n_units; t += gridDim.x) {
            const TileInfo ti = decode_tile<BN, SPARSE, WINDOW>(p, t);
            // this warp's sub-tile, selected without runtime array indexing
            const int my_valid = i ? ti.valid[1] : ti.valid[0];
            const int my_p0 = i ? ti.p0[1] : ti.p0[0];
            const int nb = i ? ti.nblk[1] : ti.nblk[0];
            const int my_full = i ? ti.full_blk[1] : ti.full_blk[0];
            // sliding window: this sub-tile's first block, and the blocks below lo_full
            // that hold keys under some row's window
            const int my_jb0 = WINDOW ? (i ? ti.jb0[1] : ti.jb0[0]) : 0;
            const int my_lo_full = WINDOW ? (i ? ti.lo_full[1] : ti.lo_full[0]) : 0;
            if (!my_valid) continue;
            int pos, head;
            if (p.pack) {
                pos = my_p0 + r / p.G;
                head = ti.hu * p.G + (r - (r / p.G) * p.G);
            } else {
                pos = my_p0 + r;
                head = ti.hu;
            }
            const bool row_valid = pos < ti.sq;
            if (p.cu_seqlens && r == 0 &&
                (ti.sq > p.Sq || ti.q_row0 + ti.sq > p.total_rows))
                raise_device_error(kDevBadTile);
            int key_lim = p.causal ? pos + ti.sk - ti.sq + 1 : ti.sk;
            key_lim = min(key_lim, ti.sk);
            // sliding window: the row's first visible key
            const int key_lo = WINDOW ? pos + ti.sk - ti.sq - p.window + 1 : 0;
            float m_run = -INFINITY, l_run = 0.f, l_rnd = 0.f;
            for (int j = my_jb0; j < nb; ++j) {
                if (!mbar_wait_warp(bar_s_full + i, s_phase, abort_flag)) goto softmax_done;
                s_phase ^= 1;
                tc_fence_after();
                uint32_t sr[4][32];
                // S in two halves: the row max of keys 0..63 runs while 64..127 load
                tmem_ld32(tS, sr[0]);
                tmem_ld32(tS + 32, sr[1]);
                tmem_ld_wait();
                reg_fence(sr[0]);
                reg_fence(sr[1]);
                tmem_ld32(tS + 64, sr[2]);
                tmem_ld32(tS + 96, sr[3]);
                // keys of this block past the row's limit (causal diagonal, sequence end)
                int kbj = j;
                bool need_mask = j >= my_full;
                if constexpr (SPARSE) {
                    kbj = sparse_block<SPARSE>(p, ti, j);
                    need_mask = (kbj + 1) * BN > key_lim;
                }
                if constexpr (WINDOW) {
                    if (j < my_lo_full) need_mask = true;
                }
                // the mask reads all four chunks; need_mask can differ between the rows of
                // a warp (block-sparse), and the wait is a warp-wide (.sync.aligned) step
                if (__any_sync(0xffffffffu, need_mask)) {
                    tmem_ld_wait();
                    reg_fence(sr[2]);
                    reg_fence(sr[3]);
                }
                if (need_mask) {
                    const int lim = key_lim - kbj * BN;
                    if constexpr (WINDOW) {
                        // keys before the row's window as well
                        const int lo = key_lo - kbj * BN;
#pragma unroll
                        for (int c = 0; c < 4; ++c)
#pragma unroll
                            for (int e = 0; e < 32; ++e)
                                if (c * 32 + e >= lim || c * 32 + e < lo)
                                    sr[c][e] = __float_as_uint(-INFINITY);
                    } else {
#pragma unroll
                        for (int c = 0; c < 4; ++c)
#pragma unroll
                            for (int e = 0; e < 32; ++e)
                                if (c * 32 + e >= lim) sr[c][e] = __float_as_uint(-INFINITY);
                    }
                }
                // block row max: four independent three-input max chains
                float mx0 = -INFINITY, mx1 = -INFINITY, mx2 = -INFINITY, mx3 = -INFINITY;
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    if (c == 2) {
                        tmem_ld_wait();
                        reg_fence(sr[2]);
                        reg_fence(sr[3]);
                    }
#pragma unroll
                    for (int e = 0; e < 32; e += 8) {
                        mx0 = fmax3(mx0, __uint_as_float(sr[c][e]), __uint_as_float(sr[c][e + 1]));
                        mx1 = fmax3(mx1, __uint_as_float(sr[c][e + 2]),
                                    __uint_as_float(sr[c][e + 3]));
                        mx2 = fmax3(mx2, __uint_as_float(sr[c][e + 4]),
                                    __uint_as_float(sr[c][e + 5]));
                        mx3 = fmax3(mx3, __uint_as_float(sr[c][e + 6]),
                                    __uint_as_float(sr[c][e + 7]));
                    }
                }
                const float mx = fmax3(fmaxf(mx0, mx1), mx2, mx3);
                const float mb = mx * sl2;
                float alpha = 1.f;
                if (mb > m_run + C::RESCALE_THRESHOLD) {
                    alpha = ex2_approx(m_run - mb);
                    m_run = mb;
                }
                const float m_use = (m_run == -INFINITY) ? 0.f : m_run;
                // FP8: p carries 2^P_SHIFT (cancels between O and l; L removes it)
                const uint64_t negm2 = f2_pack(C::P_SHIFT - m_use, C::P_SHIFT - m_use);
                // p = 2^(s*scale*log2e - m); two row sums in fp32: of the exact p (for L)
                // and of the bf16 p the P.V MMA consumes (for O / l).  The second sum
                // takes the bf16 halves either unpacked into paired adds (D = 64) or
                // through the mixed bf16 + f32 add (D = 128), whichever measured faster.
                // When P overlays S, each 32-key chunk of P goes to TMEM as soon as it is
                // packed: S(j) is complete, so P.V(j-1), issued before it, no longer reads
                // those columns.
                uint64_t se0 = 0, se1 = 0, sq0 = 0, sq1 = 0;
                float rq0 = 0.f, rq1 = 0.f, rq2 = 0.f, rq3 = 0.f;
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    uint32_t pk[16];
                    float pprev0 = 0.f, pprev1 = 0.f;  // FP8: the pair before this one
#pragma unroll
                    for (int e = 0; e < 16; ++e) {
                        const uint64_t a = ffma2(f2_pack(__uint_as_float(sr[c][2 * e]),
                                                         __uint_as_float(sr[c][2 * e + 1])),
                                                 sl2x2, negm2);
                        float a0, a1;
                        f2_unpack(a, a0, a1);
                        const float p0 = ex2_approx(a0);
                        const float p1 = ex2_approx(a1);
                        const uint64_t pe = f2_pack(p0, p1);
                        if (e & 1)
                            se1 = fadd2(se1, pe);
                        else
                            se0 = fadd2(se0, pe);
                        if constexpr (FP8) {
                            // four keys per 32-bit column, key order = byte order
                            if (e & 1) pk[e >> 1] = pack_e4m3x4(pprev0, pprev1, p0, p1);
                            pprev0 = p0;
                            pprev1 = p1;
                            continue;
                        }
                        pk[e] = pack_bf16x2(p0, p1);
                        if constexpr (HD == 128) {
                            if (e & 1)
                                add_bf16x2_to_f32(pk[e], rq2, rq3);
                            else
                                add_bf16x2_to_f32(pk[e], rq0, rq1);
                        } else {
                            const uint64_t pr = f2_pack(bf16_lo(pk[e]), bf16_hi(pk[e]));
                            if (e & 1)
                                sq1 = fadd2(sq1, pr);
                            else
                                sq0 = fadd2(sq0, pr);
                        }
                    }
                    if constexpr (FP8) {
                        tmem_st8(tP + c * 8, *reinterpret_cast<const uint32_t(*)[8]>(pk));
                    } else if constexpr (!C::P_OWN) {
                        tmem_st16(tP + c * 16, pk);
                    } else {
#pragma unroll
                        for (int e = 0; e < 16; ++e) sr[c >> 1][(c & 1) * 16 + e] = pk[e];
                    }
                }
                if constexpr (HD == 128 && !FP8) sq0 = f2_pack(rq0 + rq2, rq1 + rq3);
                if constexpr (C::P_OWN) {
                    // P in its own 64 columns: P.V(j-1), issued after S(j), has to finish
                    // before P is overwritten or O rescaled
                    if (j > my_jb0) {
                        if (!mbar_wait_warp(bar_o_done + i, o_phase, abort_flag))
                            goto softmax_done;
                        o_phase ^= 1;
                        tc_fence_after();
                    }
                    tmem_st32(tP, sr[0]);
                    tmem_st32(tP + 32, sr[1]);
                }
                float lsum, lrnd;
                {
                    float x0, x1, y0, y1;
                    f2_unpack(fadd2(se0, se1), x0, x1);
                    f2_unpack(fadd2(sq0, sq1), y0, y1);
                    lsum = x0 + x1;
                    // FP8: O is normalised by the sum of the unrounded p
                    lrnd = FP8 ? lsum : y0 + y1;
                }
                l_run = l_run * alpha + lsum;
                l_rnd = l_rnd * alpha + lrnd;
                if (j > my_jb0 && __any_sync(0xffffffffu, alpha != 1.f)) {
                    const uint64_t al2 = f2_pack(alpha, alpha);
#pragma unroll 1
                    for (int c = 0; c < HD / 32; ++c) {
                        uint32_t o[32];
                        tmem_ld32(tO + c * 32, o);
                        tmem_ld_wait();
                        reg_fence(o);
#pragma unroll
                        for (int e = 0; e < 32; e += 2) {
                            float u0, u1;
                            f2_unpack(fmul2(f2_pack(__uint_as_float(o[e]),
                                                    __uint_as_float(o[e + 1])),
                                            al2),
                                      u0, u1);
                            o[e] = __float_as_uint(u0);
                            o[e + 1] = __float_as_uint(u1);
                        }
                        tmem_st32(tO + c * 32, o);
                    }
                }
                tmem_st_wait();
                tc_fence_before();
                mbar_arrive(bar_p_full + i);
            }
            // ---------------------------------------------------------- epilogue
            {
                const size_t row = size_t(ti.q_row0 + pos) * p.Hq + head;
                if (nb > my_jb0) {
                    if (!mbar_wait_warp(bar_o_done + i, o_phase, abort_flag)) goto softmax_done;
                    o_phase ^= 1;
                    tc_fence_after();
                }
                // FP8: o_scale = v_scale (the V codes' unit)
                const float inv_l = (l_rnd > 0.f) ? (FP8 ? p.o_scale : 1.f) / l_rnd : 0.f;
                // a sub-tile whose 128 rows are all real leaves through one TMA store
                const bool tma_out = C::EPI_TMA && (my_p0 + p.sub_pos <= ti.sq);
                if constexpr (C::EPI_TMA) {
                    if (tma_out) {
                        uint8_t* stage = smem + C::OFF_O + i * C::O_SUB;
                        const uint32_t st_row = smem_u32(stage) + uint32_t(r) * 128u;
                        if (ec > 0) {  // the previous store has finished reading the box
                            if (r == 0) {
                                bulk_wait_read();
                                mbar_arrive(bar_ofree + i);
                            }
                            if (!mbar_wait_warp(bar_ofree + i, (ec - 1) & 1, abort_flag))
                                goto softmax_done;
                        }
#pragma unroll 1
                        for (int c = 0; c < HD / 32; ++c) {
                            uint32_t o[32];
                            if (nb > my_jb0) {
                                tmem_ld32(tO + c * 32, o);
                                tmem_ld_wait();
                                reg_fence(o);
                            } else {
#pragma unroll
                                for (int e = 0; e < 32; ++e) o[e] = 0u;
                            }
                            uint32_t w[16];
#pragma unroll
                            for (int e = 0; e < 16; ++e)
                                w[e] = pack_bf16x2(__uint_as_float(o[2 * e]) * inv_l,
                                                   __uint_as_float(o[2 * e + 1]) * inv_l);
                            // 16-byte chunk q of the row sits at q ^ (row % 8) (128B swizzle)
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                const uint32_t q = uint32_t(c * 4 + e);
                                st_shared_v4(st_row + ((q ^ uint32_t(r & 7)) << 4), w[4 * e],
                                             w[4 * e + 1], w[4 * e + 2], w[4 * e + 3]);
                            }
                        }
                        fence_proxy_async();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(bar_epi + i);
                        bool ok = true;
                        if (r == 0) ok = mbar_wait(bar_epi + i, ec & 1, abort_flag);
                        if (!__all_sync(0xffffffffu, ok)) goto softmax_done;
                        if (r == 0) {
                            tma_store_3d(&tm_o, stage, 0, p.pack ? ti.hu * p.G : ti.hu,
                                         ti.q_row0 + my_p0);
                            bulk_commit();
                        }
                        ++ec;
                    }
                }
#pragma unroll 1
                for (int c = 0; c < HD / 32 && !tma_out; ++c) {
                    uint32_t o[32];
                    if (nb > my_jb0) {
                        tmem_ld32(tO + c * 32, o);
                        tmem_ld_wait();
                        reg_fence(o);
                    } else {
#pragma unroll
                        for (int e = 0; e < 32; ++e) o[e] = 0u;
                    }
                    if (row_valid) {
                        uint32_t w[16];
#pragma unroll
                        for (int e = 0; e < 16; ++e)
                            w[e] = pack_bf16x2(__uint_as_float(o[2 * e]) * inv_l,
                                               __uint_as_float(o[2 * e + 1]) * inv_l);
                        uint4* dst = reinterpret_cast<uint4*>(p.out + row * HD + c * 32);
#pragma unroll
                        for (int e = 0; e < 4; ++e)
                            dst[e] = make_uint4(w[4 * e], w[4 * e + 1], w[4 * e + 2], w[4 * e + 3]);
                    }
                }
                if (row_valid) {
                    const float L = (l_run > 0.f)
                                        ? (m_run - C::P_SHIFT + __log2f(l_run)) *
                                              0.69314718055994531f
                                        : -INFINITY;
                    size_t li;
                    if (p.cu_seqlens)
                        li = size_t(head) * p.total_rows + ti.q_row0 + pos;
                    else
                        li = (size_t(ti.b) * p.Hq + head) * p.lse_ld + pos;
                    p.lse[li] = L;
                }
            }
        }
    softmax_done:
        // the thread that issued O stores waits for them before the CTA may exit
        if constexpr (C::EPI_TMA) {
            if (r == 0) bulk_wait_all();
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 8) tmem_dealloc(tmem, C::TMEM_COLS);
}

}  // namespace gqa
