// Backward pass on the 5th-generation tensor cores: one kernel template, two roles.
//
// FA-2 summary page, backward paragraph: the outer loop runs over K/V column blocks,
// each accumulating its own dK and dV; dQ is shared between them.  GQA paragraph: dK
// and dV sum over the query heads of a K/V head.  With P recomputed from L and
// D_i = rowsum(dO_i * O_i) (bwd_dot_do_o):
//   dV = P^T dO,  dS = P * (dO V^T - D),  dK = scale dS^T Q,  dQ = scale dS K.
//
// A CTA keeps 128 "resident" rows X, Y in shared memory and streams 64-row blocks A, B
// of the other side past them:
//   dK/dV (DQ = false): X = K, Y = V (128 keys of one K/V head); A = Q, B = dO (64
//     queries of each of the G query heads, every block the causal mask leaves any
//     key of the CTA);  S^T = X A^T, dP^T = Y B^T, dV += P^T B, dK += dS^T A;
//   dQ (DQ = true): X = Q, Y = dO (128 queries of one head); A = K, B = V (64 keys);
//     S = X A^T, dP = Y B^T, dQ += dS A.
// Each row of S (or S^T) is one TMEM lane, so a thread owns one resident row and the
// per-element work needs no exchange between threads:
//   warp 8       TMA producer (X, Y once; A, B and the block's L, D into a ring);
//   warp 9       MMA issuer (tcgen05.mma, one thread) and TMEM owner;
//   warps 0-7    elementwise: warp w reads lanes 32 (w & 3) .. + 31 and one half of
//                the block's 64 columns of S and dP, writes P and dS as bf16 back
//                over the columns it read (the A operand of the accumulating MMAs,
//                read from TMEM), and at the end stores the accumulators.
// TMEM: dK or dQ in columns [0, D), dV in [D, 2D), then two buffers of [S | dP] (64 +
// 64 columns): the MMAs of block t + 1 run while the elementwise warps work on block t.
// dQ is computed by its own launch (DQ = true) so that every output element has one
// writer: no atomics, bit-reproducible results.
#pragma once
#include "backward.cuh"
#include "prefill_sm100.cuh"

namespace gqa {

struct BwdTcParams {
    const float* lse;   // [B, Hq, Sq] natural log
    const float* dvec;  // [B, Hq, Sq] rowsum(dO * O)
    __nv_bfloat16* out0;  // dK [B, Sk, Hkv, D] (DQ = false) or dQ [B, Sq, Hq, D]
    __nv_bfloat16* out1;  // dV [B, Sk, Hkv, D] (DQ = false)
    int B, Hq, Hkv, Sq, Sk, G;
    int causal;
    float scale;
    float scale_log2;  // scale * log2(e)
};

template <int HD, bool DQ, int EW>
struct BwdTcCfg {
    static constexpr int M = 128;       // resident rows
    // streamed rows per block: the dQ role has TMEM room for two 96-column S/dP pairs
    static constexpr int N = DQ ? 96 : 64;
    static constexpr int NG = EW / 4;   // column groups: warps per TMEM lane quarter
    static constexpr int CW = N / NG;   // columns of S (and dP) per elementwise warp
    static constexpr int THREADS = 32 * (EW + 2);
    static constexpr int CH = HD / 64;  // 64-dimension chunks (one 128-byte swizzle atom wide)
    static constexpr int STAGES = HD == 128 ? (DQ ? 3 : 4) : 6;
    static constexpr int RES_ATOM = M * 128;  // one chunk of a resident tile
    static constexpr int RES_TILE = CH * RES_ATOM;
    static constexpr int STR_ATOM = N * 128;  // one chunk of a streamed block
    static constexpr int STR_TILE = CH * STR_ATOM;
    static constexpr int STAGE = 2 * STR_TILE;  // A and B
    static constexpr int OFF_X = 0;
    static constexpr int OFF_Y = RES_TILE;
    static constexpr int OFF_ST = 2 * RES_TILE;
    static constexpr int OFF_LD = OFF_ST + STAGES * STAGE;  // [STAGES][2][N] fp32: -L log2e, -D
    static constexpr int LD_BYTES = DQ ? 0 : STAGES * 2 * N * 4;
    static constexpr int OFF_BAR = OFF_LD + LD_BYTES;
    static constexpr int NBAR = 1 + 2 * STAGES + 2 + 2 + 1 + 1;
    static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
    static constexpr int SMEM = OFF_MISC + 16 + 1024;  // + slack to align the base to 1 KB
    static constexpr int ACC2 = 0;                      // dK or dQ
    static constexpr int ACC1 = HD;                     // dV
    static constexpr int BUF0 = DQ ? HD : 2 * HD;       // two [S | dP] buffers follow
    static constexpr int BUF = 2 * N;
    static constexpr int TMEM_COLS = 512;
    static_assert(BUF0 + 2 * BUF <= TMEM_COLS, "TMEM columns");
    static_assert(SMEM <= 227 * 1024, "shared memory");
};

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr)
        : "memory");
}
// NC consecutive columns: x32 loads when NC is a multiple of 32, else x16 loads
// (each load starts at a column aligned to its width)
template <int NC>
__device__ __forceinline__ void tmem_ld_cols(uint32_t taddr, uint32_t (&r)[NC]) {
    if constexpr (NC % 32 == 0) {
#pragma unroll
        for (int i = 0; i < NC / 32; ++i)
            tmem_ld32(taddr + 32 * i, *reinterpret_cast<uint32_t(*)[32]>(r + 32 * i));
    } else {
#pragma unroll
        for (int i = 0; i < NC / 16; ++i)
            tmem_ld16(taddr + 16 * i, *reinterpret_cast<uint32_t(*)[16]>(r + 16 * i));
    }
}
// NC consecutive columns (8, 16 or 24): x16 stores, then an x8 store for the rest
template <int NC>
__device__ __forceinline__ void tmem_st_cols(uint32_t taddr, const uint32_t (&r)[NC]) {
#pragma unroll
    for (int i = 0; i < NC / 16; ++i)
        tmem_st16(taddr + 16 * i, *reinterpret_cast<const uint32_t(*)[16]>(r + 16 * i));
    if constexpr (NC % 16 == 8)
        tmem_st8(taddr + NC - 8, *reinterpret_cast<const uint32_t(*)[8]>(r + NC - 8));
}

template <int HD, bool DQ, int EW>
__global__ void __launch_bounds__(BwdTcCfg<HD, DQ, EW>::THREADS, 1)
    bwd_tc(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_y,
           const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
           const BwdTcParams p) {
    using C = BwdTcCfg<HD, DQ, EW>;
    constexpr int N = C::N;
    constexpr int ST = C::STAGES;
    constexpr int CW = C::CW;
    constexpr int WP = EW;      // producer warp
    constexpr int WM = EW + 1;  // MMA warp
    // the elementwise warps confirm block t + 2 has landed before they release block t
    // (so the MMA thread skips that probe); the producer refills block t + 2's stage
    // only after block t + 2 - ST is released, which needs ST >= 3
    static_assert(ST >= 3, "block t + 2 must not wait on block t's release");
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
    uint64_t* bar_x = bars;                   // X and Y landed
    uint64_t* bar_full = bar_x + 1;           // [ST] A, B (and L, D) of a block landed
    uint64_t* bar_empty = bar_full + ST;      // [ST] the block's last MMA finished
    uint64_t* bar_sp = bar_empty + ST;        // [2] S and dP of a buffer computed
    uint64_t* bar_p = bar_sp + 2;             // [2] P and dS of a buffer written (8 warps)
    uint64_t* bar_acc = bar_p + 2;            // every accumulating MMA finished
    uint64_t* bar_drain = bar_acc + 1;        // MMA completion before exit
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);
    float* sLD = reinterpret_cast<float*>(smem + C::OFF_LD);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int b = blockIdx.z;
    const int shift = p.Sk - p.Sq;  // causal: key j visible to query i iff j <= i + shift

    // the CTA's resident rows and the blocks it streams
    int r0, hx, n, nq = 1, blk_first = 0, c = 0;
    if constexpr (DQ) {
        const int nrb = (p.Sq + C::M - 1) / C::M;
        r0 = (nrb - 1 - int(blockIdx.x)) * C::M;  // longest rows first (causal)
        hx = blockIdx.y;                         // query head
        int j_end = p.Sk;
        if (p.causal) j_end = max(0, min(p.Sk, min(r0 + C::M, p.Sq) + shift));
        n = (j_end + N - 1) / N;
    } else {
        r0 = blockIdx.x * C::M;
        c = blockIdx.y;  // K/V head
        hx = c;
        const int i_first = p.causal ? max(0, r0 - shift) : 0;
        blk_first = i_first / N;
        nq = i_first < p.Sq ? (p.Sq + N - 1) / N - blk_first : 0;
        n = nq * p.G;
    }
    // block t: first streamed row, and the head it belongs to
    auto block = [&](int t, int& s0, int& hs) {
        if constexpr (DQ) {
            s0 = t * N;
            hs = hx / p.G;
        } else {
            const int hh = t / nq;
            s0 = (blk_first + t - hh * nq) * N;
            hs = c * p.G + hh;
        }
    };

    if (threadIdx.x == 0) {
        mbar_init(bar_x, 1);
        for (int s = 0; s < ST; ++s) {
            mbar_init(bar_full + s, 1);
            mbar_init(bar_empty + s, 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(bar_sp + i, 1);
            mbar_init(bar_p + i, EW);
        }
        mbar_init(bar_acc, 1);
        mbar_init(bar_drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == WM) {
        tmem_alloc(tmem_slot, C::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == WP) {
        // ------------------------------------------------------------ TMA producer
        const int zx = DQ ? b * p.Sq + r0 : b * p.Sk + r0;
        if (lane == 0 && n > 0) {
            tma_prefetch_desc(&tm_x);
            tma_prefetch_desc(&tm_y);
            tma_prefetch_desc(&tm_a);
            tma_prefetch_desc(&tm_b);
            mbar_arrive_expect_tx(bar_x, 2 * C::RES_TILE);
#pragma unroll
            for (int a = 0; a < C::CH; ++a) {
                tma_load_3d(smem + C::OFF_X + a * C::RES_ATOM, &tm_x, bar_x, a * 64, hx, zx);
                tma_load_3d(smem + C::OFF_Y + a * C::RES_ATOM, &tm_y, bar_x, a * 64, hx, zx);
            }
        }
        int t = 0;
        for (; t < n; ++t) {
            const int s = t % ST;
            if (!mbar_wait_warp(bar_empty + s, ((t / ST) & 1) ^ 1, abort_flag)) break;
            int s0, hs;
            block(t, s0, hs);
            if constexpr (!DQ) {
                // -L (log2 units) and -D of the block's 64 queries; 0 past the end
                const size_t row = (size_t(b) * p.Hq + hs) * p.Sq;
                float* dst = sLD + s * 2 * N;
#pragma unroll
                for (int k = 0; k < N / 32; ++k) {
                    const int i = s0 + k * 32 + lane;
                    const bool ok = i < p.Sq;
                    dst[k * 32 + lane] = ok ? p.lse[row + i] * -1.4426950408889634f : 0.f;
                    dst[N + k * 32 + lane] = ok ? -p.dvec[row + i] : 0.f;
                }
                __syncwarp();
            }
            if (lane == 0) {
                const int zs = DQ ? b * p.Sk + s0 : b * p.Sq + s0;
                uint8_t* st = smem + C::OFF_ST + s * C::STAGE;
                mbar_arrive_expect_tx(bar_full + s, C::STAGE);
#pragma unroll
                for (int a = 0; a < C::CH; ++a) {
                    tma_load_3d(st + a * C::STR_ATOM, &tm_a, bar_full + s, a * 64, hs, zs);
                    tma_load_3d(st + C::STR_TILE + a * C::STR_ATOM, &tm_b, bar_full + s, a * 64,
                                hs, zs);
                }
            }
        }
        // every copy issued has landed before the CTA may exit
        if (lane == 0 && n > 0) {
            drain_wait(bar_x, 0);
            for (int s = 0; s < ST; ++s) {
                const int u = t / ST + (s < t % ST ? 1 : 0);
                if (u > 0) drain_wait(bar_full + s, (u - 1) & 1);
            }
        }
    } else if (warp == WM) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0 && n > 0) {
            constexpr uint32_t idesc_s = idesc_bf16_f32(128, N, 0, 0);
            constexpr uint32_t idesc_acc = idesc_bf16_f32(128, HD, 0, 1);
            const uint32_t sX = smem_u32(smem + C::OFF_X), sY = smem_u32(smem + C::OFF_Y);
            const uint32_t sS = smem_u32(smem + C::OFF_ST);
            const uint64_t dx = sw128_desc(sX, 16, 1024), dy = sw128_desc(sY, 16, 1024);
            const uint64_t dk0 = sw128_desc(sS, 16, 1024);           // K-major (S, dP)
            const uint64_t dm0 = sw128_desc(sS, C::STR_ATOM, 1024);  // MN-major (dV, dK, dQ)
            auto res_off = [](int kk) {
                return uint64_t(((kk >> 2) * C::RES_ATOM + (kk & 3) * 32) >> 4);
            };
            auto str_off = [](int kk) {
                return uint64_t(((kk >> 2) * C::STR_ATOM + (kk & 3) * 32) >> 4);
            };
            // P / dS of stream rows 16 kk .. +15: the packed columns that the warp holding
            // S columns [16 kk / CW * CW, + CW) wrote at the start of its slice
            auto p_col = [](int kk) {
                return uint32_t((16 * kk / CW) * CW + (16 * kk % CW) / 2);
            };
            if (!mbar_wait(bar_x, 0, abort_flag)) goto mma_done;
            for (int t = 0; t <= n; ++t) {
                if (t < n) {
                    const int s = t % ST;
                    // blocks 0 and 1 are waited for here; block t >= 2 was confirmed by
                    // the elementwise warps before they released block t - 2, whose
                    // release this thread has already observed
                    if (t < 2 && !mbar_wait(bar_full + s, (t / ST) & 1, abort_flag))
                        goto mma_done;
                    tc_fence_after();
                    const uint32_t tb = tmem + C::BUF0 + (t & 1) * C::BUF;
                    const uint64_t da = dk0 + uint64_t((s * C::STAGE) >> 4);
                    const uint64_t db = da + uint64_t(C::STR_TILE >> 4);
#pragma unroll
                    for (int kk = 0; kk < HD / 16; ++kk)
                        umma_ss(tb, dx + res_off(kk), da + str_off(kk), idesc_s, kk > 0);
#pragma unroll
                    for (int kk = 0; kk < HD / 16; ++kk)
                        umma_ss(tb + N, dy + res_off(kk), db + str_off(kk), idesc_s, kk > 0);
                    umma_commit(bar_sp + (t & 1));
                }
                if (t > 0) {
                    const int u = t - 1, s = u % ST;
                    if (!mbar_wait(bar_p + (u & 1), (u >> 1) & 1, abort_flag)) goto mma_done;
                    tc_fence_after();
                    const uint32_t tb = tmem + C::BUF0 + (u & 1) * C::BUF;
                    const uint64_t ma = dm0 + uint64_t((s * C::STAGE) >> 4);
                    const uint64_t mb = ma + uint64_t(C::STR_TILE >> 4);
                    if constexpr (!DQ) {
#pragma unroll
                        for (int kk = 0; kk < N / 16; ++kk)
                            umma_ts(tmem + C::ACC1, tb + p_col(kk),
                                    mb + uint64_t((kk * 16 * 128) >> 4), idesc_acc,
                                    (u > 0 || kk > 0) ? 1u : 0u);
                    }
#pragma unroll
                    for (int kk = 0; kk < N / 16; ++kk)
                        umma_ts(tmem + C::ACC2, tb + N + p_col(kk),
                                ma + uint64_t((kk * 16 * 128) >> 4), idesc_acc,
                                (u > 0 || kk > 0) ? 1u : 0u);
                    umma_commit(bar_empty + s);
                }
            }
            umma_commit(bar_acc);
        mma_done:
            umma_commit(bar_drain);
            drain_wait(bar_drain, 0);
        }
    } else {
        // ------------------------------------------------------------ elementwise warps
        const int lq = warp & 3, hf = warp >> 2;
        const int row = lq * 32 + lane;  // resident row of this thread
        const uint32_t lane_base = uint32_t(lq * 32) << 16;
        const uint64_t sl2x2 = f2_pack(p.scale_log2, p.scale_log2);
        // dQ: -L (log2 units) and -D belong to this thread's query row
        uint64_t nl_row = 0, nd_row = 0;
        if constexpr (DQ) {
            const int i = r0 + row;
            if (i < p.Sq) {
                const size_t li = (size_t(b) * p.Hq + hx) * p.Sq + i;
                const float nl = p.lse[li] * -1.4426950408889634f, nd = -p.dvec[li];
                nl_row = f2_pack(nl, nl);
                nd_row = f2_pack(nd, nd);
            }
        }
        bool ok = true;
        for (int t = 0; t < n; ++t) {
            const int bf = t & 1;
            if (!mbar_wait_warp(bar_sp + bf, (t >> 1) & 1, abort_flag)) {
                ok = false;
                break;
            }
            tc_fence_after();
            const uint32_t tS = tmem + lane_base + C::BUF0 + bf * C::BUF + hf * CW;
            uint32_t sr[CW], dr[CW];
            tmem_ld_cols(tS, sr);
            tmem_ld_cols(tS + N, dr);
            int s0, hs;
            block(t, s0, hs);
            const int col0 = s0 + hf * CW;  // first streamed row (column) of this slice
            const float* lcol = nullptr;
            if constexpr (!DQ) {
                const int s = t % ST;
                // -L, -D were written before the block's full barrier completed
                if (!mbar_wait_warp(bar_full + s, (t / ST) & 1, abort_flag)) {
                    tmem_ld_wait();
                    ok = false;
                    break;
                }
                lcol = sLD + s * 2 * N + hf * CW;
            }
            tmem_ld_wait();
            reg_fence(sr);
            reg_fence(dr);
            // causal / ragged masking, decided per warp
            bool need_mask;
            if constexpr (DQ) {
                need_mask = col0 + CW > p.Sk ||
                            (p.causal && col0 + CW - 1 > r0 + lq * 32 + shift);
            } else {
                need_mask = col0 + CW > p.Sq ||
                            (p.causal && r0 + lq * 32 + 31 > col0 + shift);
            }
            uint32_t pp[CW / 2], dd[CW / 2];
#pragma unroll
            for (int e8 = 0; e8 < CW; e8 += 8) {
                uint64_t nl[4], nd[4];
                if constexpr (DQ) {
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        nl[q] = nl_row;
                        nd[q] = nd_row;
                    }
                } else {
                    const float4 l0 = *reinterpret_cast<const float4*>(lcol + e8);
                    const float4 l1 = *reinterpret_cast<const float4*>(lcol + e8 + 4);
                    const float4 d0 = *reinterpret_cast<const float4*>(lcol + N + e8);
                    const float4 d1 = *reinterpret_cast<const float4*>(lcol + N + e8 + 4);
                    nl[0] = f2_pack(l0.x, l0.y);
                    nl[1] = f2_pack(l0.z, l0.w);
                    nl[2] = f2_pack(l1.x, l1.y);
                    nl[3] = f2_pack(l1.z, l1.w);
                    nd[0] = f2_pack(d0.x, d0.y);
                    nd[1] = f2_pack(d0.z, d0.w);
                    nd[2] = f2_pack(d1.x, d1.y);
                    nd[3] = f2_pack(d1.z, d1.w);
                }
#pragma unroll
                for (int e2 = 0; e2 < 8; e2 += 2) {
                    const int e = e8 + e2;
                    float a0, a1;
                    f2_unpack(ffma2(f2_pack(__uint_as_float(sr[e]), __uint_as_float(sr[e + 1])),
                                    sl2x2, nl[e2 >> 1]),
                              a0, a1);
                    float p0 = ex2_approx(a0), p1 = ex2_approx(a1);
                    if (need_mask) {
                        const int c0 = col0 + e;
                        bool v0, v1;
                        if constexpr (DQ) {
                            v0 = c0 < p.Sk && (!p.causal || c0 <= r0 + row + shift);
                            v1 = c0 + 1 < p.Sk && (!p.causal || c0 + 1 <= r0 + row + shift);
                        } else {
                            v0 = c0 < p.Sq && (!p.causal || r0 + row <= c0 + shift);
                            v1 = c0 + 1 < p.Sq && (!p.causal || r0 + row <= c0 + 1 + shift);
                        }
                        if (!v0) p0 = 0.f;
                        if (!v1) p1 = 0.f;
                    }
                    float s0v, s1v;
                    f2_unpack(fmul2(f2_pack(p0, p1),
                                    fadd2(f2_pack(__uint_as_float(dr[e]),
                                                  __uint_as_float(dr[e + 1])),
                                          nd[e2 >> 1])),
                              s0v, s1v);
                    pp[e >> 1] = pack_bf16x2(p0, p1);
                    dd[e >> 1] = pack_bf16x2(s0v, s1v);
                }
            }
            tmem_st_cols(tS, pp);
            tmem_st_cols(tS + N, dd);
            if (t + 2 < n) {  // block t + 2 has landed (see the MMA thread)
                const int s2 = (t + 2) % ST;
                if (!mbar_wait_warp(bar_full + s2, ((t + 2) / ST) & 1, abort_flag)) {
                    tmem_st_wait();
                    ok = false;
                    break;
                }
            }
            tmem_st_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar_p + bf);
        }
        // ------------------------------------------------------------ epilogue
        if (ok && n > 0) ok = mbar_wait_warp(bar_acc, 0, abort_flag);
        if (ok) {
            tc_fence_after();
            const int rg = r0 + row;
            const bool live = DQ ? rg < p.Sq : rg < p.Sk;
            constexpr int NACC = DQ ? 1 : 2;
            constexpr int AW = HD / C::NG;  // accumulator columns per warp
#pragma unroll
            for (int a = 0; a < NACC; ++a) {
                const uint32_t acol = a == 0 ? C::ACC2 : C::ACC1;
                const float mul = a == 0 ? p.scale : 1.f;
                __nv_bfloat16* dst =
                    DQ ? p.out0 + ((size_t(b) * p.Sq + rg) * p.Hq + hx) * HD
                       : (a == 0 ? p.out0 : p.out1) + ((size_t(b) * p.Sk + rg) * p.Hkv + c) * HD;
#pragma unroll
                for (int k = 0; k < AW / 16; ++k) {
                    const int col = hf * AW + k * 16;
                    uint32_t r[16];
                    if (n > 0) {
                        tmem_ld16(tmem + lane_base + acol + col, r);
                        tmem_ld_wait();
                        reg_fence(r);
                    } else {
#pragma unroll
                        for (int e = 0; e < 16; ++e) r[e] = 0u;
                    }
                    if (live) {
                        uint4* o4 = reinterpret_cast<uint4*>(dst + col);
#pragma unroll
                        for (int v = 0; v < 2; ++v)
                            o4[v] = make_uint4(
                                pack_bf16x2(__uint_as_float(r[8 * v]) * mul,
                                            __uint_as_float(r[8 * v + 1]) * mul),
                                pack_bf16x2(__uint_as_float(r[8 * v + 2]) * mul,
                                            __uint_as_float(r[8 * v + 3]) * mul),
                                pack_bf16x2(__uint_as_float(r[8 * v + 4]) * mul,
                                            __uint_as_float(r[8 * v + 5]) * mul),
                                pack_bf16x2(__uint_as_float(r[8 * v + 6]) * mul,
                                            __uint_as_float(r[8 * v + 7]) * mul));
                    }
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == WM) tmem_dealloc(tmem, C::TMEM_COLS);
}

}  // namespace gqa
