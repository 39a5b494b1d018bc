// Backward pass of exact grouped-query attention: dQ, dK, dV for a given dO.
//
// FA-2 summary page, backward paragraph: the outer loop runs over column blocks of K
// and V, each accumulating its dK and dV on its own; dQ is shared between column
// blocks.  GQA paragraph: dK and dV are summed over the query heads that share a K/V
// head.  With P recomputed from L (the forward's log-sum-exp, which the same page says
// FA-2 keeps for this pass) and D_i = rowsum(dO_i * O_i):
//   dV = P^T dO,  dS = P * (dO V^T - D),  dK = scale dS^T Q,  dQ = scale dS K.
//
// Three kernels, warp-level bf16 MMAs (m16n8k16, fp32 accumulate) on tiles staged in
// padded shared memory (row stride D + 8 halves: ldmatrix rows land on distinct banks),
// the streamed tiles double-buffered with cp.async (step s + 1 loads while s computes):
//   bwd_dot_do_o  D_i = sum_d dO * O, one warp per row;
//   bwd_dkdv      one CTA per 64 keys of one (batch, K/V head): 4 warps x 16 keys
//                 hold dK and dV in registers while the G query heads and their 32-row
//                 query blocks stream past (blocks the causal mask hides are skipped);
//   bwd_dq        one CTA per 64 queries of one (batch, query head): 4 warps x 16
//                 queries recompute P and dS over 32-key blocks and accumulate dQ.
// Computing dQ in its own pass costs two more products than the page's atomic
// additions into a shared dQ, and gives every output one writer: no atomics, and
// results that do not depend on the order in which blocks finish.
#pragma once
#include "decode.cuh"

namespace gqa {

struct BwdParams {
    const __nv_bfloat16* q;   // [B, Sq, Hq, D]
    const __nv_bfloat16* k;   // [B, Sk, Hkv, D]
    const __nv_bfloat16* v;   // [B, Sk, Hkv, D]
    const __nv_bfloat16* o;   // [B, Sq, Hq, D]
    const __nv_bfloat16* dout;  // [B, Sq, Hq, D]
    const float* lse;         // [B, Hq, Sq] natural log
    float* dvec;              // [B, Hq, Sq] workspace: rowsum(dO * O)
    __nv_bfloat16* dq;        // [B, Sq, Hq, D]
    __nv_bfloat16* dk;        // [B, Sk, Hkv, D]
    __nv_bfloat16* dv;        // [B, Sk, Hkv, D]
    int B, Hq, Hkv, Sq, Sk, G;
    int causal;
    float scale;
    float scale_log2;         // scale * log2(e)
};

// D_i = sum_d dO[i, d] * O[i, d], one warp per (b, i, h) row
template <int HD>
__global__ void __launch_bounds__(256) bwd_dot_do_o(const BwdParams p) {
    const long long row = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    const long long rows = (long long)p.B * p.Sq * p.Hq;
    if (row >= rows) return;
    const __nv_bfloat162* o2 = reinterpret_cast<const __nv_bfloat162*>(p.o + row * HD);
    const __nv_bfloat162* d2 = reinterpret_cast<const __nv_bfloat162*>(p.dout + row * HD);
    float acc = 0.f;
#pragma unroll
    for (int e = lane; e < HD / 2; e += 32) {
        const float2 a = __bfloat1622float2(o2[e]), b = __bfloat1622float2(d2[e]);
        acc = fmaf(a.x, b.x, fmaf(a.y, b.y, acc));
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if (lane == 0) {
        // row = (b * Sq + i) * Hq + h  ->  dvec[(b * Hq + h) * Sq + i]
        const long long h = row % p.Hq, bi = row / p.Hq;
        const long long i = bi % p.Sq, b = bi / p.Sq;
        p.dvec[(b * p.Hq + h) * p.Sq + i] = acc;
    }
}

// ---------------------------------------------------------------------------- helpers
template <int HD>
struct BwdCfg {
    static constexpr int RS = HD + 8;                 // padded row stride (halves)
    static constexpr int ROWB = RS * 2;               // bytes per staged row
};

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) { return pack_bf16x2(lo, hi); }

// Stage rows [r0, r0 + n) of a [rows, H, HD] bf16 tensor (head h, first row base) into
// shared memory with stride RS, by cp.async (16 bytes per copy); rows past `limit` are
// zero-filled, their source clamped to the first row so every address stays valid.
// All threads take part; the caller commits the group.
template <int HD>
__device__ __forceinline__ void stage_rows_async(uint8_t* dst, const __nv_bfloat16* src,
                                                 long long base, int H, int h, int r0, int n,
                                                 int limit) {
    constexpr int CH = HD / 8;
    for (int idx = threadIdx.x; idx < n * CH; idx += blockDim.x) {
        const int r = idx / CH, c = idx - r * CH;
        const bool ok = r0 + r < limit;
        const __nv_bfloat16* gp = src + ((base + (ok ? r0 + r : 0)) * H + h) * HD + c * 8;
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(
                         smem_u32(dst + r * BwdCfg<HD>::ROWB + c * 16)),
                     "l"(gp), "r"(ok ? 16 : 0)
                     : "memory");
    }
}
// n floats (rows r0..r0+n of a [rows] fp32 vector) into shared memory; past `limit`: 0
__device__ __forceinline__ void stage_f32_async(float* dst, const float* src, int r0, int n,
                                                int limit) {
    for (int r = threadIdx.x; r < n; r += blockDim.x) {
        const bool ok = r0 + r < limit;
        asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(smem_u32(dst + r)),
                     "l"(src + (ok ? r0 + r : 0)), "r"(ok ? 4 : 0)
                     : "memory");
    }
}
__device__ __forceinline__ void cp_async_commit() {
    asm volatile("cp.async.commit_group;" ::: "memory");
}
__device__ __forceinline__ void cp_async_wait_prev() {  // all but the newest group landed
    asm volatile("cp.async.wait_group 1;" ::: "memory");
}

// ---------------------------------------------------------------------------- dK, dV
constexpr int kBwdKeys = 64;     // keys per dK/dV CTA (4 warps x 16)
constexpr int kBwdQRows = 32;    // query rows per step of the dK/dV CTA

template <int HD>
__global__ void __launch_bounds__(128) bwd_dkdv(const BwdParams p) {
    using C = BwdCfg<HD>;
    constexpr int KS = HD / 16;            // k-steps over the head dimension
    constexpr int NQ = kBwdQRows / 8;      // n-tiles over a query block
    constexpr int QB = kBwdQRows * C::ROWB;
    extern __shared__ __align__(16) uint8_t smem[];
    uint8_t* sK = smem;
    uint8_t* sV = sK + kBwdKeys * C::ROWB;
    uint8_t* sQ = sV + kBwdKeys * C::ROWB;  // [2] query blocks (double buffer)
    uint8_t* sO = sQ + 2 * QB;              // [2] dO rows
    float* sL = reinterpret_cast<float*>(sO + 2 * QB);  // [2][kBwdQRows] lse (natural log)
    float* sD = sL + 2 * kBwdQRows;                      // [2][kBwdQRows] D_i

    const int j0 = blockIdx.x * kBwdKeys;
    const int c = blockIdx.y;  // K/V head
    const int b = blockIdx.z;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    const int mat = lane >> 3, mrow = lane & 7;
    const int shift = p.Sk - p.Sq;  // causal: key j visible to query i iff j <= i + shift

    // steps: (query head of the group, 32-row query block), skipping blocks the causal
    // mask hides from all of this CTA's keys
    int i_first = 0;
    if (p.causal) i_first = max(0, j0 - shift);
    i_first = (i_first / kBwdQRows) * kBwdQRows;
    const int nqb = i_first < p.Sq ? (p.Sq - i_first + kBwdQRows - 1) / kBwdQRows : 0;
    const int nsteps = nqb * p.G;
    auto load_step = [&](int st) {
        const int hh = st / nqb, i0 = i_first + (st - hh * nqb) * kBwdQRows;
        const int h = c * p.G + hh, buf = st & 1;
        stage_rows_async<HD>(sQ + buf * QB, p.q, (long long)b * p.Sq, p.Hq, h, i0, kBwdQRows,
                             p.Sq);
        stage_rows_async<HD>(sO + buf * QB, p.dout, (long long)b * p.Sq, p.Hq, h, i0,
                             kBwdQRows, p.Sq);
        const size_t lrow = ((size_t)b * p.Hq + h) * p.Sq;
        stage_f32_async(sL + buf * kBwdQRows, p.lse + lrow, i0, kBwdQRows, p.Sq);
        stage_f32_async(sD + buf * kBwdQRows, p.dvec + lrow, i0, kBwdQRows, p.Sq);
    };
    stage_rows_async<HD>(sK, p.k, (long long)b * p.Sk, p.Hkv, c, j0, kBwdKeys, p.Sk);
    stage_rows_async<HD>(sV, p.v, (long long)b * p.Sk, p.Hkv, c, j0, kBwdKeys, p.Sk);
    if (nsteps > 0) load_step(0);
    cp_async_commit();

    float dk[HD / 8][4], dv[HD / 8][4];
#pragma unroll
    for (int n = 0; n < HD / 8; ++n)
#pragma unroll
        for (int e = 0; e < 4; ++e) dk[n][e] = dv[n][e] = 0.f;

    const uint32_t aK = smem_u32(sK), aV = smem_u32(sV);
    // this warp's rows of K (A operand): row warp*16 + (mat & 1) * 8 + mrow, chunk + mat >> 1
    const int a_row = warp * 16 + (mat & 1) * 8 + mrow;

    for (int st = 0; st < nsteps; ++st) {
        if (st + 1 < nsteps) load_step(st + 1);  // into the other buffer
        cp_async_commit();
        cp_async_wait_prev();
        __syncthreads();
        const int hh = st / nqb, i0 = i_first + (st - hh * nqb) * kBwdQRows, buf = st & 1;
        const uint32_t aQ = smem_u32(sQ + buf * QB), aO = smem_u32(sO + buf * QB);
        const float* lq = sL + buf * kBwdQRows;
        const float* dq_ = sD + buf * kBwdQRows;
        // S^T = K_w Q^T and dP^T = V_w dO^T: 16 keys x 32 queries per warp
        float s[NQ][4], dp[NQ][4];
#pragma unroll
        for (int n = 0; n < NQ; ++n)
#pragma unroll
            for (int e = 0; e < 4; ++e) s[n][e] = dp[n][e] = 0.f;
#pragma unroll
        for (int kk = 0; kk < KS; ++kk) {
            uint32_t ak[4], av[4];
            ldsm_x4(aK + a_row * C::ROWB + (kk * 2 + (mat >> 1)) * 16, ak[0], ak[1], ak[2],
                    ak[3]);
            ldsm_x4(aV + a_row * C::ROWB + (kk * 2 + (mat >> 1)) * 16, av[0], av[1], av[2],
                    av[3]);
#pragma unroll
            for (int np = 0; np < NQ / 2; ++np) {
                // B = Q^T / dO^T: query rows np*16 + (mat >> 1) * 8 + mrow, chunk mat & 1
                const int br = np * 16 + (mat >> 1) * 8 + mrow;
                uint32_t b0, b1, b2, b3;
                ldsm_x4(aQ + br * C::ROWB + (kk * 2 + (mat & 1)) * 16, b0, b1, b2, b3);
                mma_bf16_16816(s[2 * np], ak, b0, b1);
                mma_bf16_16816(s[2 * np + 1], ak, b2, b3);
                ldsm_x4(aO + br * C::ROWB + (kk * 2 + (mat & 1)) * 16, b0, b1, b2, b3);
                mma_bf16_16816(dp[2 * np], av, b0, b1);
                mma_bf16_16816(dp[2 * np + 1], av, b2, b3);
            }
        }
        // P^T and dS^T, packed as the A operands of the two accumulating products
        uint32_t pa[NQ / 2][4], sa[NQ / 2][4];
#pragma unroll
        for (int n = 0; n < NQ; ++n) {
            float pv[4], sv[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int key = j0 + warp * 16 + g + 8 * (e >> 1);
                const int qr = n * 8 + 2 * t + (e & 1);  // query row within the block
                const float l2 = lq[qr] * 1.4426950408889634f;
                bool vis = i0 + qr < p.Sq && l2 != -INFINITY && key < p.Sk;
                if (p.causal) vis = vis && key <= i0 + qr + shift;
                const float pr = vis ? exp2f(s[n][e] * p.scale_log2 - l2) : 0.f;
                pv[e] = pr;
                sv[e] = pr * (dp[n][e] - dq_[qr]);
            }
            const int ks = n >> 1, half = (n & 1) * 2;
            pa[ks][half] = pack_bf16(pv[0], pv[1]);
            pa[ks][half + 1] = pack_bf16(pv[2], pv[3]);
            sa[ks][half] = pack_bf16(sv[0], sv[1]);
            sa[ks][half + 1] = pack_bf16(sv[2], sv[3]);
        }
        // dV += P^T dO and dK += dS^T Q over the block's 32 queries
#pragma unroll
        for (int ks = 0; ks < NQ / 2; ++ks) {
#pragma unroll
            for (int dn = 0; dn < HD / 16; ++dn) {
                // B = dO / Q rows (k = queries): row ks*16 + (mat & 1) * 8 + mrow, chunk
                // dn * 2 + (mat >> 1), transposed
                const int br = ks * 16 + (mat & 1) * 8 + mrow;
                uint32_t b0, b1, b2, b3;
                ldsm_x4_t(aO + br * C::ROWB + (dn * 2 + (mat >> 1)) * 16, b0, b1, b2, b3);
                mma_bf16_16816(dv[2 * dn], pa[ks], b0, b1);
                mma_bf16_16816(dv[2 * dn + 1], pa[ks], b2, b3);
                ldsm_x4_t(aQ + br * C::ROWB + (dn * 2 + (mat >> 1)) * 16, b0, b1, b2, b3);
                mma_bf16_16816(dk[2 * dn], sa[ks], b0, b1);
                mma_bf16_16816(dk[2 * dn + 1], sa[ks], b2, b3);
            }
        }
        __syncthreads();  // this buffer is refilled two steps on
    }
    asm volatile("cp.async.wait_group 0;" ::: "memory");  // nothing in flight at exit
    // this warp's rows: keys j0 + warp*16 + g (+ 8); columns n*8 + 2t (+ 1)
#pragma unroll
    for (int hr = 0; hr < 2; ++hr) {
        const int key = j0 + warp * 16 + g + 8 * hr;
        if (key >= p.Sk) continue;
        __nv_bfloat16* dkr = p.dk + (((size_t)b * p.Sk + key) * p.Hkv + c) * HD;
        __nv_bfloat16* dvr = p.dv + (((size_t)b * p.Sk + key) * p.Hkv + c) * HD;
#pragma unroll
        for (int n = 0; n < HD / 8; ++n) {
            *reinterpret_cast<uint32_t*>(dkr + n * 8 + 2 * t) =
                pack_bf16(dk[n][2 * hr] * p.scale, dk[n][2 * hr + 1] * p.scale);
            *reinterpret_cast<uint32_t*>(dvr + n * 8 + 2 * t) =
                pack_bf16(dv[n][2 * hr], dv[n][2 * hr + 1]);
        }
    }
}

// ---------------------------------------------------------------------------- dQ
constexpr int kBwdQ = 64;      // query rows per dQ CTA (4 warps x 16)
constexpr int kBwdKStep = 32;  // keys per step of the dQ CTA

template <int HD>
__global__ void __launch_bounds__(128) bwd_dq(const BwdParams p) {
    using C = BwdCfg<HD>;
    constexpr int KS = HD / 16;
    constexpr int NK = kBwdKStep / 8;      // n-tiles over a key block
    constexpr int KB = kBwdKStep * C::ROWB;
    extern __shared__ __align__(16) uint8_t smem[];
    uint8_t* sQ = smem;
    uint8_t* sO = sQ + kBwdQ * C::ROWB;     // dO rows
    uint8_t* sK = sO + kBwdQ * C::ROWB;     // [2] key blocks (double buffer)
    uint8_t* sV = sK + 2 * KB;              // [2]

    const int i0 = blockIdx.x * kBwdQ;
    const int h = blockIdx.y;
    const int b = blockIdx.z;
    const int c = h / p.G;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    const int mat = lane >> 3, mrow = lane & 7;
    const int shift = p.Sk - p.Sq;

    // keys any query of this block sees
    int j_end = p.Sk;
    if (p.causal) j_end = max(0, min(p.Sk, min(i0 + kBwdQ, p.Sq) + shift));
    const int nsteps = (j_end + kBwdKStep - 1) / kBwdKStep;
    auto load_step = [&](int st) {
        const int buf = st & 1;
        stage_rows_async<HD>(sK + buf * KB, p.k, (long long)b * p.Sk, p.Hkv, c, st * kBwdKStep,
                             kBwdKStep, p.Sk);
        stage_rows_async<HD>(sV + buf * KB, p.v, (long long)b * p.Sk, p.Hkv, c, st * kBwdKStep,
                             kBwdKStep, p.Sk);
    };
    stage_rows_async<HD>(sQ, p.q, (long long)b * p.Sq, p.Hq, h, i0, kBwdQ, p.Sq);
    stage_rows_async<HD>(sO, p.dout, (long long)b * p.Sq, p.Hq, h, i0, kBwdQ, p.Sq);
    if (nsteps > 0) load_step(0);
    cp_async_commit();
    // this thread's two rows: queries i0 + warp*16 + g (+ 8)
    float l2[2], dd[2];
#pragma unroll
    for (int hr = 0; hr < 2; ++hr) {
        const int i = i0 + warp * 16 + g + 8 * hr;
        const size_t li = ((size_t)b * p.Hq + h) * p.Sq + i;
        l2[hr] = i < p.Sq ? p.lse[li] * 1.4426950408889634f : -INFINITY;
        dd[hr] = i < p.Sq ? p.dvec[li] : 0.f;
    }
    float dq[HD / 8][4];
#pragma unroll
    for (int n = 0; n < HD / 8; ++n)
#pragma unroll
        for (int e = 0; e < 4; ++e) dq[n][e] = 0.f;

    const uint32_t aQ = smem_u32(sQ), aO = smem_u32(sO);
    const int a_row = warp * 16 + (mat & 1) * 8 + mrow;

    for (int st = 0; st < nsteps; ++st) {
        if (st + 1 < nsteps) load_step(st + 1);
        cp_async_commit();
        cp_async_wait_prev();
        __syncthreads();
        const int j0 = st * kBwdKStep, buf = st & 1;
        const uint32_t aK = smem_u32(sK + buf * KB), aV = smem_u32(sV + buf * KB);
        // S = Q_w K^T and dP = dO_w V^T: 16 queries x 32 keys per warp
        float s[NK][4], dp[NK][4];
#pragma unroll
        for (int n = 0; n < NK; ++n)
#pragma unroll
            for (int e = 0; e < 4; ++e) s[n][e] = dp[n][e] = 0.f;
#pragma unroll
        for (int kk = 0; kk < KS; ++kk) {
            uint32_t aq[4], ao[4];
            ldsm_x4(aQ + a_row * C::ROWB + (kk * 2 + (mat >> 1)) * 16, aq[0], aq[1], aq[2], aq[3]);
            ldsm_x4(aO + a_row * C::ROWB + (kk * 2 + (mat >> 1)) * 16, ao[0], ao[1], ao[2], ao[3]);
#pragma unroll
            for (int np = 0; np < NK / 2; ++np) {
                const int br = np * 16 + (mat >> 1) * 8 + mrow;
                uint32_t b0, b1, b2, b3;
                ldsm_x4(aK + br * C::ROWB + (kk * 2 + (mat & 1)) * 16, b0, b1, b2, b3);
                mma_bf16_16816(s[2 * np], aq, b0, b1);
                mma_bf16_16816(s[2 * np + 1], aq, b2, b3);
                ldsm_x4(aV + br * C::ROWB + (kk * 2 + (mat & 1)) * 16, b0, b1, b2, b3);
                mma_bf16_16816(dp[2 * np], ao, b0, b1);
                mma_bf16_16816(dp[2 * np + 1], ao, b2, b3);
            }
        }
        // dS = P * (dP - D), packed as the A operand of dQ += dS K
        uint32_t sa[NK / 2][4];
#pragma unroll
        for (int n = 0; n < NK; ++n) {
            float sv[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int hr = e >> 1;
                const int i = i0 + warp * 16 + g + 8 * hr;
                const int key = j0 + n * 8 + 2 * t + (e & 1);
                bool vis = l2[hr] != -INFINITY && key < p.Sk;
                if (p.causal) vis = vis && key <= i + shift;
                const float pr = vis ? exp2f(s[n][e] * p.scale_log2 - l2[hr]) : 0.f;
                sv[e] = pr * (dp[n][e] - dd[hr]);
            }
            const int ks = n >> 1, half = (n & 1) * 2;
            sa[ks][half] = pack_bf16(sv[0], sv[1]);
            sa[ks][half + 1] = pack_bf16(sv[2], sv[3]);
        }
#pragma unroll
        for (int ks = 0; ks < NK / 2; ++ks) {
#pragma unroll
            for (int dn = 0; dn < HD / 16; ++dn) {
                const int br = ks * 16 + (mat & 1) * 8 + mrow;
                uint32_t b0, b1, b2, b3;
                ldsm_x4_t(aK + br * C::ROWB + (dn * 2 + (mat >> 1)) * 16, b0, b1, b2, b3);
                mma_bf16_16816(dq[2 * dn], sa[ks], b0, b1);
                mma_bf16_16816(dq[2 * dn + 1], sa[ks], b2, b3);
            }
        }
        __syncthreads();  // this buffer is refilled two steps on
    }
    cp_async_commit();
    asm volatile("cp.async.wait_group 0;" ::: "memory");  // nothing in flight at exit
#pragma unroll
    for (int hr = 0; hr < 2; ++hr) {
        const int i = i0 + warp * 16 + g + 8 * hr;
        if (i >= p.Sq) continue;
        __nv_bfloat16* dqr = p.dq + (((size_t)b * p.Sq + i) * p.Hq + h) * HD;
#pragma unroll
        for (int n = 0; n < HD / 8; ++n)
            *reinterpret_cast<uint32_t*>(dqr + n * 8 + 2 * t) =
                pack_bf16(dq[n][2 * hr] * p.scale, dq[n][2 * hr + 1] * p.scale);
    }
}

template <int HD>
constexpr int bwd_dkdv_smem() {
    return (2 * kBwdKeys + 4 * kBwdQRows) * BwdCfg<HD>::ROWB + 4 * kBwdQRows * 4;
}
template <int HD>
constexpr int bwd_dq_smem() {
    return (2 * kBwdQ + 4 * kBwdKStep) * BwdCfg<HD>::ROWB;
}

}  // namespace gqa
