// fp32 forward of exact grouped-query attention on CUDA cores.
//
// Same definition as the bf16 path (scaled logits, causal mask with the
// diagonal kept and bottom-right alignment, online softmax with a running max
// and a deferred 1/l, L = m + ln l, query head h reading KV head h / G), kept in
// fp32 end to end.  It serves fp32 callers such as the Ultralytics glossary's
// fp32 example (q[1,8,16,64], k/v[1,2,16,64]); it is correct for any size but
// built for small ones: one warp per query row, lanes over keys for the scores
// and over head dimensions for the output.
#pragma once
#include <cstdint>

namespace gqa {

struct F32Params {
    const float* q;
    const float* k;
    const float* v;
    float* out;
    float* lse;
    const int* cu_seqlens;
    int B, Hq, Hkv, Sq, Sk, D;
    int G;
    int total_rows;  // varlen: packed rows (cu_seqlens[B])
    int causal;
    float scale;
    long long n_rows;  // query rows x heads covered by the grid
};

__global__ void __launch_bounds__(128) attn_fwd_f32_simt(const F32Params p) {
    constexpr int MAXD = 256;
    __shared__ float sq[4][MAXD];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long long gw = (long long)blockIdx.x * 4 + warp;
    if (gw >= p.n_rows) return;
    const int h = int(gw % p.Hq);
    const long long row = gw / p.Hq;  // global query row (dense: b*Sq + i; varlen: packed)
    int b, i, sq_len, sk_len;
    long long q_row0, k_row0;
    if (p.cu_seqlens) {
        int lo = 0, hi = p.B;  // find b with cu[b] <= row < cu[b+1]
        while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if (p.cu_seqlens[mid] <= row) lo = mid; else hi = mid;
        }
        b = lo;
        q_row0 = k_row0 = p.cu_seqlens[b];
        sq_len = sk_len = p.cu_seqlens[b + 1] - p.cu_seqlens[b];
        i = int(row - q_row0);
    } else {
        b = int(row / p.Sq);
        i = int(row - (long long)b * p.Sq);
        q_row0 = (long long)b * p.Sq;
        k_row0 = (long long)b * p.Sk;
        sq_len = p.Sq;
        sk_len = p.Sk;
    }
    const int kvh = h / p.G;
    const float* qr = p.q + ((q_row0 + i) * p.Hq + h) * p.D;
    for (int d = lane; d < p.D; d += 32) sq[warp][d] = qr[d];
    __syncwarp();
    int kend = sk_len;
    if (p.causal) kend = min(sk_len, max(0, i + sk_len - sq_len + 1));
    constexpr int PER = MAXD / 32;
    float acc[PER];
#pragma unroll
    for (int e = 0; e < PER; ++e) acc[e] = 0.f;
    float m = -INFINITY, l = 0.f;
    for (int j0 = 0; j0 < kend; j0 += 32) {
        const int j = j0 + lane;
        float s = -INFINITY;
        if (j < kend) {
            const float* kr = p.k + ((k_row0 + j) * p.Hkv + kvh) * p.D;
            float dot = 0.f;
            for (int d = 0; d < p.D; ++d) dot = fmaf(sq[warp][d], kr[d], dot);
            s = dot * p.scale;
        }
        float mx = s;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
        const float m_new = fmaxf(m, mx);
        const float alpha = (m == -INFINITY) ? 0.f : expf(m - m_new);
        const float pj = (s == -INFINITY) ? 0.f : expf(s - m_new);
        float ps = pj;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) ps += __shfl_xor_sync(0xffffffffu, ps, off);
        l = l * alpha + ps;
#pragma unroll
        for (int e = 0; e < PER; ++e) acc[e] *= alpha;
        const int nj = min(32, kend - j0);
        for (int t = 0; t < nj; ++t) {
            const float pt = __shfl_sync(0xffffffffu, pj, t);
            const float* vr = p.v + ((k_row0 + j0 + t) * p.Hkv + kvh) * p.D;
#pragma unroll
            for (int e = 0; e < PER; ++e) {
                const int d = lane + 32 * e;
                if (d < p.D) acc[e] = fmaf(pt, vr[d], acc[e]);
            }
        }
        m = m_new;
    }
    float* orow = p.out + ((q_row0 + i) * p.Hq + h) * p.D;
    const float inv = (l > 0.f) ? 1.f / l : 0.f;
#pragma unroll
    for (int e = 0; e < PER; ++e) {
        const int d = lane + 32 * e;
        if (d < p.D) orow[d] = acc[e] * inv;
    }
    if (lane == 0) {
        const float L = (l > 0.f) ? m + logf(l) : -INFINITY;
        if (p.cu_seqlens)
            p.lse[(long long)h * p.total_rows + q_row0 + i] = L;
        else
            p.lse[((long long)b * p.Hq + h) * p.Sq + i] = L;
    }
}

// O = 0 and L = -inf for every row (a problem with no keys at all).
template <typename T>
__global__ void fill_no_keys(T* out, long long n_out, float* lse, long long n_lse) {
    const long long stride = (long long)gridDim.x * blockDim.x;
    for (long long t = (long long)blockIdx.x * blockDim.x + threadIdx.x; t < n_out; t += stride)
        out[t] = T(0.f);
    for (long long t = (long long)blockIdx.x * blockDim.x + threadIdx.x; t < n_lse; t += stride)
        lse[t] = -INFINITY;
}

}  // namespace gqa
