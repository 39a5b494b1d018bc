// Backward pass of exact grouped-query attention: the shared parameter block and the
// first of its three launches, D_i = rowsum(dO_i * O_i) (FA-2 summary page, backward
// paragraph: with P recomputed from the forward's L, dS = P * (dP - D)).  The dK/dV
// and dQ kernels (tcgen05) follow in backward_tc.cuh.
#pragma once
#include "decode.cuh"

namespace gqa {

struct BwdParams {
    const __nv_bfloat16* o;     // [B, Sq, Hq, D]
    const __nv_bfloat16* dout;  // [B, Sq, Hq, D]
    float* dvec;                // [B, Hq, Sq] workspace: rowsum(dO * O)
    int B, Hq, Sq;
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

}  // namespace gqa
