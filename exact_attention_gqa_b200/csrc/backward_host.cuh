// Host side of the backward entry points declared in include/gqa_attn.h
// (gqa_attn_bwd_workspace_bytes, gqa_attn_bwd).  Included at the end of gqa_attn.cu,
// whose argument checks, device table, workspace registry and shared-memory limit
// helpers it uses; kept apart so the forward's translation unit text does not change
// with the backward.
#pragma once
#include "backward_tc.cuh"

#ifndef GQA_BWD_EW
#define GQA_BWD_EW 8
#endif

extern "C" {

size_t gqa_attn_bwd_workspace_bytes(int B, int Hq, int Sq) {
    if (B <= 0 || Hq <= 0 || Sq <= 0) return 0;
    return (size_t(B) * Hq * Sq * 4 + 255) / 256 * 256;
}

int gqa_attn_bwd(const void* q, const void* k, const void* v, const void* out, const float* lse,
                 const void* dout, void* dq, void* dk, void* dv, int B, int Hq, int Hkv, int Sq,
                 int Sk, int D, float scale, int causal, cudaStream_t stream) {
    int rc = check_shape(B, Hq, Hkv, Sq, Sk, D, scale, 1, -1, false, false);
    if (rc != GQA_OK) return rc;
    if (B > 65535 || Hq > 65535) return GQA_ERR_SHAPE;  // grid dimensions
    if (B == 0 || (Sq == 0 && Sk == 0)) return GQA_OK;
    if ((Sq > 0 && (!q || !out || !lse || !dout || !dq)) || (Sk > 0 && (!k || !v || !dk || !dv)))
        return GQA_ERR_NULL;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16) ||
        !aligned(dout, 16) || !aligned(dq, 16) || !aligned(dk, 16) || !aligned(dv, 16) ||
        !aligned(lse, 4))
        return GQA_ERR_ALIGN;
    DeviceInfo* di = nullptr;
    rc = device_info(&di);
    if (rc != GQA_OK) return rc;
    // nothing flows where one side is empty: the other side's gradient is zero
    if (Sq == 0 || Sk == 0) {
        const size_t qb = size_t(B) * Sq * Hq * D * 2, kb = size_t(B) * Sk * Hkv * D * 2;
        if ((qb && cudaMemsetAsync(dq, 0, qb, stream) != cudaSuccess) ||
            (kb && (cudaMemsetAsync(dk, 0, kb, stream) != cudaSuccess ||
                    cudaMemsetAsync(dv, 0, kb, stream) != cudaSuccess)))
            return GQA_ERR_CUDA;
        return GQA_OK;
    }
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return GQA_ERR_CUDA;
    Workspace ws;
    {
        std::lock_guard<std::mutex> lk(g_mu);
        ws = g_ws[dev];
    }
    if (!ws.ptr || ws.bytes < gqa_attn_bwd_workspace_bytes(B, Hq, Sq)) return GQA_ERR_WORKSPACE;
    gqa::BwdParams p;  // D = rowsum(dO * O)
    p.o = static_cast<const __nv_bfloat16*>(out);
    p.dout = static_cast<const __nv_bfloat16*>(dout);
    p.dvec = static_cast<float*>(ws.ptr);
    p.B = B;
    p.Hq = Hq;
    p.Sq = Sq;
    gqa::BwdTcParams tp;
    tp.lse = lse;
    tp.dvec = static_cast<const float*>(ws.ptr);
    tp.B = B;
    tp.Hq = Hq;
    tp.Hkv = Hkv;
    tp.Sq = Sq;
    tp.Sk = Sk;
    tp.G = Hq / Hkv;
    tp.causal = causal ? 1 : 0;
    tp.scale = scale;
    tp.scale_log2 = scale * kLog2e;
    // [rows, heads, D] views: 128-row boxes for the resident tiles; the streamed blocks
    // are 64 query rows (dK/dV launch) and 96 key rows (dQ launch)
    constexpr int NQB = gqa::BwdTcCfg<128, false, GQA_BWD_EW>::N;
    constexpr int NKB = gqa::BwdTcCfg<128, true, GQA_BWD_EW>::N;
    static_assert(NQB == gqa::BwdTcCfg<64, false, GQA_BWD_EW>::N &&
                      NKB == gqa::BwdTcCfg<64, true, GQA_BWD_EW>::N,
                  "block rows do not depend on D");
    CUtensorMap mq128, mo128, mk128, mv128, mqs, mos, mks, mvs;
    const long long rq = (long long)B * Sq, rk = (long long)B * Sk;
    if (!make_map(&mq128, q, rq, Hq, D, 1, 128) || !make_map(&mo128, dout, rq, Hq, D, 1, 128) ||
        !make_map(&mk128, k, rk, Hkv, D, 1, 128) || !make_map(&mv128, v, rk, Hkv, D, 1, 128) ||
        !make_map(&mqs, q, rq, Hq, D, 1, NQB) || !make_map(&mos, dout, rq, Hq, D, 1, NQB) ||
        !make_map(&mks, k, rk, Hkv, D, 1, NKB) || !make_map(&mvs, v, rk, Hkv, D, 1, NKB))
        return GQA_ERR_CUDA;
    auto launch = [&](auto tag) -> int {
        constexpr int HD = decltype(tag)::value;
        constexpr int EW = GQA_BWD_EW;
        using C1 = gqa::BwdTcCfg<HD, false, EW>;
        using C2 = gqa::BwdTcCfg<HD, true, EW>;
        constexpr int S1 = C1::SMEM, S2 = C2::SMEM;
        const int sh = HD == 64 ? 0 : 1;
        int r = ensure_smem_limit(gqa::bwd_tc<HD, false, EW>, 4096 << sh, S1);
        if (r == GQA_OK) r = ensure_smem_limit(gqa::bwd_tc<HD, true, EW>, 16384 << sh, S2);
        if (r != GQA_OK) return r;
        const long long rows = (long long)B * Sq * Hq;
        gqa::bwd_dot_do_o<HD><<<unsigned((rows + 7) / 8), 256, 0, stream>>>(p);
        gqa::BwdTcParams t1 = tp;
        t1.out0 = static_cast<__nv_bfloat16*>(dk);
        t1.out1 = static_cast<__nv_bfloat16*>(dv);
        gqa::bwd_tc<HD, false, EW><<<dim3((Sk + 127) / 128, Hkv, B), C1::THREADS, S1, stream>>>(
            mk128, mv128, mqs, mos, t1);
        gqa::BwdTcParams t2 = tp;
        t2.out0 = static_cast<__nv_bfloat16*>(dq);
        t2.out1 = nullptr;
        gqa::bwd_tc<HD, true, EW><<<dim3((Sq + 127) / 128, Hq, B), C2::THREADS, S2, stream>>>(
            mq128, mo128, mks, mvs, t2);
        return cudaGetLastError() == cudaSuccess ? GQA_OK : GQA_ERR_CUDA;
    };
    return D == 128 ? launch(std::integral_constant<int, 128>())
                    : launch(std::integral_constant<int, 64>());
}

}  // extern "C"
