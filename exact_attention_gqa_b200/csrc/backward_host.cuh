// Host side of the backward entry points declared in include/gqa_attn.h
// (gqa_attn_bwd_workspace_bytes, gqa_attn_bwd).  Included at the end of gqa_attn.cu,
// whose argument checks, device table, workspace registry and shared-memory limit
// helpers it uses; kept apart so the forward's translation unit text does not change
// with the backward.
#pragma once
#include "backward.cuh"

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
    gqa::BwdParams p;
    p.q = static_cast<const __nv_bfloat16*>(q);
    p.k = static_cast<const __nv_bfloat16*>(k);
    p.v = static_cast<const __nv_bfloat16*>(v);
    p.o = static_cast<const __nv_bfloat16*>(out);
    p.dout = static_cast<const __nv_bfloat16*>(dout);
    p.lse = lse;
    p.dvec = static_cast<float*>(ws.ptr);
    p.dq = static_cast<__nv_bfloat16*>(dq);
    p.dk = static_cast<__nv_bfloat16*>(dk);
    p.dv = static_cast<__nv_bfloat16*>(dv);
    p.B = B;
    p.Hq = Hq;
    p.Hkv = Hkv;
    p.Sq = Sq;
    p.Sk = Sk;
    p.G = Hq / Hkv;
    p.causal = causal ? 1 : 0;
    p.scale = scale;
    p.scale_log2 = scale * kLog2e;
    auto launch = [&](auto tag) -> int {
        constexpr int HD = decltype(tag)::value;
        constexpr int S1 = gqa::bwd_dkdv_smem<HD>(), S2 = gqa::bwd_dq_smem<HD>();
        const int sh = HD == 64 ? 0 : 1;
        int r = ensure_smem_limit(gqa::bwd_dkdv<HD>, 4096 << sh, S1);
        if (r == GQA_OK) r = ensure_smem_limit(gqa::bwd_dq<HD>, 16384 << sh, S2);
        if (r != GQA_OK) return r;
        const long long rows = (long long)B * Sq * Hq;
        gqa::bwd_dot_do_o<HD><<<unsigned((rows + 7) / 8), 256, 0, stream>>>(p);
        gqa::bwd_dkdv<HD><<<dim3((Sk + gqa::kBwdKeys - 1) / gqa::kBwdKeys, Hkv, B), 128, S1,
                            stream>>>(p);
        gqa::bwd_dq<HD><<<dim3((Sq + gqa::kBwdQ - 1) / gqa::kBwdQ, Hq, B), 128, S2, stream>>>(p);
        return cudaGetLastError() == cudaSuccess ? GQA_OK : GQA_ERR_CUDA;
    };
    return D == 128 ? launch(std::integral_constant<int, 128>())
                    : launch(std::integral_constant<int, 64>());
}

}  // extern "C"
