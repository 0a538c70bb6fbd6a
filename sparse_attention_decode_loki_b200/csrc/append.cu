// KV-cache append with key rotation: K~ = K_new P into the cache, V copied.
// NeurIPS 2024 poster page, "Loki's Computational Cost": keys are appended to
// the KV-cache at every decode step (named there as a limiting cost); "Visual
// Insights" Figure 1 caption: keys are used through their PCA projection.
//
// One CTA per (block of up to 8 tokens, KV head, batch); thread c owns output
// column c for all tokens of the block, so each P[h][i][c] read from L2 is
// used 8 times. fp32 accumulation in index order, rounded once to the cache
// type (nearest-even).
#include "common.cuh"
#include "launch.h"

namespace loki {

constexpr int kAppendTokens = 8;

template <class E>
__global__ void __launch_bounds__(128) k_rotate_append(const typename E::T* __restrict__ K_new,
                                                       const typename E::T* __restrict__ V_new,
                                                       const float* __restrict__ P,
                                                       typename E::T* __restrict__ Kt_cache,
                                                       typename E::T* __restrict__ V_cache,
                                                       typename E::T* __restrict__ Kt_lo, int d_lo,
                                                       int H_kv, int T, int D, int64_t S_max,
                                                       int64_t pos) {
    __shared__ float kin[kAppendTokens][128];
    const int t0 = blockIdx.x * kAppendTokens;
    const int h = blockIdx.y, b = blockIdx.z;
    const int c = threadIdx.x;
    const int64_t unit = (int64_t)b * H_kv + h;
    const int nt = min(kAppendTokens, T - t0);
    for (int t = 0; t < kAppendTokens; ++t) {
        float x = 0.f;
        if (t < nt && c < D) x = E::load1(K_new + (unit * T + t0 + t) * D + c);
        kin[t][c] = x;
    }
    __syncthreads();
    if (c >= D) return;
    float acc[kAppendTokens];
#pragma unroll
    for (int t = 0; t < kAppendTokens; ++t) acc[t] = 0.f;
    const float* Ph = P + (int64_t)h * D * D + c;
    for (int i = 0; i < D; ++i) {
        const float p = __ldg(Ph + (int64_t)i * D);
#pragma unroll
        for (int t = 0; t < kAppendTokens; ++t) acc[t] = fmaf(kin[t][i], p, acc[t]);
    }
    for (int t = 0; t < nt; ++t) {
        const int64_t row = unit * S_max + pos + t0 + t;
        const typename E::T kt = E::from_float(acc[t]);
        Kt_cache[row * D + c] = kt;
        V_cache[row * D + c] = V_new[(unit * T + t0 + t) * D + c];
        if (Kt_lo != nullptr && c < d_lo) Kt_lo[row * d_lo + c] = kt;
    }
}

cudaError_t launch_append(Dt dt, const void* K_new, const void* V_new, const float* P,
                          void* Kt_cache, void* V_cache, void* Kt_lo, int d_lo, int B, int H_kv,
                          int T, int D, int64_t S_max, int64_t pos, cudaStream_t s) {
    dim3 grid((T + kAppendTokens - 1) / kAppendTokens, H_kv, B), block(128);
    if (dt == kF32)
        k_rotate_append<ElemF32><<<grid, block, 0, s>>>(
            static_cast<const float*>(K_new), static_cast<const float*>(V_new), P,
            static_cast<float*>(Kt_cache), static_cast<float*>(V_cache),
            static_cast<float*>(Kt_lo), d_lo, H_kv, T, D, S_max, pos);
    else
        k_rotate_append<ElemBF16><<<grid, block, 0, s>>>(
            static_cast<const __nv_bfloat16*>(K_new), static_cast<const __nv_bfloat16*>(V_new), P,
            static_cast<__nv_bfloat16*>(Kt_cache), static_cast<__nv_bfloat16*>(V_cache),
            static_cast<__nv_bfloat16*>(Kt_lo), d_lo, H_kv, T, D, S_max, pos);
    return cudaGetLastError();
}

}  // namespace loki
