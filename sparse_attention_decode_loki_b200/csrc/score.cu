// The (register-staged) low-dimensional score scan of Loki.
//
// Loki (NeurIPS 2024 poster page, TL;DR and "Visual Insights" Figure 1
// caption; briefgpt.xyz abstract page): every cached token is scored on the
// first d principal components only, s_j = q~[:d] . K~_j[:d], with q~ = q P.
//
// The scan is an HBM stream over d of the D columns of each cached row. Each
// row's d columns are covered by L = next_pow2(ceil(d * elem / 16)) lanes,
// one 16-byte vector each; every thread keeps 8 rows in flight. The rows of
// all (batch, KV head) units are laid end to end and split evenly over a
// single wave of CTAs (SM count x resident CTAs), so no wave is partly empty.
// One pass over a KV head's rows serves all G of its query heads.
#include "common.cuh"
#include "launch.h"

namespace loki {

template <class E, int G>
__global__ void __launch_bounds__(256) k_score_lowdim(const float* __restrict__ q_rot,
                                                      const typename E::T* __restrict__ Kt,
                                                      float* __restrict__ scores, int H_q, int H_kv,
                                                      int S, int64_t S_max, int D, int row_len,
                                                      int d, int log2L, int64_t total,
                                                      int64_t per) {
    constexpr int kThreads = 256;
    constexpr int U = 8;
    constexpr int KV = E::kVec;
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int L = 1 << log2L;
    const int sub = lane & (L - 1);
    const int row_in_pass = warp * (32 >> log2L) + (lane >> log2L);
    const int rows_per_pass = kThreads >> log2L;
    const int nvec = (d + KV - 1) / KV;
    const bool lane_on = sub < nvec;
    const int64_t row_bytes = (int64_t)row_len * E::kBytes;
    griddep_wait();  // q_rot comes from the projection kernel
    griddep_launch_dependents();

    int64_t r = (int64_t)blockIdx.x * per;
    const int64_t r_end = min64(r + per, total);
    while (r < r_end) {
        const int64_t unit = r / S;
        const int s0 = (int)(r - unit * S);
        const int seg = (int)min64(r_end - r, (int64_t)S - s0);
        const int b = (int)(unit / H_kv);
        const int hk = (int)(unit % H_kv);
        const int64_t qrow0 = (int64_t)b * H_q + (int64_t)hk * G;

        float qv[G][KV];
#pragma unroll
        for (int g = 0; g < G; ++g) {
            const float* qp = q_rot + (qrow0 + g) * D + sub * KV;
#pragma unroll
            for (int e = 0; e < KV; ++e) {
                const int col = sub * KV + e;
                qv[g][e] = (lane_on && col < d) ? __ldg(qp + e) : 0.f;
            }
        }
        const char* base =
            reinterpret_cast<const char*>(Kt) + (unit * S_max + s0) * row_bytes + sub * 16;
        float* srow = scores + qrow0 * S + s0;

        for (int p = 0; p < seg; p += rows_per_pass * U) {
            uint4 v[U];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int row = p + u * rows_per_pass + row_in_pass;
                if (lane_on && row < seg)
                    v[u] = ld_stream(base + (int64_t)row * row_bytes);
                else
                    v[u] = make_uint4(0u, 0u, 0u, 0u);
            }
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int row = p + u * rows_per_pass + row_in_pass;
                float f[KV];
                E::unpack(v[u], f);
#pragma unroll
                for (int g = 0; g < G; ++g) {
                    float a = 0.f;
#pragma unroll
                    for (int e = 0; e < KV; ++e) a = fmaf(qv[g][e], f[e], a);
                    a = group_sum_rt(a, L);
                    if (sub == 0 && row < seg) srow[(int64_t)g * S + row] = a;
                }
            }
        }
        r += seg;
    }
}

template <class E, int G>
static cudaError_t score_impl(const float* q_rot, const void* Kt, int B, int H_q, int H_kv,
                              int64_t S, int64_t S_max, int D, int row, int d, float* scores,
                              cudaStream_t s, bool pdl) {
    DevInfo di;
    cudaError_t e = dev_info(&di);
    if (e != cudaSuccess) return e;
    const int nvec = (d + E::kVec - 1) / E::kVec;
    int log2L = 0;
    while ((1 << log2L) < nvec) ++log2L;
    const int64_t total = (int64_t)B * H_kv * S;
    const int64_t min_rows = (int64_t)(256 >> log2L) * 8;  // one unrolled pass
    auto kern = k_score_lowdim<E, G>;
    const int64_t resident = (int64_t)di.sm_count * occupancy((const void*)kern, 256, 0);
    int64_t grid = (total + min_rows - 1) / min_rows;
    if (grid > resident) grid = resident;
    const int64_t per = (total + grid - 1) / grid;
    grid = (total + per - 1) / per;
    return launch_kernel(kern, dim3((unsigned)grid), dim3(256), 0, s, pdl, q_rot,
                         static_cast<const typename E::T*>(Kt), scores, H_q, H_kv, (int)S, S_max,
                         D, row, d, log2L, total, per);
}

template <class E>
static cudaError_t score_dispatch(int G, const float* q_rot, const void* Kt, int B, int H_q,
                                  int H_kv, int64_t S, int64_t S_max, int D, int row, int d,
                                  float* scores, cudaStream_t s, bool pdl) {
    switch (G) {
#define LOKI_G(g) \
    case g:       \
        return score_impl<E, g>(q_rot, Kt, B, H_q, H_kv, S, S_max, D, row, d, scores, s, pdl);
        LOKI_G(1) LOKI_G(2) LOKI_G(3) LOKI_G(4) LOKI_G(5) LOKI_G(6) LOKI_G(7) LOKI_G(8)
#undef LOKI_G
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_score_lowdim(Dt dt, const float* q_rot, const void* Kt, int B, int H_q,
                                int H_kv, int64_t S, int64_t S_max, int D, int row, int d,
                                float* scores, cudaStream_t s, bool pdl) {
    const int G = H_q / H_kv;
    if (dt == kF32)
        return score_dispatch<ElemF32>(G, q_rot, Kt, B, H_q, H_kv, S, S_max, D, row, d, scores, s,
                                       pdl);
    return score_dispatch<ElemBF16>(G, q_rot, Kt, B, H_q, H_kv, S, S_max, D, row, d, scores, s,
                                    pdl);
}

}  // namespace loki
