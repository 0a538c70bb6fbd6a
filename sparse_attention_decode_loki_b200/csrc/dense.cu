// Dense decode attention over all S cached tokens: the full-attention
// baseline of every Loki comparison (NeurIPS 2024 poster page, "More on
// tables": full-attention rows; "More on figures": per-layer attention time
// of vanilla attention against Loki).
//
// Flash-decoding split over the sequence: the rows of all (batch, KV head)
// units are laid end to end and split evenly over one wave of CTAs. A row
// group of lanes streams contiguous key and value rows (16-byte vectors, 2-4
// rows in flight per group) and keeps an online softmax for each of the G
// query heads of its KV head, so every key/value byte is read once for all G
// heads. Partials are merged by k_combine.
//
// The same kernel computes PCAAttn, the variant of Loki that applies the
// softmax directly to the reduced-dimensional scores of every token (poster
// page, "More on tables", PCAAttn table caption): the key of token j is then
// its row of the low-dimensional key plane (d_lo columns, read by the first
// d_lo * elem / 16 lanes of the row group) and the query is q~[:d], so the
// score is s_j = q~[:d] . K~_j[:d]; the values are read in full.
#include "combine.cuh"
#include "common.cuh"
#include "launch.h"

namespace loki {

constexpr int kDenseMinRows = 256;

// per >= kDenseMinRows / 2 (see sparse_max_parts for the argument)
int64_t dense_max_parts(int64_t S) { return (S - 1) / (kDenseMinRows / 2) + 2; }

// NVK = 0: dense attention, keys are full rows and q is of type E::T.
// NVK > 0: PCAAttn, keys are plane rows of NVK 16-byte chunks and the query is
// q_rot (fp32 q~), of which the first d columns count.
// DH: head dimension (96 or 128). The lanes keep the layout of 128 columns;
// those past DH load nothing and write nothing.
template <class E, int G, int NVK, int DH>
__global__ void __launch_bounds__(256) k_dense(const typename E::T* __restrict__ q,
                                               const float* __restrict__ q_rot, int d,
                                               const typename E::T* __restrict__ K,
                                               const typename E::T* __restrict__ V, int H_q,
                                               int H_kv, int S, int64_t S_max, float scale_log2,
                                               int64_t total, int64_t per, int maxp,
                                               float2* __restrict__ part_ml,
                                               float* __restrict__ part_acc) {
    constexpr int D = DH;
    constexpr int KV = E::kVec;
    constexpr int LPR = 128 / KV;
    constexpr int NGRP = 256 / LPR;
    constexpr int U = G <= 2 ? 4 : 2;
    constexpr int64_t kRowBytes = (int64_t)D * E::kBytes;
    constexpr int64_t kKeyBytes = NVK == 0 ? kRowBytes : (int64_t)NVK * 16;
    __shared__ float sm_m[G][NGRP], sm_l[G][NGRP];
    __shared__ float sm_acc[NGRP][128];

    const int grp = threadIdx.x / LPR;
    const int sub = threadIdx.x % LPR;
    const bool lane_on = sub * KV < D;
    griddep_launch_dependents();  // lets the combine kernel be scheduled early
    if constexpr (NVK > 0) griddep_wait();  // q~ comes from the projection kernel

    int64_t w = (int64_t)blockIdx.x * per;
    const int64_t w_end = min64(w + per, total);
    while (w < w_end) {
        const int64_t unit = w / S;
        const int s0 = (int)(w - unit * S);
        const int seg = (int)min64(w_end - w, (int64_t)S - s0);
        const int b = (int)(unit / H_kv), hk = (int)(unit % H_kv);

        float qv[G][KV];
#pragma unroll
        for (int g = 0; g < G; ++g) {
            const int64_t qr = (int64_t)b * H_q + (int64_t)hk * G + g;
            if constexpr (NVK == 0) {
                const typename E::T* qp = q + qr * D + sub * KV;
#pragma unroll
                for (int e = 0; e < KV; ++e) qv[g][e] = lane_on ? E::load1(qp + e) * scale_log2 : 0.f;
            } else {
#pragma unroll
                for (int e = 0; e < KV; ++e) {
                    const int col = sub * KV + e;
                    qv[g][e] = (sub < NVK && col < d) ? __ldg(q_rot + qr * D + col) * scale_log2
                                                      : 0.f;
                }
            }
        }
        // this lane reads part of the key row
        const bool k_lane = NVK == 0 ? lane_on : sub < NVK;
        const char* Kb = reinterpret_cast<const char*>(K) + (unit * S_max + s0) * kKeyBytes +
                         (k_lane ? sub * 16 : 0);
        const char* Vb = reinterpret_cast<const char*>(V) + (unit * S_max + s0) * kRowBytes +
                         (lane_on ? sub * 16 : 0);

        float m[G], l[G], acc[G][KV];
#pragma unroll
        for (int g = 0; g < G; ++g) {
            m[g] = -INFINITY;
            l[g] = 0.f;
#pragma unroll
            for (int e = 0; e < KV; ++e) acc[g][e] = 0.f;
        }

        for (int pb = 0; pb < seg; pb += NGRP * U) {
            uint4 kv[U], vv[U];
            bool ok[U];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int row = pb + u * NGRP + grp;
                ok[u] = row < seg;
                if (ok[u]) {
                    kv[u] = k_lane ? ld_stream(Kb + (int64_t)row * kKeyBytes)
                                   : make_uint4(0u, 0u, 0u, 0u);
                    vv[u] = lane_on ? ld_stream(Vb + (int64_t)row * kRowBytes)
                                    : make_uint4(0u, 0u, 0u, 0u);
                } else {
                    kv[u] = make_uint4(0u, 0u, 0u, 0u);
                    vv[u] = kv[u];
                }
            }
            float fk[U][KV], fv[U][KV];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                E::unpack(kv[u], fk[u]);
                E::unpack(vv[u], fv[u]);
            }
#pragma unroll
            for (int g = 0; g < G; ++g) {
                float s[U];
                float mx = m[g];
#pragma unroll
                for (int u = 0; u < U; ++u) {
                    float a = 0.f;
#pragma unroll
                    for (int e = 0; e < KV; ++e) a = fmaf(qv[g][e], fk[u][e], a);
                    a = group_sum<LPR>(a);
                    s[u] = ok[u] ? a : -INFINITY;
                    mx = fmaxf(mx, s[u]);
                }
                if (mx == -INFINITY) continue;
                const float alpha = exp2f(m[g] - mx);
                l[g] *= alpha;
#pragma unroll
                for (int e = 0; e < KV; ++e) acc[g][e] *= alpha;
#pragma unroll
                for (int u = 0; u < U; ++u) {
                    const float p = exp2f(s[u] - mx);
                    l[g] += p;
#pragma unroll
                    for (int e = 0; e < KV; ++e) acc[g][e] = fmaf(p, fv[u][e], acc[g][e]);
                }
                m[g] = mx;
            }
        }

        const int part = (int)(blockIdx.x - (unit * S) / per);
#pragma unroll
        for (int g = 0; g < G; ++g) {
            if (sub == 0) {
                sm_m[g][grp] = m[g];
                sm_l[g][grp] = l[g];
            }
#pragma unroll
            for (int e = 0; e < KV; ++e) sm_acc[grp][sub * KV + e] = acc[g][e];
            __syncthreads();
            if (threadIdx.x < D) {
                float M = -INFINITY;
#pragma unroll
                for (int i = 0; i < NGRP; ++i) M = fmaxf(M, sm_m[g][i]);
                float Lsum = 0.f, A = 0.f;
                if (M != -INFINITY) {
#pragma unroll
                    for (int i = 0; i < NGRP; ++i) {
                        const float sc = exp2f(sm_m[g][i] - M);
                        Lsum += sm_l[g][i] * sc;
                        A += sm_acc[i][threadIdx.x] * sc;
                    }
                }
                const int64_t slot = (unit * maxp + part) * G + g;
                part_acc[slot * D + threadIdx.x] = A;
                if (threadIdx.x == 0) part_ml[slot] = make_float2(M, Lsum);
            }
            __syncthreads();
        }
        w += seg;
    }
}

template <class E, int G, int NVK, int DH>
static cudaError_t dense_impl(const void* q, const float* q_rot, int d, const void* K,
                              const void* V, int B, int H_q, int H_kv, int64_t S, int64_t S_max,
                              int D, float scale, void* out, float2* part_ml, float* part_acc,
                              cudaStream_t s, bool pdl) {
    DevInfo di;
    cudaError_t e = dev_info(&di);
    if (e != cudaSuccess) return e;
    const int64_t total = (int64_t)B * H_kv * S;
    auto kern = k_dense<E, G, NVK, DH>;
    const int64_t resident = (int64_t)di.sm_count * occupancy((const void*)kern, 256, 0);
    int64_t grid = (total + kDenseMinRows - 1) / kDenseMinRows;
    if (grid > resident) grid = resident;
    const int64_t per = (total + grid - 1) / grid;
    grid = (total + per - 1) / per;
    const int maxp = (int)((S - 1) / per + 2);
    if (maxp > dense_max_parts(S)) return cudaErrorInvalidValue;
    using T = typename E::T;
    e = launch_kernel(kern, dim3((unsigned)grid), dim3(256), 0, s, pdl, static_cast<const T*>(q),
                      q_rot, d, static_cast<const T*>(K), static_cast<const T*>(V), H_q, H_kv,
                      (int)S, S_max, scale * kLog2e, total, per, maxp, part_ml, part_acc);
    if (e != cudaSuccess) return e;
    return launch_kernel(k_combine<E>, dim3((unsigned)((int64_t)B * H_q)), dim3(128), 0, s, true,
                         (const float2*)part_ml, (const float*)part_acc, static_cast<T*>(out), H_q,
                         G, (int64_t)S, per, maxp, D);
}

template <class E, int NVK, int DH>
static cudaError_t dense_dispatch(int G, const void* q, const float* q_rot, int d, const void* K,
                                  const void* V, int B, int H_q, int H_kv, int64_t S,
                                  int64_t S_max, int D, float scale, void* out, float2* part_ml,
                                  float* part_acc, cudaStream_t s, bool pdl) {
    switch (G) {
#define LOKI_G(g)                                                                               \
    case g:                                                                                     \
        return dense_impl<E, g, NVK, DH>(q, q_rot, d, K, V, B, H_q, H_kv, S, S_max, D, scale, \
                                         out, part_ml, part_acc, s, pdl);
        LOKI_G(1) LOKI_G(2) LOKI_G(3) LOKI_G(4) LOKI_G(5) LOKI_G(6) LOKI_G(7) LOKI_G(8)
#undef LOKI_G
        default: return cudaErrorInvalidValue;
    }
}

template <class E, int DH>
static cudaError_t pca_nvk(int nvk, int G, const float* q_rot, int d, const void* Klo,
                           const void* V, int B, int H_q, int H_kv, int64_t S, int64_t S_max,
                           float scale, void* out, float2* part_ml, float* part_acc,
                           cudaStream_t s) {
    switch (nvk) {
#define LOKI_NVK(n)                                                                          \
    case n:                                                                                  \
        return dense_dispatch<E, n, DH>(G, nullptr, q_rot, d, Klo, V, B, H_q, H_kv, S, S_max, \
                                        DH, scale, out, part_ml, part_acc, s, true);
        LOKI_NVK(1) LOKI_NVK(2) LOKI_NVK(4) LOKI_NVK(8)
#undef LOKI_NVK
        default: return cudaErrorInvalidValue;
    }
}

bool pca_attention_supported(Dt dt, int d_lo) {
    const int row_bytes = d_lo * (dt == kF32 ? 4 : 2);
    const int nvk = row_bytes / 16;
    return row_bytes % 16 == 0 && (nvk == 1 || nvk == 2 || nvk == 4 || nvk == 8) &&
           nvk <= 128 / (dt == kF32 ? 4 : 8);
}

cudaError_t launch_pca_attention(Dt dt, const float* q_rot, const void* Klo, int d_lo, int d,
                                 const void* V, int B, int H_q, int H_kv, int64_t S, int64_t S_max,
                                 int D, float scale, void* out, float2* part_ml, float* part_acc,
                                 cudaStream_t s) {
    if (!pca_attention_supported(dt, d_lo) || (D != 96 && D != 128)) return cudaErrorInvalidValue;
    const int G = H_q / H_kv;
    const int nvk = d_lo * (dt == kF32 ? 4 : 2) / 16;
#define LOKI_PCA(E, DH) \
    pca_nvk<E, DH>(nvk, G, q_rot, d, Klo, V, B, H_q, H_kv, S, S_max, scale, out, part_ml, part_acc, s)
    if (dt == kF32) return D == 96 ? LOKI_PCA(ElemF32, 96) : LOKI_PCA(ElemF32, 128);
    return D == 96 ? LOKI_PCA(ElemBF16, 96) : LOKI_PCA(ElemBF16, 128);
#undef LOKI_PCA
}

cudaError_t launch_dense(Dt dt, const void* q, const void* K, const void* V, int B, int H_q,
                         int H_kv, int64_t S, int64_t S_max, int D, float scale, void* out,
                         float2* part_ml, float* part_acc, cudaStream_t s) {
    const int G = H_q / H_kv;
    if (D != 96 && D != 128) return cudaErrorInvalidValue;
#define LOKI_DENSE(E, DH)                                                                         \
    dense_dispatch<E, 0, DH>(G, q, nullptr, 128, K, V, B, H_q, H_kv, S, S_max, D, scale, out, \
                             part_ml, part_acc, s, false)
    if (dt == kF32) return D == 96 ? LOKI_DENSE(ElemF32, 96) : LOKI_DENSE(ElemF32, 128);
    return D == 96 ? LOKI_DENSE(ElemBF16, 96) : LOKI_DENSE(ElemBF16, 128);
#undef LOKI_DENSE
}

}  // namespace loki
