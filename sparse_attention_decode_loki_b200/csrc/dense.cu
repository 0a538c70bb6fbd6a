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
#include "combine.cuh"
#include "common.cuh"
#include "launch.h"

namespace loki {

constexpr int kDenseMinRows = 256;

// per >= kDenseMinRows / 2 (see sparse_max_parts for the argument)
int64_t dense_max_parts(int64_t S) { return (S - 1) / (kDenseMinRows / 2) + 2; }

template <class E, int G>
__global__ void __launch_bounds__(256) k_dense(const typename E::T* __restrict__ q,
                                               const typename E::T* __restrict__ K,
                                               const typename E::T* __restrict__ V, int H_q,
                                               int H_kv, int S, int64_t S_max, float scale_log2,
                                               int64_t total, int64_t per, int maxp,
                                               float2* __restrict__ part_ml,
                                               float* __restrict__ part_acc) {
    constexpr int D = 128;
    constexpr int KV = E::kVec;
    constexpr int LPR = D / KV;
    constexpr int NGRP = 256 / LPR;
    constexpr int U = G <= 2 ? 4 : 2;
    constexpr int64_t kRowBytes = (int64_t)D * E::kBytes;
    __shared__ float sm_m[G][NGRP], sm_l[G][NGRP];
    __shared__ float sm_acc[NGRP][D];

    const int grp = threadIdx.x / LPR;
    const int sub = threadIdx.x % LPR;
    griddep_launch_dependents();  // lets the combine kernel be scheduled early

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
            const typename E::T* qp = q + ((int64_t)b * H_q + (int64_t)hk * G + g) * D + sub * KV;
#pragma unroll
            for (int e = 0; e < KV; ++e) qv[g][e] = E::load1(qp + e) * scale_log2;
        }
        const char* Kb =
            reinterpret_cast<const char*>(K) + (unit * S_max + s0) * kRowBytes + sub * 16;
        const char* Vb =
            reinterpret_cast<const char*>(V) + (unit * S_max + s0) * kRowBytes + sub * 16;

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
                    kv[u] = ld_stream(Kb + (int64_t)row * kRowBytes);
                    vv[u] = ld_stream(Vb + (int64_t)row * kRowBytes);
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

template <class E, int G>
static cudaError_t dense_impl(const void* q, const void* K, const void* V, int B, int H_q,
                              int H_kv, int64_t S, int64_t S_max, int D, float scale, void* out,
                              float2* part_ml, float* part_acc, cudaStream_t s) {
    DevInfo di;
    cudaError_t e = dev_info(&di);
    if (e != cudaSuccess) return e;
    const int64_t total = (int64_t)B * H_kv * S;
    auto kern = k_dense<E, G>;
    const int64_t resident = (int64_t)di.sm_count * occupancy((const void*)kern, 256, 0);
    int64_t grid = (total + kDenseMinRows - 1) / kDenseMinRows;
    if (grid > resident) grid = resident;
    const int64_t per = (total + grid - 1) / grid;
    grid = (total + per - 1) / per;
    const int maxp = (int)((S - 1) / per + 2);
    if (maxp > dense_max_parts(S)) return cudaErrorInvalidValue;
    using T = typename E::T;
    kern<<<(unsigned)grid, 256, 0, s>>>(static_cast<const T*>(q), static_cast<const T*>(K),
                                        static_cast<const T*>(V), H_q, H_kv, (int)S, S_max,
                                        scale * kLog2e, total, per, maxp, part_ml, part_acc);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    return launch_kernel(k_combine<E>, dim3((unsigned)((int64_t)B * H_q)), dim3(128), 0, s, true,
                         (const float2*)part_ml, (const float*)part_acc, static_cast<T*>(out), H_q,
                         G, (int64_t)S, per, maxp, D);
}

template <class E>
static cudaError_t dense_dispatch(int G, const void* q, const void* K, const void* V, int B,
                                  int H_q, int H_kv, int64_t S, int64_t S_max, int D, float scale,
                                  void* out, float2* part_ml, float* part_acc, cudaStream_t s) {
    switch (G) {
#define LOKI_G(g)                                                                             \
    case g:                                                                                   \
        return dense_impl<E, g>(q, K, V, B, H_q, H_kv, S, S_max, D, scale, out, part_ml, \
                                part_acc, s);
        LOKI_G(1) LOKI_G(2) LOKI_G(3) LOKI_G(4) LOKI_G(5) LOKI_G(6) LOKI_G(7) LOKI_G(8)
#undef LOKI_G
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_dense(Dt dt, const void* q, const void* K, const void* V, int B, int H_q,
                         int H_kv, int64_t S, int64_t S_max, int D, float scale, void* out,
                         float2* part_ml, float* part_acc, cudaStream_t s) {
    const int G = H_q / H_kv;
    if (dt == kF32)
        return dense_dispatch<ElemF32>(G, q, K, V, B, H_q, H_kv, S, S_max, D, scale, out, part_ml,
                                       part_acc, s);
    return dense_dispatch<ElemBF16>(G, q, K, V, B, H_q, H_kv, S, S_max, D, scale, out, part_ml,
                                    part_acc, s);
}

}  // namespace loki
