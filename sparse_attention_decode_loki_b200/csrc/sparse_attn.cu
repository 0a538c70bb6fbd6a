// Exact attention over the selected tokens (Loki's final step; NeurIPS 2024
// poster page, TL;DR: full-dimensional scores only for the selected tokens;
// "Visual Insights" Figure 1 caption: the full-dimensional keys give the
// final attention scores).
//
// Work items are (row, j) pairs, row = (batch, query head) and j < k the
// position in its selected list; the B*H_q*k items are split evenly over one
// wave of CTAs. Each CTA stages its selected indices in shared memory (1024
// at a time), so the row gathers never wait on an index load. A row group of
// lanes (16 lanes for bf16, 32 for fp32) owns one 256/512-byte key row and
// the matching value row per step, with 8 rows in flight; each row is a
// random gather, but a contiguous one. Scores use all D
// dimensions in fp32; the softmax runs online in base 2 with the scale folded
// into q~. Each CTA merges its row groups and writes one partial per row
// segment; k_combine merges the partials of a row.
#include "combine.cuh"
#include "common.cuh"
#include "launch.h"

namespace loki {

constexpr int kSparseMinItems = 64;  // CTAs own at least this many items

// A CTA of the split owns per >= kSparseMinItems / 2 items (grid <= total /
// kSparseMinItems, rounded up), so a row of k items spans at most
// (k - 1) / per + 2 CTAs; the workspace is sized for the smallest per.
int64_t sparse_max_parts(int64_t k) { return (k - 1) / (kSparseMinItems / 2) + 2; }

template <class E>
__global__ void __launch_bounds__(256, 2) k_sparse_attn(
    const float* __restrict__ q_rot, const typename E::T* __restrict__ Kt,
    const typename E::T* __restrict__ V, const int32_t* __restrict__ idx, int H_q, int H_kv, int S,
    int64_t S_max, int k, float scale_log2, int64_t total, int64_t per, int maxp,
    float2* __restrict__ part_ml, float* __restrict__ part_acc) {
    constexpr int D = 128;
    constexpr int KV = E::kVec;
    constexpr int LPR = D / KV;           // lanes per row
    constexpr int NGRP = 256 / LPR;       // row groups per CTA
    constexpr int U = 8;                  // rows in flight per group
    constexpr int kIdxChunk = 1024;       // selected indices staged per step
    constexpr int64_t kRowBytes = (int64_t)D * E::kBytes;
    __shared__ float sm_m[NGRP], sm_l[NGRP];
    __shared__ float sm_acc[NGRP][D];
    __shared__ int s_idx[kIdxChunk];

    const int grp = threadIdx.x / LPR;
    const int sub = threadIdx.x % LPR;
    const int G = H_q / H_kv;
    griddep_wait();  // q_rot and the selected indices come from earlier kernels
    griddep_launch_dependents();

    int64_t w = (int64_t)blockIdx.x * per;
    const int64_t w_end = min64(w + per, total);
    while (w < w_end) {
        const int64_t r = w / k;
        const int j0 = (int)(w - r * k);
        const int j1 = (int)min64(k, j0 + (w_end - w));
        const int b = (int)(r / H_q), h = (int)(r % H_q);
        const int64_t unit = (int64_t)b * H_kv + h / G;

        float qv[KV];
        {
            const float* qp = q_rot + r * D + sub * KV;
#pragma unroll
            for (int e = 0; e < KV; ++e) qv[e] = __ldg(qp + e) * scale_log2;
        }
        const char* Kb = reinterpret_cast<const char*>(Kt) + unit * S_max * kRowBytes + sub * 16;
        const char* Vb = reinterpret_cast<const char*>(V) + unit * S_max * kRowBytes + sub * 16;
        const int32_t* ip = idx + r * k;

        float m = -INFINITY, l = 0.f, acc[KV];
#pragma unroll
        for (int e = 0; e < KV; ++e) acc[e] = 0.f;

        for (int cb = j0; cb < j1; cb += kIdxChunk) {
            const int n = min(kIdxChunk, j1 - cb);
            __syncthreads();  // the previous chunk's indices are no longer read
            for (int t = threadIdx.x; t < n; t += 256) {
                const int tok = __ldg(ip + cb + t);
                s_idx[t] = ((unsigned)tok < (unsigned)S) ? tok : -1;
            }
            __syncthreads();
            for (int jb = 0; jb < n; jb += NGRP * U) {
                int t[U];
                uint4 kv[U], vv[U];
#pragma unroll
                for (int u = 0; u < U; ++u) {
                    const int jj = jb + u * NGRP + grp;
                    const int tok = jj < n ? s_idx[jj] : -1;
                    t[u] = tok;
                    if (tok >= 0) {
                        kv[u] = ld_stream(Kb + (int64_t)tok * kRowBytes);
                        vv[u] = ld_stream(Vb + (int64_t)tok * kRowBytes);
                    } else {
                        kv[u] = make_uint4(0u, 0u, 0u, 0u);
                        vv[u] = kv[u];
                    }
                }
                float s[U];
                float mx = m;
#pragma unroll
                for (int u = 0; u < U; ++u) {
                    float f[KV];
                    E::unpack(kv[u], f);
                    float a = 0.f;
#pragma unroll
                    for (int e = 0; e < KV; ++e) a = fmaf(qv[e], f[e], a);
                    a = group_sum<LPR>(a);
                    s[u] = t[u] >= 0 ? a : -INFINITY;
                    mx = fmaxf(mx, s[u]);
                }
                if (mx == -INFINITY) continue;
                const float alpha = exp2f(m - mx);
                l *= alpha;
#pragma unroll
                for (int e = 0; e < KV; ++e) acc[e] *= alpha;
#pragma unroll
                for (int u = 0; u < U; ++u) {
                    const float p = exp2f(s[u] - mx);
                    l += p;
                    float f[KV];
                    E::unpack(vv[u], f);
#pragma unroll
                    for (int e = 0; e < KV; ++e) acc[e] = fmaf(p, f[e], acc[e]);
                }
                m = mx;
            }
        }

        if (sub == 0) {
            sm_m[grp] = m;
            sm_l[grp] = l;
        }
#pragma unroll
        for (int e = 0; e < KV; ++e) sm_acc[grp][sub * KV + e] = acc[e];
        __syncthreads();
        if (threadIdx.x < D) {
            float M = -INFINITY;
#pragma unroll
            for (int g = 0; g < NGRP; ++g) M = fmaxf(M, sm_m[g]);
            float Lsum = 0.f, A = 0.f;
            if (M != -INFINITY) {
#pragma unroll
                for (int g = 0; g < NGRP; ++g) {
                    const float sc = exp2f(sm_m[g] - M);
                    Lsum += sm_l[g] * sc;
                    A += sm_acc[g][threadIdx.x] * sc;
                }
            }
            const int part = (int)(blockIdx.x - (r * k) / per);
            const int64_t slot = r * maxp + part;
            part_acc[slot * D + threadIdx.x] = A;
            if (threadIdx.x == 0) part_ml[slot] = make_float2(M, Lsum);
        }
        __syncthreads();
        w += j1 - j0;
    }
}

template <class E>
static cudaError_t sparse_impl(const float* q_rot, const void* Kt, const void* V,
                               const int32_t* idx, int B, int H_q, int H_kv, int64_t S,
                               int64_t S_max, int D, int64_t k, float scale, void* out,
                               float2* part_ml, float* part_acc, cudaStream_t s, bool pdl) {
    DevInfo di;
    cudaError_t e = dev_info(&di);
    if (e != cudaSuccess) return e;
    const int64_t rows = (int64_t)B * H_q;
    const int64_t total = rows * k;
    auto kern = k_sparse_attn<E>;
    const int64_t resident = (int64_t)di.sm_count * occupancy((const void*)kern, 256, 0);
    int64_t grid = (total + kSparseMinItems - 1) / kSparseMinItems;
    if (grid > resident) grid = resident;
    const int64_t per = (total + grid - 1) / grid;
    grid = (total + per - 1) / per;
    const int maxp = (int)((k - 1) / per + 2);
    if (maxp > sparse_max_parts(k)) return cudaErrorInvalidValue;
    using T = typename E::T;
    e = launch_kernel(kern, dim3((unsigned)grid), dim3(256), 0, s, pdl, q_rot,
                      static_cast<const T*>(Kt), static_cast<const T*>(V), idx, H_q, H_kv, (int)S,
                      S_max, (int)k, scale * kLog2e, total, per, maxp, part_ml, part_acc);
    if (e != cudaSuccess) return e;
    return launch_kernel(k_combine<E>, dim3((unsigned)rows), dim3(128), 0, s, true,
                         (const float2*)part_ml, (const float*)part_acc, static_cast<T*>(out), H_q,
                         1, (int64_t)k, per, maxp, D);
}

cudaError_t launch_sparse_attention(Dt dt, const float* q_rot, const void* Kt, const void* V,
                                    const int32_t* idx, int B, int H_q, int H_kv, int64_t S,
                                    int64_t S_max, int D, int64_t k, float scale, void* out,
                                    float2* part_ml, float* part_acc, cudaStream_t s, bool pdl) {
    if (dt == kF32)
        return sparse_impl<ElemF32>(q_rot, Kt, V, idx, B, H_q, H_kv, S, S_max, D, k, scale, out,
                                    part_ml, part_acc, s, pdl);
    return sparse_impl<ElemBF16>(q_rot, Kt, V, idx, B, H_q, H_kv, S, S_max, D, k, scale, out,
                                 part_ml, part_acc, s, pdl);
}

}  // namespace loki
