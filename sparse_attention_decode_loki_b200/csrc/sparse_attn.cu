// Exact attention over the selected tokens (Loki's final step; NeurIPS 2024
// poster page, TL;DR: full-dimensional scores only for the selected tokens;
// "Visual Insights" Figure 1 caption: the full-dimensional keys give the
// final attention scores).
//
// One warp per (row, chunk of the selected list); no block barriers. The warp
// stages its selected indices in shared memory, then each row group of lanes
// (16 lanes for bf16, 32 for fp32) gathers one 256/512-byte key row and the
// matching value row per step, 8 rows in flight; every row is a random but
// contiguous gather. Scores use all D dimensions in fp32; the softmax runs
// online in base 2 with the scale folded into q~. The warp merges its row
// groups with shuffles and writes one partial; the last warp to finish a row
// (a per-row atomic counter) merges that row's partials into the output, so
// no separate combine kernel runs.
#include "common.cuh"
#include "launch.h"

namespace loki {

// Work decomposition. Each (batch, query head) row's k selected positions are
// cut into nchunk chunks; a work item is one (row, chunk) and one warp owns one
// item at a time (grid-stride over items). nchunk is chosen so the items fill
// one wave of resident warps. Partials of row r sit in slots [r*nchunk, ...).
constexpr int kMinChunk = 16;
constexpr int kWarpIdx = 256;  // indices staged per warp per step

int64_t sparse_max_parts(int64_t rows, int64_t k) {
    int64_t cap = 10240 / rows;
    if (cap < 1) cap = 1;
    const int64_t by_k = (k + kMinChunk - 1) / kMinChunk;
    return (by_k < cap ? by_k : cap) + 2;
}

template <class E>
__global__ void __launch_bounds__(256) k_sparse_attn(
    const float* __restrict__ q_rot, const typename E::T* __restrict__ Kt,
    const typename E::T* __restrict__ V, const int32_t* __restrict__ idx, int H_q, int H_kv, int S,
    int64_t S_max, int k, float scale_log2, int chunk, int nchunk, int64_t n_items,
    float2* __restrict__ part_ml, float* __restrict__ part_acc, int* __restrict__ done,
    typename E::T* __restrict__ out) {
    constexpr int D = 128;
    constexpr int KV = E::kVec;
    constexpr int LPR = D / KV;     // lanes per row
    constexpr int GPW = 32 / LPR;   // row groups per warp
    constexpr int U = 8;            // rows in flight per group
    constexpr int64_t kRowBytes = (int64_t)D * E::kBytes;
    __shared__ int s_idx[8][kWarpIdx];

    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int grp = lane / LPR, sub = lane % LPR;
    const int G = H_q / H_kv;
    int* widx = s_idx[warp];
    griddep_wait();  // q_rot and the selected indices come from earlier kernels
    griddep_launch_dependents();

    const int64_t nwarps = (int64_t)gridDim.x * 8;
    for (int64_t item = (int64_t)blockIdx.x * 8 + warp; item < n_items; item += nwarps) {
        const int64_t r = item / nchunk;
        const int c = (int)(item - r * nchunk);
        const int j0 = c * chunk;
        const int j1 = min(k, j0 + chunk);
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

        for (int cb = j0; cb < j1; cb += kWarpIdx) {
            const int n = min(kWarpIdx, j1 - cb);
            __syncwarp();
            for (int t = lane; t < n; t += 32) {
                const int tok = __ldg(ip + cb + t);
                widx[t] = ((unsigned)tok < (unsigned)S) ? tok : -1;
            }
            __syncwarp();
            for (int jb = 0; jb < n; jb += GPW * U) {
                int t[U];
                uint4 kv[U], vv[U];
#pragma unroll
                for (int u = 0; u < U; ++u) {
                    const int jj = jb + u * GPW + grp;
                    const int tok = jj < n ? widx[jj] : -1;
                    t[u] = tok;
                    if (tok >= 0) {
                        kv[u] = ld_stream(Kb + (int64_t)tok * kRowBytes);
                        vv[u] = ld_stream(Vb + (int64_t)tok * kRowBytes);
                    } else {
                        kv[u] = make_uint4(0u, 0u, 0u, 0u);
                        vv[u] = kv[u];
                    }
                }
                float sc[U];
                float mx = m;
#pragma unroll
                for (int u = 0; u < U; ++u) {
                    float f[KV];
                    E::unpack(kv[u], f);
                    float a = 0.f;
#pragma unroll
                    for (int e = 0; e < KV; ++e) a = fmaf(qv[e], f[e], a);
                    a = group_sum<LPR>(a);
                    sc[u] = t[u] >= 0 ? a : -INFINITY;
                    mx = fmaxf(mx, sc[u]);
                }
                if (mx == -INFINITY) continue;
                const float alpha = exp2f(m - mx);
                l *= alpha;
#pragma unroll
                for (int e = 0; e < KV; ++e) acc[e] *= alpha;
#pragma unroll
                for (int u = 0; u < U; ++u) {
                    const float p = exp2f(sc[u] - mx);
                    l += p;
                    float f[KV];
                    E::unpack(vv[u], f);
#pragma unroll
                    for (int e = 0; e < KV; ++e) acc[e] = fmaf(p, f[e], acc[e]);
                }
                m = mx;
            }
        }
        // merge the warp's row groups (lane l and lane l + LPR hold the same columns)
#pragma unroll
        for (int off = LPR; off < 32; off <<= 1) {
            const float mo = __shfl_xor_sync(0xffffffffu, m, off);
            const float lo = __shfl_xor_sync(0xffffffffu, l, off);
            const float M = fmaxf(m, mo);
            const float sa = M == -INFINITY ? 0.f : exp2f(m - M);
            const float sb = M == -INFINITY ? 0.f : exp2f(mo - M);
            l = l * sa + lo * sb;
#pragma unroll
            for (int e = 0; e < KV; ++e) {
                const float ao = __shfl_xor_sync(0xffffffffu, acc[e], off);
                acc[e] = acc[e] * sa + ao * sb;
            }
            m = M;
        }
        if (grp == 0) {
            float* pa = part_acc + item * D + sub * KV;
#pragma unroll
            for (int e = 0; e < KV; e += 4)
                *reinterpret_cast<float4*>(pa + e) = make_float4(acc[e], acc[e + 1], acc[e + 2], acc[e + 3]);
            if (sub == 0) part_ml[item] = make_float2(m, l);
        }
        // The last warp to finish a chunk of row r merges the row's partials
        // (its own included) into out[r]: publish, count, and only the warp
        // that sees the count reach nchunk reads the others' partials.
        __threadfence();  // each lane's partial writes are visible device-wide...
        __syncwarp();     // ...before lane 0 counts the chunk as done
        int prev = 0;
        if (lane == 0) prev = atomicAdd(done + r, 1);
        prev = __shfl_sync(0xffffffffu, prev, 0);
        if (prev == nchunk - 1) {
            __threadfence();
            const float2* ml = part_ml + r * nchunk;
            float M = -INFINITY;
            for (int p = 0; p < nchunk; ++p) M = fmaxf(M, __ldcg(&ml[p].x));
            float Lsum = 0.f, A[D / 32];
#pragma unroll
            for (int e = 0; e < D / 32; ++e) A[e] = 0.f;
            if (M != -INFINITY) {
                for (int p = 0; p < nchunk; ++p) {
                    const float2 mlp = __ldcg(&ml[p]);
                    const float sc = exp2f(mlp.x - M);
                    Lsum += mlp.y * sc;
                    const float* pa = part_acc + (r * nchunk + p) * D;
#pragma unroll
                    for (int e = 0; e < D / 32; ++e) A[e] += __ldcg(pa + e * 32 + lane) * sc;
                }
            }
            const float inv = Lsum > 0.f ? 1.f / Lsum : 0.f;
#pragma unroll
            for (int e = 0; e < D / 32; ++e) out[r * D + e * 32 + lane] = E::from_float(A[e] * inv);
            if (lane == 0) done[r] = 0;  // leave the counter ready for the next call
        }
    }
}

template <class E>
static cudaError_t sparse_impl(const float* q_rot, const void* Kt, const void* V,
                               const int32_t* idx, int B, int H_q, int H_kv, int64_t S,
                               int64_t S_max, int D, int64_t k, float scale, void* out,
                               float2* part_ml, float* part_acc, int* done, cudaStream_t s,
                               bool pdl) {
    DevInfo di;
    cudaError_t e = dev_info(&di);
    if (e != cudaSuccess) return e;
    const int64_t rows = (int64_t)B * H_q;
    auto kern = k_sparse_attn<E>;
    const int64_t warps = (int64_t)di.sm_count * occupancy((const void*)kern, 256, 0) * 8;
    int64_t nchunk = warps / rows;
    if (nchunk < 1) nchunk = 1;
    const int64_t cap = sparse_max_parts(rows, k);
    if (nchunk > cap) nchunk = cap;
    int64_t chunk = (k + nchunk - 1) / nchunk;
    chunk = (chunk + kMinChunk - 1) / kMinChunk * kMinChunk;
    nchunk = (k + chunk - 1) / chunk;
    const int64_t n_items = rows * nchunk;
    int64_t grid = (n_items + 7) / 8;
    const int64_t max_grid = warps / 8;
    if (grid > max_grid) grid = max_grid;
    using T = typename E::T;
    return launch_kernel(kern, dim3((unsigned)grid), dim3(256), 0, s, pdl, q_rot,
                         static_cast<const T*>(Kt), static_cast<const T*>(V), idx, H_q, H_kv,
                         (int)S, S_max, (int)k, scale * kLog2e, (int)chunk, (int)nchunk, n_items,
                         part_ml, part_acc, done, static_cast<T*>(out));
}

cudaError_t launch_sparse_attention(Dt dt, const float* q_rot, const void* Kt, const void* V,
                                    const int32_t* idx, int B, int H_q, int H_kv, int64_t S,
                                    int64_t S_max, int D, int64_t k, float scale, void* out,
                                    float2* part_ml, float* part_acc, int* done, cudaStream_t s,
                                    bool pdl) {
    if (dt == kF32)
        return sparse_impl<ElemF32>(q_rot, Kt, V, idx, B, H_q, H_kv, S, S_max, D, k, scale, out,
                                    part_ml, part_acc, done, s, pdl);
    return sparse_impl<ElemBF16>(q_rot, Kt, V, idx, B, H_q, H_kv, S, S_max, D, k, scale, out,
                                 part_ml, part_acc, done, s, pdl);
}

}  // namespace loki
