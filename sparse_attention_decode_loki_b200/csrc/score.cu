// Query rotation and the (register-staged) low-dimensional score scan of Loki.
//
// Loki (NeurIPS 2024 poster page, TL;DR and "Visual Insights" Figure 1
// caption; briefgpt.xyz abstract page): the query is projected onto the PCA
// basis and every cached token is scored on the first d principal components
// only, s_j = q~[:d] . K~_j[:d].
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

// q_rot[row, c] = sum_i q[row, i] P[h_kv, i, c]; also zeroes done[0, n_done)
// (the attention kernel's per-row counters) when done is given. One CTA per (KV head, block of
// 32 output columns, chunk of up to 32 query rows of that head): the P column
// block (128 x 32 fp32) is staged once in shared memory and reused by every
// query of the head; each warp computes one query's 32 columns per step.
constexpr int kProjCols = 32;
constexpr int kProjRows = 32;

template <class E>
__global__ void __launch_bounds__(256) k_project_query(const typename E::T* __restrict__ q,
                                                       const float* __restrict__ P,
                                                       float* __restrict__ q_rot, int B, int H_q,
                                                       int G, int D, int* __restrict__ done,
                                                       int n_done, int hold) {
    __shared__ float Ps[128][kProjCols];
    __shared__ float qs[kProjRows][128];
    // the next kernel (the score scan) may start streaming keys right away
    griddep_launch_dependents();
    if (done != nullptr) {
        const int nb = gridDim.x * gridDim.y * gridDim.z;
        const int bid = (blockIdx.z * gridDim.y + blockIdx.y) * gridDim.x + blockIdx.x;
        for (int i = bid * 256 + (int)threadIdx.x; i < n_done; i += nb * 256) done[i] = 0;
    }
    const int hk = blockIdx.x;
    const int c0 = blockIdx.y * kProjCols;
    const int r0 = blockIdx.z * kProjRows;
    const int nrows = min(kProjRows, B * G - r0);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const float* Ph = P + (int64_t)hk * D * D;
    // P block: 128 rows x 32 columns = 1024 float4, 4 per thread, all in flight
    float4 pv[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        const int it = tid + u * 256;
        const int i = it >> 3, c4 = (it & 7) * 4;
        pv[u] = (i < D && c0 + c4 < D)
                    ? __ldg(reinterpret_cast<const float4*>(Ph + (int64_t)i * D + c0 + c4))
                    : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    // the head's queries: row j of the chunk is (batch b, group member g);
    // 8 consecutive elements per thread per step
    constexpr int QV = 8;
    float qv[kProjRows * 128 / 256];
#pragma unroll
    for (int u = 0; u < kProjRows * 128 / 256 / QV; ++u) {
        const int it = (tid + u * 256) * QV;
        const int j = it / D, i = it % D;
        const int jr = r0 + j;
        const int64_t row = (int64_t)(jr / G) * H_q + (int64_t)hk * G + jr % G;
#pragma unroll
        for (int e = 0; e < QV; ++e)
            qv[u * QV + e] = (j < nrows) ? E::load1(q + row * D + i + e) : 0.f;
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        const int it = tid + u * 256;
        const int i = it >> 3, c4 = (it & 7) * 4;
        if (i < 128) *reinterpret_cast<float4*>(&Ps[i][c4]) = pv[u];
    }
#pragma unroll
    for (int u = 0; u < kProjRows * 128 / 256 / QV; ++u) {
        const int it = (tid + u * 256) * QV;
        const int j = it / D, i = it % D;
#pragma unroll
        for (int e = 0; e < QV; ++e) qs[j][i + e] = qv[u * QV + e];
    }
    __syncthreads();
    for (int j = warp; j < nrows; j += 8) {
        float acc = 0.f;
#pragma unroll 8
        for (int i = 0; i < D; ++i) acc = fmaf(qs[j][i], Ps[i][lane], acc);
        const int jr = r0 + j;
        const int64_t row = (int64_t)(jr / G) * H_q + (int64_t)hk * G + jr % G;
        if (c0 + lane < D) q_rot[row * D + c0 + lane] = acc;
    }
    // hold: launched beside the score scan, this grid completes only after the
    // scan does (one waiting thread is enough), so the kernels that wait on
    // it also see the scan's scores
    if (hold && threadIdx.x == 0 && blockIdx.x == 0 && blockIdx.y == 0 && blockIdx.z == 0)
        griddep_wait();
}

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

cudaError_t launch_project_query(Dt dt, const void* q, const float* P, int B, int H_q, int H_kv,
                                 int D, float* q_rot, cudaStream_t s, int* done, int n_done,
                                 bool pdl) {
    const int G = H_q / H_kv;
    dim3 grid(H_kv, (D + kProjCols - 1) / kProjCols, (B * G + kProjRows - 1) / kProjRows);
    const int hold = pdl ? 1 : 0;
    if (dt == kF32)
        return launch_kernel(k_project_query<ElemF32>, grid, dim3(256), 0, s, pdl,
                             static_cast<const float*>(q), P, q_rot, B, H_q, G, D, done, n_done,
                             hold);
    return launch_kernel(k_project_query<ElemBF16>, grid, dim3(256), 0, s, pdl,
                         static_cast<const __nv_bfloat16*>(q), P, q_rot, B, H_q, G, D, done,
                         n_done, hold);
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
