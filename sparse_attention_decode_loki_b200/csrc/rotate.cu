// Rotation of rows into a KV head's PCA basis: queries, q~ = q P, and new
// keys appended to the KV-cache, K~ = K P (the key also goes to the
// low-dimensional key plane; its value row is copied unchanged). With no P
// the rotation is the identity: rows are copied (queries widened to fp32,
// keys written to the cache as they are), which the pre-rotary variant uses
// for its post-rotary queries and keys.
//
// Loki (NeurIPS 2024 poster page, "Visual Insights" Figure 1 caption: keys
// and queries are used through their PCA projection; "Loki's Computational
// Cost": keys are appended to the KV-cache at every decode step).
//
// One CTA per (KV head, block of 32 output columns, chunk of up to 32 rows of
// that head): the 128 x 32 column block of P is staged once in shared memory
// and used by every row of the chunk; each warp computes one row's 32 columns
// per step, summing in fp32 in index order. A head's rows are, per sequence
// b, its G query heads and then its T new keys; query rows go to q_rot
// (fp32), key rows are rounded once to the cache type (nearest even) and
// written at cache rows [pos, pos + T).
#include "common.cuh"
#include "launch.h"

namespace loki {

constexpr int kRotCols = 32;
constexpr int kRotRows = 32;

template <class E>
__global__ void __launch_bounds__(256) k_rotate_rows(
    const typename E::T* __restrict__ q, const typename E::T* __restrict__ K_new,
    const typename E::T* __restrict__ V_new, const float* __restrict__ P, float* __restrict__ q_rot,
    typename E::T* __restrict__ Kt_cache, typename E::T* __restrict__ V_cache,
    typename E::T* __restrict__ Kt_lo, int d_lo, int B, int H_q, int H_kv, int G, int T, int D,
    int64_t S_max, int64_t pos, int* __restrict__ done, int n_done, int hold,
    const int* __restrict__ block_table, const int* __restrict__ positions, int page_size,
    int max_pages, int64_t n_pages, int* __restrict__ err) {
    using Tp = typename E::T;
    __shared__ float Ps[128][kRotCols];
    __shared__ float xs[kRotRows][128];
    // a programmatic dependent (the score scan) may start right away
    griddep_launch_dependents();
    if (done != nullptr) {
        const int64_t nb = gridDim.x;
        for (int64_t i = blockIdx.x * 256 + threadIdx.x; i < n_done; i += nb * 256) done[i] = 0;
    }
    const int ncb = (D + kRotCols - 1) / kRotCols;
    const int R = G + T;  // rows of the head per sequence
    // work items (row chunk, column block, KV head), head fastest, dealt to
    // the CTAs of the grid in turn (the grid may be smaller than the items)
    const int64_t nitems = ((int64_t)B * R + kRotRows - 1) / kRotRows * ncb * H_kv;
    for (int64_t bid = blockIdx.x; bid < nitems; bid += gridDim.x) {
    const int hk = (int)(bid % H_kv);
    const int cb = (int)((bid / H_kv) % ncb);
    const int c0 = cb * kRotCols;
    const int64_t r0 = (bid / H_kv / ncb) * kRotRows;
    const int nrows = (int)min64(kRotRows, (int64_t)B * R - r0);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const float* Ph = P != nullptr ? P + (int64_t)hk * D * D : nullptr;
    // the P block: 128 rows x 32 columns = 1024 float4, 4 per thread, all in
    // flight (no P: the identity's block, so each sum is one exact product)
    float4 pv[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        const int it = tid + u * 256;
        const int i = it >> 3, c4 = (it & 7) * 4;
        const int c = c0 + c4;
        if (P == nullptr)
            pv[u] = make_float4(i == c ? 1.f : 0.f, i == c + 1 ? 1.f : 0.f,
                                i == c + 2 ? 1.f : 0.f, i == c + 3 ? 1.f : 0.f);
        else
            pv[u] = (i < D && c < D)
                        ? __ldg(reinterpret_cast<const float4*>(Ph + (int64_t)i * D + c))
                        : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    // row j of the chunk: sequence b = (r0 + j) / R, member g = (r0 + j) % R
    // (a query head for g < G, else new key g - G); 8 elements per thread and
    // step, in a layout of 128 columns whose columns past D stay zero
    constexpr int QV = 8;
    float xv[kRotRows * 128 / 256];
#pragma unroll
    for (int u = 0; u < kRotRows * 128 / 256 / QV; ++u) {
        const int it = (tid + u * 256) * QV;
        const int j = it / 128, i = it % 128;
        const int64_t jr = r0 + j;
        const Tp* src = nullptr;
        if (j < nrows && i < D) {
            const int b = (int)(jr / R), g = (int)(jr % R);
            src = g < G ? q + ((int64_t)b * H_q + (int64_t)hk * G + g) * D
                        : K_new + (((int64_t)b * H_kv + hk) * T + (g - G)) * D;
        }
#pragma unroll
        for (int e = 0; e < QV; ++e) xv[u * QV + e] = src ? E::load1(src + i + e) : 0.f;
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        const int it = tid + u * 256;
        const int i = it >> 3, c4 = (it & 7) * 4;
        if (i < 128) *reinterpret_cast<float4*>(&Ps[i][c4]) = pv[u];
    }
#pragma unroll
    for (int u = 0; u < kRotRows * 128 / 256 / QV; ++u) {
        const int it = (tid + u * 256) * QV;
        const int j = it / 128, i = it % 128;
#pragma unroll
        for (int e = 0; e < QV; ++e) xs[j][i + e] = xv[u * QV + e];
    }
    __syncthreads();
    for (int j = warp; j < nrows; j += 8) {
        float acc = 0.f;
#pragma unroll 8
        for (int i = 0; i < D; ++i) acc = fmaf(xs[j][i], Ps[i][lane], acc);
        const int64_t jr = r0 + j;
        const int b = (int)(jr / R), g = (int)(jr % R);
        const int c = c0 + lane;
        if (g < G) {
            if (c < D) q_rot[((int64_t)b * H_q + (int64_t)hk * G + g) * D + c] = acc;
        } else {
            const int t = g - G;
            int64_t row;
            if (block_table == nullptr) {
                row = ((int64_t)b * H_kv + hk) * S_max + pos + t;
            } else {
                // paged: logical token positions[b] + t of sequence b
                const int64_t j = (int64_t)positions[b] + t;
                const int page = (j >= 0 && j < (int64_t)page_size * max_pages)
                                     ? __ldg(block_table + (int64_t)b * max_pages + j / page_size)
                                     : -1;
                if (page < 0 || page >= n_pages) {
                    if (lane == 0) atomicExch(err, 2);  // nowhere valid to write: skip the row
                    continue;
                }
                row = ((int64_t)page * H_kv + hk) * page_size + j % page_size;
            }
            const Tp kt = E::from_float(acc);
            if (Kt_cache != nullptr && c < D) Kt_cache[row * D + c] = kt;
            if (Kt_lo != nullptr && c < d_lo) Kt_lo[row * d_lo + c] = kt;
            if (V_cache != nullptr && cb == 0) {  // one column block copies the value row
                const Tp* vs = V_new + (((int64_t)b * H_kv + hk) * T + t) * D;
                for (int e = lane; e < D; e += 32) V_cache[row * D + e] = vs[e];
            }
        }
    }
    __syncthreads();  // Ps and xs are refilled for the next item
    }
    // hold: launched beside the score scan, this grid completes only after the
    // scan does (one waiting thread is enough), so the kernels that wait on
    // it also see the scan's scores
    if (hold && threadIdx.x == 0 && blockIdx.x == 0) griddep_wait();
}

cudaError_t launch_rotate(Dt dt, const void* q, const void* K_new, const void* V_new,
                          const float* P, float* q_rot, void* Kt_cache, void* V_cache, void* Kt_lo,
                          int d_lo, int B, int H_q, int H_kv, int T, int D, int64_t S_max,
                          int64_t pos, cudaStream_t s, int* done, int n_done, bool pdl,
                          const PagedKV* pg, const int* positions, bool one_per_sm) {
    int* err = device_error_word();
    if (err == nullptr) return cudaErrorInvalidDevice;
    const int* bt = pg != nullptr ? pg->block_table : nullptr;
    const int ps = pg != nullptr ? pg->page_size : 0;
    const int mp = pg != nullptr ? pg->max_pages : 0;
    const int64_t np = pg != nullptr ? pg->n_pages : 0;
    const int G = q != nullptr ? H_q / H_kv : 0;
    const int Tn = K_new != nullptr ? T : 0;
    const int R = G + Tn;
    if (R == 0) return cudaSuccess;
    const int64_t chunks = ((int64_t)B * R + kRotRows - 1) / kRotRows;
    int64_t nblocks = chunks * H_kv * ((D + kRotCols - 1) / kRotCols);
    if (one_per_sm) {
        // beside the score scan: at most one CTA per SM, so the scan's CTA
        // (9 warps at 128 registers) still fits next to it on every SM
        DevInfo di;
        const cudaError_t e = dev_info(&di);
        if (e != cudaSuccess) return e;
        nblocks = min64(nblocks, di.sm_count);
    }
    if (nblocks > 0x7fffffff) return cudaErrorInvalidConfiguration;
    const dim3 grid((unsigned)nblocks);
    const int hold = pdl ? 1 : 0;
    if (dt == kF32)
        return launch_kernel(k_rotate_rows<ElemF32>, grid, dim3(256), 0, s, pdl,
                             static_cast<const float*>(q), static_cast<const float*>(K_new),
                             static_cast<const float*>(V_new), P, q_rot,
                             static_cast<float*>(Kt_cache), static_cast<float*>(V_cache),
                             static_cast<float*>(Kt_lo), d_lo, B, H_q, H_kv, G, Tn, D, S_max, pos,
                             done, n_done, hold, bt, positions, ps, mp, np, err);
    using T16 = __nv_bfloat16;
    return launch_kernel(k_rotate_rows<ElemBF16>, grid, dim3(256), 0, s, pdl,
                         static_cast<const T16*>(q), static_cast<const T16*>(K_new),
                         static_cast<const T16*>(V_new), P, q_rot, static_cast<T16*>(Kt_cache),
                         static_cast<T16*>(V_cache), static_cast<T16*>(Kt_lo), d_lo, B, H_q, H_kv,
                         G, Tn, D, S_max, pos, done, n_done, hold, bt, positions, ps, mp, np, err);
}

cudaError_t launch_project_query(Dt dt, const void* q, const float* P, int B, int H_q, int H_kv,
                                 int D, float* q_rot, cudaStream_t s, int* done, int n_done,
                                 bool pdl) {
    return launch_rotate(dt, q, nullptr, nullptr, P, q_rot, nullptr, nullptr, nullptr, 0, B, H_q,
                         H_kv, 0, D, 0, 0, s, done, n_done, pdl, nullptr, nullptr, pdl);
}

cudaError_t launch_append(Dt dt, const void* K_new, const void* V_new, const float* P,
                          void* Kt_cache, void* V_cache, void* Kt_lo, int d_lo, int B, int H_kv,
                          int T, int D, int64_t S_max, int64_t pos, cudaStream_t s) {
    return launch_rotate(dt, nullptr, K_new, V_new, P, nullptr, Kt_cache, V_cache, Kt_lo, d_lo, B,
                         H_kv, H_kv, T, D, S_max, pos, s, nullptr, 0, false, nullptr, nullptr,
                         false);
}

}  // namespace loki
