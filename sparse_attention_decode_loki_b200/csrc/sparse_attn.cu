// Exact attention over the selected tokens (Loki's final step; NeurIPS 2024
// poster page, TL;DR: full-dimensional scores only for the selected tokens;
// "Visual Insights" Figure 1 caption: the full-dimensional keys give the
// final attention scores).
//
// Every warp of one wave owns an equal run of 16-key blocks of the selected
// lists (rows laid end to end); no block barriers. The warp stages its
// selected indices in shared memory, then each row group of lanes (16 lanes
// for bf16, 32 for fp32) gathers one 256/512-byte key row and the matching
// value row per step, 8 rows in flight; every row is a random but contiguous
// gather. Scores use all D dimensions in fp32; the softmax runs online in
// base 2 with the scale folded into q~. The warp merges its row groups with
// shuffles and, per row it touches, writes the output (a whole row) or one
// partial; the last warp to finish a row (a per-row atomic counter) merges
// that row's partials into the output, so no separate combine kernel runs.
// Inside a decode the score scan has already summed each selected key's
// products over the first d columns: given those scores (and d >= D / 2), the
// kernel reads only columns [d, D) of the key rows and adds the stored score,
// so the gather moves (D - d) / D of the key bytes (the value rows in full).
#include "common.cuh"
#include "launch.h"

namespace loki {

// Work decomposition. Each (batch, query head) row's k selected positions are
// cut into blocks of kBlk; the rows' blocks are laid end to end (N in all)
// and every warp of one full wave takes an equal contiguous range of them,
// warp w the blocks [w N / W, (w + 1) N / W). A range covers the tail of one
// row, whole rows and the head of another, so every SM gets the same share of
// the gather. A warp that covers a whole row writes its output directly;
// otherwise it leaves a partial (m, l, acc) for each row it touches. The
// warps touching row r are consecutive, w_first(r) .. w_last(r), and warp w's
// partial of row r goes to slot r + w: no two (row, warp) pairs share a slot
// since a later warp never touches an earlier row. Slots stay below rows + W.
constexpr int kBlk = 16;
constexpr int kWarpIdx = 256;  // indices staged per warp per step

int64_t sparse_max_parts(int64_t rows, int64_t k) {
    int64_t cap = 10240 / rows;
    if (cap < 1) cap = 1;
    const int64_t by_k = (k + kBlk - 1) / kBlk;
    return (by_k < cap ? by_k : cap) + 2;
}

// The warp whose block range holds block b (W warps over N blocks).
__device__ __forceinline__ int64_t owner_warp(int64_t b, int64_t W, int64_t N) {
    return ((b + 1) * W - 1) / N;
}

// Issue the key and value loads of one batch: U rows per row group, rows
// jb + u * GPW + grp of the staged index list (indices past n, or -1 for an
// index outside [0, S), load nothing and give zeros; so do lanes past the
// head dimension, and for the key, lanes whose columns the stored scores
// cover: k_on false).
template <int U, int GPW>
__device__ __forceinline__ void sp_load(const int* widx, int n, int jb, int grp, const char* Kb,
                                        const char* Vb, int64_t row_bytes, bool lane_on, bool k_on,
                                        int (&t)[U], uint4 (&kv)[U], uint4 (&vv)[U]) {
#pragma unroll
    for (int u = 0; u < U; ++u) {
        const int jj = jb + u * GPW + grp;
        const int tok = jj < n ? widx[jj] : -1;
        t[u] = tok;
        kv[u] = make_uint4(0u, 0u, 0u, 0u);
        vv[u] = kv[u];
        if (tok >= 0) {
            if (k_on) kv[u] = ld_stream(Kb + (int64_t)tok * row_bytes);
            if (lane_on) vv[u] = ld_stream(Vb + (int64_t)tok * row_bytes);
        }
    }
}

// Fold one loaded batch into the row group's running softmax state (m, l,
// acc) in base 2: full-D scores (with kLo, the stored part of row jb + u *
// GPW + grp from wsc plus the loaded columns), then the value rows weighted
// by 2^(s - m).
template <class E, int U, int LPR, int GPW, bool kLo>
__device__ __forceinline__ void sp_consume(const float (&qv)[E::kVec], const int (&t)[U],
                                           const uint4 (&kv)[U], const uint4 (&vv)[U],
                                           const float* wsc, int jb, int grp, float& m, float& l,
                                           float (&acc)[E::kVec]) {
    constexpr int KV = E::kVec;
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
        if constexpr (kLo) a += t[u] >= 0 ? wsc[jb + u * GPW + grp] : 0.f;
        sc[u] = t[u] >= 0 ? a : -INFINITY;
        mx = fmaxf(mx, sc[u]);
    }
    if (mx == -INFINITY) return;  // nothing in this batch for this row group
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

// rows in flight per row group, resident CTAs per SM (measured: more CTAs
// with fewer rows each, or two batches in flight per warp, are no faster)
constexpr int kSpU = 8;
constexpr int kSpMinBlocks = 2;

// DH: head dimension (96 or 128). The lanes keep the layout of 128 columns;
// those past DH load nothing and write nothing.
// kLo: sc_lo [rows, S] holds each token's score over the first skip * kVec
// columns (q~ . K~ unscaled); lanes of those columns load no key chunk.
template <class E, int DH, bool kLo>
__global__ void __launch_bounds__(256, kSpMinBlocks) k_sparse_attn(
    const float* __restrict__ q_rot, const typename E::T* __restrict__ Kt,
    const typename E::T* __restrict__ V, const int32_t* __restrict__ idx, int H_q, int H_kv, int S,
    int64_t S_max, int k, float scale_log2, int nblk, int64_t N, int64_t W,
    float2* __restrict__ part_ml, float* __restrict__ part_acc, int* __restrict__ done,
    typename E::T* __restrict__ out, const int* __restrict__ block_table, int page_size,
    int max_pages, int64_t n_pages, const int* __restrict__ lens, int* __restrict__ err,
    const float* __restrict__ sc_lo, int skip) {
    constexpr int D = DH;
    constexpr int KV = E::kVec;
    constexpr int LPR = 128 / KV;   // lanes per row
    constexpr int GPW = 32 / LPR;   // row groups per warp
    constexpr int U = kSpU;         // rows in flight per group
    constexpr int64_t kRowBytes = (int64_t)D * E::kBytes;
    __shared__ int s_idx[8][kWarpIdx];
    __shared__ float s_sc[kLo ? 8 : 1][kLo ? kWarpIdx : 1];  // stored scores, in base 2

    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int grp = lane / LPR, sub = lane % LPR;
    const bool lane_on = sub * KV < D;
    const bool k_on = lane_on && (!kLo || sub >= skip);
    const int G = H_q / H_kv;
    int* widx = s_idx[warp];
    float* wsc = s_sc[kLo ? warp : 0];

    // this warp's blocks [bcur, bend); W <= N, so no warp's range is empty
    const int64_t w = (int64_t)blockIdx.x * 8 + warp;
    int64_t bcur = w < W ? w * N / W : 0;
    const int64_t bend = w < W ? (w + 1) * N / W : 0;
    // The first row's q~ is read before the wait: this kernel is launched
    // behind top-k, whose CTAs let it start only after their own wait on the
    // kernels that wrote q~ (or, without programmatic launch, after all of
    // them). The selected indices are read after the wait.
    float qv0[KV];
    {
        const float* qp = q_rot + (bcur / nblk) * D + sub * KV;
#pragma unroll
        for (int e = 0; e < KV; ++e)
            qv0[e] = (lane_on && bcur < bend) ? __ldg(qp + e) * scale_log2 : 0.f;
    }
    bool first = true;
    griddep_wait();  // the selected indices come from top-k
    griddep_launch_dependents();

    while (bcur < bend) {
        const int64_t r = bcur / nblk;
        const int64_t rb1 = min64(bend, (r + 1) * nblk);
        const int j0 = (int)(bcur - r * nblk) * kBlk;
        const int j1 = min(k, (int)(rb1 - r * nblk) * kBlk);
        bcur = rb1;
        const int b = (int)(r / H_q), h = (int)(r % H_q);
        const int64_t unit = (int64_t)b * H_kv + h / G;

        float qv[KV];
        if (first) {
#pragma unroll
            for (int e = 0; e < KV; ++e) qv[e] = qv0[e];
            first = false;
        } else {
            const float* qp = q_rot + r * D + sub * KV;
#pragma unroll
            for (int e = 0; e < KV; ++e) qv[e] = lane_on ? __ldg(qp + e) * scale_log2 : 0.f;
        }
        // contiguous cache: rows of the unit; paged: rows of the page pool
        const int64_t base_row = block_table != nullptr ? 0 : unit * S_max;
        const char* Kb = reinterpret_cast<const char*>(Kt) + base_row * kRowBytes + sub * 16;
        const char* Vb = reinterpret_cast<const char*>(V) + base_row * kRowBytes + sub * 16;
        const int32_t* ip = idx + r * k;
        const int S_row = lens != nullptr ? min(S, max(0, lens[b])) : S;
        const int hk = h / G;

        float m = -INFINITY, l = 0.f, acc[KV];
#pragma unroll
        for (int e = 0; e < KV; ++e) acc[e] = 0.f;

        for (int cb = j0; cb < j1; cb += kWarpIdx) {
            const int n = min(kWarpIdx, j1 - cb);
            __syncwarp();
            {
                // all of a lane's indices in flight at once (n <= 256 = 8 x 32)
                int tk[kWarpIdx / 32];
#pragma unroll
                for (int u = 0; u < kWarpIdx / 32; ++u) {
                    const int t = lane + 32 * u;
                    tk[u] = t < n ? __ldg(ip + cb + t) : -1;
                }
                if constexpr (kLo) {
                    // the scan's scores of the valid tokens (all loads in flight)
                    const float* sp = sc_lo + r * S;
                    float sv[kWarpIdx / 32];
#pragma unroll
                    for (int u = 0; u < kWarpIdx / 32; ++u) {
                        const int t = lane + 32 * u;
                        sv[u] = (t < n && (unsigned)tk[u] < (unsigned)S_row) ? __ldg(sp + tk[u])
                                                                              : 0.f;
                    }
#pragma unroll
                    for (int u = 0; u < kWarpIdx / 32; ++u) {
                        const int t = lane + 32 * u;
                        if (t < n) wsc[t] = sv[u] * scale_log2;
                    }
                }
#pragma unroll
                for (int u = 0; u < kWarpIdx / 32; ++u) {
                    const int t = lane + 32 * u;
                    int tok = (t < n && (unsigned)tk[u] < (unsigned)S_row) ? tk[u] : -1;
                    if (block_table != nullptr && tok >= 0) {
                        // token -> row of the page pool (< 2^31 rows, checked on the host)
                        const int page = __ldg(block_table + (int64_t)b * max_pages + tok / page_size);
                        if (page < 0 || page >= n_pages) {
                            atomicExch(err, 2);  // a bad block-table entry: skip the token
                            tok = -1;
                        } else {
                            tok = (int)(((int64_t)page * H_kv + hk) * page_size + tok % page_size);
                        }
                    }
                    if (t < n) widx[t] = tok;
                }
            }
            __syncwarp();
            for (int jb = 0; jb < n; jb += GPW * U) {
                int t[U];
                uint4 kv[U], vv[U];
                sp_load<U, GPW>(widx, n, jb, grp, Kb, Vb, kRowBytes, lane_on, k_on, t, kv, vv);
                sp_consume<E, U, LPR, GPW, kLo>(qv, t, kv, vv, wsc, jb, grp, m, l, acc);
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
        const int64_t wf = owner_warp(r * nblk, W, N);
        const int64_t wl = owner_warp((r + 1) * nblk - 1, W, N);
        if (wf == wl) {  // the whole row is this warp's: normalise and write it
            if (grp == 0 && lane_on) {
                const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll
                for (int e = 0; e < KV; ++e) out[r * D + sub * KV + e] = E::from_float(acc[e] * inv);
            }
            continue;
        }
        const int64_t slot = r + w;
        if (grp == 0 && lane_on) {
            float* pa = part_acc + slot * D + sub * KV;
#pragma unroll
            for (int e = 0; e < KV; e += 4)
                *reinterpret_cast<float4*>(pa + e) = make_float4(acc[e], acc[e + 1], acc[e + 2], acc[e + 3]);
            if (sub == 0) part_ml[slot] = make_float2(m, l);
        }
        // The last warp to finish its part of row r merges the row's partials
        // (its own included) into out[r]: publish, count, and only the warp
        // that sees the count reach the number of parts reads the others'.
        const int nparts = (int)(wl - wf + 1);
        // the warp's partial writes, then lane 0 counts the part with a
        // release-acquire add: the last part's warp sees every other part
        __syncwarp();
        int prev = 0;
        if (lane == 0) prev = atom_add_acq_rel_gpu(done + r, 1);
        prev = __shfl_sync(0xffffffffu, prev, 0);
        __syncwarp();
        if (prev == nparts - 1) {
            // lane l merges columns [4 l, 4 l + 4) over all parts
            const float2* ml = part_ml + r + wf;
            const float* pacc = part_acc + (r + wf) * D;
            const bool col_on = 4 * lane < D;
            // (m, l) of part p on lane p (parts past 32, rare, are re-read),
            // and the parts' columns sixteen at a time, all sixteen loads in
            // flight together (the first sixteen already behind the max)
            constexpr int kPB = 16;
            const float2 mlp = lane < nparts ? __ldcg(&ml[lane]) : make_float2(-INFINITY, 0.f);
            float4 ap[kPB];
            auto load_parts = [&](int p0) {
#pragma unroll
                for (int j = 0; j < kPB; ++j)
                    ap[j] = (p0 + j < nparts && col_on)
                                ? __ldcg(reinterpret_cast<const float4*>(pacc + (int64_t)(p0 + j) * D) +
                                         lane)
                                : make_float4(0.f, 0.f, 0.f, 0.f);
            };
            load_parts(0);
            float M = mlp.x;
            for (int p = lane + 32; p < nparts; p += 32) M = fmaxf(M, __ldcg(&ml[p].x));
#pragma unroll
            for (int off = 16; off >= 1; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
            float Lsum = 0.f;
            float4 A = make_float4(0.f, 0.f, 0.f, 0.f);
            if (M != -INFINITY) {
                Lsum = lane < nparts ? mlp.y * exp2f(mlp.x - M) : 0.f;
                for (int p = lane + 32; p < nparts; p += 32) {
                    const float2 e = __ldcg(&ml[p]);
                    Lsum += e.y * exp2f(e.x - M);
                }
                for (int p0 = 0; p0 < nparts; p0 += kPB) {
                    if (p0 > 0) load_parts(p0);
#pragma unroll
                    for (int j = 0; j < kPB; ++j) {
                        const int p = p0 + j;
                        if (p < nparts) {
                            const float mp = p < 32 ? __shfl_sync(0xffffffffu, mlp.x, p & 31)
                                                    : __ldcg(&ml[p].x);
                            const float sc = exp2f(mp - M);
                            A.x = fmaf(ap[j].x, sc, A.x);
                            A.y = fmaf(ap[j].y, sc, A.y);
                            A.z = fmaf(ap[j].z, sc, A.z);
                            A.w = fmaf(ap[j].w, sc, A.w);
                        }
                    }
                }
            }
#pragma unroll
            for (int off = 16; off >= 1; off >>= 1) Lsum += __shfl_xor_sync(0xffffffffu, Lsum, off);
            const float inv = Lsum > 0.f ? 1.f / Lsum : 0.f;
            if (4 * lane < D) {
                typename E::T* o = out + r * D + 4 * lane;
                o[0] = E::from_float(A.x * inv);
                o[1] = E::from_float(A.y * inv);
                o[2] = E::from_float(A.z * inv);
                o[3] = E::from_float(A.w * inv);
            }
            if (lane == 0) done[r] = 0;  // leave the counter ready for the next call
        }
    }
}

template <class E, int DH>
static cudaError_t sparse_impl(const float* q_rot, const void* Kt, const void* V,
                               const int32_t* idx, int B, int H_q, int H_kv, int64_t S,
                               int64_t S_max, int D, int64_t k, float scale, void* out,
                               float2* part_ml, float* part_acc, int* done, cudaStream_t s,
                               bool pdl, const PagedKV& pg, const float* sc_lo, int d_sc) {
    DevInfo di;
    cudaError_t e = dev_info(&di);
    if (e != cudaSuccess) return e;
    const int64_t rows = (int64_t)B * H_q;
    // only whole 16-byte chunks are skipped, and the stored scores pay off
    // once they cover half the key row (measured at D = 128, bf16: d = 64
    // takes 4 % off the step; at d = 32 the extra score loads cost what the
    // 64 bytes fewer per key row save, the random gather being bound by its
    // row count more than its bytes)
    const int skip = (sc_lo != nullptr && d_sc < D && d_sc % E::kVec == 0 && 2 * d_sc >= D)
                         ? d_sc / E::kVec
                         : 0;
    auto kern = skip > 0 ? k_sparse_attn<E, DH, true> : k_sparse_attn<E, DH, false>;
    // the gathers in flight live in L1: the smallest shared split that still
    // holds two CTAs' staged indices (8 KB each, 16 KB with the stored
    // scores, plus 1 KB reserved per CTA)
    const int kb = skip > 0 ? 16 : 8;
    const int pct = (2 * (kb + 1) * 1024 * 100 + di.smem_optin - 1) / di.smem_optin + 1;
    e = prefer_carveout((const void*)kern, pct);
    if (e != cudaSuccess) return e;
    const int64_t nblk = (k + kBlk - 1) / kBlk;
    const int64_t N = rows * nblk;
    // one full wave of warps, but no more warps than blocks (no empty range)
    // and no more partial slots (rows + W) than the workspace holds
    int64_t W = (int64_t)di.sm_count * occupancy((const void*)kern, 256, 0) * 8;
    const int64_t cap = rows * (sparse_max_parts(rows, k) - 1);
    if (W > cap) W = cap;
    // at most 32 parts per row: every part costs its row's merge a load
    if (W > rows * 32) W = rows * 32;
    if (W > N) W = N;
    const int64_t grid = (W + 7) / 8;
    using T = typename E::T;
    return launch_kernel(kern, dim3((unsigned)grid), dim3(256), 0, s, pdl, q_rot,
                         static_cast<const T*>(Kt), static_cast<const T*>(V), idx, H_q, H_kv,
                         (int)S, S_max, (int)k, scale * kLog2e, (int)nblk, N, W, part_ml,
                         part_acc, done, static_cast<T*>(out), pg.block_table, pg.page_size,
                         pg.max_pages, pg.n_pages, pg.lens, device_error_word(),
                         skip > 0 ? sc_lo : nullptr, skip);
}

cudaError_t launch_sparse_attention(Dt dt, const float* q_rot, const void* Kt, const void* V,
                                    const int32_t* idx, int B, int H_q, int H_kv, int64_t S,
                                    int64_t S_max, int D, int64_t k, float scale, void* out,
                                    float2* part_ml, float* part_acc, int* done, cudaStream_t s,
                                    bool pdl, const PagedKV& pg, const float* sc_lo, int d_sc) {
    if (D != 96 && D != 128) return cudaErrorInvalidValue;
    if (dt == kF32)
        return D == 96 ? sparse_impl<ElemF32, 96>(q_rot, Kt, V, idx, B, H_q, H_kv, S, S_max, D, k,
                                                  scale, out, part_ml, part_acc, done, s, pdl, pg,
                                                  sc_lo, d_sc)
                       : sparse_impl<ElemF32, 128>(q_rot, Kt, V, idx, B, H_q, H_kv, S, S_max, D,
                                                   k, scale, out, part_ml, part_acc, done, s, pdl,
                                                   pg, sc_lo, d_sc);
    return D == 96 ? sparse_impl<ElemBF16, 96>(q_rot, Kt, V, idx, B, H_q, H_kv, S, S_max, D, k,
                                               scale, out, part_ml, part_acc, done, s, pdl, pg,
                                               sc_lo, d_sc)
                   : sparse_impl<ElemBF16, 128>(q_rot, Kt, V, idx, B, H_q, H_kv, S, S_max, D, k,
                                                scale, out, part_ml, part_acc, done, s, pdl, pg,
                                                sc_lo, d_sc);
}

}  // namespace loki
