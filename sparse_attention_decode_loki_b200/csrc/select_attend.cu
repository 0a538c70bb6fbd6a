// Token selection and exact attention over the selected tokens in one
// persistent kernel (Loki's top-k and final attention: NeurIPS 2024 poster
// page, TL;DR -- keep the k tokens with the largest approximate scores, then
// compute full-dimensional scores only for them; "Visual Insights" Figure 1
// caption).
//
// One CTA per SM takes the (batch, query head) rows r = blockIdx.x + i *
// gridDim.x in turn, with two warp roles:
//   * 8 selector warps read row r's fp32 scores (written by the score scan,
//     still in L2), select the k largest with the register radix select of
//     topk_select.cuh (on their own named barrier) and write the ascending
//     selection to a shared-memory buffer and to selected_idx;
//   * 8 gatherer warps take the selection of the previous row from the other
//     buffer, each gathering k / 8 of its key and value rows (16-byte loads,
//     8 rows in flight per row group) with an online softmax in base 2; the
//     warps' partials meet in shared memory and one merge writes the output.
// The two buffers pass between the roles through mbarriers, so the
// selection of row i + 1 overlaps the gather of row i, and a row is only
// ever gathered by one CTA: no partials in global memory, no atomics. Used
// for small decodes (few rows, few selected tokens), where one kernel instead
// of two saves a launch boundary.
#include "common.cuh"
#include "launch.h"
#include "tma.cuh"
#include "topk_select.cuh"

namespace loki {

constexpr int kSaSelThreads = 256;
constexpr int kSaGatThreads = 256;
constexpr int kSaThreads = kSaSelThreads + kSaGatThreads;
constexpr int kSaGatWarps = kSaGatThreads / 32;
constexpr int kSaBarSel = 1;  // named barriers of the two roles
constexpr int kSaBarGat = 2;

// Issue one batch of gathers for a row group (U rows of the warp's share,
// rows jb + u * GPW + grp of the list `sel` of n indices).
template <int U, int GPW>
__device__ __forceinline__ void sa_load(const int* sel, int n, int jb, int grp, const char* Kb,
                                        const char* Vb, int64_t row_bytes, int (&t)[U],
                                        uint4 (&kv)[U], uint4 (&vv)[U]) {
#pragma unroll
    for (int u = 0; u < U; ++u) {
        const int jj = jb + u * GPW + grp;
        const int tok = jj < n ? sel[jj] : -1;
        t[u] = tok;
        if (tok >= 0) {
            kv[u] = ld_stream(Kb + (int64_t)tok * row_bytes);
            vv[u] = ld_stream(Vb + (int64_t)tok * row_bytes);
        } else {
            kv[u] = make_uint4(0u, 0u, 0u, 0u);
            vv[u] = kv[u];
        }
    }
}

// I: groups of 4 keys per selector thread (S <= 1024 * I).
template <class E, int I>
__global__ void __launch_bounds__(kSaThreads, 1) k_select_attend(
    const float* __restrict__ scores, const float* __restrict__ q_rot,
    const typename E::T* __restrict__ Kt, const typename E::T* __restrict__ V, int H_q, int H_kv,
    int S, int64_t S_max, int k, float scale_log2, int64_t rows, int vec4,
    int32_t* __restrict__ sel_out, typename E::T* __restrict__ out, int* __restrict__ err) {
    constexpr int D = 128;
    constexpr int KV = E::kVec;
    constexpr int LPR = D / KV;    // lanes per gathered row
    constexpr int GPW = 32 / LPR;  // row groups per warp
    constexpr int U = 8;           // rows in flight per row group
    constexpr int64_t kRowBytes = (int64_t)D * E::kBytes;
    extern __shared__ __align__(16) int s_sel[];  // [2][k]
    __shared__ __align__(16) uint32_t s_tk[kTkSmemWords];
    __shared__ float s_part[kSaGatWarps][2 + D];
    __shared__ uint64_t bar_full[2], bar_empty[2];
    __shared__ int s_ok[2];  // per role: the leader's last wait succeeded

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (tid == 0) {
        for (int b = 0; b < 2; ++b) {
            mbar_init(&bar_full[b], 1);
            mbar_init(&bar_empty[b], 1);
        }
        fence_mbar_init();
    }
    __syncthreads();
    griddep_wait();  // scores and q~ come from the preceding kernels
    griddep_launch_dependents();
    const int G = H_q / H_kv;

    if (tid < kSaSelThreads) {
        // ---------------- selectors ----------------
        using SelCl = TkCluster<false, kSaBarSel, kSaSelThreads>;
        const SelCl cl;
        const TkSmem sm = tk_carve(s_tk);
        int i = 0;
        for (int64_t r = blockIdx.x; r < rows; r += gridDim.x, ++i) {
            const int b = i & 1;
            const uint32_t ph = (uint32_t)(i >> 1) & 1u;
            // buffer b is free once the gatherers are done with row i - 2
            if (tid == 0) s_ok[0] = mbar_wait(&bar_empty[b], ph ^ 1u, err) ? 1 : 0;
            tk_zero<kSaSelThreads>(sm);
            cl.bsync();
            if (!s_ok[0]) break;
            const float* src = scores + r * S;
            uint4 v[I];
#pragma unroll
            for (int u = 0; u < I; ++u) {
                const int g = warp * 32 * I + 32 * u + lane;  // keys 4g .. 4g + 3
                const int j = 4 * g;
                if (vec4 && j + 3 < S) {
                    const float4 f = __ldcg(reinterpret_cast<const float4*>(src) + g);
                    v[u] = make_uint4(order_key(f.x), order_key(f.y), order_key(f.z), order_key(f.w));
                } else {
                    v[u] = make_uint4(j < S ? order_key(__ldcg(src + j)) : 0u,
                                      j + 1 < S ? order_key(__ldcg(src + j + 1)) : 0u,
                                      j + 2 < S ? order_key(__ldcg(src + j + 2)) : 0u,
                                      j + 3 < S ? order_key(__ldcg(src + j + 3)) : 0u);
                }
            }
#pragma unroll
            for (int u = 0; u < I; ++u) {
                const uint32_t kk[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    if (kk[e] != 0u) atomicAdd(&sm.hist1[kk[e] >> 21], 1u);
            }
            int* buf = s_sel + b * k;
            tk_select<kSaSelThreads, I, false, kSaBarSel>(cl, v, 0, k, buf, sm);
            cl.bsync();  // the whole selection is in buf
            int32_t* so = sel_out + r * k;
            for (int x = tid; x < k; x += kSaSelThreads) so[x] = buf[x];
            if (tid == 0) mbar_arrive(&bar_full[b]);  // release: buf holds row r
        }
        return;
    }

    // ---------------- gatherers ----------------
    const int gt = tid - kSaSelThreads, gw = gt >> 5;
    const int grp = lane / LPR, sub = lane % LPR;
    int i = 0;
    for (int64_t r = blockIdx.x; r < rows; r += gridDim.x, ++i) {
        const int b = i & 1;
        const uint32_t ph = (uint32_t)(i >> 1) & 1u;
        if (gt == 0) s_ok[1] = mbar_wait(&bar_full[b], ph, err) ? 1 : 0;
        named_sync(kSaBarGat, kSaGatThreads);
        if (!s_ok[1]) break;
        const int* buf = s_sel + b * k;
        const int bb = (int)(r / H_q), h = (int)(r % H_q);
        const int64_t unit = (int64_t)bb * H_kv + h / G;
        float qv[KV];
        {
            const float* qp = q_rot + r * D + sub * KV;
#pragma unroll
            for (int e = 0; e < KV; ++e) qv[e] = __ldcg(qp + e) * scale_log2;
        }
        const char* Kb = reinterpret_cast<const char*>(Kt) + unit * S_max * kRowBytes + sub * 16;
        const char* Vb = reinterpret_cast<const char*>(V) + unit * S_max * kRowBytes + sub * 16;
        // this warp's share of the selection
        const int j0 = (int)((int64_t)gw * k / kSaGatWarps);
        const int j1 = (int)((int64_t)(gw + 1) * k / kSaGatWarps);
        const int* wsel = buf + j0;
        const int n = j1 - j0;
        float m = -INFINITY, l = 0.f, acc[KV];
#pragma unroll
        for (int e = 0; e < KV; ++e) acc[e] = 0.f;
        for (int jb = 0; jb < n; jb += GPW * U) {
            int t[U];
            uint4 kv[U], vv[U];
            sa_load<U, GPW>(wsel, n, jb, grp, Kb, Vb, kRowBytes, t, kv, vv);
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
            if (mx != -INFINITY) {
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
#pragma unroll
            for (int e = 0; e < KV; ++e) s_part[gw][2 + sub * KV + e] = acc[e];
            if (sub == 0) {
                s_part[gw][0] = m;
                s_part[gw][1] = l;
            }
        }
        named_sync(kSaBarGat, kSaGatThreads);  // partials written; buf no longer read
        if (gt == 0) mbar_arrive(&bar_empty[b]);
        if (gt < D) {
            float M = -INFINITY;
#pragma unroll
            for (int w = 0; w < kSaGatWarps; ++w) M = fmaxf(M, s_part[w][0]);
            float L = 0.f, A = 0.f;
            if (M != -INFINITY) {
#pragma unroll
                for (int w = 0; w < kSaGatWarps; ++w) {
                    const float s2 = exp2f(s_part[w][0] - M);
                    L += s_part[w][1] * s2;
                    A += s_part[w][2 + gt] * s2;
                }
            }
            out[r * D + gt] = E::from_float(L > 0.f ? A / L : 0.f);
        }
        named_sync(kSaBarGat, kSaGatThreads);  // s_part is reused by the next row
    }
}

// ---------------------------------------------------------------------------

bool select_attend_fits(Dt dt, int64_t rows, int64_t S, int D, int64_t k) {
    (void)dt;
    // Small decodes only (measured): there the kernel boundary between top-k
    // and attention dominates, and one CTA per row gathers few tokens. On
    // large ones, eight gatherer warps per SM keep too few rows in flight and
    // the stream-K gather over every SM wins.
    return D == 128 && S >= 1 && S <= 8192 && k >= 1 && k <= S && rows * k <= 8192;
}

template <class E, int I>
static cudaError_t sa_impl(const float* scores, const float* q_rot, const void* Kt, const void* V,
                           int B, int H_q, int H_kv, int64_t S, int64_t S_max, int64_t k,
                           float scale, void* out, int32_t* sel, cudaStream_t s, bool pdl) {
    DevInfo di;
    cudaError_t e = dev_info(&di);
    if (e != cudaSuccess) return e;
    int* err = device_error_word();
    if (err == nullptr) return cudaErrorInvalidDevice;
    auto kern = k_select_attend<E, I>;
    const size_t smem = (size_t)2 * k * sizeof(int);
    static bool attr_set[64] = {};
    if (di.device < 64 && !attr_set[di.device]) {
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, 2 * 8192 * 4);
        if (e != cudaSuccess) return e;
        attr_set[di.device] = true;
    }
    const int64_t rows = (int64_t)B * H_q;
    const int64_t grid = rows < di.sm_count ? rows : di.sm_count;
    const int vec4 = (S % 4 == 0) && (reinterpret_cast<uintptr_t>(scores) % 16 == 0);
    using T = typename E::T;
    return launch_kernel(kern, dim3((unsigned)grid), dim3(kSaThreads), smem, s, pdl, scores, q_rot,
                         static_cast<const T*>(Kt), static_cast<const T*>(V), H_q, H_kv, (int)S,
                         S_max, (int)k, scale * kLog2e, rows, vec4, sel, static_cast<T*>(out), err);
}

template <class E>
static cudaError_t sa_dispatch(const float* scores, const float* q_rot, const void* Kt,
                               const void* V, int B, int H_q, int H_kv, int64_t S, int64_t S_max,
                               int64_t k, float scale, void* out, int32_t* sel, cudaStream_t s,
                               bool pdl) {
    if (S <= 1024)
        return sa_impl<E, 1>(scores, q_rot, Kt, V, B, H_q, H_kv, S, S_max, k, scale, out, sel, s, pdl);
    if (S <= 2048)
        return sa_impl<E, 2>(scores, q_rot, Kt, V, B, H_q, H_kv, S, S_max, k, scale, out, sel, s, pdl);
    if (S <= 4096)
        return sa_impl<E, 4>(scores, q_rot, Kt, V, B, H_q, H_kv, S, S_max, k, scale, out, sel, s, pdl);
    return sa_impl<E, 8>(scores, q_rot, Kt, V, B, H_q, H_kv, S, S_max, k, scale, out, sel, s, pdl);
}

cudaError_t launch_select_attend(Dt dt, const float* scores, const float* q_rot, const void* Kt,
                                 const void* V, int B, int H_q, int H_kv, int64_t S,
                                 int64_t S_max, int64_t k, float scale, void* out, int32_t* sel,
                                 cudaStream_t s, bool pdl) {
    if (dt == kF32)
        return sa_dispatch<ElemF32>(scores, q_rot, Kt, V, B, H_q, H_kv, S, S_max, k, scale, out,
                                    sel, s, pdl);
    return sa_dispatch<ElemBF16>(scores, q_rot, Kt, V, B, H_q, H_kv, S, S_max, k, scale, out, sel,
                                 s, pdl);
}

}  // namespace loki
