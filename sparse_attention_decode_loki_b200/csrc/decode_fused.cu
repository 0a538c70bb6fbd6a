// Fused Loki decode step over a low-dimensional key plane: one CTA per
// (batch, KV head) unit runs every step of the method for that unit.
//
// Loki (briefgpt.xyz abstract page; NeurIPS 2024 poster page, TL;DR and
// "Visual Insights" Figure 1 caption): rotate the query by the unit's PCA
// basis, q~ = q P; score every cached token on the first d principal
// components, s_j = q~[:d] . K~_j[:d]; keep the k tokens with the largest
// scores; attend exactly over those k tokens with full-dimensional keys.
//
// Phases of one CTA (256 threads, G query heads of the unit):
//   0. thread 0 starts streaming the unit's plane rows (cp.async.bulk into a
//      ring of shared-memory tiles, one mbarrier per stage) while all
//      threads rotate the G queries (P read from L2, fp32) into shared memory;
//   1. score scan: one plane row per thread and tile, G dot products each,
//      stored as order-preserving keys in shared memory (the scores never
//      touch HBM);
//   2. exact radix top-k per query head over the keys in shared memory
//      (topk_select.cuh); the selection goes to shared memory and to
//      selected_idx;
//   3. sparse attention: each warp gathers its share of one head's selected
//      key and value rows (16-byte loads, U rows per row group in flight) with
//      an online softmax in base 2; the warps' partials meet in shared memory
//      and are merged into the output rows.
// Several CTAs share an SM, each in its own phase, so one unit's top-k and
// pipeline ramps overlap other units' memory streams, and the hardware block
// scheduler balances the units over the SMs.
#include "common.cuh"
#include "launch.h"
#include "tma.cuh"
#include "topk_select.cuh"

namespace loki {

constexpr int kFusedThreads = 256;
constexpr int kFusedWarps = kFusedThreads / 32;
constexpr int kFusedRows = kFusedThreads;  // plane rows per scan tile (one per thread)
constexpr int kFusedStages = 3;
constexpr int kFusedMaxS = 32 * kFusedThreads;  // rows per head the block top-k handles

__host__ __device__ constexpr int fused_align16(int x) { return (x + 15) & ~15; }

// Byte offsets of the dynamic shared-memory regions of one CTA.
struct FusedLayout {
    int ring;   // scan tiles; afterwards top-k scratch, then the warps' partials
    int keys;   // G x Spad order keys (Spad = S rounded up to 4)
    int sel;    // G x k selected indices
    int qin;    // G x 128 fp32 raw queries
    int qpart;  // 2 x G x 128 fp32 halves of the rotation
    int qrot;   // G x 128 fp32 rotated queries (the gather's)
    int qlo;    // G x C fp32 rotated queries, zero beyond column d (the scan's)
    int total;
};

// nv: 16-byte chunks per plane row; cols: plane row width in elements
__host__ __device__ inline FusedLayout fused_layout(int nv, int cols, int G, int S, int k) {
    const int tile = kFusedRows * nv * 16;
    int ring = kFusedStages * tile;
    const int topk_scratch = kTkSmemWords * 4;
    const int partials = kFusedWarps * (2 + 128) * 4;
    if (ring < topk_scratch) ring = topk_scratch;
    if (ring < partials) ring = partials;
    FusedLayout L;
    L.ring = 0;
    L.keys = fused_align16(ring);
    L.sel = L.keys + fused_align16(G * ((S + 3) & ~3) * 4);
    L.qin = L.sel + fused_align16(G * k * 4);
    L.qpart = L.qin + G * 128 * 4;
    L.qrot = L.qpart + 2 * G * 128 * 4;
    L.qlo = L.qrot + G * 128 * 4;
    L.total = L.qlo + G * cols * 4;
    return L;
}

// E: element traits; NV: 16-byte chunks per plane row; U: rows in flight per
// row group in the gather; MINB: resident CTAs per SM the registers allow.
template <class E, int NV, int U, int MINB>
__global__ void __launch_bounds__(kFusedThreads, MINB) k_decode_fused(
    const typename E::T* __restrict__ q, const float* __restrict__ P,
    const typename E::T* __restrict__ Klo, const typename E::T* __restrict__ Kt,
    const typename E::T* __restrict__ V, int H_q, int H_kv, int G, int S, int64_t S_max, int d,
    int k, float scale_log2, typename E::T* __restrict__ out, int32_t* __restrict__ sel_out,
    int* __restrict__ err) {
    using T = typename E::T;
    constexpr int D = 128;
    constexpr int KV = E::kVec;
    constexpr int C = NV * KV;             // plane row width in elements
    constexpr int kRowBytes = NV * 16;     // plane row bytes
    constexpr int kTile = kFusedRows * kRowBytes;
    constexpr int LPR = D / KV;            // gather lanes per cache row
    constexpr int GPW = 32 / LPR;          // gather row groups per warp
    constexpr int64_t kCacheRow = (int64_t)D * E::kBytes;
    extern __shared__ __align__(128) unsigned char smem[];
    __shared__ uint64_t full[kFusedStages];

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int64_t unit = blockIdx.x;
    const int b = (int)(unit / H_kv), hk = (int)(unit % H_kv);
    const int Spad = (S + 3) & ~3;
    const FusedLayout L = fused_layout(NV, C, G, S, k);
    unsigned char* ring = smem + L.ring;
    uint32_t* keys = reinterpret_cast<uint32_t*>(smem + L.keys);
    int32_t* sel = reinterpret_cast<int32_t*>(smem + L.sel);
    float* qin = reinterpret_cast<float*>(smem + L.qin);
    float* qpart = reinterpret_cast<float*>(smem + L.qpart);
    float* qrot = reinterpret_cast<float*>(smem + L.qrot);
    float* qlo = reinterpret_cast<float*>(smem + L.qlo);
    const int ntiles = (S + kFusedRows - 1) / kFusedRows;
    const char* plane = reinterpret_cast<const char*>(Klo) + unit * S_max * kRowBytes;

    if (tid == 0) {
        for (int s = 0; s < kFusedStages; ++s) mbar_init(&full[s], 1);
        fence_mbar_init();
    }
    __syncthreads();
    griddep_wait();  // inputs may come from the preceding kernel (an append)

    // ---- 0. start the key stream; rotate the queries meanwhile ------------------
    // (the plane is read once: evict-first keeps it from displacing the
    // gathered rows other CTAs are reading)
    const uint64_t pol = l2_policy_evict_first();
    auto issue = [&](int t) {
        const int st = t % kFusedStages;
        const int n = min(kFusedRows, S - t * kFusedRows);
        mbar_arrive_expect_tx(&full[st], (uint32_t)(n * kRowBytes));
        bulk_load_hint(ring + st * kTile, plane + (int64_t)t * kFusedRows * kRowBytes,
                       (uint32_t)(n * kRowBytes), &full[st], pol);
    };
    if (tid == 0)
        for (int t = 0; t < kFusedStages && t < ntiles; ++t) issue(t);
    {
        const T* qb = q + ((int64_t)b * H_q + (int64_t)hk * G) * D;  // the unit's G rows
        for (int x = tid; x < G * D; x += kFusedThreads) qin[x] = E::load1(qb + x);
    }
    __syncthreads();
    {
        // thread (half h, column c) sums rows [64h, 64h + 64) of column c of
        // P for every head, 32 loads of P in flight at a time; the halves
        // meet in shared memory
        const int c = tid & 127, h = tid >> 7;
        const float* Pc = P + ((int64_t)hk * D + h * 64) * D + c;
        float acc[8];
#pragma unroll
        for (int g = 0; g < 8; ++g) acc[g] = 0.f;
#pragma unroll
        for (int i0 = 0; i0 < 64; i0 += 32) {
            float pv[32];
#pragma unroll
            for (int i = 0; i < 32; ++i) pv[i] = __ldg(Pc + (int64_t)(i0 + i) * D);
#pragma unroll
            for (int g = 0; g < 8; ++g) {
                if (g < G) {
                    const float* qg = qin + g * D + h * 64 + i0;
#pragma unroll
                    for (int i = 0; i < 32; ++i) acc[g] = fmaf(qg[i], pv[i], acc[g]);
                }
            }
        }
        for (int g = 0; g < G; ++g) qpart[(h * G + g) * D + c] = acc[g];
    }
    __syncthreads();
    for (int x = tid; x < G * D; x += kFusedThreads) {
        const float v = qpart[x] + qpart[G * D + x];
        qrot[x] = v;
        const int c = x % D;
        if (c < C) qlo[(x / D) * C + c] = c < d ? v : 0.f;
    }
    // padding keys beyond S sort below every real key
    for (int x = tid; x < G * (Spad - S); x += kFusedThreads) {
        const int g = x / (Spad - S), j = S + x % (Spad - S);
        keys[g * Spad + j] = 0u;
    }
    __syncthreads();

    // ---- 1. score scan ----------------------------------------------------------
    // chunk c of a row is read at rotation (c + tid / 2) % NV: the 8 threads of
    // a quarter-warp then touch 8 distinct 16-byte bank groups
    const int rot = (tid >> 1) & (NV - 1);
    bool bad = false;
    int t = 0;
    for (; t < ntiles; ++t) {
        const int st = t % kFusedStages;
        const bool ok = mbar_wait(&full[st], (uint32_t)(t / kFusedStages) & 1u, err);
        const int row = t * kFusedRows + tid;
        if (ok && row < S) {
            const unsigned char* rp = ring + st * kTile + tid * kRowBytes;
            float a[8];
#pragma unroll
            for (int g = 0; g < 8; ++g) a[g] = 0.f;
#pragma unroll
            for (int cc = 0; cc < NV; ++cc) {
                const int ch = (cc + rot) & (NV - 1);
                float f[KV];
                E::unpack(*reinterpret_cast<const uint4*>(rp + ch * 16), f);
#pragma unroll
                for (int g = 0; g < 8; ++g) {
                    if (g < G) {
                        const float4* qg = reinterpret_cast<const float4*>(qlo + g * C + ch * KV);
#pragma unroll
                        for (int e4 = 0; e4 < KV / 4; ++e4) {
                            const float4 qq = qg[e4];
                            a[g] = fmaf(qq.x, f[4 * e4 + 0], a[g]);
                            a[g] = fmaf(qq.y, f[4 * e4 + 1], a[g]);
                            a[g] = fmaf(qq.z, f[4 * e4 + 2], a[g]);
                            a[g] = fmaf(qq.w, f[4 * e4 + 3], a[g]);
                        }
                    }
                }
            }
#pragma unroll
            for (int g = 0; g < 8; ++g)
                if (g < G) keys[g * Spad + row] = order_key(a[g]);
        }
        if (__syncthreads_or(!ok)) {
            bad = true;
            break;
        }
        // every thread is done with stage st: refill it
        if (tid == 0 && t + kFusedStages < ntiles) issue(t + kFusedStages);
    }
    if (bad) {
        // a copy never landed: wait (bounded) for every issued copy, then stop
        if (tid == 0)
            for (int j = t; j < ntiles && j < t + kFusedStages; ++j)
                mbar_wait(&full[j % kFusedStages], (uint32_t)(j / kFusedStages) & 1u, err);
        return;
    }

    // ---- 2. top-k per query head ---------------------------------------------------
    // (the ring is free once the scan is done: it holds the selection scratch;
    // each thread takes 8 groups of 4 keys of the head into registers)
    const TkSmem tsm = tk_carve(reinterpret_cast<uint32_t*>(ring));
    const TkCluster<false> one_cta;
    constexpr int kGroups = kFusedMaxS / (4 * kFusedThreads);
    static_assert(kGroups == 8, "fused top-k layout");
    for (int g = 0; g < G; ++g) {
        const uint4* kg = reinterpret_cast<const uint4*>(keys + g * Spad);
        tk_zero<kFusedThreads>(tsm);
        __syncthreads();
        uint4 v[kGroups];
#pragma unroll
        for (int i = 0; i < kGroups; ++i) {
            const int grp_i = warp * 32 * kGroups + 32 * i + lane;
            v[i] = grp_i < Spad / 4 ? kg[grp_i] : make_uint4(0u, 0u, 0u, 0u);
            const uint32_t kk[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
#pragma unroll
            for (int e = 0; e < 4; ++e)
                if (kk[e] != 0u) atomicAdd(&tsm.hist1[kk[e] >> 21], 1u);
        }
        tk_select<kFusedThreads, kGroups, false>(one_cta, v, 0, k, sel + g * k, tsm);
        __syncthreads();
    }
    {
        int32_t* so = sel_out + ((int64_t)b * H_q + (int64_t)hk * G) * k;
        for (int x = tid; x < G * k; x += kFusedThreads) so[x] = sel[x];
    }

    // ---- 3. sparse attention over the selected rows ----------------------------------
    const int wph = kFusedWarps / G;  // warps per head
    const int g = warp / wph, part = warp % wph;
    const int j0 = (int)((int64_t)part * k / wph), j1 = (int)((int64_t)(part + 1) * k / wph);
    const int grp = lane / LPR, sub = lane % LPR;
    float qv[KV];
#pragma unroll
    for (int e = 0; e < KV; ++e) qv[e] = qrot[g * D + sub * KV + e] * scale_log2;
    const char* Kb = reinterpret_cast<const char*>(Kt) +
                     ((int64_t)b * H_kv + hk) * S_max * kCacheRow + sub * 16;
    const char* Vb = reinterpret_cast<const char*>(V) +
                     ((int64_t)b * H_kv + hk) * S_max * kCacheRow + sub * 16;
    const int32_t* sg = sel + g * k;
    float m = -INFINITY, l = 0.f, acc[KV];
#pragma unroll
    for (int e = 0; e < KV; ++e) acc[e] = 0.f;
    for (int jb = j0; jb < j1; jb += GPW * U) {
        int tok[U];
        uint4 kv[U], vv[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int jj = jb + u * GPW + grp;
            tok[u] = jj < j1 ? sg[jj] : -1;
            if (tok[u] >= 0) {
                kv[u] = ld_stream(Kb + (int64_t)tok[u] * kCacheRow);
                vv[u] = ld_stream(Vb + (int64_t)tok[u] * kCacheRow);
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
            sc[u] = tok[u] >= 0 ? a : -INFINITY;
            mx = fmaxf(mx, sc[u]);
        }
        // (both row groups of the warp reach here: the shuffles above need
        // the whole warp; a group without tokens keeps its state)
        const bool none = mx == -INFINITY;
        const float alpha = none ? 1.f : exp2f(m - mx);
        l *= alpha;
#pragma unroll
        for (int e = 0; e < KV; ++e) acc[e] *= alpha;
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const float p = none ? 0.f : exp2f(sc[u] - mx);
            l += p;
            float f[KV];
            E::unpack(vv[u], f);
#pragma unroll
            for (int e = 0; e < KV; ++e) acc[e] = fmaf(p, f[e], acc[e]);
        }
        m = mx;
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
    // the warps' partials (m, l, acc[128]) meet in the ring area (free after top-k)
    float* parts = reinterpret_cast<float*>(ring);
    if (grp == 0) {
        float* pw = parts + warp * (2 + D);
#pragma unroll
        for (int e = 0; e < KV; ++e) pw[2 + sub * KV + e] = acc[e];
        if (sub == 0) {
            pw[0] = m;
            pw[1] = l;
        }
    }
    __syncthreads();
    for (int x = tid; x < G * D; x += kFusedThreads) {
        const int gg = x / D, c = x % D;
        const float* p0 = parts + gg * wph * (2 + D);
        float M = -INFINITY;
        for (int w = 0; w < wph; ++w) M = fmaxf(M, p0[w * (2 + D)]);
        float Ls = 0.f, A = 0.f;
        if (M != -INFINITY) {
            for (int w = 0; w < wph; ++w) {
                const float* pw = p0 + w * (2 + D);
                const float s = exp2f(pw[0] - M);
                Ls += pw[1] * s;
                A += pw[2 + c] * s;
            }
        }
        out[((int64_t)b * H_q + (int64_t)hk * G + gg) * D + c] = E::from_float(Ls > 0.f ? A / Ls : 0.f);
    }
}

// ---------------------------------------------------------------------------

static int fused_nv(Dt dt, int d_lo) { return d_lo * (dt == kF32 ? 4 : 2) / 16; }

bool decode_fused_fits(Dt dt, int H_q, int H_kv, int64_t S, int D, int d_lo, int64_t k) {
    if (D != 128 || H_kv < 1 || H_q % H_kv != 0) return false;
    const int G = H_q / H_kv;
    if (G != 1 && G != 2 && G != 4 && G != 8) return false;
    if (S < 1 || S > kFusedMaxS || k < 1 || k > S) return false;
    const int row_bytes = d_lo * (dt == kF32 ? 4 : 2);
    if (row_bytes % 16 != 0) return false;
    const int nv = row_bytes / 16;
    if (nv != 1 && nv != 2 && nv != 4 && nv != 8) return false;
    DevInfo di;
    if (dev_info(&di) != cudaSuccess) return false;
    const FusedLayout L = fused_layout(nv, nv * 16 / (dt == kF32 ? 4 : 2), G, (int)S, (int)k);
    return L.total + 1024 <= di.smem_optin;
}

#ifndef LOKI_FUSED_U
#define LOKI_FUSED_U 8
#endif
#ifndef LOKI_FUSED_MINB
#define LOKI_FUSED_MINB 2
#endif

template <class E, int NV>
static cudaError_t fused_impl(const void* q, const float* P, const void* Klo, const void* Kt,
                              const void* V, int B, int H_q, int H_kv, int64_t S, int64_t S_max,
                              int d, int64_t k, float scale, void* out, int32_t* sel, int* err,
                              cudaStream_t s, bool pdl) {
    auto kern = k_decode_fused<E, NV, LOKI_FUSED_U, LOKI_FUSED_MINB>;
    const int G = H_q / H_kv;
    const FusedLayout L = fused_layout(NV, NV * E::kVec, G, (int)S, (int)k);
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L.total);
    if (e != cudaSuccess) return e;
    using T = typename E::T;
    return launch_kernel(kern, dim3((unsigned)((int64_t)B * H_kv)), dim3(kFusedThreads),
                         (size_t)L.total, s, pdl, static_cast<const T*>(q), P,
                         static_cast<const T*>(Klo), static_cast<const T*>(Kt),
                         static_cast<const T*>(V), H_q, H_kv, G, (int)S, S_max, d, (int)k,
                         scale * kLog2e, static_cast<T*>(out), sel, err);
}

template <class E>
static cudaError_t fused_nv_dispatch(int nv, const void* q, const float* P, const void* Klo,
                                     const void* Kt, const void* V, int B, int H_q, int H_kv,
                                     int64_t S, int64_t S_max, int d, int64_t k, float scale,
                                     void* out, int32_t* sel, int* err, cudaStream_t s, bool pdl) {
    switch (nv) {
#define LOKI_NV(n)                                                                            \
    case n:                                                                                   \
        return fused_impl<E, n>(q, P, Klo, Kt, V, B, H_q, H_kv, S, S_max, d, k, scale, out, sel, \
                                err, s, pdl);
        LOKI_NV(1) LOKI_NV(2) LOKI_NV(4) LOKI_NV(8)
#undef LOKI_NV
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_decode_fused(Dt dt, const void* q, const float* P, const void* Klo,
                                const void* Kt, const void* V, int B, int H_q, int H_kv, int64_t S,
                                int64_t S_max, int d_lo, int d, int64_t k, float scale, void* out,
                                int32_t* sel, cudaStream_t s) {
    int* err = device_error_word();
    if (err == nullptr) return cudaErrorInvalidDevice;
    const int nv = fused_nv(dt, d_lo);
    if (dt == kF32)
        return fused_nv_dispatch<ElemF32>(nv, q, P, Klo, Kt, V, B, H_q, H_kv, S, S_max, d, k,
                                          scale, out, sel, err, s, false);
    return fused_nv_dispatch<ElemBF16>(nv, q, P, Klo, Kt, V, B, H_q, H_kv, S, S_max, d, k, scale,
                                       out, sel, err, s, false);
}

}  // namespace loki
