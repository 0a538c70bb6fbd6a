// Fused Loki decode step for few (batch, KV head) units: each unit is split
// over the CTAs of a thread-block cluster (2 to 8), so a decode with a
// handful of units still keeps the SMs busy in one kernel.
//
// Loki (briefgpt.xyz abstract page; NeurIPS 2024 poster page, TL;DR and
// "Visual Insights" Figure 1 caption): rotate the query by the unit's PCA
// basis, q~ = q P; score every cached token on the first d principal
// components, s_j = q~[:d] . K~_j[:d]; keep the k tokens with the largest
// scores; attend exactly over those k tokens with full-dimensional keys.
//
// CTA of rank r in the unit's cluster of CL CTAs (256 threads each):
//   0. streams plane rows [r chunk, (r + 1) chunk) of the unit into a ring of
//      shared-memory tiles (cp.async.bulk, one mbarrier per stage) while it
//      computes the first d_lo columns of the unit's G rotated queries
//      (P read from L2, fp32); the other columns, which only the gather needs,
//      are split over the cluster after the scan, each CTA storing its
//      128 / CL columns into every CTA;
//   1. scores its rows for the G query heads and stores them, as
//      order-preserving keys, straight into rank 0's shared memory
//      (distributed shared memory);
//   2. rank 0 runs the exact radix top-k of every head over all S keys
//      (topk_select.cuh, one CTA: a top-k split over the cluster was slower,
//      its histogram exchanges paying a distributed-memory latency each) and
//      writes the selection to selected_idx; every CTA copies its share of
//      the selection from rank 0;
//   3. gathers its share [r k / CL, (r + 1) k / CL) of each head's selected
//      key and value rows (16 rows in flight per warp, online softmax in
//      base 2) and merges its warps into one partial per head;
//   4. the partials of the cluster meet through distributed shared memory:
//      head g is merged and written by the CTA of rank g % CL.
#include "common.cuh"
#include "launch.h"
#include "tma.cuh"
#include "topk_select.cuh"

namespace loki {

constexpr int kCdThreads = 256;
constexpr int kCdWarps = kCdThreads / 32;
constexpr int kCdRows = kCdThreads;  // plane rows per scan tile (one per thread)
constexpr int kCdStages = 3;
constexpr int kCdMaxI = 8;           // groups of 4 keys per thread in the top-k

__host__ __device__ constexpr int cd_align16(int x) { return (x + 15) & ~15; }

// Byte offsets of the dynamic shared-memory regions of one CTA.
struct ClusterLayout {
    int ring;   // scan tiles; then top-k scratch (rank 0); then the warps' partials
    int keys;   // G x Spad order keys of all S rows (used in rank 0)
    int sel;    // G x k selected indices (rank 0: all; others: their share)
    int qin;    // G x 128 fp32 raw queries
    int qpart;  // 256 G fp32 partial sums of the rotation
    int qrot;   // G x 128 fp32 rotated queries (the gather's)
    int qlo;    // G x C fp32 rotated queries, zero beyond column d (the scan's)
    int cpart;  // G x (2 + 128) fp32: this CTA's partial (m, l, acc) per head
    int total;
};

__host__ __device__ inline ClusterLayout cluster_layout(int nv, int cols, int G, int Spad, int k) {
    const int tile = kCdRows * nv * 16;
    int ring = kCdStages * tile;
    const int topk_scratch = kTkSmemWords * 4;
    const int partials = kCdWarps * (2 + 128) * 4;
    if (ring < topk_scratch) ring = topk_scratch;
    if (ring < partials) ring = partials;
    ClusterLayout L;
    L.ring = 0;
    L.keys = cd_align16(ring);
    L.sel = L.keys + cd_align16(G * Spad * 4);
    L.qin = L.sel + cd_align16(G * k * 4);
    L.qpart = L.qin + G * 128 * 4;
    L.qrot = L.qpart + 2 * G * 128 * 4;
    L.qlo = L.qrot + G * 128 * 4;
    L.cpart = L.qlo + cd_align16(G * cols * 4);
    L.total = L.cpart + G * (2 + 128) * 4;
    return L;
}

// E: element traits; NV: 16-byte chunks per plane row; I: groups of 4 keys
// per thread in rank 0's top-k (Spad <= 4 * 256 * I); U: rows in flight per
// row group in the gather. chunk: rows per CTA (a multiple of 4); Spad: S
// rounded up to 4.
template <class E, int NV, int I, int U>
__global__ void __launch_bounds__(kCdThreads, 2) k_decode_cluster(
    const typename E::T* __restrict__ q, const float* __restrict__ P,
    const typename E::T* __restrict__ Klo, const typename E::T* __restrict__ Kt,
    const typename E::T* __restrict__ V, int H_q, int H_kv, int G, int S, int64_t S_max, int d,
    int k, int chunk, float scale_log2, typename E::T* __restrict__ out,
    int32_t* __restrict__ sel_out, int* __restrict__ err) {
    using T = typename E::T;
    constexpr int D = 128;
    constexpr int KV = E::kVec;
    constexpr int C = NV * KV;          // plane row width in elements
    constexpr int kRowBytes = NV * 16;  // plane row bytes
    constexpr int kTile = kCdRows * kRowBytes;
    constexpr int LPR = D / KV;         // gather lanes per cache row
    constexpr int GPW = 32 / LPR;       // gather row groups per warp
    constexpr int64_t kCacheRow = (int64_t)D * E::kBytes;
    extern __shared__ __align__(128) unsigned char smem[];
    __shared__ uint64_t full[kCdStages];

    TkCluster<true> cl;
    cl.init();
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int rank = cl.rank, ncl = cl.size;
    const int64_t unit = blockIdx.x / ncl;
    const int b = (int)(unit / H_kv), hk = (int)(unit % H_kv);
    const int base = rank * chunk;                // this CTA's first row
    const int n = max(0, min(chunk, S - base));  // and its row count
    const int Spad = (S + 3) & ~3;
    const ClusterLayout L = cluster_layout(NV, C, G, Spad, k);
    unsigned char* ring = smem + L.ring;
    uint32_t* keys = reinterpret_cast<uint32_t*>(smem + L.keys);
    int32_t* sel = reinterpret_cast<int32_t*>(smem + L.sel);
    float* qin = reinterpret_cast<float*>(smem + L.qin);
    float* qpart = reinterpret_cast<float*>(smem + L.qpart);
    float* qrot = reinterpret_cast<float*>(smem + L.qrot);
    float* qlo = reinterpret_cast<float*>(smem + L.qlo);
    float* cpart = reinterpret_cast<float*>(smem + L.cpart);
    const int ntiles = (n + kCdRows - 1) / kCdRows;
    const char* plane =
        reinterpret_cast<const char*>(Klo) + (unit * S_max + base) * (int64_t)kRowBytes;

    if (tid == 0) {
        for (int s = 0; s < kCdStages; ++s) mbar_init(&full[s], 1);
        fence_mbar_init();
    }
    __syncthreads();
    griddep_wait();  // inputs may come from the preceding kernel (an append)
    fence_proxy_async_global();  // whose stores precede our bulk reads

    // ---- 0. start the key stream; rotate the queries meanwhile ------------------
    const uint64_t pol = l2_policy_evict_first();
    auto issue = [&](int t) {
        const int st = t % kCdStages;
        const int nr = min(kCdRows, n - t * kCdRows);
        mbar_arrive_expect_tx(&full[st], (uint32_t)(nr * kRowBytes));
        bulk_load_hint(ring + st * kTile, plane + (int64_t)t * kCdRows * kRowBytes,
                       (uint32_t)(nr * kRowBytes), &full[st], pol);
    };
    if (tid == 0)
        for (int t = 0; t < kCdStages && t < ntiles; ++t) issue(t);
    {
        const T* qb = q + ((int64_t)b * H_q + (int64_t)hk * G) * D;  // the unit's G rows
        for (int x = tid; x < G * D; x += kCdThreads) qin[x] = E::load1(qb + x);
    }
    // every CTA of the cluster is running before any writes another's memory
    cl.sync();
    {
        // the scan's q~[:C]: this CTA computes it alone (thread: one of the C
        // columns, 128 / (256 / C) rows of P); the halves of the row range meet
        // in shared memory
        const int nblk = kCdThreads / C, rows = D / nblk;
        const int c = tid % C, h = tid / C;
        const float* Pc = P + ((int64_t)hk * D + h * rows) * D + c;
        float pv[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) pv[i] = i < rows ? __ldg(Pc + (int64_t)i * D) : 0.f;
        for (int g = 0; g < G; ++g) {
            const float* qg = qin + g * D + h * rows;
            float a = 0.f;
#pragma unroll
            for (int i = 0; i < 32; ++i)
                if (i < rows) a = fmaf(qg[i], pv[i], a);
            qpart[(h * G + g) * C + c] = a;  // [block][head][column]
        }
        __syncthreads();
        for (int x = tid; x < G * C; x += kCdThreads) {
            const int g = x / C, cc = x % C;
            float v = 0.f;
            for (int hh = 0; hh < nblk; ++hh) v += qpart[(hh * G + g) * C + cc];
            qlo[x] = cc < d ? v : 0.f;
        }
    }
    if (rank == 0)  // padding keys beyond S sort below every real key
        for (int x = tid; x < G * (Spad - S); x += kCdThreads)
            keys[(x / (Spad - S)) * Spad + S + x % (Spad - S)] = 0u;
    __syncthreads();

    // ---- 1. score scan; the keys go to rank 0 --------------------------------------
    // chunk c of a row is read at rotation (c + tid / 2) % NV: the 8 threads of
    // a quarter-warp then touch 8 distinct 16-byte bank groups
    uint32_t* keys0 = cl.at(keys, 0);
    const int rot = (tid >> 1) & (NV - 1);
    bool bad = false;
    int t = 0;
    for (; t < ntiles; ++t) {
        const int st = t % kCdStages;
        const bool ok = mbar_wait(&full[st], (uint32_t)(t / kCdStages) & 1u, err);
        const int row = t * kCdRows + tid;
        if (ok && row < n) {
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
                if (g < G) keys0[g * Spad + base + row] = order_key(a[g]);
        }
        if (__syncthreads_or(!ok)) {
            bad = true;
            break;
        }
        // every thread is done with stage st: refill it
        if (tid == 0 && t + kCdStages < ntiles) issue(t + kCdStages);
    }
    if (bad && tid == 0)
        // a copy never landed: wait (bounded) for every issued copy; the keys
        // are incomplete, but the cluster still runs every step below together
        // (its barriers need every CTA), and the error word reports it
        for (int j = t; j < ntiles && j < t + kCdStages; ++j)
            mbar_wait(&full[j % kCdStages], (uint32_t)(j / kCdStages) & 1u, err);
    {
        // the gather's full q~, split over the cluster: CTA r computes columns
        // [r 128 / CL, (r + 1) 128 / CL) for every head (thread: one column,
        // 64 / CL <= 32 rows of P) and stores them into every CTA's q~
        const int ncol = D / ncl, nblk = kCdThreads / ncol, rows = D / nblk;
        const int c = rank * ncol + tid % ncol, h = tid / ncol;
        const float* Pc = P + ((int64_t)hk * D + h * rows) * D + c;
        float pv[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) pv[i] = i < rows ? __ldg(Pc + (int64_t)i * D) : 0.f;
        for (int g = 0; g < G; ++g) {
            const float* qg = qin + g * D + h * rows;
            float a = 0.f;
#pragma unroll
            for (int i = 0; i < 32; ++i)
                if (i < rows) a = fmaf(qg[i], pv[i], a);
            qpart[(h * G + g) * ncol + tid % ncol] = a;  // [block][head][column]
        }
        __syncthreads();
        for (int x = tid; x < G * ncol; x += kCdThreads) {
            const int g = x / ncol, cc = x % ncol;
            float v = 0.f;
            for (int hh = 0; hh < nblk; ++hh) v += qpart[(hh * G + g) * ncol + cc];
            for (int rr = 0; rr < ncl; ++rr) cl.at(qrot, rr)[g * D + rank * ncol + cc] = v;
        }
    }
    cl.sync();  // every key is in rank 0, and every CTA holds all of q~

    // ---- 2. top-k per query head in rank 0; each CTA takes its share ---------------
    if (rank == 0) {
        // (the ring is free once the scan is done: it holds the selection scratch)
        const TkSmem tsm = tk_carve(reinterpret_cast<uint32_t*>(ring));
        const TkCluster<false> one_cta;
        for (int g = 0; g < G; ++g) {
            const uint4* kg = reinterpret_cast<const uint4*>(keys + g * Spad);
            tk_zero<kCdThreads>(tsm);
            __syncthreads();
            uint4 v[I];
#pragma unroll
            for (int i = 0; i < I; ++i) {
                const int gi = warp * 32 * I + 32 * i + lane;  // keys 4 gi .. 4 gi + 3
                v[i] = 4 * gi < Spad ? kg[gi] : make_uint4(0u, 0u, 0u, 0u);
                const uint32_t kk[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    if (kk[e] != 0u) atomicAdd(&tsm.hist1[kk[e] >> 21], 1u);
            }
            tk_select<kCdThreads, I, false>(one_cta, v, 0, k, sel + g * k, tsm);
            __syncthreads();
        }
        int32_t* so = sel_out + ((int64_t)b * H_q + (int64_t)hk * G) * k;
        for (int x = tid; x < G * k; x += kCdThreads) so[x] = sel[x];
    }
    cl.sync();  // the selection is in rank 0
    const int s0 = (int)((int64_t)rank * k / ncl), s1 = (int)((int64_t)(rank + 1) * k / ncl);
    if (rank != 0) {
        const int32_t* sel0 = cl.at(sel, 0);
        for (int x = tid; x < G * (s1 - s0); x += kCdThreads) {
            const int g = x / (s1 - s0), j = s0 + x % (s1 - s0);
            sel[g * k + j] = sel0[g * k + j];
        }
    }
    __syncthreads();

    // ---- 3. sparse attention over this CTA's share of each head's selection ------
    const int wph = kCdWarps / G;  // warps per head
    const int g = warp / wph, part = warp % wph;
    const int j0 = s0 + (int)((int64_t)part * (s1 - s0) / wph);
    const int j1 = s0 + (int)((int64_t)(part + 1) * (s1 - s0) / wph);
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
            if ((unsigned)tok[u] >= (unsigned)S) tok[u] = -1;
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
    // this CTA's partial per head: the head's warps merged
    for (int x = tid; x < G * D; x += kCdThreads) {
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
        float* cp = cpart + gg * (2 + D);
        cp[2 + c] = A;
        if (c == 0) {
            cp[0] = M;
            cp[1] = Ls;
        }
    }

    // ---- 4. the cluster's partials: head g merged by the CTA of rank g % CL ------
    // (all ranks' values of a column are loaded together: one round trip)
    cl.sync();
    for (int x = tid; x < G * D; x += kCdThreads) {
        const int gg = x / D, c = x % D;
        if (gg % ncl != rank) continue;
        float mr[kTkMaxCluster], lr[kTkMaxCluster], ar[kTkMaxCluster];
#pragma unroll
        for (int rr = 0; rr < kTkMaxCluster; ++rr) {
            if (rr < ncl) {
                const float* cp = cl.at(cpart, rr) + gg * (2 + D);
                mr[rr] = cp[0];
                lr[rr] = cp[1];
                ar[rr] = cp[2 + c];
            } else {
                mr[rr] = -INFINITY;
                lr[rr] = 0.f;
                ar[rr] = 0.f;
            }
        }
        float M = -INFINITY;
#pragma unroll
        for (int rr = 0; rr < kTkMaxCluster; ++rr) M = fmaxf(M, mr[rr]);
        float Ls = 0.f, A = 0.f;
        if (M != -INFINITY) {
#pragma unroll
            for (int rr = 0; rr < kTkMaxCluster; ++rr) {
                const float s = mr[rr] == -INFINITY ? 0.f : exp2f(mr[rr] - M);
                Ls += lr[rr] * s;
                A += ar[rr] * s;
            }
        }
        out[((int64_t)b * H_q + (int64_t)hk * G + gg) * D + c] =
            E::from_float(Ls > 0.f ? A / Ls : 0.f);
    }
    cl.sync();  // no CTA leaves while another still reads its partials
}

// ---------------------------------------------------------------------------

// The cluster size for a decode of `units` (batch, KV head) units: the most
// CTAs per unit (a power of two up to 8) that keep the grid within two per SM;
// 0 when fewer than two would be used (many units: the split pipeline wins).
static int cluster_size_for(int64_t units, int sm_count) {
    int cl = 8;
    while (cl >= 2 && units * cl > 2 * (int64_t)sm_count) cl /= 2;
    return cl >= 2 ? cl : 0;
}

struct ClusterShape {
    int cl, chunk, gi;
    bool pdl = false;  // launched as a programmatic dependent (behind an append)
};

static bool cluster_shape(Dt dt, int B, int H_q, int H_kv, int64_t S, int D, int d_lo, int64_t k,
                          ClusterShape* sh) {
    if (D != 128 || H_kv < 1 || H_q % H_kv != 0) return false;
    const int G = H_q / H_kv;
    if (G != 1 && G != 2 && G != 4 && G != 8) return false;
    if (S < 1 || k < 1 || k > S) return false;
    const int row_bytes = d_lo * (dt == kF32 ? 4 : 2);
    if (row_bytes % 16 != 0) return false;
    const int nv = row_bytes / 16;
    if (nv != 1 && nv != 2 && nv != 4 && nv != 8) return false;
    DevInfo di;
    if (dev_info(&di) != cudaSuccess) return false;
    const int cl = cluster_size_for((int64_t)B * H_kv, di.sm_count);
    if (cl == 0) return false;
    // rank 0 selects over all S keys of a head in one CTA
    const int64_t Spad = (S + 3) / 4 * 4;
    int gi = 1;
    while (gi < kCdMaxI && 4 * kCdThreads * gi < Spad) gi *= 2;
    if (4 * kCdThreads * gi < Spad) return false;
    const int64_t chunk = ((S + cl - 1) / cl + 3) / 4 * 4;
    const ClusterLayout L =
        cluster_layout(nv, nv * 16 / (dt == kF32 ? 4 : 2), G, (int)Spad, (int)k);
    if (L.total + 1024 > di.smem_optin) return false;
    sh->cl = cl;
    sh->chunk = (int)chunk;
    sh->gi = gi;
    return true;
}

bool decode_cluster_fits(Dt dt, int B, int H_q, int H_kv, int64_t S, int D, int d_lo, int64_t k) {
    ClusterShape sh;
    return cluster_shape(dt, B, H_q, H_kv, S, D, d_lo, k, &sh);
}

bool decode_cluster_preferred(Dt dt, int B, int H_q, int H_kv, int64_t S, int D, int d_lo,
                              int64_t k) {
    return (int64_t)B * H_kv >= 16 && decode_cluster_fits(dt, B, H_q, H_kv, S, D, d_lo, k);
}

template <class E, int NV, int I>
static cudaError_t cluster_impl(const ClusterShape& sh, const void* q, const float* P,
                                const void* Klo, const void* Kt, const void* V, int B, int H_q,
                                int H_kv, int64_t S, int64_t S_max, int d, int64_t k, float scale,
                                void* out, int32_t* sel, int* err, cudaStream_t s) {
    auto kern = k_decode_cluster<E, NV, I, 4>;
    const int G = H_q / H_kv;
    const ClusterLayout L = cluster_layout(NV, NV * E::kVec, G, (int)((S + 3) / 4 * 4), (int)k);
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L.total);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)((int64_t)B * H_kv * sh.cl));
    cfg.blockDim = dim3(kCdThreads);
    cfg.dynamicSmemBytes = (size_t)L.total;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)sh.cl;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = sh.pdl ? 2 : 1;
    using T = typename E::T;
    return cudaLaunchKernelEx(&cfg, kern, static_cast<const T*>(q), P, static_cast<const T*>(Klo),
                              static_cast<const T*>(Kt), static_cast<const T*>(V), H_q, H_kv, G,
                              (int)S, S_max, d, (int)k, sh.chunk, scale * kLog2e,
                              static_cast<T*>(out), sel, err);
}

template <class E, int NV>
static cudaError_t cluster_gi(const ClusterShape& sh, const void* q, const float* P,
                              const void* Klo, const void* Kt, const void* V, int B, int H_q,
                              int H_kv, int64_t S, int64_t S_max, int d, int64_t k, float scale,
                              void* out, int32_t* sel, int* err, cudaStream_t s) {
    switch (sh.gi) {
#define LOKI_GI(i)                                                                            \
    case i:                                                                                   \
        return cluster_impl<E, NV, i>(sh, q, P, Klo, Kt, V, B, H_q, H_kv, S, S_max, d, k, scale, \
                                      out, sel, err, s);
        LOKI_GI(1) LOKI_GI(2) LOKI_GI(4) LOKI_GI(8)
#undef LOKI_GI
        default: return cudaErrorInvalidValue;
    }
}

template <class E>
static cudaError_t cluster_nv(int nv, const ClusterShape& sh, const void* q, const float* P,
                              const void* Klo, const void* Kt, const void* V, int B, int H_q,
                              int H_kv, int64_t S, int64_t S_max, int d, int64_t k, float scale,
                              void* out, int32_t* sel, int* err, cudaStream_t s) {
    switch (nv) {
#define LOKI_NV(n)                                                                               \
    case n:                                                                                      \
        return cluster_gi<E, n>(sh, q, P, Klo, Kt, V, B, H_q, H_kv, S, S_max, d, k, scale, out, \
                                sel, err, s);
        LOKI_NV(1) LOKI_NV(2) LOKI_NV(4) LOKI_NV(8)
#undef LOKI_NV
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_decode_cluster(Dt dt, const void* q, const float* P, const void* Klo,
                                  const void* Kt, const void* V, int B, int H_q, int H_kv,
                                  int64_t S, int64_t S_max, int d_lo, int d, int64_t k,
                                  float scale, void* out, int32_t* sel, cudaStream_t s, bool pdl) {
    int* err = device_error_word();
    if (err == nullptr) return cudaErrorInvalidDevice;
    ClusterShape sh;
    if (!cluster_shape(dt, B, H_q, H_kv, S, 128, d_lo, k, &sh)) return cudaErrorInvalidValue;
    sh.pdl = pdl;
    const int nv = d_lo * (dt == kF32 ? 4 : 2) / 16;
    if (dt == kF32)
        return cluster_nv<ElemF32>(nv, sh, q, P, Klo, Kt, V, B, H_q, H_kv, S, S_max, d, k, scale,
                                   out, sel, err, s);
    return cluster_nv<ElemBF16>(nv, sh, q, P, Klo, Kt, V, B, H_q, H_kv, S, S_max, d, k, scale,
                                out, sel, err, s);
}

}  // namespace loki
