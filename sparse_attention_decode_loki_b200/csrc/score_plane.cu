// Low-dimensional score scan over a low-dim key plane, staged through shared
// memory by TMA bulk copies.
//
// Loki (NeurIPS 2024 poster page, TL;DR and "Visual Insights" Figure 1
// caption; briefgpt.xyz abstract page): every cached token is scored on the
// first d principal components, s_j = q~[:d] . K~_j[:d], with q~ = q P.
//
// A (batch, KV head) unit's plane rows are contiguous (d_lo elements each),
// so the scan is a pure stream. The rows of all units are laid end to end and
// split evenly over one wave of CTAs. In each CTA one producer warp issues
// cp.async.bulk copies of 256-row tiles into a 96 KB ring of shared-memory
// stages (full/empty mbarriers); each of 256 consumer threads scores one row
// of every tile for all G query heads of the unit (whole row per thread: no
// shuffles, coalesced score stores), reading the row's 16-byte chunks in a
// rotated order so a quarter-warp touches distinct banks. The ring keeps up
// to ~90 KB per SM in flight without holding it in registers. In the decode
// call the scan comes first and rotates the queries itself (the full query
// projection runs beside it); as a step of its own it reads q~ and may be
// launched right behind the projection (programmatic dependent launch): the
// producer then starts streaming keys at once, and only the consumers wait.
// In a decode step that appends its new keys first (rows [wait_row, S) of
// every unit, written by the preceding kernel), each CTA streams its older
// rows first and only then, after waiting for the append, gathers the new
// rows of all its segments into tiles of their own, so the append's time
// hides behind the stream.
#include "common.cuh"
#include "launch.h"
#include "tma.cuh"

namespace loki {

constexpr int kScoreConsumerWarps = 8;
constexpr int kScoreConsumers = kScoreConsumerWarps * 32;
constexpr int kScoreThreads = kScoreConsumers + 32;
// one CTA per SM (9 warps at ~104 registers leave no room for a second);
// a 192 KB ring measured no faster than this one
#ifndef LOKI_SCORE_RING_KB
#define LOKI_SCORE_RING_KB 96
#endif
constexpr int kScoreRingBytes = LOKI_SCORE_RING_KB * 1024;
constexpr int kScoreMaxStages = 16;

// NV = 16-byte chunks per plane row (d_lo * elem / 16). A tile is 256 rows,
// one per consumer thread; stages = ring bytes / tile bytes.
//
// kFuseQ: the consumers rotate the query themselves, q~[:d] = q P[:, :d], per
// (batch, KV head) unit, from q and P (head dim 128), so the scan needs no
// projection kernel before it: thread (part p, column c) keeps the 128 /
// parts rows of column c of P that it needs in registers, prefetched one unit
// ahead, and the per-part partial sums meet in shared memory. Without it the
// consumers read q~ from q_rot after the preceding kernel completes.
// kDefer: the kernel of a step that appends (wait_row < S), with the new rows
// scanned last; without it rows at or past wait_row are not expected.
template <class E, int G, int NV, bool kFuseQ, bool kDefer>
__device__ __forceinline__ void score_plane_body(
    const float* __restrict__ q_rot, const typename E::T* __restrict__ q,
    const float* __restrict__ P, const typename E::T* __restrict__ Klo,
    float* __restrict__ scores, int* __restrict__ err, int H_q, int H_kv, int S, int64_t S_max,
    int D, int d, int64_t total, int64_t per, int wait_row) {
    constexpr int KV = E::kVec;
    constexpr int kRowBytes = NV * 16;
    constexpr int kTR = kScoreConsumers;  // rows per tile
    constexpr int kTile = kTR * kRowBytes;
    constexpr int kStages = (kScoreRingBytes / kTile) < kScoreMaxStages ? (kScoreRingBytes / kTile)
                                                                      : kScoreMaxStages;
    static_assert(kStages >= 2, "ring too small");
    constexpr int C = NV * KV;                     // plane row width in elements
    constexpr int kParts = kScoreConsumers / C;    // row blocks of P
    constexpr int kR = 128 / kParts;               // rows of P per thread
    constexpr int QN = (G * 128 + kScoreConsumers - 1) / kScoreConsumers;
    extern __shared__ __align__(128) unsigned char ring[];
    __shared__ uint64_t full[kStages], empty[kStages];
    __shared__ float s_q[kFuseQ ? G * 128 : 1];
    __shared__ float s_part[kFuseQ ? kParts * G * C : 1];
    __shared__ float s_qlo[kFuseQ ? G * C : 1];

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (tid == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kScoreConsumerWarps);
        }
        fence_mbar_init();
    }
    __syncthreads();
    griddep_launch_dependents();

    const int64_t R0 = (int64_t)blockIdx.x * per;
    const int64_t R1 = min64(R0 + per, total);

    if (warp == kScoreConsumerWarps) {
        // ---------------- producer: one lane issues every tile copy ----------------
        if (lane == 0) {
            // the plane is read once per step: keep it from evicting the
            // scores, which top-k reads right after this kernel
            const uint64_t pol = l2_policy_evict_first();
            int i = 0;
            bool ok = true;
            // rows [wait_row, S) of every unit are written by the preceding
            // kernel (an append): the older rows of every segment stream
            // first (phase A), then, after the wait, the new rows of all the
            // CTA's segments are gathered into tiles of their own (phase B)
            const bool defer = kDefer && wait_row < S;
            for (int64_t r = R0; r < R1 && ok;) {
                const int64_t unit = r / S;
                const int s0 = (int)(r - unit * S);
                const int seg = (int)min64(R1 - r, (int64_t)S - s0);
                const int segA = defer ? max(0, min(seg, wait_row - s0)) : seg;
                const char* src = reinterpret_cast<const char*>(Klo) + (unit * S_max + s0) * kRowBytes;
                for (int t0 = 0; t0 < segA; t0 += kTR, ++i) {
                    const int n = min(kTR, segA - t0);
                    const int st = i % kStages;
                    const uint32_t ph = (uint32_t)(i / kStages) & 1u;
                    if (!mbar_wait(&empty[st], ph ^ 1u, err)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(&full[st], (uint32_t)(n * kRowBytes));
                    bulk_load_hint(ring + (size_t)st * kTile, src + (int64_t)t0 * kRowBytes,
                                   (uint32_t)(n * kRowBytes), &full[st], pol);
                }
                r += seg;
            }
            // the preceding kernel is complete (and, in phase B, its rows are
            // visible to our bulk reads) before any new row is read; a CTA
            // without new rows waits too, so the kernels after the scan also
            // see the preceding kernel's writes
            griddep_wait();
            if (defer && ok) {
                fence_proxy_async_global();  // its stores, then our bulk reads
                int fill = 0, st = 0;
                for (int64_t r = R0; r < R1 && ok;) {
                    const int64_t unit = r / S;
                    const int s0 = (int)(r - unit * S);
                    const int seg = (int)min64(R1 - r, (int64_t)S - s0);
                    for (int x = max(s0, wait_row); x < s0 + seg && ok;) {
                        if (fill == 0) {
                            st = i % kStages;
                            if (!mbar_wait(&empty[st], ((uint32_t)(i / kStages) & 1u) ^ 1u, err)) {
                                ok = false;
                                break;
                            }
                        }
                        const int n = min(s0 + seg - x, kTR - fill);
                        mbar_expect_tx(&full[st], (uint32_t)(n * kRowBytes));
                        bulk_load_hint(ring + (size_t)st * kTile + (size_t)fill * kRowBytes,
                                       reinterpret_cast<const char*>(Klo) +
                                           (unit * S_max + x) * kRowBytes,
                                       (uint32_t)(n * kRowBytes), &full[st], pol);
                        fill += n;
                        x += n;
                        if (fill == kTR) {
                            mbar_arrive(&full[st]);  // the tile's one arrival
                            fill = 0;
                            ++i;
                        }
                    }
                    r += seg;
                }
                if (ok && fill > 0) {
                    mbar_arrive(&full[st]);
                    ++i;
                }
            }
            // every issued copy has landed before the CTA may exit
            for (int j = max(0, i - kStages); j < i; ++j)
                mbar_wait(&full[j % kStages], (uint32_t)(j / kStages) & 1u, err);
        }
        return;
    }

    // ---------------- consumers: one row of each tile per thread ----------------
    // Unfused, q~ comes from the projection kernel, which may still be
    // running: the producer above streams keys without waiting, the consumers
    // wait here.
    if constexpr (!kFuseQ) griddep_wait();
    // chunk c of a row is read at rotation (c + tid / 2) % NV: the 8 threads
    // of a quarter-warp then hit 8 distinct 16-byte bank groups
    const int rot = (tid >> 1) & (NV - 1);
    const int pc = tid % C, pp = tid / C;  // fused rotation: column and row block of P
    float pf[kFuseQ ? kR : 1], qf[kFuseQ ? QN : 1];
    // loads P[hk][pp*kR + j][pc] (zero beyond column d) and the unit's G query rows
#define LOKI_FETCH_UNIT(unit_)                                                              \
    {                                                                                      \
        const int fb = (int)((unit_) / H_kv), fh = (int)((unit_) % H_kv);                  \
        const float* Pp = P + ((int64_t)fh * 128 + pp * kR) * 128 + pc;                    \
        _Pragma("unroll") for (int j = 0; j < kR; ++j) pf[j] =                            \
            pc < d ? __ldg(Pp + j * 128) : 0.f;                                            \
        const typename E::T* qb = q + ((int64_t)fb * H_q + (int64_t)fh * G) * 128;         \
        _Pragma("unroll") for (int e = 0; e < QN; ++e) {                                   \
            const int qi = tid + e * kScoreConsumers;                                      \
            qf[e] = qi < G * 128 ? E::load1(qb + qi) : 0.f;                                \
        }                                                                                  \
    }
    if constexpr (kFuseQ)
        if (R0 < R1) LOKI_FETCH_UNIT(R0 / S)
    bool bad = false;
    int i = 0;
    const bool defer = kDefer && wait_row < S;  // phase A: each segment's rows below wait_row
    for (int64_t r = R0; r < R1;) {
        const int64_t unit = r / S;
        const int s0 = (int)(r - unit * S);
        const int seg = (int)min64(R1 - r, (int64_t)S - s0);
        const int segA = defer ? max(0, min(seg, wait_row - s0)) : seg;
        const int b = (int)(unit / H_kv), hk = (int)(unit % H_kv);
        const int64_t qrow0 = (int64_t)b * H_q + (int64_t)hk * G;
        // qv holds q~ in this thread's rotated chunk order: slot cc holds
        // chunk (cc + rot) % NV, so the row loop indexes registers statically
        float qv[G][NV * KV];
        if constexpr (kFuseQ) {
            named_sync(1, kScoreConsumers);  // the previous unit's readers are done
#pragma unroll
            for (int e = 0; e < QN; ++e) {
                const int qi = tid + e * kScoreConsumers;
                if (qi < G * 128) s_q[qi] = qf[e];
            }
            named_sync(1, kScoreConsumers);
#pragma unroll
            for (int g = 0; g < G; ++g) {
                float a = 0.f;
#pragma unroll
                for (int j = 0; j < kR; ++j) a = fmaf(s_q[g * 128 + pp * kR + j], pf[j], a);
                s_part[(pp * G + g) * C + pc] = a;
            }
            named_sync(1, kScoreConsumers);
            for (int x = tid; x < G * C; x += kScoreConsumers) {
                float a = 0.f;
#pragma unroll 4
                for (int p2 = 0; p2 < kParts; ++p2) a += s_part[p2 * G * C + x];
                s_qlo[x] = a;
            }
            named_sync(1, kScoreConsumers);
#pragma unroll
            for (int g = 0; g < G; ++g)
#pragma unroll
                for (int cc = 0; cc < NV; ++cc)
#pragma unroll
                    for (int e = 0; e < KV; ++e)
                        qv[g][cc * KV + e] = s_qlo[g * C + ((cc + rot) & (NV - 1)) * KV + e];
            // the next unit's P block and queries load behind this unit's tiles
            if ((unit + 1) * S < R1) LOKI_FETCH_UNIT(unit + 1)
        } else {
#pragma unroll
            for (int g = 0; g < G; ++g)
#pragma unroll
                for (int cc = 0; cc < NV; ++cc)
#pragma unroll
                    for (int e = 0; e < KV; ++e) {
                        const int col = ((cc + rot) & (NV - 1)) * KV + e;
                        qv[g][cc * KV + e] = col < d ? __ldg(q_rot + (qrow0 + g) * D + col) : 0.f;
                    }
        }
#undef LOKI_FETCH_UNIT

        float* srow = scores + qrow0 * S + s0;
        for (int t0 = 0; t0 < segA; t0 += kTR, ++i) {
            const int n = min(kTR, segA - t0);
            const int st = i % kStages;
            const uint32_t ph = (uint32_t)(i / kStages) & 1u;
            // after a timed-out wait this warp stops consuming and stops
            // releasing stages, so the producer stops issuing and drains
            if (!bad && !mbar_wait(&full[st], ph, err)) bad = true;
            if (!bad && tid < n) {
                const unsigned char* rowp = ring + (size_t)st * kTile + tid * kRowBytes;
                float a[G];
#pragma unroll
                for (int g = 0; g < G; ++g) a[g] = 0.f;
#pragma unroll
                for (int cc = 0; cc < NV; ++cc) {
                    const int c = (cc + rot) & (NV - 1);
                    const uint4 v = *reinterpret_cast<const uint4*>(rowp + c * 16);
                    float f[KV];
                    E::unpack(v, f);
#pragma unroll
                    for (int g = 0; g < G; ++g)
#pragma unroll
                        for (int e = 0; e < KV; ++e) a[g] = fmaf(qv[g][cc * KV + e], f[e], a[g]);
                }
#pragma unroll
                for (int g = 0; g < G; ++g) srow[(int64_t)g * S + t0 + tid] = a[g];
            }
            __syncwarp();
            if (lane == 0 && !bad) mbar_arrive(&empty[st]);
        }
        r += seg;
    }
    if (!kDefer || !defer) return;

    // phase B: the new rows of all the CTA's segments, packed in scan order
    // into tiles of kTR rows; new row g of the CTA lands in slot g % kTR of
    // its tile. Their q~ comes from q_rot, which the preceding kernel wrote.
    griddep_wait();
    int64_t nb_all = 0;
    for (int64_t r = R0; r < R1;) {
        const int64_t unit = r / S;
        const int s0 = (int)(r - unit * S);
        const int seg = (int)min64(R1 - r, (int64_t)S - s0);
        nb_all += max(0, s0 + seg - max(s0, wait_row));
        r += seg;
    }
    for (int64_t g0 = 0; g0 < nb_all; g0 += kTR, ++i) {
        const int n = (int)min64(kTR, nb_all - g0);
        const int st = i % kStages;
        const uint32_t ph = (uint32_t)(i / kStages) & 1u;
        if (!bad && !mbar_wait(&full[st], ph, err)) bad = true;
        if (!bad && tid < n) {
            // this thread's new row: walk the CTA's segments to it
            int64_t gi = g0 + tid, unit = 0;
            int x = 0;
            for (int64_t r = R0; r < R1;) {
                unit = r / S;
                const int s0 = (int)(r - unit * S);
                const int seg = (int)min64(R1 - r, (int64_t)S - s0);
                const int a0 = max(s0, wait_row), nb = max(0, s0 + seg - a0);
                if (gi < nb) {
                    x = a0 + (int)gi;
                    break;
                }
                gi -= nb;
                r += seg;
            }
            const int b = (int)(unit / H_kv), hk = (int)(unit % H_kv);
            const int64_t qrow0 = (int64_t)b * H_q + (int64_t)hk * G;
            const unsigned char* rowp = ring + (size_t)st * kTile + tid * kRowBytes;
            float a[G];
#pragma unroll
            for (int g = 0; g < G; ++g) a[g] = 0.f;
#pragma unroll
            for (int cc = 0; cc < NV; ++cc) {
                const int c = (cc + rot) & (NV - 1);
                const uint4 v = *reinterpret_cast<const uint4*>(rowp + c * 16);
                float f[KV];
                E::unpack(v, f);
#pragma unroll
                for (int g = 0; g < G; ++g)
#pragma unroll
                    for (int e = 0; e < KV; ++e) {
                        const int col = c * KV + e;
                        const float qc = col < d ? __ldcg(q_rot + (qrow0 + g) * D + col) : 0.f;
                        a[g] = fmaf(qc, f[e], a[g]);
                    }
            }
#pragma unroll
            for (int g = 0; g < G; ++g) scores[(qrow0 + g) * S + x] = a[g];
        }
        __syncwarp();
        if (lane == 0 && !bad) mbar_arrive(&empty[st]);
    }
}

template <class E, int G, int NV, bool kFuseQ>
__global__ void __launch_bounds__(kScoreThreads, 1) k_score_plane(
    const float* __restrict__ q_rot, const typename E::T* __restrict__ q,
    const float* __restrict__ P, const typename E::T* __restrict__ Klo,
    float* __restrict__ scores, int* __restrict__ err, int H_q, int H_kv, int S, int64_t S_max,
    int D, int d, int64_t total, int64_t per, int wait_row) {
    score_plane_body<E, G, NV, kFuseQ, false>(q_rot, q, P, Klo, scores, err, H_q, H_kv, S, S_max,
                                              D, d, total, per, wait_row);
}

// The kernel of a step that appends runs beside the rotation kernel, so it
// keeps to 128 registers: 9 warps at 128 leave room on every SM for the
// rotation's CTA (at 135 the rotation waited for the scan to end).
template <class E, int G, int NV, bool kFuseQ>
__global__ void __maxnreg__(128) k_score_plane_append(
    const float* __restrict__ q_rot, const typename E::T* __restrict__ q,
    const float* __restrict__ P, const typename E::T* __restrict__ Klo,
    float* __restrict__ scores, int* __restrict__ err, int H_q, int H_kv, int S, int64_t S_max,
    int D, int d, int64_t total, int64_t per, int wait_row) {
    score_plane_body<E, G, NV, kFuseQ, true>(q_rot, q, P, Klo, scores, err, H_q, H_kv, S, S_max,
                                             D, d, total, per, wait_row);
}

// Arguments shared by every instantiation of the launch path.
struct PlaneArgs {
    const float* q_rot;  // q~ rows (unfused), or
    const void* q;       // raw queries and
    const float* P;      // the PCA bases (fused)
    const void* Klo;
    float* scores;
    int* err;
    int B, H_q, H_kv;
    int64_t S, S_max;
    int D, d;
    int64_t wait_row;  // first row written by the preceding kernel (>= S: none)
};

template <class E, int G, int NV, bool kFuseQ>
static cudaError_t plane_impl(const PlaneArgs& a, cudaStream_t s, bool pdl) {
    DevInfo di;
    cudaError_t e = dev_info(&di);
    if (e != cudaSuccess) return e;
    constexpr int kTile = kScoreConsumers * NV * 16;
    constexpr int kStages = (kScoreRingBytes / kTile) < kScoreMaxStages ? (kScoreRingBytes / kTile)
                                                                      : kScoreMaxStages;
    const bool append = a.wait_row < a.S;
    auto kern = append ? k_score_plane_append<E, G, NV, kFuseQ> : k_score_plane<E, G, NV, kFuseQ>;
    const size_t smem = (size_t)kStages * kTile;
    static bool attr_set[2][64] = {};
    if (di.device < 64 && !attr_set[append][di.device]) {
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        attr_set[append][di.device] = true;
    }
    const int64_t total = (int64_t)a.B * a.H_kv * a.S;
    const int64_t resident = (int64_t)di.sm_count * occupancy((const void*)kern, kScoreThreads, smem);
    int64_t grid = (total + kScoreConsumers - 1) / kScoreConsumers;
    if (grid > resident) grid = resident;
    const int64_t per = (total + grid - 1) / grid;
    grid = (total + per - 1) / per;
    using T = typename E::T;
    return launch_kernel(kern, dim3((unsigned)grid), dim3(kScoreThreads), smem, s, pdl, a.q_rot,
                         static_cast<const T*>(a.q), a.P, static_cast<const T*>(a.Klo), a.scores,
                         a.err, a.H_q, a.H_kv, (int)a.S, a.S_max, a.D, a.d, total, per,
                         (int)(a.wait_row < a.S ? a.wait_row : a.S));
}

template <class E, int G, int NV>
static cudaError_t plane_if(const PlaneArgs& a, cudaStream_t s, bool pdl) {
    if constexpr (G * NV * E::kVec <= 64) {
        if (a.q != nullptr) return plane_impl<E, G, NV, true>(a, s, pdl);
        return plane_impl<E, G, NV, false>(a, s, pdl);
    } else {
        return cudaErrorInvalidValue;  // not dispatched (see score_plane_supported)
    }
}

template <class E, int G>
static cudaError_t plane_nv(int nv, const PlaneArgs& a, cudaStream_t s, bool pdl) {
    switch (nv) {
        case 1: return plane_if<E, G, 1>(a, s, pdl);
        case 2: return plane_if<E, G, 2>(a, s, pdl);
        case 4: return plane_if<E, G, 4>(a, s, pdl);
        case 8: return plane_if<E, G, 8>(a, s, pdl);
        default: return cudaErrorInvalidValue;
    }
}

template <class E>
static cudaError_t plane_dispatch(int G, int nv, const PlaneArgs& a, cudaStream_t s, bool pdl) {
    switch (G) {
#define LOKI_G(g) \
    case g:       \
        return plane_nv<E, g>(nv, a, s, pdl);
        LOKI_G(1) LOKI_G(2) LOKI_G(3) LOKI_G(4) LOKI_G(5) LOKI_G(6) LOKI_G(7) LOKI_G(8)
#undef LOKI_G
        default: return cudaErrorInvalidValue;
    }
}

// Plane rows of 1, 2, 4 or 8 chunks with G * chunks * elements <= 64 take the
// thread-per-row TMA kernel; other planes take the register-staged scan.
bool score_plane_supported(Dt dt, int G, int d_lo) {
    const int row_bytes = d_lo * (dt == kF32 ? 4 : 2);
    const int nv = row_bytes / 16;
    const int kv = dt == kF32 ? 4 : 8;
    return row_bytes % 16 == 0 && (nv == 1 || nv == 2 || nv == 4 || nv == 8) && G * nv * kv <= 64;
}

bool score_plane_fuses(Dt dt, int G, int d_lo, int D) {
    return D == 128 && score_plane_supported(dt, G, d_lo);
}

cudaError_t launch_score_plane(Dt dt, const float* q_rot, const void* Klo, int B, int H_q,
                               int H_kv, int64_t S, int64_t S_max, int D, int d_lo, int d,
                               float* scores, cudaStream_t s, bool pdl, const void* q,
                               const float* P, int64_t wait_row) {
    int* err = device_error_word();
    if (err == nullptr) return cudaErrorInvalidDevice;
    const int G = H_q / H_kv;
    if (!score_plane_supported(dt, G, d_lo)) {
        // the register-staged scan reads q~ from q_rot: it cannot rotate
        if (q != nullptr) return cudaErrorInvalidValue;
        return launch_score_lowdim(dt, q_rot, Klo, B, H_q, H_kv, S, S_max, D, d_lo, d, scores, s,
                                   pdl);
    }
    const int nv = d_lo * (dt == kF32 ? 4 : 2) / 16;
    const bool fuse = q != nullptr && P != nullptr;
    if (fuse && D != 128) return cudaErrorInvalidValue;  // the fused rotation takes head dim 128
    // a scan that rotates its own queries reads q and P at once: it is
    // launched early beside the preceding kernel only when that kernel writes
    // cache rows the producer waits for (an append), never q or P
    if (fuse && wait_row >= S) pdl = false;
    const PlaneArgs a{q_rot, fuse ? q : nullptr, fuse ? P : nullptr, Klo, scores, err, B, H_q,
                      H_kv, S, S_max, D, d, wait_row};
    if (dt == kF32) return plane_dispatch<ElemF32>(G, nv, a, s, pdl);
    return plane_dispatch<ElemBF16>(G, nv, a, s, pdl);
}

}  // namespace loki
