// Low-dimensional score scan over a paged key plane, for batches whose
// sequences have their own lengths.
//
// Loki (NeurIPS 2024 poster page, TL;DR; briefgpt.xyz abstract page): every
// cached token of a sequence is scored on the first d principal components,
// s_j = q~[:d] . K~_j[:d], j < S_b.
//
// Cache layout: the key plane is a pool of pages [n_pages, H_kv, page_size,
// d_lo]; sequence b's token j lives in page block_table[b][j / page_size], at
// slot j % page_size. (A contiguous cache [B, H_kv, S_max, d_lo] is the case
// page_size = S_max with block_table[b][0] = b.)
//
// k_paged_prefix (one CTA) turns the lengths into the scan's work split
// without a host round trip: the rows of all (sequence, KV head) units laid
// end to end (H_kv * S_b rows for sequence b) are cut evenly over the scan's
// CTAs, and each CTA's first row is located. The scan then works like the
// contiguous one (one producer warp issuing bulk copies into a ring of
// shared-memory stages, 256 consumer threads scoring one row each), except
// that a tile of 256 rows is copied page segment by page segment, the page
// numbers of a unit's rows being read once into shared memory.
#include "common.cuh"
#include "launch.h"
#include "tma.cuh"

namespace loki {

// Workspace of the paged decode, in front of the usual decode workspace.
struct PagedStart {
    int64_t b;      // sequence of the CTA's first row
    int64_t off;    // row of it within the sequence's H_kv * S_b rows
    int64_t count;  // rows of the CTA
};

__global__ void __launch_bounds__(1024) k_paged_prefix(const int* __restrict__ seq_lens, int B,
                                                       int H_kv, int64_t S_cap,
                                                       int* __restrict__ lens,
                                                       int64_t* __restrict__ rowoff,
                                                       PagedStart* __restrict__ starts, int grid) {
    __shared__ int64_t s_warp[32];
    __shared__ int64_t s_carry;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    if (tid == 0) s_carry = 0;
    __syncthreads();
    // exclusive prefix of H_kv * S_b over the sequences, 1024 at a time
    for (int b0 = 0; b0 < B; b0 += 1024) {
        const int b = b0 + tid;
        int64_t v = 0;
        if (b < B) {
            int64_t L = seq_lens[b];
            L = L < 0 ? 0 : (L > S_cap ? S_cap : L);
            lens[b] = (int)L;
            v = L * H_kv;
        }
        int64_t x = v;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int64_t y = __shfl_up_sync(0xffffffffu, x, off);
            if (lane >= off) x += y;
        }
        if (lane == 31) s_warp[warp] = x;
        __syncthreads();
        int64_t before = s_carry;
        for (int w = 0; w < warp; ++w) before += s_warp[w];
        if (b < B) rowoff[b] = before + x - v;
        __syncthreads();
        if (tid == 1023) s_carry = before + x;
        __syncthreads();
    }
    if (tid == 0) rowoff[B] = s_carry;
    __syncthreads();
    const int64_t total = s_carry;
    // each scan CTA's first row: the last sequence whose offset is <= it
    for (int c = tid; c < grid; c += 1024) {
        const int64_t R0 = total * c / grid, R1 = total * (c + 1) / grid;
        int lo = 0, hi = B - 1;
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (rowoff[mid] <= R0) lo = mid;
            else hi = mid - 1;
        }
        // skip empty sequences at the boundary
        while (lo < B - 1 && rowoff[lo + 1] <= R0) ++lo;
        starts[c].b = lo;
        starts[c].off = R0 - rowoff[lo];
        starts[c].count = R1 - R0;
    }
}

constexpr int kPgConsumerWarps = 8;
constexpr int kPgConsumers = kPgConsumerWarps * 32;
constexpr int kPgThreads = kPgConsumers + 32;
constexpr int kPgRingBytes = 96 * 1024;
constexpr int kPgMaxStages = 16;
constexpr int kPgPageCache = 2048;  // page numbers of a unit held in shared memory at a time

// A walker over the CTA's rows: unit (b, hk) and row j, as both roles see them.
struct PgCursor {
    int64_t b;
    int hk;
    int64_t j;
    int64_t left;  // rows of the CTA still to visit
};

template <class E, int G, int NV>
__global__ void __launch_bounds__(kPgThreads, 1) k_score_paged(
    const float* __restrict__ q_rot, const typename E::T* __restrict__ Klo_pages,
    const int* __restrict__ block_table, const int* __restrict__ lens,
    const PagedStart* __restrict__ starts, float* __restrict__ scores, int* __restrict__ err,
    int B, int H_q, int H_kv, int page_size, int max_pages, int64_t n_pages, int64_t S_cap,
    int d, int D) {
    constexpr int KV = E::kVec;
    constexpr int kRowBytes = NV * 16;
    constexpr int kTR = kPgConsumers;  // rows per tile
    constexpr int kTile = kTR * kRowBytes;
    constexpr int kStages = (kPgRingBytes / kTile) < kPgMaxStages ? (kPgRingBytes / kTile)
                                                                  : kPgMaxStages;
    static_assert(kStages >= 2, "ring too small");
    extern __shared__ __align__(128) unsigned char ring[];
    __shared__ uint64_t full[kStages], empty[kStages];
    __shared__ int s_pages[kPgPageCache];

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (tid == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kPgConsumerWarps);
        }
        fence_mbar_init();
    }
    __syncthreads();
    griddep_wait();  // the work split, the lengths and q~ come from earlier kernels
    griddep_launch_dependents();

    const PagedStart st0 = starts[blockIdx.x];
    PgCursor cur;
    cur.b = st0.b;
    cur.left = st0.count;
    {
        const int64_t L = lens[cur.b];
        cur.hk = L > 0 ? (int)(st0.off / L) : H_kv;
        cur.j = L > 0 ? st0.off % L : 0;
    }

    if (warp == kPgConsumerWarps) {
        // ---------------- producer: every lane issues page-segment copies ----------------
        const uint64_t pol = l2_policy_evict_first();
        int i = 0;
        bool ok = true;
        PgCursor c = cur;
        int64_t cached_b = -1, cached_p0 = -1;
        while (c.left > 0 && ok && c.b < B) {
            const int64_t L = lens[c.b];
            if (c.hk >= H_kv || c.j >= L) {  // next unit
                if (++c.hk >= H_kv || L == 0) {
                    c.hk = 0;
                    ++c.b;
                }
                c.j = 0;
                continue;
            }
            const int seg = (int)min64(L - c.j, c.left);
            for (int t0 = 0; t0 < seg && ok; t0 += kTR, ++i) {
                const int n = min(kTR, seg - t0);
                const int64_t j0 = c.j + t0;
                const int64_t p_first = j0 / page_size, p_last = (j0 + n - 1) / page_size;
                // page numbers of this sequence, kPgPageCache at a time
                if (c.b != cached_b || p_first < cached_p0 || p_last >= cached_p0 + kPgPageCache) {
                    __syncwarp();
                    cached_b = c.b;
                    cached_p0 = p_first;
                    const int np = (int)min64(kPgPageCache, (int64_t)max_pages - p_first);
                    const int* bt = block_table + c.b * max_pages + p_first;
                    for (int x = lane; x < np; x += 32) s_pages[x] = __ldg(bt + x);
                    __syncwarp();
                }
                const int stg = i % kStages;
                const uint32_t ph = (uint32_t)(i / kStages) & 1u;
                int okw = 1;
                if (lane == 0) {
                    okw = mbar_wait(&empty[stg], ph ^ 1u, err) ? 1 : 0;
                    if (okw) mbar_arrive_expect_tx(&full[stg], (uint32_t)(n * kRowBytes));
                }
                okw = __shfl_sync(0xffffffffu, okw, 0);
                if (!okw) {
                    ok = false;
                    break;
                }
                __syncwarp();  // the expected bytes are registered before any copy lands
                const int nseg = (int)(p_last - p_first + 1);
                for (int sgi = lane; sgi < nseg; sgi += 32) {
                    const int64_t lp = p_first + sgi;
                    const int64_t r0 = lp * page_size > j0 ? lp * page_size : j0;
                    const int64_t r1 = min64((lp + 1) * page_size, j0 + n);
                    int64_t phys = s_pages[lp - cached_p0];
                    if (phys < 0 || phys >= n_pages) {  // a bad block-table entry: flag it and
                        atomicExch(err, kDevErrBadPage);  // read page 0 instead of faulting
                        phys = 0;
                    }
                    const char* src = reinterpret_cast<const char*>(Klo_pages) +
                                      ((phys * H_kv + c.hk) * page_size + (r0 - lp * page_size)) *
                                          (int64_t)kRowBytes;
                    bulk_load_hint(ring + (size_t)stg * kTile + (r0 - j0) * kRowBytes, src,
                                   (uint32_t)((r1 - r0) * kRowBytes), &full[stg], pol);
                }
            }
            c.j += seg;
            c.left -= seg;
        }
        // every issued copy has landed before the CTA may exit
        if (lane == 0)
            for (int j = max(0, i - kStages); j < i; ++j)
                mbar_wait(&full[j % kStages], (uint32_t)(j / kStages) & 1u, err);
        return;
    }

    // ---------------- consumers: one row of each tile per thread ----------------
    bool bad = false;
    int i = 0;
    PgCursor c = cur;
    while (c.left > 0 && c.b < B) {
        const int64_t L = lens[c.b];
        if (c.hk >= H_kv || c.j >= L) {
            if (++c.hk >= H_kv || L == 0) {
                c.hk = 0;
                ++c.b;
            }
            c.j = 0;
            continue;
        }
        const int seg = (int)min64(L - c.j, c.left);
        const int64_t qrow0 = c.b * H_q + (int64_t)c.hk * G;
        float qv[G][NV * KV];
#pragma unroll
        for (int g = 0; g < G; ++g)
#pragma unroll
            for (int x = 0; x < NV * KV; ++x)
                qv[g][x] = x < d ? __ldcg(q_rot + (qrow0 + g) * D + x) : 0.f;
        float* srow = scores + qrow0 * S_cap + c.j;
        for (int t0 = 0; t0 < seg; t0 += kTR, ++i) {
            const int n = min(kTR, seg - t0);
            const int stg = i % kStages;
            const uint32_t ph = (uint32_t)(i / kStages) & 1u;
            if (!bad && !mbar_wait(&full[stg], ph, err)) bad = true;
            if (!bad && tid < n) {
                const unsigned char* rowp = ring + (size_t)stg * kTile + tid * kRowBytes;
                float a[G];
#pragma unroll
                for (int g = 0; g < G; ++g) a[g] = 0.f;
#pragma unroll
                for (int cc = 0; cc < NV; ++cc) {
                    const uint4 v = *reinterpret_cast<const uint4*>(rowp + cc * 16);
                    float f[KV];
                    E::unpack(v, f);
#pragma unroll
                    for (int g = 0; g < G; ++g)
#pragma unroll
                        for (int e = 0; e < KV; ++e) a[g] = fmaf(qv[g][cc * KV + e], f[e], a[g]);
                }
#pragma unroll
                for (int g = 0; g < G; ++g) srow[(int64_t)g * S_cap + t0 + tid] = a[g];
            }
            __syncwarp();
            if (lane == 0 && !bad) mbar_arrive(&empty[stg]);
        }
        c.j += seg;
        c.left -= seg;
    }
}

// ---------------------------------------------------------------------------

int paged_scan_grid() {
    DevInfo di;
    if (dev_info(&di) != cudaSuccess) return 0;
    return di.sm_count;  // one CTA per SM (the ring takes most of its shared memory)
}

size_t paged_start_bytes(int B, int grid) {
    return (size_t)(B + 1) * sizeof(int64_t) + (size_t)B * sizeof(int) +
           (size_t)grid * sizeof(PagedStart) + 64;
}

template <class E, int G, int NV>
static cudaError_t paged_impl(const float* q_rot, const void* Klo, const int* bt, const int* lens,
                              const void* starts, float* scores, int* err, int B, int H_q,
                              int H_kv, int page_size, int max_pages, int64_t n_pages,
                              int64_t S_cap, int d, int D, int grid, cudaStream_t s) {
    constexpr int kTile = kPgConsumers * NV * 16;
    constexpr int kStages = (kPgRingBytes / kTile) < kPgMaxStages ? (kPgRingBytes / kTile)
                                                                  : kPgMaxStages;
    auto kern = k_score_paged<E, G, NV>;
    const size_t smem = (size_t)kStages * kTile;
    DevInfo di;
    cudaError_t e = dev_info(&di);
    if (e != cudaSuccess) return e;
    static bool attr_set[64] = {};
    if (di.device < 64 && !attr_set[di.device]) {
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        attr_set[di.device] = true;
    }
    using T = typename E::T;
    return launch_kernel(kern, dim3((unsigned)grid), dim3(kPgThreads), smem, s, true, q_rot,
                         static_cast<const T*>(Klo), bt, lens,
                         static_cast<const PagedStart*>(starts), scores, err, B, H_q, H_kv,
                         page_size, max_pages, n_pages, S_cap, d, D);
}

template <class E, int G>
static cudaError_t paged_nv(int nv, const float* q_rot, const void* Klo, const int* bt,
                            const int* lens, const void* starts, float* scores, int* err, int B,
                            int H_q, int H_kv, int page_size, int max_pages, int64_t n_pages,
                            int64_t S_cap, int d, int D, int grid, cudaStream_t s) {
    switch (nv) {
#define LOKI_NV(n)                                                                              \
    case n:                                                                                     \
        if constexpr (G * n * E::kVec <= 64)                                                    \
            return paged_impl<E, G, n>(q_rot, Klo, bt, lens, starts, scores, err, B, H_q, H_kv, \
                                       page_size, max_pages, n_pages, S_cap, d, D, grid, s);    \
        return cudaErrorInvalidValue;
        LOKI_NV(1) LOKI_NV(2) LOKI_NV(4) LOKI_NV(8)
#undef LOKI_NV
        default: return cudaErrorInvalidValue;
    }
}

bool paged_scan_supported(Dt dt, int G, int d_lo) {
    const int row_bytes = d_lo * (dt == kF32 ? 4 : 2);
    const int nv = row_bytes / 16;
    const int kv = dt == kF32 ? 4 : 8;
    return row_bytes % 16 == 0 && (nv == 1 || nv == 2 || nv == 4 || nv == 8) && G >= 1 && G <= 8 &&
           G * nv * kv <= 64;
}

cudaError_t launch_paged_prefix(const int* seq_lens, int B, int H_kv, int64_t S_cap, void* start_ws,
                                int grid, cudaStream_t s) {
    char* w = static_cast<char*>(start_ws);
    int64_t* rowoff = reinterpret_cast<int64_t*>(w);
    int* lens = reinterpret_cast<int*>(w + (size_t)(B + 1) * sizeof(int64_t));
    const size_t off = ((size_t)(B + 1) * sizeof(int64_t) + (size_t)B * sizeof(int) + 15) / 16 * 16;
    PagedStart* starts = reinterpret_cast<PagedStart*>(w + off);
    return launch_kernel(k_paged_prefix, dim3(1), dim3(1024), 0, s, false, seq_lens, B, H_kv,
                         S_cap, lens, rowoff, starts, grid);
}

const int* paged_lens(const void* start_ws, int B) {
    return reinterpret_cast<const int*>(static_cast<const char*>(start_ws) +
                                        (size_t)(B + 1) * sizeof(int64_t));
}

cudaError_t launch_score_paged(Dt dt, const float* q_rot, const void* Klo_pages, int d_lo,
                               const int* block_table, const void* start_ws, int B, int H_q,
                               int H_kv, int page_size, int max_pages, int64_t n_pages,
                               int64_t S_cap, int d, int D, float* scores, int grid,
                               cudaStream_t s) {
    int* err = device_error_word();
    if (err == nullptr) return cudaErrorInvalidDevice;
    const int G = H_q / H_kv;
    if (!paged_scan_supported(dt, G, d_lo)) return cudaErrorInvalidValue;
    const int nv = d_lo * (dt == kF32 ? 4 : 2) / 16;
    const char* w = static_cast<const char*>(start_ws);
    const int* lens = reinterpret_cast<const int*>(w + (size_t)(B + 1) * sizeof(int64_t));
    const size_t off = ((size_t)(B + 1) * sizeof(int64_t) + (size_t)B * sizeof(int) + 15) / 16 * 16;
    const void* starts = w + off;
    switch (G) {
#define LOKI_G(g)                                                                              \
    case g:                                                                                    \
        if (dt == kF32)                                                                        \
            return paged_nv<ElemF32, g>(nv, q_rot, Klo_pages, block_table, lens, starts,       \
                                        scores, err, B, H_q, H_kv, page_size, max_pages,       \
                                        n_pages, S_cap, d, D, grid, s);                        \
        return paged_nv<ElemBF16, g>(nv, q_rot, Klo_pages, block_table, lens, starts, scores,   \
                                     err, B, H_q, H_kv, page_size, max_pages, n_pages, S_cap,  \
                                     d, D, grid, s);
        LOKI_G(1) LOKI_G(2) LOKI_G(3) LOKI_G(4) LOKI_G(5) LOKI_G(6) LOKI_G(7) LOKI_G(8)
#undef LOKI_G
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace loki
