// Top-k token selection of Loki (NeurIPS 2024 poster page, TL;DR and "Visual
// Insights" Figure 1 caption: keep the k tokens with the largest approximate
// scores), as a kernel over rows of fp32 scores in global memory.
//
// k_topk: each row is held in the registers of one CTA (up to 32 keys per
// thread) or, when the row is long or there are few rows for the SMs, split
// over the CTAs of a thread-block cluster (2, 4 or 8 CTAs) that cooperate
// through distributed shared memory (topk_select.cuh). The first radix digit
// is histogrammed while the scores are loaded and turned into keys. Rows too
// long for an 8-CTA cluster (more than 262144 keys) take k_topk_long, which
// re-reads the scores from global memory in each pass.
#include "launch.h"
#include "topk_select.cuh"

namespace loki {

#ifndef LOKI_TOPK_CHUNK_TARGET
#define LOKI_TOPK_CHUNK_TARGET 32768  // keys one CTA holds before a row is split over a cluster
#endif
#ifndef LOKI_TOPK_SPLIT_FEW_ROWS
#define LOKI_TOPK_SPLIT_FEW_ROWS 0    // also split rows when they are fewer than 2 per SM
#endif
constexpr int kTopkChunkTarget = LOKI_TOPK_CHUNK_TARGET;

// One CTA (or one cluster of CTAs) per row. CTA rank r of the row's cluster
// holds keys [r * chunk, min((r + 1) * chunk, S)); chunk is a multiple of 4
// and at most 4 * NT * I.
// With lens (a per-sequence length, row r belonging to sequence r / H_q) a
// row holds lens[r / H_q] <= S keys at stride S: it selects min(k, length)
// and pads its output with -1.
// Rows of up to 4096 keys keep to 48 registers, so five 256-thread CTAs fit
// on an SM: a decode's rows (640 at the Llama2-13B shape) then all start in
// one wave on 148 SMs.
// Rows of 16384 keys (512 threads of 32 keys) keep to 64 registers, two CTAs
// per SM.
template <int NT, int I, bool kCl>
constexpr int kTopkMinBlocks = (!kCl && NT * I <= 1024) ? 1280 / NT : (!kCl && NT == 512) ? 2 : 1;

template <int NT, int I, bool kCl>
__global__ void __launch_bounds__(NT, (kTopkMinBlocks<NT, I, kCl>)) k_topk(
    const float* __restrict__ scores, int S, int k, int chunk, int32_t* __restrict__ out, int vec4,
    const int* __restrict__ lens, int H_q) {
    __shared__ __align__(16) uint32_t scratch[kTkSmemWords];
    TkCluster<kCl> cl;
    cl.init();
    const TkSmem sm = tk_carve(scratch);
    tk_zero<NT>(sm);
    __syncthreads();
    griddep_wait();  // scores come from the score kernel
    griddep_launch_dependents();

    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int64_t row = blockIdx.x / cl.size;
    const int base = cl.rank * chunk;
    const int S_row = lens != nullptr ? min(S, max(0, lens[row / H_q])) : S;
    const int k_row = min(k, S_row);
    const int n = max(0, min(chunk, S_row - base));
    const float* src = scores + row * S + base;
    int32_t* o = out + row * k;
    if (cl.rank == 0)
        for (int x = k_row + (int)threadIdx.x; x < k; x += NT) o[x] = -1;  // padding
    if (k_row == 0) return;  // an empty sequence (uniform over the cluster)
    uint4 v[I];
#pragma unroll
    for (int i = 0; i < I; ++i) {
        const int g = warp * 32 * I + 32 * i + lane;  // group of keys 4g .. 4g + 3
        const int j = 4 * g;
        if (vec4 && j + 3 < n) {
            const float4 f = __ldg(reinterpret_cast<const float4*>(src) + g);
            v[i] = make_uint4(order_key(f.x), order_key(f.y), order_key(f.z), order_key(f.w));
        } else {
            v[i] = make_uint4(j < n ? order_key(__ldg(src + j)) : 0u,
                              j + 1 < n ? order_key(__ldg(src + j + 1)) : 0u,
                              j + 2 < n ? order_key(__ldg(src + j + 2)) : 0u,
                              j + 3 < n ? order_key(__ldg(src + j + 3)) : 0u);
        }
    }
#pragma unroll
    for (int i = 0; i < I; ++i) {
        const uint32_t kk[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
        // only a group that reaches past the row's end holds padding (key 0)
        const bool whole = 4 * (warp * 32 * I + 32 * i + lane) + 3 < n;
#pragma unroll
        for (int e = 0; e < 4; ++e)
            if (whole || kk[e] != 0u) atomicAdd(&sm.hist1[kk[e] >> 21], 1u);
    }
    // rows of up to 4096 keys share each SM with four or more other CTAs:
    // searching in one warp saves the instructions of the others
    tk_select<NT, I, kCl, 0, (!kCl && NT * I <= 1024)>(cl, v, base, k_row, o, sm);
}

// exclusive prefix sum over the block; `total` gets the block sum
__device__ __forceinline__ int block_excl_scan(int v, int* buf, int* total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int nw = (blockDim.x + 31) >> 5;
    int x = v;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, off);
        if (lane >= off) x += y;
    }
    if (lane == 31) buf[warp] = x;
    __syncthreads();
    if (warp == 0) {
        int w = lane < nw ? buf[lane] : 0;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, w, off);
            if (lane >= off) w += y;
        }
        if (lane < nw) buf[lane] = w;  // inclusive warp totals
    }
    __syncthreads();
    const int before = (warp > 0 ? buf[warp - 1] : 0) + x - v;
    *total = buf[nw - 1];
    __syncthreads();
    return before;
}

// Long rows: keys in shared memory (kSmem) or re-read from global memory,
// 8-bit digits with warp-aggregated shared-memory atomics.
template <bool kSmem>
__global__ void __launch_bounds__(512) k_topk_long(const float* __restrict__ scores, int S, int k,
                                                   int32_t* __restrict__ out) {
    extern __shared__ uint32_t keys[];
    __shared__ uint32_t hist[256];
    __shared__ int s_bin, s_krem;
    __shared__ int scan_buf[32];
    const int tid = threadIdx.x, nt = blockDim.x, lane = tid & 31;
    const float* row = scores + (int64_t)blockIdx.x * S;
    griddep_wait();
    griddep_launch_dependents();

    if (kSmem) {
        for (int j = tid; j < S; j += nt) keys[j] = order_key(__ldg(row + j));
    }
    uint32_t prefix = 0u, mask = 0u;
    int krem = k;
    const int S_round = (S + 31) & ~31;
    for (int pass = 0; pass < 4; ++pass) {
        const int shift = 24 - 8 * pass;
        for (int i = tid; i < 256; i += nt) hist[i] = 0u;
        __syncthreads();
        for (int j = tid; j < S_round; j += nt) {
            int bin = 256;
            if (j < S) {
                const uint32_t key = kSmem ? keys[j] : order_key(__ldg(row + j));
                if ((key & mask) == prefix) bin = (int)((key >> shift) & 0xffu);
            }
            const unsigned peers = __match_any_sync(0xffffffffu, bin);
            if (bin < 256 && lane == __ffs(peers) - 1) atomicAdd(&hist[bin], (uint32_t)__popc(peers));
        }
        __syncthreads();
        // 256 bins over 512 threads: the first 256 threads own one bin each
        {
            const int c = tid < 256 ? (int)hist[tid] : 0;
            int total;
            const int before = block_excl_scan(c, scan_buf, &total);
            const int above = total - before - c;
            if (tid < 256 && above < krem && above + c >= krem) {
                s_bin = tid;
                s_krem = krem - above;
            }
        }
        __syncthreads();
        prefix |= (uint32_t)s_bin << shift;
        mask |= 0xffu << shift;
        krem = s_krem;
        __syncthreads();
    }
    const uint32_t T = prefix;

    const int per = (S + nt - 1) / nt;
    const int j0 = min(S, tid * per), j1 = min(S, j0 + per);
    int gt = 0, eq = 0;
    for (int j = j0; j < j1; ++j) {
        const uint32_t key = kSmem ? keys[j] : order_key(__ldg(row + j));
        gt += key > T;
        eq += key == T;
    }
    int total;
    const int eq_before = block_excl_scan(eq, scan_buf, &total);
    const int take_eq = max(0, min(eq, krem - eq_before));
    int pos = block_excl_scan(gt + take_eq, scan_buf, &total);
    int32_t* o = out + (int64_t)blockIdx.x * k;
    int eq_seen = 0;
    for (int j = j0; j < j1; ++j) {
        const uint32_t key = kSmem ? keys[j] : order_key(__ldg(row + j));
        bool take = key > T;
        if (key == T) {
            take = eq_seen < take_eq;
            ++eq_seen;
        }
        if (take) {
            if (pos < k) o[pos] = j;
            ++pos;
        }
    }
}

template <int NT, int I, bool kCl>
static cudaError_t launch_rows(const float* scores, int64_t rows, int S, int k, int C, int chunk,
                               int32_t* idx, cudaStream_t s, bool pdl, const int* lens, int H_q) {
    auto kern = k_topk<NT, I, kCl>;
    cudaError_t e = prefer_carveout(reinterpret_cast<const void*>(kern),
                                    cudaSharedmemCarveoutMaxShared);
    if (e != cudaSuccess) return e;
    const int vec4 = (S % 4 == 0) && (chunk % 4 == 0) &&
                     (reinterpret_cast<uintptr_t>(scores) % 16 == 0);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(rows * C));
    cfg.blockDim = dim3(NT);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    int na = 0;
    if (kCl) {
        attr[na].id = cudaLaunchAttributeClusterDimension;
        attr[na].val.clusterDim.x = (unsigned)C;
        attr[na].val.clusterDim.y = 1;
        attr[na].val.clusterDim.z = 1;
        ++na;
    }
    if (pdl) {
        attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[na].val.programmaticStreamSerializationAllowed = 1;
        ++na;
    }
    cfg.attrs = na ? attr : nullptr;
    cfg.numAttrs = (unsigned)na;
    return cudaLaunchKernelEx(&cfg, kern, scores, S, k, chunk, idx, vec4, lens, H_q);
}

template <bool kCl>
static cudaError_t launch_shape(int nt, int gi, const float* scores, int64_t rows, int S, int k,
                                int C, int chunk, int32_t* idx, cudaStream_t s, bool pdl,
                                const int* lens, int H_q) {
#define LOKI_TK(NT_, I_)                                                                        \
    if (nt == NT_ && gi == I_)                                                                  \
        return launch_rows<NT_, I_, kCl>(scores, rows, S, k, C, chunk, idx, s, pdl, lens, H_q);
    LOKI_TK(128, 1) LOKI_TK(128, 2) LOKI_TK(128, 4)
    LOKI_TK(256, 4) LOKI_TK(256, 8) LOKI_TK(512, 8)
    LOKI_TK(256, 1) LOKI_TK(512, 1)
    LOKI_TK(1024, 1) LOKI_TK(1024, 2) LOKI_TK(1024, 4) LOKI_TK(1024, 8)
#undef LOKI_TK
    return cudaErrorInvalidValue;
}

// Launch shape of k_topk for a [rows, S] problem: cluster size C, keys per
// CTA (chunk), threads per CTA (nt) and groups of 4 keys per thread (gi);
// false when S is too long for it.
bool topk_shape(int64_t rows, int64_t S, int sm_count, int* C_out, int* chunk_out, int* nt_out,
                int* gi_out) {
    int C = 1;
    auto chunk_of = [&](int c) { return (int)(((S + c - 1) / c + 3) / 4 * 4); };
    // split a row over a cluster only while its CTA would hold more than the
    // target (measured: one CTA per row beats a cluster at 4096 and 32768 keys)
    while (C < kTkMaxCluster &&
           (chunk_of(C) > kTopkChunkTarget ||
            (LOKI_TOPK_SPLIT_FEW_ROWS && rows * C < 2 * sm_count && chunk_of(2 * C) >= 1024)))
        C *= 2;
    const int chunk = chunk_of(C);
    // 128 threads up to 2048 keys, then 256 threads with up to 8 groups of 4
    // keys each, then more threads (measured: 256 x 4 beats 128 x 8 at 4096)
    // Many rows (at least two CTAs per SM): 128 threads up to 2048 keys, then
    // 256 threads with up to 8 groups of 4 keys each (measured: 256 x 4 beats
    // 128 x 8 at 4096 keys), then more threads. Few rows: one group of 4 keys
    // per thread up to 1024 threads (measured: 1024 x 1 takes two thirds of
    // the 256 x 4 time at 32 rows of 4096 keys).
    const bool few = rows * C < 2 * sm_count;
    int nt = chunk > 2048 ? 256 : 128, gi = 1;
    if (few)
        while (nt < 1024 && 4 * nt < chunk) nt *= 2;  // one group of 4 keys per thread
    while (4 * nt * gi < chunk && gi < 8) gi *= 2;
    while (4 * nt * gi < chunk && nt < 1024) nt *= 2;
    if (4 * nt * gi < chunk) return false;
    *C_out = C;
    *chunk_out = chunk;
    *nt_out = nt;
    *gi_out = gi;
    return true;
}

cudaError_t launch_topk(const float* scores, int64_t rows, int64_t S, int64_t k, int32_t* idx,
                        cudaStream_t s, bool pdl, const int* lens, int H_q) {
    const int Si = (int)S, ki = (int)k;
    DevInfo di;
    cudaError_t e = dev_info(&di);
    if (e != cudaSuccess) return e;
    int C, chunk, nt, gi;
    if (topk_shape(rows, S, di.sm_count, &C, &chunk, &nt, &gi)) {
        if (C == 1)
            return launch_shape<false>(nt, gi, scores, rows, Si, ki, 1, chunk, idx, s, pdl, lens,
                                       H_q);
        return launch_shape<true>(nt, gi, scores, rows, Si, ki, C, chunk, idx, s, pdl, lens, H_q);
    }
    if (lens != nullptr) return cudaErrorInvalidValue;  // per-row lengths: up to 262144 keys
    {
        const size_t need = (size_t)S * 4;
        if (need + 4096 <= (size_t)di.smem_optin) {
            e = cudaFuncSetAttribute(k_topk_long<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     (int)need);
            if (e != cudaSuccess) return e;
            return launch_kernel(k_topk_long<true>, dim3((unsigned)rows), dim3(512), need, s, pdl,
                                 scores, Si, ki, idx);
        }
        return launch_kernel(k_topk_long<false>, dim3((unsigned)rows), dim3(512), 0, s, pdl,
                             scores, Si, ki, idx);
    }
}

}  // namespace loki
