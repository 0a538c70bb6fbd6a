// Top-k token selection of Loki (NeurIPS 2024 poster page, TL;DR and "Visual
// Insights" Figure 1 caption: keep the k tokens with the largest approximate
// scores), as a kernel over rows of fp32 scores in global memory.
//
// One CTA per (batch, query head) row. Rows of up to 32768 keys
// (k_topk_smem) load their keys into shared memory and run the block-level
// radix select of topk_core.cuh. Longer rows (k_topk_long) keep keys in
// shared memory, or re-read them from L2 when they do not fit, with 8-bit
// digits and warp-aggregated atomics.
#include "launch.h"
#include "topk_core.cuh"

namespace loki {

// Rows of up to 32 * NT keys: keys in shared memory (zero-padded to a
// multiple of 4; key 0 never comes from a score), every loop rolled and over
// uint4 groups of 4 keys (a small kernel body that stays in the instruction
// cache, and few instructions per key).
template <int NT>
__global__ void __launch_bounds__(NT) k_topk_smem(const float* __restrict__ scores, int S, int k,
                                                  int32_t* __restrict__ out, int vec4) {
    extern __shared__ uint4 keys4[];
    __shared__ __align__(16) uint32_t hist[4096];
    __shared__ uint32_t cand[kTopkCandCap];
    __shared__ int scan_buf[32];
    __shared__ int small[5];
    const int tid = threadIdx.x;
    const int S4 = (S + 3) >> 2;
    const float* row = scores + (int64_t)blockIdx.x * S;
#pragma unroll 1
    for (int i = tid; i < 1024; i += NT) reinterpret_cast<uint4*>(hist)[i] = make_uint4(0u, 0u, 0u, 0u);
    griddep_wait();  // scores come from the score kernel
    griddep_launch_dependents();

    if (vec4) {  // S % 4 == 0 and scores 16-byte aligned
        // 8 loads in flight per thread before any is used: the row arrives in
        // one or two memory round trips instead of one per group
        constexpr int kInFlight = 8;
        const float4* r4 = reinterpret_cast<const float4*>(row);
#pragma unroll 1
        for (int j0 = tid; j0 < S4; j0 += kInFlight * NT) {
            float4 v[kInFlight];
#pragma unroll
            for (int u = 0; u < kInFlight; ++u) {
                const int j = j0 + u * NT;
                v[u] = j < S4 ? __ldg(r4 + j) : make_float4(0.f, 0.f, 0.f, 0.f);
            }
#pragma unroll
            for (int u = 0; u < kInFlight; ++u) {
                const int j = j0 + u * NT;
                if (j < S4)
                    keys4[j] = make_uint4(order_key(v[u].x), order_key(v[u].y), order_key(v[u].z),
                                          order_key(v[u].w));
            }
        }
    } else {
#pragma unroll 1
        for (int j = tid; j < S4; j += NT) {
            const int j4 = 4 * j;
            keys4[j] = make_uint4(order_key(__ldg(row + j4)),
                                  j4 + 1 < S ? order_key(__ldg(row + j4 + 1)) : 0u,
                                  j4 + 2 < S ? order_key(__ldg(row + j4 + 2)) : 0u,
                                  j4 + 3 < S ? order_key(__ldg(row + j4 + 3)) : 0u);
        }
    }
    __syncthreads();
    topk_block_select<NT>(keys4, S, k, out + (int64_t)blockIdx.x * k,
                          TopkScratch{hist, cand, scan_buf, small});
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

template <int NT>
static cudaError_t launch_smem(const float* scores, int64_t rows, int S, int k, int32_t* idx,
                              cudaStream_t s, bool pdl) {
    const size_t smem = ((size_t)S + 3) / 4 * 16;
    if (smem > 48 * 1024) {
        const cudaError_t e = cudaFuncSetAttribute(
            k_topk_smem<NT>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
    }
    const int vec4 = (S % 4 == 0) && (reinterpret_cast<uintptr_t>(scores) % 16 == 0);
    return launch_kernel(k_topk_smem<NT>, dim3((unsigned)rows), dim3(NT), smem, s, pdl, scores, S,
                         k, idx, vec4);
}

cudaError_t launch_topk(const float* scores, int64_t rows, int64_t S, int64_t k, int32_t* idx,
                        cudaStream_t s, bool pdl) {
    const int Si = (int)S, ki = (int)k;
    // each thread owns at most 16 consecutive keys of the row (32 for rows
    // longer than 16 x 512): shorter per-thread loops in a latency-bound kernel
    if (S <= 128 * 16) return launch_smem<128>(scores, rows, Si, ki, idx, s, pdl);
    if (S <= 256 * 16) return launch_smem<256>(scores, rows, Si, ki, idx, s, pdl);
    if (S <= 512 * 16) return launch_smem<512>(scores, rows, Si, ki, idx, s, pdl);
    if (S <= 1024 * 32) return launch_smem<1024>(scores, rows, Si, ki, idx, s, pdl);
    {
        DevInfo di;
        cudaError_t e = dev_info(&di);
        if (e != cudaSuccess) return e;
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
