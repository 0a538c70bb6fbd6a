// Top-k token selection of Loki (NeurIPS 2024 poster page, TL;DR and
// "Visual Insights" Figure 1 caption: keep the k tokens with the largest
// approximate scores).
//
// One CTA per (batch, query head) row. Scores become order-preserving 32-bit
// keys (larger float -> larger key; -0 folded onto +0; NaN folded onto -inf),
// held in shared memory when the row fits. An MSB-first radix select with
// 8-bit digits finds the k-th largest key T and how many keys equal to T
// belong to the set; warp-aggregated shared-memory atomics keep the
// histograms cheap when many keys share a digit. A stable compaction then
// writes the selected indices in ascending token order, taking keys equal to
// T from the lowest indices first. All decisions are integer compares, so the
// result is exact and deterministic.
#include "common.cuh"
#include "launch.h"

namespace loki {

__device__ __forceinline__ uint32_t order_key(float x) {
    uint32_t u = __float_as_uint(x);
    if ((u & 0x7f800000u) == 0x7f800000u && (u & 0x007fffffu)) u = 0xff800000u;  // NaN -> -inf
    if (u == 0x80000000u) u = 0u;                                                // -0 -> +0
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
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

template <bool kSmem>
__global__ void __launch_bounds__(512) k_topk(const float* __restrict__ scores, int S, int k,
                                              int32_t* __restrict__ out) {
    extern __shared__ uint32_t keys[];
    __shared__ uint32_t hist[256];
    __shared__ int s_digit, s_krem;
    __shared__ int scan_buf[32];
    const int tid = threadIdx.x, nt = blockDim.x, lane = tid & 31;
    if (tid == 0) {
        s_digit = 0;
        s_krem = k;
    }
    const float* row = scores + (int64_t)blockIdx.x * S;

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
        if (tid < 32) {
            // lane l owns bins [8l, 8l + 8); higher bins hold larger keys
            int c[8], tot = 0;
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                c[e] = (int)hist[8 * lane + e];
                tot += c[e];
            }
            int suf = tot;  // inclusive suffix sum over lanes
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const int y = __shfl_down_sync(0xffffffffu, suf, off);
                if (lane + off < 32) suf += y;
            }
            int above = suf - tot;
#pragma unroll
            for (int e = 7; e >= 0; --e) {
                if (above < krem && above + c[e] >= krem) {
                    s_digit = 8 * lane + e;
                    s_krem = krem - above;
                }
                above += c[e];
            }
        }
        __syncthreads();
        prefix |= (uint32_t)s_digit << shift;
        mask |= 0xffu << shift;
        krem = s_krem;
    }
    const uint32_t T = prefix;  // the k-th largest key; take `krem` of the keys equal to T

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
    const int off = block_excl_scan(gt + take_eq, scan_buf, &total);
    int32_t* o = out + (int64_t)blockIdx.x * k;
    int pos = off;  // stays below k by construction; the bound keeps a row's writes in the row
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

cudaError_t launch_topk(const float* scores, int64_t rows, int64_t S, int64_t k, int32_t* idx,
                        cudaStream_t s) {
    DevInfo di;
    cudaError_t e = dev_info(&di);
    if (e != cudaSuccess) return e;
    const size_t static_smem = 256 * 4 + 32 * 4 + 16;
    const size_t need = (size_t)S * 4;
    const int threads = 512;
    if (need + static_smem <= (size_t)di.smem_optin) {
        if (need > 48 * 1024) {
            e = cudaFuncSetAttribute(k_topk<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     (int)need);
            if (e != cudaSuccess) return e;
        }
        k_topk<true><<<(unsigned)rows, threads, need, s>>>(scores, (int)S, (int)k, idx);
    } else {
        k_topk<false><<<(unsigned)rows, threads, 0, s>>>(scores, (int)S, (int)k, idx);
    }
    return cudaGetLastError();
}

}  // namespace loki
