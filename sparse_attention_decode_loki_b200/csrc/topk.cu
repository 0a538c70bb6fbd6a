// Top-k token selection of Loki (NeurIPS 2024 poster page, TL;DR and
// "Visual Insights" Figure 1 caption: keep the k tokens with the largest
// approximate scores).
//
// One CTA per (batch, query head) row. Scores become order-preserving 32-bit
// keys (larger float -> larger key; -0 folded onto +0; NaN folded onto -inf).
// A most-significant-digit radix select finds the k-th largest key T and how
// many keys equal to T belong to the set; a stable compaction then writes the
// selected indices in ascending token order, taking keys equal to T from the
// lowest indices first. All decisions are integer compares: the result is
// exact and deterministic.
//
// Rows of up to 32768 keys (k_topk_reg): each thread holds a contiguous run of
// keys in registers. One block pass histograms the top 12 key bits (4096
// shared-memory bins: sign, exponent and 3 mantissa bits), which already
// narrows the threshold to one bin holding a few percent of the row; those
// keys are gathered and warp 0 resolves the remaining 20 bits alone with two
// 10-bit passes over a warp-private histogram, so no further block barriers
// are paid. (A bin too crowded
// for the gather buffer -- heavy ties -- takes two 10-bit block passes.)
// Longer rows (k_topk_long) keep keys in shared memory, or re-read them from
// L2 when they do not fit, with 8-bit digits and warp-aggregated atomics.
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

// Given per-bin counts in hist[0, nbins) (bins ordered by key), find the bin
// holding the krem-th largest counted key. Thread t owns bins [t*per, (t+1)*per)
// and reads them in a rotated order (bank-conflict free for per <= 32).
// Writes the bin, the rank left inside it and the bin's count to shared memory.
__device__ __forceinline__ void find_bin(const uint32_t* hist, int nbins, int krem, int* buf,
                                         int* s_bin, int* s_krem, int* s_cnt) {
    const int per = nbins / (int)blockDim.x;
    const int b0 = threadIdx.x * per;
    const int rot = threadIdx.x & (per - 1);
    int local = 0;
    for (int i = 0; i < per; ++i) local += (int)hist[b0 + ((i + rot) & (per - 1))];
    int total;
    const int before = block_excl_scan(local, buf, &total);
    int above = total - before - local;  // keys in bins owned by higher threads
    if (above < krem && above + local >= krem) {
        for (int i = per - 1; i >= 0; --i) {
            const int c = (int)hist[b0 + i];
            if (above < krem && above + c >= krem) {
                *s_bin = b0 + i;
                *s_krem = krem - above;
                *s_cnt = c;
            }
            above += c;
        }
    }
    __syncthreads();
}

// Warp-synchronous select over n candidate keys (all sharing their top 12
// bits) held in shared memory: finds the krem-th largest with two 10-bit
// passes over a warp-private 1024-bin histogram `h`. Lane l owns bins
// [32l, 32l + 32) and reads them rotated by l (bank-conflict free). Returns
// (low 20 bits of the threshold, rank left inside it, count of keys equal to it).
__device__ __forceinline__ void warp_select20(const uint32_t* cand, int n, int krem, uint32_t* h,
                                              uint32_t* low, int* krem_out, int* cnt_out) {
    const int lane = threadIdx.x & 31;
    uint32_t hi10 = 0u;
    int cnt_sel = 0;
#pragma unroll
    for (int pass = 0; pass < 2; ++pass) {
        const int shift = pass == 0 ? 10 : 0;
#pragma unroll
        for (int i = 0; i < 32; ++i) h[32 * i + lane] = 0u;
        __syncwarp();
        for (int i = lane; i < n; i += 32) {
            const uint32_t c = cand[i];
            if (pass == 0 || ((c >> 10) & 1023u) == hi10) atomicAdd(&h[(c >> shift) & 1023u], 1u);
        }
        __syncwarp();
        int local = 0;
#pragma unroll
        for (int i = 0; i < 32; ++i) local += (int)h[32 * lane + ((i + lane) & 31)];
        int suf = local;  // inclusive suffix sum over lanes
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int y = __shfl_down_sync(0xffffffffu, suf, off);
            if (lane + off < 32) suf += y;
        }
        int above = suf - local;
        int bin = -1, kr = 0, cnt = 0;
        if (above < krem && above + local >= krem) {
            for (int i = 31; i >= 0; --i) {
                const int c = (int)h[32 * lane + i];
                if (above < krem && above + c >= krem) {
                    bin = 32 * lane + i;
                    kr = krem - above;
                    cnt = c;
                }
                above += c;
            }
        }
        const int src = __ffs(__ballot_sync(0xffffffffu, bin >= 0)) - 1;
        bin = __shfl_sync(0xffffffffu, bin, src);
        krem = __shfl_sync(0xffffffffu, kr, src);
        cnt_sel = __shfl_sync(0xffffffffu, cnt, src);
        if (pass == 0) hi10 = (uint32_t)bin;
        else *low = (hi10 << 10) | (uint32_t)bin;
        __syncwarp();
    }
    *krem_out = krem;
    *cnt_out = cnt_sel;
}

template <int KPT, int NT>
__global__ void __launch_bounds__(NT) k_topk_reg(const float* __restrict__ scores, int S, int k,
                                                 int32_t* __restrict__ out) {
    constexpr int kCandCap = 2048;
    __shared__ uint32_t hist[4096];
    __shared__ uint32_t cand[kCandCap];
    __shared__ int scan_buf[32];
    __shared__ int s_bin, s_krem, s_cnt, s_ncand;
    __shared__ uint32_t s_T;
    const int tid = threadIdx.x;
    const float* row = scores + (int64_t)blockIdx.x * S;
    const int j0 = tid * KPT;
    for (int i = tid; i < 4096; i += NT) hist[i] = 0u;
    if (tid == 0) s_ncand = 0;
    griddep_wait();  // scores come from the score kernel
    griddep_launch_dependents();

    uint32_t key[KPT];
    if ((S & 3) == 0) {
#pragma unroll
        for (int e = 0; e < KPT; e += 4) {
            if (j0 + e < S) {
                const float4 v = __ldg(reinterpret_cast<const float4*>(row + j0 + e));
                key[e] = order_key(v.x);
                key[e + 1] = order_key(v.y);
                key[e + 2] = order_key(v.z);
                key[e + 3] = order_key(v.w);
            } else {
                key[e] = key[e + 1] = key[e + 2] = key[e + 3] = 0u;
            }
        }
    } else {
#pragma unroll
        for (int e = 0; e < KPT; ++e) key[e] = (j0 + e < S) ? order_key(__ldg(row + j0 + e)) : 0u;
    }
    // key 0 never comes from a score (NaN maps to the -inf key), so it marks
    // padding: it is never counted, selected or histogrammed
    __syncthreads();

    // pass 1: top 12 bits over the whole row
#pragma unroll
    for (int e = 0; e < KPT; ++e)
        if (key[e]) atomicAdd(&hist[key[e] >> 20], 1u);
    __syncthreads();
    find_bin(hist, 4096, k, scan_buf, &s_bin, &s_krem, &s_cnt);
    const uint32_t bin1 = (uint32_t)s_bin;
    int krem = s_krem;
    const int n1 = s_cnt;  // keys in the threshold bin

    uint32_t T;
    int cnt_T;
    if (n1 <= kCandCap) {
        // gather the threshold bin's keys (one shared atomic per warp reserves
        // the warp's slots); warp 0 then resolves the low 20 bits
        int mine = 0;
#pragma unroll
        for (int e = 0; e < KPT; ++e) mine += (key[e] && (key[e] >> 20) == bin1);
        const int lane = tid & 31;
        int incl = mine;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, incl, off);
            if (lane >= off) incl += y;
        }
        int base = 0;
        if (lane == 31 && incl > 0) base = atomicAdd(&s_ncand, incl);
        base = __shfl_sync(0xffffffffu, base, 31) + incl - mine;
#pragma unroll
        for (int e = 0; e < KPT; ++e)
            if (key[e] && (key[e] >> 20) == bin1) cand[base++] = key[e];
        __syncthreads();
        if (tid < 32) {
            uint32_t low;
            int kr, c;
            // the pass-1 histogram is no longer read: its first 1024 bins serve warp 0
            warp_select20(cand, s_ncand, krem, hist, &low, &kr, &c);
            if (tid == 0) {
                s_T = (bin1 << 20) | low;
                s_krem = kr;
                s_cnt = c;
            }
        }
        __syncthreads();
        T = s_T;
        krem = s_krem;
        cnt_T = s_cnt;
    } else {
        // a crowded bin (heavy ties): two more block passes of 10 bits each
        __syncthreads();
        for (int i = tid; i < 1024; i += NT) hist[i] = 0u;
        __syncthreads();
#pragma unroll
        for (int e = 0; e < KPT; ++e)
            if (key[e] && (key[e] >> 20) == bin1) atomicAdd(&hist[(key[e] >> 10) & 1023u], 1u);
        __syncthreads();
        find_bin(hist, 1024, krem, scan_buf, &s_bin, &s_krem, &s_cnt);
        const uint32_t pre2 = (bin1 << 10) | (uint32_t)s_bin;
        krem = s_krem;
        __syncthreads();
        for (int i = tid; i < 1024; i += NT) hist[i] = 0u;
        __syncthreads();
#pragma unroll
        for (int e = 0; e < KPT; ++e)
            if (key[e] && (key[e] >> 10) == pre2) atomicAdd(&hist[key[e] & 1023u], 1u);
        __syncthreads();
        find_bin(hist, 1024, krem, scan_buf, &s_bin, &s_krem, &s_cnt);
        T = (pre2 << 10) | (uint32_t)s_bin;
        krem = s_krem;
        cnt_T = s_cnt;
    }
    // T is the k-th largest key; krem of the cnt_T keys equal to T are taken,
    // lowest indices first

    int gt = 0, eq = 0;
#pragma unroll
    for (int e = 0; e < KPT; ++e) {
        gt += key[e] > T;
        eq += key[e] == T;
    }
    int total, take_eq;
    if (krem == cnt_T) {
        take_eq = eq;  // every key equal to T is selected: no tie scan needed
    } else {
        const int eq_before = block_excl_scan(eq, scan_buf, &total);
        take_eq = max(0, min(eq, krem - eq_before));
    }
    int pos = block_excl_scan(gt + take_eq, scan_buf, &total);
    int32_t* o = out + (int64_t)blockIdx.x * k;
    int eq_seen = 0;
#pragma unroll
    for (int e = 0; e < KPT; ++e) {
        bool take = key[e] > T;
        if (key[e] == T) {
            take = eq_seen < take_eq;
            ++eq_seen;
        }
        if (take) {
            if (pos < k) o[pos] = j0 + e;  // pos < k by construction; the bound keeps writes in the row
            ++pos;
        }
    }
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

template <int KPT, int NT>
static cudaError_t launch_reg(const float* scores, int64_t rows, int S, int k, int32_t* idx,
                              cudaStream_t s, bool pdl) {
    return launch_kernel(k_topk_reg<KPT, NT>, dim3((unsigned)rows), dim3(NT), 0, s, pdl, scores,
                         S, k, idx);
}

cudaError_t launch_topk(const float* scores, int64_t rows, int64_t S, int64_t k, int32_t* idx,
                        cudaStream_t s, bool pdl) {
    const int Si = (int)S, ki = (int)k;
    // find_bin needs 4096 and 1024 bins to split evenly over the threads (NT <= 1024)
    if (S <= 128 * 4) return launch_reg<4, 128>(scores, rows, Si, ki, idx, s, pdl);
    if (S <= 128 * 8) return launch_reg<8, 128>(scores, rows, Si, ki, idx, s, pdl);
    if (S <= 128 * 16) return launch_reg<16, 128>(scores, rows, Si, ki, idx, s, pdl);
    if (S <= 256 * 16) return launch_reg<16, 256>(scores, rows, Si, ki, idx, s, pdl);
    if (S <= 256 * 32) return launch_reg<32, 256>(scores, rows, Si, ki, idx, s, pdl);
    if (S <= 512 * 32) return launch_reg<32, 512>(scores, rows, Si, ki, idx, s, pdl);
    if (S <= 512 * 64) return launch_reg<64, 512>(scores, rows, Si, ki, idx, s, pdl);
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
