// Exact top-k selection over order-preserving 32-bit keys held in shared
// memory (Loki's token selection: NeurIPS 2024 poster page, TL;DR and "Visual
// Insights" Figure 1 caption -- keep the k tokens with the largest approximate
// scores). Shared by the standalone top-k kernel and the fused decode kernel.
//
// Scores become order-preserving keys (larger float -> larger key; -0 folded
// onto +0; NaN folded onto -inf). A most-significant-digit radix select finds
// the k-th largest key T and how many keys equal to T belong to the set; a
// stable compaction then writes the selected indices in ascending token
// order, taking keys equal to T from the lowest indices first. All decisions
// are integer compares: the result is exact and deterministic.
//
// One block pass histograms the top 12 key bits (4096 shared-memory bins:
// sign, exponent and 3 mantissa bits), which already narrows the threshold to
// one bin holding a few percent of the row; those keys are gathered and warp
// 0 resolves the remaining 20 bits alone with two 10-bit passes over a
// warp-private histogram, so no further block barriers are paid. (A bin too
// crowded for the gather buffer -- heavy ties -- takes two 10-bit block
// passes.) The compaction reads each thread's run of keys once into bit masks
// and writes the selected indices in ascending order from them.
#pragma once

#include "common.cuh"

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

// Within one chunk of 32 consecutive bins (base b0) of which the krem-th
// largest counted key is known to lie in, find that bin with the whole warp:
// lane l holds bin b0 + l, a suffix scan over lanes gives the keys above each
// bin. Returns (bin, rank left inside it, its count) on every lane.
__device__ __forceinline__ void warp_find_in_chunk(const uint32_t* h, int b0, int nb, int krem,
                                                   int* bin, int* kr, int* cnt) {
    const int lane = threadIdx.x & 31;
    const int c = lane < nb ? (int)h[b0 + lane] : 0;
    int suf = c;  // inclusive suffix sum over lanes (higher lanes = higher bins)
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int y = __shfl_down_sync(0xffffffffu, suf, off);
        if (lane + off < 32) suf += y;
    }
    const int above = suf - c;
    const unsigned hit = __ballot_sync(0xffffffffu, lane < nb && above < krem && above + c >= krem);
    const int src = hit ? __ffs(hit) - 1 : 0;  // a hit always exists when the counts hold krem
    *bin = b0 + src;
    *kr = krem - __shfl_sync(0xffffffffu, above, src);
    *cnt = __shfl_sync(0xffffffffu, c, src);
}

// Given per-bin counts in hist[0, nbins) (bins ordered by key), find the bin
// holding the krem-th largest counted key. Thread t owns bins [t*per, (t+1)*per)
// (per <= 32, a power of two) and reads them in a rotated order (bank-conflict
// free); the thread whose range holds the bin hands it to warp 0, which
// searches the range in parallel. Writes the bin, the rank left inside it and
// the bin's count to shared memory (valid after the function returns).
__device__ __forceinline__ void find_bin(const uint32_t* hist, int nbins, int krem, int* buf,
                                         int* s_bin, int* s_krem, int* s_cnt) {
    const int per = nbins / (int)blockDim.x;
    const int b0 = threadIdx.x * per;
    const int rot = threadIdx.x & (per - 1);
    int local = 0;
    for (int i = 0; i < per; ++i) local += (int)hist[b0 + ((i + rot) & (per - 1))];
    int total;
    const int before = block_excl_scan(local, buf, &total);
    const int above = total - before - local;  // keys in bins owned by higher threads
    if (above < krem && above + local >= krem) {
        buf[0] = b0;
        buf[1] = krem - above;
    }
    __syncthreads();
    if (threadIdx.x < 32) {
        int bin, kr, cnt;
        const int cb0 = min(max(buf[0], 0), nbins - per);  // stays inside hist whatever buf holds
        warp_find_in_chunk(hist, cb0, per, buf[1], &bin, &kr, &cnt);
        if (threadIdx.x == 0) {
            *s_bin = bin;
            *s_krem = kr;
            *s_cnt = cnt;
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
#pragma unroll 1
    for (int pass = 0; pass < 2; ++pass) {
        const int shift = pass == 0 ? 10 : 0;
#pragma unroll 8
        for (int i = 0; i < 32; ++i) h[32 * i + lane] = 0u;
        __syncwarp();
        for (int i = lane; i < n; i += 32) {
            const uint32_t c = cand[i];
            if (pass == 0 || ((c >> 10) & 1023u) == hi10) atomicAdd(&h[(c >> shift) & 1023u], 1u);
        }
        __syncwarp();
        int local = 0;
#pragma unroll 8
        for (int i = 0; i < 32; ++i) local += (int)h[32 * lane + ((i + lane) & 31)];
        int suf = local;  // inclusive suffix sum over lanes
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int y = __shfl_down_sync(0xffffffffu, suf, off);
            if (lane + off < 32) suf += y;
        }
        const int above = suf - local;
        const unsigned hit = __ballot_sync(0xffffffffu, above < krem && above + local >= krem);
        const int src = hit ? __ffs(hit) - 1 : 0;
        int bin, kr, cnt;
        warp_find_in_chunk(h, 32 * src, 32, krem - __shfl_sync(0xffffffffu, above, src), &bin, &kr,
                           &cnt);
        krem = kr;
        cnt_sel = cnt;
        if (pass == 0) hi10 = (uint32_t)bin;
        else *low = (hi10 << 10) | (uint32_t)bin;
        __syncwarp();
    }
    *krem_out = krem;
    *cnt_out = cnt_sel;
}

// Scratch of one block-level selection (shared memory).
struct TopkScratch {
    uint32_t* hist;  // 4096 bins, 16-byte aligned
    uint32_t* cand;  // kTopkCandCap keys
    int* scan_buf;   // 32 ints
    int* small;      // 5 ints: bin, rank, count, candidates, threshold
};
constexpr int kTopkCandCap = 2048;

// Selects the k largest of the S keys in keys4 (zero padded to a multiple of
// 4; key 0 never comes from a score) with all NT threads of the block (NT a
// power of two, S <= 32 * NT) and writes their indices in ascending order to
// out[0, k) (global or shared memory). hist must be zero on entry. Ends with
// every thread past its last barrier; the caller synchronises before reusing
// the scratch or reading out.
template <int NT>
__device__ __forceinline__ void topk_block_select(const uint4* keys4, int S, int k, int32_t* out,
                                                  const TopkScratch& sc) {
    constexpr int kCandCap = kTopkCandCap;
    const uint32_t* keys = reinterpret_cast<const uint32_t*>(keys4);
    uint32_t* hist = sc.hist;
    uint32_t* cand = sc.cand;
    int* scan_buf = sc.scan_buf;
    int& s_bin = sc.small[0];
    int& s_krem = sc.small[1];
    int& s_cnt = sc.small[2];
    int& s_ncand = sc.small[3];
    uint32_t& s_T = reinterpret_cast<uint32_t&>(sc.small[4]);
    const int tid = threadIdx.x, lane = tid & 31;
    const int S4 = (S + 3) >> 2;
    if (tid == 0) s_ncand = 0;
    __syncthreads();

    // pass 1: top 12 bits over the whole row (padding keys land in bin 0,
    // below every real key, and never reach the threshold)
#pragma unroll 1
    for (int j = tid; j < S4; j += NT) {
        const uint4 v = keys4[j];
        atomicAdd(&hist[v.x >> 20], 1u);
        atomicAdd(&hist[v.y >> 20], 1u);
        atomicAdd(&hist[v.z >> 20], 1u);
        atomicAdd(&hist[v.w >> 20], 1u);
    }
    __syncthreads();
    find_bin(hist, 4096, k, scan_buf, &s_bin, &s_krem, &s_cnt);
    const uint32_t bin1 = (uint32_t)s_bin;
    int krem = s_krem;
    const int n1 = s_cnt;  // keys in the threshold bin

    uint32_t T;
    int cnt_T;
    if (n1 <= kCandCap) {
        // gather the threshold bin's keys (one shared atomic per warp and
        // step); warp 0 then resolves the low 20 bits
        const int S4r = (S4 + 31) & ~31;
#pragma unroll 1
        for (int j = tid; j < S4r; j += NT) {
            const uint4 v = j < S4 ? keys4[j] : make_uint4(0u, 0u, 0u, 0u);
            const uint32_t kk[4] = {v.x, v.y, v.z, v.w};
            const int mine = ((kk[0] >> 20) == bin1) + ((kk[1] >> 20) == bin1) +
                             ((kk[2] >> 20) == bin1) + ((kk[3] >> 20) == bin1);
            const unsigned any = __ballot_sync(0xffffffffu, mine > 0);
            if (any) {
                int incl = mine;
#pragma unroll
                for (int off = 1; off < 32; off <<= 1) {
                    const int y = __shfl_up_sync(0xffffffffu, incl, off);
                    if (lane >= off) incl += y;
                }
                int base = 0;
                if (lane == 31) base = atomicAdd(&s_ncand, incl);
                base = __shfl_sync(0xffffffffu, base, 31) + incl - mine;
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    if ((kk[e] >> 20) == bin1) cand[base++] = kk[e];
            }
        }
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
#pragma unroll 1
        for (int i = tid; i < 1024; i += NT) hist[i] = 0u;
        __syncthreads();
#pragma unroll 1
        for (int j = tid; j < 4 * S4; j += NT)
            if ((keys[j] >> 20) == bin1) atomicAdd(&hist[(keys[j] >> 10) & 1023u], 1u);
        __syncthreads();
        find_bin(hist, 1024, krem, scan_buf, &s_bin, &s_krem, &s_cnt);
        const uint32_t pre2 = (bin1 << 10) | (uint32_t)s_bin;
        krem = s_krem;
        __syncthreads();
#pragma unroll 1
        for (int i = tid; i < 1024; i += NT) hist[i] = 0u;
        __syncthreads();
#pragma unroll 1
        for (int j = tid; j < 4 * S4; j += NT)
            if ((keys[j] >> 10) == pre2) atomicAdd(&hist[keys[j] & 1023u], 1u);
        __syncthreads();
        find_bin(hist, 1024, krem, scan_buf, &s_bin, &s_krem, &s_cnt);
        T = (pre2 << 10) | (uint32_t)s_bin;
        krem = s_krem;
        cnt_T = s_cnt;
    }
    // T is the k-th largest key; krem of the cnt_T keys equal to T are taken,
    // lowest indices first. Thread t owns the q4 uint4 groups [t*q4, t*q4 + q4)
    // (4*q4 <= 32 keys), read in a rotated order into bit masks.
    const int q4 = (S4 + NT - 1) / NT;
    const int g0 = tid * q4;
    const int ng = max(0, min(q4, S4 - g0));
    const bool pow2 = (q4 & (q4 - 1)) == 0;
    uint32_t gtm = 0u, eqm = 0u;
    const int nloop = pow2 ? q4 : ng;
#pragma unroll 1
    for (int i = 0; i < nloop; ++i) {
        const int ii = pow2 ? ((i + tid) & (q4 - 1)) : i;
        if (ii < ng) {
            const uint4 v = keys4[g0 + ii];
            const uint32_t kk[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                gtm |= (uint32_t)(kk[e] > T) << (4 * ii + e);
                eqm |= (uint32_t)(kk[e] == T) << (4 * ii + e);
            }
        }
    }
    const int gt = __popc(gtm), eq = __popc(eqm);
    int total, take_eq;
    if (krem == cnt_T) {
        take_eq = eq;  // every key equal to T is selected: no tie scan needed
    } else {
        const int eq_before = block_excl_scan(eq, scan_buf, &total);
        take_eq = max(0, min(eq, krem - eq_before));
    }
    int pos = block_excl_scan(gt + take_eq, scan_buf, &total);
    // keys equal to T beyond the first take_eq (in index order) are dropped
    uint32_t em = eqm;
    for (int t = 0; t < take_eq; ++t) em &= em - 1u;
    uint32_t take = gtm | (eqm & ~em);
    int32_t* o = out;
    const int j0 = 4 * g0;
#pragma unroll 1
    while (take) {
        const int ii = __ffs(take) - 1;
        take &= take - 1u;
        if (pos < k) o[pos] = j0 + ii;  // pos < k by construction; the bound keeps writes in the row
        ++pos;
    }
}

}  // namespace loki
