// Exact top-k selection over order-preserving 32-bit keys held in registers
// (Loki's token selection: NeurIPS 2024 poster page, TL;DR and "Visual
// Insights" Figure 1 caption -- keep the k tokens with the largest approximate
// scores). Shared by the standalone top-k kernel (topk.cu) and the fused
// decode kernel (decode_fused.cu).
//
// Scores become order-preserving keys (larger float -> larger key; -0 folded
// onto +0; NaN folded onto -inf; key 0 marks padding and never counts). A
// most-significant-digit radix select finds the k-th largest key T in three
// passes over the digits 31..21, 20..10 and 9..0 (2048, 2048 and 1024 bins):
// each pass adds every key that still matches the known prefix into a
// shared-memory histogram (fire-and-forget atomics from registers), and a
// scan over the bins (block-wide, or in one warp when several CTAs share the
// SM) finds the bin holding the k-th key. That also gives how many keys equal
// to T belong to the set (ties go to the lowest token indices). A pass whose
// threshold bin is taken whole ends the search early (for continuous scores
// the 22-bit prefix of pass 2 almost always isolates the k-th key, so pass 3
// rarely runs). A compaction then writes the selected indices in ascending
// token order: each warp scans its lanes' per-step counts packed as 8-bit
// fields, and warp and CTA prefixes place every key. Every decision is an
// integer compare, so the result is exact and deterministic.
//
// Key layout: thread (warp w, lane) holds I uint4 groups of 4 keys in
// registers; its group i is group w * 32 I + 32 i + lane of the CTA, so every
// step of a warp covers 128 consecutive keys (coalesced loads) and key order
// is (warp, step, lane, element).
//
// A row may be split over the CTAs of a thread-block cluster: CTA r holds
// keys [r * chunk, r * chunk + n). Each pass then sums the cluster's
// histograms through distributed shared memory (every CTA reads all copies
// for its share of bins, so all CTAs reach the same decisions), and the
// compaction adds the counts of the lower-ranked CTAs. Without a cluster
// (kCl = false) the same code runs with block barriers only.
#pragma once

#include <cooperative_groups.h>

#include "common.cuh"

namespace loki {

namespace cg = cooperative_groups;

__device__ __forceinline__ uint32_t order_key(float x) {
    // fmaxf with -inf turns NaN into -inf (IEEE maxNum returns the operand
    // that is a number); adding +0 turns -0 into +0
    const uint32_t u = __float_as_uint(fmaxf(x, -INFINITY) + 0.0f);
    // negative: all bits flipped; positive: the sign bit set
    return u ^ ((uint32_t)((int32_t)u >> 31) | 0x80000000u);
}
// (no score maps to key 0: -inf maps to 0x007fffff, so every real key lies in
// bin 3 or above of the first digit and a threshold never admits padding)

constexpr int kTkBins1 = 2048;  // digit 1: key bits 31..21
constexpr int kTkBins2 = 2048;  // digit 2: key bits 20..10
constexpr int kTkBins3 = 1024;  // digit 3: key bits 9..0
constexpr int kTkMaxKeysPerThread = 32;

// Shared-memory scratch of one selection: the histograms and 64 words of
// reduction slots. The third histogram reuses the first one's words (cleared
// once the first pass's bin search is over), so the scratch stays small
// enough for five 256-thread top-k CTAs per SM.
struct TkSmem {
    uint32_t* hist1;
    uint32_t* hist2;
    uint32_t* hist3;
    int* red;
};
constexpr int kTkSmemWords = kTkBins1 + kTkBins2 + 64;
static_assert(kTkBins3 <= kTkBins1, "the third histogram lives in the first");

// red[] slots (0..31: per-warp partial sums)
constexpr int kRedBin = 32, kRedKrem = 33, kRedCnt = 34, kRedTotal = 35;

__device__ __forceinline__ TkSmem tk_carve(uint32_t* base) {
    TkSmem s;
    s.hist1 = base;
    s.hist2 = base + kTkBins1;
    s.hist3 = base;
    s.red = reinterpret_cast<int*>(s.hist2 + kTkBins2);
    return s;
}

// Zero the histograms (all threads of the block; visible after the next
// barrier).
template <int NT>
__device__ __forceinline__ void tk_zero(const TkSmem& sm) {
    constexpr int n4 = (kTkBins1 + kTkBins2) / 4;
    for (int i = threadIdx.x; i < n4; i += NT)
        reinterpret_cast<uint4*>(sm.hist1)[i] = make_uint4(0u, 0u, 0u, 0u);
}

// The CTA's place in its cluster (rank 0 of 1 without one), and the block
// barrier of the selecting threads: __syncthreads() (kBar = 0), or named
// barrier kBar over the first kBarThreads threads of the block when the
// selection runs on a subset of its warps.
template <bool kCl, int kBar = 0, int kBarThreads = 0>
struct TkCluster {
    int rank = 0, size = 1;
    __device__ __forceinline__ void bsync() const {
        if constexpr (kBar == 0) __syncthreads();
        else asm volatile("bar.sync %0, %1;" ::"n"(kBar), "n"(kBarThreads) : "memory");
    }
    __device__ __forceinline__ void init() {
        if constexpr (kCl) {
            cg::cluster_group c = cg::this_cluster();
            rank = (int)c.block_rank();
            size = (int)c.num_blocks();
        }
    }
    __device__ __forceinline__ void sync() const {
        if constexpr (kCl) cg::this_cluster().sync();
        else bsync();
    }
    // the copy of a shared-memory object in the CTA of rank r
    template <class T>
    __device__ __forceinline__ T* at(T* p, int r) const {
        if constexpr (kCl) return cg::this_cluster().map_shared_rank(p, r);
        else return p;
    }
};
constexpr int kTkMaxCluster = 8;

// Sum of v over the lanes above this one (exclusive suffix), and the warp total.
__device__ __forceinline__ int warp_suffix_excl(int v, int* total) {
    const int lane = threadIdx.x & 31;
    int x = v;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int y = __shfl_down_sync(0xffffffffu, x, off);
        if (lane + off < 32) x += y;
    }
    *total = __shfl_sync(0xffffffffu, x, 0);
    return x - v;
}

// Inclusive scan over the lanes of a word of packed counters (the fields
// must not overflow).
__device__ __forceinline__ uint32_t warp_incl_scan(uint32_t x) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, x, off);
        if (lane >= off) x += y;
    }
    return x;
}

// Sum of v over all warps before this one (and over all warps), through
// red[0, NW); ends with every thread past one block barrier.
template <int NT, class CL>
__device__ __forceinline__ int block_warp_prefix(const CL& cl, int v, int* red, int* all) {
    constexpr int NW = NT / 32;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    if (lane == 0) red[warp] = v;
    cl.bsync();
    int lo = (lane < warp) ? red[lane] : 0;
    int tot = (lane < NW) ? red[lane] : 0;
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) {
        lo += __shfl_xor_sync(0xffffffffu, lo, off);
        tot += __shfl_xor_sync(0xffffffffu, tot, off);
    }
    *all = tot;
    return lo;
}

// Given the per-bin counts of this CTA's `hist` (NB bins ordered by key,
// 1 <= krem <= their total), warp 0 alone finds the bin holding the krem-th
// largest counted key in two levels: lane l sums bins [l * PER, (l + 1) * PER)
// (reading its 16-byte chunks in a lane-rotated order, so the 8 lanes of a
// quarter-warp hit distinct banks) and a suffix scan over the lanes finds the
// block; then lane j takes bins [j * Q, (j + 1) * Q) of that block. The bin,
// the rank left inside it and its count go to red[] and are valid for every
// thread on return; the caller has made hist complete (block barrier).
template <int NB, class CL>
__device__ __forceinline__ void tk_find_bin_warp(const CL& cl, const uint32_t* hist, int krem,
                                                 int* red) {
    constexpr int PER = NB / 32;  // 64 or 32
    constexpr int NV = PER / 4;   // 16-byte chunks per lane
    constexpr int Q = PER / 32;   // bins per lane in the second level
    static_assert(NB % 1024 == 0 && Q >= 1, "bins");
    if (threadIdx.x < 32) {
        const int lane = threadIdx.x;
        const uint4* h4 = reinterpret_cast<const uint4*>(hist) + lane * NV;
        uint32_t s0 = 0u, s1 = 0u, s2 = 0u, s3 = 0u;
        // two chunks in flight: the selecting threads still hold their keys
#pragma unroll 2
        for (int v = 0; v < NV; ++v) {
            const uint4 x = h4[(v + lane) & (NV - 1)];
            s0 += x.x;
            s1 += x.y;
            s2 += x.z;
            s3 += x.w;
        }
        const int local = (int)(s0 + s1 + s2 + s3);
        int tot;
        const int above = warp_suffix_excl(local, &tot);  // keys in higher lanes' blocks
        const uint32_t m = __ballot_sync(0xffffffffu, above < krem && above + local >= krem);
        const int L = m ? __ffs(m) - 1 : 0;  // one lane by construction
        const int aboveL = __shfl_sync(0xffffffffu, above, L);
        const uint32_t* hb = hist + L * PER + lane * Q;
        uint32_t c[Q];
        int loc2 = 0;
#pragma unroll
        for (int e = 0; e < Q; ++e) {
            c[e] = hb[e];
            loc2 += (int)c[e];
        }
        int tot2;
        const int above2 = aboveL + warp_suffix_excl(loc2, &tot2);
        if (above2 < krem && above2 + loc2 >= krem) {
            int cum = above2;
            bool found = false;
#pragma unroll
            for (int e = Q - 1; e >= 0; --e) {
                if (!found && cum + (int)c[e] >= krem) {
                    red[kRedBin] = L * PER + lane * Q + e;
                    red[kRedKrem] = krem - cum;
                    red[kRedCnt] = (int)c[e];
                    found = true;
                }
                cum += (int)c[e];
            }
        }
    }
    cl.bsync();
}

// Given per-bin counts summed over the cluster's copies of `hist` (NB bins,
// ordered by key), find the bin holding the krem-th largest counted key.
// Thread t owns bins [t * PER, (t + 1) * PER) and keeps their sums in
// registers. The bin, the rank left inside it and its cluster count go to
// red[] and are valid for every thread on return. The caller has made every
// copy of hist complete and visible (block or cluster barrier). With kWarp
// (one CTA) the one-warp search above runs instead.
template <int NT, int NB, bool kCl, class CL, bool kWarp = false>
__device__ __forceinline__ void tk_find_bin(const CL& cl, const uint32_t* hist, int krem, int* red) {
    if constexpr (kWarp && !kCl) {
        tk_find_bin_warp<NB, CL>(cl, hist, krem, red);
        return;
    }
    constexpr int PER = NB / NT;  // 1..16
    static_assert(PER >= 1 && NB % NT == 0, "bins per thread");
    constexpr int NW = NT / 32;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int b0 = tid * PER;
    uint32_t c[PER];
#pragma unroll
    for (int e = 0; e < PER; ++e) c[e] = 0u;
#pragma unroll
    for (int r = 0; r < (kCl ? kTkMaxCluster : 1); ++r) {
        if (r < cl.size) {
            const uint32_t* h = cl.at(hist, r) + b0;
            if constexpr (PER % 4 == 0) {
#pragma unroll
                for (int v = 0; v < PER / 4; ++v) {
                    const uint4 x = reinterpret_cast<const uint4*>(h)[v];
                    c[4 * v] += x.x;
                    c[4 * v + 1] += x.y;
                    c[4 * v + 2] += x.z;
                    c[4 * v + 3] += x.w;
                }
            } else {
#pragma unroll
                for (int e = 0; e < PER; ++e) c[e] += h[e];
            }
        }
    }
    int local = 0;
#pragma unroll
    for (int e = 0; e < PER; ++e) local += (int)c[e];
    // keys in bins owned by higher threads
    int wtot;
    const int in_warp_above = warp_suffix_excl(local, &wtot);
    if (lane == 0) red[warp] = wtot;
    cl.bsync();
    int hi = (lane > warp && lane < NW) ? red[lane] : 0;
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) hi += __shfl_xor_sync(0xffffffffu, hi, off);
    const int above = hi + in_warp_above;
    if (above < krem && above + local >= krem) {
        // this thread's range holds the bin: walk its registers from the top
        int cum = above;
        bool found = false;
#pragma unroll
        for (int e = PER - 1; e >= 0; --e) {
            if (!found && cum + (int)c[e] >= krem) {
                red[kRedBin] = b0 + e;
                red[kRedKrem] = krem - cum;
                red[kRedCnt] = (int)c[e];
                found = true;
            }
            cum += (int)c[e];
        }
    }
    cl.bsync();
}

// Selects the k largest keys of a row and writes their global indices in
// ascending order to out[0, k) (global or shared memory).
//   v      this thread's I groups of keys (layout above); padding keys are 0
//   base   global index of the CTA's first key (rank * chunk in a cluster)
//   sm     scratch: hist1 holds this CTA's histogram of key bits 31..21 over
//          its keys, hist2 is zero (the call's first barrier publishes
//          them; hist3 shares hist1's words and is cleared here)
//   k      1 <= k <= the row's number of keys
// Every thread of every CTA of the cluster must call it. On return every
// thread is past its last barrier (in a cluster: past a final cluster
// barrier, so no CTA's shared memory is still read by another).
// kWarpFind: the bin searches run in one warp (fewer instructions, more
// latency: for CTAs that share their SM with several others).
template <int NT, int I, bool kCl, int kBar = 0, bool kWarpFind = false>
__device__ __forceinline__ void tk_select(const TkCluster<kCl, kBar, (kBar ? NT : 0)>& cl,
                                          const uint4 (&v)[I], int base, int k, int32_t* out,
                                          const TkSmem& sm) {
    using CL = TkCluster<kCl, kBar, (kBar ? NT : 0)>;
    static_assert(I == 1 || I == 2 || I == 4 || I == 8, "groups per thread");
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    int* red = sm.red;
    // every CTA's pass-1 histogram is complete
    cl.sync();
    tk_find_bin<NT, kTkBins1, kCl, CL, kWarpFind>(cl, sm.hist1, k, red);
    const uint32_t bin1 = (uint32_t)red[kRedBin];
    int krem = red[kRedKrem];
    // A pass whose threshold bin is taken whole ends the search: the set is
    // then every key at or above the bin's lowest key, with no tie to break.
    // The counts are the cluster's, so every thread takes the same branch.
    // lo: that lowest key; T, take_T, cnt_T: the exact threshold of pass 3.
    uint32_t lo = 0u, T = 0u;
    int take_T = 0, cnt_T = 0;
    bool whole = krem == red[kRedCnt];
    if (whole) {
        lo = bin1 << 21;
    } else {
        // pass 2: bits 20..10 of the keys in the threshold bin
#pragma unroll
        for (int i = 0; i < I; ++i) {
            const uint32_t kk[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
#pragma unroll
            for (int e = 0; e < 4; ++e)
                if ((kk[e] >> 21) == bin1)
                    atomicAdd(&sm.hist2[(kk[e] >> 10) & 2047u], 1u);
        }
        cl.sync();
        // no CTA of the cluster reads the pass-1 histograms any more: clear
        // the words pass 3 counts into (the bin search's barriers publish it)
        for (int i = tid; i < kTkBins3 / 4; i += NT)
            reinterpret_cast<uint4*>(sm.hist3)[i] = make_uint4(0u, 0u, 0u, 0u);
        tk_find_bin<NT, kTkBins2, kCl, CL, kWarpFind>(cl, sm.hist2, krem, red);
        const uint32_t pre = (bin1 << 11) | (uint32_t)red[kRedBin];
        krem = red[kRedKrem];
        whole = krem == red[kRedCnt];
        if (whole) {
            lo = pre << 10;
        } else {
            // pass 3: bits 9..0 of the keys sharing the 22-bit prefix
#pragma unroll
            for (int i = 0; i < I; ++i) {
                const uint32_t kk[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    if ((kk[e] >> 10) == pre) atomicAdd(&sm.hist3[kk[e] & 1023u], 1u);
            }
            cl.sync();
            tk_find_bin<NT, kTkBins3, kCl, CL, kWarpFind>(cl, sm.hist3, krem, red);
            T = (pre << 10) | (uint32_t)red[kRedBin];
            take_T = red[kRedKrem];  // keys equal to T in the set (the lowest-index ones)
            cnt_T = red[kRedCnt];    // keys equal to T in the row
        }
    }

    // ---- compaction ----------------------------------------------------------
    // per-thread masks: bit 4 i + e is element e of group i (padding keys, 0,
    // are never selected)
    uint32_t gtm = 0u, eqm = 0u;
#pragma unroll
    for (int i = 0; i < I; ++i) {
        const uint32_t kk[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            if (whole) {
                gtm |= (uint32_t)(kk[e] >= lo) << (4 * i + e);
            } else {
                gtm |= (uint32_t)(kk[e] > T) << (4 * i + e);
                eqm |= (uint32_t)(kk[e] == T) << (4 * i + e);
            }
        }
    }
    // packed per-step counts: field i (8 bits) of word i / 4; a field sums at
    // most 4 x 32 = 128 over the warp
    constexpr int NWD = (I + 3) / 4;
    auto pack = [&](uint32_t m, uint32_t (&w)[NWD]) {
#pragma unroll
        for (int j = 0; j < NWD; ++j) w[j] = 0u;
#pragma unroll
        for (int i = 0; i < I; ++i) w[i / 4] |= (uint32_t)__popc((m >> (4 * i)) & 15u) << (8 * (i % 4));
    };
    // exclusive position of each step's first key in the warp's order
    // (earlier steps of every lane, then earlier lanes of the same step);
    // returns the warp total
    auto warp_positions = [&](uint32_t m, int (&pos)[I]) -> int {
        uint32_t w[NWD], inc[NWD];
        pack(m, w);
#pragma unroll
        for (int j = 0; j < NWD; ++j) inc[j] = warp_incl_scan(w[j]);
        int run = 0;
#pragma unroll
        for (int i = 0; i < I; ++i) {
            const int sh = 8 * (i % 4);
            const int excl = (int)(((inc[i / 4] - w[i / 4]) >> sh) & 255u);
            const int tot = (int)((__shfl_sync(0xffffffffu, inc[i / 4], 31) >> sh) & 255u);
            pos[i] = run + excl;
            run += tot;
        }
        return run;
    };
    auto cluster_prefix = [&](int cta_total, int slot) -> int {
        int add = 0;
        if constexpr (kCl) {
            if (tid == 0) red[slot] = cta_total;
            cl.sync();
            for (int r = 0; r < cl.rank; ++r) add += cl.at(red, r)[slot];
        }
        (void)cta_total;
        (void)slot;
        return add;
    };
    uint32_t sel = gtm | eqm;
    if (take_T < cnt_T) {
        // only the first take_T keys equal to T (in index order) are kept
        int epos[I];
        const int wtot = warp_positions(eqm, epos);
        int all;
        const int wpre = block_warp_prefix<NT>(cl, wtot, red, &all);
        const int before = wpre + cluster_prefix(all, kRedTotal);
        uint32_t keep = 0u;
#pragma unroll
        for (int i = 0; i < I; ++i) {
            const uint32_t g = (eqm >> (4 * i)) & 15u;
            int rank = before + epos[i];
#pragma unroll
            for (int e = 0; e < 4; ++e)
                if ((g >> e) & 1u) {
                    if (rank < take_T) keep |= 1u << (4 * i + e);
                    ++rank;
                }
        }
        sel = gtm | keep;
        cl.bsync();  // red[0, NW) is reused below
    }
    int spos[I];
    const int wtot = warp_positions(sel, spos);
    int all;
    const int wpre = block_warp_prefix<NT>(cl, wtot, red, &all);
    const int before = wpre + cluster_prefix(all, kRedTotal + 1);
    const int gw = warp * 32 * I + lane;
#pragma unroll
    for (int i = 0; i < I; ++i) {
        uint32_t g = (sel >> (4 * i)) & 15u;
        int p = before + spos[i];
        const int j0 = base + 4 * (gw + 32 * i);
        while (g) {
            const int e = __ffs(g) - 1;
            g &= g - 1u;
            if (p < k) out[p] = j0 + e;  // p < k by construction; the bound keeps writes in the row
            ++p;
        }
    }
    // no CTA leaves while another may still read its shared memory
    if constexpr (kCl) cl.sync();
}

}  // namespace loki
