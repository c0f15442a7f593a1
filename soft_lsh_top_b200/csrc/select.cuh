// Block-wide selection helpers (512-thread CTAs): prefix sums, radix digits
// over bit patterns, and the compaction of a selection in index order.  Used
// by the top-k kernel and by the merge of sharded selections.
#pragma once

#include "common.cuh"

namespace socket_attn {
namespace select512 {

constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;
constexpr int kBins = 2048;  // radix bins of a digit pass

struct Shared {
    uint32_t warp_sums[kWarps];
    uint32_t digit, krem, last;
    uint32_t count;  // keys in the bin found by the last digit; candidates of this CTA during the read
    uint32_t base;   // offset of this CTA's candidates in the unit list
    uint32_t bin_count;  // keys in the bin find_bin found
    __align__(16) uint32_t hist[kBins];
};

// Block-wide exclusive prefix sum of one uint32 per thread; also returns the total.
__device__ __forceinline__ uint32_t block_exclusive_scan(uint32_t v, uint32_t* warp_sums, uint32_t& total)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    uint32_t x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(kFullMask, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) warp_sums[warp] = x;
    __syncthreads();
    if (warp == 0) {
        uint32_t w = lane < kWarps ? warp_sums[lane] : 0u;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t y = __shfl_up_sync(kFullMask, w, o);
            if (lane >= o) w += y;
        }
        if (lane < kWarps) warp_sums[lane] = w;  // inclusive over warps
    }
    __syncthreads();
    total = warp_sums[kWarps - 1];
    const uint32_t before = warp == 0 ? 0u : warp_sums[warp - 1];
    const uint32_t excl = before + x - v;
    __syncthreads();  // warp_sums reusable after return
    return excl;
}

// Over bins given in descending order as per-thread runs c[0..NB) (thread
// t's run precedes thread t+1's), finds the bin holding the krem-th key from
// the top: writes its id (bin_of(q)) to sh.digit, the keys still needed
// inside it to sh.krem and the keys it holds to sh.bin_count.  Every thread
// must call it; sh is valid after the next barrier.
template <int NB, typename BinOf>
__device__ __forceinline__ void find_bin(const uint32_t (&c)[NB], uint32_t krem, Shared& sh, BinOf bin_of)
{
    uint32_t sum = 0;
#pragma unroll
    for (int q = 0; q < NB; ++q) sum += c[q];
    uint32_t total;
    uint32_t run = block_exclusive_scan(sum, sh.warp_sums, total);
#pragma unroll
    for (int q = 0; q < NB; ++q) {
        if (run < krem && krem <= run + c[q]) {
            sh.digit = bin_of(q);
            sh.krem = krem - run;
            sh.bin_count = c[q];
        }
        run += c[q];
    }
}

// One radix digit over `n` values produced by get(i) (bit pattern), counting
// only those with (x & mask) == prefix, digit (x >> shift) & dmask (<= 2048
// bins).  Updates prefix / mask / krem to the bin of the krem-th largest
// (descending == true) or smallest value.
template <typename Get>
__device__ __forceinline__ void radix_digit(Shared& sh, int n, Get get, int shift, uint32_t dmask, bool descending,
                                            uint32_t& prefix, uint32_t& mask, uint32_t& krem)
{
    const int tid = threadIdx.x;
    for (int b = tid; b < kBins; b += kThreads) sh.hist[b] = 0;
    if (tid == 0) {  // kept if no bin holds the krem-th value (inconsistent input)
        sh.digit = 0;
        sh.krem = krem;
    }
    __syncthreads();
    for (int i = tid; i < n; i += kThreads) {
        const uint32_t x = get(i);
        if ((x & mask) == prefix) atomicAdd(&sh.hist[(x >> shift) & dmask], 1u);
    }
    __syncthreads();
    constexpr int kPer = kBins / kThreads;  // 4 bins per thread
    uint32_t c[kPer];
    int bins[kPer];
#pragma unroll
    for (int q = 0; q < kPer; ++q) {
        bins[q] = descending ? kBins - 1 - (kPer * tid + q) : kPer * tid + q;
        c[q] = sh.hist[bins[q]];
    }
    find_bin<kPer>(c, krem, sh, [&](int q) { return (uint32_t)bins[q]; });
    __syncthreads();
    if (threadIdx.x == 0) sh.count = sh.hist[sh.digit];
    __syncthreads();
    prefix |= sh.digit << shift;
    mask |= dmask << shift;
    krem = sh.krem;
    __syncthreads();
}

// Writes the selection from a pass over the scores: keys of [0, n) above t,
// plus the first `budget` keys equal to t, in index order.
__device__ inline void compact_scores(const uint32_t* su, int n, uint32_t t, uint32_t budget, int k, int32_t* out,
                               Shared& sh)
{
    constexpr int kPer = 16;  // consecutive keys per thread and tile
    const int tid = threadIdx.x;
    uint32_t out_base = 0, ties_seen = 0;
    for (int tile = 0; tile < n; tile += kThreads * kPer) {
        const int i0 = tile + tid * kPer;
        uint32_t vals[kPer];
#pragma unroll
        for (int q = 0; q < kPer / 4; ++q) {
            uint4 v = make_uint4(0, 0, 0, 0);
            if (i0 + 4 * q < n) v = __ldcg(reinterpret_cast<const uint4*>(su + i0 + 4 * q));
            vals[4 * q] = v.x;
            vals[4 * q + 1] = v.y;
            vals[4 * q + 2] = v.z;
            vals[4 * q + 3] = v.w;
        }
        uint32_t gt = 0, eq = 0;
#pragma unroll
        for (int e = 0; e < kPer; ++e)
            if (i0 + e < n) {
                gt += vals[e] > t;
                eq += vals[e] == t;
            }
        uint32_t tot_gt, tot_eq;
        const uint32_t gt_before = block_exclusive_scan(gt, sh.warp_sums, tot_gt);
        const uint32_t eq_before = block_exclusive_scan(eq, sh.warp_sums, tot_eq);
        const uint32_t left = budget > ties_seen ? budget - ties_seen : 0u;
        uint32_t pos = out_base + gt_before + min(eq_before, left);
        uint32_t my_eq = eq_before;
#pragma unroll
        for (int e = 0; e < kPer; ++e) {
            if (i0 + e >= n) continue;
            const bool take = vals[e] > t || (vals[e] == t && my_eq < left);
            my_eq += vals[e] == t;
            // pos < k whenever the threshold is exact; the guard keeps every
            // store inside the unit's k slots regardless.
            if (take) {
                if (pos < (uint32_t)k) out[pos] = i0 + e;
                ++pos;
            }
        }
        out_base += tot_gt + min(tot_eq, left);
        ties_seen += tot_eq;
    }
}

}  // namespace select512
}  // namespace socket_attn
