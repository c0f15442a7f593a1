// Deterministic top-k selection of every unit's keys by soft score.
//
// Method: "Resumen Técnico: SOCKET ..." (gist.science/es/paper/2602.06283),
// "Mecanismo Central: LSH Suave" step 4 "Selección" and "Contribuciones
// Clave" 1 (stable top-k selection with no ad-hoc voting); "SOCKET: SOft
// Collision Kernel EsTimator for Sparse Attention"
// (gist.science/de/paper/2602.06283), "Auswahl".  The k keys with the
// largest scores are chosen deterministically; equal scores go to the lower
// index, and the chosen indices are written in ascending order.
//
// Scores are non-negative float32, so their bit patterns order like the
// values.  The selection finds the bit pattern t of the k-th largest score
// and the number of keys equal to t to keep (the lowest-index ones), then
// writes every key above t and those ties in index order.  A unit is handled
// by a thread-block cluster of up to 16 CTAs that exchange counts through
// distributed shared memory; the paths are described at the kernel.
#include <cooperative_groups.h>

#include "common.cuh"
#include "internal.h"

namespace cg = cooperative_groups;

namespace socket_attn {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kBins = 2048;                           // radix bins of the multi-pass path
constexpr int kKeysPerThread = 16;                    // compaction: 16 consecutive keys per thread
constexpr int kTileKeys = kThreads * kKeysPerThread;  // 4096
constexpr int kSliceKeys = 32768;                     // target keys per CTA of a cluster
constexpr int kBatch = 8;                             // 16-byte loads in flight per thread
constexpr int kMaxCluster = 16;
constexpr int kWindowShift = 15;                      // multi-pass first digit: 2^15 ulps (1/256 octave)
constexpr int kCand = kTopkCandidates;
constexpr int kBitmapKeys = 65536;                    // fast path compacts from a bitmap of up to this many keys
constexpr int kBitmapWords = kBitmapKeys / 32;

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

struct Shared {
    uint32_t warp_sums[32];
    uint32_t digit, krem, sure, total, pick, pick_above, grand;
    uint32_t counts[2];
    uint32_t nlocal, local_base;  // this CTA's candidates, and their offset in the unit list
    __align__(16) uint32_t hist[kBins];
    union {  // the multi-pass path uses `slice`, the candidate path `cand`
        __align__(16) uint32_t slice[kBins];
        uint2 cand[kCand];  // (global index, bit pattern) of the unit's candidates
    };
    // Candidate path: bit i set for key lo + i of the slice if it is selected
    // (first every key in or above the threshold bin, then pruned).
    __align__(16) uint32_t bits[kBitmapWords];
};

// Finds, over bins given in descending order as per-thread runs of `nb`
// counts c[0..nb) (thread t's run precedes thread t+1's), the bin holding the
// krem-th key from the top: writes (bin id via `bin_of(t, q)`, keys still
// needed inside it) to sh.digit / sh.krem.  `above` is the count above all bins.
template <int NB, typename BinOf>
__device__ __forceinline__ void find_bin(const uint32_t (&c)[NB], uint32_t above, uint32_t krem, Shared& sh,
                                         BinOf bin_of)
{
    uint32_t sum = 0;
#pragma unroll
    for (int q = 0; q < NB; ++q) sum += c[q];
    uint32_t total;
    uint32_t run = above + block_exclusive_scan(sum, sh.warp_sums, total);
#pragma unroll
    for (int q = 0; q < NB; ++q) {
        if (run < krem && krem <= run + c[q]) {
            sh.digit = bin_of(q);
            sh.krem = krem - run;
        }
        run += c[q];
    }
}

// Writes this CTA's selected indices (keys of [lo, hi) above t, plus the first
// `budget` keys equal to t) in index order from position out_base.
__device__ __forceinline__ void load_tile(uint32_t (&vals)[kKeysPerThread], const uint32_t* su, int lo, int n, int i0)
{
#pragma unroll
    for (int q = 0; q < kKeysPerThread / 4; ++q) {
        uint4 v = make_uint4(0, 0, 0, 0);
        if (i0 + 4 * q < n) v = __ldcg(reinterpret_cast<const uint4*>(su + lo + i0 + 4 * q));
        vals[4 * q + 0] = v.x;
        vals[4 * q + 1] = v.y;
        vals[4 * q + 2] = v.z;
        vals[4 * q + 3] = v.w;
    }
}

// Writes this CTA's selected indices (keys of [lo, hi) above t, plus the first
// `budget` keys equal to t) in index order from position out_base.  Each
// tile's loads are issued before the previous tile's scan.
__device__ __forceinline__ void compact(const uint32_t* su, int lo, int hi, uint32_t t, uint32_t budget,
                                        uint32_t out_base, int k, int32_t* out, Shared& sh)
{
    const int tid = threadIdx.x;
    const int n = hi - lo;
    uint32_t ties_seen = 0;
    uint32_t vals[kKeysPerThread];
    load_tile(vals, su, lo, n, tid * kKeysPerThread);
    for (int tile = 0; tile < n; tile += kTileKeys) {
        const int i0 = tile + tid * kKeysPerThread;
        uint32_t next[kKeysPerThread];
        if (tile + kTileKeys < n) load_tile(next, su, lo, n, i0 + kTileKeys);
        uint32_t tgt = 0, teq = 0;
#pragma unroll
        for (int e = 0; e < kKeysPerThread; ++e) {
            if (i0 + e < n) {
                tgt += vals[e] > t;
                teq += vals[e] == t;
            }
        }
        uint32_t total;
        const uint32_t excl = block_exclusive_scan((tgt << 16) | teq, sh.warp_sums, total);
        const uint32_t gt_before = excl >> 16, eq_before = excl & 0xffffu;
        const uint32_t left = budget > ties_seen ? budget - ties_seen : 0u;
        uint32_t pos = out_base + gt_before + min(eq_before, left);
        uint32_t my_eq = eq_before;
#pragma unroll
        for (int e = 0; e < kKeysPerThread; ++e) {
            if (i0 + e < n) {
                // pos < k always holds when the threshold is exact; the guard keeps
                // every store inside the unit's k slots regardless.
                if (vals[e] > t) {
                    if (pos < (uint32_t)k) out[pos] = lo + i0 + e;
                    ++pos;
                } else if (vals[e] == t) {
                    if (my_eq < left) {
                        if (pos < (uint32_t)k) out[pos] = lo + i0 + e;
                        ++pos;
                    }
                    ++my_eq;
                }
            }
        }
        out_base += (total >> 16) + min(total & 0xffffu, left);
        ties_seen += total & 0xffffu;
#pragma unroll
        for (int e = 0; e < kKeysPerThread; ++e) vals[e] = next[e];
    }
}

// Multi-pass radix select over the cluster (any score distribution): three
// digits of the bit pattern; the first covers the 8 octaves below the unit's
// largest score in 2048 bins of 1/256 octave, redone over the full range
// (bits 30-20) if fewer than k keys fall in that window.  Histograms are
// combined through distributed shared memory: CTA r sums the r-th 1/C of the
// bins over the cluster, the slice totals locate the slice holding the k-th
// key, and every CTA scans that slice, so all pick the same digit.
// Returns the threshold pattern t and the ties at t to keep in *need.
__device__ uint32_t select_multipass(cg::cluster_group& cluster, const uint32_t* su, int lo, int hi,
                                     uint32_t maxbits, int k, Shared& sh, uint32_t* need)
{
    const unsigned rank = cluster.block_rank(), C = cluster.num_blocks();
    const int tid = threadIdx.x;
    const int n = hi - lo;
    const uint32_t dmax = maxbits >> kWindowShift;
    const uint32_t dlow = dmax >= (uint32_t)(kBins - 1) ? dmax - (kBins - 1) : 0u;
    bool windowed = true;
    uint32_t prefix = 0, mask = 0, krem = (uint32_t)k;
    for (int pass = 0; pass < 3; ++pass) {
        int shift, width;
        if (windowed) {
            shift = pass == 0 ? kWindowShift : pass == 1 ? 4 : 0;
            width = pass == 0 ? 17 : pass == 1 ? 11 : 4;
        } else {
            shift = pass == 0 ? 20 : pass == 1 ? 9 : 0;
            width = pass == 0 ? 11 : pass == 1 ? 11 : 9;
        }
        const uint32_t dmask = (1u << width) - 1u;
        for (int b = tid; b < kBins; b += kThreads) sh.hist[b] = 0;
        __syncthreads();
        for (int i = tid * 4; i < n; i += kThreads * 4) {
            const uint4 v = __ldcg(reinterpret_cast<const uint4*>(su + lo + i));
            const uint32_t vals[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                if (i + e < n) {
                    const uint32_t x = vals[e];
                    if (pass == 0 && windowed) {
                        const uint32_t dgt = x >> kWindowShift;
                        if (dgt >= dlow) atomicAdd(&sh.hist[min(dgt - dlow, (uint32_t)(kBins - 1))], 1u);
                    } else if ((x & mask) == prefix) {
                        atomicAdd(&sh.hist[(x >> shift) & dmask], 1u);
                    }
                }
            }
        }
        cluster.sync();  // every CTA's histogram is complete
        const int S = kBins / (int)C;
        const int s0 = (int)rank * S;
        uint32_t part = 0;
        for (int i = tid; i < S / 4; i += kThreads) {
            uint4 acc4 = make_uint4(0, 0, 0, 0);
            for (unsigned r = 0; r < C; ++r) {
                const uint4 v = *reinterpret_cast<const uint4*>(cluster.map_shared_rank(sh.hist, r) + s0 + 4 * i);
                acc4.x += v.x;
                acc4.y += v.y;
                acc4.z += v.z;
                acc4.w += v.w;
            }
            *reinterpret_cast<uint4*>(sh.slice + 4 * i) = acc4;
            part += acc4.x + acc4.y + acc4.z + acc4.w;
        }
        uint32_t slice_total;
        block_exclusive_scan(part, sh.warp_sums, slice_total);
        if (tid == 0) sh.total = slice_total;
        cluster.sync();  // slices and slice totals complete
        if (tid == 0) {
            uint32_t above = 0, pick_above = 0;
            int pick = -1;
            for (int r = (int)C - 1; r >= 0; --r) {
                const uint32_t t = *cluster.map_shared_rank(&sh.total, (unsigned)r);
                if (pick < 0 && above + t >= krem) {
                    pick = r;
                    pick_above = above;
                }
                above += t;
            }
            sh.pick = pick < 0 ? 0u : (uint32_t)pick;
            sh.pick_above = pick_above;
            sh.grand = above;
        }
        __syncthreads();
        {
            // Thread t owns bins b0, b0-1, ..., b0-7 (b0 = S-1-8t) of the picked slice.
            const uint32_t* ps = cluster.map_shared_rank(sh.slice, sh.pick);
            const int b0 = S - 1 - 8 * tid;
            uint32_t c[8] = {0, 0, 0, 0, 0, 0, 0, 0};
            if (b0 >= 7) {
                const uint4 v0 = *reinterpret_cast<const uint4*>(ps + b0 - 7);
                const uint4 v1 = *reinterpret_cast<const uint4*>(ps + b0 - 3);
                c[0] = v1.w; c[1] = v1.z; c[2] = v1.y; c[3] = v1.x;
                c[4] = v0.w; c[5] = v0.z; c[6] = v0.y; c[7] = v0.x;
            }
            const uint32_t pick = sh.pick;
            find_bin<8>(c, sh.pick_above, krem, sh, [&](int q) { return pick * (uint32_t)S + (uint32_t)(b0 - q); });
        }
        cluster.sync();  // remote slices read; digit, krem, grand visible
        if (pass == 0 && windowed && sh.grand < krem) {
            windowed = false;  // the k-th score lies below the window
            pass = -1;
            continue;
        }
        if (pass == 0 && windowed) {
            prefix = (sh.digit + dlow) << kWindowShift;
            mask = 0xffffffffu << kWindowShift;
        } else {
            prefix |= sh.digit << shift;
            mask |= dmask << shift;
        }
        krem = sh.krem;
    }
    *need = krem;
    return prefix;
}

// Grid: U * C CTAs in clusters of C (a power of two; one cluster per unit).
// CTA r of a cluster owns keys [r*R, min(N, (r+1)*R)) of its unit.
//
// Fast path.  The scoring kernel left a histogram of the unit's score bit
// patterns >> 19 (1/16 octave per bin).  Every CTA reads it and finds the bin
// d0 holding the k-th largest score; the keys above that bin are selected for
// sure, and the keys inside it (a few hundred on typical data) are the
// candidates.  Each CTA appends its candidates (index, pattern) to the unit's
// candidate list, every CTA then loads the whole list and selects among it
// with two more radix digits (11 + 8 bits) in its own shared memory -- the
// same exact threshold t and tie count everywhere.  The CTA's output offset
// follows from the "sure" counts of lower-ranked CTAs (distributed shared
// memory) and the candidate list.  The same single read of the scores marks
// every key in or above bin d0 in a bitmap of the CTA's slice; the slice's
// candidates below t (and ties past the tie budget, by index) are cleared,
// and the CTA writes the set bits in index order from one block scan over
// the words' popcounts.  Slices over kBitmapKeys keys re-read the scores
// instead (compact).  If the threshold bin holds more than kTopkCandidates
// keys, the cluster takes the multi-pass path.
__global__ __launch_bounds__(kThreads, 2) void topk_kernel(const float* __restrict__ scores,
                                                        const uint32_t* __restrict__ unit_max,
                                                        const uint32_t* __restrict__ unit_hist,
                                                        uint32_t* __restrict__ cand_cnt, uint2* __restrict__ cand,
                                                        int64_t Ncap, int N, int k, int R,
                                                        int32_t* __restrict__ idx_out)
{
    extern __shared__ __align__(16) char topk_smem[];
    Shared& sh = *reinterpret_cast<Shared*>(topk_smem);
    cg::cluster_group cluster = cg::this_cluster();
    const unsigned rank = cluster.block_rank(), C = cluster.num_blocks();
    const int tid = threadIdx.x;
    const int64_t u = blockIdx.x / C;
    const uint32_t* su = reinterpret_cast<const uint32_t*>(scores + u * Ncap);
    int32_t* out = idx_out + u * (int64_t)k;
    const int lo = (int)min64((int64_t)rank * R, N), hi = (int)min64((int64_t)lo + R, N);
    const int n = hi - lo;

    // The grid fits in one wave, so the attention kernel's CTAs may be placed
    // now; they wait for this grid to finish before they read anything.
    pdl_launch_dependents();
    pdl_wait();  // scores, maxima and histograms come from the previous kernel on the stream

    // ---- the unit histogram: bin d0 of the k-th largest score.
    {
        constexpr int kPer = kScoreHistBins / kThreads;  // 16 bins per thread, descending
        const int b0 = kScoreHistBins - 1 - kPer * tid;
        const uint4* hp = reinterpret_cast<const uint4*>(unit_hist + u * kScoreHistBins + (b0 - (kPer - 1)));
        uint32_t c[kPer];
#pragma unroll
        for (int v = 0; v < kPer / 4; ++v) {
            const uint4 w = __ldcg(hp + (kPer / 4 - 1 - v));
            c[4 * v + 0] = w.w;
            c[4 * v + 1] = w.z;
            c[4 * v + 2] = w.y;
            c[4 * v + 3] = w.x;
        }
        if (tid == 0) {
            sh.digit = 0;
            sh.krem = (uint32_t)k;
        }
        __syncthreads();
        find_bin<kPer>(c, 0u, (uint32_t)k, sh, [&](int q) { return (uint32_t)(b0 - q); });
        __syncthreads();
    }
    const uint32_t d0 = sh.digit, krem0 = sh.krem;
    const uint32_t ncand = __ldcg(unit_hist + u * kScoreHistBins + d0);

    uint32_t t, need, out_base, budget;
    if (ncand > (uint32_t)kCand) {
        t = select_multipass(cluster, su, lo, hi, __ldcg(unit_max + u), k, sh, &need);
        uint32_t gt = 0, eq = 0;
        for (int i = tid * 4; i < n; i += kThreads * 4) {
            const uint4 v = __ldcg(reinterpret_cast<const uint4*>(su + lo + i));
            const uint32_t vals[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                if (i + e < n) {
                    gt += vals[e] > t;
                    eq += vals[e] == t;
                }
            }
        }
        uint32_t tot_gt, tot_eq;
        block_exclusive_scan(gt, sh.warp_sums, tot_gt);
        block_exclusive_scan(eq, sh.warp_sums, tot_eq);
        if (tid == 0) {
            sh.counts[0] = tot_gt;
            sh.counts[1] = tot_eq;
        }
        cluster.sync();
        out_base = 0;
        uint32_t ties_before = 0;
        for (unsigned r = 0; r < rank; ++r) {
            const uint32_t* rc = cluster.map_shared_rank(sh.counts, r);
            const uint32_t b = need > ties_before ? need - ties_before : 0u;
            out_base += rc[0] + min(rc[1], b);
            ties_before += rc[1];
        }
        budget = need > ties_before ? need - ties_before : 0u;
        cluster.sync();  // no remote shared-memory access after this point
    } else {
        // ---- candidates of this slice -> the unit list; count keys above bin d0;
        // mark every key in or above bin d0 in the slice bitmap.
        const bool use_bits = n <= kBitmapKeys;
        const int words = (n + 31) / 32;
        if (use_bits)
            for (int w = tid; w < words; w += kThreads) sh.bits[w] = 0u;
        if (tid == 0) sh.nlocal = 0;
        __syncthreads();
        const int lane = tid & 31;
        uint32_t sure = 0;
        for (int base = tid * 4; base - tid * 4 < n; base += kThreads * 4 * kBatch) {
            uint4 v[kBatch];
#pragma unroll
            for (int b = 0; b < kBatch; ++b) {
                const int i = base + b * kThreads * 4;
                v[b] = i < n ? __ldcg(reinterpret_cast<const uint4*>(su + lo + i)) : make_uint4(0, 0, 0, 0);
            }
#pragma unroll
            for (int b = 0; b < kBatch; ++b) {
                const int i = base + b * kThreads * 4;
                const uint32_t vals[4] = {v[b].x, v[b].y, v[b].z, v[b].w};
                uint32_t nib = 0;
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    if (i + e < n) {
                        const uint32_t top = vals[e] >> kScoreHistShift;
                        sure += top > d0;
                        nib |= (uint32_t)(top >= d0) << e;
                        if (top == d0) {
                            // The unit's bin holds <= kCand keys, so the slice's do too.
                            const uint32_t slot = atomicAdd(&sh.nlocal, 1u);
                            if (slot < (uint32_t)kCand) sh.cand[slot] = make_uint2((uint32_t)(lo + i + e), vals[e]);
                        }
                    }
                }
                if (use_bits) {
                    // Lanes 8m .. 8m + 7 hold the 32 consecutive keys of one bitmap word.
                    uint32_t word = nib << ((lane & 7) * 4);
                    word |= __shfl_xor_sync(kFullMask, word, 1);
                    word |= __shfl_xor_sync(kFullMask, word, 2);
                    word |= __shfl_xor_sync(kFullMask, word, 4);
                    if ((lane & 7) == 0 && i < n) sh.bits[i >> 5] = word;
                }
            }
        }
        uint32_t sure_total;
        block_exclusive_scan(sure, sh.warp_sums, sure_total);  // (its barriers also order sh.nlocal)
        if (tid == 0) {
            sh.sure = sure_total;
            sh.local_base = atomicAdd(cand_cnt + u, min(sh.nlocal, (uint32_t)kCand));
        }
        __syncthreads();
        {
            // Append this slice's candidates to the unit list with one atomic per CTA.
            const uint32_t nl = min(sh.nlocal, (uint32_t)kCand), lb = sh.local_base;
            for (uint32_t i = tid; i < nl; i += kThreads)
                if (lb + i < (uint32_t)kCand) cand[u * kCand + lb + i] = sh.cand[i];
        }
        __threadfence();
        cluster.sync();  // candidate list complete; sure counts visible
        if (tid == 0) {
            uint32_t before = 0;
            for (unsigned r = 0; r < rank; ++r) before += *cluster.map_shared_rank(&sh.sure, r);
            sh.pick_above = before;
        }
        const int nc = (int)min(ncand, (uint32_t)kCand);
        for (int i = tid; i < nc; i += kThreads) sh.cand[i] = __ldcg(cand + u * kCand + i);
        cluster.sync();  // no remote shared-memory access after this point
        const uint32_t sure_before = sh.pick_above;

        // ---- the krem0-th largest among the candidates: digits 18-8 and 7-0.
        uint32_t prefix = d0 << kScoreHistShift, mask = 0xffffffffu << kScoreHistShift, krem = krem0;
        for (int pass = 0; pass < 2; ++pass) {
            const int shift = pass == 0 ? 8 : 0;
            const uint32_t dmask = pass == 0 ? 0x7ffu : 0xffu;
            for (int b = tid; b < kBins; b += kThreads) sh.hist[b] = 0;
            __syncthreads();
            for (int i = tid; i < nc; i += kThreads) {
                const uint32_t x = sh.cand[i].y;
                if ((x & mask) == prefix) atomicAdd(&sh.hist[(x >> shift) & dmask], 1u);
            }
            __syncthreads();
            constexpr int kPer = kBins / kThreads;  // 8 bins per thread, descending
            const int b0 = kBins - 1 - kPer * tid;
            uint32_t c[kPer];
#pragma unroll
            for (int q = 0; q < kPer; ++q) c[q] = sh.hist[b0 - q];
            find_bin<kPer>(c, 0u, krem, sh, [&](int q) { return (uint32_t)(b0 - q); });
            __syncthreads();
            prefix |= sh.digit << shift;
            mask |= dmask << shift;
            krem = sh.krem;
            __syncthreads();
        }
        t = prefix;
        need = krem;
        // Keys before this slice that are selected: sure keys of lower CTAs,
        // candidates above t before lo, and ties at t before lo (up to need).
        uint32_t gt_before = 0, eq_before = 0, eq_all = 0;
        for (int i = tid; i < nc; i += kThreads) {
            const uint2 e = sh.cand[i];
            if ((int)e.x < lo) {
                gt_before += e.y > t;
                eq_before += e.y == t;
            }
            eq_all += e.y == t;
        }
        uint32_t tg, te, tall;
        block_exclusive_scan(gt_before, sh.warp_sums, tg);
        block_exclusive_scan(eq_before, sh.warp_sums, te);
        block_exclusive_scan(eq_all, sh.warp_sums, tall);
        out_base = sure_before + tg + min(te, need);
        budget = need > te ? need - te : 0u;
        if (use_bits) {
            // Prune the slice's candidates: keep those above t, and ties at t
            // whose rank by index among all of the unit's ties is below need.
            for (int i = tid; i < nc; i += kThreads) {
                const uint2 e = sh.cand[i];
                if ((int)e.x < lo || (int)e.x >= hi) continue;
                bool keep = e.y > t;
                if (e.y == t) {
                    if (tall <= need) {
                        keep = true;
                    } else {
                        uint32_t rank_t = 0;
                        for (int j = 0; j < nc; ++j) rank_t += sh.cand[j].y == t && sh.cand[j].x < e.x;
                        keep = rank_t < need;
                    }
                }
                if (!keep) atomicAnd(&sh.bits[(e.x - lo) >> 5], ~(1u << ((e.x - lo) & 31)));
            }
            __syncthreads();
            // Selected keys in index order: each thread takes consecutive words
            // (read 16 bytes at a time; words past the slice are zero).
            constexpr int kWordsPerThread = kBitmapWords / kThreads;
            const int w0 = tid * kWordsPerThread;
            uint32_t wv[kWordsPerThread];
#pragma unroll
            for (int q = 0; q < kWordsPerThread; q += 4) {
                const uint4 x4 = w0 + q < words ? *reinterpret_cast<const uint4*>(&sh.bits[w0 + q]) : make_uint4(0, 0, 0, 0);
                wv[q] = x4.x;
                wv[q + 1] = w0 + q + 1 < words ? x4.y : 0u;
                wv[q + 2] = w0 + q + 2 < words ? x4.z : 0u;
                wv[q + 3] = w0 + q + 3 < words ? x4.w : 0u;
            }
            uint32_t cnt = 0;
#pragma unroll
            for (int q = 0; q < kWordsPerThread; ++q) cnt += __popc(wv[q]);
            uint32_t total;
            uint32_t pos = out_base + block_exclusive_scan(cnt, sh.warp_sums, total);
#pragma unroll
            for (int q = 0; q < kWordsPerThread; ++q) {
                uint32_t x = wv[q];
                while (x) {
                    const int bit = __ffs(x) - 1;
                    x &= x - 1;
                    // pos < k always holds when the threshold is exact; the guard
                    // keeps every store inside the unit's k slots regardless.
                    if (pos < (uint32_t)k) out[pos] = lo + 32 * (w0 + q) + bit;
                    ++pos;
                }
            }
            return;
        }
    }
    compact(su, lo, hi, t, budget, out_base, k, out, sh);
}

}  // namespace

cudaError_t launch_topk(const float* scores, const uint32_t* unit_max, const uint32_t* unit_hist,
                        uint32_t* cand_cnt, uint2* cand, const DecodeShape& s, int32_t* idx_out, cudaStream_t stream)
{
    const int64_t want = (s.N + kSliceKeys - 1) / kSliceKeys;
    int C = 1;  // a power of two, so the multi-pass bins split evenly over the cluster
    while (C < kMaxCluster && C < want) C *= 2;
    const int R = (int)(((s.N + C - 1) / C + 31) / 32 * 32);
    cudaError_t e = cudaFuncSetAttribute(topk_kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sizeof(Shared));
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(s.U * C));
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = sizeof(Shared);
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)C;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl_enabled() ? 2 : 1;
    e = cudaLaunchKernelEx(&cfg, topk_kernel, scores, unit_max, unit_hist, cand_cnt, cand, s.Ncap, (int)s.N, s.k, R,
                           idx_out);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace socket_attn
