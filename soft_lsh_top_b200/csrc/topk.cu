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
// values.  The scoring kernel leaves, per unit, a histogram of the score bit
// patterns >> 19 (1/16 octave per bin).  From it every CTA finds the bin d0
// that holds the k-th largest score: keys above d0 are selected for sure,
// keys inside it are the candidates.
//
// One read of the scores, slice by slice (CTA r of a unit takes keys
// [r S, (r + 1) S)): each CTA writes the unit's selection bitmap for its
// slice -- bit n set when key n lies in or above bin d0 -- and appends its
// candidates (index, bit pattern) to the unit's candidate list.  The last CTA
// of the unit to finish (an atomic ticket; nobody waits) then
//   * radix-selects the exact k-th bit pattern t among the candidates (two
//     more digits) and the number of keys equal to t still to take,
//   * clears the bitmap bits of the candidates below t, and of the ties at t
//     beyond that number (the lowest indices are kept: a radix select over
//     the ties' indices when they do not all fit),
//   * writes the set bits of the bitmap in index order from one block-wide
//     scan of the words' population counts.
// If the threshold bin holds more keys than the candidate list can take, the
// last CTA instead selects over all of the unit's scores (three radix digits)
// and writes the selection from a compaction pass over the scores.
#include "common.cuh"
#include "internal.h"

namespace socket_attn {
namespace {

constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;
constexpr int kSliceKeys = 32768;                      // keys per CTA
constexpr int kLoads = 8;                              // 16-byte score loads per thread in flight
constexpr int kRounds = kSliceKeys / (4 * kThreads * kLoads);
constexpr int kBins = 2048;                            // radix bins of the digit passes
constexpr int kWordsPerThread = 8;                     // bitmap words per thread and tile of the compaction

struct Shared {
    uint32_t warp_sums[kWarps];
    uint32_t digit, krem, last;
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
// the top: writes its id (bin_of(q)) to sh.digit and the keys still needed
// inside it to sh.krem.  Every thread must call it; sh is valid after the
// next barrier.
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
    prefix |= sh.digit << shift;
    mask |= dmask << shift;
    krem = sh.krem;
    __syncthreads();
}

// Writes the selection from a pass over the scores: keys of [0, n) above t,
// plus the first `budget` keys equal to t, in index order.
__device__ void compact_scores(const uint32_t* su, int n, uint32_t t, uint32_t budget, int k, int32_t* out,
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

struct TopkArgs {
    const float* scores;       // [U][Ncap]
    const uint32_t* unit_hist; // [U][kScoreHistBins]
    uint32_t* cand_cnt;        // [U] candidates appended (zeroed before the step)
    uint2* cand;               // [U][cap] (index, bit pattern)
    uint32_t* bitmap;          // [U][Ncap / 32]
    uint32_t* done;            // [U] tickets of finished CTAs (zeroed before the step)
    int32_t* idx_out;          // [U][k]
    int64_t Ncap;
    int N, k, C, cap;
};

// Grid: U * C CTAs of kThreads; CTA r of unit u reads keys [r S, min(N, (r+1) S)).
__global__ __launch_bounds__(kThreads, 2) void topk_kernel(const TopkArgs a)
{
    __shared__ Shared sh;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int64_t u = blockIdx.x / a.C;
    const int r = blockIdx.x % a.C;
    const uint32_t* su = reinterpret_cast<const uint32_t*>(a.scores + u * a.Ncap);
    uint32_t* bm = a.bitmap + u * (a.Ncap / 32);
    const int lo = r * kSliceKeys, hi = min(a.N, lo + kSliceKeys);

    // The grid fits in one wave, so the attention kernel's CTAs may be placed
    // now; they wait for this grid to finish before they read anything.
    pdl_launch_dependents();
    pdl_wait();  // scores and histograms come from the previous kernel on the stream

    // ---- the unit histogram: bin d0 of the k-th largest score.
    {
        constexpr int kPer = kScoreHistBins / kThreads;  // 8 bins per thread, descending
        const int b0 = kScoreHistBins - 1 - kPer * tid;
        const uint4* hp = reinterpret_cast<const uint4*>(a.unit_hist + u * kScoreHistBins + (b0 - (kPer - 1)));
        uint32_t c[kPer];
#pragma unroll
        for (int v = 0; v < kPer / 4; ++v) {
            const uint4 w = __ldcg(hp + (kPer / 4 - 1 - v));
            c[4 * v] = w.w;
            c[4 * v + 1] = w.z;
            c[4 * v + 2] = w.y;
            c[4 * v + 3] = w.x;
        }
        if (tid == 0) {
            sh.digit = 0;
            sh.krem = (uint32_t)a.k;
        }
        __syncthreads();
        find_bin<kPer>(c, (uint32_t)a.k, sh, [&](int q) { return (uint32_t)(b0 - q); });
        __syncthreads();
    }
    const uint32_t d0 = sh.digit, krem0 = sh.krem;

    // ---- one read of the slice: bitmap words and candidates.  In load i of
    // a round thread t holds keys base + 2048 i + 4 t .. + 3, so lanes
    // 8m .. 8m + 7 of a warp hold the 32 keys of one bitmap word.
    for (int round = 0; round < kRounds; ++round) {
        const int base = lo + round * kLoads * 4 * kThreads;
        if (base >= hi) break;
        uint4 v[kLoads];
#pragma unroll
        for (int i = 0; i < kLoads; ++i) {
            const int n0 = base + i * 4 * kThreads + 4 * tid;
            v[i] = n0 < hi ? __ldcg(reinterpret_cast<const uint4*>(su + n0)) : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int i = 0; i < kLoads; ++i) {
            const int n0 = base + i * 4 * kThreads + 4 * tid;
            const uint32_t vals[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
            uint32_t nib = 0, cmask = 0;
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const uint32_t top = vals[e] >> kScoreHistShift;
                const bool live = n0 + e < hi;
                nib |= (uint32_t)(live && top >= d0) << e;
                cmask |= (uint32_t)(live && top == d0) << e;
            }
            uint32_t word = nib << ((lane & 7) * 4);
            word |= __shfl_xor_sync(kFullMask, word, 1);
            word |= __shfl_xor_sync(kFullMask, word, 2);
            word |= __shfl_xor_sync(kFullMask, word, 4);
            if ((lane & 7) == 0 && n0 < hi) bm[n0 >> 5] = word;
            // Candidates: one atomic per warp and load round that has any.
            const uint32_t cnt = __popc(cmask);
            if (__any_sync(kFullMask, cnt != 0)) {
                uint32_t incl = cnt;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const uint32_t y = __shfl_up_sync(kFullMask, incl, o);
                    if (lane >= o) incl += y;
                }
                uint32_t slot = 0;
                if (lane == 31) slot = atomicAdd(a.cand_cnt + u, incl);
                slot = __shfl_sync(kFullMask, slot, 31) + incl - cnt;
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    if (cmask >> e & 1u) {
                        if (slot < (uint32_t)a.cap) a.cand[u * a.cap + slot] = make_uint2((uint32_t)(n0 + e), vals[e]);
                        ++slot;
                    }
                }
            }
        }
    }

    // ---- the unit's last CTA to get here selects.
    __threadfence();
    __syncthreads();
    if (tid == 0) sh.last = atomicAdd(a.done + u, 1u) == (uint32_t)(a.C - 1);
    __syncthreads();
    if (!sh.last) return;
    __threadfence();

    int32_t* out = a.idx_out + u * (int64_t)a.k;
    const uint32_t ncand = __ldcg(a.unit_hist + u * kScoreHistBins + d0);  // == candidates appended
    if (ncand > (uint32_t)a.cap) {
        // The threshold bin holds more keys than the list: three digits over
        // all of the unit's scores, then a compaction pass over them.
        uint32_t prefix = 0, mask = 0, krem = (uint32_t)a.k;
        auto get = [&](int i) { return __ldcg(su + i); };
        radix_digit(sh, a.N, get, 20, 0x7ffu, true, prefix, mask, krem);
        radix_digit(sh, a.N, get, 9, 0x7ffu, true, prefix, mask, krem);
        radix_digit(sh, a.N, get, 0, 0x1ffu, true, prefix, mask, krem);
        compact_scores(su, a.N, prefix, krem, a.k, out, sh);
        if (tid == 0) a.done[u] = 0u;
        return;
    }

    // ---- the krem0-th largest among the candidates: digits 18-8 and 7-0.
    const uint2* cu = a.cand + u * a.cap;
    const int nc = (int)ncand;
    uint32_t prefix = d0 << kScoreHistShift, mask = 0xffffffffu << kScoreHistShift, need = krem0;
    {
        auto get = [&](int i) { return __ldcg(&cu[i].y); };
        radix_digit(sh, nc, get, 8, 0x7ffu, true, prefix, mask, need);
        radix_digit(sh, nc, get, 0, 0xffu, true, prefix, mask, need);
    }
    const uint32_t t = prefix;
    // Ties at t: if more than `need`, keep the `need` lowest indices, i.e.
    // those at or below the need-th smallest tie index ti.
    uint32_t ties = 0;
    for (int i = tid; i < nc; i += kThreads) ties += __ldcg(&cu[i].y) == t;
    uint32_t ties_total;
    block_exclusive_scan(ties, sh.warp_sums, ties_total);
    uint32_t ti = 0xffffffffu;
    if (ties_total > need) {
        uint32_t ik = need;
        // Indices below 2^31: digits 30-20, 19-9, 8-0 of the ties' indices, ascending.
        auto get = [&](int i) {
            const uint2 e = __ldcg(&cu[i]);
            return e.y == t ? e.x : 0xffffffffu;  // non-ties never match the prefix once bit 31 is fixed
        };
        uint32_t p31 = 0, m31 = 0x80000000u;
        radix_digit(sh, nc, [&](int i) { return get(i); }, 20, 0x7ffu, false, p31, m31, ik);
        radix_digit(sh, nc, [&](int i) { return get(i); }, 9, 0x7ffu, false, p31, m31, ik);
        radix_digit(sh, nc, [&](int i) { return get(i); }, 0, 0x1ffu, false, p31, m31, ik);
        ti = p31;
    }
    // Clear the bits of the candidates that are not selected.
    for (int i = tid; i < nc; i += kThreads) {
        const uint2 e = __ldcg(&cu[i]);
        const bool keep = e.y > t || (e.y == t && e.x <= ti);
        if (!keep) atomicAnd(bm + (e.x >> 5), ~(1u << (e.x & 31)));
    }
    __threadfence();
    __syncthreads();

    // ---- selected keys in index order from the bitmap: tiles of
    // kThreads x 8 words, each thread a run of consecutive words.
    const int words = (a.N + 31) / 32;
    uint32_t out_base = 0;
    for (int w0 = 0; w0 < words; w0 += kThreads * kWordsPerThread) {
        const int wt = w0 + tid * kWordsPerThread;
        uint32_t wv[kWordsPerThread];
#pragma unroll
        for (int q = 0; q < kWordsPerThread; ++q) wv[q] = wt + q < words ? __ldcg(bm + wt + q) : 0u;
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
                // pos < k whenever the threshold is exact; the guard keeps every
                // store inside the unit's k slots regardless.
                if (pos < (uint32_t)a.k) out[pos] = 32 * (wt + q) + bit;
                ++pos;
            }
        }
        out_base += total;
    }
    if (tid == 0) a.done[u] = 0u;
}

}  // namespace

int topk_candidate_capacity(int64_t Ncap) { return (int)min64(Ncap, (int64_t)kTopkCandidates); }

cudaError_t launch_topk(const float* scores, const uint32_t* unit_hist, uint32_t* cand_cnt, uint2* cand,
                        uint32_t* bitmap, uint32_t* done, const DecodeShape& s, int32_t* idx_out,
                        cudaStream_t stream)
{
    TopkArgs a;
    a.scores = scores;
    a.unit_hist = unit_hist;
    a.cand_cnt = cand_cnt;
    a.cand = cand;
    a.bitmap = bitmap;
    a.done = done;
    a.idx_out = idx_out;
    a.Ncap = s.Ncap;
    a.N = (int)s.N;
    a.k = s.k;
    a.C = (int)((s.N + kSliceKeys - 1) / kSliceKeys);
    a.cap = topk_candidate_capacity(s.Ncap);
    cudaError_t e = set_smem_limit_once((const void*)topk_kernel, 0);
    if (e != cudaSuccess) return e;
    return launch_pdl(topk_kernel, dim3((unsigned)(s.U * a.C)), dim3(kThreads), 0, stream, a);
}

}  // namespace socket_attn
