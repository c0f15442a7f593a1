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
//     more digits; one when the first digit's bin holds exactly the keys
//     still needed, which are then all kept) and the number of keys equal to
//     t still to take,
//   * clears the bitmap bits of the candidates below t, and of the ties at t
//     beyond that number (the lowest indices are kept: a radix select over
//     the ties' indices when they do not all fit),
//   * writes the set bits of the bitmap in index order from one block-wide
//     scan of the words' population counts.
// If the threshold bin holds more keys than the candidate list can take, the
// last CTA instead selects over all of the unit's scores (three radix digits)
// and writes the selection from a compaction pass over the scores.
//
// When a unit has many slices and the whole grid is resident at once
// (`spread`), the unit's CTAs share
// the writing instead: the last CTA clears the dropped candidates' bits in
// the unit's bitmap, works out every slice's first output slot (its keys in
// or above d0, less its dropped candidates, summed over the slices before
// it), and publishes them behind a flag in the ticket word; every CTA of the
// unit then writes its own slice's selection from its slot.  The other CTAs
// wait for that flag, a bounded wait (SOCKET_DEVERR_SELECT_TIMEOUT on
// expiry); they can wait safely because the last CTA is the last to take a
// ticket, so it is running once anyone waits.
#include "common.cuh"
#include "internal.h"
#include "select.cuh"
#include "socket_attn.h"

namespace socket_attn {
namespace {

using namespace select512;
constexpr int kSliceKeys = 32768;                      // keys per CTA
constexpr int kLoadsPerThread = kSliceKeys / (4 * kThreads);  // 16-byte score loads per thread
constexpr int kInFlight = 6;                           // of them in flight at a time
constexpr int kRankMax = 96;                           // candidates ranked by counting (nc^2 comparisons)
constexpr int kWordsPerThread = 8;                     // bitmap words per thread and tile of the compaction
constexpr int kTileWords = kThreads * kWordsPerThread;  // bitmap words per tile (131072 keys)

struct TopkArgs {
    const float* scores;       // [U][Ncap]
    const uint32_t* unit_hist; // [U][kScoreHistBins]
    uint32_t* cand_cnt;        // [U] candidates appended (zeroed before the step)
    uint2* cand;               // [U][cap] (index, bit pattern)
    uint32_t* bitmap;          // [U][bm_stride] (Ncap / 32 words used)
    uint32_t* done;            // [U] tickets of finished CTAs (zeroed before the step)
    int32_t* idx_out;          // [U][k]
    uint32_t* info;            // [U][info_stride]: keys in or above d0 per slice [C], first slot per slice [C]
    uint32_t* err_word;
    int64_t Ncap, bm_stride, info_stride;
    int N, k, C, cap;
    int spread;                // every CTA writes its own slice's selection (grid resident at once)
    uint32_t max_polls;
};

constexpr uint32_t kPublished = 0x80000000u;  // set in the unit's ticket word once the slots are out
constexpr int kSpreadMinSlices = 8;
constexpr int kSpreadMaxSlices = 256;

__device__ __forceinline__ uint32_t ld_acquire_u32(const uint32_t* p)
{
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// Writes slice r's selected keys (the set bits of its words of the unit's
// bitmap, final once the slots are published) in index order from output
// slot `slot` on: two words per thread, one block-wide scan.
__device__ __forceinline__ void write_slice(const TopkArgs& a, int64_t u, int r, uint32_t slot, Shared& sh)
{
    static_assert(kSliceKeys / 32 == 2 * kThreads, "two bitmap words of the slice per thread");
    const int tid = threadIdx.x;
    const int words = (a.N + 31) / 32;
    const int w = r * (kSliceKeys / 32) + 2 * tid;
    const uint32_t* bm = a.bitmap + u * a.bm_stride;
    const uint32_t x0 = w < words ? __ldcg(bm + w) : 0u, x1 = w + 1 < words ? __ldcg(bm + w + 1) : 0u;
    uint32_t total;
    uint32_t pos = slot + block_exclusive_scan(__popc(x0) + __popc(x1), sh.warp_sums, total);
    int32_t* out = a.idx_out + u * (int64_t)a.k;
    const uint32_t xs[2] = {x0, x1};
#pragma unroll
    for (int q = 0; q < 2; ++q) {
        uint32_t x = xs[q];
        while (x) {
            const int b = __ffs(x) - 1;
            x &= x - 1;
            // pos < k whenever the threshold is exact; the guard keeps every
            // store inside the unit's k slots regardless.
            if (pos < (uint32_t)a.k) out[pos] = 32 * (w + q) + b;
            ++pos;
        }
    }
}

// Grid: U * C CTAs of kThreads; CTA r of unit u reads keys [r S, min(N, (r+1) S)).
// Dynamic shared memory: the CTA's candidates (then the unit's) and one tile
// of the selection bitmap.
// SPREAD: every CTA writes its own slice of the selection (a.spread).
template <bool SPREAD>
__global__ __launch_bounds__(kThreads, 2) void topk_kernel(const TopkArgs a)
{
    __shared__ Shared sh;
    extern __shared__ __align__(16) char topk_dyn[];
    uint2* scand = reinterpret_cast<uint2*>(topk_dyn);                               // [a.cap]
    uint32_t* sbits = reinterpret_cast<uint32_t*>(topk_dyn + sizeof(uint2) * a.cap);  // [kTileWords]
    const int tid = threadIdx.x, lane = tid & 31;
    const int64_t u = blockIdx.x / a.C;
    // With many slices per unit, consecutive CTAs (which tend to share an SM:
    // the grid is placed two per SM as the scoring grid's CTAs leave) take
    // slices from opposite ends of the unit, so that where keys drift along a
    // long sequence the crowded late slices share SMs with sparse early ones.
    // With few slices the plain order measured faster.
    const int b = blockIdx.x % a.C;
    const int r = !SPREAD ? b : (b & 1) ? a.C - 1 - (b >> 1) : (b >> 1);
    const bool single = a.C == 1;  // one CTA holds the whole unit: bitmap and candidates stay in shared memory
    const uint32_t* su = reinterpret_cast<const uint32_t*>(a.scores + u * a.Ncap);
    uint32_t* bm = a.bitmap + u * a.bm_stride;  // 16-byte aligned rows
    const int lo = r * kSliceKeys, hi = min(a.N, lo + kSliceKeys);

    // The grid fits in one wave, so the attention kernel's CTAs may be placed
    // now; they wait for this grid to finish before they read anything.
    pdl_launch_dependents();
    pdl_wait();  // scores and histograms come from the previous kernel on the stream

    // Load g of this thread covers keys lo + 2048 g + 4 tid .. + 3 (lanes
    // 8m .. 8m + 7 of a warp: the 32 keys of one bitmap word).  The first
    // kInFlight loads are issued right after the histogram's, so they stream
    // while d0 is found, without delaying the histogram behind them.
    auto key_of = [&](int g) { return lo + g * 4 * kThreads + 4 * tid; };
    auto load = [&](int g) {
        const int n0 = key_of(g);
        return n0 < hi ? __ldcg(reinterpret_cast<const uint4*>(su + n0)) : make_uint4(0, 0, 0, 0);
    };
    uint4 v[kInFlight];

    // ---- the unit histogram: bin d0 of the k-th largest score.
    {
        constexpr int kPer = kScoreHistBins / kThreads;  // 8 bins per thread, descending
        const int b0 = kScoreHistBins - 1 - kPer * tid;
        const uint4* hp = reinterpret_cast<const uint4*>(a.unit_hist + u * kScoreHistBins + (b0 - (kPer - 1)));
        uint4 hw[kPer / 4];
#pragma unroll
        for (int q = 0; q < kPer / 4; ++q) hw[q] = __ldcg(hp + (kPer / 4 - 1 - q));
#pragma unroll
        for (int g = 0; g < kInFlight; ++g) v[g] = load(g);
        uint32_t c[kPer];
#pragma unroll
        for (int q = 0; q < kPer / 4; ++q) {
            c[4 * q] = hw[q].w;
            c[4 * q + 1] = hw[q].z;
            c[4 * q + 2] = hw[q].y;
            c[4 * q + 3] = hw[q].x;
        }
        if (tid == 0) {
            sh.digit = 0;
            sh.krem = (uint32_t)a.k;
            sh.count = 0;
            sh.bin_count = 0;
        }
        __syncthreads();
        find_bin<kPer>(c, (uint32_t)a.k, sh, [&](int q) { return (uint32_t)(b0 - q); });
        __syncthreads();
    }
    const uint32_t d0 = sh.digit, krem0 = sh.krem;
    const uint32_t ncand = sh.bin_count;  // keys of the unit in bin d0
    const bool fits = ncand <= (uint32_t)a.cap;

    // ---- one read of the slice: bitmap words, and the candidates into
    // shared memory (one shared atomic per warp and load that has any).
#pragma unroll
    for (int g = 0; g < kLoadsPerThread; ++g) {
        if (lo + g * 4 * kThreads + 128 * (tid >> 5) >= hi) continue;  // the warp's keys all lie past the slice
        const uint4 x = v[g % kInFlight];
        if (g + kInFlight < kLoadsPerThread) v[g % kInFlight] = load(g + kInFlight);
        const int n0 = key_of(g);
        const uint32_t vals[4] = {x.x, x.y, x.z, x.w};
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
        if ((lane & 7) == 0 && n0 < hi) {
            if (single) sbits[n0 >> 5] = word;
            else bm[n0 >> 5] = word;
        }
        const uint32_t cnt = fits ? __popc(cmask) : 0u;
        if (__any_sync(kFullMask, cnt != 0)) {
            uint32_t incl = cnt;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const uint32_t y = __shfl_up_sync(kFullMask, incl, o);
                if (lane >= o) incl += y;
            }
            uint32_t slot = 0;
            if (lane == 31) slot = atomicAdd(&sh.count, incl);
            slot = __shfl_sync(kFullMask, slot, 31) + incl - cnt;
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                if (cmask >> e & 1u) {
                    // slot < ncand <= cap: the slice's candidates are a subset of the unit's
                    if (slot < (uint32_t)a.cap) scand[slot] = make_uint2((uint32_t)(n0 + e), vals[e]);
                    ++slot;
                }
            }
        }
    }
    __syncthreads();
    if (!single) {
        // The CTA's candidates -> the unit list (one global atomic per CTA).
        const uint32_t nl = min(sh.count, (uint32_t)a.cap);
        if (tid == 0 && nl) sh.base = atomicAdd(a.cand_cnt + u, nl);
        __syncthreads();
        const uint32_t base = sh.base;
        uint2* cu = a.cand + u * a.cap;
        for (uint32_t i = tid; i < nl; i += kThreads)
            if (base + i < (uint32_t)a.cap) cu[base + i] = scand[i];
        if (SPREAD && fits) {
            // Keys of this slice in or above d0, from its bitmap words (written above).
            __syncthreads();
            const int words = (a.N + 31) / 32, w = r * (kSliceKeys / 32) + 2 * tid;
            const uint32_t my_ge = (w < words ? __popc(__ldcg(bm + w)) : 0) + (w + 1 < words ? __popc(__ldcg(bm + w + 1)) : 0);
            uint32_t ge_total;
            block_exclusive_scan(my_ge, sh.warp_sums, ge_total);
            if (tid == 0) a.info[u * a.info_stride + r] = ge_total;
        }
        // ---- the unit's last CTA to get here selects.
        if (!cta_ticket(a.done + u, (uint32_t)(a.C - 1), sh.last)) {
            if (!(SPREAD && fits)) return;
            // Wait (bounded) for the last CTA's slots, then write this slice.
            if (tid == 0) {
                bool got = false;
                for (uint32_t polls = 0; polls < a.max_polls; ++polls) {
                    if (ld_acquire_u32(a.done + u) & kPublished) {
                        got = true;
                        break;
                    }
                    __nanosleep(128);
                }
                sh.base = got ? __ldcg(a.info + u * a.info_stride + a.C + r) : 0xffffffffu;
                if (!got) atomicOr(a.err_word, SOCKET_DEVERR_SELECT_TIMEOUT);
            }
            __syncthreads();
            if (sh.base != 0xffffffffu) write_slice(a, u, r, sh.base, sh);
            return;
        }
    }

    int32_t* out = a.idx_out + u * (int64_t)a.k;
    if (!fits) {
        // The threshold bin holds more keys than the candidate list: three
        // digits over all of the unit's scores, then a compaction pass.
        uint32_t prefix = 0, mask = 0, krem = (uint32_t)a.k;
        auto get = [&](int i) { return __ldcg(su + i); };
        radix_digit(sh, a.N, get, 20, 0x7ffu, true, prefix, mask, krem);
        radix_digit(sh, a.N, get, 9, 0x7ffu, true, prefix, mask, krem);
        radix_digit(sh, a.N, get, 0, 0x1ffu, true, prefix, mask, krem);
        compact_scores(su, a.N, prefix, krem, a.k, out, sh);
        if (tid == 0) a.done[u] = 0u;
        return;
    }

    // The first bitmap tile is fetched while the candidates are ranked.
    const int words = (a.N + 31) / 32;
    uint4 tw[kWordsPerThread / 4];
    auto load_tile = [&](int w0) {
#pragma unroll
        for (int q = 0; q < kWordsPerThread / 4; ++q) {
            // Rows are padded to whole 16-byte groups; words past the last key are dropped.
            const int wi = w0 + tid * kWordsPerThread + 4 * q;
            uint4 x = wi < words ? __ldcg(reinterpret_cast<const uint4*>(bm + wi)) : make_uint4(0, 0, 0, 0);
            if (wi + 1 >= words) x.y = 0u;
            if (wi + 2 >= words) x.z = 0u;
            if (wi + 3 >= words) x.w = 0u;
            tw[q] = x;
        }
    };
    const int nc = (int)ncand;
    if (!single) {
        if (!SPREAD) load_tile(0);
        // ---- the unit's candidates in shared memory.
        const uint2* cu = a.cand + u * a.cap;
        for (int i = tid; i < nc; i += kThreads) scand[i] = __ldcg(cu + i);
        __syncthreads();
    }
    // ---- among the nc candidates (every key of bin d0), keep the krem0 with
    // the largest scores, ties to the lower index; the decision replaces each
    // candidate's bit pattern (1 keep, 0 drop).  A few hundred: rank each by
    // counting those ahead of it (T lanes per candidate, a power of two);
    // more: two radix digits for the krem0-th pattern t, then the ties at t by
    // a radix select over their indices.
    if (nc <= kRankMax) {
        int T = 1;
        while (T < 32 && T * 2 * nc <= kThreads) T *= 2;
        const int sub = lane & (T - 1);
        uint32_t keep[(kRankMax + kThreads - 1) / kThreads] = {};
        for (int i0 = 0, it = 0; i0 < nc * T; i0 += kThreads, ++it) {
            const int i = (i0 + tid) / T;
            uint32_t ahead = 0;
            if (i < nc) {
                const uint2 me = scand[i];
                int j = sub;
                for (; j + 3 * T < nc; j += 4 * T) {
                    const uint2 o0 = scand[j], o1 = scand[j + T], o2 = scand[j + 2 * T], o3 = scand[j + 3 * T];
                    ahead += (o0.y > me.y || (o0.y == me.y && o0.x < me.x)) +
                             (o1.y > me.y || (o1.y == me.y && o1.x < me.x)) +
                             (o2.y > me.y || (o2.y == me.y && o2.x < me.x)) +
                             (o3.y > me.y || (o3.y == me.y && o3.x < me.x));
                }
                for (; j < nc; j += T) {
                    const uint2 o = scand[j];
                    ahead += o.y > me.y || (o.y == me.y && o.x < me.x);
                }
            }
            for (int o = 1; o < T; o <<= 1) ahead += __shfl_xor_sync(kFullMask, ahead, o);
            keep[it] = ahead < krem0;
        }
        __syncthreads();  // every rank counted before the patterns are overwritten
        for (int i0 = 0, it = 0; i0 < nc * T; i0 += kThreads, ++it) {
            const int i = (i0 + tid) / T;
            if (i < nc && sub == 0) scand[i].y = keep[it];
        }
    } else {
        uint32_t prefix = d0 << kScoreHistShift, mask = 0xffffffffu << kScoreHistShift, need = krem0;
        auto bits_of = [&](int i) { return scand[i].y; };
        radix_digit(sh, nc, bits_of, 8, 0x7ffu, true, prefix, mask, need);
        // When the bin found holds exactly the keys still needed, all of them
        // are kept: the threshold is the bin's lowest pattern, with no ties to
        // resolve, and the last digit is skipped (the common case: a few
        // hundred candidates spread over 2048 bins).
        if (sh.count != need) radix_digit(sh, nc, bits_of, 0, 0xffu, true, prefix, mask, need);
        const uint32_t t = prefix, ties_total = sh.count;  // keys equal to t (or the bin's keys, all kept)
        // Ties at t beyond `need`: keep the `need` lowest indices, i.e. those at
        // or below the need-th smallest tie index ti (digits 30-20, 19-9, 8-0 of
        // the ties' indices, ascending; non-ties map to 2^32 - 1 and never match).
        uint32_t ti = 0xffffffffu;
        if (ties_total > need) {
            auto idx_of_tie = [&](int i) {
                const uint2 e = scand[i];
                return e.y == t ? e.x : 0xffffffffu;
            };
            uint32_t ip = 0, im = 0x80000000u, ik = need;
            radix_digit(sh, nc, idx_of_tie, 20, 0x7ffu, false, ip, im, ik);
            radix_digit(sh, nc, idx_of_tie, 9, 0x7ffu, false, ip, im, ik);
            radix_digit(sh, nc, idx_of_tie, 0, 0x1ffu, false, ip, im, ik);
            ti = ip;
        }
        for (int i = tid; i < nc; i += kThreads) {
            const uint2 e = scand[i];
            scand[i].y = e.y > t || (e.y == t && e.x <= ti);
        }
    }

    if constexpr (SPREAD) {
        // The dropped candidates' bits cleared in the unit's bitmap, counted
        // per slice; each slice's first slot; the flag; then this slice.
        uint32_t* dropped = sh.hist;  // [C] (the radix bins are free again)
        __syncthreads();
        for (int i = tid; i < a.C; i += kThreads) dropped[i] = 0u;
        __syncthreads();
        for (int i = tid; i < nc; i += kThreads) {
            const uint2 e = scand[i];
            if (!e.y) {
                atomicAnd(bm + (e.x >> 5), ~(1u << (e.x & 31)));
                atomicAdd(&dropped[e.x / (uint32_t)kSliceKeys], 1u);
            }
        }
        __syncthreads();
        uint32_t mine = 0;
        if (tid < a.C) mine = __ldcg(a.info + u * a.info_stride + tid) - dropped[tid];
        uint32_t total;
        const uint32_t slot = block_exclusive_scan(mine, sh.warp_sums, total);
        if (tid < a.C) a.info[u * a.info_stride + a.C + tid] = slot;
        if (tid == r) sh.base = slot;
        __syncthreads();  // the bits and the slots precede the release below
        if (tid == 0) {
            __threadfence();
            atomicOr(a.done + u, kPublished);
        }
        write_slice(a, u, r, sh.base, sh);
        return;
    }

    // ---- selected keys in index order, tile by tile of the bitmap: the
    // tile's words in shared memory, the candidates that are not selected
    // cleared there, then each thread's run of consecutive words written out
    // from one block-wide scan of their population counts.
    uint32_t out_base = 0;
    for (int w0 = 0; w0 < words; w0 += kTileWords) {
        if (!single) {  // a single CTA's words (one tile at most) are in shared memory already
            __syncthreads();  // the previous tile's words have been read
#pragma unroll
            for (int q = 0; q < kWordsPerThread / 4; ++q)
                *reinterpret_cast<uint4*>(sbits + tid * kWordsPerThread + 4 * q) = tw[q];
        }
        __syncthreads();
        if (!single && w0 + kTileWords < words) load_tile(w0 + kTileWords);
        const uint32_t klo = 32u * (uint32_t)w0, khi = klo + 32u * kTileWords;
        for (int i = tid; i < nc; i += kThreads) {
            const uint2 e = scand[i];
            if (!e.y && e.x >= klo && e.x < khi) atomicAnd(sbits + ((e.x - klo) >> 5), ~(1u << (e.x & 31)));
        }
        __syncthreads();
        uint32_t wv[kWordsPerThread];
#pragma unroll
        for (int q = 0; q < kWordsPerThread; ++q) wv[q] = w0 + tid * kWordsPerThread + q < words ? sbits[tid * kWordsPerThread + q] : 0u;
        uint32_t cnt = 0;
#pragma unroll
        for (int q = 0; q < kWordsPerThread; ++q) cnt += __popc(wv[q]);
        uint32_t total;
        uint32_t pos = out_base + block_exclusive_scan(cnt, sh.warp_sums, total);
        const int wt = w0 + tid * kWordsPerThread;
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

int64_t topk_bitmap_stride(int64_t Ncap) { return (Ncap / 32 + 3) / 4 * 4; }

int64_t topk_info_stride(int64_t Ncap) { return 2 * ((Ncap + kSliceKeys - 1) / kSliceKeys); }

namespace {
int topk_smem_bytes(int cap) { return (int)sizeof(uint2) * cap + 4 * kTileWords; }
}  // namespace

cudaError_t launch_topk(const float* scores, const uint32_t* unit_hist, uint32_t* cand_cnt, uint2* cand,
                        uint32_t* bitmap, uint32_t* done, uint32_t* info, uint32_t* err_word, const DecodeShape& s,
                        int32_t* idx_out, cudaStream_t stream)
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
    a.bm_stride = topk_bitmap_stride(s.Ncap);
    a.N = (int)s.N;
    a.k = s.k;
    a.C = (int)((s.N + kSliceKeys - 1) / kSliceKeys);
    a.cap = topk_candidate_capacity(s.Ncap);
    a.info = info;
    a.err_word = err_word;
    a.info_stride = topk_info_stride(s.Ncap);
    a.max_polls = wait_poll_limit();
    // Every CTA writes its own slice when a unit has many slices (one CTA
    // compacting a long bitmap is slow; with a few slices, CTAs that exit
    // after their ticket free their SMs sooner, which pays more) and the
    // grid (two CTAs per SM) is resident at once.
    a.spread = a.C >= kSpreadMinSlices && a.C <= kSpreadMaxSlices && s.U * a.C <= 2 * (int64_t)device_num_sms() ? 1 : 0;
    auto kern = a.spread ? topk_kernel<true> : topk_kernel<false>;
    cudaError_t e = set_smem_limit_once((const void*)kern, topk_smem_bytes(kTopkCandidates));
    if (e != cudaSuccess) return e;
    return launch_pdl(kern, dim3((unsigned)(s.U * a.C)), dim3(kThreads), (size_t)topk_smem_bytes(a.cap), stream, a);
}

}  // namespace socket_attn
