// Top-k selection fused with the exact attention over the selected keys, for
// bfloat16 q, K, V and at most 8 query heads per unit.
//
// Method: "Resumen Técnico: SOCKET ..." (gist.science/es/paper/2602.06283),
// "Mecanismo Central: LSH Suave" step 4 "Selección": the k keys with the
// largest scores are chosen deterministically (ties to the lower index, the
// indices written in ascending order) and exact softmax attention is computed
// over them; "SOCKET: SOft Collision Kernel EsTimator for Sparse Attention"
// (gist.science/de/paper/2602.06283), "Auswahl".
//
// The scoring kernel leaves, per unit, a histogram of the score bit patterns
// >> 19 (scores are non-negative, so the patterns order like the values).
// From it every CTA finds the bin d0 that holds the k-th largest score.  Keys
// above d0 are selected whatever the exact threshold is ("sure" keys); only
// the keys inside d0 (the candidates) need the exact comparison.  So the
// attention over the sure keys need not wait for the selection.
//
// Grid: C slices per unit, one CTA per slice, at most one CTA per SM (the
// grid is resident all at once).  CTA r of unit u:
//   A. finds d0 from the unit histogram (its first score reads in flight);
//   B. reads its slice of scores once (from L2, where the scoring kernel left
//      them) into a bitmap of the sure keys, and appends the candidates
//      (index, bit pattern) to shared memory and to the unit's list;
//   C. takes a ticket; the unit's last CTA to arrive selects among the
//      candidates: the exact k-th pattern t and the highest index ti among
//      the ties at t that are kept (ties go to the lower index), then the
//      number of keys each slice keeps and each slice's first output slot;
//      it publishes (t, ti, slots) with a release flag;
//   D. attends over its sure keys in index order, chunk c of 16 by warp
//      c mod 16: the warp gathers the chunk's key and value rows into its
//      stage (16-byte cp.async copies) and adds them to its online softmax
//      (WarpAttn: both contractions on mma.sync);
//   E. waits (bounded) for the flag; keeps the candidates of its slice with
//      pattern > t, or = t and index <= ti; writes its slice's selection
//      (sure and kept keys, ascending) from its first output slot on; attends
//      over the kept keys;
//   F. merges its 16 warps' softmax states into one partial per head; the
//      unit's last CTA merges the C partials into the output.
// Every merge runs in a fixed order, so the output is deterministic.  The
// flag wait is the only wait on another CTA and the kernel's only wait that
// can fail to end (copies always complete); it is bounded, and on expiry the
// CTA sets SOCKET_DEVERR_SELECT_TIMEOUT in the error word and skips the rest
// of its selection (the outputs are then undefined, as the header states).
//
// This kernel runs where the separate top-k kernel would leave SMs idle (few
// units; see select_attend_supported): every slice of every unit gets an SM.
#include "common.cuh"
#include "internal.h"
#include "select.cuh"
#include "socket_attn.h"
#include "warp_attn.cuh"

namespace socket_attn {
namespace {

using namespace select512;

constexpr int kRoundKeys = 4 * kThreads;           // keys of one read round of the CTA (4 per thread)
constexpr int kRing = 12;                          // read rounds in flight (one 16-byte cp.async per thread each)
constexpr int kRingStageBytes = kThreads * 16;
constexpr int kSliceCand = 1024;                   // a slice's candidates kept in shared memory
constexpr int kMaxSliceKeys = 131072;
constexpr int kMaxWordsPerThread = kMaxSliceKeys / 32 / kThreads;  // 8
constexpr int kMaxK = 4096;
constexpr int kMaxSlices = 256;
constexpr uint32_t kPublished = 0x80000000u;       // set in the unit's ticket word once (t, ti, slots) are out
constexpr int kStagesBytes = kWarps * kWStageBytes;  // one chunk stage per warp
constexpr int kUnitCandMax = kStagesBytes / 8;     // candidates the selecting CTA ranks in shared memory
constexpr int kSliceCandBytes = kSliceCand * 8;
constexpr int kQfragBytes = 8 * 32 * 8;
static_assert(kRing * kRingStageBytes <= kStagesBytes, "the read ring fits the stages");

struct FusedArgs {
    const float* scores;        // [U][Ncap]
    const uint32_t* unit_hist;  // [U][kScoreHistBins]
    uint32_t* cand_cnt;         // [U] candidates appended (zeroed before the step)
    uint2* cand;                // [U][cap] (index, bit pattern)
    uint32_t* info;             // [U][info_stride]: t, ti, sure count [C], first slot [C]
    uint32_t* done;             // [U] slice tickets, then the published flag (zeroed before the step)
    uint32_t* tickets;          // [U] partial tickets (zeroed before the step)
    int32_t* idx_out;           // [U][k]
    const uint16_t* q;          // [U * G][d]
    const uint16_t* K;          // [B][Hkv][Ncap][d]
    const uint16_t* V;
    float* part_o;              // [U][G][C][d] per slice, unnormalised
    float2* part_ml;            // [U][G][C] (largest logit, sum of weights)
    uint32_t* err_word;
    float* out;                 // [U * G][d]
    int64_t Ncap, info_stride;
    int N, k, C, S, cap, share;
    uint32_t max_polls;
};

__device__ __forceinline__ uint32_t ld_acquire(const uint32_t* p)
{
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

template <int G>
__global__ __launch_bounds__(kThreads, 1) void select_attend_kernel(const FusedArgs a)
{
    __shared__ Shared sh;
    __shared__ __align__(8) uint64_t bar[kWarps];
    __shared__ float wm[kWarps][8], wl[kWarps][8];
    __shared__ uint32_t kept_cnt[kMaxSlices];
    __shared__ uint32_t s_t, s_ti, s_slot, s_ok;
    extern __shared__ __align__(128) char dyn[];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int Sw = a.S / 32;  // bitmap words of a slice (a multiple of 64)
    // Stages: the read ring of B; then (selecting CTA) the unit's candidates;
    // then one chunk stage per warp (D, E); then the warps' states (F).
    char* stages = dyn;
    uint2* ucand = reinterpret_cast<uint2*>(stages);
    uint2* scand = reinterpret_cast<uint2*>(stages + kStagesBytes);  // [kSliceCand] this slice's candidates
    uint32_t* sure_w = reinterpret_cast<uint32_t*>(stages + kStagesBytes + kSliceCandBytes);  // [Sw]
    uint32_t* kept_w = sure_w + Sw;                                                           // [Sw]
    uint2* qfrag = reinterpret_cast<uint2*>(kept_w + Sw);
    int32_t* list = reinterpret_cast<int32_t*>(reinterpret_cast<char*>(qfrag) + kQfragBytes);  // [k]

    const int64_t u = blockIdx.x / a.C;
    const int r = blockIdx.x % a.C;
    const int64_t rowbase = (u / a.share) * a.Ncap;  // the unit's first row of K and V
    const int64_t qrow0 = u * G;                     // the unit's query rows of [B][Hq]
    const uint32_t* su = reinterpret_cast<const uint32_t*>(a.scores + u * a.Ncap);
    uint32_t* info = a.info + u * a.info_stride;
    const int lo = r * a.S, hi = min(a.N, lo + a.S);
    const int wpt = (Sw + kThreads - 1) / kThreads;  // bitmap words per thread in the scans (<= 8)

    if (tid < kWarps) mbar_init(&bar[tid], 1);
    if (tid == 0) {
        fence_mbarrier_init();
        sh.count = 0u;
        sh.digit = 0u;
        sh.krem = (uint32_t)a.k;
        sh.bin_count = 0u;
    }
    for (int i = tid; i < Sw; i += kThreads) sure_w[i] = 0u;
    if (tid < kMaxSlices) kept_cnt[tid] = 0u;
    // q is an input of the step, complete before the step's first kernel ran.
    if (tid < 8 * 32) qfrag[tid] = q_fragment<G>(a.q, qrow0, tid >> 5, tid & 31);
    __syncthreads();
    // The grid is resident all at once, so the next kernel's CTAs may be
    // placed now; they wait for this grid to finish before they read anything.
    pdl_launch_dependents();
    pdl_wait();  // scores and histograms come from the previous kernel on the stream

    // ---- A. Round g of this thread covers keys lo + 2048 g + 4 tid .. + 3
    // (lanes 8m .. 8m + 7 of a warp: the 32 keys of one bitmap word).  The
    // thread copies its 16 bytes of round g into ring stage g mod kRing (one
    // commit group per round, empty past the slice) and reads them back
    // itself; the first kRing - 1 rounds are issued right after the
    // histogram's loads, so they stream while d0 is found.
    const int rounds = (hi - lo + kRoundKeys - 1) / kRoundKeys;
    auto key_of = [&](int g) { return lo + g * kRoundKeys + 4 * tid; };
    const uint32_t my_slot = smem_addr(stages) + 16u * (uint32_t)tid;
    auto issue_round = [&](int g) {
        const int n0 = key_of(g);
        if (g < rounds && n0 < hi) cp_async16(my_slot + (uint32_t)(g % kRing) * kRingStageBytes, su + n0);
        cp_async_commit();
    };
    {
        constexpr int kPer = kScoreHistBins / kThreads;  // 8 bins per thread, descending
        const int b0 = kScoreHistBins - 1 - kPer * tid;
        const uint4* hp = reinterpret_cast<const uint4*>(a.unit_hist + u * kScoreHistBins + (b0 - (kPer - 1)));
        uint4 hw[kPer / 4];
#pragma unroll
        for (int qq = 0; qq < kPer / 4; ++qq) hw[qq] = __ldcg(hp + (kPer / 4 - 1 - qq));
#pragma unroll
        for (int g = 0; g < kRing - 1; ++g) issue_round(g);
        uint32_t c[kPer];
#pragma unroll
        for (int qq = 0; qq < kPer / 4; ++qq) {
            c[4 * qq] = hw[qq].w;
            c[4 * qq + 1] = hw[qq].z;
            c[4 * qq + 2] = hw[qq].y;
            c[4 * qq + 3] = hw[qq].x;
        }
        find_bin<kPer>(c, (uint32_t)a.k, sh, [&](int qq) { return (uint32_t)(b0 - qq); });
        __syncthreads();
    }
    const uint32_t d0 = sh.digit, krem0 = sh.krem;
    const uint32_t ncand = sh.bin_count;  // keys of the unit in bin d0
    const bool fits = ncand <= (uint32_t)a.cap;

    // ---- B. one read of the slice.
    uint32_t nsure = 0;
    for (int g = 0; g < rounds; ++g) {
        // Round g has landed once at most kRing - 2 younger groups are pending.
        cp_async_wait<kRing - 2>();
        uint4 x;
        asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
                     : "=r"(x.x), "=r"(x.y), "=r"(x.z), "=r"(x.w)
                     : "r"(my_slot + (uint32_t)(g % kRing) * kRingStageBytes)
                     : "memory");
        // Round g + kRing - 1 goes into the stage read one round ago.
        issue_round(g + kRing - 1);
        if (lo + g * kRoundKeys + 128 * warp >= hi) continue;  // the warp's keys all lie past the slice
        const int n0 = key_of(g);
        const uint32_t vals[4] = {x.x, x.y, x.z, x.w};
        uint32_t gt = 0, eq = 0;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const uint32_t top = vals[j] >> kScoreHistShift;
            const bool live = n0 + j < hi;
            gt |= (uint32_t)(live && top > d0) << j;
            eq |= (uint32_t)(live && top == d0) << j;
        }
        uint32_t wg = gt << ((lane & 7) * 4);
#pragma unroll
        for (int o = 1; o < 8; o <<= 1) wg |= __shfl_xor_sync(kFullMask, wg, o);
        if ((lane & 7) == 0) sure_w[(n0 - lo) >> 5] = wg;  // n0 - lo < rounds * 2048 <= S
        // Candidates -> shared memory (one shared atomic per warp and round
        // that has any); slots >= kSliceCand go to the unit's list at once.
        const uint32_t cnt = fits ? __popc(eq) : 0u;
        if (__any_sync(kFullMask, cnt != 0)) {
            uint32_t incl = cnt;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const uint32_t y = __shfl_up_sync(kFullMask, incl, o);
                if (lane >= o) incl += y;
            }
            uint32_t slot = 0;
            if (lane == 31) slot = atomicAdd(&sh.count, incl);
            slot = __shfl_sync(kFullMask, slot, 31);
            const uint32_t total = __shfl_sync(kFullMask, incl, 31);
            const uint32_t spill_from = max(slot, (uint32_t)kSliceCand);
            uint32_t gbase = 0;
            if (slot + total > spill_from) {
                if (lane == 31) gbase = atomicAdd(a.cand_cnt + u, slot + total - spill_from);
                gbase = __shfl_sync(kFullMask, gbase, 31);
            }
            uint32_t p = slot + incl - cnt;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                if (eq >> j & 1u) {
                    const uint2 c = make_uint2((uint32_t)(n0 + j), vals[j]);
                    if (p < (uint32_t)kSliceCand) scand[p] = c;
                    else if (gbase + (p - spill_from) < (uint32_t)a.cap)  // a subset of the unit's (<= cap)
                        a.cand[u * a.cap + gbase + (p - spill_from)] = c;
                    ++p;
                }
            }
        }
        nsure += __popc(gt);
    }
    cp_async_wait<0>();  // only empty groups remain
    uint32_t my_sure;
    block_exclusive_scan(nsure, sh.warp_sums, my_sure);  // also the barrier after the read
    const uint32_t slice_cand = sh.count;  // candidates this slice found (also those past kSliceCand)

    // ---- C. the candidates to the unit's list, then the ticket.
    const bool own_only = a.C == 1 && slice_cand <= (uint32_t)kSliceCand;  // every candidate is in scand
    if (!own_only) {
        const uint32_t nl = min(slice_cand, (uint32_t)kSliceCand);
        if (tid == 0) {
            sh.base = nl ? atomicAdd(a.cand_cnt + u, nl) : 0u;
            info[2 + r] = my_sure;
        }
        __syncthreads();
        const uint32_t base = sh.base;
        uint2* cu = a.cand + u * a.cap;
        for (uint32_t i = tid; i < nl; i += kThreads)
            if (base + i < (uint32_t)a.cap) cu[base + i] = scand[i];
    }
    // One slice: this CTA selects (after a barrier: its own list entries are
    // written).  Else the last to take a ticket, which then sees the other
    // slices' lists and counts.
    bool selector = true;
    if (a.C > 1) selector = cta_ticket(a.done + u, (uint32_t)(a.C - 1), sh.last);
    else __syncthreads();
    if (selector) {
        uint32_t t, ti = 0xffffffffu;
        if (fits && ncand <= (uint32_t)kUnitCandMax) {
            const int nc = (int)ncand;
            const uint2* selc = own_only ? scand : ucand;
            if (!own_only) {
                const uint2* cu = a.cand + u * a.cap;
                for (int i = tid; i < nc; i += kThreads) ucand[i] = __ldcg(cu + i);
                __syncthreads();
            }
            // The krem0-th largest pattern t among the candidates (two more digits).
            uint32_t prefix = d0 << kScoreHistShift, mask = 0xffffffffu << kScoreHistShift, need = krem0;
            auto bits_of = [&](int i) { return selc[i].y; };
            radix_digit(sh, nc, bits_of, 8, 0x7ffu, true, prefix, mask, need);
            // A bin holding exactly the keys still needed is kept whole: its
            // lowest pattern is the threshold, with no ties to resolve.
            if (sh.count != need) radix_digit(sh, nc, bits_of, 0, 0xffu, true, prefix, mask, need);
            t = prefix;
            // Ties at t beyond `need`: the need lowest indices are kept, i.e. those
            // at or below the need-th smallest tie index ti (digits 30-20, 19-9,
            // 8-0 of the ties' indices; other candidates map to 2^32 - 1).
            if (sh.count > need) {
                auto idx_of_tie = [&](int i) {
                    const uint2 e = selc[i];
                    return e.y == t ? e.x : 0xffffffffu;
                };
                uint32_t ip = 0, im = 0x80000000u, ik = need;
                radix_digit(sh, nc, idx_of_tie, 20, 0x7ffu, false, ip, im, ik);
                radix_digit(sh, nc, idx_of_tie, 9, 0x7ffu, false, ip, im, ik);
                radix_digit(sh, nc, idx_of_tie, 0, 0x1ffu, false, ip, im, ik);
                ti = ip;
            }
            for (int i = tid; i < nc; i += kThreads) {
                const uint2 e = selc[i];
                if (e.y > t || (e.y == t && e.x <= ti)) atomicAdd(&kept_cnt[e.x / (uint32_t)a.S], 1u);
            }
        } else {
            // The threshold bin holds more keys than shared memory takes: the
            // same digits over all of the unit's scores.
            uint32_t prefix = 0, mask = 0, krem = (uint32_t)a.k;
            auto get = [&](int i) { return __ldcg(su + i); };
            radix_digit(sh, a.N, get, 20, 0x7ffu, true, prefix, mask, krem);
            radix_digit(sh, a.N, get, 9, 0x7ffu, true, prefix, mask, krem);
            radix_digit(sh, a.N, get, 0, 0x1ffu, true, prefix, mask, krem);
            t = prefix;
            if (sh.count > krem) {
                auto idx_of_tie = [&](int i) { return __ldcg(su + i) == t ? (uint32_t)i : 0xffffffffu; };
                uint32_t ip = 0, im = 0x80000000u, ik = krem;
                radix_digit(sh, a.N, idx_of_tie, 20, 0x7ffu, false, ip, im, ik);
                radix_digit(sh, a.N, idx_of_tie, 9, 0x7ffu, false, ip, im, ik);
                radix_digit(sh, a.N, idx_of_tie, 0, 0x1ffu, false, ip, im, ik);
                ti = ip;
            }
            for (int i = tid; i < a.N; i += kThreads) {
                const uint32_t x = __ldcg(su + i);
                if ((x >> kScoreHistShift) == d0 && (x > t || (x == t && (uint32_t)i <= ti)))
                    atomicAdd(&kept_cnt[i / a.S], 1u);
            }
        }
        __syncthreads();
        // First output slot of every slice: the keys of the slices before it.
        uint32_t mine = 0;
        if (tid < a.C) mine = (tid == r ? my_sure : __ldcg(info + 2 + tid)) + kept_cnt[tid];
        uint32_t total;
        const uint32_t slot = block_exclusive_scan(mine, sh.warp_sums, total);
        if (tid < a.C) info[2 + a.C + tid] = slot;
        if (tid == r) s_slot = slot;
        if (tid == 0) {
            info[0] = t;
            info[1] = ti;
            s_t = t;
            s_ti = ti;
            s_ok = 1u;
        }
        __syncthreads();  // the record's words precede the release below
        if (tid == 0 && a.C > 1) {
            __threadfence();
            atomicOr(a.done + u, kPublished);
        }
    }

    __syncthreads();  // the stages are free again (ring drained, candidates ranked)

    // The keys of `words` (a bitmap of the slice, per-thread runs of wpt
    // words) in index order -> list[0..), at most k; returns the count.
    auto compact = [&](const uint32_t* words) {
        uint32_t cnt = 0;
        for (int qq = 0; qq < wpt; ++qq) {
            const int wi = tid * wpt + qq;
            if (wi < Sw) cnt += __popc(words[wi]);
        }
        uint32_t total;
        uint32_t pos = block_exclusive_scan(cnt, sh.warp_sums, total);
        for (int qq = 0; qq < wpt; ++qq) {
            const int wi = tid * wpt + qq;
            if (wi >= Sw) break;
            uint32_t x = words[wi];
            while (x) {
                const int b = __ffs(x) - 1;
                x &= x - 1;
                if (pos < (uint32_t)a.k) list[pos] = lo + 32 * wi + b;
                ++pos;
            }
        }
        __syncthreads();
        return (int)min(total, (uint32_t)a.k);
    };
    // Attention over list[0..n): chunk c of 16 by warp c mod 16.
    WarpAttn<G, true> at;
    at.init(qfrag);
    char* stw = stages + warp * kWStageBytes;
    auto attend = [&](int n) {
        for (int c = warp; c * kWChunk < n; c += kWarps) {
            const int nr = min(kWChunk, n - c * kWChunk);
            int32_t key = (lane & 15) < nr ? list[c * kWChunk + (lane & 15)] : 0;
            key = min(max(key, 0), a.N - 1);  // a gather never leaves the unit's rows
            at.issue_lsu(stw, a.K, a.V, rowbase + key, nr);
            cp_async_wait<0>();
            __syncwarp();
            at.consume(smem_addr(stw), nr);
        }
    };

    // ---- D. the sure keys.
    attend(compact(sure_w));
    __syncthreads();  // every warp is done with the list

    // ---- E. the selection's outcome for this slice.
    if (!selector) {
        if (tid == 0) {
            bool got = false;
            for (uint32_t polls = 0; polls < a.max_polls; ++polls) {
                if (ld_acquire(a.done + u) & kPublished) {
                    got = true;
                    break;
                }
                __nanosleep(128);
            }
            s_ok = got ? 1u : 0u;
            if (got) {
                s_t = __ldcg(info);
                s_ti = __ldcg(info + 1);
                s_slot = __ldcg(info + 2 + a.C + r);
            } else {
                atomicOr(a.err_word, SOCKET_DEVERR_SELECT_TIMEOUT);
            }
        }
    }
    __syncthreads();
    if (s_ok) {
        const uint32_t t = s_t, ti = s_ti;
        // Kept candidates of the slice -> kept_w: from scand when it holds them
        // all, else from a second read of the slice's scores.
        for (int i = tid; i < Sw; i += kThreads) kept_w[i] = 0u;
        __syncthreads();
        if (fits && slice_cand <= (uint32_t)kSliceCand) {
            for (uint32_t i = tid; i < slice_cand; i += kThreads) {
                const uint2 e = scand[i];
                if (e.y > t || (e.y == t && e.x <= ti)) atomicOr(&kept_w[(e.x - lo) >> 5], 1u << (e.x & 31));
            }
        } else {
            for (int n = lo + tid; n < hi; n += kThreads) {
                const uint32_t x = __ldcg(su + n);
                if ((x >> kScoreHistShift) == d0 && (x > t || (x == t && (uint32_t)n <= ti)))
                    atomicOr(&kept_w[(n - lo) >> 5], 1u << (n & 31));
            }
        }
        __syncthreads();
        uint32_t kcnt = 0, fcnt = 0;
#pragma unroll
        for (int qq = 0; qq < kMaxWordsPerThread; ++qq) {
            const int wi = tid * wpt + qq;
            if (qq < wpt && wi < Sw) {
                kcnt += __popc(kept_w[wi]);
                fcnt += __popc(sure_w[wi] | kept_w[wi]);
            }
        }
        uint32_t ktot, ftot;
        uint32_t kpos = block_exclusive_scan(kcnt, sh.warp_sums, ktot);
        uint32_t fpos = s_slot + block_exclusive_scan(fcnt, sh.warp_sums, ftot);
        int32_t* outi = a.idx_out + u * (int64_t)a.k;
#pragma unroll
        for (int qq = 0; qq < kMaxWordsPerThread; ++qq) {
            const int wi = tid * wpt + qq;
            if (qq < wpt && wi < Sw) {
                const uint32_t kq = kept_w[wi];
                uint32_t x = sure_w[wi] | kq;
                while (x) {
                    const int b = __ffs(x) - 1;
                    x &= x - 1;
                    const int32_t key = lo + 32 * wi + b;
                    // fpos < k whenever the threshold is exact; the guards keep every
                    // store inside the unit's k slots regardless.
                    if (fpos < (uint32_t)a.k) outi[fpos] = key;
                    ++fpos;
                    if (kq >> b & 1u) {
                        if (kpos < (uint32_t)a.k) list[kpos] = key;
                        ++kpos;
                    }
                }
            }
        }
        __syncthreads();
        attend((int)min(ktot, (uint32_t)a.k));
    }

    // ---- F. this slice's partial: the 16 warps' states merged per head.
    __syncthreads();  // every stage is idle
    float* o_sm = reinterpret_cast<float*>(stages);  // [16 warps][8 heads][d]
    at.store(o_sm + warp * 8 * kHeadDim, wm[warp], wl[warp]);
    __syncthreads();
    for (int e = tid; e < G * kHeadDim; e += kThreads) {
        const int h = e / kHeadDim, ch = e % kHeadDim;
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) M = fmaxf(M, wm[w][h]);
        float o = 0.0f, l = 0.0f;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) {
            const float wt = wm[w][h] == -INFINITY ? 0.0f : expf(wm[w][h] - M);
            o += wt * o_sm[(w * 8 + h) * kHeadDim + ch];
            l += wt * wl[w][h];
        }
        const int64_t p = (qrow0 + h) * a.C + r;  // [U][G][C]
        a.part_o[p * kHeadDim + ch] = o;
        if (ch == 0) a.part_ml[p] = make_float2(M, l);
    }
    if (!cta_ticket(a.tickets + u, (uint32_t)(a.C - 1), sh.last)) return;
    // The unit's output: the C slice partials merged per head in slice order,
    // 16 slices at a time with all their loads in flight, and a running
    // maximum rescaling the tiles already summed.
    constexpr int kMergeTile = 16;
    for (int e = tid; e < G * kHeadDim; e += kThreads) {
        const int h = e / kHeadDim, ch = e % kHeadDim;
        const float2* pml = a.part_ml + (qrow0 + h) * a.C;
        const float* po = a.part_o + (qrow0 + h) * a.C * kHeadDim + ch;
        float M = -INFINITY, o = 0.0f, l = 0.0f;
        for (int s0 = 0; s0 < a.C; s0 += kMergeTile) {
            float2 ml[kMergeTile];
            float ov[kMergeTile];
#pragma unroll
            for (int j = 0; j < kMergeTile; ++j) {
                const bool in = s0 + j < a.C;
                ml[j] = in ? __ldcg(pml + s0 + j) : make_float2(-INFINITY, 0.0f);
                ov[j] = in ? __ldcg(po + (int64_t)(s0 + j) * kHeadDim) : 0.0f;
            }
            float mt = -INFINITY;
#pragma unroll
            for (int j = 0; j < kMergeTile; ++j) mt = fmaxf(mt, ml[j].x);
            const float Mn = fmaxf(M, mt);
            if (Mn == -INFINITY) continue;
            const float sc = M == -INFINITY ? 0.0f : expf(M - Mn);
            o *= sc;
            l *= sc;
#pragma unroll
            for (int j = 0; j < kMergeTile; ++j) {
                const float wt = ml[j].x == -INFINITY ? 0.0f : expf(ml[j].x - Mn);
                o += wt * ov[j];
                l += wt * ml[j].y;
            }
            M = Mn;
        }
        a.out[(qrow0 + h) * kHeadDim + ch] = l > 0.0f ? o / l : 0.0f;
    }
    if (tid == 0) {
        a.done[u] = 0u;
        a.tickets[u] = 0u;
    }
}

int slice_keys(int64_t N, int C) { return (int)(((N + C - 1) / C + kRoundKeys - 1) / kRoundKeys * kRoundKeys); }

int smem_bytes(int S, int k) { return kStagesBytes + kSliceCandBytes + 2 * (S / 32) * 4 + kQfragBytes + (k + 3) / 4 * 16; }

}  // namespace

int select_attend_slices(const DecodeShape& s, int num_sms)
{
    int64_t C = max64(1, num_sms / max64(1, s.U));
    C = min64(C, (s.k + kWChunk - 1) / kWChunk);
    C = min64(C, (s.N + kRoundKeys - 1) / kRoundKeys);
    C = min64(max64(C, 1), kMaxSlices);
    const int S = slice_keys(s.N, (int)C);
    return (int)((s.N + S - 1) / S);
}

bool select_attend_supported(int kv_dtype, int q_dtype, const DecodeShape& s, int num_sms)
{
    if (kv_dtype != SOCKET_BF16 || q_dtype != SOCKET_BF16 || s.G > 8 || s.d != kHeadDim) return false;
    if (s.k > kMaxK || s.U > num_sms || s.N > (int64_t(1) << 30)) return false;
    // Only where the separate top-k kernel (one CTA per 32768 keys of a unit)
    // would not fill the SMs: with more units the two-kernel path is faster.
    if (s.U * ((s.N + 32767) / 32768) >= num_sms) return false;
    const int C = select_attend_slices(s, num_sms);
    return slice_keys(s.N, C) <= kMaxSliceKeys && 2 + 2 * (int64_t)C <= topk_bitmap_stride(s.Ncap);
}

cudaError_t launch_select_attend(const float* scores, const uint32_t* unit_hist, uint32_t* cand_cnt, uint2* cand,
                                 uint32_t* info, uint32_t* done, uint32_t* tickets, const void* q, const void* K,
                                 const void* V, const DecodeShape& s, float* part_o, float2* part_ml,
                                 uint32_t* err_word, int32_t* idx_out, float* out, cudaStream_t stream)
{
    FusedArgs a;
    a.scores = scores;
    a.unit_hist = unit_hist;
    a.cand_cnt = cand_cnt;
    a.cand = cand;
    a.info = info;
    a.done = done;
    a.tickets = tickets;
    a.idx_out = idx_out;
    a.q = static_cast<const uint16_t*>(q);
    a.K = static_cast<const uint16_t*>(K);
    a.V = static_cast<const uint16_t*>(V);
    a.part_o = part_o;
    a.part_ml = part_ml;
    a.err_word = err_word;
    a.out = out;
    a.Ncap = s.Ncap;
    a.info_stride = topk_bitmap_stride(s.Ncap);
    a.N = (int)s.N;
    a.k = s.k;
    a.C = s.nsplit;
    a.S = slice_keys(s.N, a.C);
    a.cap = topk_candidate_capacity(s.Ncap);
    a.share = s.share;
    a.max_polls = wait_poll_limit();
    const dim3 grid((unsigned)(s.U * a.C)), block(kThreads);
    const int smem = smem_bytes(a.S, a.k);
#define SOCKET_FUSED_CASE(g)                                                                          \
    case g: {                                                                                         \
        cudaError_t e = set_smem_limit_once((const void*)select_attend_kernel<g>,                     \
                                            smem_bytes(kMaxSliceKeys, kMaxK));                        \
        if (e != cudaSuccess) return e;                                                               \
        e = launch_pdl(select_attend_kernel<g>, grid, block, (size_t)smem, stream, a);                \
        if (e != cudaSuccess) return e;                                                               \
        return cudaGetLastError();                                                                    \
    }
    switch (s.G) {
        SOCKET_FUSED_CASE(1) SOCKET_FUSED_CASE(2) SOCKET_FUSED_CASE(3) SOCKET_FUSED_CASE(4)
        SOCKET_FUSED_CASE(5) SOCKET_FUSED_CASE(6) SOCKET_FUSED_CASE(7) SOCKET_FUSED_CASE(8)
        default: return cudaErrorInvalidValue;
    }
#undef SOCKET_FUSED_CASE
}

}  // namespace socket_attn
