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
// values.  A three-digit radix select (11 + 11 + 9 bits of the 31 magnitude
// bits) finds the k-th largest pattern t and how many keys equal to t are
// needed; one ordered compaction pass then keeps every key above t plus the
// lowest-index keys equal to t.  A unit is handled by a thread-block cluster
// of up to 16 CTAs that exchange histograms and counts through distributed
// shared memory, so no global scratch and no second kernel are needed.
#include <cooperative_groups.h>

#include "common.cuh"
#include "internal.h"

namespace cg = cooperative_groups;

namespace socket_attn {
namespace {

constexpr int kThreads = 512;
constexpr int kBins = 2048;
constexpr int kBinsPerThread = kBins / kThreads;      // 4
constexpr int kKeysPerThread = 16;                    // compaction: 16 consecutive keys per thread
constexpr int kTileKeys = kThreads * kKeysPerThread;  // 8192
constexpr int kSliceKeys = 16384;                     // target keys per CTA of a cluster
constexpr int kCacheKeys = 16384;                     // keys of the CTA's slice kept in shared memory
constexpr int kMaxCluster = 16;
constexpr int kWindowShift = 15;                      // first-digit bin = 2^15 ulps (1/256 octave)

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
        uint32_t w = lane < kThreads / 32 ? warp_sums[lane] : 0u;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t y = __shfl_up_sync(kFullMask, w, o);
            if (lane >= o) w += y;
        }
        if (lane < kThreads / 32) warp_sums[lane] = w;  // inclusive over warps
    }
    __syncthreads();
    total = warp_sums[kThreads / 32 - 1];
    const uint32_t before = warp == 0 ? 0u : warp_sums[warp - 1];
    const uint32_t excl = before + x - v;
    __syncthreads();  // warp_sums reusable after return
    return excl;
}

// Position of 16-byte chunk c in the shared cache: XOR swizzle that keeps both
// the coalesced pattern (chunk = base + lane) and the compaction pattern
// (chunk = 4 * lane + q) free of bank conflicts.
__device__ __forceinline__ int cache_pos(int c) { return c ^ ((c >> 3) & 3); }

// Grid: U * C CTAs in clusters of C (one cluster per unit).  CTA r of a
// cluster owns keys [r*R, min(N, (r+1)*R)) of its unit and keeps up to
// kCacheKeys of them in shared memory.  Three radix digits of the score bit
// pattern select the k-th largest: the first digit covers the 8 octaves
// below the unit's largest score in 2048 bins of 1/256 octave (spread scores
// over many bins, so the shared-memory atomics rarely collide); if fewer
// than k keys fall in that window, the first digit is redone over the full
// range (bits 30-20).  Every CTA sums the cluster's histograms through
// distributed shared memory and picks the same digit.  Then each CTA counts
// its keys above the threshold and equal to it; the counts of lower-ranked
// CTAs give its output offset and tie budget, and it writes its selected
// indices in index order.
__global__ __launch_bounds__(kThreads) void topk_kernel(const float* __restrict__ scores,
                                                        const uint32_t* __restrict__ unit_max, int64_t Ncap,
                                                        int N, int k, int R, int32_t* __restrict__ idx_out)
{
    extern __shared__ uint4 cache[];
    __shared__ uint32_t hist[kBins];
    __shared__ uint32_t warp_sums[32];
    __shared__ uint32_t s_digit, s_krem, s_total;
    __shared__ uint32_t s_counts[2];

    cg::cluster_group cluster = cg::this_cluster();
    const unsigned rank = cluster.block_rank(), C = cluster.num_blocks();
    const int tid = threadIdx.x;
    const int64_t u = blockIdx.x / C;
    const uint32_t* su = reinterpret_cast<const uint32_t*>(scores + u * Ncap);
    int32_t* out = idx_out + u * (int64_t)k;
    const int lo = (int)min64((int64_t)rank * R, N), hi = (int)min64((int64_t)lo + R, N);
    const int n = hi - lo, ncache = min(n, kCacheKeys);

    pdl_wait();  // scores and the unit maxima come from the previous kernel on the stream

    const uint32_t maxbits = __ldcg(unit_max + u);
    for (int i = tid * 4; i < ncache; i += kThreads * 4)
        cache[cache_pos(i >> 2)] = __ldcg(reinterpret_cast<const uint4*>(su + lo + i));
    // Four keys starting at offset i (a multiple of 4) of the CTA's range.
    auto get4 = [&](int i) -> uint4 {
        return i < ncache ? cache[cache_pos(i >> 2)] : __ldcg(reinterpret_cast<const uint4*>(su + lo + i));
    };

    const uint32_t dmax = maxbits >> kWindowShift;
    const uint32_t dlow = dmax >= (uint32_t)(kBins - 1) ? dmax - (kBins - 1) : 0u;
    bool windowed = true;
    uint32_t prefix = 0, mask = 0, krem = (uint32_t)k;
    if (tid == 0) {
        s_digit = 0;
        s_krem = krem;
    }
    for (int pass = 0; pass < 3; ++pass) {
        // Digit of this pass: bits [shift, shift + width) of the pattern
        // (the first windowed digit is taken relative to dlow).
        int shift, width;
        if (windowed) {
            shift = pass == 0 ? kWindowShift : pass == 1 ? 4 : 0;
            width = pass == 0 ? 17 : pass == 1 ? 11 : 4;
        } else {
            shift = pass == 0 ? 20 : pass == 1 ? 9 : 0;
            width = pass == 0 ? 11 : pass == 1 ? 11 : 9;
        }
        const uint32_t dmask = width >= 32 ? 0xffffffffu : (1u << width) - 1u;
        for (int b = tid; b < kBins; b += kThreads) hist[b] = 0;
        __syncthreads();
        for (int i = tid * 4; i < n; i += kThreads * 4) {
            const uint4 v = get4(i);
            const uint32_t vals[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                if (i + e < n) {
                    const uint32_t x = vals[e];
                    if (pass == 0 && windowed) {
                        const uint32_t dgt = x >> kWindowShift;
                        if (dgt >= dlow) atomicAdd(&hist[min(dgt - dlow, (uint32_t)(kBins - 1))], 1u);
                    } else if ((x & mask) == prefix) {
                        atomicAdd(&hist[(x >> shift) & dmask], 1u);
                    }
                }
            }
        }
        cluster.sync();  // every CTA's histogram is complete
        // Thread t owns bins b0, b0-1, b0-2, b0-3 with b0 = 2047 - 4t (descending order).
        const int b0 = kBins - 1 - kBinsPerThread * tid;
        uint32_t c[kBinsPerThread] = {0, 0, 0, 0};
        for (unsigned r = 0; r < C; ++r) {
            const uint32_t* rh = cluster.map_shared_rank(hist, r);
#pragma unroll
            for (int q = 0; q < kBinsPerThread; ++q) c[q] += rh[b0 - q];
        }
        uint32_t total;
        uint32_t run = block_exclusive_scan(c[0] + c[1] + c[2] + c[3], warp_sums, total);
#pragma unroll
        for (int q = 0; q < kBinsPerThread; ++q) {
            if (run < krem && krem <= run + c[q]) {
                s_digit = (uint32_t)(b0 - q);
                s_krem = krem - run;
            }
            run += c[q];
        }
        if (tid == 0) s_total = total;
        cluster.sync();  // remote histograms read; s_digit, s_total visible
        if (pass == 0 && windowed && s_total < krem) {
            // The k-th largest score lies below the window: redo the first
            // digit over the full range.
            windowed = false;
            pass = -1;
            continue;
        }
        if (pass == 0 && windowed) {
            prefix = (s_digit + dlow) << kWindowShift;
            mask = 0xffffffffu << kWindowShift;
        } else {
            prefix |= s_digit << shift;
            mask |= dmask << shift;
        }
        krem = s_krem;
    }

    // prefix = bit pattern of the unit's k-th largest score; krem = keys equal
    // to it that are kept (the lowest-index ones).
    const uint32_t t = prefix, need_ties = krem;
    uint32_t gt = 0, eq = 0;
    for (int i = tid * 4; i < n; i += kThreads * 4) {
        const uint4 v = get4(i);
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
    block_exclusive_scan(gt, warp_sums, tot_gt);
    block_exclusive_scan(eq, warp_sums, tot_eq);
    if (tid == 0) {
        s_counts[0] = tot_gt;
        s_counts[1] = tot_eq;
    }
    cluster.sync();
    uint32_t out_base = 0, ties_before = 0;
    for (unsigned r = 0; r < rank; ++r) {
        const uint32_t* rc = cluster.map_shared_rank(s_counts, r);
        const uint32_t rgt = rc[0], req = rc[1];
        const uint32_t budget = need_ties > ties_before ? need_ties - ties_before : 0u;
        out_base += rgt + min(req, budget);
        ties_before += req;
    }
    cluster.sync();  // no remote shared-memory access after this point

    uint32_t ties_seen = ties_before;
    for (int tile = 0; tile < n; tile += kTileKeys) {
        const int i0 = tile + tid * kKeysPerThread;
        uint32_t vals[kKeysPerThread];
#pragma unroll
        for (int q = 0; q < kKeysPerThread / 4; ++q) {
            uint4 v = make_uint4(0, 0, 0, 0);
            if (i0 + 4 * q < n) v = get4(i0 + 4 * q);
            vals[4 * q + 0] = v.x;
            vals[4 * q + 1] = v.y;
            vals[4 * q + 2] = v.z;
            vals[4 * q + 3] = v.w;
        }
        uint32_t tgt = 0, teq = 0;
#pragma unroll
        for (int e = 0; e < kKeysPerThread; ++e) {
            if (i0 + e < n) {
                tgt += vals[e] > t;
                teq += vals[e] == t;
            }
        }
        uint32_t total;
        const uint32_t excl = block_exclusive_scan((tgt << 16) | teq, warp_sums, total);
        const uint32_t gt_before = excl >> 16, eq_before = excl & 0xffffu;
        const uint32_t budget = need_ties > ties_seen ? need_ties - ties_seen : 0u;
        uint32_t pos = out_base + gt_before + min(eq_before, budget);
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
                    if (my_eq < budget) {
                        if (pos < (uint32_t)k) out[pos] = lo + i0 + e;
                        ++pos;
                    }
                    ++my_eq;
                }
            }
        }
        out_base += (total >> 16) + min(total & 0xffffu, budget);
        ties_seen += total & 0xffffu;
    }
}

}  // namespace

cudaError_t launch_topk(const float* scores, const uint32_t* unit_max, const DecodeShape& s, int32_t* idx_out,
                        cudaStream_t stream)
{
    const int64_t want = (s.N + kSliceKeys - 1) / kSliceKeys;
    const int C = (int)max64(1, min64(kMaxCluster, want));
    const int R = (int)(((s.N + C - 1) / C + 31) / 32 * 32);
    const int smem = (int)min64(R, kCacheKeys) * 4;
    cudaError_t e = cudaFuncSetAttribute(topk_kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kCacheKeys * 4);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(s.U * C));
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = (size_t)smem;
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
    e = cudaLaunchKernelEx(&cfg, topk_kernel, scores, unit_max, s.Ncap, (int)s.N, s.k, R, idx_out);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace socket_attn
