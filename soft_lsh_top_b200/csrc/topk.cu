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
// lowest-index keys equal to t.
#include "common.cuh"
#include "internal.h"

namespace socket_attn {
namespace {

constexpr int kThreads = 1024;
constexpr int kBins = 2048;
constexpr int kKeysPerThread = 16;
constexpr int kTileKeys = kThreads * kKeysPerThread;

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
        uint32_t w = warp_sums[lane];
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t y = __shfl_up_sync(kFullMask, w, o);
            if (lane >= o) w += y;
        }
        warp_sums[lane] = w;  // inclusive over warps
    }
    __syncthreads();
    total = warp_sums[31];
    const uint32_t before = warp == 0 ? 0u : warp_sums[warp - 1];
    const uint32_t excl = before + x - v;
    __syncthreads();  // warp_sums reusable after return
    return excl;
}

// Grid: U.  Block: kThreads.
__global__ __launch_bounds__(kThreads, 1) void topk_kernel(const float* __restrict__ scores, int64_t Ncap, int N,
                                                           int k, int32_t* __restrict__ idx_out)
{
    __shared__ uint32_t hist[kBins];
    __shared__ uint32_t warp_sums[32];
    __shared__ uint32_t s_digit, s_krem;

    const int tid = threadIdx.x;
    const int64_t u = blockIdx.x;
    const uint32_t* su = reinterpret_cast<const uint32_t*>(scores + u * Ncap);
    int32_t* out = idx_out + u * (int64_t)k;

    uint32_t prefix = 0, mask = 0, krem = (uint32_t)k;
    if (tid == 0) {
        s_digit = 0;
        s_krem = krem;
    }
    const int shifts[3] = {20, 9, 0};
    const int widths[3] = {11, 11, 9};

    for (int pass = 0; pass < 3; ++pass) {
        const int shift = shifts[pass];
        const uint32_t dmask = (1u << widths[pass]) - 1u;
        for (int b = tid; b < kBins; b += kThreads) hist[b] = 0;
        __syncthreads();
        for (int i = tid * 4; i < N; i += kThreads * 4) {
            const uint4 v = *reinterpret_cast<const uint4*>(su + i);
            const uint32_t vals[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int e = 0; e < 4; ++e)
                if (i + e < N && (vals[e] & mask) == prefix) atomicAdd(&hist[(vals[e] >> shift) & dmask], 1u);
        }
        __syncthreads();
        // Thread t owns bins hi = 2047 - 2t and lo = 2046 - 2t (descending order).
        const int hi = kBins - 1 - 2 * tid, lo = hi - 1;
        const uint32_t chi = hist[hi], clo = hist[lo];
        uint32_t total;
        const uint32_t above = block_exclusive_scan(chi + clo, warp_sums, total);
        if (above < krem && krem <= above + chi) {
            s_digit = (uint32_t)hi;
            s_krem = krem - above;
        } else if (above + chi < krem && krem <= above + chi + clo) {
            s_digit = (uint32_t)lo;
            s_krem = krem - above - chi;
        }
        __syncthreads();
        prefix |= s_digit << shift;
        mask |= dmask << shift;
        krem = s_krem;
        __syncthreads();
    }

    // prefix = bit pattern of the k-th largest score; krem = keys equal to it to keep.
    const uint32_t t = prefix, need_ties = krem;
    uint32_t out_base = 0, ties_seen = 0;
    for (int tile = 0; tile < N; tile += kTileKeys) {
        const int i0 = tile + tid * kKeysPerThread;
        uint32_t vals[kKeysPerThread];
#pragma unroll
        for (int q = 0; q < kKeysPerThread / 4; ++q) {
            uint4 v = make_uint4(0, 0, 0, 0);
            if (i0 + 4 * q < N) v = *reinterpret_cast<const uint4*>(su + i0 + 4 * q);
            vals[4 * q + 0] = v.x;
            vals[4 * q + 1] = v.y;
            vals[4 * q + 2] = v.z;
            vals[4 * q + 3] = v.w;
        }
        uint32_t gt = 0, eq = 0;
#pragma unroll
        for (int e = 0; e < kKeysPerThread; ++e) {
            if (i0 + e < N) {
                gt += vals[e] > t;
                eq += vals[e] == t;
            }
        }
        uint32_t total;
        const uint32_t excl = block_exclusive_scan((gt << 16) | eq, warp_sums, total);
        const uint32_t gt_before = excl >> 16, eq_before = excl & 0xffffu;
        const uint32_t budget = need_ties > ties_seen ? need_ties - ties_seen : 0u;
        uint32_t pos = out_base + gt_before + min(eq_before, budget);
        uint32_t my_eq = eq_before;
#pragma unroll
        for (int e = 0; e < kKeysPerThread; ++e) {
            if (i0 + e < N) {
                // pos < k always holds when the threshold is exact; the guard keeps
                // every store inside the unit's k slots regardless.
                if (vals[e] > t) {
                    if (pos < (uint32_t)k) out[pos] = i0 + e;
                    ++pos;
                } else if (vals[e] == t) {
                    if (my_eq < budget) {
                        if (pos < (uint32_t)k) out[pos] = i0 + e;
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

size_t topk_scratch_words(const DecodeShape&) { return 0; }

cudaError_t launch_topk(const float* scores, const DecodeShape& s, uint32_t*, int32_t* idx_out,
                        cudaStream_t stream)
{
    topk_kernel<<<(unsigned)s.U, kThreads, 0, stream>>>(scores, s.Ncap, (int)s.N, s.k, idx_out);
    return cudaGetLastError();
}

}  // namespace socket_attn
