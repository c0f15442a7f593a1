// Soft collision scoring: score(n) = vnorm(n) * sum_l T_l[id_l(n)] for every
// live key of every unit, where T_l is the unit's summed soft-assignment
// table of hash table l.
//
// Method: "Resumen Técnico: SOCKET ..." (gist.science/es/paper/2602.06283),
// "Mecanismo Central: LSH Suave" step 3 "Puntuación"; "SOCKET: SOft Collision
// Kernel EsTimator for Sparse Attention" (gist.science/de/paper/2602.06283),
// "Bewertung": the probability mass the query puts on the key's own bucket,
// aggregated over the L tables and weighted by the key's value norm.  The
// pages implement this step as "a custom CUDA scoring kernel"
// ("Contribuciones Clave" 2 / "Hauptbeiträge").
//
// B200 design.  The step streams L + 4 bytes per key from HBM (one uint8 id
// per table, table-major, plus the fp32 norm) and performs L random lookups
// into 2^P-entry tables.  Lookups go to shared memory in a lane-private
// layout: a buffer holds two tables as float[256 buckets][2 tables][32 lanes],
// so lane j only ever touches bank j and a warp's 32 lookups are one
// conflict-free wavefront whatever the ids are.  One byte-permute builds the
// address (id << 8) | (lane << 2) straight from the packed id word.  Each
// thread keeps 64 keys' accumulators in registers across all L tables, so a
// pass covers 32768 keys per CTA and the 64 KB table staging per table pair
// is amortised over them.  Ids are read with 16-byte streaming loads one table
// ahead in registers and several tables ahead through bulk L2 prefetches.
// The grid is persistent (at most one CTA per SM) and splits the flattened
// (unit, key-group) range evenly, so every SM streams the same byte count.
#include "common.cuh"
#include "internal.h"

namespace socket_attn {
namespace {

constexpr int kThreads = 512;
constexpr int kGroupsPerThread = 4;                      // 16-key groups per thread per pass
constexpr int kPassGroups = kThreads * kGroupsPerThread;  // 2048 groups = 32768 keys
constexpr int kBufFloats = 256 * 2 * 32;                 // [bucket][table pair][lane]
constexpr int kBufBytes = kBufFloats * 4;                // 64 KB
constexpr int kSmemBytes = 2 * kBufBytes;                // double-buffered
constexpr int kStageSlots = kBufFloats / 4 / kThreads;   // float4 stores per thread per buffer (8)
constexpr int kPrefetchAhead = 3;                        // tables prefetched into L2 ahead

struct Pass {
    int64_t unit;
    int64_t first_group;  // first 16-key group of the pass inside the unit
    int npg;              // groups in the pass (<= kPassGroups)
};

__device__ __forceinline__ void load_ids(uint4 (&v)[kGroupsPerThread], const uint8_t* row, int npg, int tid)
{
#pragma unroll
    for (int j = 0; j < kGroupsPerThread; ++j) {
        const int g = j * kThreads + tid;
        v[j] = g < npg ? ldg_stream_u4(row + (int64_t)g * 16) : make_uint4(0, 0, 0, 0);
    }
}

// Accumulate one table's contribution.  `tab` points at the table's column
// block inside a staging buffer (buffer base + 128 * table-in-pair).
__device__ __forceinline__ void lookup(float (&acc)[kGroupsPerThread][16], const uint4 (&v)[kGroupsPerThread],
                                       const char* tab, uint32_t lane4)
{
#pragma unroll
    for (int j = 0; j < kGroupsPerThread; ++j) {
        const uint32_t words[4] = {v[j].x, v[j].y, v[j].z, v[j].w};
#pragma unroll
        for (int w = 0; w < 4; ++w) {
#pragma unroll
            for (int byte = 0; byte < 4; ++byte) {
                // result byte 0 = lane*4, byte 1 = id, bytes 2-3 = 0  ->  (id << 8) | (lane << 2)
                const uint32_t off = __byte_perm(lane4, words[w], 0x1140u + (byte << 4));
                acc[j][w * 4 + byte] += *reinterpret_cast<const float*>(tab + off);
            }
        }
    }
}

__global__ __launch_bounds__(kThreads, 1) void score_kernel(
    const float* __restrict__ tables, const uint8_t* __restrict__ ids, const float* __restrict__ vnorm,
    float* __restrict__ scores, int L, int NB, int64_t Ncap, int64_t groups_per_unit, int64_t total_groups,
    int64_t groups_per_cta)
{
    extern __shared__ __align__(128) char smem[];
    const int tid = threadIdx.x;
    const uint32_t lane4 = (uint32_t)(tid & 31) << 2;
    const int nbuf = (L + 1) >> 1;

    int64_t g0 = (int64_t)blockIdx.x * groups_per_cta;
    const int64_t g1 = min(total_groups, g0 + groups_per_cta);

    while (g0 < g1) {
        Pass ps;
        ps.unit = g0 / groups_per_unit;
        ps.first_group = g0 % groups_per_unit;
        ps.npg = (int)min64(min64(g1 - g0, groups_per_unit - ps.first_group), kPassGroups);
        g0 += ps.npg;

        const float* tu = tables + ps.unit * L * (int64_t)NB;
        const uint8_t* idu = ids + ps.unit * L * Ncap + ps.first_group * 16;
        const float* vu = vnorm + ps.unit * Ncap + ps.first_group * 16;
        float* su = scores + ps.unit * Ncap + ps.first_group * 16;
        const uint32_t pass_bytes = (uint32_t)ps.npg * 16u;

        if (tid == 0) {
            prefetch_l2_bulk(vu, pass_bytes * 4u);
            for (int l = 0; l < min(L, kPrefetchAhead); ++l) prefetch_l2_bulk(idu + l * Ncap, pass_bytes);
        }

        // Stage values for buffer bi: float4 slot e = i*kThreads + tid holds
        // bucket e >> 4, table-in-pair (e >> 3) & 1, four lanes' copies.
        float stage[kStageSlots];
        auto load_stage = [&](int bi) {
#pragma unroll
            for (int i = 0; i < kStageSlots; ++i) {
                const int e = i * kThreads + tid;
                const int bucket = e >> 4, l = 2 * bi + ((e >> 3) & 1);
                stage[i] = (bucket < NB && l < L) ? __ldg(tu + (int64_t)l * NB + bucket) : 0.0f;
            }
        };
        auto store_stage = [&](int buf) {
            float4* dst = reinterpret_cast<float4*>(smem + buf * kBufBytes);
#pragma unroll
            for (int i = 0; i < kStageSlots; ++i) {
                const int e = i * kThreads + tid;
                if ((e >> 4) < NB) dst[e] = make_float4(stage[i], stage[i], stage[i], stage[i]);
            }
        };

        __syncthreads();  // previous pass finished reading both buffers
        load_stage(0);
        store_stage(0);
        if (nbuf > 1) load_stage(1);
        __syncthreads();

        float acc[kGroupsPerThread][16];
#pragma unroll
        for (int j = 0; j < kGroupsPerThread; ++j)
#pragma unroll
            for (int e = 0; e < 16; ++e) acc[j][e] = 0.0f;

        uint4 cur[kGroupsPerThread];
        load_ids(cur, idu, ps.npg, tid);

        for (int bi = 0; bi < nbuf; ++bi) {
            const char* buf = smem + (bi & 1) * kBufBytes;
#pragma unroll
            for (int tt = 0; tt < 2; ++tt) {
                const int l = 2 * bi + tt;
                if (l < L) {
                    if (tid == 0 && l + kPrefetchAhead < L)
                        prefetch_l2_bulk(idu + (l + kPrefetchAhead) * Ncap, pass_bytes);
                    uint4 nxt[kGroupsPerThread];
                    if (l + 1 < L) load_ids(nxt, idu + (l + 1) * Ncap, ps.npg, tid);
                    lookup(acc, cur, buf + tt * 128, lane4);
                    if (l + 1 < L) {
#pragma unroll
                        for (int j = 0; j < kGroupsPerThread; ++j) cur[j] = nxt[j];
                    }
                }
            }
            if (bi + 1 < nbuf) {
                store_stage((bi + 1) & 1);
                if (bi + 2 < nbuf) load_stage(bi + 2);
            }
            __syncthreads();
        }

#pragma unroll
        for (int j = 0; j < kGroupsPerThread; ++j) {
            const int g = j * kThreads + tid;
            if (g < ps.npg) {
#pragma unroll
                for (int w = 0; w < 4; ++w) {
                    const float4 vn = ldg_stream_f4(vu + (int64_t)g * 16 + w * 4);
                    float4 sc;
                    sc.x = acc[j][w * 4 + 0] * vn.x;
                    sc.y = acc[j][w * 4 + 1] * vn.y;
                    sc.z = acc[j][w * 4 + 2] * vn.z;
                    sc.w = acc[j][w * 4 + 3] * vn.w;
                    *reinterpret_cast<float4*>(su + (int64_t)g * 16 + w * 4) = sc;
                }
            }
        }
    }
}

int num_sms()
{
    int dev = 0, n = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    return n > 0 ? n : 1;
}

}  // namespace

cudaError_t launch_score(const float* tables, const uint8_t* ids, const float* vnorm, const DecodeShape& s,
                         float* scores, cudaStream_t stream)
{
    const int64_t gpu = (s.N + 15) / 16;
    const int64_t total = s.U * gpu;
    // At least ~8192 keys per CTA so the table staging stays amortised.
    const int64_t want = (total + 511) / 512;
    const int grid = (int)max64(1, min64(num_sms(), want));
    const int64_t per_cta = (total + grid - 1) / grid;
    cudaError_t e = cudaFuncSetAttribute(score_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return e;
    score_kernel<<<grid, kThreads, kSmemBytes, stream>>>(tables, ids, vnorm, scores, s.L, s.NB, s.Ncap, gpu,
                                                          total, per_cta);
    return cudaGetLastError();
}

}  // namespace socket_attn
