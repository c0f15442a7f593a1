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
// conflict-free wavefront whatever the ids are.  The buffers sit at 64 KB-
// aligned shared addresses, so one byte-permute of the packed id word yields
// the full shared address of a lookup.  Each
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
constexpr uint32_t kBufBytes = 1u << 16;                 // [bucket 256][table pair 2][lane 32] floats
constexpr int kStageSlots = kBufBytes / 16 / kThreads;   // float4 stores per thread per buffer (8)
constexpr int kPrefetchAhead = 4;                        // tables prefetched into L2 ahead
// The two staging buffers sit at 64 KB-aligned shared addresses A and
// A + 64 KB.  A lookup address is then A_buf | (id << 8) | (tt << 7) | (lane << 2):
// one byte-permute of the packed id word with a per-thread base that already
// holds A_buf, the table-in-pair and the lane.  The dynamic allocation spans
// three 64 KB windows so an aligned pair fits wherever the window starts.
constexpr int kSmemBytes = 3 * (int)kBufBytes;

__device__ __forceinline__ void load_ids(uint4 (&v)[kGroupsPerThread], const uint8_t* row, int npg, int tid)
{
#pragma unroll
    for (int j = 0; j < kGroupsPerThread; ++j) {
        const int g = j * kThreads + tid;
        v[j] = g < npg ? ldg_stream_u4(row + (int64_t)g * 16) : make_uint4(0, 0, 0, 0);
    }
}

__device__ __forceinline__ float lds_f32(uint32_t addr)
{
    float v;
    asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(addr));
    return v;
}

// Accumulate one table's contribution for this thread's live groups.
// `base` = shared address of the buffer | (table-in-pair << 7) | (lane << 2),
// whose byte 1 is zero.
__device__ __forceinline__ void lookup(float (&acc)[kGroupsPerThread][16], const uint4 (&v)[kGroupsPerThread],
                                       uint32_t base, int npg, int tid)
{
#pragma unroll
    for (int j = 0; j < kGroupsPerThread; ++j) {
        if (j * kThreads + tid < npg) {
            const uint32_t words[4] = {v[j].x, v[j].y, v[j].z, v[j].w};
#pragma unroll
            for (int w = 0; w < 4; ++w) {
#pragma unroll
                for (int byte = 0; byte < 4; ++byte) {
                    // bytes 0, 2, 3 from base; byte 1 = the id
                    const uint32_t addr = __byte_perm(base, words[w], 0x3240u + (byte << 4));
                    acc[j][w * 4 + byte] += lds_f32(addr);
                }
            }
        }
    }
}

// One pass: groups [first_group, first_group + npg) of one unit, npg <= kPassGroups.
__device__ __forceinline__ void score_pass(const float* __restrict__ tables, const uint8_t* __restrict__ ids,
                                           const float* __restrict__ vnorm, float* __restrict__ scores,
                                           uint32_t* __restrict__ unit_max, char* smem, uint32_t buf0, int L,
                                           int NB, int64_t Ncap, int64_t N, int64_t unit, int64_t first_group,
                                           int npg, bool first_pass, uint32_t* red)
{
    const int tid = threadIdx.x;
    const uint32_t lane4 = (uint32_t)(tid & 31) << 2;
    const int nbuf = (L + 1) >> 1;
    const float* tu = tables + unit * L * (int64_t)NB;
    const uint8_t* idu = ids + unit * L * Ncap + first_group * 16;
    const float* vu = vnorm + unit * Ncap + first_group * 16;
    float* su = scores + unit * Ncap + first_group * 16;
    const uint32_t pass_bytes = (uint32_t)npg * 16u;
    char* bufp0 = smem + (buf0 - smem_addr(smem));

    if (tid == 0) {
        prefetch_l2_bulk(vu, pass_bytes * 4u);
        for (int l = 0; l < min(L, kPrefetchAhead); ++l) prefetch_l2_bulk(idu + l * Ncap, pass_bytes);
    }
    uint4 cur[kGroupsPerThread];
    load_ids(cur, idu, npg, tid);
    // The soft tables come from the previous kernel on the stream.
    if (first_pass) pdl_wait();

    // Stage values for buffer bi: float4 slot e = i*kThreads + tid holds
    // bucket e >> 4, table-in-pair (e >> 3) & 1, four lanes' copies.
    float stage[kStageSlots];
    auto load_stage = [&](int bi) {
#pragma unroll
        for (int i = 0; i < kStageSlots; ++i) {
            const int e = i * kThreads + tid;
            const int bucket = e >> 4, l = 2 * bi + ((e >> 3) & 1);
            stage[i] = (bucket < NB && l < L) ? __ldcg(tu + (int64_t)l * NB + bucket) : 0.0f;
        }
    };
    auto store_stage = [&](int buf) {
        float4* dst = reinterpret_cast<float4*>(bufp0 + buf * kBufBytes);
#pragma unroll
        for (int i = 0; i < kStageSlots; ++i) {
            const int e = i * kThreads + tid;
            if ((e >> 4) < NB) dst[e] = make_float4(stage[i], stage[i], stage[i], stage[i]);
        }
    };

    __syncthreads();  // the previous pass finished reading both buffers
    load_stage(0);
    store_stage(0);
    if (nbuf > 1) load_stage(1);
    __syncthreads();

    float acc[kGroupsPerThread][16];
#pragma unroll
    for (int j = 0; j < kGroupsPerThread; ++j)
#pragma unroll
        for (int e = 0; e < 16; ++e) acc[j][e] = 0.0f;

    for (int bi = 0; bi < nbuf; ++bi) {
        const uint32_t bbase = buf0 + (uint32_t)(bi & 1) * kBufBytes + lane4;
#pragma unroll
        for (int tt = 0; tt < 2; ++tt) {
            const int l = 2 * bi + tt;
            if (l < L) {
                if (tid == 0 && l + kPrefetchAhead < L)
                    prefetch_l2_bulk(idu + (l + kPrefetchAhead) * Ncap, pass_bytes);
                uint4 nxt[kGroupsPerThread];
                if (l + 1 < L) load_ids(nxt, idu + (l + 1) * Ncap, npg, tid);
                lookup(acc, cur, bbase + (uint32_t)tt * 128u, npg, tid);
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

    // Scores, and the largest score of a live key (n < N) of the pass.
    uint32_t mx = 0;
    const int64_t key0 = first_group * 16;
#pragma unroll
    for (int j = 0; j < kGroupsPerThread; ++j) {
        const int g = j * kThreads + tid;
        if (g < npg) {
#pragma unroll
            for (int w = 0; w < 4; ++w) {
                const float4 vn = ldg_stream_f4(vu + (int64_t)g * 16 + w * 4);
                float4 sc;
                sc.x = acc[j][w * 4 + 0] * vn.x;
                sc.y = acc[j][w * 4 + 1] * vn.y;
                sc.z = acc[j][w * 4 + 2] * vn.z;
                sc.w = acc[j][w * 4 + 3] * vn.w;
                *reinterpret_cast<float4*>(su + (int64_t)g * 16 + w * 4) = sc;
                const int64_t n = key0 + (int64_t)g * 16 + w * 4;
                if (n + 0 < N) mx = max(mx, __float_as_uint(sc.x));
                if (n + 1 < N) mx = max(mx, __float_as_uint(sc.y));
                if (n + 2 < N) mx = max(mx, __float_as_uint(sc.z));
                if (n + 3 < N) mx = max(mx, __float_as_uint(sc.w));
            }
        }
    }
    for (int o = 16; o > 0; o >>= 1) mx = max(mx, __shfl_xor_sync(kFullMask, mx, o));
    if ((tid & 31) == 0) red[tid >> 5] = mx;
    __syncthreads();
    if (tid == 0) {
        uint32_t m = 0;
        for (int w = 0; w < kThreads / 32; ++w) m = max(m, red[w]);
        atomicMax(unit_max + unit, m);
    }
}

// Persistent grid: CTA c owns groups [c * per_cta, (c+1) * per_cta) of the
// flattened (unit, 16-key group) range.  The range is cut at unit boundaries
// and each piece into equal passes of at most kPassGroups groups.
__global__ __launch_bounds__(kThreads, 1) void score_kernel(
    const float* __restrict__ tables, const uint8_t* __restrict__ ids, const float* __restrict__ vnorm,
    float* __restrict__ scores, uint32_t* __restrict__ unit_max, int L, int NB, int64_t Ncap, int64_t N,
    int64_t groups_per_unit, int64_t total_groups, int64_t groups_per_cta)
{
    extern __shared__ __align__(1024) char smem[];
    __shared__ uint32_t red[kThreads / 32];
    const uint32_t buf0 = (smem_addr(smem) + kBufBytes - 1) & ~(kBufBytes - 1);
    int64_t g = (int64_t)blockIdx.x * groups_per_cta;
    const int64_t g1 = min(total_groups, g + groups_per_cta);
    bool first = true;
    if (g >= g1) pdl_wait();
    while (g < g1) {
        const int64_t unit = g / groups_per_unit;
        const int64_t seg_end = min(g1, (unit + 1) * groups_per_unit);
        const int64_t seg = seg_end - g;
        const int64_t npass = (seg + kPassGroups - 1) / kPassGroups;
        for (int64_t ip = 0; ip < npass; ++ip) {
            const int64_t a = g + seg * ip / npass, e = g + seg * (ip + 1) / npass;
            score_pass(tables, ids, vnorm, scores, unit_max, smem, buf0, L, NB, Ncap, N, unit,
                       a - unit * groups_per_unit, (int)(e - a), first, red);
            first = false;
        }
        g = seg_end;
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
                         float* scores, uint32_t* unit_max, cudaStream_t stream)
{
    const int64_t gpu = (s.N + 15) / 16;
    const int64_t total = s.U * gpu;
    // At least ~8192 keys per CTA so the table staging stays amortised.
    const int64_t want = (total + 511) / 512;
    const int grid = (int)max64(1, min64(num_sms(), want));
    const int64_t per_cta = (total + grid - 1) / grid;
    cudaError_t e = cudaFuncSetAttribute(score_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return e;
    e = launch_pdl(score_kernel, dim3(grid), dim3(kThreads), kSmemBytes, stream, tables, ids, vnorm, scores,
                   unit_max, s.L, s.NB, s.Ncap, s.N, gpu, total, per_cta);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace socket_attn
