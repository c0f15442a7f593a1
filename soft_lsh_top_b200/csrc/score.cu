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
// layout: a 64 KB buffer holds four tables as float[256 buckets][4 tables]
// [16 replicas]; lane j uses replica j % 16, and the two half-warps look up
// different tables of the buffer in the same instruction (round t: slot
// t ^ half), so a warp's 32 random lookups land in 32 distinct banks -- one
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
constexpr uint32_t kBufBytes = 1u << 16;                 // [bucket 256][table 4][replica 16] floats
constexpr int kTablesPerBuf = 4;
constexpr int kStageSlots = kBufBytes / 16 / kThreads;   // float4 stores per thread per buffer (8)
constexpr int kPrefetchAhead = 8;                        // tables prefetched into L2 ahead
constexpr int kHistBins = kScoreHistBins;                // unit histogram of score bit patterns >> kHistShift
constexpr int kHistShift = kScoreHistShift;
// The two staging buffers sit at 64 KB-aligned shared addresses A and
// A + 64 KB.  A lookup address is then A_buf | (id << 8) | (slot << 6) | (replica << 2):
// one byte-permute of the packed id word with a per-lane base that already
// holds A_buf, the table slot and the replica.  The dynamic allocation spans
// three 64 KB windows so an aligned pair fits wherever the window starts.
constexpr int kSmemBytes = 3 * (int)kBufBytes;

__device__ __forceinline__ float lds_f32(uint32_t addr)
{
    float v;
    asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(addr));
    return v;
}

// Ids of round rr for this lane's 4 groups: table (rr & ~3) + ((rr & 3) ^ half).
// Groups past the pass read the pass's last group instead (their sums are
// never stored), so the lookup loop needs no per-group condition.
__device__ __forceinline__ void load_round(uint4 (&v)[kGroupsPerThread], const uint8_t* idu, int64_t Ncap, int L,
                                           int npg, int tid, int half, int rr)
{
    const int tab = (rr & ~(kTablesPerBuf - 1)) + ((rr & (kTablesPerBuf - 1)) ^ half);
    const uint8_t* row = idu + (int64_t)min(tab, L - 1) * Ncap;
#pragma unroll
    for (int j = 0; j < kGroupsPerThread; ++j) {
        const int g = min(j * kThreads + tid, npg - 1);
        v[j] = ldg_stream_u4(row + (int64_t)g * 16);
    }
}

// One pass: groups [first_group, first_group + npg) of one unit, npg <= kPassGroups.
__device__ __forceinline__ void score_pass(const float* __restrict__ tables, const uint8_t* __restrict__ ids,
                                           const float* __restrict__ vnorm, float* __restrict__ scores,
                                           uint32_t* __restrict__ unit_max, uint32_t* __restrict__ unit_hist,
                                           uint32_t* shist, char* smem, uint32_t buf0, int L,
                                           int NB, int64_t Ncap, int64_t N, int64_t unit, int64_t first_group,
                                           int npg, bool first_pass, uint32_t* red)
{
    const int tid = threadIdx.x, lane = tid & 31;
    const int half = lane >> 4;
    // byte 0 of a lookup address for slot s: (s << 6) | (replica << 2); slot = t ^ half.
    const uint32_t rep4 = (uint32_t)(lane & 15) << 2;
    const int nbuf = (L + kTablesPerBuf - 1) / kTablesPerBuf;
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
    load_round(cur, idu, Ncap, L, npg, tid, half, 0);
    // The soft tables come from the previous kernel on the stream.
    if (first_pass) pdl_wait();

    // Stage values for buffer bi: float4 slot e = i*kThreads + tid holds
    // bucket e >> 4, table slot (e >> 2) & 3, replicas 4*(e & 3) .. +3.
    float stage[kStageSlots];
    auto load_stage = [&](int bi) {
#pragma unroll
        for (int i = 0; i < kStageSlots; ++i) {
            const int e = i * kThreads + tid;
            const int bucket = e >> 4, l = kTablesPerBuf * bi + ((e >> 2) & 3);
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

    const int nrounds = nbuf * kTablesPerBuf;
    for (int bi = 0; bi < nbuf; ++bi) {
        if (tid == 0) {
            const int l0 = kTablesPerBuf * bi + kPrefetchAhead;
            for (int l = l0; l < min(L, l0 + kTablesPerBuf); ++l) prefetch_l2_bulk(idu + l * Ncap, pass_bytes);
        }
        const uint32_t bbase = buf0 + (uint32_t)(bi & 1) * kBufBytes + rep4;
#pragma unroll
        for (int t = 0; t < kTablesPerBuf; ++t) {
            const int rr = kTablesPerBuf * bi + t;
            uint4 nxt[kGroupsPerThread];
            if (rr + 1 < nrounds) load_round(nxt, idu, Ncap, L, npg, tid, half, rr + 1);
            // Rounds past table L-1 look up the zero-filled slots of the last buffer.
            const uint32_t base = bbase + ((uint32_t)(t ^ half) << 6);
#pragma unroll
            for (int j = 0; j < kGroupsPerThread; ++j) {
                const uint32_t words[4] = {cur[j].x, cur[j].y, cur[j].z, cur[j].w};
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
#pragma unroll
            for (int j = 0; j < kGroupsPerThread; ++j) cur[j] = nxt[j];
        }
        if (bi + 1 < nbuf) {
            store_stage((bi + 1) & 1);
            if (bi + 2 < nbuf) load_stage(bi + 2);
        }
        __syncthreads();
    }

    // Scores, the largest score of a live key (n < N) of the pass, and the
    // histogram of the live scores' top bits (bit pattern >> kHistShift).
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
                const uint32_t bits[4] = {__float_as_uint(sc.x), __float_as_uint(sc.y), __float_as_uint(sc.z),
                                          __float_as_uint(sc.w)};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    if (n + e < N) {
                        mx = max(mx, bits[e]);
                        atomicAdd(shist + min(bits[e] >> kHistShift, (uint32_t)(kHistBins - 1)), 1u);
                    }
                }
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
    // Flush the pass histogram into the unit's histogram and clear it.
    uint32_t* gh = unit_hist + unit * kHistBins;
    for (int b = tid; b < kHistBins; b += kThreads) {
        const uint32_t c = shist[b];
        if (c) {
            atomicAdd(gh + b, c);
            shist[b] = 0;
        }
    }
}

// Persistent grid: CTA c owns groups [c * per_cta, (c+1) * per_cta) of the
// flattened (unit, 16-key group) range.  The range is cut at unit boundaries
// and each piece into equal passes of at most kPassGroups groups.
__global__ __launch_bounds__(kThreads, 1) void score_kernel(
    const float* __restrict__ tables, const uint8_t* __restrict__ ids, const float* __restrict__ vnorm,
    float* __restrict__ scores, uint32_t* __restrict__ unit_max, uint32_t* __restrict__ unit_hist, int L, int NB,
    int64_t Ncap, int64_t N, int64_t groups_per_unit, int64_t total_groups, int64_t groups_per_cta)
{
    extern __shared__ __align__(1024) char smem[];
    __shared__ uint32_t red[kThreads / 32];
    __shared__ uint32_t shist[kHistBins];
    for (int b = threadIdx.x; b < kHistBins; b += kThreads) shist[b] = 0;
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
            score_pass(tables, ids, vnorm, scores, unit_max, unit_hist, shist, smem, buf0, L, NB, Ncap, N, unit,
                       a - unit * groups_per_unit, (int)(e - a), first, red);
            first = false;
        }
        g = seg_end;
    }
}

}  // namespace

int device_num_sms()
{
    int dev = 0, n = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    return n > 0 ? n : 1;
}

cudaError_t launch_score(const float* tables, const uint8_t* ids, const float* vnorm, const DecodeShape& s,
                         float* scores, uint32_t* unit_max, uint32_t* unit_hist, cudaStream_t stream)
{
    const int64_t gpu = (s.N + 15) / 16;
    const int64_t total = s.U * gpu;
    // At least ~8192 keys per CTA so the table staging stays amortised.
    const int64_t want = (total + 511) / 512;
    const int grid = (int)max64(1, min64(device_num_sms(), want));
    const int64_t per_cta = (total + grid - 1) / grid;
    cudaError_t e = cudaFuncSetAttribute(score_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return e;
    e = launch_pdl(score_kernel, dim3(grid), dim3(kThreads), kSmemBytes, stream, tables, ids, vnorm, scores,
                   unit_max, unit_hist, s.L, s.NB, s.Ncap, s.N, gpu, total, per_cta);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace socket_attn
