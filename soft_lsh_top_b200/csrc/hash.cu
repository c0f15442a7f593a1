// Prefill hashing: one uint8 bucket id per (key, table) and the value norm of
// every key in [n_begin, n_end) of every unit.
//
// Method: "Resumen Técnico: SOCKET ..." (gist.science/es/paper/2602.06283),
// "Mecanismo Central: LSH Suave" step 1 "Pre-cálculo (Prellenado)";
// "SOCKET: SOft Collision Kernel EsTimator for Sparse Attention"
// (gist.science/de/paper/2602.06283), "Vorverarbeitung (Prefill)": keys are
// hashed into L independent tables by random projections, one bucket id per
// table, and the value-vector norms are cached.
//
// id_l(k) = sum_p [<W_{l,p}, k> > 0] 2^p with the projections in float32:
// for bfloat16 keys on the fifth-generation tensor cores (hash_umma_kernel),
// for float32 keys with one fused multiply-add per element in channel order
// (hash_kernel).
// vnorm = sqrt(sum v^2) summed in float64, rounded to float32.
#include <cuda.h>
#include <stdlib.h>

#include "common.cuh"
#include "internal.h"
#include "socket_attn.h"

namespace socket_attn {
namespace {

constexpr int kThreads = 256;
constexpr int kKeys = 64;                         // keys per CTA
constexpr int kTableGroups = kThreads / kKeys;    // threads per key, each a subset of tables
constexpr int kTablesPerStage = 4;                // tables of W staged in shared memory at once
constexpr int kKPad = kHeadDim + 1;               // padded key row (conflict-free column reads)

template <typename KT>
__device__ __forceinline__ float elem(const KT* p, int64_t i);
template <>
__device__ __forceinline__ float elem<float>(const float* p, int64_t i) { return p[i]; }

// Grid: (ceil((n_end - n_begin) / kKeys), U).  Block: kThreads.
template <typename KT>
__global__ __launch_bounds__(kThreads) void hash_kernel(const KT* __restrict__ K, const KT* __restrict__ V,
                                                        int64_t Ncap, int64_t n_begin, int64_t n_end,
                                                        const uint16_t* __restrict__ W, int L, int P,
                                                        uint8_t* __restrict__ ids, float* __restrict__ vnorm)
{
    __shared__ float ks[kKeys][kKPad];
    __shared__ uint32_t ws[kTablesPerStage * 8 * kHeadDim / 2];  // bf16 pairs, [table][plane][d/2]
    extern __shared__ __align__(16) uint8_t idrow[];              // [kKeys][Lr] rotated id rows
    const int Lr = 32 * ((L + 31) / 32);

    const int tid = threadIdx.x;
    const int64_t u = blockIdx.y;
    const int64_t n0 = n_begin + (int64_t)blockIdx.x * kKeys;
    const int nk = (int)min64(kKeys, n_end - n0);
    const KT* Ku = K + u * Ncap * kHeadDim;
    const KT* Vu = V + u * Ncap * kHeadDim;

    for (int e = tid; e < kKeys * kHeadDim; e += kThreads) {
        const int r = e / kHeadDim, j = e % kHeadDim;
        ks[r][j] = r < nk ? elem(Ku, (n0 + r) * kHeadDim + j) : 0.0f;
    }
    for (int e = tid; e < kKeys * Lr / 16; e += kThreads) reinterpret_cast<uint4*>(idrow)[e] = make_uint4(0, 0, 0, 0);

    const int key = tid % kKeys, tg = tid / kKeys;
    const int64_t n = n0 + key;

    if (tg == 0 && key < nk) {
        // Squares of float32 / bfloat16 values are exact in float64 and the
        // 128-term sum loses at most ~1e-14 relative, so the float32 norm is
        // the correctly rounded norm except in rare rounding ties.
        double s = 0.0;
        for (int j = 0; j < kHeadDim; ++j) {
            const double v = (double)elem(Vu, n * kHeadDim + j);
            s = fma(v, v, s);
        }
        vnorm[u * Ncap + n] = (float)sqrt(s);
    }

    const int wpr = P * kHeadDim / 2;  // 32-bit words of W per table
    for (int l0 = 0; l0 < L; l0 += kTablesPerStage) {
        const int nt = min(kTablesPerStage, L - l0);
        __syncthreads();
        const uint32_t* wsrc = reinterpret_cast<const uint32_t*>(W + (int64_t)l0 * P * kHeadDim);
        for (int e = tid; e < nt * wpr; e += kThreads) ws[e] = wsrc[e];
        __syncthreads();
        for (int lt = tg; lt < nt; lt += kTableGroups) {
            float y[8];
#pragma unroll
            for (int p = 0; p < 8; ++p) y[p] = 0.0f;
            const uint32_t* wl = ws + lt * wpr;
            for (int j2 = 0; j2 < kHeadDim / 2; ++j2) {
                const float k0 = ks[key][2 * j2], k1 = ks[key][2 * j2 + 1];
#pragma unroll
                for (int p = 0; p < 8; ++p) {
                    if (p < P) {
                        const float2 w = bf16x2_to_f32x2(wl[p * (kHeadDim / 2) + j2]);
                        y[p] = fmaf(w.x, k0, y[p]);
                        y[p] = fmaf(w.y, k1, y[p]);
                    }
                }
            }
            uint32_t id = 0;
#pragma unroll
            for (int p = 0; p < 8; ++p)
                if (p < P && y[p] > 0.0f) id |= 1u << p;
            // Slot of table l in key n's row: 32 (l / 32) + (l - n) mod 32.
            const int l = l0 + lt;
            idrow[key * Lr + (l & ~31) + (((l & 31) - (int)(n & 31)) & 31)] = (uint8_t)id;
        }
    }
    __syncthreads();
    // Chunked layout: piece p (16 bytes) of key n = 32m + j sits at [m][p][j];
    // neighbouring threads write neighbouring keys' pieces.
    const int pieces = Lr / 16;
    uint8_t* idu = ids + u * Ncap * Lr;
    for (int e = tid; e < nk * pieces; e += kThreads) {
        const int p = e / nk, k = e % nk;
        const int64_t nn = n0 + k;
        *reinterpret_cast<uint4*>(idu + ((nn >> 5) * pieces + p) * 512 + (nn & 31) * 16) =
            *reinterpret_cast<const uint4*>(idrow + k * Lr + 16 * p);
    }
}

// ---------------------------------------------------------------------------
// bfloat16 keys on the fifth-generation tensor cores (tcgen05), in passes over
// whole 32-table blocks of at most 256 hyperplanes (one pass when L*P <= 256;
// a pass writes the 16-byte pieces of its own blocks, the first also the
// value norms).  The projections of a 128-key tile on every hyperplane are one
// UMMA product per 16 channels, y [128 keys x Np planes] = K_tile * W^T
// (bf16 in, fp32 accumulate in tensor memory), with Np = L*P rounded up to a
// multiple of 16 (the extra hyperplane rows are zero-filled by the copy and
// their signs ignored).  bf16 x bf16 products are exact in fp32, so as for the
// other kernels only the accumulation order differs from a plain sum.
//
// Persistent grid, one CTA per SM, three warp roles:
//   warp 0    one thread issues tensor copies (TMA): W once, then each key
//             tile (two 64-channel boxes, 128-byte swizzle) into a ring of
//             kUStages stages;
//   warp 1    owns the tensor-memory allocation (two accumulators of 256
//             fp32 columns); one thread issues the UMMAs of a tile into the
//             free accumulator and commits them to the stage's "empty" and
//             the accumulator's "full" barriers;
//   warps 2-9 the epilogue, two groups of four warps taking alternate tiles
//             (one accumulator each), one key per thread (tensor-memory lane = key row):
//             load the key's projections 32 columns at a time, fold their
//             signs into words, release the accumulator, then cut the table
//             ids, write the key's rotated id row, and the value norm (the
//             value row of the group's next tile is loaded from global memory
//             while the current one is processed).
// Every wait is bounded; on expiry the kernel records it in the error word,
// lets its own copies and MMAs land, frees tensor memory and exits.
// ---------------------------------------------------------------------------
constexpr int kUKeys = 128;                            // keys per tile (UMMA M)
constexpr int kUStages = 2;
constexpr int kUThreads = 320;
constexpr uint32_t kUBoxBytes = kUKeys * 128u;         // 128 rows x 64 bf16 channels
constexpr uint32_t kUTileBytes = 2u * kUBoxBytes;      // 32 KB
constexpr int kUMaxPlanes = 256;
constexpr uint32_t kUTmemCols = 512;                   // two accumulators of 256 columns
constexpr int kUSgnStride = 9;                         // sign words per key row (8 + zero pad)
constexpr uint32_t kUMaxPolls = 1u << 22;

__device__ uint32_t g_hash_err;  // bit 0: a bounded wait of the tensor-core hash expired

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void mbar_arrive(uint64_t* bar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}

// 3-D tensor copy global -> this CTA's shared memory, completion on `bar`.
__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap* map, int x, int y, int z, uint64_t* bar)
{
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(smem_addr(bar))
        : "memory");
}

// Shared-memory matrix descriptor: K-major operand in 128-byte swizzled
// atoms of 8 rows x 128 bytes (1024 bytes apart along the rows).
__device__ __forceinline__ uint64_t umma_desc_sw128(uint32_t saddr)
{
    return (uint64_t)((saddr >> 4) & 0x3fffu)   // start address
         | (uint64_t)1u << 16                    // leading byte offset (unused for swizzled K-major)
         | (uint64_t)(1024u >> 4) << 32          // stride byte offset: next 8-row group
         | (uint64_t)1u << 46                    // descriptor version
         | (uint64_t)2u << 61;                   // 128-byte swizzle
}

__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                          uint32_t accumulate)
{
    asm volatile(
        "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
        " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Arrives once on `bar` when every tcgen05 operation this thread issued so far has completed.
__device__ __forceinline__ void umma_commit(uint64_t* bar)
{
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_addr(bar))
                 : "memory");
}

__device__ __forceinline__ void tmem_ld_32cols(uint32_t taddr, uint32_t (&v)[32])
{
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
          "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15]),
          "=r"(v[16]), "=r"(v[17]), "=r"(v[18]), "=r"(v[19]), "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]),
          "=r"(v[24]), "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
        : "r"(taddr));
}

__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// Bit j = [y_j > 0] for 32 fp32 projections given as bit patterns (finite y).
__device__ __forceinline__ uint32_t sign_word(const uint32_t (&v)[32])
{
    uint32_t w = 0;
#pragma unroll
    for (int j = 0; j < 32; ++j) w |= (uint32_t)((int)v[j] > 0) << j;
    return w;
}

struct HashUArgs {
    const uint16_t* V;
    uint8_t* ids;
    float* vnorm;
    int64_t Ncap, n_begin, n_end;
    int L, P, Np;      // tables of this pass, planes per table, hyperplane rows rounded up to 16
    int blk0;          // first 32-table block of this pass
    int pieces_full;   // 16-byte pieces of a key's whole id row
    int norms;         // this pass also loads V and writes the value norms
    int tiles_per_unit;
    int64_t tiles;
};

__global__ __launch_bounds__(kUThreads, 1) void hash_umma_kernel(const __grid_constant__ CUtensorMap tmK,
                                                                 const __grid_constant__ CUtensorMap tmV,
                                                                 const __grid_constant__ CUtensorMap tmW,
                                                                 const HashUArgs a)
{
    extern __shared__ __align__(1024) char dsm[];
    __shared__ __align__(8) uint64_t full[kUStages], empty[kUStages], tfull[2], tempty[2], vfull[2], vempty[2], wbar,
        done;
    __shared__ uint32_t tmem_slot;

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const uint32_t raw = smem_addr(dsm);
    const uint32_t sW = (raw + 1023u) & ~1023u;                 // [2 boxes][Np rows][128 B]
    const uint32_t sK = sW + (uint32_t)a.Np * 256u;             // [kUStages][2 boxes][128 rows][128 B]
    const uint32_t sV = sK + kUStages * kUTileBytes;            // [2 groups][2 boxes][128 rows][128 B]
    uint32_t* sgn = reinterpret_cast<uint32_t*>(dsm + (sV + 2 * kUTileBytes - raw));  // [2][128][9]
    const int Lr = 32 * ((a.L + 31) / 32);

    if (tid == 0) {
        for (int s = 0; s < kUStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&tfull[b], 1);
            mbar_init(&tempty[b], 4);  // one arrival per epilogue warp of group b
            mbar_init(&vfull[b], 1);
            mbar_init(&vempty[b], 4);
        }
        mbar_init(&wbar, 1);
        mbar_init(&done, 1);
        fence_mbarrier_init();
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_addr(&tmem_slot)),
                     "r"(kUTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_slot;

    if (warp == 0) {
        if (lane == 0) {
            // ---- copies: W once, then the key tiles through the ring.
            mbar_arrive_expect_tx(&wbar, (uint32_t)a.Np * 256u);
            tma_load_3d(sW, &tmW, 0, 0, 0, &wbar);
            tma_load_3d(sW + (uint32_t)a.Np * 128u, &tmW, 64, 0, 0, &wbar);
            int i = 0;
            bool ok = true;
            for (int64_t t = blockIdx.x; t < a.tiles; t += gridDim.x, ++i) {
                const int s = i % kUStages, g = i & 1;
                if (!mbar_wait_bounded(&empty[s], ((i / kUStages) & 1) ^ 1, kUMaxPolls) ||
                    (a.norms && !mbar_wait_bounded(&vempty[g], ((i >> 1) & 1) ^ 1, kUMaxPolls))) {
                    ok = false;
                    break;
                }
                const int u = (int)(t / a.tiles_per_unit);
                const int n0 = (int)(a.n_begin + (t % a.tiles_per_unit) * kUKeys);
                mbar_arrive_expect_tx(&full[s], kUTileBytes);
                tma_load_3d(sK + s * kUTileBytes, &tmK, 0, n0, u, &full[s]);
                tma_load_3d(sK + s * kUTileBytes + kUBoxBytes, &tmK, 64, n0, u, &full[s]);
                if (a.norms) {
                    mbar_arrive_expect_tx(&vfull[g], kUTileBytes);
                    tma_load_3d(sV + g * kUTileBytes, &tmV, 0, n0, u, &vfull[g]);
                    tma_load_3d(sV + g * kUTileBytes + kUBoxBytes, &tmV, 64, n0, u, &vfull[g]);
                }
            }
            if (!ok) atomicOr(&g_hash_err, 1u);
            // The last copies of every stage and buffer have landed before the CTA exits.
            mbar_wait_bounded(&wbar, 0, kUMaxPolls);
            for (int j = max(0, i - kUStages); j < i; ++j)
                mbar_wait_bounded(&full[j % kUStages], (j / kUStages) & 1, kUMaxPolls);
            if (a.norms)
                for (int j = max(0, i - 2); j < i; ++j) mbar_wait_bounded(&vfull[j & 1], (j >> 1) & 1, kUMaxPolls);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // ---- MMA issue: D[128 x Np] (+)= A[128 x 16] * B[Np x 16]^T, 8 steps over 128 channels.
            const uint32_t idesc = (1u << 4)                       // D: fp32
                                 | (1u << 7) | (1u << 10)          // A, B: bf16
                                 | ((uint32_t)(a.Np >> 3) << 17)   // N
                                 | ((uint32_t)(kUKeys >> 4) << 24);  // M
            bool ok = mbar_wait_bounded(&wbar, 0, kUMaxPolls);
            int i = 0;
            for (int64_t t = blockIdx.x; ok && t < a.tiles; t += gridDim.x, ++i) {
                const int s = i % kUStages, b = i & 1;
                if (!mbar_wait_bounded(&tempty[b], ((i >> 1) & 1) ^ 1, kUMaxPolls) ||
                    !mbar_wait_bounded(&full[s], (i / kUStages) & 1, kUMaxPolls)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d = tmem + (uint32_t)b * 256u;
#pragma unroll
                for (int kk = 0; kk < kHeadDim / 16; ++kk) {
                    const uint32_t koff = (uint32_t)(kk >> 2) * kUBoxBytes + (uint32_t)(kk & 3) * 32u;
                    const uint32_t woff = (uint32_t)(kk >> 2) * (uint32_t)a.Np * 128u + (uint32_t)(kk & 3) * 32u;
                    umma_bf16(d, umma_desc_sw128(sK + s * kUTileBytes + koff), umma_desc_sw128(sW + woff), idesc,
                              kk > 0 ? 1u : 0u);
                }
                umma_commit(&empty[s]);
                umma_commit(&tfull[b]);
            }
            if (!ok) atomicOr(&g_hash_err, 1u);
            umma_commit(&done);  // every MMA of this CTA has completed once `done` flips
            mbar_wait_bounded(&done, 0, kUMaxPolls);
        }
    } else {
        // ---- epilogue: two groups of four warps take alternate tiles (group
        // g drains accumulator g); key row r of a tile <-> tensor-memory lane r.
        const int grp = (warp - 2) >> 2;
        const int q = warp & 3;  // the lane quarter this warp may access
        const int r = q * 32 + lane;
        const int ng = (a.Np + 31) / 32;
        const int pieces = Lr / 16;
        uint32_t* srow = sgn + (grp * kUKeys + r) * kUSgnStride;
        srow[8] = 0u;
        const int64_t step = 2 * (int64_t)gridDim.x;
        // This thread's value row: the 16-byte chunks of row r in the group's
        // two swizzled boxes, read in an order staggered by r so that a warp's
        // loads spread over all banks (only the sum of squares is taken).
        const uint32_t vrow = sV + (uint32_t)grp * kUTileBytes + (uint32_t)r * 128u;
        for (int64_t t = blockIdx.x + grp * (int64_t)gridDim.x, j = 0; t < a.tiles; t += step, ++j) {
            const int64_t u = t / a.tiles_per_unit;
            const int64_t n = a.n_begin + (t % a.tiles_per_unit) * kUKeys + r;
            const bool live = n < a.n_end;
            const bool ok = (!a.norms || mbar_wait_bounded(&vfull[grp], j & 1, kUMaxPolls)) &&
                            mbar_wait_bounded(&tfull[grp], j & 1, kUMaxPolls);
            if (!__all_sync(kFullMask, ok)) {
                if (lane == 0) atomicOr(&g_hash_err, 1u);
                break;
            }
            tc_fence_after();
            // Sign words: bit j of sw[g] is [y > 0] for hyperplane 32 g + j.
            const uint32_t tbase = tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)grp * 256u;
            uint32_t sw[8];
#pragma unroll
            for (int g = 0; g < 8; g += 2) {
                sw[g] = 0u;
                sw[g + 1] = 0u;
                if (g < ng) {
                    uint32_t v0[32], v1[32];
                    tmem_ld_32cols(tbase + (uint32_t)g * 32u, v0);
                    if (g + 1 < ng) tmem_ld_32cols(tbase + (uint32_t)(g + 1) * 32u, v1);
                    tmem_wait_ld();
                    sw[g] = sign_word(v0);
                    if (g + 1 < ng) sw[g + 1] = sign_word(v1);
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&tempty[grp]);

            if (a.norms && live) {
                // Value norm: squares summed in float64 (exact squares), rounded once.
                double s0 = 0.0, s1 = 0.0;
#pragma unroll
                for (int c = 0; c < kHeadDim / 8; ++c) {
                    uint4 x;
                    asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
                                 : "=r"(x.x), "=r"(x.y), "=r"(x.z), "=r"(x.w)
                                 : "r"(vrow + (uint32_t)(c >> 3) * kUBoxBytes + (uint32_t)((c ^ r) & 7) * 16u));
                    const uint32_t w4[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float2 f = bf16x2_to_f32x2(w4[e]);
                        s0 = fma((double)f.x, (double)f.x, s0);
                        s1 = fma((double)f.y, (double)f.y, s1);
                    }
                }
                a.vnorm[u * a.Ncap + n] = (float)sqrt(s0 + s1);
            }
            if (a.norms) {
                fence_proxy_async_shared();  // these reads precede the next tensor copy into the buffer
                __syncwarp();
                if (lane == 0) mbar_arrive(&vempty[grp]);
            }
            if (!live) continue;

            // Rotated id row: slot s of block c holds table 32c + (s + n) mod 32;
            // this pass writes the pieces of its own blocks.
            uint8_t* dst = a.ids + u * a.Ncap * (a.pieces_full * 16) +
                           ((n >> 5) * a.pieces_full + 2 * a.blk0) * 512 + (n & 31) * 16;
            const int rot = (int)(n & 31);
            if (a.P == 8) {
                // One byte per hyperplane group: the sign words are the ids in
                // table order (L <= 32); zero the bytes past L, then rotate the
                // 32-byte row by n mod 32 bytes in registers.
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    const int lo = 4 * k;
                    if (lo >= a.L) sw[k] = 0u;
                    else if (lo + 4 > a.L) sw[k] &= 0xffffffffu >> (8 * (lo + 4 - a.L));
                }
#pragma unroll
                for (int k = 1; k < 8; k <<= 1) {
                    if ((rot >> 2) & k) {
                        uint32_t tmp[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e) tmp[e] = sw[(e + k) & 7];
#pragma unroll
                        for (int e = 0; e < 8; ++e) sw[e] = tmp[e];
                    }
                }
                const uint32_t sh = 8u * (uint32_t)(rot & 3);
                uint32_t o[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) o[e] = __funnelshift_r(sw[e], sw[(e + 1) & 7], sh);
                *reinterpret_cast<uint4*>(dst) = make_uint4(o[0], o[1], o[2], o[3]);
                *reinterpret_cast<uint4*>(dst + 512) = make_uint4(o[4], o[5], o[6], o[7]);
                continue;
            }
            // Any P: table l's id is sign bits l P .. l P + P - 1, cut from this
            // thread's sign words in shared memory.
#pragma unroll
            for (int g = 0; g < 8; ++g)
                if (g < ng) srow[g] = sw[g];
            const uint32_t mask = (1u << a.P) - 1u;
            for (int p = 0; p < pieces; ++p) {
                uint32_t wv[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    uint32_t word = 0;
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        const int slot = 16 * p + 4 * e + k;
                        const int l = (slot & ~31) + (((slot & 31) + rot) & 31);
                        uint32_t id = 0;
                        if (l < a.L) {
                            const int bit = l * a.P;
                            id = __funnelshift_r(srow[bit >> 5], srow[(bit >> 5) + 1], bit & 31) & mask;
                        }
                        word |= id << (8 * k);
                    }
                    wv[e] = word;
                }
                *reinterpret_cast<uint4*>(dst + p * 512) = make_uint4(wv[0], wv[1], wv[2], wv[3]);
            }
        }
    }
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kUTmemCols) : "memory");
    }
}

// cuTensorMapEncodeTiled through the runtime's driver entry point (no libcuda link).
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_tiled()
{
    static EncodeTiledFn fn = [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return (EncodeTiledFn) nullptr;
        return reinterpret_cast<EncodeTiledFn>(p);
    }();
    return fn;
}

// [z][y][128 channels] bf16 rows viewed as a 3-D tensor; boxes of 64 channels
// x box_rows rows x 1, 128-byte swizzle, zero fill outside.
bool encode_rows(CUtensorMap* m, const void* base, uint64_t rows, uint64_t planes, uint32_t box_rows)
{
    EncodeTiledFn f = encode_tiled();
    if (!f) return false;
    const cuuint64_t dims[3] = {(cuuint64_t)kHeadDim, rows, planes};
    const cuuint64_t strides[2] = {(cuuint64_t)kHeadDim * 2, (cuuint64_t)kHeadDim * 2 * rows};
    const cuuint32_t box[3] = {64, box_rows, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    return f(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

cudaError_t launch_hash_keys(const void* K, const void* V, int kv_dtype, int64_t B, int64_t Hkv, int64_t Ncap,
                             int64_t n_begin, int64_t n_end, const uint16_t* W, int L, int P, uint8_t* ids,
                             float* vnorm, cudaStream_t stream)
{
    const int64_t nkeys = n_end - n_begin;
    if (kv_dtype == 1) {
        // Passes over whole 32-table blocks of at most 256 hyperplanes each
        // (one pass when L * P <= 256); the first also writes the value norms.
        const int tpp = 32 * max(1, kUMaxPlanes / (32 * P));
        const int npass = (L + tpp - 1) / tpp;  // <= 4
        HashUArgs a;
        a.V = static_cast<const uint16_t*>(V);
        a.ids = ids;
        a.vnorm = vnorm;
        a.Ncap = Ncap;
        a.n_begin = n_begin;
        a.n_end = n_end;
        a.P = P;
        a.pieces_full = 2 * ((L + 31) / 32);
        a.tiles_per_unit = (int)((nkeys + kUKeys - 1) / kUKeys);
        a.tiles = B * Hkv * a.tiles_per_unit;
        // The tensor maps are the kernel's only way to its operands; failing to
        // encode one is an error, not a reason to take another kernel.
        CUtensorMap tmK, tmV, tmW[4];
        bool ok = npass <= 4 && encode_rows(&tmK, K, (uint64_t)Ncap, (uint64_t)(B * Hkv), kUKeys) &&
                  encode_rows(&tmV, V, (uint64_t)Ncap, (uint64_t)(B * Hkv), kUKeys);
        for (int ps = 0; ok && ps < npass; ++ps) {
            const int lp = min(tpp, L - ps * tpp);
            ok = encode_rows(&tmW[ps], W + (int64_t)ps * tpp * P * kHeadDim, (uint64_t)(lp * P), 1,
                             (uint32_t)((lp * P + 15) / 16 * 16));
        }
        if (!ok) return cudaErrorInvalidValue;
        const int max_smem = 1024 + kUMaxPlanes * 256 + (kUStages + 2) * (int)kUTileBytes + 2 * kUKeys * kUSgnStride * 4;
        cudaError_t e = set_smem_limit_once((const void*)hash_umma_kernel, max_smem);
        if (e != cudaSuccess) return e;
        const int grid = (int)min64(device_num_sms(), a.tiles);
        for (int ps = 0; ps < npass; ++ps) {
            a.blk0 = ps * tpp / 32;
            a.L = min(tpp, L - ps * tpp);
            a.Np = (a.L * P + 15) / 16 * 16;
            a.norms = ps == 0;
            const int smem = 1024 + a.Np * 256 + (kUStages + 2) * (int)kUTileBytes + 2 * kUKeys * kUSgnStride * 4;
            hash_umma_kernel<<<grid, kUThreads, smem, stream>>>(tmK, tmV, tmW[ps], a);
            e = cudaGetLastError();
            if (e != cudaSuccess) return e;
        }
        return cudaSuccess;
    }
    dim3 grid((unsigned)((nkeys + kKeys - 1) / kKeys), (unsigned)(B * Hkv));
    const int smem = kKeys * 32 * ((L + 31) / 32);
    cudaError_t e = set_smem_limit_once((const void*)hash_kernel<float>, smem);
    if (e != cudaSuccess) return e;
    hash_kernel<float><<<grid, kThreads, smem, stream>>>(static_cast<const float*>(K), static_cast<const float*>(V),
                                                         Ncap, n_begin, n_end, W, L, P, ids, vnorm);
    return cudaGetLastError();
}

int hash_device_error(cudaStream_t stream, uint32_t* bits)
{
    cudaError_t e = cudaStreamSynchronize(stream);
    if (e != cudaSuccess) return (int)e;
    e = cudaMemcpyFromSymbol(bits, g_hash_err, sizeof(uint32_t));
    if (e != cudaSuccess) return (int)e;
    const uint32_t zero = 0;
    return (int)cudaMemcpyToSymbol(g_hash_err, &zero, sizeof(uint32_t));
}

}  // namespace socket_attn
