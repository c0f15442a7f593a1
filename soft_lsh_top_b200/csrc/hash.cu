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
// id_l(k) = sum_p [<W_{l,p}, k> > 0] 2^p, accumulated in float32 with one
// fused multiply-add per element in channel order (bfloat16 x bfloat16
// products are exact in float32, so the only error is the float32
// accumulation).  vnorm = sqrt(sum v^2) summed in float64, rounded to float32.
#include "common.cuh"
#include "internal.h"

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
__device__ __forceinline__ float elem<uint16_t>(const uint16_t* p, int64_t i) { return bf16_to_f32(p[i]); }
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

}  // namespace

cudaError_t launch_hash_keys(const void* K, const void* V, int kv_dtype, int64_t B, int64_t Hkv, int64_t Ncap,
                             int64_t n_begin, int64_t n_end, const uint16_t* W, int L, int P, uint8_t* ids,
                             float* vnorm, cudaStream_t stream)
{
    const int64_t nkeys = n_end - n_begin;
    dim3 grid((unsigned)((nkeys + kKeys - 1) / kKeys), (unsigned)(B * Hkv));
    const int smem = kKeys * 32 * ((L + 31) / 32);
    cudaError_t e = cudaFuncSetAttribute(kv_dtype == 1 ? (const void*)hash_kernel<uint16_t> : (const void*)hash_kernel<float>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    if (kv_dtype == 1)
        hash_kernel<uint16_t><<<grid, kThreads, smem, stream>>>(static_cast<const uint16_t*>(K),
                                                            static_cast<const uint16_t*>(V), Ncap, n_begin, n_end,
                                                            W, L, P, ids, vnorm);
    else
        hash_kernel<float><<<grid, kThreads, smem, stream>>>(static_cast<const float*>(K), static_cast<const float*>(V),
                                                         Ncap, n_begin, n_end, W, L, P, ids, vnorm);
    return cudaGetLastError();
}

}  // namespace socket_attn
