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
// for bfloat16 keys on the tensor cores (hash_mma_kernel), for float32 keys
// with one fused multiply-add per element in channel order (hash_kernel).
// vnorm = sqrt(sum v^2) summed in float64, rounded to float32.
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

// ---------------------------------------------------------------------------
// bfloat16 keys: the projections of a 64-key tile on every hyperplane as a
// tensor-core product, y [64 keys x L*P planes] = K_tile [64 x 128] *
// W^T [128 x L*P] (warp-level mma.sync m16n8k16, bf16 in, fp32 accumulate;
// bf16 x bf16 products are exact in fp32, so only the fp32 accumulation order
// differs from the CUDA-core kernel).  Warp w holds keys 16w .. 16w+15; the
// hyperplanes are staged 64 at a time.  Each 8-plane column tile's signs fold
// into one byte per key (the four lanes of a quad hold two planes each), and
// every table's id is cut from the key's sign bytes at bit l*P.  Rows are
// padded to 272 bytes so an ldmatrix phase's 8 rows hit distinct banks.
// ---------------------------------------------------------------------------
constexpr int kMKeys = 64;
constexpr int kMThreads = 128;
constexpr int kMPlanes = 64;
constexpr int kMRow = 272;
constexpr int kMSignBytes = SOCKET_MAX_L * SOCKET_MAX_P / 8;  // per key

__global__ __launch_bounds__(kMThreads) void hash_mma_kernel(const uint16_t* __restrict__ K,
                                                             const uint16_t* __restrict__ V, int64_t Ncap,
                                                             int64_t n_begin, int64_t n_end,
                                                             const uint16_t* __restrict__ W, int L, int P,
                                                             uint8_t* __restrict__ ids, float* __restrict__ vnorm)
{
    extern __shared__ __align__(128) char hsm[];
    char* ks = hsm;                                                     // [kMKeys][kMRow] key rows
    char* ws = ks + kMKeys * kMRow;                                     // [kMPlanes][kMRow] hyperplane rows
    uint8_t* sgn = reinterpret_cast<uint8_t*>(ws + kMPlanes * kMRow);   // [kMKeys][kMSignBytes]
    uint8_t* idrow = sgn + kMKeys * kMSignBytes;                        // [kMKeys][Lr] rotated id rows
    const int Lr = 32 * ((L + 31) / 32);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int64_t u = blockIdx.y;
    const int64_t n0 = n_begin + (int64_t)blockIdx.x * kMKeys;
    const int nk = (int)min64(kMKeys, n_end - n0);
    const uint16_t* Ku = K + u * Ncap * kHeadDim;
    const uint16_t* Vu = V + u * Ncap * kHeadDim;

    for (int e = tid; e < kMKeys * 16; e += kMThreads) {
        const int r = e >> 4, c = e & 15;
        uint4 v = make_uint4(0, 0, 0, 0);
        if (r < nk) v = __ldg(reinterpret_cast<const uint4*>(Ku + (n0 + r) * kHeadDim) + c);
        *reinterpret_cast<uint4*>(ks + r * kMRow + c * 16) = v;
    }
    for (int e = tid; e < kMKeys * Lr / 16; e += kMThreads) reinterpret_cast<uint4*>(idrow)[e] = make_uint4(0, 0, 0, 0);

    // Value norms: two threads per key, squares summed in float64.
    {
        const int r = tid >> 1, h = tid & 1;
        double s = 0.0;
        if (r < nk) {
            const uint4* vp = reinterpret_cast<const uint4*>(Vu + (n0 + r) * kHeadDim + h * (kHeadDim / 2));
#pragma unroll
            for (int c = 0; c < kHeadDim / 16; ++c) {
                const uint4 w = __ldg(vp + c);
                const uint32_t w4[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const float2 f = bf16x2_to_f32x2(w4[i]);
                    s = fma((double)f.x, (double)f.x, s);
                    s = fma((double)f.y, (double)f.y, s);
                }
            }
        }
        s += __shfl_xor_sync(kFullMask, s, 1);
        if (h == 0 && r < nk) vnorm[u * Ncap + n0 + r] = (float)sqrt(s);
    }

    const int nplanes = L * P;
    const uint32_t ks_s = smem_addr(ks), ws_s = smem_addr(ws);
    const int q4 = lane >> 3;
    // ldmatrix lane rows: A = keys 16 warp + 8 (q4 & 1) + lane % 8, channel half q4 >> 1;
    // B = hyperplanes 8 (q4 >> 1) + lane % 8 of a 16-plane pair, channel half q4 & 1.
    const uint32_t a_addr = ks_s + (uint32_t)((warp * 16 + (q4 & 1) * 8 + (lane & 7)) * kMRow + (q4 >> 1) * 16);
    const uint32_t b_off = (uint32_t)(((q4 >> 1) * 8 + (lane & 7)) * kMRow + (q4 & 1) * 16);
    const int g = lane >> 2, t2 = (lane & 3) * 2;
    for (int p0 = 0; p0 < nplanes; p0 += kMPlanes) {
        __syncthreads();  // the previous tile of hyperplanes is consumed
        for (int e = tid; e < kMPlanes * 16; e += kMThreads) {
            const int r = e >> 4, c = e & 15;
            uint4 v = make_uint4(0, 0, 0, 0);
            if (p0 + r < nplanes) v = __ldg(reinterpret_cast<const uint4*>(W + (int64_t)(p0 + r) * kHeadDim) + c);
            *reinterpret_cast<uint4*>(ws + r * kMRow + c * 16) = v;
        }
        __syncthreads();
        float acc[8][4];
#pragma unroll
        for (int nt = 0; nt < 8; ++nt)
#pragma unroll
            for (int i = 0; i < 4; ++i) acc[nt][i] = 0.0f;
#pragma unroll
        for (int kk = 0; kk < kHeadDim / 16; ++kk) {
            uint32_t a[4];
            ldsm_x4(a_addr + kk * 32, a);
#pragma unroll
            for (int np = 0; np < 4; ++np) {
                uint32_t b[4];
                ldsm_x4(ws_s + b_off + np * 16 * kMRow + kk * 32, b);
                mma_bf16(acc[2 * np], a, b[0], b[1]);
                mma_bf16(acc[2 * np + 1], a, b[2], b[3]);
            }
        }
        // Column tile nt: planes p0 + 8 nt .. + 7; this lane holds planes t2, t2 + 1
        // of keys g ([0], [1]) and g + 8 ([2], [3]).
#pragma unroll
        for (int nt = 0; nt < 8; ++nt) {
            uint32_t lo = (uint32_t)(acc[nt][0] > 0.0f) << t2 | (uint32_t)(acc[nt][1] > 0.0f) << (t2 + 1);
            uint32_t hi = (uint32_t)(acc[nt][2] > 0.0f) << t2 | (uint32_t)(acc[nt][3] > 0.0f) << (t2 + 1);
            lo |= __shfl_xor_sync(kFullMask, lo, 1);
            lo |= __shfl_xor_sync(kFullMask, lo, 2);
            hi |= __shfl_xor_sync(kFullMask, hi, 1);
            hi |= __shfl_xor_sync(kFullMask, hi, 2);
            if ((lane & 3) == 0 && p0 / 8 + nt < kMSignBytes) {
                sgn[(warp * 16 + g) * kMSignBytes + p0 / 8 + nt] = (uint8_t)lo;
                sgn[(warp * 16 + g + 8) * kMSignBytes + p0 / 8 + nt] = (uint8_t)hi;
            }
        }
    }
    __syncthreads();
    // Table l's id: sign bits l*P .. l*P + P - 1 (bit p <-> plane p), into the
    // slot 32 (l / 32) + (l - n) mod 32 of key n's row.
    for (int e = tid; e < kMKeys * L; e += kMThreads) {
        const int r = e / L, l = e % L;
        const int bit = l * P;
        const uint8_t* sb = sgn + r * kMSignBytes + (bit >> 3);
        uint32_t w = sb[0];
        if ((bit & 7) + P > 8) w |= (uint32_t)sb[1] << 8;
        const uint32_t id = (w >> (bit & 7)) & ((1u << P) - 1u);
        const int64_t n = n0 + r;
        idrow[r * Lr + (l & ~31) + (((l & 31) - (int)(n & 31)) & 31)] = (uint8_t)id;
    }
    __syncthreads();
    const int pieces = Lr / 16;
    uint8_t* idu = ids + u * Ncap * Lr;
    for (int e = tid; e < nk * pieces; e += kMThreads) {
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
    if (kv_dtype == 1) {
        dim3 grid((unsigned)((nkeys + kMKeys - 1) / kMKeys), (unsigned)(B * Hkv));
        const int smem = 2 * kMKeys * kMRow + kMKeys * kMSignBytes + kMKeys * 32 * ((L + 31) / 32);
        cudaError_t e = cudaFuncSetAttribute(hash_mma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return e;
        hash_mma_kernel<<<grid, kMThreads, smem, stream>>>(static_cast<const uint16_t*>(K), static_cast<const uint16_t*>(V),
                                                           Ncap, n_begin, n_end, W, L, P, ids, vnorm);
        return cudaGetLastError();
    }
    dim3 grid((unsigned)((nkeys + kKeys - 1) / kKeys), (unsigned)(B * Hkv));
    const int smem = kKeys * 32 * ((L + 31) / 32);
    cudaError_t e = cudaFuncSetAttribute(hash_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    hash_kernel<float><<<grid, kThreads, smem, stream>>>(static_cast<const float*>(K), static_cast<const float*>(V),
                                                         Ncap, n_begin, n_end, W, L, P, ids, vnorm);
    return cudaGetLastError();
}

}  // namespace socket_attn
