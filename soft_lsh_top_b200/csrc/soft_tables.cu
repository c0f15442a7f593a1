// Soft bucket assignment: per unit, the 2^P-entry probability table of every
// hash table, summed over the unit's query heads.
//
// Method: "Resumen Técnico: SOCKET ..." (gist.science/es/paper/2602.06283),
// "Mecanismo Central: LSH Suave" step 2 "Asignación Suave (Decodificación)";
// "SOCKET: SOft Collision Kernel EsTimator for Sparse Attention"
// (gist.science/de/paper/2602.06283), "Weiche Zuweisung (Decoding)".  The
// query's projections on the random hyperplanes go through a temperature
// softmax over the buckets of each table.  Reading of the open soft hash:
// softmax over the 2^P sign patterns of <s_b, z>/tau with z = W_l q/||q||,
// which factorises per plane into sigmoid(2 s_{b,p} z_p / tau); this kernel
// uses the factorised form, in float64, and rounds each summed entry once to
// float32.
#include "common.cuh"
#include "internal.h"

namespace socket_attn {
namespace {

constexpr int kThreads = 256;
constexpr int kTablesPerBlock = 8;
constexpr int kMaxGroup = 16;
constexpr int kMaxP = 8;

// Grid: (U, ceil(L / kTablesPerBlock)).  Block: kThreads.
template <typename QT>
__global__ __launch_bounds__(kThreads) void soft_tables_kernel(
    const QT* __restrict__ q, const uint16_t* __restrict__ W, int64_t Hq, int64_t Hkv, int G, int L,
    int P, double tau, float* __restrict__ tables, uint32_t* __restrict__ err_word,
    uint32_t* __restrict__ counters)
{
    __shared__ double qd[kMaxGroup][kHeadDim];
    __shared__ double qnorm[kMaxGroup];
    __shared__ double sig[kMaxGroup][kTablesPerBlock][kMaxP][2];

    const int64_t u = blockIdx.x;
    const int64_t b = u / Hkv, kvh = u % Hkv;
    const int l0 = blockIdx.y * kTablesPerBlock;
    const int nt = min(kTablesPerBlock, L - l0);
    const int NB = 1 << P;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

    if (blockIdx.y == 0 && tid == 0) {
        counters[u] = 0u;
        if (u == 0) *err_word = 0u;
    }

    const QT* qu = q + (b * Hq + kvh * G) * kHeadDim;
    for (int e = tid; e < G * kHeadDim; e += kThreads) {
        if constexpr (sizeof(QT) == 2) qd[e / kHeadDim][e % kHeadDim] = (double)bf16_to_f32(qu[e]);
        else qd[e / kHeadDim][e % kHeadDim] = (double)qu[e];
    }
    __syncthreads();

    for (int h = warp; h < G; h += kThreads / 32) {
        double s = 0.0;
        for (int j = lane; j < kHeadDim; j += 32) s += qd[h][j] * qd[h][j];
        for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(kFullMask, s, o);
        if (lane == 0) qnorm[h] = sqrt(s);
    }
    __syncthreads();

    // One warp per (head, table, plane) row: z = <W_{l,p}, q_h> / ||q_h||.
    const int rows = G * nt * P;
    for (int r = warp; r < rows; r += kThreads / 32) {
        const int h = r / (nt * P), lt = (r / P) % nt, p = r % P;
        const uint16_t* w = W + ((int64_t)(l0 + lt) * P + p) * kHeadDim;
        const uint2 wv = *reinterpret_cast<const uint2*>(w + lane * 4);
        const float2 w01 = bf16x2_to_f32x2(wv.x), w23 = bf16x2_to_f32x2(wv.y);
        double y = (double)w01.x * qd[h][lane * 4 + 0] + (double)w01.y * qd[h][lane * 4 + 1] +
                   (double)w23.x * qd[h][lane * 4 + 2] + (double)w23.y * qd[h][lane * 4 + 3];
        for (int o = 16; o > 0; o >>= 1) y += __shfl_xor_sync(kFullMask, y, o);
        if (lane == 0) {
            const double z = qnorm[h] > 0.0 ? y / qnorm[h] : 0.0;
            const double x = 2.0 * z / tau;
            sig[h][lt][p][1] = 1.0 / (1.0 + exp(-x));  // sign +1: bit set
            sig[h][lt][p][0] = 1.0 / (1.0 + exp(x));   // sign -1: bit clear
        }
    }
    __syncthreads();

    float* tu = tables + (u * L + l0) * (int64_t)NB;
    for (int e = tid; e < nt * NB; e += kThreads) {
        const int lt = e / NB, bucket = e % NB;
        double acc = 0.0;
        for (int h = 0; h < G; ++h) {
            double prod = 1.0;
            for (int p = 0; p < P; ++p) prod *= sig[h][lt][p][(bucket >> p) & 1];
            acc += prod;
        }
        tu[e] = (float)acc;
    }
}

}  // namespace

cudaError_t launch_soft_tables(const void* q, int q_dtype, const uint16_t* W, const DecodeShape& s,
                               double tau, float* tables, uint32_t* err_word, uint32_t* counters,
                               cudaStream_t stream)
{
    dim3 grid((unsigned)s.U, (unsigned)((s.L + kTablesPerBlock - 1) / kTablesPerBlock));
    if (q_dtype == 1)
        soft_tables_kernel<uint16_t><<<grid, kThreads, 0, stream>>>(
            static_cast<const uint16_t*>(q), W, s.Hq, s.Hkv, s.G, s.L, s.P, tau, tables, err_word, counters);
    else
        soft_tables_kernel<float><<<grid, kThreads, 0, stream>>>(
            static_cast<const float*>(q), W, s.Hq, s.Hkv, s.G, s.L, s.P, tau, tables, err_word, counters);
    return cudaGetLastError();
}

}  // namespace socket_attn
