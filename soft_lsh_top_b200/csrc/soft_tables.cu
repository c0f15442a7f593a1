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
// uses the factorised form (split into two 4-plane halves), in float64, and
// rounds each group-summed entry once to float32.
#include "common.cuh"
#include "internal.h"

namespace socket_attn {
namespace {

constexpr int kThreads = 256;
constexpr int kTablesPerBlock = 8;
constexpr int kMaxGroup = 16;
constexpr int kMaxP = 8;

// Grid: (U, ceil(L / kTablesPerBlock)).  Block: kThreads.
//   1. the unit's G query rows are widened to float64 and their norms taken;
//   2. one thread per (head, table, plane) row forms z = <W_{l,p}, q_h>/||q_h||
//      (all 16 loads of its hyperplane row in flight at once) and the two
//      per-plane factors sigmoid(+-2z/tau);
//   3. the per-plane factors of planes 0-3 and 4-7 are multiplied into two
//      16-entry nibble tables per (head, table);
//   4. each entry T_l(b) = sum_h lo_h(b & 15) * hi_h(b >> 4), rounded once to
//      float32.
template <typename QT>
__global__ __launch_bounds__(kThreads) void soft_tables_kernel(
    const QT* __restrict__ q, const uint16_t* __restrict__ W, int64_t Hq, int64_t Hkv, int G, int L,
    int P, double tau, float* __restrict__ tables, uint32_t* __restrict__ err_word,
    uint32_t* __restrict__ counters, uint32_t* __restrict__ unit_max, uint32_t* __restrict__ unit_hist,
    uint32_t* __restrict__ cand_cnt)
{
    // Dynamic shared memory, sized for the unit's G heads (see soft_tables_smem).
    extern __shared__ __align__(16) double dsm[];
    double (*qd)[kHeadDim] = reinterpret_cast<double (*)[kHeadDim]>(dsm);
    double* qnorm = dsm + G * kHeadDim;
    double (*sig)[kTablesPerBlock][kMaxP][2] =
        reinterpret_cast<double (*)[kTablesPerBlock][kMaxP][2]>(qnorm + kMaxGroup);
    double (*nib)[kTablesPerBlock][2][16] = reinterpret_cast<double (*)[kTablesPerBlock][2][16]>(sig + G);

    const int64_t u = blockIdx.x;
    const int64_t b = u / Hkv, kvh = u % Hkv;
    const int l0 = blockIdx.y * kTablesPerBlock;
    const int nt = min(kTablesPerBlock, L - l0);
    const int NB = 1 << P;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

    if (blockIdx.y == 0) {
        if (tid == 0) {
            counters[u] = 0u;
            unit_max[u] = 0u;
            cand_cnt[u] = 0u;
            if (u == 0) *err_word = 0u;
        }
        uint4* h = reinterpret_cast<uint4*>(unit_hist + u * kScoreHistBins);
        for (int i = tid; i < kScoreHistBins / 4; i += kThreads) h[i] = make_uint4(0, 0, 0, 0);
    }
    // Let the scoring kernel start its table-independent prologue.
    pdl_launch_dependents();

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

    // Rows ordered (head, table, plane) so neighbouring threads share q_h.
    const int rows = G * nt * P;
    for (int r = tid; r < rows; r += kThreads) {
        const int h = r / (nt * P), lt = (r / P) % nt, p = r % P;
        const uint4* w = reinterpret_cast<const uint4*>(W + ((int64_t)(l0 + lt) * P + p) * kHeadDim);
        uint4 wv[kHeadDim / 8];
#pragma unroll
        for (int c = 0; c < kHeadDim / 8; ++c) wv[c] = __ldg(w + c);
        double acc[4] = {0.0, 0.0, 0.0, 0.0};
#pragma unroll
        for (int c = 0; c < kHeadDim / 8; ++c) {
            const uint32_t words[4] = {wv[c].x, wv[c].y, wv[c].z, wv[c].w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float2 f = bf16x2_to_f32x2(words[i]);
                acc[i] = fma((double)f.x, qd[h][c * 8 + 2 * i], acc[i]);
                acc[i] = fma((double)f.y, qd[h][c * 8 + 2 * i + 1], acc[i]);
            }
        }
        const double y = (acc[0] + acc[1]) + (acc[2] + acc[3]);
        const double z = qnorm[h] > 0.0 ? y / qnorm[h] : 0.0;
        const double x = 2.0 * z / tau;
        sig[h][lt][p][1] = 1.0 / (1.0 + exp(-x));  // sign +1: bit set
        sig[h][lt][p][0] = 1.0 / (1.0 + exp(x));   // sign -1: bit clear
    }
    __syncthreads();

    // Nibble tables: lo over planes 0..min(P,4)-1, hi over planes 4..P-1.
    const int plo = min(P, 4);
    for (int e = tid; e < G * nt * 32; e += kThreads) {
        const int h = e / (nt * 32), lt = (e / 32) % nt, half = (e / 16) & 1, v = e & 15;
        double prod = 1.0;
        const int p0 = half ? 4 : 0, p1 = half ? P : plo;
        for (int p = p0; p < p1; ++p) prod *= sig[h][lt][p][(v >> (p - p0)) & 1];
        nib[h][lt][half][v] = prod;
    }
    __syncthreads();

    float* tu = tables + (u * L + l0) * (int64_t)NB;
    for (int e = tid; e < nt * NB; e += kThreads) {
        const int lt = e / NB, bucket = e % NB;
        double acc = 0.0;
        for (int h = 0; h < G; ++h)
            acc += nib[h][lt][0][bucket & 15] * nib[h][lt][1][bucket >> 4];
        tu[e] = (float)acc;
    }
}

}  // namespace

cudaError_t launch_soft_tables(const void* q, int q_dtype, const uint16_t* W, const DecodeShape& s,
                               double tau, float* tables, uint32_t* err_word, uint32_t* counters,
                               uint32_t* unit_max, uint32_t* unit_hist, uint32_t* cand_cnt, cudaStream_t stream)
{
    dim3 grid((unsigned)s.U, (unsigned)((s.L + kTablesPerBlock - 1) / kTablesPerBlock));
    const size_t smem = sizeof(double) * ((size_t)s.G * kHeadDim + kMaxGroup + (size_t)s.G * kTablesPerBlock * kMaxP * 2 +
                                          (size_t)s.G * kTablesPerBlock * 32);
    cudaError_t e = cudaFuncSetAttribute(q_dtype == 1 ? (const void*)soft_tables_kernel<uint16_t>
                                                      : (const void*)soft_tables_kernel<float>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    if (q_dtype == 1)
        soft_tables_kernel<uint16_t><<<grid, kThreads, smem, stream>>>(
            static_cast<const uint16_t*>(q), W, s.Hq, s.Hkv, s.G, s.L, s.P, tau, tables, err_word, counters,
            unit_max, unit_hist, cand_cnt);
    else
        soft_tables_kernel<float><<<grid, kThreads, smem, stream>>>(
            static_cast<const float*>(q), W, s.Hq, s.Hkv, s.G, s.L, s.P, tau, tables, err_word, counters,
            unit_max, unit_hist, cand_cnt);
    return cudaGetLastError();
}

}  // namespace socket_attn
