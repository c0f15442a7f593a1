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

constexpr int kThreads = 128;
constexpr int kTablesPerBlock = 2;
constexpr int kMaxGroup = 16;
constexpr int kMaxP = 8;
constexpr int kHalf = kHeadDim / 2;  // channels per thread of a dot product

// Grid: (U, ceil(L / kTablesPerBlock)).  Block: kThreads.
//   1. two threads per (head, table, plane) row load the two halves of the
//      hyperplane row W_{l,p} (issued first, so they are in flight while the
//      query is staged); the unit's G query rows are widened to float64 and
//      their norms taken;
//   2. each pair forms z = <W_{l,p}, q_h>/||q_h|| (its halves added with one
//      shuffle) and the two per-plane factors sigmoid(+-2z/tau);
//   3. the per-plane factors of planes 0-3 and 4-7 are multiplied into two
//      16-entry nibble tables per (head, table);
//   4. each entry T_l(b) = sum_h lo_h(b & 15) * hi_h(b >> 4) is rounded once
//      to float32 and written in the expanded layout the scoring kernel
//      copies into shared memory: per 32-table block c a [bucket][64] row
//      whose column j holds table 32c + j mod 32 (tables past L are zero).
template <typename QT>
__global__ __launch_bounds__(kThreads) void soft_tables_kernel(
    const QT* __restrict__ q, const uint16_t* __restrict__ W, int G, int L,
    int P, double tau, const AppendHash app, int64_t Ncap, int share, float* __restrict__ tables,
    uint32_t* __restrict__ err_word, uint32_t* __restrict__ counters, uint32_t* __restrict__ unit_max,
    uint32_t* __restrict__ unit_hist, uint32_t* __restrict__ cand_cnt)
{
    __shared__ uint32_t aid[kMaxAppend][kTablesPerBlock];  // ids of the appended keys (bit p <-> plane p)
    __shared__ double qd[kMaxGroup][kHeadDim];
    __shared__ double qnorm[kMaxGroup];
    __shared__ double sig[kMaxGroup][kTablesPerBlock][kMaxP][2];
    __shared__ double nib[kMaxGroup][kTablesPerBlock][2][16];

    const int64_t u = blockIdx.x;  // the unit's query rows are u G .. u G + G - 1 of [B][Hq]
    const int l0 = blockIdx.y * kTablesPerBlock;
    const int nt = min(kTablesPerBlock, L - l0);
    const int NB = 1 << P;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

    // Rows ordered (head, table, plane); thread pair (2r, 2r + 1) takes row r.
    // This kernel may be launched before the previous kernel on the stream
    // has finished (programmatic dependent launch): q and W may come from
    // it, so nothing is read before the wait.  The scoring kernel may start
    // once the wait is over (its early id loads then see every earlier
    // kernel's writes).
    pdl_wait();
    pdl_launch_dependents();

    // The unit's G query rows in 16-byte pieces (8 bf16 or 4 fp32 each), one
    // load per thread, issued before the hyperplane loads.
    constexpr int kPer16 = 16 / (int)sizeof(QT);             // elements per piece
    const int npieces = G * kHeadDim / kPer16;               // <= 512 for G <= 16
    const uint4* qu4 = reinterpret_cast<const uint4*>(q + u * G * kHeadDim);
    uint4 qv[(kMaxGroup * kHeadDim / kPer16 + kThreads - 1) / kThreads];
#pragma unroll
    for (int i = 0; i < (int)(sizeof(qv) / sizeof(qv[0])); ++i)
        if (tid + i * kThreads < npieces) qv[i] = __ldg(qu4 + tid + i * kThreads);

    const int rows = G * nt * P;
    const int half = tid & 1;
    int r = tid >> 1;
    uint4 wv[kHalf / 8];
    auto load_w = [&](int row) {
        const int lt = (row / P) % nt, p = row % P;
        const uint4* w = reinterpret_cast<const uint4*>(W + ((int64_t)(l0 + lt) * P + p) * kHeadDim + half * kHalf);
#pragma unroll
        for (int c = 0; c < kHalf / 8; ++c) wv[c] = __ldg(w + c);
    };
    if (r < rows) load_w(r);

#pragma unroll
    for (int i = 0; i < (int)(sizeof(qv) / sizeof(qv[0])); ++i) {
        const int piece = tid + i * kThreads;
        if (piece < npieces) {
            double* dst = &qd[0][0] + piece * kPer16;  // qd rows are contiguous
            const uint32_t w4[4] = {qv[i].x, qv[i].y, qv[i].z, qv[i].w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                if constexpr (sizeof(QT) == 2) {
                    const float2 f = bf16x2_to_f32x2(w4[e]);
                    dst[2 * e] = (double)f.x;
                    dst[2 * e + 1] = (double)f.y;
                } else {
                    dst[e] = (double)__uint_as_float(w4[e]);
                }
            }
        }
    }
    __syncthreads();
    for (int h = warp; h < G; h += kThreads / 32) {
        double s = 0.0;
        for (int j = lane; j < kHeadDim; j += 32) s += qd[h][j] * qd[h][j];
        for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(kFullMask, s, o);
        if (lane == 0) qnorm[h] = sqrt(s);
    }
    __syncthreads();

    // Every pair runs the same number of rounds so the shuffle sees both halves.
    for (; r < (rows + kThreads / 2 - 1) / (kThreads / 2) * (kThreads / 2); r += kThreads / 2) {
        const bool live = r < rows;
        const int h = live ? r / (nt * P) : 0;
        double acc[4] = {0.0, 0.0, 0.0, 0.0};
        if (live) {
            const double* qh = qd[h] + half * kHalf;
#pragma unroll
            for (int c = 0; c < kHalf / 8; ++c) {
                const uint32_t words[4] = {wv[c].x, wv[c].y, wv[c].z, wv[c].w};
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const float2 f = bf16x2_to_f32x2(words[i]);
                    acc[i] = fma((double)f.x, qh[c * 8 + 2 * i], acc[i]);
                    acc[i] = fma((double)f.y, qh[c * 8 + 2 * i + 1], acc[i]);
                }
            }
        }
        double y = (acc[0] + acc[1]) + (acc[2] + acc[3]);
        y += __shfl_xor_sync(kFullMask, y, 1);
        if (live && half == 0) {
            const int lt = (r / P) % nt, p = r % P;
            if (tau == 0.0) {
                // Hard LSH: the plane's bit is [<W_{l,p}, q_h> > 0], as for keys.
                sig[h][lt][p][1] = y > 0.0 ? 1.0 : 0.0;
                sig[h][lt][p][0] = y > 0.0 ? 0.0 : 1.0;
            } else {
                const double z = qnorm[h] > 0.0 ? y / qnorm[h] : 0.0;
                const double x = 2.0 * z / tau;
                sig[h][lt][p][1] = 1.0 / (1.0 + exp(-x));  // sign +1: bit set
                sig[h][lt][p][0] = 1.0 / (1.0 + exp(x));   // sign -1: bit clear
            }
        }
        if (r + kThreads / 2 < rows) load_w(r + kThreads / 2);
    }
    __syncthreads();

    // Nibble tables: lo over planes 0..min(P,4)-1, hi over planes 4..P-1.
    const int plo = min(P, 4);
    for (int e = tid; e < G * nt * 32; e += kThreads) {
        const int h = e / (nt * 32), lt = (e / 32) % nt, hi = (e / 16) & 1, v = e & 15;
        double prod = 1.0;
        const int p0 = hi ? 4 : 0, p1 = hi ? P : plo;
        for (int p = p0; p < p1; ++p) prod *= sig[h][lt][p][(v >> (p - p0)) & 1];
        nib[h][lt][hi][v] = prod;
    }
    __syncthreads();

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
    const int nblk = (L + 31) / 32;
    float* tu = tables + u * nblk * (int64_t)NB * 64;
    for (int e = tid; e < nt * NB; e += kThreads) {
        const int lt = e % nt, bucket = e / nt;
        double acc = 0.0;
        for (int h = 0; h < G; ++h)
            acc += nib[h][lt][0][bucket & 15] * nib[h][lt][1][bucket >> 4];
        const int l = l0 + lt;
        float* row = tu + ((int64_t)(l >> 5) * NB + bucket) * 64;
        row[l & 31] = (float)acc;
        row[(l & 31) + 32] = (float)acc;
    }
    if (blockIdx.y == 0) {
        const int npad = 32 * nblk - L;
        for (int e = tid; e < npad * NB; e += kThreads) {
            const int l = L + e % npad, bucket = e / npad;
            float* row = tu + ((int64_t)(l >> 5) * NB + bucket) * 64;
            row[l & 31] = 0.0f;
            row[(l & 31) + 32] = 0.0f;
        }
    }

    // Keys appended in this step (the step 1 hash of those keys, "Pre-cálculo"):
    // the ids of this CTA's tables, and for the first table block the norms and
    // the row padding.  Projections in float32 (one warp per (key, table,
    // plane), four channels per lane, tree sum); norms in float64.  The first
    // unit of each kv unit does it; the scoring kernel reads these rows only
    // after this grid has completed.
    if (app.end > app.begin && u % share == 0) {
        const int64_t ukv = u / share;
        const int nk = (int)(app.end - app.begin);
        const int Lr = 32 * nblk, pieces = Lr / 16;
        uint8_t* idu = app.ids + ukv * Ncap * Lr;
        for (int e = tid; e < nk * kTablesPerBlock; e += kThreads) aid[e / kTablesPerBlock][e % kTablesPerBlock] = 0u;
        __syncthreads();
        for (int row = warp; row < nk * nt * P; row += kThreads / 32) {
            const int key = row / (nt * P), lt = (row / P) % nt, p = row % P;
            const int64_t off = (ukv * Ncap + app.begin + key) * kHeadDim + 4 * lane;
            const uint2 wq = *reinterpret_cast<const uint2*>(W + ((int64_t)(l0 + lt) * P + p) * kHeadDim + 4 * lane);
            const float2 w01 = bf16x2_to_f32x2(wq.x), w23 = bf16x2_to_f32x2(wq.y);
            float4 kf;
            if (app.kv_dtype == 1) {
                const uint2 kq = *reinterpret_cast<const uint2*>(static_cast<const uint16_t*>(app.K) + off);
                const float2 k01 = bf16x2_to_f32x2(kq.x), k23 = bf16x2_to_f32x2(kq.y);
                kf = make_float4(k01.x, k01.y, k23.x, k23.y);
            } else {
                kf = *reinterpret_cast<const float4*>(static_cast<const float*>(app.K) + off);
            }
            float y = fmaf(w23.y, kf.w, fmaf(w23.x, kf.z, fmaf(w01.y, kf.y, w01.x * kf.x)));
            for (int o = 16; o > 0; o >>= 1) y += __shfl_xor_sync(kFullMask, y, o);
            if (lane == 0 && y > 0.0f) atomicOr(&aid[key][lt], 1u << p);
        }
        __syncthreads();
        // Byte of table l in key n's rotated row: block l / 32, slot (l - n) mod 32.
        auto id_byte = [&](int64_t n, int l) -> uint8_t* {
            const int b = (l & ~31) + (((l & 31) - (int)(n & 31)) & 31);
            return idu + ((n >> 5) * pieces + (b >> 4)) * 512 + (n & 31) * 16 + (b & 15);
        };
        for (int e = tid; e < nk * nt; e += kThreads) {
            const int key = e / nt, lt = e % nt;
            *id_byte(app.begin + key, l0 + lt) = (uint8_t)aid[key][lt];
        }
        if (blockIdx.y == 0) {
            const int npad = Lr - L;
            for (int e = tid; e < nk * npad; e += kThreads) *id_byte(app.begin + e / npad, L + e % npad) = 0;
            for (int key = warp; key < nk; key += kThreads / 32) {
                const int64_t off = (ukv * Ncap + app.begin + key) * kHeadDim + 4 * lane;
                float4 vf;
                if (app.kv_dtype == 1) {
                    const uint2 vq = *reinterpret_cast<const uint2*>(static_cast<const uint16_t*>(app.V) + off);
                    const float2 v01 = bf16x2_to_f32x2(vq.x), v23 = bf16x2_to_f32x2(vq.y);
                    vf = make_float4(v01.x, v01.y, v23.x, v23.y);
                } else {
                    vf = *reinterpret_cast<const float4*>(static_cast<const float*>(app.V) + off);
                }
                double s = (double)vf.x * vf.x + (double)vf.y * vf.y + (double)vf.z * vf.z + (double)vf.w * vf.w;
                for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(kFullMask, s, o);
                if (lane == 0) app.vnorm[ukv * Ncap + app.begin + key] = (float)sqrt(s);
            }
        }
    }
}

}  // namespace

cudaError_t launch_soft_tables(const void* q, int q_dtype, const uint16_t* W, const DecodeShape& s,
                               double tau, const AppendHash& app, float* tables, uint32_t* err_word,
                               uint32_t* counters, uint32_t* unit_max, uint32_t* unit_hist, uint32_t* cand_cnt,
                               cudaStream_t stream)
{
    dim3 grid((unsigned)s.U, (unsigned)((s.L + kTablesPerBlock - 1) / kTablesPerBlock));
    if (q_dtype == 1)
        return launch_pdl(soft_tables_kernel<uint16_t>, grid, dim3(kThreads), 0, stream,
                          static_cast<const uint16_t*>(q), W, s.G, s.L, s.P, tau, app, s.Ncap, s.share, tables,
                          err_word, counters, unit_max, unit_hist, cand_cnt);
    return launch_pdl(soft_tables_kernel<float>, grid, dim3(kThreads), 0, stream, static_cast<const float*>(q), W,
                      s.G, s.L, s.P, tau, app, s.Ncap, s.share, tables, err_word, counters, unit_max, unit_hist,
                      cand_cnt);
}

}  // namespace socket_attn
