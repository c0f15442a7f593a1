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
constexpr int kMaxTablesPerBlock = 8;  // tables per CTA: 2, 4 or 8, chosen at launch
constexpr int kMaxGroup = 16;
constexpr int kMaxP = 8;
constexpr int kHalf = kHeadDim / 2;  // channels per thread of a dot product
constexpr int kWRow = kHeadDim + 8;  // padded bf16 hyperplane row in shared memory (272 bytes)

// Grid: (U, ceil(L / tpb)).  Block: kThreads.  Dynamic shared memory sized by G and tpb.
//   1. the CTA's hyperplane rows are staged in shared memory; the unit's G
//      query rows are widened to float64 and their norms taken;
//   2. two threads per (head, table, plane) row form z = <W_{l,p}, q_h>/||q_h||
//      (their channel halves added with one shuffle) and the two per-plane
//      factors sigmoid(+-2z/tau), both from one exponential;
//   3. the per-plane factors of planes 0-3 and 4-7 are multiplied into two
//      16-entry nibble tables per (head, table);
//   4. each entry T_l(b) = sum_h lo_h(b & 15) * hi_h(b >> 4) is rounded once
//      to float32 and written in the expanded layout the scoring kernel
//      copies into shared memory: per 32-table block c a [bucket][64] row
//      whose column j holds table 32c + j mod 32 (tables past L are zero).
template <typename QT>
__global__ __launch_bounds__(kThreads) void soft_tables_kernel(
    const QT* __restrict__ q, const uint16_t* __restrict__ W, int G, int L,
    int P, int tpb, double tau, const AppendHash app, int64_t Ncap, int share, float* __restrict__ tables,
    uint32_t* __restrict__ err_word, uint32_t* __restrict__ counters, uint32_t* __restrict__ unit_max,
    uint32_t* __restrict__ unit_hist, uint32_t* __restrict__ cand_cnt)
{
    __shared__ uint32_t aid[kMaxAppend][kMaxTablesPerBlock];  // ids of the appended keys (bit p <-> plane p)
    extern __shared__ __align__(16) char st_dyn[];
    uint16_t* wsm = reinterpret_cast<uint16_t*>(st_dyn);  // [tpb * P][kWRow] bf16 hyperplane rows
    double* qd = reinterpret_cast<double*>(st_dyn + tpb * P * kWRow * 2);  // [G][kHeadDim]
    double* qnorm = qd + G * kHeadDim;               // [G]: 2 / (tau ||q_h||)
    double* sig = qnorm + G;                         // [G][tpb][kMaxP][2]
    double* nib = sig + G * tpb * kMaxP * 2;         // [G][tpb][2][16]
    auto SIG = [&](int h, int lt, int p, int s) -> double& { return sig[((h * tpb + lt) * kMaxP + p) * 2 + s]; };
    auto NIB = [&](int h, int lt, int hi, int v) -> double& { return nib[((h * tpb + lt) * 2 + hi) * 16 + v]; };

    const int64_t u = blockIdx.x;  // the unit's query rows are u G .. u G + G - 1 of [B][Hq]
    const int l0 = blockIdx.y * tpb;
    const int nt = min(tpb, L - l0);
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

    // This CTA's hyperplane rows (nt tables x P planes, contiguous in W),
    // staged once in shared memory with rows padded to 272 bytes so that a
    // warp's 16-byte reads of 16 rows x 2 halves fall on distinct banks.
    const int wrows = nt * P;
    const uint4* wsrc = reinterpret_cast<const uint4*>(W + (int64_t)l0 * P * kHeadDim);
    for (int e = tid; e < wrows * (kHeadDim / 8); e += kThreads)
        *reinterpret_cast<uint4*>(wsm + (e >> 4) * kWRow + (e & 15) * 8) = __ldg(wsrc + e);

#pragma unroll
    for (int i = 0; i < (int)(sizeof(qv) / sizeof(qv[0])); ++i) {
        const int piece = tid + i * kThreads;
        if (piece < npieces) {
            double* dst = qd + piece * kPer16;  // qd rows are contiguous
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
    // Per head, the factor taking <W_{l,p}, q_h> to the sigmoid argument
    // 2 z / tau with z = <W_{l,p}, q_h> / ||q_h|| (0 for a zero query).
    for (int h = warp; h < G; h += kThreads / 32) {
        double s = 0.0;
        for (int j = lane; j < kHeadDim; j += 32) s += qd[h * kHeadDim + j] * qd[h * kHeadDim + j];
        for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(kFullMask, s, o);
        if (lane == 0) qnorm[h] = (s > 0.0 && tau > 0.0) ? 2.0 / (tau * sqrt(s)) : 0.0;
    }
    __syncthreads();

    // Rows ordered (head, table, plane); thread pair (2r, 2r + 1) takes the two
    // channel halves of row r, and every pair runs the same number of rounds
    // so the shuffle sees both halves.
    const int rows = G * wrows;
    const int half = tid & 1;
    for (int r = tid >> 1; r < (rows + kThreads / 2 - 1) / (kThreads / 2) * (kThreads / 2); r += kThreads / 2) {
        const bool live = r < rows;
        const int h = live ? r / wrows : 0, wr = live ? r - h * wrows : 0;
        double acc[8] = {0.0, 0.0, 0.0, 0.0, 0.0, 0.0, 0.0, 0.0};
        if (live) {
            const double* qh = qd + h * kHeadDim + half * kHalf;
            const uint16_t* wh = wsm + wr * kWRow + half * kHalf;
#pragma unroll
            for (int c = 0; c < kHalf / 8; ++c) {
                const uint4 wq = *reinterpret_cast<const uint4*>(wh + c * 8);
                const uint32_t words[4] = {wq.x, wq.y, wq.z, wq.w};
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const float2 f = bf16x2_to_f32x2(words[i]);
                    acc[2 * i] = fma((double)f.x, qh[c * 8 + 2 * i], acc[2 * i]);
                    acc[2 * i + 1] = fma((double)f.y, qh[c * 8 + 2 * i + 1], acc[2 * i + 1]);
                }
            }
        }
        double y = ((acc[0] + acc[1]) + (acc[2] + acc[3])) + ((acc[4] + acc[5]) + (acc[6] + acc[7]));
        y += __shfl_xor_sync(kFullMask, y, 1);
        if (live && half == 0) {
            const int lt = wr / P, p = wr - lt * P;
            if (tau == 0.0) {
                // Hard LSH: the plane's bit is [<W_{l,p}, q_h> > 0], as for keys.
                SIG(h, lt, p, 1) = y > 0.0 ? 1.0 : 0.0;
                SIG(h, lt, p, 0) = y > 0.0 ? 0.0 : 1.0;
            } else {
                // sigmoid(+-x) from one exponential: e = exp(-|x|),
                // sigmoid(|x|) = 1 / (1 + e), sigmoid(-|x|) = e / (1 + e).
                const double x = y * qnorm[h];
                const double e = exp(-fabs(x));
                const double big = 1.0 / (1.0 + e), small = e * big;
                SIG(h, lt, p, 1) = x >= 0.0 ? big : small;  // sign +1: bit set
                SIG(h, lt, p, 0) = x >= 0.0 ? small : big;  // sign -1: bit clear
            }
        }
    }
    __syncthreads();

    // Nibble tables: lo over planes 0..min(P,4)-1, hi over planes 4..P-1.
    const int plo = min(P, 4);
    for (int e = tid; e < G * nt * 32; e += kThreads) {
        const int h = e / (nt * 32), lt = (e / 32) % nt, hi = (e / 16) & 1, v = e & 15;
        double prod = 1.0;
        const int p0 = hi ? 4 : 0, p1 = hi ? P : plo;
        for (int p = p0; p < p1; ++p) prod *= SIG(h, lt, p, (v >> (p - p0)) & 1);
        NIB(h, lt, hi, v) = prod;
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
    // One bucket of all nt tables per thread: the row's nt adjacent columns
    // (and their copies 32 columns on) go out as whole vector stores.  tpb
    // divides 32 and l0 is a multiple of it, so the CTA's tables sit in one
    // 32-table block and its columns start on an nt-float boundary.
    for (int bucket = tid; bucket < NB; bucket += kThreads) {
        float vals[kMaxTablesPerBlock];
#pragma unroll
        for (int lt = 0; lt < kMaxTablesPerBlock; ++lt) {
            double acc = 0.0;
            if (lt < nt)
                for (int h = 0; h < G; ++h) acc += NIB(h, lt, 0, bucket & 15) * NIB(h, lt, 1, bucket >> 4);
            vals[lt] = (float)acc;
        }
        float* row = tu + ((int64_t)(l0 >> 5) * NB + bucket) * 64 + (l0 & 31);
        if (nt == 8) {
            const float4 a = make_float4(vals[0], vals[1], vals[2], vals[3]);
            const float4 b = make_float4(vals[4], vals[5], vals[6], vals[7]);
            *reinterpret_cast<float4*>(row) = a;
            *reinterpret_cast<float4*>(row + 4) = b;
            *reinterpret_cast<float4*>(row + 32) = a;
            *reinterpret_cast<float4*>(row + 36) = b;
        } else if (nt == 4) {
            const float4 a = make_float4(vals[0], vals[1], vals[2], vals[3]);
            *reinterpret_cast<float4*>(row) = a;
            *reinterpret_cast<float4*>(row + 32) = a;
        } else if (nt == 2) {
            const float2 a = make_float2(vals[0], vals[1]);
            *reinterpret_cast<float2*>(row) = a;
            *reinterpret_cast<float2*>(row + 32) = a;
        } else {
#pragma unroll
            for (int lt = 0; lt < kMaxTablesPerBlock; ++lt)
                if (lt < nt) {
                    row[lt] = vals[lt];
                    row[lt + 32] = vals[lt];
                }
        }
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
        for (int e = tid; e < nk * kMaxTablesPerBlock; e += kThreads) aid[e / kMaxTablesPerBlock][e % kMaxTablesPerBlock] = 0u;
        __syncthreads();
        for (int key = 0; key < nk; ++key) {
            // The key row once per warp (four channels per lane); the CTA's
            // hyperplane rows from shared memory.
            const int64_t off = (ukv * Ncap + app.begin + key) * kHeadDim + 4 * lane;
            float4 kf;
            if (app.kv_dtype == 1) {
                const uint2 kq = *reinterpret_cast<const uint2*>(static_cast<const uint16_t*>(app.K) + off);
                const float2 k01 = bf16x2_to_f32x2(kq.x), k23 = bf16x2_to_f32x2(kq.y);
                kf = make_float4(k01.x, k01.y, k23.x, k23.y);
            } else {
                kf = *reinterpret_cast<const float4*>(static_cast<const float*>(app.K) + off);
            }
            for (int wr = warp; wr < wrows; wr += kThreads / 32) {
                const uint2 wq = *reinterpret_cast<const uint2*>(wsm + wr * kWRow + 4 * lane);
                const float2 w01 = bf16x2_to_f32x2(wq.x), w23 = bf16x2_to_f32x2(wq.y);
                float y = fmaf(w23.y, kf.w, fmaf(w23.x, kf.z, fmaf(w01.y, kf.y, w01.x * kf.x)));
                for (int o = 16; o > 0; o >>= 1) y += __shfl_xor_sync(kFullMask, y, o);
                if (lane == 0 && y > 0.0f) atomicOr(&aid[key][wr / P], 1u << (wr % P));
            }
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
    // Tables per CTA: the fewest (2, 4, 8) whose grid fits in one wave of
    // resident CTAs, so many units or tables do not queue in waves.
    const int qi = q_dtype == 1 ? 1 : 0;
    auto kern = qi ? (void*)soft_tables_kernel<uint16_t> : (void*)soft_tables_kernel<float>;
    // Resident CTAs per SM by (q dtype, G, P, log2 tpb - 1), looked up once per thread and device.
    static thread_local int cached_dev = -1;
    static thread_local int per_sm_cache[2][kMaxGroup + 1][kMaxP + 1][3];
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev != cached_dev) {
        for (auto& a : per_sm_cache)
            for (auto& b : a)
                for (auto& c : b)
                    for (int& e : c) e = -1;
        for (void* kf : {(void*)soft_tables_kernel<uint16_t>, (void*)soft_tables_kernel<float>}) {
            const int max_smem = (int)sizeof(double) * kMaxGroup * (kHeadDim + 1 + kMaxTablesPerBlock * (kMaxP * 2 + 32)) +
                                 kMaxTablesPerBlock * kMaxP * kWRow * 2;
            cudaError_t e = cudaFuncSetAttribute(kf, cudaFuncAttributeMaxDynamicSharedMemorySize, max_smem);
            if (e != cudaSuccess) return e;
        }
        cached_dev = dev;
    }
    int tpb = 2, smem = 0;
    for (int li = 0;; ++li, tpb *= 2) {
        smem = (int)sizeof(double) * s.G * (kHeadDim + 1 + tpb * (kMaxP * 2 + 32)) + tpb * s.P * kWRow * 2;
        int& per_sm = per_sm_cache[qi][s.G][s.P][li];
        if (per_sm < 0) {
            cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kThreads, smem);
            if (e != cudaSuccess) return e;
        }
        const int64_t ctas = s.U * ((s.L + tpb - 1) / tpb);
        if (tpb == kMaxTablesPerBlock || ctas <= (int64_t)per_sm * device_num_sms()) break;
    }
    dim3 grid((unsigned)s.U, (unsigned)((s.L + tpb - 1) / tpb));
    if (q_dtype == 1)
        return launch_pdl(soft_tables_kernel<uint16_t>, grid, dim3(kThreads), (size_t)smem, stream,
                          static_cast<const uint16_t*>(q), W, s.G, s.L, s.P, tpb, tau, app, s.Ncap, s.share, tables,
                          err_word, counters, unit_max, unit_hist, cand_cnt);
    return launch_pdl(soft_tables_kernel<float>, grid, dim3(kThreads), (size_t)smem, stream, static_cast<const float*>(q),
                      W, s.G, s.L, s.P, tpb, tau, app, s.Ncap, s.share, tables, err_word, counters, unit_max,
                      unit_hist, cand_cnt);
}

}  // namespace socket_attn
