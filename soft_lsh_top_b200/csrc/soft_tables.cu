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
constexpr int kMaxGroup = 16;
constexpr int kMaxP = 8;
constexpr int kTpr = 8;                    // threads per hyperplane row (16 channels each)
constexpr int kChan = kHeadDim / kTpr;     // 16
constexpr int kQSeg = kChan + 2;           // padded fp64 segment of a query row (bank spread)
constexpr int kHeadsPerPass = 4;           // heads whose dot products share one read of a row

// bfloat16 bits (low 16) -> float64, exact.  Normal values are rebuilt with
// integer operations (sign, exponent rebiased by 1023 - 127, the 7 mantissa
// bits at the top of the fp64 mantissa); zero, subnormals, infinities and NaN
// take the hardware widening.
__device__ __forceinline__ double bf16_bits_to_f64(uint32_t b)
{
    const uint32_t mag = b & 0x7fffu, e = mag >> 7;
    if (e == 0u || e == 0xffu) return (double)__uint_as_float(b << 16);
    return __hiloint2double((int)(((b & 0x8000u) << 16) | ((mag << 13) + (896u << 20))), 0);
}

// Four channels of a value row (element offset `off`) as float32.
__device__ __forceinline__ float4 load_v4(const AppendHash& app, int64_t off)
{
    if (app.kv_dtype == 1) {
        const uint2 vq = *reinterpret_cast<const uint2*>(static_cast<const uint16_t*>(app.V) + off);
        const float2 v01 = bf16x2_to_f32x2(vq.x), v23 = bf16x2_to_f32x2(vq.y);
        return make_float4(v01.x, v01.y, v23.x, v23.y);
    }
    return *reinterpret_cast<const float4*>(static_cast<const float*>(app.V) + off);
}

constexpr int kKeySlots = 16;              // appended keys projected per pass group (extra rows of qd)

// Dynamic shared memory of a CTA for group size G, with `slots` rows for
// appended keys.
__host__ __device__ constexpr int smem_bytes(int G, int slots, int tpb)
{
    return (G + slots) * kTpr * kQSeg * 8         // query rows, then key rows (fp64), padded channel slices
           + G * 8                                // per-head factor 2 / (tau ||q_h||)
           + G * tpb * kMaxP * 2 * 8              // per-plane sigmoid pairs
           + G * tpb * 2 * 16 * 8;                // nibble tables
}

// Grid: (U, 32 / TPB * ceil(L / 32)); CTA y covers tables TPB y .. TPB y +
// TPB - 1 (the ones >= L are written as zero columns).  TPB = 4, or 8 for
// per-head tables when the grid would need several waves: a thread then takes
// two hyperplane rows, one after the other, and the CTAs (each a chain of
// short dependent phases) are half as many.  Block: kThreads.  Many small CTAs keep
// every step's dependent chain short and enough warps resident to hide it.
//   1. the unit's G query rows are widened to float64 in shared memory, with
//      their norms; each thread holds 16 channels of one hyperplane row
//      (eight threads per row, 32 B each, read straight from W), widened once;
//   2. the eight threads of a row form <W_{l,p}, q_h> for four heads per pass
//      (partial sums added by shuffles), and thread j of the row turns head
//      j's projection into the two per-plane factors sigmoid(+-2z/tau), both
//      from one exponential;
//   3. the per-plane factors of planes 0-3 and 4-7 are multiplied into two
//      16-entry nibble tables per (head, table);
//   4. thread b forms entry b of the CTA's four tables,
//      T_l(b) = sum_h lo_h(b & 15) hi_h(b >> 4), rounds it once to float32
//      and writes the four adjacent columns (and their copies 32 columns on)
//      of row b of the expanded layout the scoring kernel copies into shared
//      memory: per 32-table block c a [bucket][64] row whose column j holds
//      table 32c + j mod 32.
template <typename QT, int TPB>
__global__ __launch_bounds__(kThreads, 4) void soft_tables_kernel(
    const QT* __restrict__ q, const uint16_t* __restrict__ W, int G, int L, int P, double tau,
    const AppendHash app, int64_t Ncap, int share, bool sep, float* __restrict__ tables,
    uint32_t* __restrict__ err_word, uint32_t* __restrict__ counters, uint32_t* __restrict__ topk_done,
    uint32_t* __restrict__ unit_hist, uint32_t* __restrict__ cand_cnt)
{
    static_assert(TPB == 4 || TPB == 8, "four or eight tables per CTA");
    constexpr int kTpb = TPB;
    constexpr int kRowPasses = TPB * kMaxP / (kThreads / kTpr);  // hyperplane rows per thread, at most
    __shared__ uint32_t aid[kMaxAppend][kTpb];  // ids of the appended keys (bit p <-> plane p)
    extern __shared__ __align__(16) char st_dyn[];
    // Keys appended in this step are hashed here too (step 1 of the method,
    // "Pre-cálculo"), by the first unit of each kv unit: their rows take
    // kKeySlots extra rows of qd and the same dot products as the queries.
    const bool appending = app.end > app.begin && blockIdx.x % share == 0;
    const int slots = appending ? kKeySlots : 0;
    double* qd = reinterpret_cast<double*>(st_dyn);  // [G + slots][kTpr][kQSeg]
    double* qscale = qd + (G + slots) * kTpr * kQSeg;  // [G]
    double* sig = qscale + G;                        // [G][kTpb][kMaxP][2]
    double* nib = sig + G * kTpb * kMaxP * 2;        // [G][kTpb][2][16]
    auto QD = [&](int h, int c) -> double& { return qd[(h * kTpr + (c >> 4)) * kQSeg + (c & 15)]; };
    auto SIG = [&](int h, int lt, int p, int s) -> double& { return sig[((h * kTpb + lt) * kMaxP + p) * 2 + s]; };
    auto NIB = [&](int h, int lt, int hi, int v) -> double& { return nib[((h * kTpb + lt) * 2 + hi) * 16 + v]; };
    // Appended keys k0 .. k0 + nk - 1 of the kv unit into rows G .. G + nk - 1
    // of qd, widened to float64, from 16-byte pieces (8 bf16 or 4 float32).
    auto stage_keys = [&](int k0, int nk) {
        const int per = app.kv_dtype == 1 ? 8 : 4;
        const char* kbase = static_cast<const char*>(app.K) +
                            ((int64_t)(blockIdx.x / share) * Ncap + app.begin + k0) * kHeadDim * (int64_t)(16 / per);
        for (int e = threadIdx.x; e < nk * kHeadDim / per; e += kThreads) {
            const uint4 v = *reinterpret_cast<const uint4*>(kbase + 16 * (int64_t)e);
            const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
            const int key = e * per / kHeadDim, c0 = e * per % kHeadDim;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                if (per == 8) {
                    QD(G + key, c0 + 2 * j) = bf16_bits_to_f64(w4[j] & 0xffffu);
                    QD(G + key, c0 + 2 * j + 1) = bf16_bits_to_f64(w4[j] >> 16);
                } else {
                    QD(G + key, c0 + j) = (double)__uint_as_float(w4[j]);
                }
            }
        }
    };

    const int64_t u = blockIdx.x;  // the unit's query rows are u G .. u G + G - 1 of [B][Hq]
    const int l0 = blockIdx.y * kTpb;
    const int nt = max(0, min(kTpb, L - l0));
    const int NB = 1 << P;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

    // This kernel may be launched before the previous kernel on the stream
    // has finished (programmatic dependent launch): q and W may come from
    // it, so nothing is read before the wait.  The scoring kernel may start
    // once the wait is over (its early id loads then see every earlier
    // kernel's writes).
    pdl_wait();
    pdl_launch_dependents();
    const int nk_all = appending ? (int)(app.end - app.begin) : 0;
    const int nk0 = min(kKeySlots, nk_all);  // keys projected in the same passes as the queries
    const int64_t ukv = u / share;
    // The first unit CTA's warp j fetches appended key j's value row now, for
    // its norm at the end (the load's latency overlaps the projections).
    float4 vpre = make_float4(0.f, 0.f, 0.f, 0.f);
    if (blockIdx.y == 0 && warp < nk_all) vpre = load_v4(app, (ukv * Ncap + app.begin + warp) * kHeadDim + 4 * lane);
    if (appending) {
        for (int e = tid; e < kMaxAppend * kTpb; e += kThreads) aid[e / kTpb][e % kTpb] = 0u;
    }

    if (nt > 0) {
        // This thread's slices of its hyperplane rows (pass rp: row tid / 8 +
        // 32 rp), loaded before the query is staged, so all the loads are in
        // flight together.
        const int part = tid % kTpr;
        const int wrows = nt * P;
        uint4 w2[kRowPasses][2];
#pragma unroll
        for (int rp = 0; rp < kRowPasses; ++rp) {
            const int r = tid / kTpr + rp * (kThreads / kTpr);
            w2[rp][0] = w2[rp][1] = make_uint4(0, 0, 0, 0);
            if (r < wrows) {
                const uint4* wsrc = reinterpret_cast<const uint4*>(W + ((int64_t)l0 * P + r) * kHeadDim + kChan * part);
                w2[rp][0] = __ldg(wsrc);
                w2[rp][1] = __ldg(wsrc + 1);
            }
        }
        // The unit's G query rows in 16-byte pieces (8 bf16 or 4 fp32 each).
        constexpr int kPer16 = 16 / (int)sizeof(QT);
        const int npieces = G * kHeadDim / kPer16;  // <= 512 for G <= 16
        const uint4* qu4 = reinterpret_cast<const uint4*>(q + u * G * kHeadDim);
        constexpr int kQv = (kMaxGroup * kHeadDim / kPer16 + kThreads - 1) / kThreads;
#pragma unroll
        for (int i = 0; i < kQv; ++i) {
            const int piece = tid + i * kThreads;
            if (piece < npieces) {
                const uint4 v = __ldg(qu4 + piece);
                const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
                const int h = piece * kPer16 / kHeadDim, c0 = piece * kPer16 % kHeadDim;
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    if constexpr (sizeof(QT) == 2) {
                        QD(h, c0 + 2 * e) = bf16_bits_to_f64(w4[e] & 0xffffu);
                        QD(h, c0 + 2 * e + 1) = bf16_bits_to_f64(w4[e] >> 16);
                    } else {
                        QD(h, c0 + e) = (double)__uint_as_float(w4[e]);
                    }
                }
            }
        }
        stage_keys(0, nk0);
        __syncthreads();
        // Per head, the factor taking <W_{l,p}, q_h> to the sigmoid argument
        // 2 z / tau with z = <W_{l,p}, q_h> / ||q_h|| (0 for a zero query).
        for (int h = warp; h < G; h += kThreads / 32) {
            double s = 0.0;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const double x = QD(h, 4 * lane + j);
                s = fma(x, x, s);
            }
            for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(kFullMask, s, o);
            if (lane == 0) qscale[h] = (s > 0.0 && tau > 0.0) ? 2.0 / (tau * sqrt(s)) : 0.0;
        }
#pragma unroll 1
        for (int rp = 0; rp < kRowPasses; ++rp) {
            if (rp * (kThreads / kTpr) >= wrows) break;  // no row of this pass is live (CTA-uniform)
            const int r = tid / kTpr + rp * (kThreads / kTpr);
            const bool live = r < wrows;
            if (rp > 0 && nk_all > kKeySlots) {
                // The first appended keys again (later ones took their rows).
                __syncthreads();
                stage_keys(0, nk0);
            }
            double wd[kChan];  // this thread's 16 channels of the row, widened once
            {
                const uint32_t words[8] = {w2[rp][0].x, w2[rp][0].y, w2[rp][0].z, w2[rp][0].w,
                                           w2[rp][1].x, w2[rp][1].y, w2[rp][1].z, w2[rp][1].w};
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    wd[2 * i] = bf16_bits_to_f64(words[i] & 0xffffu);
                    wd[2 * i + 1] = bf16_bits_to_f64(words[i] >> 16);
                }
            }
            __syncthreads();
            // Rows 0 .. G-1 of qd are the queries, rows G .. G + nk0 - 1 the first
            // appended keys: bit p of a key's id in table l is [<W_{l,p}, k> > 0].
            const int lt = live ? r / P : 0, p = live ? r - lt * P : 0;
            const int Ht = G + nk0;
            for (int h0 = 0; h0 < Ht; h0 += kHeadsPerPass) {
                double acc[kHeadsPerPass];
#pragma unroll
                for (int hh = 0; hh < kHeadsPerPass; ++hh) {
                    double a0 = 0.0, a1 = 0.0;
                    if (h0 + hh < Ht) {
                        const double* qh = &QD(h0 + hh, kChan * part);
#pragma unroll
                        for (int i = 0; i < kChan; i += 2) {
                            const double2 qv2 = *reinterpret_cast<const double2*>(qh + i);
                            a0 = fma(wd[i], qv2.x, a0);
                            a1 = fma(wd[i + 1], qv2.y, a1);
                        }
                    }
                    acc[hh] = a0 + a1;
                }
                // Sum the row's eight slices; thread hh of the row finishes head h0 + hh.
#pragma unroll
                for (int hh = 0; hh < kHeadsPerPass; ++hh) {
                    acc[hh] += __shfl_xor_sync(kFullMask, acc[hh], 1);
                    acc[hh] += __shfl_xor_sync(kFullMask, acc[hh], 2);
                    acc[hh] += __shfl_xor_sync(kFullMask, acc[hh], 4);
                }
                const double y = part == 0 ? acc[0] : part == 1 ? acc[1] : part == 2 ? acc[2] : acc[3];
                const int h = h0 + part;
                if (live && part < kHeadsPerPass && h >= G && h < Ht) {
                    if (y > 0.0) atomicOr(&aid[h - G][lt], 1u << p);
                } else if (live && part < kHeadsPerPass && h < G) {
                    if (tau == 0.0) {
                        // Hard LSH: the plane's bit is [<W_{l,p}, q_h> > 0], as for keys.
                        SIG(h, lt, p, 1) = y > 0.0 ? 1.0 : 0.0;
                        SIG(h, lt, p, 0) = y > 0.0 ? 0.0 : 1.0;
                    } else {
                        // sigmoid(+-x) from one exponential: e = exp(-|x|),
                        // sigmoid(|x|) = 1 / (1 + e), sigmoid(-|x|) = e / (1 + e).
                        const double x = y * qscale[h];
                        const double e = exp(-fabs(x));
                        const double big = 1.0 / (1.0 + e), small = e * big;
                        SIG(h, lt, p, 1) = x >= 0.0 ? big : small;  // sign +1: bit set
                        SIG(h, lt, p, 0) = x >= 0.0 ? small : big;  // sign -1: bit clear
                    }
                }
            }
            // Any further appended keys, kKeySlots at a time, on the same rows.
            for (int k0 = kKeySlots; k0 < nk_all; k0 += kKeySlots) {
                const int nk = min(kKeySlots, nk_all - k0);
                __syncthreads();  // the previous keys' rows have been read
                stage_keys(k0, nk);
                __syncthreads();
                for (int h0 = 0; h0 < nk; h0 += kHeadsPerPass) {
                    double acc[kHeadsPerPass];
#pragma unroll
                    for (int hh = 0; hh < kHeadsPerPass; ++hh) {
                        double a0 = 0.0, a1 = 0.0;
                        if (h0 + hh < nk) {
                            const double* kh = &QD(G + h0 + hh, kChan * part);
#pragma unroll
                            for (int i = 0; i < kChan; i += 2) {
                                const double2 kv2 = *reinterpret_cast<const double2*>(kh + i);
                                a0 = fma(wd[i], kv2.x, a0);
                                a1 = fma(wd[i + 1], kv2.y, a1);
                            }
                        }
                        acc[hh] = a0 + a1;
                    }
#pragma unroll
                    for (int hh = 0; hh < kHeadsPerPass; ++hh) {
                        acc[hh] += __shfl_xor_sync(kFullMask, acc[hh], 1);
                        acc[hh] += __shfl_xor_sync(kFullMask, acc[hh], 2);
                        acc[hh] += __shfl_xor_sync(kFullMask, acc[hh], 4);
                    }
                    const double y = part == 0 ? acc[0] : part == 1 ? acc[1] : part == 2 ? acc[2] : acc[3];
                    if (live && part < kHeadsPerPass && h0 + part < nk && y > 0.0)
                        atomicOr(&aid[k0 + h0 + part][lt], 1u << p);
                }
            }
        }
        __syncthreads();

        // Nibble tables: lo over planes 0..min(P,4)-1, hi over planes 4..P-1.
        const int plo = min(P, 4);
        for (int e = tid; e < G * kTpb * 32; e += kThreads) {
            const int h = e / (kTpb * 32), t = (e >> 5) % kTpb, hi = (e >> 4) & 1, v = e & 15;
            if (t >= nt) continue;
            double prod = 1.0;
            const int p0 = hi ? 4 : 0, p1 = hi ? P : plo;
            for (int pp = p0; pp < p1; ++pp) prod *= SIG(h, t, pp, (v >> (pp - p0)) & 1);
            NIB(h, t, hi, v) = prod;
        }
        __syncthreads();
    }

    // Units whose tables this CTA writes: u itself, or (sep) the G units
    // u G .. u G + G - 1, one per query head.
    const int nunits = sep ? G : 1;
    const int64_t unit0 = sep ? u * G : u;
    if (blockIdx.y == 0) {
        if (tid < nunits) {
            const int64_t uu = unit0 + tid;
            counters[uu] = 0u;
            topk_done[uu] = 0u;
            cand_cnt[uu] = 0u;
            if (uu == 0) *err_word = 0u;
        }
        uint4* hz = reinterpret_cast<uint4*>(unit_hist + unit0 * kScoreHistBins);
        for (int i = tid; i < nunits * kScoreHistBins / 4; i += kThreads) hz[i] = make_uint4(0, 0, 0, 0);
    }
    const int nblk = (L + 31) / 32;
    // Entry `bucket` of the CTA's four tables: four adjacent columns (and
    // their copies 32 columns on) of one row, as vector stores.  Summed over
    // the G heads, or (sep) one table per head, T = lo x hi rounded once.
    for (int e = tid; e < nunits * NB; e += kThreads) {
        const int bucket = e % NB, hs = e / NB;
        float vals[kTpb];
#pragma unroll
        for (int t = 0; t < kTpb; ++t) {
            double acc = 0.0;
            if (t < nt) {
                if (sep) {
                    acc = fma(NIB(hs, t, 0, bucket & 15), NIB(hs, t, 1, bucket >> 4), acc);
                } else {
                    for (int h0 = 0; h0 < G; h0 += 4)
#pragma unroll
                        for (int hh = 0; hh < 4; ++hh)
                            if (h0 + hh < G)
                                acc = fma(NIB(h0 + hh, t, 0, bucket & 15), NIB(h0 + hh, t, 1, bucket >> 4), acc);
                }
            }
            vals[t] = (float)acc;
        }
        float* tu = tables + (unit0 + hs) * nblk * (int64_t)NB * 64;
        float* row = tu + ((int64_t)(l0 >> 5) * NB + bucket) * 64 + (l0 & 31);
#pragma unroll
        for (int t4 = 0; t4 < kTpb; t4 += 4) {
            const float4 a = make_float4(vals[t4], vals[t4 + 1], vals[t4 + 2], vals[t4 + 3]);
            *reinterpret_cast<float4*>(row + t4) = a;
            *reinterpret_cast<float4*>(row + t4 + 32) = a;
        }
    }

    // The appended keys' id slots of this CTA's four tables (0 for tables
    // >= L), and for the unit's first CTA their norms (float64 sums).  The
    // scoring kernel reads these rows only after this grid has completed.
    // (aid is complete: its last writes precede the barrier before the
    // nibble tables; a CTA with nt == 0 writes zeros without reading it.)
    if (appending) {
        const int nk = nk_all;
        const int Lr = 32 * nblk, pieces = Lr / 16;
        uint8_t* idu = app.ids + ukv * Ncap * Lr;
        // Byte of table l in key n's rotated row: block l / 32, slot (l - n) mod 32.
        auto id_byte = [&](int64_t n, int l) -> uint8_t* {
            const int b = (l & ~31) + (((l & 31) - (int)(n & 31)) & 31);
            return idu + ((n >> 5) * pieces + (b >> 4)) * 512 + (n & 31) * 16 + (b & 15);
        };
        for (int e = tid; e < nk * kTpb; e += kThreads) {
            const int key = e / kTpb, t = e % kTpb;
            *id_byte(app.begin + key, l0 + t) = t < nt ? (uint8_t)aid[key][t] : (uint8_t)0;
        }
        if (blockIdx.y == 0) {
            for (int key = warp; key < nk; key += kThreads / 32) {
                const float4 vf =
                    key == warp ? vpre : load_v4(app, (ukv * Ncap + app.begin + key) * kHeadDim + 4 * lane);
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
                               uint32_t* counters, uint32_t* topk_done, uint32_t* unit_hist, uint32_t* cand_cnt,
                               cudaStream_t stream)
{
    // When every query head selects its own keys (G = 1, share heads per kv
    // unit), a CTA builds the tables of all `share` heads of a kv unit: their
    // dot products share the hyperplane rows' reads, as a group's do, and
    // each head keeps its own table (the same operations as one head alone).
    const bool sep = s.G == 1 && s.share > 1;
    const int G = sep ? s.share : s.G;
    const int share = sep ? 1 : s.share;
    const int64_t ctas = sep ? s.U / s.share : s.U;
    // Four tables per CTA; eight for per-head tables when four would need
    // several waves (there each CTA writes all its heads' tables, and halving
    // the CTAs pays; for grouped tables it measured slower).
    const int nblk = (s.L + 31) / 32;
    const int tpb = sep && ctas * 8 * nblk > 4 * (int64_t)device_num_sms() ? 8 : 4;
    const int slots = app.end > app.begin ? kKeySlots : 0;
    const int smem = smem_bytes(G, slots, tpb);
    const dim3 grid((unsigned)ctas, (unsigned)(32 / tpb * nblk));
#define SOCKET_ST_CASE(QTT, TPBV)                                                                              \
    {                                                                                                          \
        cudaError_t e = set_smem_limit_once((const void*)soft_tables_kernel<QTT, TPBV>,                        \
                                            smem_bytes(kMaxGroup, kKeySlots, TPBV));                           \
        if (e != cudaSuccess) return e;                                                                        \
        return launch_pdl(soft_tables_kernel<QTT, TPBV>, grid, dim3(kThreads), (size_t)smem, stream,          \
                          static_cast<const QTT*>(q), W, G, s.L, s.P, tau, app, s.Ncap, share, sep, tables,    \
                          err_word, counters, topk_done, unit_hist, cand_cnt);                                 \
    }
    if (q_dtype == 1) {
        if (tpb == 8) SOCKET_ST_CASE(uint16_t, 8)
        SOCKET_ST_CASE(uint16_t, 4)
    }
    if (tpb == 8) SOCKET_ST_CASE(float, 8)
    SOCKET_ST_CASE(float, 4)
#undef SOCKET_ST_CASE
}

}  // namespace socket_attn
