// The whole decode step in one kernel for small problems: soft tables,
// soft collision scores, deterministic top-k and exact attention, one CTA per
// unit, with nothing left in global memory between the steps.
//
// Method: "Resumen Técnico: SOCKET ..." (gist.science/es/paper/2602.06283),
// "Mecanismo Central: LSH Suave" steps 2-4; "SOCKET: SOft Collision Kernel
// EsTimator for Sparse Attention" (gist.science/de/paper/2602.06283),
// "Weiche Zuweisung (Decoding)", "Bewertung", "Auswahl".
//
// For a few thousand keys the separate kernels are bound by their launch and
// hand-off latencies, not by their work.  Here a CTA of 512 threads runs the
// four steps of one unit back to back in shared memory:
//   1. soft tables T_l(b) = sum_h prod_p sigmoid(2 s_{b,p} z_{h,l,p} / tau)
//      in float64, rounded once to float32 -- the same operations, in the
//      same order, as the soft-table kernel, so every entry is bit-identical;
//      stored as [bucket][64 columns], column c holding table c mod 32, so
//      the lookups below hit 32 distinct banks;
//   2. scores s(n) = vnorm(n) * sum over the id row's 32 slots of T, added
//      slot by slot in the scoring kernel's order (slot r of key n holds
//      table (r + n) mod 32; slots past L hold zero entries), so every score
//      is bit-identical to the scoring kernel's;
//   3. the k largest scores, ties to the lower index: three radix digits over
//      the score bit patterns, then the selection written in index order;
//   4. attention over the selected keys in float32 on the CUDA cores: each
//      warp keeps an online softmax per head over its share of the keys, the
//      16 warps' states are merged in a fixed order.
// No wait in this kernel depends on another CTA or on a copy: it has no
// bounded waits and sets no error bits.
#include "common.cuh"
#include "internal.h"
#include "select.cuh"
#include "socket_attn.h"

namespace socket_attn {
namespace {

using namespace select512;

constexpr int kSmallMaxN = 8192;      // scores of a unit in shared memory
constexpr int kSmallMaxK = 1024;
constexpr int kSmallMaxG = 8;
constexpr int kSmallMaxGL = 64;       // G * L: nibble tables of the soft step
constexpr int kSmallMaxGLP = 512;     // G * L * P: sigmoid pairs of the soft step
constexpr int kTpr = 8;               // threads per hyperplane row (16 channels each)
constexpr int kChan = kHeadDim / kTpr;
constexpr int kQSeg = kChan + 2;      // padded float64 segment of a query row
constexpr float kInvSqrtD = 0.088388347648318440550f;  // 1 / sqrt(128)
constexpr int kKeysPerRound = 4;      // keys a thread scores per round (loads in flight together)

// bfloat16 bits (low 16) -> float64, exact (as the soft-table kernel widens).
__device__ __forceinline__ double bf16_bits_to_f64_exact(uint32_t b)
{
    const uint32_t mag = b & 0x7fffu, e = mag >> 7;
    if (e == 0u || e == 0xffu) return (double)__uint_as_float(b << 16);
    return __hiloint2double((int)(((b & 0x8000u) << 16) | ((mag << 13) + (896u << 20))), 0);
}

struct SmallArgs {
    const void* q;          // [U * G][128], q_dtype
    const uint16_t* W;      // [L][P][128] bf16
    const uint8_t* ids;     // [U / share][Ncap / 32][Lr / 16][32][16] rotated id rows (Lr = 32)
    const float* vnorm;     // [U / share][Ncap]
    const void* K;          // [U / share][Ncap][128], kv_dtype
    const void* V;
    int32_t* idx_out;       // [U][k]
    float* out;             // [U * G][128]
    float* scores_out;      // [U][Ncap] or null
    uint32_t* err_word;
    int64_t Ncap;
    int N, k, G, L, P, share;
    double tau;
};

// Dynamic shared memory: tables [NB][64] float32 (later the warps' attention
// states [16][8][128]); scores [kSmallMaxN] (first the soft step's float64
// scratch); the selection [kSmallMaxK].
constexpr int kTablesBytes = 256 * 64 * 4;
constexpr int kStatesBytes = 16 * 8 * kHeadDim * 4;
constexpr int kRegionA = kTablesBytes > kStatesBytes ? kTablesBytes : kStatesBytes;
constexpr int kScoresBytes = 36 * 1024;  // kSmallMaxN scores, or the soft step's scratch
constexpr int kSmallSmem = kRegionA + kScoresBytes + kSmallMaxK * 4;
static_assert(kSmallMaxN * 4 <= kScoresBytes, "the scores fit the score region");
static_assert(kSmallMaxG * kTpr * kQSeg * 8 + kSmallMaxG * 8 + kSmallMaxGLP * 16 + kSmallMaxGL * 32 * 8 <= kScoresBytes,
              "the soft step's scratch fits the score region");

// MAXG: query heads per unit the attention registers are sized for (G <= MAXG).
template <typename QT, typename KT, int MAXG>
__global__ __launch_bounds__(kThreads, 1) void small_step_kernel(const SmallArgs a)
{
    __shared__ Shared sh;
    __shared__ float wm[kWarps][kSmallMaxG], wl[kWarps][kSmallMaxG];
    extern __shared__ __align__(16) char small_dyn[];
    float* T64 = reinterpret_cast<float*>(small_dyn);                        // [NB][64]
    float* st_o = reinterpret_cast<float*>(small_dyn);                       // [16][8][128] (step 4)
    float* sc = reinterpret_cast<float*>(small_dyn + kRegionA);              // [N]
    uint32_t* scb = reinterpret_cast<uint32_t*>(sc);
    int32_t* sel = reinterpret_cast<int32_t*>(small_dyn + kRegionA + kScoresBytes);  // [k]
    // Soft step scratch, inside the score region.
    double* qd = reinterpret_cast<double*>(sc);                              // [G][kTpr][kQSeg]
    double* qscale = qd + kSmallMaxG * kTpr * kQSeg;                         // [G]
    double* sig = qscale + kSmallMaxG;                                       // [G][L][P][2]
    double* nib = sig + kSmallMaxGLP * 2;                                    // [G][L][2][16]

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int G = a.G, L = a.L, P = a.P, NB = 1 << a.P, N = a.N, k = a.k;
    const int64_t u = blockIdx.x;
    const int64_t ukv = u / a.share;
    const int64_t qrow0 = u * G;
    auto QD = [&](int h, int c) -> double& { return qd[(h * kTpr + (c >> 4)) * kQSeg + (c & 15)]; };
    auto SIG = [&](int h, int l, int p, int s) -> double& { return sig[((h * L + l) * P + p) * 2 + s]; };
    auto NIB = [&](int h, int l, int hi, int v) -> double& { return nib[((h * L + l) * 2 + hi) * 16 + v]; };

    // q and W may come from the previous kernel on the stream.
    pdl_wait();
    pdl_launch_dependents();
    if (u == 0 && tid == 0) *a.err_word = 0u;

    // ---- 1. soft tables.
    // The unit's query rows, widened to float64.
    for (int e = tid; e < G * kHeadDim; e += kThreads) {
        const int h = e / kHeadDim, c = e % kHeadDim;
        double x;
        if constexpr (sizeof(QT) == 2)
            x = bf16_bits_to_f64_exact(static_cast<const uint16_t*>(a.q)[(qrow0 + h) * kHeadDim + c]);
        else
            x = (double)static_cast<const float*>(a.q)[(qrow0 + h) * kHeadDim + c];
        QD(h, c) = x;
    }
    __syncthreads();
    // Per head, 2 / (tau ||q_h||) (0 for a zero query or tau = 0).
    for (int h = warp; h < G; h += kWarps) {
        double s = 0.0;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const double x = QD(h, 4 * lane + j);
            s = fma(x, x, s);
        }
        for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(kFullMask, s, o);
        if (lane == 0) qscale[h] = (s > 0.0 && a.tau > 0.0) ? 2.0 / (a.tau * sqrt(s)) : 0.0;
    }
    __syncthreads();
    // <W_{l,p}, q_h>: eight threads per hyperplane row, 16 channels each,
    // even and odd channels in two sums, the slices added by shuffles; thread
    // `part` of the row turns head `part`'s projection into its sigmoid pair.
    {
        const int part = tid % kTpr;
        for (int r0 = 0; r0 < L * P; r0 += kThreads / kTpr) {
            const int r = r0 + tid / kTpr;
            const bool live = r < L * P;
            double wd[kChan];
            {
                uint4 w2[2] = {make_uint4(0, 0, 0, 0), make_uint4(0, 0, 0, 0)};
                if (live) {
                    const uint4* src = reinterpret_cast<const uint4*>(a.W + (int64_t)r * kHeadDim + kChan * part);
                    w2[0] = __ldg(src);
                    w2[1] = __ldg(src + 1);
                }
                const uint32_t words[8] = {w2[0].x, w2[0].y, w2[0].z, w2[0].w, w2[1].x, w2[1].y, w2[1].z, w2[1].w};
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    wd[2 * i] = bf16_bits_to_f64_exact(words[i] & 0xffffu);
                    wd[2 * i + 1] = bf16_bits_to_f64_exact(words[i] >> 16);
                }
            }
            const int l = live ? r / P : 0, p = live ? r % P : 0;
            for (int h = 0; h < G; ++h) {
                double a0 = 0.0, a1 = 0.0;
                const double* qh = &QD(h, kChan * part);
#pragma unroll
                for (int i = 0; i < kChan; i += 2) {
                    a0 = fma(wd[i], qh[i], a0);
                    a1 = fma(wd[i + 1], qh[i + 1], a1);
                }
                double y = a0 + a1;
                y += __shfl_xor_sync(kFullMask, y, 1);
                y += __shfl_xor_sync(kFullMask, y, 2);
                y += __shfl_xor_sync(kFullMask, y, 4);
                if (live && part == h % kTpr) {
                    if (a.tau == 0.0) {
                        // Hard LSH: the plane's bit is [<W_{l,p}, q_h> > 0], as for keys.
                        SIG(h, l, p, 1) = y > 0.0 ? 1.0 : 0.0;
                        SIG(h, l, p, 0) = y > 0.0 ? 0.0 : 1.0;
                    } else {
                        // sigmoid(+-x) from one exponential.
                        const double x = y * qscale[h];
                        const double e = exp(-fabs(x));
                        const double big = 1.0 / (1.0 + e), small = e * big;
                        SIG(h, l, p, 1) = x >= 0.0 ? big : small;
                        SIG(h, l, p, 0) = x >= 0.0 ? small : big;
                    }
                }
            }
        }
    }
    __syncthreads();
    // Nibble tables: lo over planes 0..min(P,4)-1, hi over planes 4..P-1.
    {
        const int plo = min(P, 4);
        for (int e = tid; e < G * L * 32; e += kThreads) {
            const int v = e & 15, hi = (e >> 4) & 1, hl = e >> 5;
            const int h = hl / L, l = hl % L;
            double prod = 1.0;
            const int p0 = hi ? 4 : 0, p1 = hi ? P : plo;
            for (int pp = p0; pp < p1; ++pp) prod *= SIG(h, l, pp, (v >> (pp - p0)) & 1);
            NIB(h, l, hi, v) = prod;
        }
    }
    __syncthreads();
    // T64[b][c] = T_{c mod 32}(b) for tables < L, else 0.
    for (int e = tid; e < NB * 64; e += kThreads) {
        const int b = e >> 6, l = e & 31;
        double acc = 0.0;
        if (l < L)
            for (int h = 0; h < G; ++h) acc = fma(NIB(h, l, 0, b & 15), NIB(h, l, 1, b >> 4), acc);
        T64[e] = (float)acc;
    }
    __syncthreads();  // the scratch (in the score region) is dead from here on

    // ---- 2. scores.  Thread t scores keys t, t + 512, ... (lane = key mod 32).
    {
        const uint8_t* idu = a.ids + ukv * a.Ncap * 32;
        const float* vu = a.vnorm + ukv * a.Ncap;
        const uint32_t tb = smem_addr(T64) + 4u * (uint32_t)lane;
        for (int n0 = tid; n0 < N; n0 += kThreads * kKeysPerRound) {
            uint4 w[kKeysPerRound][2];
            float vn[kKeysPerRound];
#pragma unroll
            for (int j = 0; j < kKeysPerRound; ++j) {
                const int n = n0 + j * kThreads;
                if (n < N) {
                    const uint4* row = reinterpret_cast<const uint4*>(idu + ((int64_t)(n >> 5) * 2 * 32 + (n & 31)) * 16);
                    w[j][0] = __ldg(row);
                    w[j][1] = __ldg(row + 32);
                    vn[j] = __ldg(vu + n);
                } else {
                    w[j][0] = w[j][1] = make_uint4(0, 0, 0, 0);
                    vn[j] = 0.0f;
                }
            }
#pragma unroll
            for (int j = 0; j < kKeysPerRound; ++j) {
                const int n = n0 + j * kThreads;
                const uint32_t words[8] = {w[j][0].x, w[j][0].y, w[j][0].z, w[j][0].w,
                                           w[j][1].x, w[j][1].y, w[j][1].z, w[j][1].w};
                float acc = 0.0f;
#pragma unroll
                for (int s = 0; s < 32; ++s) {
                    const uint32_t id = (words[s >> 2] >> (8 * (s & 3))) & 0xffu;
                    float t;
                    asm volatile("ld.shared.f32 %0, [%1];" : "=f"(t) : "r"(tb + (id * 64u + (uint32_t)s) * 4u));
                    acc += t;
                }
                if (n < N) {
                    const float s = acc * vn[j];
                    sc[n] = s;
                    if (a.scores_out) a.scores_out[u * a.Ncap + n] = s;
                }
            }
        }
    }
    __syncthreads();

    // ---- 3. the k largest, ties to the lower index, in index order.
    {
        uint32_t prefix = 0, mask = 0, krem = (uint32_t)k;
        auto get = [&](int i) { return scb[i]; };
        // A digit's bin holding exactly the keys still needed is taken whole:
        // its lowest pattern is the threshold and the later digits are skipped.
        radix_digit(sh, N, get, 20, 0x7ffu, true, prefix, mask, krem);
        if (sh.count != krem) {
            radix_digit(sh, N, get, 9, 0x7ffu, true, prefix, mask, krem);
            if (sh.count != krem) radix_digit(sh, N, get, 0, 0x1ffu, true, prefix, mask, krem);
        }
        const uint32_t t = prefix;
        // Keys above t, and the first krem keys equal to t, in index order
        // (tiles of 16 consecutive keys per thread, block-wide scans).
        constexpr int kPer = 16;
        int32_t* outi = a.idx_out + u * (int64_t)k;
        uint32_t out_base = 0, ties_seen = 0;
        for (int tile = 0; tile < N; tile += kThreads * kPer) {
            const int i0 = tile + tid * kPer;
            uint32_t gt = 0, eq = 0;
#pragma unroll
            for (int e = 0; e < kPer; ++e)
                if (i0 + e < N) {
                    gt += scb[i0 + e] > t;
                    eq += scb[i0 + e] == t;
                }
            uint32_t tot_gt, tot_eq;
            const uint32_t gt_before = block_exclusive_scan(gt, sh.warp_sums, tot_gt);
            const uint32_t eq_before = block_exclusive_scan(eq, sh.warp_sums, tot_eq);
            const uint32_t left = krem > ties_seen ? krem - ties_seen : 0u;
            uint32_t pos = out_base + gt_before + min(eq_before, left);
            uint32_t my_eq = eq_before;
#pragma unroll
            for (int e = 0; e < kPer; ++e) {
                if (i0 + e >= N) continue;
                const uint32_t x = scb[i0 + e];
                const bool take = x > t || (x == t && my_eq < left);
                my_eq += x == t;
                // pos < k whenever the threshold is exact; the guard keeps every
                // store inside the unit's k slots regardless.
                if (take) {
                    if (pos < (uint32_t)k) {
                        outi[pos] = i0 + e;
                        sel[pos] = i0 + e;
                    }
                    ++pos;
                }
            }
            out_base += tot_gt + min(tot_eq, left);
            ties_seen += tot_eq;
        }
        __syncthreads();
    }

    // ---- 4. attention: warp w takes selected keys w, w + 16, ...; lane c
    // holds channels 4c .. 4c + 3 of each head's query and output.
    float qv[MAXG][4], ov[MAXG][4], m_run[MAXG], l_run[MAXG];
#pragma unroll
    for (int h = 0; h < MAXG; ++h) {
        m_run[h] = -INFINITY;
        l_run[h] = 0.0f;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            ov[h][c] = 0.0f;
            float x = 0.0f;
            if (h < G) {
                const int64_t off = (qrow0 + h) * kHeadDim + 4 * lane + c;
                if constexpr (sizeof(QT) == 2)
                    x = bf16_to_f32(static_cast<const uint16_t*>(a.q)[off]);
                else
                    x = static_cast<const float*>(a.q)[off];
            }
            qv[h][c] = x;
        }
    }
    auto load4 = [&](const void* base, int64_t row) -> float4 {
        if constexpr (sizeof(KT) == 2) {
            const uint2 w2 = __ldg(reinterpret_cast<const uint2*>(static_cast<const uint16_t*>(base) + row * kHeadDim) + lane);
            const float2 x01 = bf16x2_to_f32x2(w2.x), x23 = bf16x2_to_f32x2(w2.y);
            return make_float4(x01.x, x01.y, x23.x, x23.y);
        } else {
            return __ldg(reinterpret_cast<const float4*>(static_cast<const float*>(base) + row * kHeadDim) + lane);
        }
    };
    constexpr int kAK = MAXG <= 2 ? 8 : 2;  // keys of a warp in flight together (as registers allow)
    for (int i0 = warp; i0 < k; i0 += kWarps * kAK) {
        float4 kr[kAK], vr[kAK];
#pragma unroll
        for (int j = 0; j < kAK; ++j) {
            const int i = i0 + j * kWarps;
            const int64_t row = ukv * a.Ncap + (i < k ? sel[i] : 0);
            kr[j] = load4(a.K, row);
            vr[j] = load4(a.V, row);
        }
#pragma unroll
        for (int j = 0; j < kAK; ++j) {
            if (i0 + j * kWarps >= k) break;
#pragma unroll
            for (int h = 0; h < MAXG; ++h) {
                if (h >= G) break;
                float d = qv[h][0] * kr[j].x;
                d = fmaf(qv[h][1], kr[j].y, d);
                d = fmaf(qv[h][2], kr[j].z, d);
                d = fmaf(qv[h][3], kr[j].w, d);
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) d += __shfl_xor_sync(kFullMask, d, o);
                const float logit = d * kInvSqrtD;
                const float m_new = fmaxf(m_run[h], logit);
                const float sc_old = expf(m_run[h] - m_new);  // 0 on the first key
                const float wgt = expf(logit - m_new);
                l_run[h] = l_run[h] * sc_old + wgt;
                ov[h][0] = ov[h][0] * sc_old + wgt * vr[j].x;
                ov[h][1] = ov[h][1] * sc_old + wgt * vr[j].y;
                ov[h][2] = ov[h][2] * sc_old + wgt * vr[j].z;
                ov[h][3] = ov[h][3] * sc_old + wgt * vr[j].w;
                m_run[h] = m_new;
            }
        }
    }
    // The warps' states -> shared memory; merged per head in warp order.
#pragma unroll
    for (int h = 0; h < MAXG; ++h) {
        if (h >= G) break;
        if (lane == 0) {
            wm[warp][h] = m_run[h];
            wl[warp][h] = l_run[h];
        }
        *reinterpret_cast<float4*>(st_o + (warp * kSmallMaxG + h) * kHeadDim + 4 * lane) =
            make_float4(ov[h][0], ov[h][1], ov[h][2], ov[h][3]);
    }
    __syncthreads();
    for (int e = tid; e < G * kHeadDim; e += kThreads) {
        const int h = e / kHeadDim, c = e % kHeadDim;
        float M = -INFINITY;
        for (int w = 0; w < kWarps; ++w) M = fmaxf(M, wm[w][h]);
        float o = 0.0f, l = 0.0f;
        for (int w = 0; w < kWarps; ++w) {
            const float wt = wm[w][h] == -INFINITY ? 0.0f : expf(wm[w][h] - M);
            o += wt * st_o[(w * kSmallMaxG + h) * kHeadDim + c];
            l += wt * wl[w][h];
        }
        a.out[(qrow0 + h) * kHeadDim + c] = l > 0.0f ? o / l : 0.0f;
    }
}

template <typename QT, typename KT, int MAXG>
cudaError_t launch_small(const SmallArgs& a, dim3 grid, dim3 block, cudaStream_t stream)
{
    cudaError_t e = set_smem_limit_once((const void*)small_step_kernel<QT, KT, MAXG>, kSmallSmem);
    if (e != cudaSuccess) return e;
    e = launch_pdl(small_step_kernel<QT, KT, MAXG>, grid, block, (size_t)kSmallSmem, stream, a);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace

bool small_step_supported(const DecodeShape& s, int num_sms)
{
    return s.d == kHeadDim && s.N <= kSmallMaxN && s.k <= kSmallMaxK && s.G <= kSmallMaxG && s.L <= 32 &&
           s.G * s.L <= kSmallMaxGL && s.G * s.L * s.P <= kSmallMaxGLP && s.U <= num_sms;
}

cudaError_t launch_small_step(const void* q, int q_dtype, const uint16_t* W, const uint8_t* ids, const float* vnorm,
                              const void* K, const void* V, int kv_dtype, const DecodeShape& s, double tau,
                              int32_t* idx_out, float* out, float* scores_out, uint32_t* err_word,
                              cudaStream_t stream)
{
    SmallArgs a;
    a.q = q;
    a.W = W;
    a.ids = ids;
    a.vnorm = vnorm;
    a.K = K;
    a.V = V;
    a.idx_out = idx_out;
    a.out = out;
    a.scores_out = scores_out;
    a.err_word = err_word;
    a.Ncap = s.Ncap;
    a.N = (int)s.N;
    a.k = s.k;
    a.G = s.G;
    a.L = s.L;
    a.P = s.P;
    a.share = s.share;
    a.tau = tau;
    const dim3 grid((unsigned)s.U), block(kThreads);
#define SOCKET_SMALL_CASE(QTT, KTT)                                                                       \
    return s.G <= 2 ? launch_small<QTT, KTT, 2>(a, grid, block, stream) : launch_small<QTT, KTT, 8>(a, grid, block, stream);
    if (q_dtype == SOCKET_BF16) {
        if (kv_dtype == SOCKET_BF16) SOCKET_SMALL_CASE(uint16_t, uint16_t)
        SOCKET_SMALL_CASE(uint16_t, float)
    }
    if (kv_dtype == SOCKET_BF16) SOCKET_SMALL_CASE(float, uint16_t)
    SOCKET_SMALL_CASE(float, float)
#undef SOCKET_SMALL_CASE
}

}  // namespace socket_attn
