// Exact softmax attention over the selected keys (split-K flash decode).
//
// Method: "Resumen Técnico: SOCKET ..." (gist.science/es/paper/2602.06283),
// "Mecanismo Central: LSH Suave" step 4 "Selección": exact attention is
// computed over the selected subset; "SOCKET: SOft Collision Kernel EsTimator
// for Sparse Attention" (gist.science/de/paper/2602.06283), "Auswahl".  The
// pages run this step with a "Flash Decode" backend ("Contribuciones Clave"
// 2 / "Hauptbeiträge"); here it is a hand-written split-K kernel.
//
// Each CTA takes a run of a unit's selected rows, in chunks of 64 rows with
// two chunks in flight: the chunk's key and value rows are gathered into
// shared memory with bulk asynchronous copies (one 256-byte row per copy,
// completion counted on that stage's mbarrier) while the previous chunk is
// being used.  The CTA computes the logits of all query heads of the unit
// (scale 1/sqrt(d)) and keeps an online softmax (running max, running sum,
// rescaled weighted value sum).  The last CTA of a unit to finish (an atomic
// ticket, no waiting) merges the CTAs' partials in split order with the
// usual log-sum-exp rescaling and writes the normalised float32 output, so
// the merge is deterministic.
#include "common.cuh"
#include "internal.h"
#include "socket_attn.h"

namespace socket_attn {
namespace {

constexpr int kThreads = 128;
constexpr uint32_t kMaxPolls = 1u << 22;
constexpr float kScale = 0.088388347648318440550f;  // 1 / sqrt(128)

template <typename KT>
struct Rows;
template <>
struct Rows<uint16_t> {  // bfloat16
    static constexpr int kChunk = 64;
    static constexpr int kRowBytes = kHeadDim * 2;
};
template <>
struct Rows<float> {
    static constexpr int kChunk = 32;
    static constexpr int kRowBytes = kHeadDim * 4;
};

// Four consecutive elements of a row, as floats.
__device__ __forceinline__ float4 load4(const uint16_t* row, int j)
{
    const uint2 w = *reinterpret_cast<const uint2*>(row + j);
    const float2 a = bf16x2_to_f32x2(w.x), b = bf16x2_to_f32x2(w.y);
    return make_float4(a.x, a.y, b.x, b.y);
}
__device__ __forceinline__ float4 load4(const float* row, int j) { return *reinterpret_cast<const float4*>(row + j); }

__device__ __forceinline__ float load1(const uint16_t* row, int j) { return bf16_to_f32(row[j]); }
__device__ __forceinline__ float load1(const float* row, int j) { return row[j]; }

// The last CTA of a unit to finish (an atomic ticket, no waiting) merges the
// unit's partials in split order: per head, M = max_s m_s, w_s = exp(m_s - M),
// out = sum_s w_s o_s / sum_s w_s l_s.  Weights are staged in shared memory,
// kThreads splits at a time, and the partial rows are read with many loads in
// flight.  Thread j handles column j.
template <int G>
__device__ __forceinline__ void merge_unit(int64_t u, int nsplit, int64_t pbase, int64_t qrow0,
                                           const float* __restrict__ part_o, const float2* __restrict__ part_ml,
                                           uint32_t* __restrict__ counters, float* __restrict__ out,
                                           float (*red)[G], float* wsm, uint32_t& s_last)
{
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    __threadfence();
    __syncthreads();
    if (tid == 0) s_last = atomicAdd(&counters[u], 1u) == (uint32_t)(nsplit - 1);
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    // Per head: M = max_s m_s; w_s = exp(m_s - M); out = sum_s w_s o_s / sum_s w_s l_s,
    // accumulated in split order.  Weights are staged in shared memory, kThreads
    // splits at a time, and the partial rows are read with many loads in flight.
    for (int h = 0; h < G; ++h) {
        const int64_t base = pbase + h * nsplit;
        float m = -INFINITY;
        for (int sp = tid; sp < nsplit; sp += kThreads) m = fmaxf(m, __ldcg(&part_ml[base + sp]).x);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(kFullMask, m, o));
        __syncthreads();
        if (lane == 0) red[warp][0] = m;
        __syncthreads();
        float M = red[0][0];
#pragma unroll
        for (int w = 1; w < kThreads / 32; ++w) M = fmaxf(M, red[w][0]);
        float lsum = 0.0f, acc = 0.0f;
        for (int s0 = 0; s0 < nsplit; s0 += kThreads) {
            const int cnt = min(kThreads, nsplit - s0);
            __syncthreads();
            if (tid < cnt) {
                const float2 t = __ldcg(&part_ml[base + s0 + tid]);
                const float w = expf(t.x - M);
                wsm[tid] = w;
                lsum += t.y * w;
            }
            __syncthreads();
            const float* po = part_o + (base + s0) * kHeadDim + tid;
            int i = 0;
            for (; i + 16 <= cnt; i += 16) {
                float v[16];
#pragma unroll
                for (int r = 0; r < 16; ++r) v[r] = __ldcg(po + (int64_t)(i + r) * kHeadDim);
#pragma unroll
                for (int r = 0; r < 16; ++r) acc += v[r] * wsm[i + r];
            }
            for (; i < cnt; ++i) acc += __ldcg(po + (int64_t)i * kHeadDim) * wsm[i];
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) lsum += __shfl_xor_sync(kFullMask, lsum, o);
        __syncthreads();
        if (lane == 0) red[warp][0] = lsum;
        __syncthreads();
        float L = 0.0f;
#pragma unroll
        for (int w = 0; w < kThreads / 32; ++w) L += red[w][0];
        out[(qrow0 + h) * kHeadDim + tid] = acc / L;
    }
    if (tid == 0) counters[u] = 0u;
}

// Grid: U * nsplit.  CTA (u, split) takes the unit's selected rows
// [split * rpc, min(k, (split + 1) * rpc)) in chunks of kChunk rows, with two
// chunks in flight: while one chunk is being used, the next one's key and
// value rows are already arriving (bulk copies on that stage's mbarrier).
// The softmax runs online across the chunks (running max, running sum,
// rescaled weighted value sum); the CTA writes one partial per head and the
// last CTA of the unit merges the partials in split order.
// Dynamic smem: 2 stages x (keys + values) x kChunk rows.
template <typename KT, int G>
__global__ __launch_bounds__(kThreads) void attention_kernel(
    const void* __restrict__ q, int q_dtype, const KT* __restrict__ K, const KT* __restrict__ V,
    const int32_t* __restrict__ idx, int64_t Hq, int64_t Hkv, int64_t Ncap, int k, int nsplit, int rpc,
    float* __restrict__ part_o, float2* __restrict__ part_ml, uint32_t* __restrict__ counters,
    uint32_t* __restrict__ err_word, float* __restrict__ out)
{
    constexpr int kChunk = Rows<KT>::kChunk;
    constexpr int kRowBytes = Rows<KT>::kRowBytes;
    constexpr int kStageBytes = 2 * kChunk * kRowBytes;
    constexpr int kRowsPerStep = 32 / G;  // rows whose G logits fill one warp transpose
    extern __shared__ __align__(128) char smem[];
    __shared__ float qs[G][kHeadDim];
    __shared__ float S[G][kChunk];
    __shared__ float red[kThreads / 32][G];
    __shared__ float m_run[G], l_run[G], m_new[G], scale[G];
    __shared__ __align__(8) uint64_t bar[2];
    __shared__ uint32_t s_last;
    __shared__ float wsm[kThreads];  // merge weights

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int64_t u = blockIdx.x / nsplit;
    const int split = blockIdx.x % nsplit;
    const int64_t b = u / Hkv, kvh = u % Hkv;
    const int r_begin = split * rpc;
    const int r_end = min(k, r_begin + rpc);
    const int nchunks = (r_end - r_begin + kChunk - 1) / kChunk;

    const int64_t qrow0 = b * Hq + kvh * G;
    for (int e = tid; e < G * kHeadDim; e += kThreads) {
        const int64_t off = qrow0 * kHeadDim + e;
        qs[e / kHeadDim][e % kHeadDim] = q_dtype == 1 ? bf16_to_f32(static_cast<const uint16_t*>(q)[off])
                                                      : static_cast<const float*>(q)[off];
    }
    if (tid < G) {
        m_run[tid] = -INFINITY;
        l_run[tid] = 0.0f;
    }
    if (tid == 0) {
        mbar_init(&bar[0], 1);
        mbar_init(&bar[1], 1);
        fence_mbarrier_init();
    }
    __syncthreads();
    pdl_wait();  // the selected indices come from the previous kernel on the stream

    // Gather chunk c into stage st: thread i < rows copies one key row and one value row.
    auto issue = [&](int c, int st) {
        const int r0 = r_begin + c * kChunk;
        const int nr = min(kChunk, r_end - r0);
        char* ks = smem + st * kStageBytes;
        char* vs = ks + kChunk * kRowBytes;
        if (tid < nr) {
            // Indices come from the top-k kernel and are < N; clamp anyway so a
            // gather can never leave the unit's cache rows.
            int32_t r = __ldcg(idx + u * k + r0 + tid);
            r = (r >= 0 && r < Ncap) ? r : 0;
            const int64_t row = u * Ncap + r;
            bulk_copy_g2s(ks + tid * kRowBytes, K + row * kHeadDim, kRowBytes, &bar[st]);
            bulk_copy_g2s(vs + tid * kRowBytes, V + row * kHeadDim, kRowBytes, &bar[st]);
        }
        if (tid == 0) mbar_arrive_expect_tx(&bar[st], (uint32_t)nr * 2u * kRowBytes);
    };
    issue(0, 0);
    if (nchunks > 1) issue(1, 1);

    float qreg[G][4];
#pragma unroll
    for (int h = 0; h < G; ++h) {
        const float4 t = *reinterpret_cast<const float4*>(&qs[h][lane * 4]);
        qreg[h][0] = t.x;
        qreg[h][1] = t.y;
        qreg[h][2] = t.z;
        qreg[h][3] = t.w;
    }
    float o[G];
#pragma unroll
    for (int h = 0; h < G; ++h) o[h] = 0.0f;

    for (int c = 0; c < nchunks; ++c) {
        const int st = c & 1;
        const int nrows = min(kChunk, r_end - (r_begin + c * kChunk));
        const char* ks = smem + st * kStageBytes;
        const char* vs = ks + kChunk * kRowBytes;
        if (!mbar_wait_bounded(&bar[st], (uint32_t)((c >> 1) & 1), kMaxPolls)) {
            if (tid == 0) atomicOr(err_word, SOCKET_DEVERR_GATHER_TIMEOUT);
            // let copies in flight land before exiting
            mbar_wait_bounded(&bar[st], (uint32_t)((c >> 1) & 1), kMaxPolls);
            if (c + 1 < nchunks) mbar_wait_bounded(&bar[st ^ 1], (uint32_t)(((c + 1) >> 1) & 1), kMaxPolls);
            return;
        }

        // ---- logits: lanes split d, rows in groups of kRowsPerStep, one warp transpose-reduce per group.
        const int nsteps = (nrows + kRowsPerStep - 1) / kRowsPerStep;
        for (int sp = warp; sp < nsteps; sp += kThreads / 32) {
            float vals[32];
#pragma unroll
            for (int i = 0; i < 32; ++i) vals[i] = 0.0f;
#pragma unroll
            for (int rr = 0; rr < kRowsPerStep; ++rr) {
                const int r = sp * kRowsPerStep + rr;
                if (r < nrows) {
                    const float4 kv = load4(reinterpret_cast<const KT*>(ks + r * kRowBytes), lane * 4);
#pragma unroll
                    for (int h = 0; h < G; ++h)
                        vals[rr * G + h] = qreg[h][0] * kv.x + qreg[h][1] * kv.y + qreg[h][2] * kv.z + qreg[h][3] * kv.w;
                }
            }
            // After the butterfly, lane l holds the full sum of value index l.
#pragma unroll
            for (int sh = 16; sh >= 1; sh >>= 1) {
                const bool upper = (lane & sh) != 0;
#pragma unroll
                for (int i = 0; i < sh; ++i) {
                    const float send = upper ? vals[i] : vals[i + sh];
                    const float keep = upper ? vals[i + sh] : vals[i];
                    vals[i] = keep + __shfl_xor_sync(kFullMask, send, sh);
                }
            }
            const int rr = lane / G, h = lane % G;
            const int r = sp * kRowsPerStep + rr;
            if (rr < kRowsPerStep && r < nrows) S[h][r] = vals[0] * kScale;
        }
        __syncthreads();

        // ---- running max per head.
#pragma unroll
        for (int h = 0; h < G; ++h) {
            float v = tid < nrows ? S[h][tid] : -INFINITY;
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) v = fmaxf(v, __shfl_xor_sync(kFullMask, v, off));
            if (lane == 0) red[warp][h] = v;
        }
        __syncthreads();
        if (tid < G) {
            float mc = red[0][tid];
#pragma unroll
            for (int w = 1; w < kThreads / 32; ++w) mc = fmaxf(mc, red[w][tid]);
            const float mn = fmaxf(m_run[tid], mc);
            m_new[tid] = mn;
            scale[tid] = expf(m_run[tid] - mn);  // 0 on the first chunk (m_run = -inf)
        }
        __syncthreads();
        // ---- weights of this chunk and their sums.
#pragma unroll
        for (int h = 0; h < G; ++h) {
            float p = 0.0f;
            if (tid < nrows) {
                p = expf(S[h][tid] - m_new[h]);
                S[h][tid] = p;
            }
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) p += __shfl_xor_sync(kFullMask, p, off);
            if (lane == 0) red[warp][h] = p;
        }
        __syncthreads();
        // ---- rescale the running state and add this chunk's weighted values (thread j: column j).
        float sc[G];
#pragma unroll
        for (int h = 0; h < G; ++h) {
            sc[h] = scale[h];
            o[h] *= sc[h];
        }
        for (int r = 0; r < nrows; ++r) {
            const float v = load1(reinterpret_cast<const KT*>(vs + r * kRowBytes), tid);
#pragma unroll
            for (int h = 0; h < G; ++h) o[h] += S[h][r] * v;
        }
        if (tid < G) {
            float lc = 0.0f;
#pragma unroll
            for (int w = 0; w < kThreads / 32; ++w) lc += red[w][tid];
            l_run[tid] = l_run[tid] * sc[tid] + lc;
            m_run[tid] = m_new[tid];
        }
        __syncthreads();  // stage st and S are free again
        if (c + 2 < nchunks) issue(c + 2, st);
    }

    const int64_t pbase = u * G * (int64_t)nsplit;
#pragma unroll
    for (int h = 0; h < G; ++h) part_o[((pbase + h * nsplit) + split) * kHeadDim + tid] = o[h];
    if (tid < G) part_ml[pbase + tid * nsplit + split] = make_float2(m_run[tid], l_run[tid]);

    merge_unit<G>(u, nsplit, pbase, qrow0, part_o, part_ml, counters, out, red, wsm, s_last);
}

// ---------------------------------------------------------------------------
// bfloat16 K/V and q, G <= 8: the same chunked online softmax with both
// contractions on the tensor cores (warp-level mma.sync m16n8k16, bf16 in,
// fp32 accumulate):
//   logits^T [64 rows x 8 heads] = K_chunk [64 x 128] * q^T [128 x 8]
//     (warp w: rows 16w..16w+15; A from ldmatrix, B = q held in registers),
//   out^T   [128 x 8 heads]      += V_chunk^T [128 x 64] * P^T [64 x 8]
//     (warp w: columns 32w..32w+31; A from ldmatrix.trans of the value rows,
//      B = the weights, split into a bfloat16 high part and a bfloat16
//      remainder so the weights keep ~16 bits).
// bf16 x bf16 products are exact in fp32, so the logits carry only fp32
// accumulation error, as on the CUDA cores.  Key/value rows are padded to
// 272 bytes in shared memory so the 8 rows an ldmatrix phase reads fall in
// distinct banks.  Heads G..7 of the n = 8 tile are zero padding.
// ---------------------------------------------------------------------------
constexpr int kMmaChunk = 64;
constexpr int kMmaRowStride = 272;
constexpr int kMmaStageBytes = 2 * kMmaChunk * kMmaRowStride;

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t (&r)[4])
{
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t (&r)[4])
{
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}
__device__ __forceinline__ void mma_bf16(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1)
{
    asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
// Two floats -> bfloat16x2 (round to nearest even), first in the low half.
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi)
{
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}
__device__ __forceinline__ float bf16_round(float x) { return __uint_as_float(pack_bf16(x, 0.0f) << 16); }

template <int G>
__global__ __launch_bounds__(kThreads) void attention_mma_kernel(
    const uint16_t* __restrict__ q, const uint16_t* __restrict__ K, const uint16_t* __restrict__ V,
    const int32_t* __restrict__ idx, int64_t Hq, int64_t Hkv, int64_t Ncap, int k, int nsplit, int rpc,
    float* __restrict__ part_o, float2* __restrict__ part_ml, uint32_t* __restrict__ counters,
    uint32_t* __restrict__ err_word, float* __restrict__ out)
{
    static_assert(G <= 8, "the n = 8 tile holds up to 8 heads");
    extern __shared__ __align__(128) char smem[];
    // Logits, then weights; rows padded to 72 floats so the weight fragments
    // (8 heads x 4 row pairs per warp) read from 32 distinct banks.
    __shared__ __align__(8) float S[G][kMmaChunk + 8];
    __shared__ float red[kThreads / 32][G];
    __shared__ float m_run[G], l_run[G], m_new[G], scale[G];
    __shared__ __align__(8) uint64_t bar[2];
    __shared__ uint32_t s_last;
    __shared__ float wsm[kThreads];

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int64_t u = blockIdx.x / nsplit;
    const int split = blockIdx.x % nsplit;
    const int64_t b = u / Hkv, kvh = u % Hkv;
    const int r_begin = split * rpc;
    const int r_end = min(k, r_begin + rpc);
    const int nchunks = (r_end - r_begin + kMmaChunk - 1) / kMmaChunk;
    const int64_t qrow0 = b * Hq + kvh * G;
    const uint32_t sbase = smem_addr(smem);

    // q^T fragments: b0/b1 of k-step ks = q[head lane/4][16 ks + 2 (lane%4) + {0, 1} (+8)].
    uint32_t qb[8][2];
    {
        const int h = lane >> 2, c = (lane & 3) * 2;
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
            uint32_t v0 = 0, v1 = 0;
            if (h < G) {
                const uint16_t* qh = q + (qrow0 + h) * kHeadDim + ks * 16 + c;
                v0 = (uint32_t)qh[0] | ((uint32_t)qh[1] << 16);
                v1 = (uint32_t)qh[8] | ((uint32_t)qh[9] << 16);
            }
            qb[ks][0] = v0;
            qb[ks][1] = v1;
        }
    }
    if (tid < G) {
        m_run[tid] = -INFINITY;
        l_run[tid] = 0.0f;
    }
    if (tid == 0) {
        mbar_init(&bar[0], 1);
        mbar_init(&bar[1], 1);
        fence_mbarrier_init();
    }
    __syncthreads();
    pdl_wait();  // the selected indices come from the previous kernel on the stream

    // Gather chunk c into stage st: thread i < rows copies one key row and one
    // value row; value rows past the chunk's end are zeroed (their weights are 0).
    auto issue = [&](int c, int st) {
        const int r0 = r_begin + c * kMmaChunk;
        const int nr = min(kMmaChunk, r_end - r0);
        char* ks = smem + st * kMmaStageBytes;
        char* vs = ks + kMmaChunk * kMmaRowStride;
        if (tid < nr) {
            // Indices come from the top-k kernel and are < N; clamp anyway so a
            // gather can never leave the unit's cache rows.
            int32_t r = __ldcg(idx + u * k + r0 + tid);
            r = (r >= 0 && r < Ncap) ? r : 0;
            const int64_t row = u * Ncap + r;
            bulk_copy_g2s(ks + tid * kMmaRowStride, K + row * kHeadDim, kHeadDim * 2, &bar[st]);
            bulk_copy_g2s(vs + tid * kMmaRowStride, V + row * kHeadDim, kHeadDim * 2, &bar[st]);
        } else if (tid < kMmaChunk) {
            uint4* z = reinterpret_cast<uint4*>(vs + tid * kMmaRowStride);
#pragma unroll
            for (int i = 0; i < kHeadDim * 2 / 16; ++i) z[i] = make_uint4(0, 0, 0, 0);
        }
        if (tid == 0) mbar_arrive_expect_tx(&bar[st], (uint32_t)nr * 2u * kHeadDim * 2u);
    };
    issue(0, 0);
    if (nchunks > 1) issue(1, 1);
    __syncthreads();  // zeroed value rows visible

    // out^T accumulators: warp w, m-tiles mt = 2w, 2w+1 (columns 16 mt ..), c[mt][i]:
    // i = 0,1: column 16 mt + lane/4, heads 2 (lane%4) + {0,1}; i = 2,3: column + 8.
    float acc[2][4];
#pragma unroll
    for (int t = 0; t < 2; ++t)
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[t][i] = 0.0f;

    for (int c = 0; c < nchunks; ++c) {
        const int st = c & 1;
        const int nrows = min(kMmaChunk, r_end - (r_begin + c * kMmaChunk));
        const uint32_t ks_addr = sbase + st * kMmaStageBytes;
        const uint32_t vs_addr = ks_addr + kMmaChunk * kMmaRowStride;
        if (!mbar_wait_bounded(&bar[st], (uint32_t)((c >> 1) & 1), kMaxPolls)) {
            if (tid == 0) atomicOr(err_word, SOCKET_DEVERR_GATHER_TIMEOUT);
            mbar_wait_bounded(&bar[st], (uint32_t)((c >> 1) & 1), kMaxPolls);
            if (c + 1 < nchunks) mbar_wait_bounded(&bar[st ^ 1], (uint32_t)(((c + 1) >> 1) & 1), kMaxPolls);
            return;
        }
        // ---- logits of rows 16 warp .. +15 for all heads.
        {
            float cl[4] = {0.0f, 0.0f, 0.0f, 0.0f};
            // ldmatrix x4 lane address: matrix q4 = lane/8 -> (rows +8 if q4 odd, cols +8 if q4 >= 2)
            const int q4 = lane >> 3;
            const uint32_t a_row = ks_addr + (uint32_t)((warp * 16 + (q4 & 1) * 8 + (lane & 7)) * kMmaRowStride) +
                                   (uint32_t)((q4 >> 1) * 16);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                uint32_t a[4];
                ldsm_x4(a_row + kk * 32, a);
                mma_bf16(cl, a, qb[kk][0], qb[kk][1]);
            }
            const int r = warp * 16 + (lane >> 2), h = (lane & 3) * 2;
            if (r < nrows) {
                if (h < G) S[h][r] = cl[0] * kScale;
                if (h + 1 < G) S[h + 1][r] = cl[1] * kScale;
            }
            if (r + 8 < nrows) {
                if (h < G) S[h][r + 8] = cl[2] * kScale;
                if (h + 1 < G) S[h + 1][r + 8] = cl[3] * kScale;
            }
        }
        __syncthreads();
        // ---- running max per head.
#pragma unroll
        for (int h = 0; h < G; ++h) {
            float v = tid < nrows ? S[h][tid] : -INFINITY;
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) v = fmaxf(v, __shfl_xor_sync(kFullMask, v, off));
            if (lane == 0) red[warp][h] = v;
        }
        __syncthreads();
        if (tid < G) {
            float mc = red[0][tid];
#pragma unroll
            for (int w = 1; w < kThreads / 32; ++w) mc = fmaxf(mc, red[w][tid]);
            const float mn = fmaxf(m_run[tid], mc);
            m_new[tid] = mn;
            scale[tid] = expf(m_run[tid] - mn);  // 0 on the first chunk (m_run = -inf)
        }
        __syncthreads();
        // ---- weights (0 for rows past the chunk's end) and their sums.
#pragma unroll
        for (int h = 0; h < G; ++h) {
            float p = 0.0f;
            if (tid < kMmaChunk) {
                if (tid < nrows) p = expf(S[h][tid] - m_new[h]);
                S[h][tid] = p;
            }
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) p += __shfl_xor_sync(kFullMask, p, off);
            if (lane == 0) red[warp][h] = p;
        }
        __syncthreads();
        // ---- rescale and add this chunk's weighted values on the tensor cores.
        {
            const int hb = (lane & 3) * 2;
            const float s0 = hb < G ? scale[hb] : 0.0f, s1 = hb + 1 < G ? scale[hb + 1] : 0.0f;
#pragma unroll
            for (int t = 0; t < 2; ++t) {
                acc[t][0] *= s0;
                acc[t][1] *= s1;
                acc[t][2] *= s0;
                acc[t][3] *= s1;
            }
            const int hn = lane >> 2;  // B fragment head (n index)
            const int q4 = lane >> 3;
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
                // P^T fragments: rows 16 kk + 2 (lane%4) + {0,1} (+8), head lane/4.
                const int r0 = kk * 16 + (lane & 3) * 2;
                float p0 = 0.f, p1 = 0.f, p2 = 0.f, p3 = 0.f;
                if (hn < G) {
                    const float2 pa = *reinterpret_cast<const float2*>(&S[hn][r0]);
                    const float2 pb = *reinterpret_cast<const float2*>(&S[hn][r0 + 8]);
                    p0 = pa.x;
                    p1 = pa.y;
                    p2 = pb.x;
                    p3 = pb.y;
                }
                const float h0 = bf16_round(p0), h1 = bf16_round(p1), h2 = bf16_round(p2), h3 = bf16_round(p3);
                const uint32_t bh0 = pack_bf16(h0, h1), bh1 = pack_bf16(h2, h3);
                const uint32_t bl0 = pack_bf16(p0 - h0, p1 - h1), bl1 = pack_bf16(p2 - h2, p3 - h3);
                // V^T tile via ldmatrix.trans: matrix q4 -> value rows 16 kk + 8 (q4 >> 1) + lane%8,
                // columns 16 mt + 8 (q4 & 1).
                const uint32_t v_row =
                    vs_addr + (uint32_t)((kk * 16 + (q4 >> 1) * 8 + (lane & 7)) * kMmaRowStride) + (uint32_t)((q4 & 1) * 16);
#pragma unroll
                for (int t = 0; t < 2; ++t) {
                    const int mt = warp * 2 + t;
                    uint32_t a[4];
                    ldsm_x4_t(v_row + mt * 32, a);
                    mma_bf16(acc[t], a, bh0, bh1);
                    mma_bf16(acc[t], a, bl0, bl1);
                }
            }
        }
        if (tid < G) {
            float lc = 0.0f;
#pragma unroll
            for (int w = 0; w < kThreads / 32; ++w) lc += red[w][tid];
            l_run[tid] = l_run[tid] * scale[tid] + lc;
            m_run[tid] = m_new[tid];
        }
        __syncthreads();  // stage st and S are free again
        if (c + 2 < nchunks) issue(c + 2, st);
    }

    // ---- partials: out^T accumulators -> part_o[(unit, head, split)][column].
    const int64_t pbase = u * G * (int64_t)nsplit;
    {
        const int hb = (lane & 3) * 2;
#pragma unroll
        for (int t = 0; t < 2; ++t) {
            const int j = (warp * 2 + t) * 16 + (lane >> 2);
            if (hb < G) {
                part_o[((pbase + hb * nsplit) + split) * kHeadDim + j] = acc[t][0];
                part_o[((pbase + hb * nsplit) + split) * kHeadDim + j + 8] = acc[t][2];
            }
            if (hb + 1 < G) {
                part_o[((pbase + (hb + 1) * nsplit) + split) * kHeadDim + j] = acc[t][1];
                part_o[((pbase + (hb + 1) * nsplit) + split) * kHeadDim + j + 8] = acc[t][3];
            }
        }
    }
    if (tid < G) part_ml[pbase + tid * nsplit + split] = make_float2(m_run[tid], l_run[tid]);
    merge_unit<G>(u, nsplit, pbase, qrow0, part_o, part_ml, counters, out, red, wsm, s_last);
}

template <int G>
cudaError_t launch_mma(const void* q, const void* K, const void* V, const int32_t* idx, const DecodeShape& s,
                       float* part_o, float2* part_ml, uint32_t* counters, uint32_t* err_word, float* out,
                       cudaStream_t stream)
{
    constexpr int smem = 2 * kMmaStageBytes;
    static_assert(kMmaChunk == Rows<uint16_t>::kChunk, "splits are sized with the bfloat16 chunk");
    const int rpc = attention_rows_per_cta(s.k, s.nsplit, kMmaChunk);
    auto kern = attention_mma_kernel<G>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    e = launch_pdl(kern, dim3((unsigned)(s.U * s.nsplit)), dim3(kThreads), smem, stream,
                   static_cast<const uint16_t*>(q), static_cast<const uint16_t*>(K), static_cast<const uint16_t*>(V),
                   idx, s.Hq, s.Hkv, s.Ncap, s.k, s.nsplit, rpc, part_o, part_ml, counters, err_word, out);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

template <typename KT, int G>
cudaError_t launch_g(const void* q, int q_dtype, const void* K, const void* V, const int32_t* idx,
                     const DecodeShape& s, float* part_o, float2* part_ml, uint32_t* counters, uint32_t* err_word,
                     float* out, cudaStream_t stream)
{
    constexpr int smem = 2 * 2 * Rows<KT>::kChunk * Rows<KT>::kRowBytes;
    const int rpc = attention_rows_per_cta(s.k, s.nsplit, Rows<KT>::kChunk);
    auto kern = attention_kernel<KT, G>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    e = launch_pdl(kern, dim3((unsigned)(s.U * s.nsplit)), dim3(kThreads), smem, stream, q, q_dtype,
                   static_cast<const KT*>(K), static_cast<const KT*>(V), idx, s.Hq, s.Hkv, s.Ncap, s.k, s.nsplit, rpc,
                   part_o, part_ml, counters, err_word, out);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

template <typename KT>
cudaError_t launch_kt(const void* q, int q_dtype, const void* K, const void* V, const int32_t* idx,
                      const DecodeShape& s, float* part_o, float2* part_ml, uint32_t* counters, uint32_t* err_word,
                      float* out, cudaStream_t stream)
{
#define SOCKET_G_CASE(g) \
    case g: return launch_g<KT, g>(q, q_dtype, K, V, idx, s, part_o, part_ml, counters, err_word, out, stream);
    switch (s.G) {
        SOCKET_G_CASE(1) SOCKET_G_CASE(2) SOCKET_G_CASE(3) SOCKET_G_CASE(4)
        SOCKET_G_CASE(5) SOCKET_G_CASE(6) SOCKET_G_CASE(7) SOCKET_G_CASE(8)
        SOCKET_G_CASE(9) SOCKET_G_CASE(10) SOCKET_G_CASE(11) SOCKET_G_CASE(12)
        SOCKET_G_CASE(13) SOCKET_G_CASE(14) SOCKET_G_CASE(15) SOCKET_G_CASE(16)
        default: return cudaErrorInvalidValue;
    }
#undef SOCKET_G_CASE
}

}  // namespace

int attention_chunk_rows(int kv_dtype) { return kv_dtype == 1 ? Rows<uint16_t>::kChunk : Rows<float>::kChunk; }

int attention_rows_per_cta(int k, int nsplit, int chunk)
{
    const int per = (k + nsplit - 1) / nsplit;
    return (per + chunk - 1) / chunk * chunk;
}

int attention_splits(int kv_dtype, int64_t U, int k, int num_sms)
{
    // About three CTAs per SM in one wave, each over whole chunks.
    const int chunk = attention_chunk_rows(kv_dtype);
    const int max_splits = (k + chunk - 1) / chunk;
    int64_t want = (3 * (int64_t)num_sms + U - 1) / U;
    int splits = (int)max64(1, min64(want, max_splits));
    const int rpc = attention_rows_per_cta(k, splits, chunk);
    return (k + rpc - 1) / rpc;
}

cudaError_t launch_attention(const void* q, int q_dtype, const void* K, const void* V, int kv_dtype,
                             const int32_t* idx, const DecodeShape& s, float* part_o, float2* part_ml,
                             uint32_t* counters, uint32_t* err_word, float* out, cudaStream_t stream)
{
    if (kv_dtype == 1 && q_dtype == 1 && s.G <= 8) {
#define SOCKET_MMA_CASE(g) \
    case g: return launch_mma<g>(q, K, V, idx, s, part_o, part_ml, counters, err_word, out, stream);
        switch (s.G) {
            SOCKET_MMA_CASE(1) SOCKET_MMA_CASE(2) SOCKET_MMA_CASE(3) SOCKET_MMA_CASE(4)
            SOCKET_MMA_CASE(5) SOCKET_MMA_CASE(6) SOCKET_MMA_CASE(7) SOCKET_MMA_CASE(8)
            default: break;
        }
#undef SOCKET_MMA_CASE
    }
    if (kv_dtype == 1)
        return launch_kt<uint16_t>(q, q_dtype, K, V, idx, s, part_o, part_ml, counters, err_word, out, stream);
    return launch_kt<float>(q, q_dtype, K, V, idx, s, part_o, part_ml, counters, err_word, out, stream);
}

}  // namespace socket_attn
