// Exact softmax attention over the selected keys (split-K flash decode).
//
// Method: "Resumen Técnico: SOCKET ..." (gist.science/es/paper/2602.06283),
// "Mecanismo Central: LSH Suave" step 4 "Selección": exact attention is
// computed over the selected subset; "SOCKET: SOft Collision Kernel EsTimator
// for Sparse Attention" (gist.science/de/paper/2602.06283), "Auswahl".  The
// pages run this step with a "Flash Decode" backend ("Contribuciones Clave"
// 2 / "Hauptbeiträge"); here it is a hand-written split-K kernel.
//
// Each CTA takes one chunk (64 rows) of a unit's selected rows: it gathers the
// chunk's key and value rows into shared memory with bulk asynchronous copies
// (one 256-byte row per copy, completion counted on an mbarrier), computes the
// logits of all query heads of the unit (scale 1/sqrt(d)), the chunk's
// running max and exp-sum, and the unnormalised weighted value sum.  The
// last CTA of a unit to finish (an atomic ticket, no waiting) merges the
// chunks in chunk order with the usual log-sum-exp rescaling and writes the
// normalised float32 output, so the merge is deterministic.
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

// Grid: U * nsplit.  Block: kThreads.  Dynamic smem: 2 * kChunk * kRowBytes.
template <typename KT, int G>
__global__ __launch_bounds__(kThreads) void attention_kernel(
    const void* __restrict__ q, int q_dtype, const KT* __restrict__ K, const KT* __restrict__ V,
    const int32_t* __restrict__ idx, int64_t Hq, int64_t Hkv, int64_t Ncap, int k, int nsplit,
    float* __restrict__ part_o, float2* __restrict__ part_ml, uint32_t* __restrict__ counters,
    uint32_t* __restrict__ err_word, float* __restrict__ out)
{
    constexpr int kChunk = Rows<KT>::kChunk;
    constexpr int kRowBytes = Rows<KT>::kRowBytes;
    constexpr int kRowsPerStep = 32 / G;  // rows whose G logits fill one warp transpose
    extern __shared__ __align__(128) char smem[];
    char* ks = smem;
    char* vs = smem + kChunk * kRowBytes;
    __shared__ float qs[G][kHeadDim];
    __shared__ float S[G][kChunk];
    __shared__ float2 ml[G];
    __shared__ float mhead[G];
    __shared__ float red[kThreads / 32][G];
    __shared__ int32_t rows[kChunk];
    __shared__ __align__(8) uint64_t bar;
    __shared__ uint32_t s_last;
    __shared__ float wsm[kThreads];  // merge weights

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int64_t u = blockIdx.x / nsplit;
    const int split = blockIdx.x % nsplit;
    const int64_t b = u / Hkv, kvh = u % Hkv;
    const int r0 = split * kChunk;
    const int nrows = min(kChunk, k - r0);

    const int64_t qrow0 = b * Hq + kvh * G;
    for (int e = tid; e < G * kHeadDim; e += kThreads) {
        const int64_t off = qrow0 * kHeadDim + e;
        qs[e / kHeadDim][e % kHeadDim] = q_dtype == 1 ? bf16_to_f32(static_cast<const uint16_t*>(q)[off])
                                                      : static_cast<const float*>(q)[off];
    }
    if (tid == 0) {
        mbar_init(&bar, 1);
        fence_mbarrier_init();
    }
    pdl_wait();  // the selected indices come from the previous kernel on the stream
    if (tid < nrows) {
        // Indices come from the top-k kernel and are < N; clamp anyway so a
        // gather can never leave the unit's cache rows.
        const int32_t r = __ldcg(idx + u * k + r0 + tid);
        rows[tid] = (r >= 0 && r < Ncap) ? r : 0;
    }
    __syncthreads();
    if (tid == 0) mbar_arrive_expect_tx(&bar, (uint32_t)nrows * 2u * kRowBytes);
    __syncthreads();
    if (tid < nrows) {
        const int64_t row = u * Ncap + rows[tid];
        bulk_copy_g2s(ks + tid * kRowBytes, K + row * kHeadDim, kRowBytes, &bar);
        bulk_copy_g2s(vs + tid * kRowBytes, V + row * kHeadDim, kRowBytes, &bar);
    }
    if (!mbar_wait_bounded(&bar, 0, kMaxPolls)) {
        if (tid == 0) atomicOr(err_word, SOCKET_DEVERR_GATHER_TIMEOUT);
        mbar_wait_bounded(&bar, 0, kMaxPolls);  // let copies in flight land before exiting
        return;
    }

    // ---- logits: lanes split d, rows in groups of kRowsPerStep, one warp transpose-reduce per group.
    float qreg[G][4];
#pragma unroll
    for (int h = 0; h < G; ++h) {
        const float4 t = *reinterpret_cast<const float4*>(&qs[h][lane * 4]);
        qreg[h][0] = t.x;
        qreg[h][1] = t.y;
        qreg[h][2] = t.z;
        qreg[h][3] = t.w;
    }
    const int nsteps = (nrows + kRowsPerStep - 1) / kRowsPerStep;
    for (int st = warp; st < nsteps; st += kThreads / 32) {
        float vals[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) vals[i] = 0.0f;
#pragma unroll
        for (int rr = 0; rr < kRowsPerStep; ++rr) {
            const int r = st * kRowsPerStep + rr;
            if (r < nrows) {
                const float4 kv = load4(reinterpret_cast<const KT*>(ks + r * kRowBytes), lane * 4);
#pragma unroll
                for (int h = 0; h < G; ++h)
                    vals[rr * G + h] = qreg[h][0] * kv.x + qreg[h][1] * kv.y + qreg[h][2] * kv.z + qreg[h][3] * kv.w;
            }
        }
        // After the butterfly, lane l holds the full sum of value index l.
#pragma unroll
        for (int s = 16; s >= 1; s >>= 1) {
            const bool upper = (lane & s) != 0;
#pragma unroll
            for (int i = 0; i < s; ++i) {
                const float send = upper ? vals[i] : vals[i + s];
                const float keep = upper ? vals[i + s] : vals[i];
                vals[i] = keep + __shfl_xor_sync(kFullMask, send, s);
            }
        }
        const int rr = lane / G, h = lane % G;
        const int r = st * kRowsPerStep + rr;
        if (rr < kRowsPerStep && r < nrows) S[h][r] = vals[0] * kScale;
    }
    __syncthreads();

    // ---- chunk max and exp-sum per head.
#pragma unroll
    for (int h = 0; h < G; ++h) {
        float v = tid < nrows ? S[h][tid] : -INFINITY;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(kFullMask, v, o));
        if (lane == 0) red[warp][h] = v;
    }
    __syncthreads();
    if (tid < G) {
        float m = red[0][tid];
#pragma unroll
        for (int w = 1; w < kThreads / 32; ++w) m = fmaxf(m, red[w][tid]);
        mhead[tid] = m;
    }
    __syncthreads();
#pragma unroll
    for (int h = 0; h < G; ++h) {
        float p = 0.0f;
        if (tid < nrows) {
            p = expf(S[h][tid] - mhead[h]);
            S[h][tid] = p;
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) p += __shfl_xor_sync(kFullMask, p, o);
        if (lane == 0) red[warp][h] = p;
    }
    __syncthreads();
    if (tid < G) {
        float l = 0.0f;
#pragma unroll
        for (int w = 0; w < kThreads / 32; ++w) l += red[w][tid];
        ml[tid] = make_float2(mhead[tid], l);
    }

    // ---- weighted value sum: thread j owns column j.
    float o[G];
#pragma unroll
    for (int h = 0; h < G; ++h) o[h] = 0.0f;
    for (int r = 0; r < nrows; ++r) {
        const float v = load1(reinterpret_cast<const KT*>(vs + r * kRowBytes), tid);
#pragma unroll
        for (int h = 0; h < G; ++h) o[h] += S[h][r] * v;
    }
    __syncthreads();

    const int64_t pbase = u * G * (int64_t)nsplit;
#pragma unroll
    for (int h = 0; h < G; ++h) part_o[((pbase + h * nsplit) + split) * kHeadDim + tid] = o[h];
    if (tid < G) part_ml[pbase + tid * nsplit + split] = ml[tid];

    // ---- the last CTA of the unit merges the chunks in order.
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

template <typename KT, int G>
cudaError_t launch_g(const void* q, int q_dtype, const void* K, const void* V, const int32_t* idx,
                     const DecodeShape& s, float* part_o, float2* part_ml, uint32_t* counters, uint32_t* err_word,
                     float* out, cudaStream_t stream)
{
    constexpr int smem = 2 * Rows<KT>::kChunk * Rows<KT>::kRowBytes;
    auto kern = attention_kernel<KT, G>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    e = launch_pdl(kern, dim3((unsigned)(s.U * s.nsplit)), dim3(kThreads), smem, stream, q, q_dtype,
                   static_cast<const KT*>(K), static_cast<const KT*>(V), idx, s.Hq, s.Hkv, s.Ncap, s.k, s.nsplit,
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

cudaError_t launch_attention(const void* q, int q_dtype, const void* K, const void* V, int kv_dtype,
                             const int32_t* idx, const DecodeShape& s, float* part_o, float2* part_ml,
                             uint32_t* counters, uint32_t* err_word, float* out, cudaStream_t stream)
{
    if (kv_dtype == 1)
        return launch_kt<uint16_t>(q, q_dtype, K, V, idx, s, part_o, part_ml, counters, err_word, out, stream);
    return launch_kt<float>(q, q_dtype, K, V, idx, s, part_o, part_ml, counters, err_word, out, stream);
}

}  // namespace socket_attn
