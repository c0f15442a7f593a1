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
#include "warp_attn.cuh"

namespace socket_attn {
namespace {

constexpr int kThreads = 128;
constexpr uint32_t kMaxPolls = 1u << 22;
constexpr float kScale = kInvSqrtD;

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
template <int G, int NT>
__device__ __forceinline__ void merge_unit(int64_t u, int nsplit, int64_t pbase, int64_t qrow0,
                                           const float* __restrict__ part_o, const float2* __restrict__ part_ml,
                                           uint32_t* __restrict__ counters, float* __restrict__ out,
                                           float2* __restrict__ ml_out, float (*red)[G], float* wsm,
                                           uint32_t& s_last)
{
    static_assert(kHeadDim % NT == 0 && NT % 32 == 0, "NT threads cover the head dimension evenly");
    constexpr int kCols = kHeadDim / NT;  // output columns per thread: tid, tid + NT, ...
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    if (!cta_ticket(&counters[u], (uint32_t)(nsplit - 1), s_last)) return;
    // Per head: M = max_s m_s; w_s = exp(m_s - M); out = sum_s w_s o_s / sum_s w_s l_s,
    // accumulated in split order.  Weights are staged in shared memory, NT
    // splits at a time, and the partial rows are read with many loads in flight.
    for (int h = 0; h < G; ++h) {
        const int64_t base = pbase + h * nsplit;
        float m = -INFINITY;
        for (int sp = tid; sp < nsplit; sp += NT) m = fmaxf(m, __ldcg(&part_ml[base + sp]).x);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(kFullMask, m, o));
        __syncthreads();
        if (lane == 0) red[warp][0] = m;
        __syncthreads();
        float M = red[0][0];
#pragma unroll
        for (int w = 1; w < NT / 32; ++w) M = fmaxf(M, red[w][0]);
        float lsum = 0.0f, acc[kCols];
#pragma unroll
        for (int j = 0; j < kCols; ++j) acc[j] = 0.0f;
        for (int s0 = 0; s0 < nsplit; s0 += NT) {
            const int cnt = min(NT, nsplit - s0);
            __syncthreads();
            if (tid < cnt) {
                const float2 t = __ldcg(&part_ml[base + s0 + tid]);
                const float w = t.x == -INFINITY ? 0.0f : expf(t.x - M);  // empty splits weigh nothing
                wsm[tid] = w;
                lsum += t.y * w;
            }
            __syncthreads();
#pragma unroll
            for (int j = 0; j < kCols; ++j) {
                const float* po = part_o + (base + s0) * kHeadDim + tid + j * NT;
                int i = 0;
                for (; i + 16 <= cnt; i += 16) {
                    float v[16];
#pragma unroll
                    for (int r = 0; r < 16; ++r) v[r] = __ldcg(po + (int64_t)(i + r) * kHeadDim);
#pragma unroll
                    for (int r = 0; r < 16; ++r) acc[j] += v[r] * wsm[i + r];
                }
                for (; i < cnt; ++i) acc[j] += __ldcg(po + (int64_t)i * kHeadDim) * wsm[i];
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) lsum += __shfl_xor_sync(kFullMask, lsum, o);
        __syncthreads();
        if (lane == 0) red[warp][0] = lsum;
        __syncthreads();
        float L = 0.0f;
#pragma unroll
        for (int w = 0; w < NT / 32; ++w) L += red[w][0];
        // No rows at all (an empty share of a sharded selection): zero output.
#pragma unroll
        for (int j = 0; j < kCols; ++j) out[(qrow0 + h) * kHeadDim + tid + j * NT] = L > 0.0f ? acc[j] / L : 0.0f;
        if (ml_out && tid == 0) ml_out[qrow0 + h] = make_float2(M, L);
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
    const int32_t* __restrict__ idx, const int32_t* __restrict__ counts, int share, int64_t Ncap, int k,
    int nsplit, int rpc, float* __restrict__ part_o, float2* __restrict__ part_ml, uint32_t* __restrict__ counters,
    uint32_t* __restrict__ err_word, float* __restrict__ out, float2* __restrict__ ml_out, uint32_t max_polls)
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
    const int64_t ukv = u / share;  // the unit's key/value rows
    const int r_begin = split * rpc;

    const int64_t qrow0 = u * G;  // the unit's query rows of [B][Hq]
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
    // Rows of the unit: k, or its own count when the selection is a share of a
    // sharded one (counts, clamped to [0, k]).
    const int rows = counts ? max(0, min(k, __ldcg(counts + u))) : k;
    const int r_end = min(rows, r_begin + rpc);
    const int nchunks = r_end > r_begin ? (r_end - r_begin + kChunk - 1) / kChunk : 0;

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
            const int64_t row = ukv * Ncap + r;
            bulk_copy_g2s(ks + tid * kRowBytes, K + row * kHeadDim, kRowBytes, &bar[st]);
            bulk_copy_g2s(vs + tid * kRowBytes, V + row * kHeadDim, kRowBytes, &bar[st]);
        }
        if (tid == 0) mbar_arrive_expect_tx(&bar[st], (uint32_t)nr * 2u * kRowBytes);
    };
    if (nchunks > 0) issue(0, 0);
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
        if (!mbar_wait_bounded(&bar[st], (uint32_t)((c >> 1) & 1), max_polls)) {
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

    merge_unit<G, kThreads>(u, nsplit, pbase, qrow0, part_o, part_ml, counters, out, ml_out, red, wsm, s_last);
}

// ---------------------------------------------------------------------------
// bfloat16 K/V and q, G <= 8: flash-decode split-K with every warp on its own
// 16-key chunks and both contractions on the tensor cores (WarpAttn, in
// warp_attn.cuh).  Each warp gathers its chunks itself (16-byte cp.async
// copies, each lane's completion arriving on the stage's mbarrier) on its own
// two-stage ring, so the chunk loop has no CTA-wide barrier and every wait is
// a bounded mbarrier wait.  The two warps
// of a CTA then merge in shared memory and the last CTA of the unit merges
// the CTAs' partials.
// ---------------------------------------------------------------------------
constexpr int kWStages = 2;
constexpr int kWWarps = 2;
constexpr int kWThreads = 32 * kWWarps;
constexpr int kWSmemBytes = kWWarps * kWStages * kWStageBytes;
constexpr int kWCtasPerSm = 6;

// The tensor-core kernel takes bfloat16 q, K, V and groups of up to 8 heads.
bool warp_path(int kv_dtype, int q_dtype, int G) { return kv_dtype == 1 && q_dtype == 1 && G <= 8; }

// The unit's last CTA merges the splits' partials: head h is merged by warp
// h % kWWarps with no CTA barrier.  Splits are taken TILE at a time (16, or 32
// when a unit has more than 16 splits: fewer round trips, more registers),
// their (m, l) pairs (split s in lane s) and 16-byte loads of their rows issued
// together; the weights w_s = exp(m_s - M) reach the other lanes by shuffle,
// and each lane accumulates four output columns in split order, rescaling
// when a later tile raises the running max M:
// out = sum_s w_s o_s / sum_s w_s l_s with M = max_s m_s.
template <int G, int TILE>
__device__ __forceinline__ void merge_unit_warps(int64_t u, int nsplit, int64_t pbase, int64_t qrow0,
                                                 const float* __restrict__ part_o, const float2* __restrict__ part_ml,
                                                 uint32_t* __restrict__ counters, float* __restrict__ out,
                                                 float2* __restrict__ ml_out, uint32_t& s_last)
{
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    if (!cta_ticket(&counters[u], (uint32_t)(nsplit - 1), s_last)) return;
    constexpr int kTile = TILE;  // splits whose rows are loaded at once
    for (int h = warp; h < G; h += kWWarps) {
        const int64_t base = pbase + h * nsplit;
        float M = -INFINITY, lsum = 0.0f;  // lsum: this lane's splits, at the running max M
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int s0 = 0; s0 < nsplit; s0 += kTile) {
            // The tile's (m, l) pairs (split s0 + i in lane i) and rows, all in flight at once.
            const int cnt = min(kTile, nsplit - s0);
            const float2 t = lane < cnt ? __ldcg(&part_ml[base + s0 + lane]) : make_float2(-INFINITY, 0.0f);
            const float4* po = reinterpret_cast<const float4*>(part_o + (base + s0) * kHeadDim) + lane;
            float4 v[kTile];
#pragma unroll
            for (int r = 0; r < kTile; ++r)
                v[r] = r < cnt ? __ldcg(po + (int64_t)r * (kHeadDim / 4)) : make_float4(0.f, 0.f, 0.f, 0.f);
            float mt = t.x;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) mt = fmaxf(mt, __shfl_xor_sync(kFullMask, mt, o));
            const float Mn = fmaxf(M, mt);
            if (Mn != -INFINITY) {
                const float sc = M == -INFINITY ? 0.0f : expf(M - Mn);  // rescale the earlier tiles
                acc.x *= sc;
                acc.y *= sc;
                acc.z *= sc;
                acc.w *= sc;
                lsum *= sc;
                const float w = t.x == -INFINITY ? 0.0f : expf(t.x - Mn);
                lsum += t.y * w;
#pragma unroll
                for (int r = 0; r < kTile; ++r) {
                    const float wr = __shfl_sync(kFullMask, w, r);
                    acc.x += wr * v[r].x;
                    acc.y += wr * v[r].y;
                    acc.z += wr * v[r].z;
                    acc.w += wr * v[r].w;
                }
                M = Mn;
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) lsum += __shfl_xor_sync(kFullMask, lsum, o);
        // No rows at all (an empty share of a sharded selection): zero output.
        const float inv = lsum > 0.0f ? 1.0f / lsum : 0.0f;
        reinterpret_cast<float4*>(out + (qrow0 + h) * kHeadDim)[lane] =
            make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
        if (ml_out && lane == 0) ml_out[qrow0 + h] = make_float2(M, lsum);
    }
    if (tid == 0) counters[u] = 0u;
}

template <int G, int TILE>
__global__ __launch_bounds__(kWThreads) void attention_warp_kernel(
    const uint16_t* __restrict__ q, const uint16_t* __restrict__ K, const uint16_t* __restrict__ V,
    const int32_t* __restrict__ idx, const int32_t* __restrict__ counts, int share, int64_t Ncap, int k,
    int nsplit, int rpc, float* __restrict__ part_o, float2* __restrict__ part_ml, uint32_t* __restrict__ counters,
    uint32_t* __restrict__ err_word, float* __restrict__ out, float2* __restrict__ ml_out, uint32_t max_polls)
{
    extern __shared__ __align__(128) char smem[];
    __shared__ __align__(8) uint64_t bar[kWWarps][kWStages];
    __shared__ float xm[kWWarps][8], xl[kWWarps][8];
    __shared__ uint32_t s_last;

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int64_t u = blockIdx.x / nsplit;
    const int split = blockIdx.x % nsplit;
    const int64_t ukv = u / share;  // the unit's key/value rows
    const int r_begin = split * rpc;
    const int64_t qrow0 = u * G;  // the unit's query rows of [B][Hq]
    char* wsm_base = smem + warp * kWStages * kWStageBytes;
    const uint32_t wbase = smem_addr(wsm_base);

    WarpAttn<G> at;
    at.init(q, qrow0);
    if (tid == 0) {
        // One arrival per lane and chunk (issue_lsu_mbar).
        for (int w = 0; w < kWWarps; ++w)
            for (int st = 0; st < kWStages; ++st) mbar_init(&bar[w][st], 32);
        fence_mbarrier_init();
    }
    __syncthreads();
    // The grid fits in one wave, so the next decode's first kernel may be
    // placed now; it waits for this grid to finish before it reads anything.
    pdl_launch_dependents();
    pdl_wait();  // the selected indices come from the previous kernel on the stream
    // Rows of the unit: k, or its own count when the selection is a share of a
    // sharded one (counts, clamped to [0, k]).
    const int rows = counts ? max(0, min(k, __ldcg(counts + u))) : k;
    const int r_end = min(rows, r_begin + rpc);
    const int nch = r_end > r_begin ? (r_end - r_begin + kWChunk - 1) / kWChunk : 0;  // chunks of this CTA
    const int cw = nch > warp ? (nch - warp + kWWarps - 1) / kWWarps : 0;               // chunks of this warp

    // Row index of this lane's row (lane % 16) of chunk j, or -1 past the end.
    auto row_index = [&](int j) -> int32_t {
        const int r0 = r_begin + (warp + kWWarps * j) * kWChunk;
        const int i = lane & 15;
        return (j < cw && i < r_end - r0) ? __ldcg(idx + u * k + r0 + i) : -1;
    };
    // Gather this warp's chunk j into stage st.  Indices come from the top-k
    // kernel and are < N; they are clamped anyway so a gather can never leave
    // the unit's cache rows.
    auto issue = [&](int j, int st, int32_t r) {
        const int r0 = r_begin + (warp + kWWarps * j) * kWChunk;
        const int nr = min(kWChunk, r_end - r0);
        r = (r >= 0 && r < Ncap) ? r : 0;
        at.issue_lsu_mbar(wsm_base + st * kWStageBytes, K, V, ukv * Ncap + r, nr, &bar[warp][st]);
    };
    if (cw > 0) issue(0, 0, row_index(0));
    if (cw > 1) issue(1, 1, row_index(1));
    __syncwarp();  // zeroed value rows visible to the warp

    bool ok = true;
    for (int j = 0; j < cw; ++j) {
        const int st = j & 1;
        const int32_t next_row = row_index(j + 2);  // in flight while chunk j is used
        const bool got = mbar_wait_bounded(&bar[warp][st], (uint32_t)((j >> 1) & 1), max_polls);
        if (__any_sync(kFullMask, !got)) {
            if (lane == 0) atomicOr(err_word, SOCKET_DEVERR_GATHER_TIMEOUT);
            mbar_wait_bounded(&bar[warp][st], (uint32_t)((j >> 1) & 1), kMaxPolls);
            if (j + 1 < cw) mbar_wait_bounded(&bar[warp][st ^ 1], (uint32_t)(((j + 1) >> 1) & 1), kMaxPolls);
            ok = false;
            break;
        }
        const int nr = min(kWChunk, r_end - (r_begin + (warp + kWWarps * j) * kWChunk));
        at.consume(wbase + st * kWStageBytes, nr);
        if (j + 2 < cw) {
            issue(j + 2, st, next_row);
            __syncwarp();
        }
    }
    if (!ok) at.reset();

    // ---- merge the two warps: warp 1 leaves (m, l, o^T) in its own stage memory.
    float* xo = reinterpret_cast<float*>(smem + kWStages * kWStageBytes);  // warp 1's area, [8 heads][128]
    if (warp == 1) at.store(xo, xm[1], xl[1]);
    else if ((lane & 3) == 0 && (lane >> 2) < G) {
        xm[0][lane >> 2] = at.m_run;
        xl[0][lane >> 2] = at.l_run;
    }
    __syncthreads();
    const int64_t pbase = u * G * (int64_t)nsplit;
    if (warp == 0) {
        const int t2 = (lane & 3) * 2;
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            const int h = t2 + hh;
            if (h < G) {
                const float M = fmaxf(xm[0][h], xm[1][h]);
                const float w0 = xm[0][h] == -INFINITY ? 0.0f : expf(xm[0][h] - M);
                const float w1 = xm[1][h] == -INFINITY ? 0.0f : expf(xm[1][h] - M);
                float* po = part_o + ((pbase + h * nsplit) + split) * kHeadDim;
#pragma unroll
                for (int mt = 0; mt < 8; ++mt) {
                    const int ch = mt * 16 + (lane >> 2);
                    po[ch] = w0 * at.acc[mt][hh] + w1 * xo[h * kHeadDim + ch];
                    po[ch + 8] = w0 * at.acc[mt][2 + hh] + w1 * xo[h * kHeadDim + ch + 8];
                }
                if ((lane >> 2) == 0) part_ml[pbase + h * nsplit + split] = make_float2(M, w0 * xl[0][h] + w1 * xl[1][h]);
            }
        }
    }
    merge_unit_warps<G, TILE>(u, nsplit, pbase, qrow0, part_o, part_ml, counters, out, ml_out, s_last);
}

template <int G>
cudaError_t launch_warp(const void* q, const void* K, const void* V, const int32_t* idx, const int32_t* counts,
                        const DecodeShape& s, float* part_o, float2* part_ml, uint32_t* counters, uint32_t* err_word,
                        float* out, float2* ml_out, cudaStream_t stream)
{
    const int rpc = attention_rows_per_cta(s.k, s.nsplit, kWChunk);
    // The wide merge tile only where a unit has more than 16 splits: its
    // registers would otherwise cost every shape (the kernel's CTAs share SMs
    // with the top-k grid while they wait for it).
    auto kern = s.nsplit > 16 ? attention_warp_kernel<G, 32> : attention_warp_kernel<G, 16>;
    cudaError_t e = set_smem_limit_once((const void*)kern, kWSmemBytes);
    if (e != cudaSuccess) return e;
    e = launch_pdl(kern, dim3((unsigned)(s.U * s.nsplit)), dim3(kWThreads), kWSmemBytes, stream,
                   static_cast<const uint16_t*>(q), static_cast<const uint16_t*>(K), static_cast<const uint16_t*>(V),
                   idx, counts, s.share, s.Ncap, s.k, s.nsplit, rpc, part_o, part_ml, counters, err_word, out,
                   ml_out, wait_poll_limit());
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

template <typename KT, int G>
cudaError_t launch_g(const void* q, int q_dtype, const void* K, const void* V, const int32_t* idx,
                     const int32_t* counts, const DecodeShape& s, float* part_o, float2* part_ml, uint32_t* counters,
                     uint32_t* err_word, float* out, float2* ml_out, cudaStream_t stream)
{
    constexpr int smem = 2 * 2 * Rows<KT>::kChunk * Rows<KT>::kRowBytes;
    const int rpc = attention_rows_per_cta(s.k, s.nsplit, Rows<KT>::kChunk);
    auto kern = attention_kernel<KT, G>;
    cudaError_t e = set_smem_limit_once((const void*)kern, smem);
    if (e != cudaSuccess) return e;
    e = launch_pdl(kern, dim3((unsigned)(s.U * s.nsplit)), dim3(kThreads), smem, stream, q, q_dtype,
                   static_cast<const KT*>(K), static_cast<const KT*>(V), idx, counts, s.share, s.Ncap, s.k, s.nsplit,
                   rpc, part_o, part_ml, counters, err_word, out, ml_out, wait_poll_limit());
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

template <typename KT>
cudaError_t launch_kt(const void* q, int q_dtype, const void* K, const void* V, const int32_t* idx,
                      const int32_t* counts, const DecodeShape& s, float* part_o, float2* part_ml, uint32_t* counters,
                      uint32_t* err_word, float* out, float2* ml_out, cudaStream_t stream)
{
#define SOCKET_G_CASE(g) \
    case g:              \
        return launch_g<KT, g>(q, q_dtype, K, V, idx, counts, s, part_o, part_ml, counters, err_word, out, ml_out, stream);
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

int attention_splits(int kv_dtype, int q_dtype, int G, int64_t U, int k, int num_sms)
{
    // One wave: about kWCtasPerSm two-warp CTAs per SM on the tensor-core path,
    // three four-warp CTAs per SM otherwise, each over whole chunks.
    const bool wp = warp_path(kv_dtype, q_dtype, G);
    const int chunk = wp ? kWChunk : attention_chunk_rows(kv_dtype);
    const int per_sm = wp ? kWCtasPerSm : 3;
    const int max_splits = (k + chunk - 1) / chunk;
    // At most kMaxSplits per unit: the unit's last CTA merges every split's
    // partial, so with few units (a million-token sequence: 8) more splits
    // cost more in the merge than they gain in gather parallelism.
    constexpr int64_t kMaxSplits = 48;
    const int64_t want = min64(kMaxSplits, max64(1, (int64_t)per_sm * num_sms / U));
    const int splits = (int)max64(1, min64(want, max_splits));
    const int rpc = attention_rows_per_cta(k, splits, chunk);
    return (k + rpc - 1) / rpc;
}

cudaError_t launch_attention(const void* q, int q_dtype, const void* K, const void* V, int kv_dtype,
                             const int32_t* idx, const int32_t* counts, const DecodeShape& s, float* part_o,
                             float2* part_ml, uint32_t* counters, uint32_t* err_word, float* out, float2* ml_out,
                             cudaStream_t stream)
{
    if (warp_path(kv_dtype, q_dtype, s.G)) {
#define SOCKET_MMA_CASE(g) \
    case g: return launch_warp<g>(q, K, V, idx, counts, s, part_o, part_ml, counters, err_word, out, ml_out, stream);
        switch (s.G) {
            SOCKET_MMA_CASE(1) SOCKET_MMA_CASE(2) SOCKET_MMA_CASE(3) SOCKET_MMA_CASE(4)
            SOCKET_MMA_CASE(5) SOCKET_MMA_CASE(6) SOCKET_MMA_CASE(7) SOCKET_MMA_CASE(8)
            default: break;
        }
#undef SOCKET_MMA_CASE
    }
    if (kv_dtype == 1)
        return launch_kt<uint16_t>(q, q_dtype, K, V, idx, counts, s, part_o, part_ml, counters, err_word, out, ml_out,
                                   stream);
    return launch_kt<float>(q, q_dtype, K, V, idx, counts, s, part_o, part_ml, counters, err_word, out, ml_out, stream);
}

}  // namespace socket_attn
