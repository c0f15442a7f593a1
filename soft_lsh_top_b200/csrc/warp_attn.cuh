// One warp's flash-decode state over 16-key chunks of a unit's selected keys:
// bfloat16 q, K and V, at most 8 query heads, both contractions on the
// tensor cores (warp-level mma.sync m16n8k16, bf16 in, fp32 accumulate):
//   logits^T [16 heads x 16 keys] = q [16 x 128] * K_chunk^T [128 x 16]
//     (A = q, held in registers or read from shared memory, heads G..15
//      zero; B from ldmatrix of the key rows, which are B's columns);
//   out^T   [128 x 16 heads]     += V_chunk^T [128 x 16] * P^T [16 x 8]
//     (A from ldmatrix.trans of the value rows; B = the weights).
// The logits' accumulator fragment (head lane/4, keys 2 (lane%4) + {0,1}
// and + 8) is exactly the B fragment the second product needs, so weights
// never leave registers; the online softmax of a head reduces over one lane
// quad.  Weights enter the second product as a bfloat16 high part plus a
// bfloat16 remainder (~16 bits).  bf16 x bf16 products are exact in fp32, so
// the logits carry only fp32 accumulation error.
//
// Exact attention over the selected keys is step 4 of the method ("Resumen
// Técnico: SOCKET ...", "Mecanismo Central: LSH Suave", "Selección";
// "SOCKET: SOft Collision Kernel EsTimator for Sparse Attention", "Auswahl").
//
// A chunk's rows are gathered by the warp itself into one stage of shared
// memory, into rows padded to 272 bytes so an ldmatrix phase's 8 rows hit
// distinct banks: 16-byte cp.async copies, completion counted on the stage's
// mbarrier (issue_lsu_mbar) or in a commit group (issue_lsu), or one bulk
// copy per 256-byte key or value row (issue).  The cp.async copies cost the
// copy engine nothing per row, which pays where an SM gathers thousands of
// rows.
#pragma once

#include "common.cuh"

namespace socket_attn {

constexpr int kWChunk = 16;                               // keys per warp chunk
constexpr int kWRowStride = 272;                          // padded row bytes in shared memory
constexpr int kWStageBytes = 2 * kWChunk * kWRowStride;   // keys + values of one chunk
constexpr float kInvSqrtD = 0.088388347648318440550f;    // 1 / sqrt(128)

// Two floats -> bfloat16x2 (round to nearest even), first in the low half.
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi)
{
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}
__device__ __forceinline__ float bf16_round(float x) { return __uint_as_float(pack_bf16(x, 0.0f) << 16); }

// q as the mma A operand, for k-step kk (channels 16 kk ..) and lane: row
// h = lane/4 (zero for h >= G), channels 16 kk + 2 (lane%4) + {0,1} (.x) and
// + 8 (.y), two bfloat16 each.
template <int G>
__device__ __forceinline__ uint2 q_fragment(const uint16_t* __restrict__ q, int64_t qrow0, int kk, int lane)
{
    const int h = lane >> 2, c = (lane & 3) * 2;
    uint2 f = make_uint2(0u, 0u);
    if (h < G) {
        const uint16_t* qh = q + (qrow0 + h) * kHeadDim + kk * 16 + c;
        f.x = (uint32_t)qh[0] | ((uint32_t)qh[1] << 16);
        f.y = (uint32_t)qh[8] | ((uint32_t)qh[9] << 16);
    }
    return f;
}

// QS: the q fragments are read from shared memory (qfrag[kk * 32 + lane], as
// q_fragment gives them) at every chunk instead of being held in registers.
template <int G, bool QS = false>
struct WarpAttn {
    static_assert(G >= 1 && G <= 8, "heads are the M rows 0..7 of the 16-row tile");
    uint32_t qa[QS ? 1 : 8][2];  // q fragments in registers (QS false)
    const uint2* qfrag;          // q fragments in shared memory (QS true)
    // out^T accumulators: m-tile mt = channels 16 mt ..; [0], [1]: channel
    // 16 mt + lane/4, heads 2 (lane%4) + {0,1}; [2], [3]: channel + 8.
    float acc[8][4];
    float m_run, l_run;  // of head lane/4: running max logit, running sum of weights

    // The unit's query rows qrow0 .. qrow0 + G - 1 of [B][Hq][128].
    __device__ __forceinline__ void init(const uint16_t* __restrict__ q, int64_t qrow0)
    {
        static_assert(!QS, "registers hold q");
        const int lane = threadIdx.x & 31;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
            const uint2 f = q_fragment<G>(q, qrow0, kk, lane);
            qa[kk][0] = f.x;
            qa[kk][1] = f.y;
        }
        qfrag = nullptr;
        reset();
    }
    // q fragments staged in shared memory by the caller.
    __device__ __forceinline__ void init(const uint2* qf)
    {
        static_assert(QS, "shared memory holds q");
        qfrag = qf;
        reset();
    }

    __device__ __forceinline__ void reset()
    {
#pragma unroll
        for (int mt = 0; mt < 8; ++mt)
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[mt][e] = 0.0f;
        m_run = -INFINITY;
        l_run = 0.0f;
    }

    // Gathers a chunk of nr (1..16) rows into `stage`: lane i < 16 copies key
    // row `row` (the lane's own row i), lane 16 + i the value row of the same
    // row; value rows past nr are zeroed (their weights are 0, and 0 * NaN
    // from stale bytes must not happen).  `row` is the row's offset in rows
    // of K and V.  Lane 0 posts the expected bytes on `bar`.  The caller
    // orders the zeroing before the chunk is consumed (__syncwarp).
    __device__ __forceinline__ void issue(char* stage, const uint16_t* __restrict__ K,
                                          const uint16_t* __restrict__ V, int64_t row, int nr, uint64_t* bar)
    {
        const int lane = threadIdx.x & 31, i = lane & 15;
        char* dst = stage + (lane >> 4) * kWChunk * kWRowStride + i * kWRowStride;
        if (i < nr) {
            const uint16_t* src = (lane < 16 ? K : V) + row * kHeadDim;
            bulk_copy_g2s(dst, src, kHeadDim * 2, bar);
        } else if (lane >= 16) {
            uint4* z = reinterpret_cast<uint4*>(dst);
#pragma unroll
            for (int e = 0; e < kHeadDim * 2 / 16; ++e) z[e] = make_uint4(0, 0, 0, 0);
        }
        if (lane == 0) mbar_arrive_expect_tx(bar, (uint32_t)nr * 2u * kHeadDim * 2u);
    }

    // The same gather through the load/store path: 16-byte cp.async copies,
    // lane l taking pieces l, l + 32, ... of the chunk's 32 rows (keys 0-15,
    // then values 0-15; 16 pieces each), rows past nr zero-filled.  `row`:
    // lane i < 16 holds the row offset of key i.  One commit group per chunk;
    // the caller waits for it (cp_async_wait) and syncs the warp before
    // consume().
    __device__ __forceinline__ void issue_lsu(char* stage, const uint16_t* __restrict__ K,
                                              const uint16_t* __restrict__ V, int64_t row, int nr)
    {
        const int lane = threadIdx.x & 31;
        const uint32_t s0 = smem_addr(stage);
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const int rr = 2 * i + (lane >> 4);  // stage row: 0-15 keys, 16-31 values
            const int kr = rr & 15;
            const int64_t rk = __shfl_sync(kFullMask, row, kr);
            const uint16_t* src = (rr < 16 ? K : V) + rk * kHeadDim + (lane & 15) * 8;
            cp_async16_zfill(s0 + (uint32_t)(rr * kWRowStride + (lane & 15) * 16), src, kr < nr ? 16u : 0u);
        }
        cp_async_commit();
    }

    // The same copies as issue_lsu, with their completion counted on `bar`
    // instead of in a commit group: each lane's arrival (cp.async.mbarrier.
    // arrive.noinc) lands once its own copies have, so `bar` must expect 32
    // arrivals per phase (mbar_init(bar, 32)) and the chunk has landed when the
    // phase completes; a wait on it can be bounded.
    __device__ __forceinline__ void issue_lsu_mbar(char* stage, const uint16_t* __restrict__ K,
                                                   const uint16_t* __restrict__ V, int64_t row, int nr, uint64_t* bar)
    {
        const int lane = threadIdx.x & 31;
        const uint32_t s0 = smem_addr(stage);
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const int rr = 2 * i + (lane >> 4);  // stage row: 0-15 keys, 16-31 values
            const int kr = rr & 15;
            const int64_t rk = __shfl_sync(kFullMask, row, kr);
            const uint16_t* src = (rr < 16 ? K : V) + rk * kHeadDim + (lane & 15) * 8;
            cp_async16_zfill(s0 + (uint32_t)(rr * kWRowStride + (lane & 15) * 16), src, kr < nr ? 16u : 0u);
        }
        asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_addr(bar)) : "memory");
    }

    // Adds the chunk of nr rows that has landed in the stage at shared address
    // `ks` (keys, then values) to the online softmax.  Ends with every lane's
    // reads of the stage ordered before later bulk copies into it.
    __device__ __forceinline__ void consume(uint32_t ks, int nr)
    {
        const int lane = threadIdx.x & 31;
        const uint32_t vs = ks + kWChunk * kWRowStride;
        const int q4 = lane >> 3;
        // ldmatrix lane address: key row (q4 >> 1) * 8 + lane % 8, channel half q4 & 1
        const uint32_t lrow = (uint32_t)(((q4 >> 1) * 8 + (lane & 7)) * kWRowStride + (q4 & 1) * 16);
        const int t2 = (lane & 3) * 2;
        // ---- logits^T: keys 0-7 (c0) and 8-15 (c1) of head lane/4.
        float c0[4] = {0.f, 0.f, 0.f, 0.f}, c1[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
            uint32_t bk[4];
            ldsm_x4(ks + lrow + kk * 32, bk);
            uint2 qv;
            if constexpr (QS) qv = qfrag[kk * 32 + lane];
            else qv = make_uint2(qa[kk][0], qa[kk][1]);
            const uint32_t a[4] = {qv.x, 0u, qv.y, 0u};
            mma_bf16(c0, a, bk[0], bk[1]);
            mma_bf16(c1, a, bk[2], bk[3]);
        }
        float sv[4] = {c0[0] * kInvSqrtD, c0[1] * kInvSqrtD, c1[0] * kInvSqrtD, c1[1] * kInvSqrtD};
        sv[0] = t2 < nr ? sv[0] : -INFINITY;
        sv[1] = t2 + 1 < nr ? sv[1] : -INFINITY;
        sv[2] = t2 + 8 < nr ? sv[2] : -INFINITY;
        sv[3] = t2 + 9 < nr ? sv[3] : -INFINITY;
        // ---- online softmax of head lane/4 over the quad's 16 keys.
        float mc = fmaxf(fmaxf(sv[0], sv[1]), fmaxf(sv[2], sv[3]));
        mc = fmaxf(mc, __shfl_xor_sync(kFullMask, mc, 1));
        mc = fmaxf(mc, __shfl_xor_sync(kFullMask, mc, 2));
        const float m_new = fmaxf(m_run, mc);
        const float sc = expf(m_run - m_new);  // 0 on the first chunk (m_run = -inf)
        float p[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) p[e] = expf(sv[e] - m_new);
        float ps = (p[0] + p[1]) + (p[2] + p[3]);
        ps += __shfl_xor_sync(kFullMask, ps, 1);
        ps += __shfl_xor_sync(kFullMask, ps, 2);
        l_run = l_run * sc + ps;
        m_run = m_new;
        // ---- rescale: the accumulators hold heads 2 (lane%4) and + 1 (quads 2 (lane%4), + 1).
        const float sa = __shfl_sync(kFullMask, sc, (lane & 3) * 8);
        const float sb = __shfl_sync(kFullMask, sc, (lane & 3) * 8 + 4);
#pragma unroll
        for (int mt = 0; mt < 8; ++mt) {
            acc[mt][0] *= sa;
            acc[mt][1] *= sb;
            acc[mt][2] *= sa;
            acc[mt][3] *= sb;
        }
        // ---- weights as B: (keys 2 (lane%4) + {0,1}, head lane/4) and keys + 8.
        const float h0 = bf16_round(p[0]), h1 = bf16_round(p[1]), h2 = bf16_round(p[2]), h3 = bf16_round(p[3]);
        const uint32_t bh0 = pack_bf16(h0, h1), bh1 = pack_bf16(h2, h3);
        const uint32_t bl0 = pack_bf16(p[0] - h0, p[1] - h1), bl1 = pack_bf16(p[2] - h2, p[3] - h3);
#pragma unroll
        for (int mt = 0; mt < 8; ++mt) {
            uint32_t av[4];
            ldsm_x4_t(vs + lrow + mt * 32, av);
            // .trans of (keys (q4>>1)*8.., channels 16 mt + (q4&1)*8..) gives A = V^T in
            // the order (ch 0-7, k 0-7), (ch 8-15, k 0-7), (ch 0-7, k 8-15), (ch 8-15, k 8-15).
            mma_bf16(acc[mt], av, bh0, bh1);
            mma_bf16(acc[mt], av, bl0, bl1);
        }
        // Every lane's reads of this stage precede the next copies into it.
        fence_proxy_async_shared();
        __syncwarp();
    }

    // Stores the warp's state for a merge in shared memory: o_sm [8][128]
    // (head-major, unnormalised weighted value sums), m_sm[h], l_sm[h].
    __device__ __forceinline__ void store(float* o_sm, float* m_sm, float* l_sm) const
    {
        const int lane = threadIdx.x & 31, t2 = (lane & 3) * 2;
        if ((lane & 3) == 0 && (lane >> 2) < G) {
            m_sm[lane >> 2] = m_run;
            l_sm[lane >> 2] = l_run;
        }
#pragma unroll
        for (int mt = 0; mt < 8; ++mt) {
            const int ch = mt * 16 + (lane >> 2);
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                if (t2 + hh < G) {
                    o_sm[(t2 + hh) * kHeadDim + ch] = acc[mt][hh];
                    o_sm[(t2 + hh) * kHeadDim + ch + 8] = acc[mt][2 + hh];
                }
            }
        }
    }
};

}  // namespace socket_attn
