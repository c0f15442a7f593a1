// Sequence-sharded decode: the kernels of the exchange between shards.
//
// When one sequence's cache is split by position across shards (e.g. GPUs),
// every shard selects its own top-k, the shards' (score, global index) pairs
// are gathered, and the global top-k is re-selected from them: a key of the
// global top-k is in its own shard's top-k, because fewer than k keys of
// that shard beat it (ties go to the lower index in both).  Each shard then
// attends over the selected keys it holds and the shards' partial softmax
// states (largest logit, sum of weights, normalised output) are merged with
// the log-sum-exp rule.  The method's pages describe no multi-device scheme;
// they claim the estimator scales to contexts of millions of tokens
// ("Resumen Técnico: SOCKET ...", "Significado y Afirmaciones";
// "SOCKET: SOft Collision Kernel EsTimator for Sparse Attention", "Bedeutung
// und Behauptungen"), and this split is how such a context is spread over
// devices with the selection unchanged.
#include "common.cuh"
#include "internal.h"
#include "select.cuh"

namespace socket_attn {
namespace {

using namespace select512;

// cand[u][i] = (score of the i-th selected key, its global index) for
// i < k_eff; (-1, -1) pads the remaining slots up to k.
__global__ void shard_pairs_kernel(const float* __restrict__ scores, const int32_t* __restrict__ sel, int64_t Ncap,
                                   int k_eff, int k, int64_t n_offset, float* __restrict__ cand_score,
                                   int32_t* __restrict__ cand_index)
{
    const int64_t u = blockIdx.y;
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= k) return;
    pdl_wait();  // the selection comes from the previous kernel on the stream
    float sc = -1.0f;
    int32_t gi = -1;
    if (i < k_eff) {
        const int32_t n = __ldcg(sel + u * k_eff + i);
        sc = __ldcg(scores + u * Ncap + n);
        gi = (int32_t)(n + n_offset);
    }
    cand_score[u * k + i] = sc;
    cand_index[u * k + i] = gi;
}

// One CTA per unit over the S shards' k pairs each, in shard order (shard s's
// global indices precede shard s+1's, each shard's list ascending): the k
// pairs with the largest scores, ties to the lower index, written in index
// order to idx_out; the ones in [n_offset, n_offset + n_local) also to this
// shard's local list (as local indices) and their number to local_count.
__global__ __launch_bounds__(kThreads) void shard_merge_kernel(const float* __restrict__ cand_score,
                                                               const int32_t* __restrict__ cand_index, int S,
                                                               int64_t U, int k, int64_t n_offset, int64_t n_local,
                                                               int32_t* __restrict__ idx_out,
                                                               int32_t* __restrict__ local_idx,
                                                               int32_t* __restrict__ local_count)
{
    __shared__ Shared sh;
    const int tid = threadIdx.x;
    const int64_t u = blockIdx.x;
    const int n = S * k;
    // Entry e = s k + i of this unit: shard s, slot i.
    auto at = [&](int e) -> int64_t { return ((int64_t)(e / k) * U + u) * k + (e % k); };
    pdl_wait();  // the gathered pairs may come from the previous kernel on the stream

    // Valid pairs (index >= 0; scores are >= 0, so their bit patterns order
    // like the values) and how many to keep.
    uint32_t valid = 0;
    for (int e = tid; e < n; e += kThreads) valid += __ldcg(cand_index + at(e)) >= 0;
    uint32_t nvalid;
    block_exclusive_scan(valid, sh.warp_sums, nvalid);
    const uint32_t keep = min(nvalid, (uint32_t)k);

    // The keep-th largest score: three digits of the bit pattern.
    auto bits_of = [&](int e) -> uint32_t {
        const int64_t a = at(e);
        // invalid pairs get a pattern no prefix with bit 31 clear can match
        return __ldcg(cand_index + a) >= 0 ? __float_as_uint(__ldcg(cand_score + a)) : 0xffffffffu;
    };
    uint32_t t = 0, need = 0;
    if (keep > 0) {
        uint32_t prefix = 0, mask = 0x80000000u, krem = keep;
        radix_digit(sh, n, bits_of, 20, 0x7ffu, true, prefix, mask, krem);
        radix_digit(sh, n, bits_of, 9, 0x7ffu, true, prefix, mask, krem);
        radix_digit(sh, n, bits_of, 0, 0x1ffu, true, prefix, mask, krem);
        t = prefix;
        need = krem;  // pairs equal to t to keep: the first `need` of them in entry order
    }

    // Selected pairs in entry order (= index order): positions from block
    // scans, tile by tile.
    int32_t* out = idx_out + u * k;
    int32_t* lout = local_idx + u * k;
    uint32_t out_base = 0, ties_seen = 0, local_base = 0;
    for (int e0 = 0; e0 < n && keep > 0; e0 += kThreads) {
        const int e = e0 + tid;
        uint32_t x = 0xffffffffu;
        int32_t gi = -1;
        if (e < n) {
            gi = __ldcg(cand_index + at(e));
            if (gi >= 0) x = __float_as_uint(__ldcg(cand_score + at(e)));
        }
        const bool above = gi >= 0 && x > t && x != 0xffffffffu;
        const bool tie = gi >= 0 && x == t;
        uint32_t ties_total;
        const uint32_t tie_rank = ties_seen + block_exclusive_scan(tie ? 1u : 0u, sh.warp_sums, ties_total);
        const bool take = above || (tie && tie_rank < need);
        uint32_t taken;
        const uint32_t pos = out_base + block_exclusive_scan(take ? 1u : 0u, sh.warp_sums, taken);
        const bool mine = take && gi >= n_offset && gi < n_offset + n_local;
        uint32_t mine_total;
        const uint32_t lpos = local_base + block_exclusive_scan(mine ? 1u : 0u, sh.warp_sums, mine_total);
        if (take && pos < (uint32_t)k) out[pos] = gi;
        if (mine && lpos < (uint32_t)k) lout[lpos] = (int32_t)(gi - n_offset);
        out_base += taken;
        ties_seen += ties_total;
        local_base += mine_total;
    }
    for (int i = (int)min(out_base, (uint32_t)k) + tid; i < k; i += kThreads) out[i] = -1;
    if (tid == 0) local_count[u] = (int32_t)min(local_base, (uint32_t)k);
}

// One warp per query row: out = sum_s w_s o_s / sum_s w_s with
// w_s = exp(m_s - M) l_s over the shards that had rows (l_s > 0), M their
// largest m_s; zero when no shard had rows.
__global__ void shard_combine_kernel(const float* __restrict__ outs, const float2* __restrict__ mls, int S,
                                     int64_t rows, float* __restrict__ out)
{
    const int lane = threadIdx.x & 31;
    const int64_t r = (int64_t)blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);
    if (r >= rows) return;
    pdl_wait();
    float M = -INFINITY;
    for (int s = 0; s < S; ++s) {
        const float2 ml = __ldcg(mls + (int64_t)s * rows + r);
        if (ml.y > 0.0f) M = fmaxf(M, ml.x);
    }
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    float wsum = 0.0f;
    for (int s = 0; s < S; ++s) {
        const float2 ml = __ldcg(mls + (int64_t)s * rows + r);
        if (!(ml.y > 0.0f)) continue;
        const float w = expf(ml.x - M) * ml.y;
        const float4 o = __ldcg(reinterpret_cast<const float4*>(outs + ((int64_t)s * rows + r) * kHeadDim) + lane);
        acc.x += w * o.x;
        acc.y += w * o.y;
        acc.z += w * o.z;
        acc.w += w * o.w;
        wsum += w;
    }
    const float inv = wsum > 0.0f ? 1.0f / wsum : 0.0f;
    reinterpret_cast<float4*>(out + r * kHeadDim)[lane] = make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
}

}  // namespace

cudaError_t launch_shard_pairs(const float* scores, const int32_t* sel, const DecodeShape& s, int k_eff, int k,
                               int64_t n_offset, float* cand_score, int32_t* cand_index, cudaStream_t stream)
{
    const dim3 grid((unsigned)((k + 255) / 256), (unsigned)s.U);
    return launch_pdl(shard_pairs_kernel, grid, dim3(256), 0, stream, scores, sel, s.Ncap, k_eff, k, n_offset,
                      cand_score, cand_index);
}

cudaError_t launch_shard_merge(const float* cand_score, const int32_t* cand_index, int S, int64_t U, int k,
                               int64_t n_offset, int64_t n_local, int32_t* idx_out, int32_t* local_idx,
                               int32_t* local_count, cudaStream_t stream)
{
    return launch_pdl(shard_merge_kernel, dim3((unsigned)U), dim3(kThreads), 0, stream, cand_score, cand_index, S, U,
                      k, n_offset, n_local, idx_out, local_idx, local_count);
}

cudaError_t launch_shard_combine(const float* outs, const float2* mls, int S, int64_t rows, float* out,
                                 cudaStream_t stream)
{
    constexpr int kRowsPerBlock = 8;
    const dim3 grid((unsigned)((rows + kRowsPerBlock - 1) / kRowsPerBlock));
    return launch_pdl(shard_combine_kernel, grid, dim3(32 * kRowsPerBlock), 0, stream, outs, mls, S, rows, out);
}

}  // namespace socket_attn
