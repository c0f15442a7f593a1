// Internal launchers and workspace layout of the SOCKET library.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace socket_attn {

// Sizes of one decode call, validated by the API layer.
struct DecodeShape {
    int64_t B, Hq, Hkv, Ncap, N, d;
    int L, P, k;
    int G;         // query heads per unit: Hq / Hkv, or 1 when every head selects its own keys
    int64_t U;     // units: B * Hkv, or B * Hq when every head selects its own keys
    int share;     // units reading one kv unit's ids, norms, keys and values (1, or Hq / Hkv)
    int NB;        // 2^P
    int nsplit;    // attention splits per unit
};

// Per-unit histogram of live scores, taken by the scoring kernel over the
// score bit pattern >> kScoreHistShift (1/16 octave per bin; finite
// non-negative scores land below bin 4081).
constexpr int kScoreHistBins = 4096;
constexpr int kScoreHistShift = 19;
// Top-k candidate capacity per unit (keys in the threshold bin of the
// histogram, at most Ncap); above it the top-k kernel selects over all of
// the unit's scores instead.
constexpr int kTopkCandidates = 8192;
int topk_candidate_capacity(int64_t Ncap);
// Words per unit row of the top-k selection bitmap (Ncap / 32 rounded up to
// a multiple of 4, so every row starts on a 16-byte boundary).
int64_t topk_bitmap_stride(int64_t Ncap);
// Words per unit of the top-k slices' record (keys in or above d0 per slice,
// first output slot per slice).
int64_t topk_info_stride(int64_t Ncap);

// Workspace regions (byte offsets from the workspace base, 256-aligned).
struct DecodeWorkspace {
    size_t err;        // uint32 device error word (offset 0)
    size_t counters;   // uint32 [U] merge counters
    size_t topk_done;  // uint32 [U] top-k tickets
    size_t unit_hist;  // uint32 [U][kScoreHistBins] score histogram
    size_t cand_cnt;   // uint32 [U] top-k candidate counters
    size_t cand;       // uint2 [U][cap] top-k candidates (index, bit pattern), cap = topk_candidate_capacity
    size_t bitmap;     // uint32 [U][topk_bitmap_stride(Ncap)] top-k selection bitmap; in the fused
                       // selection + attention, each unit's record (t, ti, sure counts, first slots)
    size_t tables;     // float [U][ceil(L/32)][NB][64], column j = table 32c + j mod 32
    size_t scores;     // float [U][Ncap]
    size_t part_o;     // float [U][G][nsplit][d]
    size_t part_ml;    // float2 [U][G][nsplit]
    size_t sel_idx;    // int32 [U][k] a shard's own selection (local indices)
    size_t topk_info;  // uint32 [U][topk_info_stride(Ncap)] top-k slices' counts and first slots
    size_t total;
};

DecodeWorkspace decode_workspace_layout(const DecodeShape& s);

// Rows of one attention chunk (the gather unit of the attention kernel).
int attention_chunk_rows(int kv_dtype);
// Attention CTAs per unit for these sizes (<= ceil(k / 16)).
int attention_splits(int kv_dtype, int q_dtype, int G, int64_t U, int k, int num_sms);
int attention_rows_per_cta(int k, int nsplit, int chunk);
// Multiprocessors of the current device (looked up once per device).
int device_num_sms();
// Forgets the calling thread's last decode path (socket_last_decode_path
// then returns -1 until a decode launches its kernels).
void clear_last_decode_path();
// Raises `func`'s dynamic shared-memory limit to `bytes` unless an earlier
// call already did so on the current device (one runtime call per kernel and
// device, not per launch).
cudaError_t set_smem_limit_once(const void* func, int bytes);

// --- kernels (each returns cudaGetLastError() after its launch) -------------
cudaError_t launch_hash_keys(const void* K, const void* V, int kv_dtype, int64_t B, int64_t Hkv,
                             int64_t Ncap, int64_t n_begin, int64_t n_end, const uint16_t* W,
                             int L, int P, uint8_t* ids, float* vnorm, cudaStream_t stream);

// Keys [begin, end) of every kv unit, just written to K and V by the caller,
// hashed inside the decode step (their ids and norms written) before scoring.
constexpr int kMaxAppend = 64;
struct AppendHash {
    const void* K = nullptr;
    const void* V = nullptr;
    int kv_dtype = 0;
    uint8_t* ids = nullptr;
    float* vnorm = nullptr;
    int64_t begin = 0, end = 0;  // empty: nothing hashed
};

// Also zeroes the error word, the merge counters, the top-k tickets, the
// score histograms and the candidate counters, and hashes `app`'s keys.
cudaError_t launch_soft_tables(const void* q, int q_dtype, const uint16_t* W, const DecodeShape& s,
                               double tau, const AppendHash& app, float* tables, uint32_t* err_word,
                               uint32_t* counters, uint32_t* topk_done, uint32_t* unit_hist, uint32_t* cand_cnt,
                               cudaStream_t stream);

// fresh_chunk: first 32-key chunk of a unit whose ids the preceding soft-table
// kernel writes in this step (none: a value >= Ncap / 32); such chunks are
// not fetched before that kernel has completed.
cudaError_t launch_score(const float* tables, const uint8_t* ids, const float* vnorm, const DecodeShape& s,
                         int64_t fresh_chunk, float* scores, uint32_t* unit_hist, uint32_t* err_word,
                         cudaStream_t stream);
// Bytes of one key's rotated id row (32 per started block of 32 tables).
int ids_row_bytes(int L);

cudaError_t launch_topk(const float* scores, const uint32_t* unit_hist, uint32_t* cand_cnt, uint2* cand,
                        uint32_t* bitmap, uint32_t* done, uint32_t* info, uint32_t* err_word, const DecodeShape& s,
                        int32_t* idx_out, cudaStream_t stream);

// Top-k fused with the attention over the selected keys (select_attend.cu):
// bfloat16 q, K and V, d = 128, G <= 8, k <= 4096, at most one unit per SM.
// s.nsplit must be select_attend_slices(s, num_sms): the slices per unit,
// whose partials part_o / part_ml hold ([U][G][C]).  info ([U][bitmap
// stride] words), done and tickets ([U], zero at entry, zero again at exit)
// are scratch.
bool select_attend_supported(int kv_dtype, int q_dtype, const DecodeShape& s, int num_sms);
int select_attend_slices(const DecodeShape& s, int num_sms);
cudaError_t launch_select_attend(const float* scores, const uint32_t* unit_hist, uint32_t* cand_cnt, uint2* cand,
                                 uint32_t* info, uint32_t* done, uint32_t* tickets, const void* q, const void* K,
                                 const void* V, const DecodeShape& s, float* part_o, float2* part_ml,
                                 uint32_t* err_word, int32_t* idx_out, float* out, cudaStream_t stream);

// The whole step (soft tables, scores, top-k, attention) in one kernel, one
// CTA per unit (small_step.cu): N <= 8192, k <= 1024, L <= 32, G <= 8,
// G*L <= 64, G*L*P <= 512, at most one unit per SM.  Writes only idx_out,
// out, scores_out (nullable) and clears the error word.
bool small_step_supported(const DecodeShape& s, int num_sms);
cudaError_t launch_small_step(const void* q, int q_dtype, const uint16_t* W, const uint8_t* ids, const float* vnorm,
                              const void* K, const void* V, int kv_dtype, const DecodeShape& s, double tau,
                              int32_t* idx_out, float* out, float* scores_out, uint32_t* err_word,
                              cudaStream_t stream);

// counts (nullable): rows of each unit's selection to use (the first
// counts[u] of its k slots; all k when null).  ml_out (nullable): per query
// row the largest logit and the sum of exp(logit - largest) over those rows
// (the log-sum-exp state a merge across shards needs); out is normalised by
// that sum (zero for a unit with no rows).
cudaError_t launch_attention(const void* q, int q_dtype, const void* K, const void* V, int kv_dtype,
                             const int32_t* idx, const int32_t* counts, const DecodeShape& s, float* part_o,
                             float2* part_ml, uint32_t* counters, uint32_t* err_word, float* out, float2* ml_out,
                             cudaStream_t stream);

// --- sequence-sharded decode (shard.cu) -------------------------------------
cudaError_t launch_shard_pairs(const float* scores, const int32_t* sel, const DecodeShape& s, int k_eff, int k,
                               int64_t n_offset, float* cand_score, int32_t* cand_index, cudaStream_t stream);
cudaError_t launch_shard_merge(const float* cand_score, const int32_t* cand_index, int S, int64_t U, int k,
                               int64_t n_offset, int64_t n_local, int32_t* idx_out, int32_t* local_idx,
                               int32_t* local_count, cudaStream_t stream);
cudaError_t launch_shard_combine(const float* outs, const float2* mls, int S, int64_t rows, float* out,
                                 cudaStream_t stream);

// Waits for `stream`, then reads and clears the hash kernels' device error
// bits; returns a cudaError_t value.
int hash_device_error(cudaStream_t stream, uint32_t* bits);

// Polls after which a decode kernel's wait for data gives up (the
// socket_set_wait_limit diagnostic; waits that drain copies already issued
// keep their own, long limit).
uint32_t wait_poll_limit();

// Sets the calling thread's socket_last_error() message; returns `status`.
int record_error(int status, const char* message);

}  // namespace socket_attn
