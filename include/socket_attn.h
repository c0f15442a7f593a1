/*
 * socket_attn.h -- C ABI of the SOCKET decode hot path on NVIDIA B200 (sm_100a).
 *
 * SOCKET (SOft Collision Kernel EsTimator) replaces dense decode attention by
 * attention over the k keys with the largest "soft collision" score.  The
 * method, as summarised on
 *   [ES] "Resumen Técnico: SOCKET - Estimador de Núcleo de Colisión Suave para
 *        Atención Escasa" (gist.science/es/paper/2602.06283),
 *        "Metodología: SOCKET" > "Mecanismo Central: LSH Suave", steps 1-4;
 *   [DE] "SOCKET: SOft Collision Kernel EsTimator for Sparse Attention"
 *        (gist.science/de/paper/2602.06283), "Technische Zusammenfassung" >
 *        "Methodik: SOCKET" > "Kernmechanismus: Soft LSH",
 * has a prefill part (hash every key into L tables, cache value norms) and a
 * decode part (soft-assign the query, score keys, select top-k, attend).
 *
 * Conventions shared by every entry point
 *   - Pointers named "device" are device memory (cudaMalloc'ed, e.g. by
 *     PyTorch) owned by the caller.  The library never allocates or frees.
 *   - Every compute call is asynchronous on `stream` (a cudaStream_t passed as
 *     void*; NULL = the legacy default stream).  It never synchronises the
 *     host.  A non-OK status means nothing was launched, except SOCKET_ECUDA
 *     after a launch error; outputs are then undefined.
 *   - No exceptions, device traps or device asserts.  Host-side checks reject
 *     bad arguments before any launch; socket_last_error() explains why.
 *   - Element types: SOCKET_F32 (IEEE binary32) or SOCKET_BF16 (bfloat16).
 *   - Tensor layouts are dense, row-major, innermost dimension last.
 *   - Head dimension d must be 128.  B, Hq, Hkv, N, Ncap are int64.
 *   - Units: a (batch row, kv head) pair is a "unit"; U = B * Hkv.  The Hq/Hkv
 *     query heads of a unit (grouped-query attention) share one selection.
 */
#ifndef SOCKET_ATTN_H
#define SOCKET_ATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Status codes. */
#define SOCKET_OK            0  /* success (work queued on the stream)            */
#define SOCKET_EINVAL        1  /* bad argument: null pointer, size, alignment    */
#define SOCKET_EUNSUPPORTED  2  /* valid but not built: d != 128, P > 8, ...      */
#define SOCKET_ECUDA         3  /* a CUDA launch failed; message has the reason   */
#define SOCKET_EWORKSPACE    4  /* workspace too small or misaligned              */

/* Element types. */
#define SOCKET_F32  0
#define SOCKET_BF16 1

/* Limits. */
#define SOCKET_HEAD_DIM   128
#define SOCKET_MAX_P      8    /* bucket ids are one byte: 2^P <= 256 buckets */
#define SOCKET_MAX_L      128
#define SOCKET_MAX_GROUP  16   /* Hq / Hkv */

/*
 * Device error word.  The first 4 bytes of the decode workspace hold a word
 * that socket_decode clears at its start and that a kernel sets (bitwise OR)
 * when one of its bounded waits expires (it then skips its work and leaves
 * its outputs undefined).  The host may read it after the stream has drained;
 * 0 means every wait completed.
 */
#define SOCKET_WS_ERROR_OFFSET 0
#define SOCKET_DEVERR_GATHER_TIMEOUT 0x1u  /* attention: a key/value row gather */
#define SOCKET_DEVERR_TABLE_TIMEOUT  0x2u  /* scoring: a copy into shared memory (soft tables, ids) */
#define SOCKET_DEVERR_SELECT_TIMEOUT 0x4u  /* selection + attention: a slice's wait for the unit's threshold */

/*
 * socket_hash_keys -- prefill hashing ([ES] step 1 "Pre-cálculo (Prellenado)";
 * [DE] "Vorverarbeitung (Prefill)").  Keys are hashed into L independent
 * tables by random projection, one bucket id per table, and the value norms
 * are cached:
 *     id_l(k)  = sum_{p<P} [ <W_{l,p}, k> > 0 ] * 2^p      (bit p <-> plane p)
 *     vnorm(k) = ||v||_2
 * Only keys n_begin <= n < n_end of every unit are written, so the same call
 * hashes a whole prefill (0, N) or appends one decode-step key (N, N + 1).
 *
 *   K, V      device, [B][Hkv][Ncap][d] of kv_dtype, 16-byte aligned.
 *   W         device, [L][P][d] bfloat16 bits (one set of hyperplanes shared
 *             by every batch row and head), 16-byte aligned.
 *   ids       device out, [B][Hkv][Ncap/32][Lr/16][32][16] uint8,
 *             Lr = socket_ids_row_bytes(L) = 32 * ceil(L / 32), 16-byte aligned.
 *             Every key has an id row of Lr bytes, in blocks of 32 slots: slot
 *             s of block c of key n holds the id of table 32c + (s + n) mod 32
 *             when that table is < L, else 0.  Keys are grouped in chunks of 32
 *             and a chunk stores its rows piece-major: the 16-byte piece p of
 *             the row of key 32m + j sits at [m][p][j].  (The rotation lets
 *             the 32 lanes of a warp, scoring keys 32m .. 32m + 31, read 32
 *             different tables in every lookup; the chunking makes each
 *             lane's 16-byte load part of one contiguous 512-byte warp load.)
 *   vnorm     device out, [B][Hkv][Ncap] float32, 16-byte aligned.
 * Preconditions: d == 128; 1 <= P <= 8; 1 <= L <= 128; Ncap % 32 == 0;
 * 0 <= n_begin <= n_end <= Ncap.  n_begin == n_end queues nothing.
 * Bucket ids are exact except where some |<W_{l,p}, k>| is within float32
 * accumulation error of 0 (below ~1e-6 * ||k|| for d = 128).
 */
int socket_hash_keys(const void* K, const void* V, int kv_dtype,
                     int64_t B, int64_t Hkv, int64_t Ncap,
                     int64_t n_begin, int64_t n_end, int64_t d,
                     const uint16_t* W, int L, int P,
                     uint8_t* ids, float* vnorm, void* stream);

/*
 * socket_ids_row_bytes -- bytes of one key's id row for L tables
 * (32 * ceil(L / 32)), or 0 if L is outside 1..SOCKET_MAX_L.
 */
int socket_ids_row_bytes(int L);

/*
 * socket_hash_check -- waits for `stream`, then reports whether a hashing
 * kernel of this library gave up on one of its bounded waits since the last
 * check (SOCKET_ECUDA with a message; its ids and norms are then
 * unspecified) and clears that record.  SOCKET_OK otherwise.  The record is
 * per device and process.
 */
int socket_hash_check(void* stream);

/*
 * socket_decode_workspace_size -- bytes of device scratch socket_decode needs
 * for these sizes (0 if the sizes are invalid).  The workspace needs no
 * initialisation, must be 256-byte aligned, and may be reused by later calls
 * on the same stream; calls that overlap in time need separate workspaces.
 */
size_t socket_decode_workspace_size(int64_t B, int64_t Hq, int64_t Hkv, int64_t Ncap,
                                    int64_t d, int L, int P, int k);

/*
 * socket_decode -- one decode step for all B*Hq query heads of one layer
 * ([ES] steps 2-4 "Asignación Suave", "Puntuación", "Selección"; [DE] "Weiche
 * Zuweisung (Decoding)", "Bewertung", "Auswahl"):
 *   1. soft assignment: z_{h,l} = W_l q_h / ||q_h|| (z = 0 if q_h = 0), and
 *      p_{h,l}(b) = softmax over the 2^P sign patterns s_b of <s_b, z_{h,l}>/tau,
 *      which factorises to prod_p sigmoid(2 s_{b,p} z_{h,l,p} / tau);
 *      evaluated in float64, rounded once to float32.
 *   2. soft collision score of every live key n < N of a unit, summed over
 *      the unit's query heads:
 *         score(n) = vnorm(n) * sum_l sum_h p_{h,l}(id_l(n))      (float32)
 *   3. deterministic top-k: the k keys of largest score, equal scores going
 *      to the lower index; written in ascending index order.
 *   4. exact softmax attention of every query head of the unit over its k
 *      selected keys, with scale 1/sqrt(d); float32 output.
 *
 *   q          device, [B][Hq][d] of q_dtype, 16-byte aligned.
 *   W          device, [L][P][d] bfloat16 bits (the same as for hashing).
 *   ids, vnorm device, as written by socket_hash_keys.
 *   K, V       device, [B][Hkv][Ncap][d] of kv_dtype, 16-byte aligned.
 *   N          live keys per unit (the same for every unit), k <= N <= Ncap.
 *   tau        temperature, finite and >= 0.  tau = 0 is hard LSH: each
 *              query is hashed like a key (bit p = [<W_{l,p}, q> > 0]) and
 *              p_{h,l} is 1 on that bucket and 0 elsewhere, so a key's score
 *              is vnorm times its collision count over tables and heads.
 *   workspace  device scratch of >= socket_decode_workspace_size() bytes,
 *              256-byte aligned.
 *   idx_out    device out, [B][Hkv][k] int32, ascending per unit.
 *   out        device out, [B][Hq][d] float32, 16-byte aligned.
 *   scores_out device out or NULL, [B][Hkv][Ncap] float32, 16-byte aligned:
 *              if given, the scores of step 2 land here (entries n >= N are
 *              unspecified).
 * Preconditions: d == 128; 1 <= P <= 8; 1 <= L <= 128; Hq % Hkv == 0;
 * 1 <= Hq / Hkv <= 16; Ncap % 32 == 0; 1 <= k <= N <= Ncap; N < 2^31.
 * Inputs must be finite; non-finite values give an unspecified selection.
 */
int socket_decode(const void* q, int q_dtype, const uint16_t* W,
                  const uint8_t* ids, const float* vnorm,
                  const void* K, const void* V, int kv_dtype,
                  int64_t B, int64_t Hq, int64_t Hkv, int64_t Ncap, int64_t N, int64_t d,
                  int L, int P, double tau, int k,
                  void* workspace, size_t workspace_bytes,
                  int32_t* idx_out, float* out, float* scores_out, void* stream);

/*
 * socket_decode_append -- a decode step whose last n_new keys were just
 * appended: the caller has written keys and values N - n_new .. N - 1 of
 * every unit into K and V; this call hashes them (step 1, [ES] "Pre-cálculo
 * (Prellenado)" / [DE] "Vorverarbeitung (Prefill)": their rows of ids and
 * their vnorm are written, as socket_hash_keys would write them) inside the
 * step's first kernel, then runs socket_decode over N keys.  One call
 * replaces socket_hash_keys(N - n_new, N) followed by socket_decode.
 *
 *   Arguments as for socket_decode, except that ids and vnorm are also
 *   written (the rows of the n_new keys) and:
 *   n_new      1 <= n_new <= min(64, N).
 * The appended keys' projections are formed in float64 (by the kernel that
 * projects the queries), so an id can differ from socket_hash_keys' (float32
 * accumulation) only where some |<W_{l,p}, k>| is within float32
 * accumulation error of 0.  The workspace is
 * socket_decode_workspace_size()'s.
 */
int socket_decode_append(const void* q, int q_dtype, const uint16_t* W,
                         uint8_t* ids, float* vnorm,
                         const void* K, const void* V, int kv_dtype,
                         int64_t B, int64_t Hq, int64_t Hkv, int64_t Ncap, int64_t N, int64_t d,
                         int L, int P, double tau, int k, int64_t n_new,
                         void* workspace, size_t workspace_bytes,
                         int32_t* idx_out, float* out, float* scores_out, void* stream);

/*
 * socket_decode_per_head_workspace_size / socket_decode_per_head -- the same
 * step with one selection per query head instead of one per kv head: every
 * query is scored and selects on its own, as the pages state the method for
 * a single query ([ES] "Mecanismo Central: LSH Suave" steps 2-4: each new
 * query induces its own bucket distribution, its own scores and its own
 * top-k).  For query head h of batch row b, with kv head h / (Hq / Hkv):
 *     score_{b,h}(n) = vnorm(n) * sum_l p_{h,l}(id_l(n))
 * then top-k and exact attention of head h over its own k keys.  With
 * Hq == Hkv this is socket_decode.
 *
 *   Arguments as for socket_decode, except:
 *   idx_out    device out, [B][Hq][k] int32, ascending per query head.
 *   scores_out device out or NULL, [B][Hq][Ncap] float32, 16-byte aligned.
 *   workspace  >= socket_decode_per_head_workspace_size() bytes.
 * Preconditions: those of socket_decode, and B * Hq <= 65535.
 * The Hq / Hkv heads of a kv head read its ids and norms from HBM about once
 * (their scoring runs side by side); the lookups, the selections and the
 * gathers are per head.
 */
size_t socket_decode_per_head_workspace_size(int64_t B, int64_t Hq, int64_t Hkv, int64_t Ncap,
                                             int64_t d, int L, int P, int k);
int socket_decode_per_head(const void* q, int q_dtype, const uint16_t* W,
                           const uint8_t* ids, const float* vnorm,
                           const void* K, const void* V, int kv_dtype,
                           int64_t B, int64_t Hq, int64_t Hkv, int64_t Ncap, int64_t N, int64_t d,
                           int L, int P, double tau, int k,
                           void* workspace, size_t workspace_bytes,
                           int32_t* idx_out, float* out, float* scores_out, void* stream);

/*
 * socket_decode_static -- socket_decode for callers that cannot allocate
 * device memory.  The paper has no counterpart: this is a packaging variant
 * of socket_decode, same arguments minus the workspace, same results.
 *
 * Who needs it: code that runs where cudaMalloc is off limits and no one
 * hands it scratch memory -- e.g. a kernel library embedded in a serving
 * runtime that has already reserved (nearly) all device memory for its own
 * pool and exposes no scratch allocator, or a caller that must not risk the
 * device-wide synchronisation an allocation can cause in a latency-critical
 * path.  Such callers still pass their inputs and outputs.
 *
 * Scratch: a file-scope device array of SOCKET_STATIC_WORKSPACE_BYTES (64 MiB)
 * inside this library; every GPU that loads the library holds it until the
 * process exits.  Calls whose socket_decode_workspace_size() exceeds it are
 * rejected with SOCKET_EWORKSPACE before anything is launched.  The first
 * call on a device looks up the array's device address (once per device,
 * with that device current), so make that first call before any stream
 * capture.  Nothing here calls cudaMalloc, cudaFree or an allocating library
 * routine.  Every call on a device shares the same array, which keeps the
 * previous call's contents; the decode clears what must start at zero (its
 * counters and error word) itself.  Calls that overlap on the GPU (other
 * streams, other host threads) race on the array: serialise them.  The
 * looked-up address is kept for the life of the process: do not call this
 * entry point again on a device after cudaDeviceReset() in the same process
 * (the array may then live elsewhere).
 */
#define SOCKET_STATIC_WORKSPACE_BYTES (64u << 20)
int socket_decode_static(const void* q, int q_dtype, const uint16_t* W,
                         const uint8_t* ids, const float* vnorm,
                         const void* K, const void* V, int kv_dtype,
                         int64_t B, int64_t Hq, int64_t Hkv, int64_t Ncap, int64_t N, int64_t d,
                         int L, int P, double tau, int k,
                         int32_t* idx_out, float* out, float* scores_out, void* stream);

/*
 * Sequence-sharded decode -- one sequence's cache split by position over S
 * shards (e.g. S GPUs, one rank each), with the same selection and output
 * as socket_decode over the whole cache.  The method's pages claim scaling
 * to contexts of millions of tokens ([ES] "Significado y Afirmaciones";
 * [DE] "Bedeutung und Behauptungen") but describe no multi-device scheme;
 * this one rests on a fact of the selection: a key of the global top-k is in
 * its own shard's top-k (fewer than k keys of that shard beat it; ties go to
 * the lower index everywhere), so each shard selects locally, the shards
 * exchange k (score, global index) pairs per kv head, re-select, attend over
 * the selected keys they hold, and merge their softmax states.  Per step:
 *   1. socket_shard_select on every shard;
 *   2. gather the pairs of all shards in shard order (an all-gather);
 *   3. socket_shard_merge on every shard (the same global selection
 *      everywhere, plus each shard's own rows);
 *   4. socket_shard_attend on every shard;
 *   5. gather the partial outputs and states, socket_shard_combine.
 * Shard s holds global keys [n_offset_s, n_offset_s + N_s), the shards in
 * increasing order of n_offset with no gaps or overlaps; every shard uses the
 * same W, q, L, P, tau and k.  Global indices stay below 2^31.
 *
 * socket_shard_select -- steps a2-a4 on this shard's keys (its own cache
 * arrays, laid out as for socket_decode with N = N_s keys):
 *   cand_score, cand_index  device out, [B][Hkv][k] float32 / int32: the
 *             shard's min(k, N_s) selected keys in increasing index order,
 *             (score, n_offset + local index); slots past min(k, N_s) hold
 *             (-1, -1).
 *   workspace  as for socket_decode: socket_decode_workspace_size with this
 *             shard's Ncap and k' = min(k, N_s).
 * Preconditions as for socket_decode with N = N_s >= 1;
 * 0 <= n_offset, n_offset + N_s < 2^31.
 */
int socket_shard_select(const void* q, int q_dtype, const uint16_t* W,
                        const uint8_t* ids, const float* vnorm,
                        int64_t B, int64_t Hq, int64_t Hkv, int64_t Ncap, int64_t N, int64_t d,
                        int L, int P, double tau, int k, int64_t n_offset,
                        void* workspace, size_t workspace_bytes,
                        float* cand_score, int32_t* cand_index, void* stream);

/*
 * socket_shard_merge -- step a4 across shards: from the S shards' pairs,
 * cand_score / cand_index [S][B][Hkv][k] (shard order), the k with the
 * largest scores, ties to the lower index, in increasing index order:
 *   idx_out      device out, [B][Hkv][k] int32 global indices (as
 *                socket_decode's idx_out; -1 past the number of pairs when
 *                the shards hold fewer than k keys together).
 *   local_idx    device out, [B][Hkv][k] int32: the selected keys in
 *                [n_offset, n_offset + n_local) (the calling shard's),
 *                as local indices, increasing.
 *   local_count  device out, [B][Hkv] int32: how many of them.
 * Arrays 4-byte aligned.  S >= 1, S * k <= 2^30.
 */
int socket_shard_merge(const float* cand_score, const int32_t* cand_index, int S,
                       int64_t B, int64_t Hkv, int k, int64_t n_offset, int64_t n_local,
                       int32_t* idx_out, int32_t* local_idx, int32_t* local_count, void* stream);

/*
 * socket_shard_attend_workspace_size -- bytes of device scratch that
 * socket_shard_attend needs for these sizes (256-byte aligned), or 0 if the
 * sizes are invalid.
 */
size_t socket_shard_attend_workspace_size(int64_t B, int64_t Hq, int64_t Hkv, int64_t Ncap, int64_t d, int k);

/*
 * socket_shard_attend -- step a5 on this shard's share of the selection:
 * for each query row, softmax attention (scale 1/sqrt(d)) over the
 * local_count[b][h] keys local_idx[b][h][0 ..) of its kv head, in the
 * shard's own K and V ([B][Hkv][Ncap][d]):
 *   out  device out, [B][Hq][d] float32, normalised over those keys (0 for a
 *        kv head with none);
 *   ml   device out, [B][Hq][2] float32: the largest logit m and the sum l
 *        of exp(logit - m) over those keys (l = 0 when there are none).
 * The workspace (socket_shard_attend_workspace_size) is cleared by the call
 * itself.  Alignment as for socket_decode; ml 8-byte aligned.
 */
int socket_shard_attend(const void* q, int q_dtype, const void* K, const void* V, int kv_dtype,
                        int64_t B, int64_t Hq, int64_t Hkv, int64_t Ncap, int64_t d, int k,
                        const int32_t* local_idx, const int32_t* local_count,
                        void* workspace, size_t workspace_bytes, float* out, float* ml, void* stream);

/*
 * socket_shard_combine -- the log-sum-exp merge of the S shards' partial
 * results, outs [S][B][Hq][d] and mls [S][B][Hq][2] (shard order): per query
 * row, out = sum_s w_s o_s / sum_s w_s with w_s = exp(m_s - M) l_s over the
 * shards with l_s > 0, M their largest m_s.  out [B][Hq][d] float32.
 * outs and out 16-byte aligned, mls 8-byte.  d == 128.
 */
int socket_shard_combine(const float* outs, const float* mls, int S, int64_t B, int64_t Hq, int64_t d,
                         float* out, void* stream);

/*
 * socket_last_error -- message for the last non-OK status returned on the
 * calling host thread ("" if none).  The pointer stays valid until the next
 * call on that thread.
 */
const char* socket_last_error(void);

/*
 * socket_set_step_events -- timing diagnostics.  Until called again with
 * n = 0, every socket_decode call made on the calling host thread records
 * events[0] on its stream before its first kernel and events[i] after its
 * i-th kernel, for i = 1 .. min(n - 1, SOCKET_DECODE_KERNELS).  The events
 * are cudaEvent_t handles (passed as void*) that the caller created and
 * reads with cudaEventElapsedTime; the library only records them.  Inside a
 * stream capture they are recorded as external event nodes.  Returns
 * SOCKET_EINVAL if n < 0, n > SOCKET_DECODE_KERNELS + 1, or a handle is NULL.
 * The kernels, in order: soft tables, scoring, top-k, attention.  When a
 * shape runs fewer kernels (socket_set_selection_path), the events after the
 * last one are recorded right after it: with the fused selection + attention
 * kernel, events[3] and events[4] follow it; with the whole step in one
 * kernel, events[1] .. events[4] follow that kernel.
 */
#define SOCKET_DECODE_KERNELS 4
int socket_set_step_events(void* const* events, int n);

/*
 * socket_set_wait_limit -- failure-path diagnostic.  Sets how many times a
 * decode kernel polls before it gives up on a wait: scoring and attention
 * for data they have requested, the fused selection + attention for the
 * unit's threshold that another of its CTAs publishes.  On expiry the kernel
 * sets its bit in the workspace error word (SOCKET_DEVERR_TABLE_TIMEOUT,
 * SOCKET_DEVERR_GATHER_TIMEOUT, SOCKET_DEVERR_SELECT_TIMEOUT), lets the
 * copies it has already issued land, and returns without its results.
 * Default 4194304 polls (~ a second or more); 0 makes every such wait give
 * up at once, which is how tests drive the give-up path without a fault;
 * 0xffffffff restores the default.  Process-wide; affects calls made after
 * it.  Returns the previous limit.  No counterpart in the method.
 */
uint32_t socket_set_wait_limit(uint32_t polls);

/*
 * socket_set_selection_path -- diagnostic.  Chooses the kernels of a decode
 * step for later decode calls of this process.  U is the number of units
 * (B*Hkv, or B*Hq for per-head calls), G the query heads per unit.
 *   SOCKET_PATH_AUTO (0): by shape.
 *     - Small problems take one kernel for the whole step (soft tables,
 *       scores, top-k, attention): N <= 8192, k <= 1024, L <= 32, G <= 8,
 *       G*L <= 64, G*L*P <= 512, U at most the SM count, no keys appended in
 *       the call.
 *     - Otherwise bf16 q and K/V with G <= 8 and k <= 4096 take a soft-table
 *       kernel, a scoring kernel and one fused selection + attention kernel
 *       when the separate top-k kernel would not fill the SMs
 *       (U*ceil(N/32768) below the SM count).
 *     - Every other shape takes the four separate kernels: soft tables,
 *       scoring, top-k, attention.
 *   SOCKET_PATH_SEPARATE (1): always the four separate kernels.
 * All paths write the same scores and indices (bit for bit) and outputs that
 * agree to float32 rounding; tests use this to compare them on the same
 * inputs.  Returns the previous path, or -1 (and changes nothing) for
 * another value.  No counterpart in the method.
 */
#define SOCKET_PATH_AUTO     0
#define SOCKET_PATH_SEPARATE 1
int socket_set_selection_path(int path);

/*
 * socket_last_decode_path -- diagnostic.  Which kernels the calling host
 * thread's most recent successful socket_decode, socket_decode_static,
 * socket_decode_append or socket_decode_per_head launched:
 *   SOCKET_STEP_SEPARATE (0): soft tables, scoring, top-k, attention;
 *   SOCKET_STEP_FUSED (1): soft tables, scoring, fused selection + attention;
 *   SOCKET_STEP_ONE_KERNEL (2): the whole step in one kernel.
 * -1 if the thread has made no such call, or its last one failed before it
 * launched anything.  Timing tools use it to name the intervals between the
 * events of socket_set_step_events.  No counterpart in the method.
 */
#define SOCKET_STEP_SEPARATE   0
#define SOCKET_STEP_FUSED      1
#define SOCKET_STEP_ONE_KERNEL 2
int socket_last_decode_path(void);

/* socket_version -- ABI version of this library (major * 100 + minor). */
int socket_version(void);

#ifdef __cplusplus
}
#endif

#endif /* SOCKET_ATTN_H */
