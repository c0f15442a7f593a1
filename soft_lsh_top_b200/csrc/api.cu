// C ABI of the SOCKET library: argument checks, workspace layout, launches.
#include <math.h>
#include <stdarg.h>
#include <stdio.h>
#include <stdlib.h>

#include <atomic>
#include <mutex>
#include <string>
#include <vector>

#include "internal.h"
#include "socket_attn.h"

namespace socket_attn {
namespace {

thread_local std::string g_last_error;
thread_local cudaEvent_t g_step_events[SOCKET_DECODE_KERNELS + 1];
thread_local int g_num_step_events = 0;

// Records diagnostic step event i (if registered) on the stream.
cudaError_t mark_step(int i, cudaStream_t stream)
{
    if (i >= g_num_step_events) return cudaSuccess;
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    cudaError_t e = cudaStreamIsCapturing(stream, &cap);
    if (e != cudaSuccess) return e;
    return cudaEventRecordWithFlags(g_step_events[i], stream,
                                    cap == cudaStreamCaptureStatusActive ? cudaEventRecordExternal : 0);
}

int fail(int status, const char* fmt, ...)
{
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof buf, fmt, ap);
    va_end(ap);
    g_last_error = buf;
    return status;
}

int cuda_status(cudaError_t e, const char* what)
{
    if (e == cudaSuccess) return SOCKET_OK;
    return fail(SOCKET_ECUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// Shape checks shared by both entry points; returns SOCKET_OK or a status.
int check_common(int64_t B, int64_t Hkv, int64_t Ncap, int64_t d, int L, int P)
{
    if (d != SOCKET_HEAD_DIM) return fail(SOCKET_EUNSUPPORTED, "head dim d=%lld unsupported (only 128)", (long long)d);
    if (P < 1 || P > SOCKET_MAX_P) return fail(SOCKET_EUNSUPPORTED, "P=%d outside [1, 8]", P);
    if (L < 1 || L > SOCKET_MAX_L) return fail(SOCKET_EUNSUPPORTED, "L=%d outside [1, 128]", L);
    if (B < 1 || Hkv < 1) return fail(SOCKET_EINVAL, "B=%lld and Hkv=%lld must be >= 1", (long long)B, (long long)Hkv);
    if (B * Hkv > 65535) return fail(SOCKET_EUNSUPPORTED, "B*Hkv=%lld above 65535", (long long)(B * Hkv));
    if (Ncap < 32 || Ncap % 32 != 0) return fail(SOCKET_EINVAL, "Ncap=%lld must be a positive multiple of 32", (long long)Ncap);
    if (Ncap >= (int64_t(1) << 31)) return fail(SOCKET_EUNSUPPORTED, "Ncap=%lld must be < 2^31", (long long)Ncap);
    return SOCKET_OK;
}

bool valid_dtype(int t) { return t == SOCKET_F32 || t == SOCKET_BF16; }

int fill_shape(DecodeShape& s, int64_t B, int64_t Hq, int64_t Hkv, int64_t Ncap, int64_t N, int64_t d, int L, int P,
               int k)
{
    int st = check_common(B, Hkv, Ncap, d, L, P);
    if (st != SOCKET_OK) return st;
    if (Hq < 1 || Hq % Hkv != 0) return fail(SOCKET_EINVAL, "Hq=%lld must be a positive multiple of Hkv=%lld", (long long)Hq, (long long)Hkv);
    if (Hq / Hkv > SOCKET_MAX_GROUP) return fail(SOCKET_EUNSUPPORTED, "group size Hq/Hkv=%lld above 16", (long long)(Hq / Hkv));
    if (k < 1) return fail(SOCKET_EINVAL, "k=%d must be >= 1", k);
    if (N < k || N > Ncap) return fail(SOCKET_EINVAL, "need k <= N <= Ncap (k=%d N=%lld Ncap=%lld)", k, (long long)N, (long long)Ncap);
    s.B = B;
    s.Hq = Hq;
    s.Hkv = Hkv;
    s.Ncap = Ncap;
    s.N = N;
    s.d = d;
    s.L = L;
    s.P = P;
    s.k = k;
    s.G = (int)(Hq / Hkv);
    s.U = B * Hkv;
    s.share = 1;
    s.NB = 1 << P;
    s.nsplit = 0;
    return SOCKET_OK;
}

// Every query head selects its own keys: each head is a unit of one query
// row, and the Hq / Hkv units of a kv head read that head's ids, norms, keys
// and values.
void select_per_head(DecodeShape& s)
{
    s.share = s.G;
    s.U = s.B * s.Hq;
    s.G = 1;
}

size_t workspace_size(bool per_head, int64_t B, int64_t Hq, int64_t Hkv, int64_t Ncap, int64_t d, int L, int P,
                      int k)
{
    DecodeShape s;
    const std::string saved = g_last_error;
    // N = k is the smallest valid N; the layout does not depend on N.
    if (fill_shape(s, B, Hq, Hkv, Ncap, k, d, L, P, k) != SOCKET_OK) {
        g_last_error = saved;
        return 0;
    }
    if (per_head) {
        if (B * Hq > 65535) return 0;
        select_per_head(s);
    }
    s.nsplit = (k + 15) / 16;  // attention splits never exceed ceil(k / 16)
    return decode_workspace_layout(s).total;
}

// Scratch of socket_shard_attend: error word, merge counters, split partials.
struct AttendWorkspace {
    size_t counters, part_o, part_ml, total;
};
AttendWorkspace attend_layout(const DecodeShape& s)
{
    AttendWorkspace w;
    size_t off = align256(4);  // error word at 0
    w.counters = off;
    off = align256(off + 4 * (size_t)s.U);
    w.part_o = off;
    off = align256(off + 4 * (size_t)s.U * s.G * s.nsplit * s.d);
    w.part_ml = off;
    off = align256(off + 8 * (size_t)s.U * s.G * s.nsplit);
    w.total = off;
    return w;
}

// Shape of an attention-only call (no hashing parameters involved).  k is
// the row capacity of the selection lists, which may exceed this shard's keys.
int fill_attend_shape(DecodeShape& s, int64_t B, int64_t Hq, int64_t Hkv, int64_t Ncap, int64_t d, int k)
{
    if (k < 1) return fail(SOCKET_EINVAL, "k=%d must be >= 1", k);
    const int st = fill_shape(s, B, Hq, Hkv, Ncap, Ncap, d, 1, 1, (int)(k < Ncap ? k : Ncap));
    s.k = k;
    return st;
}

}  // namespace

cudaError_t set_smem_limit_once(const void* func, int bytes)
{
    struct Entry {
        const void* func;
        int dev, bytes;
    };
    static std::mutex lock;
    static std::vector<Entry> done;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    std::lock_guard<std::mutex> guard(lock);
    for (const Entry& x : done)
        if (x.func == func && x.dev == dev && x.bytes >= bytes) return cudaSuccess;
    e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e != cudaSuccess) return e;
    // Every decode kernel asks for the largest shared-memory carveout, so
    // consecutive kernels of a step never need an SM's L1/shared split changed.
    e = cudaFuncSetAttribute(func, cudaFuncAttributePreferredSharedMemoryCarveout, (int)cudaSharedmemCarveoutMaxShared);
    if (e != cudaSuccess) return e;
    done.push_back({func, dev, bytes});
    return cudaSuccess;
}

int device_num_sms()
{
    constexpr int kMaxDevices = 128;
    static int sms[kMaxDevices];  // 0: not looked up yet
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 1;
    if (sms[dev] == 0) {
        int n = 0;
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
        sms[dev] = n > 0 ? n : 1;
    }
    return sms[dev];
}

namespace {
constexpr uint32_t kDefaultWaitPolls = 1u << 22;
std::atomic<uint32_t> g_wait_polls{kDefaultWaitPolls};
}  // namespace

uint32_t wait_poll_limit() { return g_wait_polls.load(std::memory_order_relaxed); }

std::atomic<int> g_selection_path{SOCKET_PATH_AUTO};
thread_local int g_last_path = -1;  // SOCKET_STEP_* of this thread's last decode, or -1

void clear_last_decode_path() { g_last_path = -1; }

bool pdl_enabled()
{
    static const bool on = getenv("SOCKET_NO_PDL") == nullptr;
    return on;
}

int record_error(int status, const char* message)
{
    g_last_error = message;
    return status;
}

DecodeWorkspace decode_workspace_layout(const DecodeShape& s)
{
    DecodeWorkspace w;
    size_t off = 0;
    w.err = off;
    off = align256(off + 4);
    w.counters = off;
    off = align256(off + 4 * (size_t)s.U);
    w.topk_done = off;
    off = align256(off + 4 * (size_t)s.U);
    w.unit_hist = off;
    off = align256(off + 4 * (size_t)s.U * kScoreHistBins);
    w.cand_cnt = off;
    off = align256(off + 4 * (size_t)s.U);
    w.cand = off;
    off = align256(off + 8 * (size_t)s.U * topk_candidate_capacity(s.Ncap));
    w.bitmap = off;
    off = align256(off + 4 * (size_t)s.U * (size_t)topk_bitmap_stride(s.Ncap));
    w.tables = off;
    off = align256(off + 4 * (size_t)s.U * ((s.L + 31) / 32) * s.NB * 64);
    w.scores = off;
    off = align256(off + 4 * (size_t)s.U * s.Ncap);
    w.part_o = off;
    off = align256(off + 4 * (size_t)s.U * s.G * s.nsplit * s.d);
    w.part_ml = off;
    off = align256(off + 8 * (size_t)s.U * s.G * s.nsplit);
    w.sel_idx = off;
    off = align256(off + 4 * (size_t)s.U * s.k);
    w.topk_info = off;
    off = align256(off + 4 * (size_t)s.U * (size_t)topk_info_stride(s.Ncap));
    w.total = off;
    return w;
}

// One decode step; per_head: every query head selects its own keys; the
// last n_new keys of every unit are hashed inside the step (ids and norms
// written through app_ids / app_vnorm) when n_new > 0.
int decode(bool per_head, const void* q, int q_dtype, const uint16_t* W, const uint8_t* ids, const float* vnorm,
           const void* K, const void* V, int kv_dtype, int64_t B, int64_t Hq, int64_t Hkv, int64_t Ncap, int64_t N,
           int64_t d, int L, int P, double tau, int k, void* workspace, size_t workspace_bytes, int32_t* idx_out,
           float* out, float* scores_out, cudaStream_t cs, int64_t n_new = 0, uint8_t* app_ids = nullptr,
           float* app_vnorm = nullptr)
{
    g_last_error.clear();
    g_last_path = -1;
    DecodeShape s;
    int st = fill_shape(s, B, Hq, Hkv, Ncap, N, d, L, P, k);
    if (st != SOCKET_OK) return st;
    if (!valid_dtype(q_dtype) || !valid_dtype(kv_dtype))
        return fail(SOCKET_EINVAL, "q_dtype=%d / kv_dtype=%d unknown", q_dtype, kv_dtype);
    if (!(tau >= 0.0) || !isfinite(tau)) return fail(SOCKET_EINVAL, "tau=%g must be finite and >= 0", tau);
    if (!q || !W || !ids || !vnorm || !K || !V || !idx_out || !out || !workspace)
        return fail(SOCKET_EINVAL, "null pointer argument");
    if (!aligned(q, 16) || !aligned(W, 16) || !aligned(ids, 16) || !aligned(vnorm, 16) || !aligned(K, 16) ||
        !aligned(V, 16) || !aligned(out, 16) || !aligned(idx_out, 4) || (scores_out && !aligned(scores_out, 16)))
        return fail(SOCKET_EINVAL, "q, W, ids, vnorm, K, V, out, scores_out must be 16-byte aligned, idx_out 4-byte");
    if (n_new < 0 || n_new > kMaxAppend || n_new > N)
        return fail(SOCKET_EINVAL, "n_new=%lld outside [0, min(%d, N)]", (long long)n_new, kMaxAppend);
    if (!aligned(workspace, 256)) return fail(SOCKET_EWORKSPACE, "workspace must be 256-byte aligned");
    if (per_head) {
        if (B * Hq > 65535) return fail(SOCKET_EUNSUPPORTED, "B*Hq=%lld above 65535", (long long)(B * Hq));
        select_per_head(s);
    }
    // Attention splits (or slices of the fused selection + attention) never
    // exceed ceil(k / 16), the count the advertised size covers.
    const int num_sms = device_num_sms();
    const bool by_shape = g_selection_path.load(std::memory_order_relaxed) == SOCKET_PATH_AUTO;
    const bool small = by_shape && n_new == 0 && small_step_supported(s, num_sms);
    const bool fused = by_shape && !small && select_attend_supported(kv_dtype, q_dtype, s, num_sms);
    s.nsplit = fused ? select_attend_slices(s, num_sms) : attention_splits(kv_dtype, q_dtype, s.G, s.U, k, num_sms);
    const size_t need = workspace_size(per_head, B, Hq, Hkv, Ncap, d, L, P, k);
    if (workspace_bytes < need)
        return fail(SOCKET_EWORKSPACE, "workspace has %zu bytes, needs %zu", workspace_bytes, need);

    const DecodeWorkspace w = decode_workspace_layout(s);
    char* base = static_cast<char*>(workspace);
    uint32_t* err_word = reinterpret_cast<uint32_t*>(base + w.err);
    uint32_t* counters = reinterpret_cast<uint32_t*>(base + w.counters);
    float* tables = reinterpret_cast<float*>(base + w.tables);
    float* scores = scores_out ? scores_out : reinterpret_cast<float*>(base + w.scores);
    uint32_t* topk_done = reinterpret_cast<uint32_t*>(base + w.topk_done);
    uint32_t* bitmap = reinterpret_cast<uint32_t*>(base + w.bitmap);
    uint32_t* unit_hist = reinterpret_cast<uint32_t*>(base + w.unit_hist);
    uint32_t* cand_cnt = reinterpret_cast<uint32_t*>(base + w.cand_cnt);
    uint2* cand = reinterpret_cast<uint2*>(base + w.cand);
    float* part_o = reinterpret_cast<float*>(base + w.part_o);
    float2* part_ml = reinterpret_cast<float2*>(base + w.part_ml);

    if ((st = cuda_status(mark_step(0, cs), "step event record")) != SOCKET_OK) return st;
    g_last_path = small ? SOCKET_STEP_ONE_KERNEL : fused ? SOCKET_STEP_FUSED : SOCKET_STEP_SEPARATE;
    if (small) {
        // One kernel for the whole step; the step's other events follow at once.
        st = cuda_status(launch_small_step(q, q_dtype, W, ids, vnorm, K, V, kv_dtype, s, tau, idx_out, out,
                                           scores_out, err_word, cs),
                         "small-step kernel launch");
        if (st != SOCKET_OK) return st;
        for (int i = 1; i <= 4; ++i)
            if ((st = cuda_status(mark_step(i, cs), "step event record")) != SOCKET_OK) return st;
        return SOCKET_OK;
    }
    AppendHash app;
    if (n_new > 0) {
        app.K = K;
        app.V = V;
        app.kv_dtype = kv_dtype;
        app.ids = app_ids;
        app.vnorm = app_vnorm;
        app.begin = N - n_new;
        app.end = N;
    }
    st = cuda_status(launch_soft_tables(q, q_dtype, W, s, tau, app, tables, err_word, counters, topk_done, unit_hist,
                                        cand_cnt, cs),
                     "soft-table kernel launch");
    if (st != SOCKET_OK) return st;
    if ((st = cuda_status(mark_step(1, cs), "step event record")) != SOCKET_OK) return st;
    const int64_t fresh_chunk = n_new > 0 ? (N - n_new) / 32 : Ncap / 32;
    st = cuda_status(launch_score(tables, ids, vnorm, s, fresh_chunk, scores, unit_hist, err_word, cs),
                     "score kernel launch");
    if (st != SOCKET_OK) return st;
    if ((st = cuda_status(mark_step(2, cs), "step event record")) != SOCKET_OK) return st;
    if (fused) {
        // One kernel selects and attends; the step's fourth event follows the third at once.
        st = cuda_status(launch_select_attend(scores, unit_hist, cand_cnt, cand, bitmap, topk_done, counters, q, K, V,
                                              s, part_o, part_ml, err_word, idx_out, out, cs),
                         "selection + attention kernel launch");
        if (st != SOCKET_OK) return st;
        if ((st = cuda_status(mark_step(3, cs), "step event record")) != SOCKET_OK) return st;
        return cuda_status(mark_step(4, cs), "step event record");
    }
    st = cuda_status(launch_topk(scores, unit_hist, cand_cnt, cand, bitmap, topk_done,
                                 reinterpret_cast<uint32_t*>(base + w.topk_info), err_word, s, idx_out, cs),
                     "top-k kernel launch");
    if (st != SOCKET_OK) return st;
    if ((st = cuda_status(mark_step(3, cs), "step event record")) != SOCKET_OK) return st;
    st = cuda_status(launch_attention(q, q_dtype, K, V, kv_dtype, idx_out, nullptr, s, part_o, part_ml, counters,
                                      err_word, out, nullptr, cs),
                     "attention kernel launch");
    if (st != SOCKET_OK) return st;
    return cuda_status(mark_step(4, cs), "step event record");
}

}  // namespace socket_attn

using namespace socket_attn;

extern "C" {

int socket_version(void) { return 200; }

int socket_set_step_events(void* const* events, int n)
{
    g_last_error.clear();
    if (n < 0 || n > SOCKET_DECODE_KERNELS + 1) return fail(SOCKET_EINVAL, "n=%d outside [0, %d]", n, SOCKET_DECODE_KERNELS + 1);
    if (n > 0 && !events) return fail(SOCKET_EINVAL, "null event array");
    for (int i = 0; i < n; ++i)
        if (!events[i]) return fail(SOCKET_EINVAL, "null event handle %d", i);
    for (int i = 0; i < n; ++i) g_step_events[i] = static_cast<cudaEvent_t>(events[i]);
    g_num_step_events = n;
    return SOCKET_OK;
}

const char* socket_last_error(void) { return g_last_error.c_str(); }

uint32_t socket_set_wait_limit(uint32_t polls)
{
    return g_wait_polls.exchange(polls == 0xffffffffu ? kDefaultWaitPolls : polls);
}

int socket_set_selection_path(int path)
{
    if (path != SOCKET_PATH_AUTO && path != SOCKET_PATH_SEPARATE) return -1;
    return g_selection_path.exchange(path);
}

int socket_last_decode_path(void) { return g_last_path; }

int socket_hash_keys(const void* K, const void* V, int kv_dtype, int64_t B, int64_t Hkv, int64_t Ncap,
                     int64_t n_begin, int64_t n_end, int64_t d, const uint16_t* W, int L, int P, uint8_t* ids,
                     float* vnorm, void* stream)
{
    g_last_error.clear();
    int st = check_common(B, Hkv, Ncap, d, L, P);
    if (st != SOCKET_OK) return st;
    if (!valid_dtype(kv_dtype)) return fail(SOCKET_EINVAL, "kv_dtype=%d unknown", kv_dtype);
    if (n_begin < 0 || n_begin > n_end || n_end > Ncap)
        return fail(SOCKET_EINVAL, "need 0 <= n_begin <= n_end <= Ncap (got %lld, %lld, %lld)", (long long)n_begin,
                    (long long)n_end, (long long)Ncap);
    if (!K || !V || !W || !ids || !vnorm) return fail(SOCKET_EINVAL, "null pointer argument");
    if (!aligned(K, 16) || !aligned(V, 16) || !aligned(W, 16) || !aligned(ids, 16) || !aligned(vnorm, 16))
        return fail(SOCKET_EINVAL, "K, V, W, ids and vnorm must be 16-byte aligned");
    if (n_begin == n_end) return SOCKET_OK;
    return cuda_status(launch_hash_keys(K, V, kv_dtype, B, Hkv, Ncap, n_begin, n_end, W, L, P, ids, vnorm,
                                        static_cast<cudaStream_t>(stream)),
                       "hash kernel launch");
}

int socket_hash_check(void* stream)
{
    g_last_error.clear();
    uint32_t bits = 0;
    const int e = hash_device_error(static_cast<cudaStream_t>(stream), &bits);
    if (e != 0) return cuda_status(static_cast<cudaError_t>(e), "hash error check");
    if (bits) return fail(SOCKET_ECUDA, "hash kernel: a bounded wait expired (device error bits 0x%x)", bits);
    return SOCKET_OK;
}

int socket_ids_row_bytes(int L) { return (L >= 1 && L <= SOCKET_MAX_L) ? ids_row_bytes(L) : 0; }

size_t socket_decode_workspace_size(int64_t B, int64_t Hq, int64_t Hkv, int64_t Ncap, int64_t d, int L, int P,
                                    int k)
{
    return workspace_size(false, B, Hq, Hkv, Ncap, d, L, P, k);
}

size_t socket_decode_per_head_workspace_size(int64_t B, int64_t Hq, int64_t Hkv, int64_t Ncap, int64_t d, int L,
                                             int P, int k)
{
    return workspace_size(true, B, Hq, Hkv, Ncap, d, L, P, k);
}

int socket_decode(const void* q, int q_dtype, const uint16_t* W, const uint8_t* ids, const float* vnorm,
                  const void* K, const void* V, int kv_dtype, int64_t B, int64_t Hq, int64_t Hkv, int64_t Ncap,
                  int64_t N, int64_t d, int L, int P, double tau, int k, void* workspace, size_t workspace_bytes,
                  int32_t* idx_out, float* out, float* scores_out, void* stream)
{
    return decode(false, q, q_dtype, W, ids, vnorm, K, V, kv_dtype, B, Hq, Hkv, Ncap, N, d, L, P, tau, k, workspace,
                  workspace_bytes, idx_out, out, scores_out, static_cast<cudaStream_t>(stream));
}

int socket_decode_append(const void* q, int q_dtype, const uint16_t* W, uint8_t* ids, float* vnorm, const void* K,
                         const void* V, int kv_dtype, int64_t B, int64_t Hq, int64_t Hkv, int64_t Ncap, int64_t N,
                         int64_t d, int L, int P, double tau, int k, int64_t n_new, void* workspace,
                         size_t workspace_bytes, int32_t* idx_out, float* out, float* scores_out, void* stream)
{
    if (n_new < 1) {
        g_last_error.clear();
        return fail(SOCKET_EINVAL, "n_new=%lld must be >= 1", (long long)n_new);
    }
    return decode(false, q, q_dtype, W, ids, vnorm, K, V, kv_dtype, B, Hq, Hkv, Ncap, N, d, L, P, tau, k, workspace,
                  workspace_bytes, idx_out, out, scores_out, static_cast<cudaStream_t>(stream), n_new, ids, vnorm);
}

int socket_decode_per_head(const void* q, int q_dtype, const uint16_t* W, const uint8_t* ids, const float* vnorm,
                           const void* K, const void* V, int kv_dtype, int64_t B, int64_t Hq, int64_t Hkv,
                           int64_t Ncap, int64_t N, int64_t d, int L, int P, double tau, int k, void* workspace,
                           size_t workspace_bytes, int32_t* idx_out, float* out, float* scores_out, void* stream)
{
    return decode(true, q, q_dtype, W, ids, vnorm, K, V, kv_dtype, B, Hq, Hkv, Ncap, N, d, L, P, tau, k, workspace,
                  workspace_bytes, idx_out, out, scores_out, static_cast<cudaStream_t>(stream));
}


int socket_shard_select(const void* q, int q_dtype, const uint16_t* W, const uint8_t* ids, const float* vnorm,
                        int64_t B, int64_t Hq, int64_t Hkv, int64_t Ncap, int64_t N, int64_t d, int L, int P,
                        double tau, int k, int64_t n_offset, void* workspace, size_t workspace_bytes,
                        float* cand_score, int32_t* cand_index, void* stream)
{
    g_last_error.clear();
    if (k < 1) return fail(SOCKET_EINVAL, "k=%d must be >= 1", k);
    if (N < 1) return fail(SOCKET_EINVAL, "a shard holds at least one key (N=%lld)", (long long)N);
    const int k_eff = (int)(N < k ? N : k);
    DecodeShape s;
    int st = fill_shape(s, B, Hq, Hkv, Ncap, N, d, L, P, k_eff);
    if (st != SOCKET_OK) return st;
    if (!valid_dtype(q_dtype)) return fail(SOCKET_EINVAL, "q_dtype=%d unknown", q_dtype);
    if (!(tau >= 0.0) || !isfinite(tau)) return fail(SOCKET_EINVAL, "tau=%g must be finite and >= 0", tau);
    if (n_offset < 0 || n_offset + N > (int64_t(1) << 31) - 1)
        return fail(SOCKET_EINVAL, "n_offset=%lld: global indices must stay below 2^31", (long long)n_offset);
    if (!q || !W || !ids || !vnorm || !workspace || !cand_score || !cand_index)
        return fail(SOCKET_EINVAL, "null pointer argument");
    if (!aligned(q, 16) || !aligned(W, 16) || !aligned(ids, 16) || !aligned(vnorm, 16) || !aligned(cand_score, 4) ||
        !aligned(cand_index, 4))
        return fail(SOCKET_EINVAL, "q, W, ids, vnorm must be 16-byte aligned, cand_score and cand_index 4-byte");
    if (!aligned(workspace, 256)) return fail(SOCKET_EWORKSPACE, "workspace must be 256-byte aligned");
    const size_t need = workspace_size(false, B, Hq, Hkv, Ncap, d, L, P, k_eff);
    if (workspace_bytes < need)
        return fail(SOCKET_EWORKSPACE, "workspace has %zu bytes, needs %zu", workspace_bytes, need);
    s.nsplit = 0;  // no attention here
    const DecodeWorkspace w = decode_workspace_layout(s);
    char* base = static_cast<char*>(workspace);
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    uint32_t* err_word = reinterpret_cast<uint32_t*>(base + w.err);
    float* scores = reinterpret_cast<float*>(base + w.scores);
    int32_t* sel = reinterpret_cast<int32_t*>(base + w.sel_idx);
    AppendHash none;
    st = cuda_status(launch_soft_tables(q, q_dtype, W, s, tau, none, reinterpret_cast<float*>(base + w.tables), err_word,
                                        reinterpret_cast<uint32_t*>(base + w.counters),
                                        reinterpret_cast<uint32_t*>(base + w.topk_done),
                                        reinterpret_cast<uint32_t*>(base + w.unit_hist),
                                        reinterpret_cast<uint32_t*>(base + w.cand_cnt), cs),
                     "soft-table kernel launch");
    if (st != SOCKET_OK) return st;
    st = cuda_status(launch_score(reinterpret_cast<float*>(base + w.tables), ids, vnorm, s, Ncap / 32, scores,
                                  reinterpret_cast<uint32_t*>(base + w.unit_hist), err_word, cs),
                     "score kernel launch");
    if (st != SOCKET_OK) return st;
    st = cuda_status(launch_topk(scores, reinterpret_cast<uint32_t*>(base + w.unit_hist),
                                 reinterpret_cast<uint32_t*>(base + w.cand_cnt), reinterpret_cast<uint2*>(base + w.cand),
                                 reinterpret_cast<uint32_t*>(base + w.bitmap),
                                 reinterpret_cast<uint32_t*>(base + w.topk_done),
                                 reinterpret_cast<uint32_t*>(base + w.topk_info), err_word, s, sel, cs),
                     "top-k kernel launch");
    if (st != SOCKET_OK) return st;
    return cuda_status(launch_shard_pairs(scores, sel, s, k_eff, k, n_offset, cand_score, cand_index, cs),
                       "shard pair kernel launch");
}

int socket_shard_merge(const float* cand_score, const int32_t* cand_index, int S, int64_t B, int64_t Hkv, int k,
                       int64_t n_offset, int64_t n_local, int32_t* idx_out, int32_t* local_idx, int32_t* local_count,
                       void* stream)
{
    g_last_error.clear();
    if (S < 1 || k < 1 || B < 1 || Hkv < 1) return fail(SOCKET_EINVAL, "S, k, B, Hkv must be >= 1");
    if (B * Hkv > 65535) return fail(SOCKET_EUNSUPPORTED, "B*Hkv=%lld above 65535", (long long)(B * Hkv));
    if ((int64_t)S * k > (int64_t(1) << 30)) return fail(SOCKET_EUNSUPPORTED, "S*k above 2^30");
    if (n_offset < 0 || n_local < 0) return fail(SOCKET_EINVAL, "n_offset and n_local must be >= 0");
    if (!cand_score || !cand_index || !idx_out || !local_idx || !local_count)
        return fail(SOCKET_EINVAL, "null pointer argument");
    if (!aligned(cand_score, 4) || !aligned(cand_index, 4) || !aligned(idx_out, 4) || !aligned(local_idx, 4) ||
        !aligned(local_count, 4))
        return fail(SOCKET_EINVAL, "arrays must be 4-byte aligned");
    return cuda_status(launch_shard_merge(cand_score, cand_index, S, B * Hkv, k, n_offset, n_local, idx_out, local_idx,
                                          local_count, static_cast<cudaStream_t>(stream)),
                       "shard merge kernel launch");
}

size_t socket_shard_attend_workspace_size(int64_t B, int64_t Hq, int64_t Hkv, int64_t Ncap, int64_t d, int k)
{
    DecodeShape s;
    const std::string saved = g_last_error;
    if (fill_attend_shape(s, B, Hq, Hkv, Ncap, d, k) != SOCKET_OK) {
        g_last_error = saved;
        return 0;
    }
    s.nsplit = (k + 15) / 16;  // attention splits never exceed ceil(k / 16)
    return attend_layout(s).total;
}

int socket_shard_attend(const void* q, int q_dtype, const void* K, const void* V, int kv_dtype, int64_t B,
                        int64_t Hq, int64_t Hkv, int64_t Ncap, int64_t d, int k, const int32_t* local_idx,
                        const int32_t* local_count, void* workspace, size_t workspace_bytes, float* out, float* ml,
                        void* stream)
{
    g_last_error.clear();
    DecodeShape s;
    int st = fill_attend_shape(s, B, Hq, Hkv, Ncap, d, k);
    if (st != SOCKET_OK) return st;
    if (!valid_dtype(q_dtype) || !valid_dtype(kv_dtype))
        return fail(SOCKET_EINVAL, "q_dtype=%d / kv_dtype=%d unknown", q_dtype, kv_dtype);
    if (!q || !K || !V || !local_idx || !local_count || !workspace || !out || !ml)
        return fail(SOCKET_EINVAL, "null pointer argument");
    if (!aligned(q, 16) || !aligned(K, 16) || !aligned(V, 16) || !aligned(out, 16) || !aligned(ml, 8) ||
        !aligned(local_idx, 4) || !aligned(local_count, 4))
        return fail(SOCKET_EINVAL, "q, K, V, out must be 16-byte aligned, ml 8-byte, local_idx and local_count 4-byte");
    if (!aligned(workspace, 256)) return fail(SOCKET_EWORKSPACE, "workspace must be 256-byte aligned");
    const size_t need = socket_shard_attend_workspace_size(B, Hq, Hkv, Ncap, d, k);
    if (workspace_bytes < need)
        return fail(SOCKET_EWORKSPACE, "workspace has %zu bytes, needs %zu", workspace_bytes, need);
    s.nsplit = attention_splits(kv_dtype, q_dtype, s.G, s.U, k, device_num_sms());
    const AttendWorkspace w = attend_layout(s);
    char* base = static_cast<char*>(workspace);
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    // The error word and the merge counters start at zero.
    if ((st = cuda_status(cudaMemsetAsync(base, 0, w.part_o, cs), "workspace clear")) != SOCKET_OK) return st;
    return cuda_status(launch_attention(q, q_dtype, K, V, kv_dtype, local_idx, local_count, s,
                                        reinterpret_cast<float*>(base + w.part_o),
                                        reinterpret_cast<float2*>(base + w.part_ml),
                                        reinterpret_cast<uint32_t*>(base + w.counters),
                                        reinterpret_cast<uint32_t*>(base), out, reinterpret_cast<float2*>(ml), cs),
                       "attention kernel launch");
}

int socket_shard_combine(const float* outs, const float* mls, int S, int64_t B, int64_t Hq, int64_t d, float* out,
                         void* stream)
{
    g_last_error.clear();
    if (d != SOCKET_HEAD_DIM) return fail(SOCKET_EUNSUPPORTED, "head dim d=%lld unsupported (only 128)", (long long)d);
    if (S < 1 || B < 1 || Hq < 1) return fail(SOCKET_EINVAL, "S, B, Hq must be >= 1");
    if (!outs || !mls || !out) return fail(SOCKET_EINVAL, "null pointer argument");
    if (!aligned(outs, 16) || !aligned(out, 16) || !aligned(mls, 8))
        return fail(SOCKET_EINVAL, "outs and out must be 16-byte aligned, mls 8-byte");
    return cuda_status(launch_shard_combine(outs, reinterpret_cast<const float2*>(mls), S, B * Hq, out,
                                            static_cast<cudaStream_t>(stream)),
                       "shard combine kernel launch");
}

}  // extern "C"
