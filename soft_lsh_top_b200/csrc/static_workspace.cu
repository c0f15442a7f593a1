// socket_decode_static: socket_decode with its scratch in a file-scope device
// array, for callers that cannot allocate device memory.  There is no
// counterpart in the method's description; this only changes where the
// scratch lives.
#include <stdio.h>

#include <mutex>

#include "internal.h"
#include "socket_attn.h"

namespace socket_attn {
namespace {

// The scratch.  In host code this name is a host-side stand-in, not a device
// address: it is only ever passed to cudaGetSymbolAddress below.
__device__ __align__(256) unsigned char g_static_workspace[SOCKET_STATIC_WORKSPACE_BYTES];

constexpr int kMaxDevices = 128;
std::mutex g_lock;
void* g_device_address[kMaxDevices];  // per device ordinal, set once

// Device address of the scratch on the current device, looked up once per
// device with that device current.
int static_workspace_address(void** out)
{
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) {
        char msg[256];
        snprintf(msg, sizeof msg, "socket_decode_static: cudaGetDevice failed: %s", cudaGetErrorString(e));
        return record_error(SOCKET_ECUDA, msg);
    }
    if (dev < 0 || dev >= kMaxDevices) return record_error(SOCKET_EUNSUPPORTED, "socket_decode_static: device ordinal out of range");
    std::lock_guard<std::mutex> guard(g_lock);
    if (!g_device_address[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_static_workspace);
        if (e != cudaSuccess || !p) {
            char msg[256];
            snprintf(msg, sizeof msg, "socket_decode_static: cudaGetSymbolAddress failed: %s", cudaGetErrorString(e));
            return record_error(SOCKET_ECUDA, msg);
        }
        g_device_address[dev] = p;
    }
    *out = g_device_address[dev];
    return SOCKET_OK;
}

}  // namespace
}  // namespace socket_attn

extern "C" int socket_decode_static(const void* q, int q_dtype, const uint16_t* W, const uint8_t* ids,
                                    const float* vnorm, const void* K, const void* V, int kv_dtype, int64_t B,
                                    int64_t Hq, int64_t Hkv, int64_t Ncap, int64_t N, int64_t d, int L, int P,
                                    double tau, int k, int32_t* idx_out, float* out, float* scores_out,
                                    void* stream)
{
    using namespace socket_attn;
    clear_last_decode_path();
    const size_t need = socket_decode_workspace_size(B, Hq, Hkv, Ncap, d, L, P, k);
    if (need > SOCKET_STATIC_WORKSPACE_BYTES) {
        char msg[320];
        snprintf(msg, sizeof msg,
                 "socket_decode_static: these sizes need %zu bytes of scratch but the static scratch holds %u "
                 "(SOCKET_STATIC_WORKSPACE_BYTES); use socket_decode with a caller-provided workspace",
                 need, (unsigned)SOCKET_STATIC_WORKSPACE_BYTES);
        return record_error(SOCKET_EWORKSPACE, msg);
    }
    void* ws = nullptr;
    const int st = static_workspace_address(&ws);
    if (st != SOCKET_OK) return st;
    // All argument checks (including sizes socket_decode_workspace_size
    // rejects with 0) happen inside socket_decode before any launch.
    return socket_decode(q, q_dtype, W, ids, vnorm, K, V, kv_dtype, B, Hq, Hkv, Ncap, N, d, L, P, tau, k, ws,
                         SOCKET_STATIC_WORKSPACE_BYTES, idx_out, out, scores_out, stream);
}
