// vsa_forward_noalloc: the whole attention call without any allocation.
//
// Some callers cannot call cudaMalloc or take memory from a caching allocator:
// a plugin or custom operator that a host runtime hands only its input and
// output buffers, with no allocator handle; a runtime whose memory pool owns
// the whole device and forbids out-of-band allocations, because cudaMalloc
// synchronizes the device and fragments that pool; real-time code that must not
// allocate after start-up.  For them this entry point runs vsa_forward on a
// workspace that lives in this file's static device array instead of a
// caller buffer.
//
// The array is kNoallocWorkspaceBytes (VSA_NOALLOC_WORKSPACE_BYTES, 32 MiB).
// Every GPU on which this file's module is loaded holds it until the process
// exits; with CUDA's lazy module loading that is from the first call of this
// entry point on that GPU.
// In host code `g_noalloc_workspace` names a host-side stand-in, not device
// memory, so its device address is looked up once per device, with that
// device current, by cudaGetSymbolAddress on the first call there (cached
// afterwards).  All calls on a device share the array and it keeps the last
// call's contents; the forward call writes every byte it reads before reading
// it, so nothing needs clearing.  Calls that overlap on the GPU (other streams,
// other host threads) race on the array.
#include <cstdio>
#include <mutex>

#include "vsa_internal.h"

namespace {

constexpr size_t kNoallocWorkspaceBytes = VSA_NOALLOC_WORKSPACE_BYTES;
static_assert(kNoallocWorkspaceBytes % 256 == 0, "workspace size must keep 256-byte alignment");

static __device__ __align__(256) unsigned char g_noalloc_workspace[kNoallocWorkspaceBytes];

constexpr int kMaxDevices = 64;
std::mutex g_setup_mutex;
void* g_device_addr[kMaxDevices] = {};

// Device address of the static workspace on the current device (set-up on first use).
vsa_status noalloc_workspace(void** out) {
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return vsa::set_last_error(VSA_ERR_CUDA, "vsa_forward_noalloc: cudaGetDevice failed");
    if (dev < 0 || dev >= kMaxDevices)
        return vsa::set_last_error(VSA_ERR_UNSUPPORTED, "vsa_forward_noalloc: device ordinal out of range");
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    if (!g_device_addr[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_workspace);
        if (e != cudaSuccess || p == nullptr)
            return vsa::set_last_error(VSA_ERR_CUDA,
                                       "vsa_forward_noalloc: cudaGetSymbolAddress of the static workspace failed");
        g_device_addr[dev] = p;
    }
    *out = g_device_addr[dev];
    return VSA_OK;
}

}  // namespace

extern "C" vsa_status vsa_forward_noalloc(const vsa_shape* shape, const vsa_bf16* q, const vsa_bf16* k,
                                          const vsa_bf16* v, const vsa_bf16* g_coarse, const vsa_bf16* g_fine,
                                          int32_t topk, float scale, vsa_bf16* out, vsa_stream_t stream) {
    const size_t need = vsa_workspace_bytes(shape, topk);
    if (need == 0)   // malformed shape or top-k: let vsa_forward report the exact reason
        return vsa_forward(shape, q, k, v, g_coarse, g_fine, topk, scale, nullptr, 0, out, stream);
    if (need > kNoallocWorkspaceBytes) {
        char msg[256];
        snprintf(msg, sizeof(msg),
                 "vsa_forward_noalloc: this shape and top-k need %zu workspace bytes but the static workspace "
                 "holds %zu; call vsa_forward with a caller workspace",
                 need, kNoallocWorkspaceBytes);
        return vsa::set_last_error(VSA_ERR_WORKSPACE, msg);
    }
    void* ws = nullptr;
    const vsa_status st = noalloc_workspace(&ws);
    if (st != VSA_OK) return st;
    return vsa_forward(shape, q, k, v, g_coarse, g_fine, topk, scale, ws, kNoallocWorkspaceBytes, out, stream);
}
