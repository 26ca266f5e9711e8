// static_ws.cu -- attn_decode for callers that cannot allocate device memory.
//
// Some callers cannot call cudaMalloc (or any allocator) at the point where
// they decode: code running under a custom allocator that must not be
// re-entered, hooks that run inside another library's critical section, or
// processes whose device memory is fully reserved up front.  For them,
// attn_decode_static_ws runs exactly the same kernels as attn_decode, but uses
// as scratch a fixed array that lives in this library's device image instead
// of a caller-provided workspace.  It allocates nothing.
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/sparsekv.h"

namespace {

// The scratch array (kStaticWorkspaceBytes on every device that loads this
// library, held until the process exits).  In host code `g_static_ws` is only
// a host-side stand-in for the symbol, never a device address: the device
// address comes from cudaGetSymbolAddress below.
constexpr size_t kStaticWorkspaceBytes = SKV_STATIC_WORKSPACE_BYTES;
static __device__ __align__(256) unsigned char g_static_ws[kStaticWorkspaceBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_dev_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device; looked up once
// per device (the first call on a device does it, with that device current).
skv_status static_ws_ptr(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return SKV_ECUDA;
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_dev_ptr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_static_ws) != cudaSuccess || p == nullptr) return SKV_ECUDA;
    g_dev_ptr[dev] = p;
  }
  *out = g_dev_ptr[dev];
  return SKV_OK;
}

}  // namespace

extern "C" {

SKV_API skv_status attn_decode_static_ws(const skv_decode_args* args, skv_stream_t stream) {
  if (!args) return SKV_EINVAL;
  // Same validation and plan as attn_decode; only the scratch source differs.
  skv_decode_args a = *args;
  a.workspace = nullptr;
  a.workspace_bytes = 0;
  const size_t need = skv_decode_workspace_size(&a);
  if (need > kStaticWorkspaceBytes) return SKV_EWORKSPACE;
  if (need > 0) {
    void* p = nullptr;
    const skv_status st = static_ws_ptr(&p);
    if (st != SKV_OK) return st;
    a.workspace = p;
    a.workspace_bytes = kStaticWorkspaceBytes;
  }
  return attn_decode(&a, stream);
}

}  // extern "C"
