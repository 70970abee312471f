// sla_forward_noalloc: the forward pass for callers that cannot allocate
// device memory. Some host programs own every byte of GPU memory themselves
// (a plugin inside an inference server or game engine with a fixed memory
// pool, a statically planned embedded deployment) or must not call
// cudaMalloc once they are running, because it can synchronise the device and
// stall latency-critical work. Such callers still pass Q, K, V and O, but they
// have no way to supply the scratch workspace sla_forward needs.
//
// This entry point takes that scratch from one file-scope __device__ array of
// SLA_NOALLOC_WORKSPACE_BYTES. The array exists on every GPU that loads the
// library and stays resident until the process exits. Kernels need its device
// address, which host code obtains with cudaGetSymbolAddress (the array's name
// in host code is only a host-side stand-in); that lookup runs once per device,
// with that device current, on the first call made on it (or on the first
// sla_read_device_status(NULL, ...) there).
#include <mutex>

#include "sla_internal.cuh"

namespace {

static __device__ __align__(256) unsigned char g_noalloc_workspace[SLA_NOALLOC_WORKSPACE_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_mutex;
void* g_dev_ptr[kMaxDevices] = {};

}  // namespace

namespace sla {

// Device address of the static workspace on the current device (looked up once).
sla_status noalloc_workspace_address(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return SLA_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return SLA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_mutex);
  if (g_dev_ptr[dev] == nullptr) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_noalloc_workspace) != cudaSuccess || ptr == nullptr)
      return SLA_ERR_CUDA;
    g_dev_ptr[dev] = ptr;
  }
  *out = g_dev_ptr[dev];
  return SLA_OK;
}

}  // namespace sla

extern "C" sla_status sla_forward_noalloc(const void* Q, const void* K, const void* V, void* O,
                                          const sla_params* p, void* stream) {
  const sla_status st = sla_validate(p);
  if (st != SLA_OK) return st;
  if (sla_workspace_size(p) > size_t(SLA_NOALLOC_WORKSPACE_BYTES)) return SLA_ERR_WORKSPACE;
  void* ws = nullptr;
  const sla_status ws_st = sla::noalloc_workspace_address(&ws);
  if (ws_st != SLA_OK) return ws_st;
  // sla_forward clears the part of the workspace that must start at zero (the
  // device status word) and overwrites everything else it reads.
  return sla_forward(Q, K, V, O, p, ws, size_t(SLA_NOALLOC_WORKSPACE_BYTES), stream);
}
