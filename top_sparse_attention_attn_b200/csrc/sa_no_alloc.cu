// sa_no_alloc.cu -- sa_bwd_no_alloc: the backward pass without a
// caller-supplied workspace, for callers that cannot allocate device memory.
//
// Some callers have no way to obtain device memory at the point where they
// run the backward: a plugin invoked by a host framework that owns every byte
// of device memory through its own pre-reserved pool and forbids allocation
// during execution, or a latency-critical loop where the implicit device
// synchronisation of cudaMalloc / cudaFree is not acceptable.  For them the
// scratch the backward needs (fp32 accumulators, rowsum(dO o O), a status
// word) lives in one fixed array in device memory, defined below.
//
// The array is part of the library's device image, so every GPU that loads
// the library holds kNoAllocScratchBytes of it until the process exits.  All
// calls share it: two calls whose work overlaps on the GPU (different streams,
// or different host threads on one device) race on it.  Each call overwrites
// and re-zeroes the parts it uses (sa_bwd clears its accumulators first).
#include <cuda_runtime.h>
#include <mutex>

#include "../../include/sparse_attn.h"

namespace {

constexpr size_t kNoAllocScratchBytes = 32u << 20;  // 32 MiB
constexpr int kMaxDevices = 64;

// Host code must not use this name as a device address: it is only a host-side
// stand-in; the device address comes from cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_no_alloc_scratch[kNoAllocScratchBytes];

std::mutex g_setup_mutex;
void* g_scratch_ptr[kMaxDevices] = {};

// Resolve the device address of the scratch array for the current device,
// once per device (with that device current).
sa_status scratch_for_current_device(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return SA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  if (!g_scratch_ptr[dev]) {
    void* ptr = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&ptr, g_no_alloc_scratch);
    if (e != cudaSuccess || !ptr) return SA_ERR_CUDA;
    g_scratch_ptr[dev] = ptr;
  }
  *out = g_scratch_ptr[dev];
  return SA_OK;
}

}  // namespace

extern "C" {

size_t sa_bwd_no_alloc_max_workspace(void) { return kNoAllocScratchBytes; }

sa_status sa_bwd_no_alloc(const sa_args* args, const sa_bwd_io* io, void* stream) {
  size_t need = 0;
  sa_status st = sa_bwd_get_workspace_size(args, &need);
  if (st != SA_OK) return st;
  if (need > kNoAllocScratchBytes) return SA_ERR_WORKSPACE;
  void* scratch = nullptr;
  st = scratch_for_current_device(&scratch);
  if (st != SA_OK) return st;
  return sa_bwd(args, io, scratch, kNoAllocScratchBytes, stream);
}

}  // extern "C"
