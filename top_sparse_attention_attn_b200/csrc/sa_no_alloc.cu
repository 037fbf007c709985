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
// the library holds kNoAllocScratchBytes of it until the process exits.  The
// first call in a CUDA context resolves the array's address (make it before
// any stream capture); sa_bwd_no_alloc_read_status reads its status word.  All
// calls share it: two calls whose work overlaps on the GPU (different streams,
// or different host threads on one device) race on it.  Each call overwrites
// and re-zeroes the parts it uses (sa_bwd clears its accumulators first).
#include <cuda.h>
#include <cuda_runtime.h>
#include <mutex>

#include "../../include/sparse_attn.h"

namespace {

constexpr size_t kNoAllocScratchBytes = 32u << 20;  // 32 MiB
constexpr int kMaxContexts = 64;

// Host code must not use this name as a device address: it is only a host-side
// stand-in; the device address comes from cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_no_alloc_scratch[kNoAllocScratchBytes];

// The array's address is resolved once per CUDA context (the device's primary
// context for runtime users; a context created after cudaDeviceReset, or one a
// driver-API caller made current, gets its own entry), with that context current.
struct ScratchEntry {
  CUcontext ctx;
  void* ptr;
};
std::mutex g_setup_mutex;
ScratchEntry g_scratch[kMaxContexts] = {};
int g_n_scratch = 0;

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
CtxGetCurrentFn ctx_get_current() {
  static CtxGetCurrentFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<CtxGetCurrentFn>(f);
  });
  return fn;
}

// The scratch array's device address in the current context.
sa_status scratch_for_current_context(void** out) {
  CtxGetCurrentFn get = ctx_get_current();
  if (!get) return SA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  CUcontext ctx = nullptr;
  if (get(&ctx) != CUDA_SUCCESS) return SA_ERR_CUDA;
  if (ctx) {
    for (int i = 0; i < g_n_scratch; ++i)
      if (g_scratch[i].ctx == ctx) {
        *out = g_scratch[i].ptr;
        return SA_OK;
      }
  }
  // first call in this context: resolve the address (this also makes the
  // runtime's primary context current when none was)
  void* ptr = nullptr;
  cudaError_t e = cudaGetSymbolAddress(&ptr, g_no_alloc_scratch);
  if (e != cudaSuccess || !ptr) return SA_ERR_CUDA;
  if (get(&ctx) != CUDA_SUCCESS || !ctx) return SA_ERR_CUDA;
  if (g_n_scratch < kMaxContexts) g_scratch[g_n_scratch++] = ScratchEntry{ctx, ptr};
  *out = ptr;
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
  st = scratch_for_current_context(&scratch);
  if (st != SA_OK) return st;
  return sa_bwd(args, io, scratch, kNoAllocScratchBytes, stream);
}

sa_status sa_bwd_no_alloc_read_status(void* stream) {
  void* scratch = nullptr;
  sa_status st = scratch_for_current_context(&scratch);
  if (st != SA_OK) return st;
  return sa_read_status(scratch, kNoAllocScratchBytes, stream);
}

}  // extern "C"
