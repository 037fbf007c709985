// sa_launch.h -- host-side launchers behind the C ABI (internal).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>

#include "sa_device.cuh"

namespace sa {

// Pointers the backward kernels write (device).
struct BwdOut {
  bf16* dq;
  float* dk_acc;    // [Tkv, Hkv, dqk] fp32 (dKV when shared)
  float* dv_acc;    // [Tkv, Hkv, dv] fp32 (unused when shared)
  float* dcmp_acc;  // [Tcmp, Hkv, dqk] fp32
  float* dsinks;    // [Hq] fp32 (accumulated)
};

// Process-wide benchmarking hooks (see sa_set_timing_events).
extern cudaEvent_t g_ev_begin, g_ev_end;
extern long long g_launches;
inline void count_launch() { __atomic_fetch_add(&g_launches, 1, __ATOMIC_RELAXED); }
inline void mark_begin(cudaStream_t st) { if (g_ev_begin && g_ev_end) cudaEventRecord(g_ev_begin, st); }
inline void mark_end(cudaStream_t st) { if (g_ev_begin && g_ev_end) cudaEventRecord(g_ev_end, st); }

// Returns false when no kernel is built for (dqk, dv, shared).
bool kernels_built(int dqk, int dv, bool shared);

cudaError_t launch_fwd(const Prob& p, bf16* o, float* lse, cudaStream_t st);
cudaError_t launch_delta(const bf16* o, const bf16* d_o, float* delta, long long rows, int dv,
                         cudaStream_t st);
cudaError_t launch_bwd(const Prob& p, const bf16* o, const bf16* d_o, const float* lse,
                       const float* delta, const BwdOut& out, cudaStream_t st);
cudaError_t launch_to_bf16(const float* src, bf16* dst, long long n, cudaStream_t st);
cudaError_t launch_check(const Prob& p, cudaStream_t st);
cudaError_t launch_debug_resolve(const Prob& p, int* rows, int* counts, int max_rows,
                                 cudaStream_t st);

}  // namespace sa
