// sa_launch.h -- host-side launchers behind the C ABI (internal).
#pragma once

#include <cuda.h>
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
enum { kTimeFwd = 0, kTimeBwdKV = 1, kTimeBwdDQ = 2 };
extern cudaEvent_t g_ev_begin, g_ev_end;
extern int g_ev_which;
extern long long g_launches;
inline void count_launch() { __atomic_fetch_add(&g_launches, 1, __ATOMIC_RELAXED); }
inline void mark_begin(cudaStream_t st, int which) {
  if (g_ev_begin && g_ev_end && which == g_ev_which) cudaEventRecord(g_ev_begin, st);
}
inline void mark_end(cudaStream_t st, int which) {
  if (g_ev_begin && g_ev_end && which == g_ev_which) cudaEventRecord(g_ev_end, st);
}

// Launch with programmatic stream serialization (the kernel calls pdl_wait()
// before it reads or writes global memory); captures into CUDA graphs as a
// programmatic edge.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), unsigned grid, unsigned block, size_t smem, cudaStream_t st,
                       Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(block);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}

// launch_pdl with thread-block clusters of `cluster_x` consecutive CTAs (grid a
// multiple of cluster_x).
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl_cluster(void (*kernel)(KArgs...), unsigned grid, unsigned block, size_t smem,
                               cudaStream_t st, unsigned cluster_x, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(block);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = cluster_x;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}

// TMA tensor map over a [rows][cols] bf16 matrix (row stride in bytes), boxes
// of box_rows x 64 columns, 128-byte swizzle, zero fill out of range.
bool make_tmap_bf16(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols, uint64_t row_stride_bytes,
                    uint32_t box_rows);

// Returns false when no kernel is built for (dqk, dv, shared).
bool kernels_built(int dqk, int dv, bool shared);

cudaError_t launch_fwd(const Prob& p, bf16* o, float* lse, cudaStream_t st);
cudaError_t launch_bwd_dq(const Prob& p, const bf16* d_o, const float* lse, const float* delta,
                          const BwdOut& out, cudaStream_t st);
cudaError_t launch_delta(const bf16* o, const bf16* d_o, float* delta, long long rows, int dv,
                         cudaStream_t st, bool f16 = false);
cudaError_t launch_bwd(const Prob& p, const bf16* o, const bf16* d_o, const float* lse,
                       const float* delta, const BwdOut& out, cudaStream_t st);
// fp32 -> the 2-byte output type (bf16, or fp16 with f16); n a multiple of 8.
cudaError_t launch_to_bf16(const float* src, bf16* dst, long long n, cudaStream_t st, bool f16 = false);
// Token-level backward over one shared KV head (d 576 / 512) on tcgen05: dQ to
// bf16 directly, dKV (dCmpKv) into the fp32 accumulators, dSinks accumulated.
bool tk_path_built(int dqk, int dv, int shared, int G);
cudaError_t launch_tk_bwd(const Prob& p, const float* lse, const float* delta, const bf16* d_o, const BwdOut& out,
                          cudaStream_t st);
cudaError_t launch_tk_fwd(const Prob& p, bf16* o, float* lse, bool pair, cudaStream_t st);
// Up to four fp32 -> bf16 conversions in one launch (each n a multiple of 8).
struct Cvt {
  const float* src;
  bf16* dst;
  long long n;
};
cudaError_t launch_to_bf16_multi(const Cvt* jobs, int njobs, cudaStream_t st, bool f16 = false);
cudaError_t launch_check(const Prob& p, cudaStream_t st);
// The lightning indexer's KL-loss backward (one CTA per token).
struct IxArgs {
  int layout, B, s_q, s_kv, Tq, Tkv, H, D, topk;
  const bf16* q;        // [Tq, H, D]
  const bf16* k;        // [Tkv, D]
  const float* w;       // [Tq, H]
  const int* idx;       // [Tq, topk]
  const int* topk_len;  // [Tq] or null
  const float* p;       // [Tq, topk]
  const int *cu_q, *cu_kv;
  float* loss;          // [Tq] or null
  bf16* dq;             // [Tq, H, D]
  float* dk_acc;        // [Tkv, D] fp32, zeroed by the caller
  float* dw;            // [Tq, H]
  int* status;
};
bool ix_built(int H, int D);
cudaError_t launch_indexer_kl(const IxArgs& a, cudaStream_t st);
// SoftmaxL1Norm outputs: ori_out [Tq, Hkv, topk] and / or cmp_out [Tq, Hkv,
// cmp_topk] fp32 (either may be null), from the forward's lse.
cudaError_t launch_softmax_l1norm(const Prob& p, const float* lse, float* ori_out, float* cmp_out, cudaStream_t st);
cudaError_t launch_debug_resolve(const Prob& p, int* rows, int* counts, int max_rows,
                                 cudaStream_t st);

}  // namespace sa
