// sa_qblock.h -- arguments of the query-stationary block kernels (forward, dQ pass).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "sa_device.cuh"

namespace sa {

// Most usable slots per work item the query-stationary block kernels hold.
constexpr int kQbMaxSlots = 256;

struct QbArgs {
  int layout, B, s_q, s_kv, Tq, Tkv, Hq, Hkv, G, dqk, dv, topk, ori_mask;
  long long wl, wr;
  float scale, scale_log2;
  const bf16* q;
  const bf16* d_o;      // dQ pass
  const int* ori_idx;
  const int* ori_len;
  const int* cu_q;
  const int* cu_kv;
  const float* sinks;   // forward
  bf16* o;              // forward output
  float* lse;           // forward output / dQ-pass input
  const float* delta;   // dQ pass
  bf16* dq;             // dQ-pass output
  int* status;
};

bool qb_path_built(int dqk, int dv);
cudaError_t launch_qb(const QbArgs& a, const void* k, const void* v, bool dq, cudaStream_t st);
// Forward on tcgen05 (64-row blocks, 16-head slices, scores held transposed in TMEM).
cudaError_t launch_bq_fwd(const QbArgs& a, const void* k, const void* v, cudaStream_t st);
// Inspection: the usable slots and row ranges of every unit as the block kernels see them.
cudaError_t launch_qb_debug_slots(const QbArgs& a, int4* rec, long long max_rec, int* n_rec, cudaStream_t st);

}  // namespace sa
