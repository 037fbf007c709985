// sa_kv_bwd.h -- arguments of the key-stationary backward and its inverse index.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "sa_device.cuh"

namespace sa {

// Inverse index over block selections (block size 64, BSND, S_q == S_kv).
struct KvIndexArgs {
  const int* ori_idx;   // [Tq, Hkv, topk]
  const int* ori_len;   // [Tq, Hkv] or null
  long long n_slots;    // Tq * Hkv * topk
  int topk, Hkv, S, nblk, n_lists, chunk_tokens, ori_mask;
  int nwin, win_tokens;  // lists are keyed by (batch, token window, kv-head, block)
  long long wl, wr;
  int* counts;          // [n_lists]
  int* cursor;          // [n_lists]
  int* list_off;        // [n_lists + 1]
  int* chunk_off;       // [n_lists + 1]
  int* entries;         // [n_slots] token ids grouped by list
  int* work_count;      // [1]
};

struct KvArgs {
  int S, Hq, Hkv, G, RPT, TPT, nblk, n_lists, chunk_tokens, ori_mask;
  int nwin;
  long long wl, wr;
  float scale, scale_log2;
  const int* list_off;
  const int* chunk_off;
  const int* entries;
  const int* work_count;
  const float* lse;     // [Tq, Hq]
  const float* delta;   // [Tq, Hq]
  float* dk_acc;        // [Tkv, Hkv, DQK]
  float* dv_acc;        // [Tkv, Hkv, DV]
  float* dq_acc;        // [Tq, Hq, DQK] (dQ in this kernel) or null
  int* status;
};

struct KvLaunch {
  KvArgs args;
  const void* q;
  const void* d_o;
  const void* k;
  const void* v;
  long long Tq, Tkv;
  int dqk, dv;
  long long max_work;   // grid size: an upper bound on the work items
};

bool kv_path_built(int dqk, int dv);
cudaError_t launch_kv_index(const KvIndexArgs& a, cudaStream_t st);
cudaError_t launch_kv_bwd(const KvLaunch& L, bool with_dq, cudaStream_t st);

}  // namespace sa
