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
  int4* items;          // [max_work] work items {list, first entry, entries, 0}
  int* entries;         // [n_slots] token ids grouped by list
  int* work_count;      // [1]
  // bucketed index (small problems): bucket b = slots [b * kBucketSlots, ...) keeps
  // its own inverse index at entries + b * kBucketSlots, lists at bucket_off[b][L],
  // bucket_cnt[b][L] entries each
  int n_buckets;
  int* bucket_cnt;      // [n_buckets][n_lists]
  int* bucket_off;      // [n_buckets][n_lists]
  int* bucket_flag;     // [n_buckets]: the bucket held an index past its sequence
  int* status;          // status word (index bit), cleared before the index is built
};

struct KvArgs {
  int S, Hq, Hkv, G, RPT, TPT, nblk, n_lists, chunk_tokens, ori_mask;
  int nwin;
  long long wl, wr;
  float scale, scale_log2;
  const int4* items;    // [work_count] {list, first entry, entries, 0}
  const int* entries;
  const int* work_count;
  const float* lse;     // [Tq, Hq]
  const float* delta;   // [Tq, Hq]
  float* dk_acc;        // [Tkv, Hkv, DQK]
  float* dv_acc;        // [Tkv, Hkv, DV]
  float* dq_acc;        // [Tq, Hq, DQK] (dQ in this kernel) or null
  int* status;
  // row gather (G = 1, 2, 4): a tile packs TPT = 128 / G tokens with no padding
  // rows, copied row piece by row piece with cp.async instead of a TMA box per
  // token (TMA boxes must start on 8-row swizzle groups)
  int gather_rows, log2_G;
  const bf16* q;        // [Tq, Hq, DQK]
  const bf16* d_o;      // [Tq, Hq, DV]
  // bucketed mode (small problems): every CTA derives its work item from the
  // per-bucket index (items and work_count unused)
  int n_buckets;
  const int* bucket_cnt;  // [n_buckets][n_lists]
  const int* bucket_off;  // [n_buckets][n_lists]
  const int* bucket_flag; // [n_buckets]
};

// Bucketed index: buckets of 512 slots, each built by one CTA (512 threads) of
// the preparation launch; the KV kernel combines at most 32 of them, and a
// chunk's token ids stay in its shared memory.
constexpr int kBucketSlots = 512;
constexpr int kBucketMax = 32;
constexpr int kBucketMaxLists = 1024;
constexpr int kBucketMaxCells = 8192;  // n_buckets * n_lists
constexpr int kBucketMaxChunk = 512;

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

// One-launch preparation for small problems: CTAs [0, n_buckets) build the
// bucketed index; the others clear [zero, zero + 16 * zero_n16) (a range that
// must not hold Delta) and form Delta (rows of dv bf16); CTA 0 also clears the
// status word.
struct KvPrepArgs {
  int* status;
  float4* zero;
  long long zero_n16;
  const bf16* o;
  const bf16* d_o;
  float* delta;
  long long rows;
  int dv;
};

bool kv_path_built(int dqk, int dv);
int kv_bucket_count(long long n_slots);
bool kv_bucketed_fits(long long n_slots, int n_lists, int chunk);
cudaError_t launch_kv_prep_small(const KvIndexArgs& a, const KvPrepArgs& p, cudaStream_t st);
cudaError_t launch_kv_index(const KvIndexArgs& a, cudaStream_t st);
cudaError_t launch_kv_bwd(const KvLaunch& L, bool with_dq, cudaStream_t st);
// Inspection walk over the work items (grid max_work), after the index is built.
cudaError_t launch_kv_debug_walk(const KvArgs& a, long long max_work, int4* rec, long long max_rec, int* n_rec,
                                 cudaStream_t st);

}  // namespace sa
