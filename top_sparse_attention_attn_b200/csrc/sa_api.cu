// sa_api.cu -- the extern "C" entry points declared in include/sparse_attn.h:
// host-side argument validation, workspace sizing and kernel dispatch.
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>
#include <string.h>

#include "../../include/sparse_attn.h"
#include "sa_device.cuh"
#include "sa_kv_bwd.h"
#include "sa_launch.h"
#include "sa_qblock.h"

namespace {

using sa::bf16;

constexpr size_t kAlign = 256;
// BAND windows wider than any sequence change nothing; clamping keeps the
// kernels' 64-bit window arithmetic far from overflow.
constexpr long long kWinClamp = 1ll << 40;
long long clamp_win(long long w) { return w < kWinClamp ? w : kWinClamp; }
size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

struct Sizes {
  long long Tq, Tkv, Tcmp;
};

// Compressed rows take part when cmp indices are given (SCFA: Gather(cmpKv,
// topkIndices)), or when a compressed KV comes without indices and a compression
// ratio above 1 (CFA: concat(oriKv, cmpKv), every compressed row);
// SparseFlashMlaGrad "Computation formula" Stage 1.
bool cfa(const sa_args* a) { return a->cmp_topk == 0 && a->cmp_kv != nullptr && a->cmp_ratio > 1; }
bool has_cmp(const sa_args* a) { return a->cmp_topk > 0 || cfa(a); }
// sequsedQ / sequsedOriKv / sequsedCmpKv given (the block kernels do not take them)
bool has_used(const sa_args* a) { return a->seqused_q || a->seqused_kv || a->seqused_cmp; }
// A paged KV cache (block_table): the forward only
bool paged(const sa_args* a) { return a->block_table != nullptr; }

Sizes sizes_of(const sa_args* a) {
  Sizes s;
  if (a->layout_q == SA_LAYOUT_BSND) {
    s.Tq = (long long)a->batch * a->s_q;
    s.Tkv = paged(a) ? (long long)a->t_kv : (long long)a->batch * a->s_kv;  // a paged cache has t_kv rows
    s.Tcmp = has_cmp(a) ? (long long)a->batch * (a->s_kv / (a->cmp_ratio > 0 ? a->cmp_ratio : 1)) : 0;
  } else {
    s.Tq = a->t_q;
    s.Tkv = a->t_kv;
    s.Tcmp = has_cmp(a) ? a->t_cmp : 0;
  }
  return s;
}

sa_status validate(const sa_args* a) {
  if (!a) return SA_ERR_NULLPTR;
  if (a->dtype != SA_DTYPE_BF16 && a->dtype != SA_DTYPE_FP16) return SA_ERR_PARAM;
  if (a->layout_q != SA_LAYOUT_BSND && a->layout_q != SA_LAYOUT_TND) return SA_ERR_PARAM;
  if (a->layout_kv != SA_LAYOUT_BSND && a->layout_kv != SA_LAYOUT_TND) return SA_ERR_PARAM;
  if (a->layout_q != a->layout_kv) return SA_ERR_UNSUPPORTED;  // mixed layouts are not built
  if (a->batch < 0) return SA_ERR_PARAM;
  if (a->layout_q == SA_LAYOUT_BSND) {
    if (a->s_q < 0 || a->s_kv < 0) return SA_ERR_PARAM;
  } else {
    if (a->t_q < 0 || a->t_kv < 0 || a->t_cmp < 0) return SA_ERR_PARAM;
  }
  if (a->n_heads_q < 1 || a->n_heads_kv < 1 || a->n_heads_q % a->n_heads_kv) return SA_ERR_PARAM;
  if (a->d_qk < 16 || a->d_v < 16 || a->d_qk % 16 || a->d_v % 16) return SA_ERR_PARAM;
  if (a->d_qk > 576 || a->d_v > 512) return SA_ERR_PARAM;
  if (a->kv_shared && a->d_v > a->d_qk) return SA_ERR_PARAM;
  if (a->block_size < 1 || (a->block_size > sa::kTileRows && a->block_size % sa::kTileRows)) return SA_ERR_PARAM;
  if (a->topk < 0 || a->cmp_topk < 0) return SA_ERR_PARAM;
  if (a->cmp_ratio < 1) return SA_ERR_PARAM;
  if (a->ori_mask_mode < SA_MASK_NONE || a->ori_mask_mode > SA_MASK_BAND) return SA_ERR_PARAM;
  if (a->cmp_mask_mode != SA_MASK_NONE && a->cmp_mask_mode != SA_MASK_CAUSAL) return SA_ERR_PARAM;
  if (a->ori_mask_mode == SA_MASK_BAND && (a->ori_win_left < 0 || a->ori_win_right < 0)) return SA_ERR_PARAM;
  if (!isfinite(a->scale)) return SA_ERR_PARAM;
  if (paged(a)) {
    if (a->layout_q != SA_LAYOUT_BSND) return SA_ERR_UNSUPPORTED;
    if (a->page_size < 1 || a->max_pages < 1 || a->t_kv < 1) return SA_ERR_PARAM;
    if ((long long)a->max_pages * a->page_size < a->s_kv) return SA_ERR_PARAM;
    if (has_cmp(a)) return SA_ERR_UNSUPPORTED;
  }
  Sizes s = sizes_of(a);
  if (s.Tq >= (1ll << 30) || s.Tkv >= (1ll << 30) || s.Tcmp >= (1ll << 30)) return SA_ERR_PARAM;
  const int G = a->n_heads_q / a->n_heads_kv;
  if (s.Tq * a->n_heads_kv * ((G + 15) / 16) >= (1ll << 31)) return SA_ERR_PARAM;
  // pointers
  if (s.Tq > 0) {
    if (!a->q) return SA_ERR_NULLPTR;
    if (a->kv_shared ? !a->kv : (!a->k || !a->v)) return SA_ERR_NULLPTR;
    if (a->topk > 0 && !a->ori_idx) return SA_ERR_NULLPTR;
    if (a->cmp_topk > 0 && (!a->cmp_kv || !a->cmp_idx)) return SA_ERR_NULLPTR;
    if (a->layout_q == SA_LAYOUT_TND) {
      if (!a->cu_seqlens_q || !a->cu_seqlens_kv) return SA_ERR_NULLPTR;
      if (has_cmp(a) && !a->cu_seqlens_cmp) return SA_ERR_NULLPTR;
      if (a->batch < 1) return SA_ERR_PARAM;
    }
  }
  // combinations that are valid on the pages but not built here
  if (has_cmp(a) && !a->kv_shared) return SA_ERR_UNSUPPORTED;
  if (!sa::kernels_built(a->d_qk, a->d_v, a->kv_shared != 0)) return SA_ERR_UNSUPPORTED;
  return SA_OK;
}

sa::Prob make_prob(const sa_args* a, int* status) {
  sa::Prob p;
  memset(&p, 0, sizeof(p));
  Sizes s = sizes_of(a);
  p.layout = a->layout_q;
  p.B = a->batch;
  p.s_q = a->s_q;
  p.s_kv = a->s_kv;
  p.Tq = (int)s.Tq;
  p.Tkv = (int)s.Tkv;
  p.Tcmp = (int)s.Tcmp;
  p.Hq = a->n_heads_q;
  p.Hkv = a->n_heads_kv;
  p.G = a->n_heads_q / a->n_heads_kv;
  p.dqk = a->d_qk;
  p.dv = a->d_v;
  p.shared = a->kv_shared ? 1 : 0;
  p.bs = a->block_size;
  p.topk = a->topk;
  p.cmp_topk = a->cmp_topk;
  p.ratio = a->cmp_ratio;
  p.ori_mask = a->ori_mask_mode;
  p.cmp_mask = a->cmp_mask_mode;
  p.wl = clamp_win(a->ori_win_left);
  p.wr = clamp_win(a->ori_win_right);
  p.scale = a->scale;
  p.scale_log2 = a->scale * 1.4426950408889634f;
  p.q = static_cast<const bf16*>(a->q);
  if (a->kv_shared) {
    p.k = static_cast<const bf16*>(a->kv);
    p.v = static_cast<const bf16*>(a->kv);
  } else {
    p.k = static_cast<const bf16*>(a->k);
    p.v = static_cast<const bf16*>(a->v);
  }
  p.cmpk = has_cmp(a) ? static_cast<const bf16*>(a->cmp_kv) : nullptr;
  p.ori_idx = a->topk > 0 ? a->ori_idx : nullptr;
  p.cmp_idx = a->cmp_topk > 0 ? a->cmp_idx : nullptr;
  p.cu_q = a->cu_seqlens_q;
  p.cu_kv = a->cu_seqlens_kv;
  p.cu_cmp = a->cu_seqlens_cmp;
  p.ori_len = a->topk > 0 ? a->ori_topk_len : nullptr;
  p.cmp_len = a->cmp_topk > 0 ? a->cmp_topk_len : nullptr;
  p.sinks = a->sinks;
  p.used_q = a->seqused_q;
  p.used_kv = a->seqused_kv;
  p.used_cmp = has_cmp(a) ? a->seqused_cmp : nullptr;
  p.page_table = a->block_table;
  p.page_size = a->page_size;
  p.max_pages = a->max_pages;
  p.status = status;
  p.f16 = a->dtype == SA_DTYPE_FP16 ? 1 : 0;
  return p;
}

bool aligned16(const void* ptr) { return ((uintptr_t)ptr & 15u) == 0; }

sa_status check_tensor_alignment(const sa_args* a) {
  if (!aligned16(a->q) || !aligned16(a->k) || !aligned16(a->v) || !aligned16(a->kv) ||
      !aligned16(a->cmp_kv))
    return SA_ERR_PARAM;
  return SA_OK;
}

// The key-stationary backward applies to block-level BSND selection with
// 64-row blocks, equal query / key lengths, separate K / V and no sinks.
bool use_kv_path(const sa_args* a) {
  if (a->flags & SA_FLAG_QUERY_STATIONARY_BWD) return false;
  const int G = a->n_heads_q / a->n_heads_kv;
  return a->dtype == SA_DTYPE_BF16 && a->layout_q == SA_LAYOUT_BSND && a->topk > 0 && a->block_size == 64 &&
         a->s_q == a->s_kv && !a->kv_shared && !has_cmp(a) && !has_used(a) && !paged(a) && a->sinks == nullptr &&
         G <= 128 && sa::kv_path_built(a->d_qk, a->d_v);
}

// Query-stationary block kernels (TMA-fed): 64-row blocks, separate K / V, no compressed KV.
bool use_qb_path(const sa_args* a) {
  return a->dtype == SA_DTYPE_BF16 && a->topk > 0 && a->topk <= sa::kQbMaxSlots && a->block_size == 64 &&
         !a->kv_shared && !has_cmp(a) && !has_used(a) && !paged(a) && sa::qb_path_built(a->d_qk, a->d_v);
}

// SA_FLAG_DQ_SEPARATE applies only where the query-stationary block kernels do
// (they hold at most kQbMaxSlots usable slots per unit); elsewhere the
// key-stationary kernel forms dQ with atomics as by default.
bool dq_separate(const sa_args* a) { return (a->flags & SA_FLAG_DQ_SEPARATE) && use_qb_path(a); }

sa::QbArgs make_qb_args(const sa_args* a, int* status) {
  sa::QbArgs q;
  memset(&q, 0, sizeof(q));
  Sizes s = sizes_of(a);
  q.layout = a->layout_q;
  q.B = a->batch;
  q.s_q = a->s_q;
  q.s_kv = a->s_kv;
  q.Tq = (int)s.Tq;
  q.Tkv = (int)s.Tkv;
  q.Hq = a->n_heads_q;
  q.Hkv = a->n_heads_kv;
  q.G = a->n_heads_q / a->n_heads_kv;
  q.dqk = a->d_qk;
  q.dv = a->d_v;
  q.topk = a->topk;
  q.ori_mask = a->ori_mask_mode;
  q.wl = clamp_win(a->ori_win_left);
  q.wr = clamp_win(a->ori_win_right);
  q.scale = a->scale;
  q.scale_log2 = a->scale * 1.4426950408889634f;
  q.q = static_cast<const bf16*>(a->q);
  q.ori_idx = a->ori_idx;
  q.ori_len = a->ori_topk_len;
  q.cu_q = a->cu_seqlens_q;
  q.cu_kv = a->cu_seqlens_kv;
  q.sinks = a->sinks;
  q.status = status;
  return q;
}

struct KvGeom {
  int RPT, TPT, nblk, n_lists, chunk, nwin, win_tokens;
  long long n_slots, max_work;
};

KvGeom kv_geometry(const sa_args* a) {
  KvGeom k;
  const int G = a->n_heads_q / a->n_heads_kv;
  // rows per token in a 128-row tile: G itself for G = 1, 2, 4 (gathered row by
  // row), else G rounded up to whole 8-row swizzle groups (a TMA box per token)
  const bool with_dq = !dq_separate(a);  // the gather runs in the dQ role
  k.RPT = with_dq && (G == 1 || G == 2 || G == 4) ? G : (G + 7) / 8 * 8;
  k.TPT = 128 / k.RPT;
  k.nblk = (a->s_kv + 63) / 64;
  // token windows: with dQ added by atomics, a window's fp32 dQ rows (~24 MB) stay
  // in L2 while the CTAs of that window run
  // Windows pay off only when a window's dQ rows fit in L2 (<= 48 MB) while each
  // (window, block) cell still holds enough tokens (>= 128 on average) that the
  // extra dK / dV flushes stay cheap; otherwise one window spans the sequence.
  k.win_tokens = a->s_q > 0 ? a->s_q : 1;
  if (with_dq && a->topk > 0) {
    long long fit = (48ll << 20) / ((long long)a->n_heads_q * a->d_qk * 4);
    fit = fit / 64 * 64;
    const long long need = 128ll * k.nblk / a->topk;
    if (fit >= 64 && fit >= need && fit < k.win_tokens) k.win_tokens = (int)fit;
  }
  k.nwin = (a->s_q + k.win_tokens - 1) / k.win_tokens;
  if (k.nwin < 1) k.nwin = 1;
  k.n_lists = a->batch * k.nwin * a->n_heads_kv * k.nblk;
  k.n_slots = (long long)a->batch * a->s_q * a->n_heads_kv * a->topk;
  // chunk of tokens per CTA: ~4 work items per SM, at most 512 tokens.  A problem
  // too small for that gets one wave of CTAs (about one item per SM) instead:
  // latency bounds it, and each extra chunk of a block costs one more dK / dV flush.
  long long want = (k.n_slots + 148 * 4 - 1) / (148 * 4);
  long long lo = k.TPT, hi = (512 / k.TPT) * k.TPT;
  if (want < lo) want = (k.n_slots + 147) / 148;
  if (want < lo) want = lo;
  if (want > hi) want = hi;
  want = (want + k.TPT - 1) / k.TPT * k.TPT;
  k.chunk = (int)want;
  k.max_work = (k.n_slots + k.chunk - 1) / k.chunk + k.n_lists;
  return k;
}

// Workspace: [status word][delta][dK or dKV acc][dV acc][dCmp acc]
//            + key-stationary path: [dQ acc][counts][cursor] | [list_off][items][work][entries]
//              [bucket counts][bucket offsets][bucket flags]
// Everything before `zero_end` is cleared at the start of each call with one memset
// (the bucketed preparation launch clears it instead).
struct BwdWs {
  size_t status, delta, dk, dv, dcmp;
  size_t dq, counts, cursor, list_off, items, work, entries, bucket_cnt, bucket_off, bucket_flag;
  size_t zero_end, total;
};

// Small key-stationary problems take the bucketed index (one preparation launch).
bool kv_bucketed(const sa_args* a, const KvGeom& k) { return sa::kv_bucketed_fits(k.n_slots, k.n_lists, k.chunk); }

BwdWs bwd_ws_layout(const sa_args* a) {
  Sizes s = sizes_of(a);
  BwdWs w;
  memset(&w, 0, sizeof(w));
  size_t off = 0;
  w.status = off;
  off += kAlign;
  w.delta = off;
  off += align_up((size_t)s.Tq * a->n_heads_q * sizeof(float));
  w.dk = off;
  off += align_up((size_t)s.Tkv * a->n_heads_kv * a->d_qk * sizeof(float));
  w.dv = off;
  if (!a->kv_shared) off += align_up((size_t)s.Tkv * a->n_heads_kv * a->d_v * sizeof(float));
  w.dcmp = off;
  off += align_up((size_t)s.Tcmp * a->n_heads_kv * a->d_qk * sizeof(float));
  if (use_kv_path(a)) {
    KvGeom k = kv_geometry(a);
    if (!dq_separate(a)) {
      w.dq = off;
      off += align_up((size_t)s.Tq * a->n_heads_q * a->d_qk * sizeof(float));
    }
    w.counts = off;
    off += align_up(sizeof(int) * k.n_lists);
    w.cursor = off;
    off += align_up(sizeof(int) * k.n_lists);
    w.zero_end = off;
    w.list_off = off;
    off += align_up(sizeof(int) * (k.n_lists + 1));
    w.items = off;
    off += align_up(sizeof(int4) * (size_t)k.max_work);
    w.work = off;
    off += kAlign;
    w.entries = off;
    off += align_up(sizeof(int) * (size_t)k.n_slots);
    if (kv_bucketed(a, k)) {
      const size_t nb = (size_t)sa::kv_bucket_count(k.n_slots);
      const size_t cells = nb * k.n_lists;
      w.bucket_cnt = off;
      off += align_up(sizeof(int) * cells);
      w.bucket_off = off;
      off += align_up(sizeof(int) * cells);
      w.bucket_flag = off;
      off += align_up(sizeof(int) * nb);
    }
  } else {
    w.zero_end = off;
  }
  w.total = off;
  return w;
}

sa_status cuda_status(cudaError_t e) { return e == cudaSuccess ? SA_OK : SA_ERR_CUDA; }

// Status word bits -> sa_status (the first that applies).
sa_status status_of_bits(int bits) {
  if (bits & sa::kStatusTimeout) return SA_ERR_TIMEOUT;
  if (bits & sa::kStatusIndexRange) return SA_ERR_INDEX;
  if (bits & sa::kStatusSmemAlign) return SA_ERR_CUDA;
  return SA_OK;
}

// SA_FLAG_CHECK: validate every usable index on the device, synchronously.
sa_status run_check(const sa_args* a, int* status, cudaStream_t st) {
  sa::Prob p = make_prob(a, status);
  if (cudaMemsetAsync(status, 0, sizeof(int), st) != cudaSuccess) return SA_ERR_CUDA;
  if (sa::launch_check(p, st) != cudaSuccess) return SA_ERR_CUDA;
  int host = 0;
  if (cudaMemcpyAsync(&host, status, sizeof(int), cudaMemcpyDeviceToHost, st) != cudaSuccess) return SA_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return SA_ERR_CUDA;
  return (host & sa::kStatusIndexRange) ? SA_ERR_INDEX : SA_OK;
}

// Kernel choices (sa_plan reports them; sa_fwd / sa_bwd dispatch on them).
bool tk_path(const sa_args* a) {
  // the row gathers need at least one KV row to point at (an empty KV takes the generic path)
  return a->dtype == SA_DTYPE_BF16 && sa::tk_path_built(a->d_qk, a->d_v, a->kv_shared, a->n_heads_q / a->n_heads_kv) &&
         sizes_of(a).Tkv >= 1;
}

int32_t fwd_choice(const sa_args* a) {
  if (use_qb_path(a)) return (a->flags & SA_FLAG_FWD_BLOCK_TC) ? SA_KERNEL_FWD_BLOCK_TC : SA_KERNEL_FWD_BLOCK;
  if (tk_path(a)) return SA_KERNEL_FWD_TOKEN_TC;
  return SA_KERNEL_FWD_GENERIC;
}

int32_t bwd_choice(const sa_args* a) {
  if (use_kv_path(a)) return dq_separate(a) ? SA_KERNEL_BWD_KEY_STATIONARY_DQ_PASS : SA_KERNEL_BWD_KEY_STATIONARY;
  if (tk_path(a) && !(a->flags & SA_FLAG_QUERY_STATIONARY_BWD)) return SA_KERNEL_BWD_TOKEN_TC;
  return SA_KERNEL_BWD_GENERIC;
}

// The key-stationary inverse index of one backward call, built into the workspace
// exactly as sa_bwd builds it: the bucketed preparation launch (which also clears
// the accumulators and, when o / d_o are given, forms Delta), or a memset of
// [0, zero_end) then the count / scan / fill launches.
struct KvIndexBuild {
  KvGeom k;
  sa::KvIndexArgs ia;
  bool bucketed;
};

sa_status build_kv_index(const sa_args* args, const BwdWs& w, char* base, const void* o, const void* d_o,
                         cudaStream_t cs, KvIndexBuild* out) {
  Sizes s = sizes_of(args);
  KvIndexBuild& r = *out;
  memset(&r, 0, sizeof(r));
  r.k = kv_geometry(args);
  r.bucketed = kv_bucketed(args, r.k);
  int* status = reinterpret_cast<int*>(base + w.status);
  float* delta = reinterpret_cast<float*>(base + w.delta);
  sa::KvIndexArgs& ia = r.ia;
  ia.ori_idx = args->ori_idx;
  ia.ori_len = args->ori_topk_len;
  ia.n_slots = r.k.n_slots;
  ia.topk = args->topk;
  ia.Hkv = args->n_heads_kv;
  ia.S = args->s_q;
  ia.nblk = r.k.nblk;
  ia.n_lists = r.k.n_lists;
  ia.nwin = r.k.nwin;
  ia.win_tokens = r.k.win_tokens;
  ia.chunk_tokens = r.k.chunk;
  ia.ori_mask = args->ori_mask_mode;
  ia.wl = clamp_win(args->ori_win_left);
  ia.wr = clamp_win(args->ori_win_right);
  ia.counts = reinterpret_cast<int*>(base + w.counts);
  ia.cursor = reinterpret_cast<int*>(base + w.cursor);
  ia.list_off = reinterpret_cast<int*>(base + w.list_off);
  ia.items = reinterpret_cast<int4*>(base + w.items);
  ia.entries = reinterpret_cast<int*>(base + w.entries);
  ia.work_count = reinterpret_cast<int*>(base + w.work);
  ia.status = status;
  if (r.bucketed) {
    ia.n_buckets = sa::kv_bucket_count(r.k.n_slots);
    ia.bucket_cnt = reinterpret_cast<int*>(base + w.bucket_cnt);
    ia.bucket_off = reinterpret_cast<int*>(base + w.bucket_off);
    ia.bucket_flag = reinterpret_cast<int*>(base + w.bucket_flag);
    sa::KvPrepArgs pa;
    // the accumulators and counters after Delta (Delta is formed in the same launch)
    pa.status = status;
    pa.zero = reinterpret_cast<float4*>(base + w.dk);
    pa.zero_n16 = (long long)((w.zero_end - w.dk) / 16);
    pa.o = static_cast<const bf16*>(o);
    pa.d_o = static_cast<const bf16*>(d_o);
    pa.delta = delta;
    pa.rows = (o && d_o) ? s.Tq * args->n_heads_q : 0;
    pa.dv = args->d_v;
    return cuda_status(sa::launch_kv_prep_small(ia, pa, cs));
  }
  // zero the accumulators and the index counters (one memset), then Delta
  if (cudaMemsetAsync(base, 0, w.zero_end, cs) != cudaSuccess) return SA_ERR_CUDA;
  if (o && d_o) {
    if (sa::launch_delta(static_cast<const bf16*>(o), static_cast<const bf16*>(d_o), delta, s.Tq * args->n_heads_q,
                         args->d_v, cs) != cudaSuccess)
      return SA_ERR_CUDA;
  }
  return cuda_status(sa::launch_kv_index(ia, cs));
}

// The key-stationary kernel's arguments for an index built by build_kv_index.
sa::KvArgs kv_args(const sa_args* args, const KvIndexBuild& r, const BwdWs& w, char* base, const void* d_o,
                   const float* lse, float* dk_acc, float* dv_acc) {
  sa::KvArgs ka;
  memset(&ka, 0, sizeof(ka));
  const KvGeom& k = r.k;
  ka.S = args->s_q;
  ka.Hq = args->n_heads_q;
  ka.Hkv = args->n_heads_kv;
  ka.G = args->n_heads_q / args->n_heads_kv;
  ka.RPT = k.RPT;
  ka.TPT = k.TPT;
  ka.gather_rows = k.RPT == ka.G ? (k.RPT < 8 ? 1 : 0) : 0;
  ka.log2_G = ka.G == 4 ? 2 : (ka.G == 2 ? 1 : 0);
  ka.q = static_cast<const bf16*>(args->q);
  ka.d_o = static_cast<const bf16*>(d_o);
  ka.nblk = k.nblk;
  ka.n_lists = k.n_lists;
  ka.nwin = k.nwin;
  ka.chunk_tokens = k.chunk;
  ka.ori_mask = args->ori_mask_mode;
  ka.wl = clamp_win(args->ori_win_left);
  ka.wr = clamp_win(args->ori_win_right);
  ka.scale = args->scale;
  ka.scale_log2 = args->scale * 1.4426950408889634f;
  ka.items = r.ia.items;
  ka.entries = r.ia.entries;
  ka.work_count = r.ia.work_count;
  ka.lse = lse;
  ka.delta = reinterpret_cast<float*>(base + w.delta);
  ka.dk_acc = dk_acc;
  ka.dv_acc = dv_acc;
  ka.dq_acc = w.dq ? reinterpret_cast<float*>(base + w.dq) : nullptr;
  ka.status = reinterpret_cast<int*>(base + w.status);
  ka.n_buckets = r.ia.n_buckets;
  ka.bucket_cnt = r.ia.bucket_cnt;
  ka.bucket_off = r.ia.bucket_off;
  ka.bucket_flag = r.ia.bucket_flag;
  return ka;
}

}  // namespace

extern "C" {

int32_t sa_abi_version(void) { return SA_ABI_VERSION; }

void sa_set_timing_events(void* ev_begin, void* ev_end, int32_t which) {
  sa::g_ev_begin = static_cast<cudaEvent_t>(ev_begin);
  sa::g_ev_end = static_cast<cudaEvent_t>(ev_end);
  sa::g_ev_which = which;
}

int64_t sa_kernel_launch_count(void) { return __atomic_load_n(&sa::g_launches, __ATOMIC_RELAXED); }

const char* sa_status_string(int32_t s) {
  switch (s) {
    case SA_OK: return "SA_OK";
    case SA_ERR_NULLPTR: return "SA_ERR_NULLPTR: a required pointer is NULL";
    case SA_ERR_PARAM: return "SA_ERR_PARAM: a size, mode or attribute is out of range";
    case SA_ERR_UNSUPPORTED: return "SA_ERR_UNSUPPORTED: combination not built";
    case SA_ERR_WORKSPACE: return "SA_ERR_WORKSPACE: workspace missing or too small";
    case SA_ERR_INDEX: return "SA_ERR_INDEX: an index lies past its sequence";
    case SA_ERR_TIMEOUT: return "SA_ERR_TIMEOUT: a bounded device wait gave up";
    case SA_ERR_CUDA: return "SA_ERR_CUDA: CUDA runtime error";
    default: return "unknown sa_status";
  }
}

sa_status sa_fwd_get_workspace_size(const sa_args* args, size_t* ws_bytes) {
  if (!ws_bytes) return SA_ERR_NULLPTR;
  sa_status st = validate(args);
  if (st != SA_OK) return st;
  *ws_bytes = kAlign;  // status word
  return SA_OK;
}

sa_status sa_fwd(const sa_args* args, const sa_fwd_out* out, void* ws, size_t ws_bytes, void* stream) {
  sa_status st = validate(args);
  if (st != SA_OK) return st;
  if (!out) return SA_ERR_NULLPTR;
  Sizes s = sizes_of(args);
  if (s.Tq == 0) return SA_OK;
  if (!out->o || !out->lse) return SA_ERR_NULLPTR;
  if (!ws || ws_bytes < kAlign) return SA_ERR_WORKSPACE;
  if (check_tensor_alignment(args) != SA_OK || !aligned16(out->o)) return SA_ERR_PARAM;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  int* status = static_cast<int*>(ws);
  if (args->flags & SA_FLAG_CHECK) {
    st = run_check(args, status, cs);
    if (st != SA_OK) return st;
  }
  sa::Prob p = make_prob(args, status);
  if (cudaMemsetAsync(status, 0, sizeof(int), cs) != cudaSuccess) return SA_ERR_CUDA;
  const int32_t choice = fwd_choice(args);
  if (choice == SA_KERNEL_FWD_BLOCK || choice == SA_KERNEL_FWD_BLOCK_TC) {
    sa::QbArgs q = make_qb_args(args, status);
    q.o = static_cast<bf16*>(out->o);
    q.lse = out->lse;
    if (choice == SA_KERNEL_FWD_BLOCK_TC) return cuda_status(sa::launch_bq_fwd(q, args->k, args->v, cs));
    return cuda_status(sa::launch_qb(q, args->k, args->v, false, cs));
  }
  if (choice == SA_KERNEL_FWD_TOKEN_TC)
    return cuda_status(sa::launch_tk_fwd(p, static_cast<bf16*>(out->o), out->lse,
                                         !(args->flags & SA_FLAG_TOKEN_FWD_UNPAIRED), cs));
  return cuda_status(sa::launch_fwd(p, static_cast<bf16*>(out->o), out->lse, cs));
}

sa_status sa_bwd_get_workspace_size(const sa_args* args, size_t* ws_bytes) {
  if (!ws_bytes) return SA_ERR_NULLPTR;
  sa_status st = validate(args);
  if (st != SA_OK) return st;
  if (paged(args)) return SA_ERR_UNSUPPORTED;  // a paged cache is an inference input: no backward
  *ws_bytes = bwd_ws_layout(args).total;
  return SA_OK;
}

sa_status sa_bwd(const sa_args* args, const sa_bwd_io* io, void* ws, size_t ws_bytes, void* stream) {
  sa_status st = validate(args);
  if (st != SA_OK) return st;
  if (paged(args)) return SA_ERR_UNSUPPORTED;
  if (!io) return SA_ERR_NULLPTR;
  Sizes s = sizes_of(args);
  const bool sinks = args->sinks != nullptr;
  if (s.Tq == 0) return SA_OK;
  if (!io->o || !io->d_o || !io->lse || !io->dq) return SA_ERR_NULLPTR;
  if (args->kv_shared ? !io->dkv : (!io->dk || !io->dv)) return SA_ERR_NULLPTR;
  if (has_cmp(args) && !io->dcmp_kv) return SA_ERR_NULLPTR;
  if (sinks && !io->dsinks) return SA_ERR_NULLPTR;
  BwdWs w = bwd_ws_layout(args);
  if (!ws || ws_bytes < w.total) return SA_ERR_WORKSPACE;
  if (check_tensor_alignment(args) != SA_OK || !aligned16(io->o) || !aligned16(io->d_o) ||
      !aligned16(io->dq) || !aligned16(io->dk) || !aligned16(io->dv) || !aligned16(io->dkv) ||
      !aligned16(io->dcmp_kv))
    return SA_ERR_PARAM;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  char* base = static_cast<char*>(ws);
  int* status = reinterpret_cast<int*>(base + w.status);
  if (args->flags & SA_FLAG_CHECK) {
    st = run_check(args, status, cs);
    if (st != SA_OK) return st;
  }
  sa::Prob p = make_prob(args, status);
  float* delta = reinterpret_cast<float*>(base + w.delta);
  sa::BwdOut out;
  out.dq = static_cast<bf16*>(io->dq);
  out.dk_acc = reinterpret_cast<float*>(base + w.dk);
  out.dv_acc = args->kv_shared ? nullptr : reinterpret_cast<float*>(base + w.dv);
  out.dcmp_acc = has_cmp(args) ? reinterpret_cast<float*>(base + w.dcmp) : nullptr;
  out.dsinks = sinks ? io->dsinks : nullptr;
  const long long nk = s.Tkv * args->n_heads_kv * args->d_qk;
  const long long nv = s.Tkv * args->n_heads_kv * args->d_v;
  const long long nc = s.Tcmp * args->n_heads_kv * args->d_qk;
  const int32_t choice = bwd_choice(args);
  cudaError_t e = cudaSuccess;
  KvIndexBuild kib;
  if (w.counts) {
    // key-stationary: the inverse index (with the cleared accumulators and Delta)
    st = build_kv_index(args, w, base, io->o, io->d_o, cs, &kib);
    if (st != SA_OK) return st;
  } else {
    // zero the accumulators and the status word (one memset), then Delta
    if (cudaMemsetAsync(base, 0, w.zero_end, cs) != cudaSuccess) return SA_ERR_CUDA;
    e = sa::launch_delta(static_cast<const bf16*>(io->o), static_cast<const bf16*>(io->d_o), delta,
                         s.Tq * args->n_heads_q, args->d_v, cs, p.f16 != 0);
    if (e != cudaSuccess) return SA_ERR_CUDA;
  }
  if (sinks && cudaMemsetAsync(io->dsinks, 0, sizeof(float) * args->n_heads_q, cs) != cudaSuccess)
    return SA_ERR_CUDA;
  if (w.counts) {
    // dK / dV per KV block (+ dQ)
    sa::KvLaunch kl;
    memset(&kl, 0, sizeof(kl));
    kl.args = kv_args(args, kib, w, base, io->d_o, io->lse, out.dk_acc, out.dv_acc);
    kl.q = args->q;
    kl.d_o = io->d_o;
    kl.k = args->k;
    kl.v = args->v;
    kl.Tq = s.Tq;
    kl.Tkv = s.Tkv;
    kl.dqk = args->d_qk;
    kl.dv = args->d_v;
    kl.max_work = kib.k.max_work;
    if (sa::launch_kv_bwd(kl, w.dq != 0, cs) != cudaSuccess) return SA_ERR_CUDA;
    if (!w.dq) {
      sa::QbArgs q = make_qb_args(args, status);
      q.d_o = static_cast<const bf16*>(io->d_o);
      q.lse = const_cast<float*>(io->lse);
      q.delta = delta;
      q.dq = static_cast<bf16*>(io->dq);
      e = sa::launch_qb(q, args->k, args->v, true, cs);
    }
  } else if (choice == SA_KERNEL_BWD_TOKEN_TC) {
    // token-level shared KV (576 / 512): the tcgen05 kernel, 64 heads per CTA
    e = sa::launch_tk_bwd(p, io->lse, delta, static_cast<const bf16*>(io->d_o), out, cs);
  } else {
    e = sa::launch_bwd(p, static_cast<const bf16*>(io->o), static_cast<const bf16*>(io->d_o), io->lse, delta,
                       out, cs);
  }
  if (e != cudaSuccess) return SA_ERR_CUDA;
  {
    sa::Cvt jobs[4];
    int nj = 0;
    if (args->kv_shared) {
      jobs[nj++] = sa::Cvt{out.dk_acc, static_cast<bf16*>(io->dkv), nk};
    } else {
      jobs[nj++] = sa::Cvt{out.dk_acc, static_cast<bf16*>(io->dk), nk};
      jobs[nj++] = sa::Cvt{out.dv_acc, static_cast<bf16*>(io->dv), nv};
    }
    if (has_cmp(args)) jobs[nj++] = sa::Cvt{out.dcmp_acc, static_cast<bf16*>(io->dcmp_kv), nc};
    if (w.dq) jobs[nj++] = sa::Cvt{reinterpret_cast<float*>(base + w.dq), static_cast<bf16*>(io->dq),
                                   s.Tq * args->n_heads_q * args->d_qk};
    e = sa::launch_to_bf16_multi(jobs, nj, cs, p.f16 != 0);
  }
  return cuda_status(e);
}

sa_status sa_softmax_grad_preprocess(const sa_args* args, const void* o, const void* d_o, float* delta,
                                     void* stream) {
  sa_status st = validate(args);
  if (st != SA_OK) return st;
  Sizes s = sizes_of(args);
  if (s.Tq == 0) return SA_OK;
  if (!o || !d_o || !delta) return SA_ERR_NULLPTR;
  if (!aligned16(o) || !aligned16(d_o)) return SA_ERR_PARAM;
  return cuda_status(sa::launch_delta(static_cast<const bf16*>(o), static_cast<const bf16*>(d_o), delta,
                                      s.Tq * args->n_heads_q, args->d_v, static_cast<cudaStream_t>(stream),
                                      args->dtype == SA_DTYPE_FP16));
}

sa_status sa_softmax_l1norm(const sa_args* args, const float* lse, float* ori_out, float* cmp_out, void* stream) {
  sa_status st = validate(args);
  if (st != SA_OK) return st;
  if (!ori_out && !cmp_out) return SA_ERR_NULLPTR;
  // each output needs its index list: ori indices (token or block selection), cmp indices
  if (ori_out && args->topk <= 0) return SA_ERR_PARAM;
  if (cmp_out && (args->cmp_topk <= 0 || !args->cmp_kv)) return SA_ERR_PARAM;
  Sizes s = sizes_of(args);
  if (s.Tq == 0) return SA_OK;
  if (!lse) return SA_ERR_NULLPTR;
  if (check_tensor_alignment(args) != SA_OK) return SA_ERR_PARAM;
  if (!sa::kernels_built(args->d_qk, args->d_v, args->kv_shared != 0)) return SA_ERR_UNSUPPORTED;
  sa::Prob p = make_prob(args, nullptr);
  return cuda_status(sa::launch_softmax_l1norm(p, lse, ori_out, cmp_out, static_cast<cudaStream_t>(stream)));
}

static sa_status ix_validate(const sa_indexer_args* a, long long* Tq, long long* Tkv) {
  if (!a) return SA_ERR_NULLPTR;
  if (a->layout != SA_LAYOUT_BSND && a->layout != SA_LAYOUT_TND) return SA_ERR_PARAM;
  if (a->batch < 0 || a->topk < 1) return SA_ERR_PARAM;
  if (a->layout == SA_LAYOUT_BSND) {
    if (a->s_q < 0 || a->s_kv < 0) return SA_ERR_PARAM;
    *Tq = (long long)a->batch * a->s_q;
    *Tkv = (long long)a->batch * a->s_kv;
  } else {
    if (a->t_q < 0 || a->t_kv < 0) return SA_ERR_PARAM;
    *Tq = a->t_q;
    *Tkv = a->t_kv;
  }
  if (*Tq >= (1ll << 31) || *Tkv >= (1ll << 30)) return SA_ERR_PARAM;
  if (!sa::ix_built(a->n_heads, a->d)) return SA_ERR_UNSUPPORTED;
  if (*Tq > 0) {
    if (!a->q || !a->k || !a->w || !a->idx || !a->p) return SA_ERR_NULLPTR;
    if (a->layout == SA_LAYOUT_TND && (!a->cu_seqlens_q || !a->cu_seqlens_kv || a->batch < 1)) return SA_ERR_NULLPTR;
    if (!aligned16(a->q) || !aligned16(a->k)) return SA_ERR_PARAM;
  }
  return SA_OK;
}

sa_status sa_indexer_kl_grad_get_workspace_size(const sa_indexer_args* args, size_t* ws_bytes) {
  if (!ws_bytes) return SA_ERR_NULLPTR;
  long long Tq = 0, Tkv = 0;
  sa_status st = ix_validate(args, &Tq, &Tkv);
  if (st != SA_OK) return st;
  *ws_bytes = kAlign + align_up((size_t)Tkv * args->d * sizeof(float));
  return SA_OK;
}

sa_status sa_indexer_kl_grad(const sa_indexer_args* args, const sa_indexer_grads* g, void* ws, size_t ws_bytes,
                             void* stream) {
  long long Tq = 0, Tkv = 0;
  sa_status st = ix_validate(args, &Tq, &Tkv);
  if (st != SA_OK) return st;
  if (!g) return SA_ERR_NULLPTR;
  if (Tq == 0) return SA_OK;
  if (!g->dq || !g->dk || !g->dw) return SA_ERR_NULLPTR;
  if (!aligned16(g->dq) || !aligned16(g->dk)) return SA_ERR_PARAM;
  const size_t need = kAlign + align_up((size_t)Tkv * args->d * sizeof(float));
  if (!ws || ws_bytes < need) return SA_ERR_WORKSPACE;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  char* base = static_cast<char*>(ws);
  if (cudaMemsetAsync(base, 0, need, cs) != cudaSuccess) return SA_ERR_CUDA;
  sa::IxArgs a;
  memset(&a, 0, sizeof(a));
  a.layout = args->layout;
  a.B = args->batch;
  a.s_q = args->s_q;
  a.s_kv = args->s_kv;
  a.Tq = (int)Tq;
  a.Tkv = (int)Tkv;
  a.H = args->n_heads;
  a.D = args->d;
  a.topk = args->topk;
  a.q = static_cast<const bf16*>(args->q);
  a.k = static_cast<const bf16*>(args->k);
  a.w = args->w;
  a.idx = args->idx;
  a.topk_len = args->topk_len;
  a.p = args->p;
  a.cu_q = args->cu_seqlens_q;
  a.cu_kv = args->cu_seqlens_kv;
  a.loss = g->loss;
  a.dq = static_cast<bf16*>(g->dq);
  a.dk_acc = reinterpret_cast<float*>(base + kAlign);
  a.dw = g->dw;
  a.status = reinterpret_cast<int*>(base);
  cudaError_t e = sa::launch_indexer_kl(a, cs);
  if (e != cudaSuccess) return SA_ERR_CUDA;
  if (Tkv > 0) e = sa::launch_to_bf16(a.dk_acc, static_cast<bf16*>(g->dk), Tkv * args->d, cs);
  return cuda_status(e);
}

sa_status sa_debug_resolve(const sa_args* args, int32_t* rows, int32_t* counts, int32_t max_rows, void* stream) {
  sa_status st = validate(args);
  if (st != SA_OK) return st;
  if (max_rows < 0) return SA_ERR_PARAM;
  Sizes s = sizes_of(args);
  if (s.Tq == 0) return SA_OK;
  if (!counts || (max_rows > 0 && !rows)) return SA_ERR_NULLPTR;
  sa::Prob p = make_prob(args, nullptr);
  return cuda_status(sa::launch_debug_resolve(p, rows, counts, max_rows, static_cast<cudaStream_t>(stream)));
}

sa_status sa_plan(const sa_args* args, int32_t* fwd_kernel, int32_t* bwd_kernel) {
  sa_status st = validate(args);
  if (st != SA_OK) return st;
  if (fwd_kernel) *fwd_kernel = fwd_choice(args);
  if (bwd_kernel) *bwd_kernel = bwd_choice(args);
  return SA_OK;
}

sa_status sa_read_status(const void* ws, size_t ws_bytes, void* stream) {
  if (!ws) return SA_ERR_NULLPTR;
  if (ws_bytes < sizeof(int)) return SA_ERR_WORKSPACE;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  int host = 0;
  if (cudaMemcpyAsync(&host, ws, sizeof(int), cudaMemcpyDeviceToHost, cs) != cudaSuccess) return SA_ERR_CUDA;
  if (cudaStreamSynchronize(cs) != cudaSuccess) return SA_ERR_CUDA;
  return status_of_bits(host);
}

sa_status sa_debug_block_index(const sa_args* args, int32_t view, void* ws, size_t ws_bytes, int32_t* records,
                               int64_t max_records, int32_t* n_records, void* stream) {
  sa_status st = validate(args);
  if (st != SA_OK) return st;
  if (!n_records || (max_records > 0 && !records)) return SA_ERR_NULLPTR;
  if (max_records < 0) return SA_ERR_PARAM;
  if (view != SA_INDEX_VIEW_QUERY_BLOCKS && view != SA_INDEX_VIEW_KEY_LISTS) return SA_ERR_PARAM;
  if (view == SA_INDEX_VIEW_QUERY_BLOCKS && !use_qb_path(args)) return SA_ERR_UNSUPPORTED;
  if (view == SA_INDEX_VIEW_KEY_LISTS && !use_kv_path(args)) return SA_ERR_UNSUPPORTED;
  BwdWs w = bwd_ws_layout(args);
  if (view == SA_INDEX_VIEW_KEY_LISTS && (!ws || ws_bytes < w.total)) return SA_ERR_WORKSPACE;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(n_records, 0, sizeof(int32_t), cs) != cudaSuccess) return SA_ERR_CUDA;
  if (sizes_of(args).Tq == 0) return SA_OK;
  int4* rec = reinterpret_cast<int4*>(records);
  if (view == SA_INDEX_VIEW_QUERY_BLOCKS) {
    sa::QbArgs q = make_qb_args(args, nullptr);
    return cuda_status(sa::launch_qb_debug_slots(q, rec, max_records, n_records, cs));
  }
  char* base = static_cast<char*>(ws);
  KvIndexBuild kib;
  st = build_kv_index(args, w, base, nullptr, nullptr, cs, &kib);
  if (st != SA_OK) return st;
  sa::KvArgs ka = kv_args(args, kib, w, base, nullptr, nullptr, nullptr, nullptr);
  return cuda_status(sa::launch_kv_debug_walk(ka, kib.k.max_work, rec, max_records, n_records, cs));
}

}  // extern "C"
