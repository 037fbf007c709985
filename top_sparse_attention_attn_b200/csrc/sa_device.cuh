// sa_device.cuh -- device-side problem description, selection (Stage 1) and
// warp-level MMA helpers shared by the sparse-attention kernels.
//
// Selection follows aclnnSparseFlashAttentionGrad "Formula" (block Gather
// through topkIndices) and SparseFlashMlaGrad "Computation formula" Stage 1
// (original KV, optionally through token indices, concatenated with gathered
// compressed KV), with the masks and topk lengths of the SparseFlashMlaGrad
// "Parameter Description" table.  Every (query token, kv-head) "unit" sees a
// list of tiles; a tile is 64 KV rows, each resolved to a global row code or
// to -1 (invisible).  Row codes: original-KV row -> its global row number;
// compressed row -> kCmpFlag | global compressed row.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace sa {

typedef __nv_bfloat16 bf16;

constexpr int kTileRows = 64;
constexpr int kCmpFlag = 0x40000000;

enum { kLayoutBSND = 0, kLayoutTND = 1 };
enum { kMaskNone = 0, kMaskCausal = 1, kMaskBand = 2 };
enum { kOriNone = 0, kOriBlock = 1, kOriToken = 2, kOriRange = 3 };

// Status bits written by kernels into the workspace status word.
enum { kStatusIndexRange = 1, kStatusTimeout = 2, kStatusSmemAlign = 4 };

struct Prob {
  int layout, B, s_q, s_kv;
  int Tq, Tkv, Tcmp;
  int Hq, Hkv, G, dqk, dv, shared, bs, topk, cmp_topk, ratio, ori_mask, cmp_mask;
  const int *used_q, *used_kv, *used_cmp;  // sequsedQ / OriKv / CmpKv ([B]) or null
  const int* page_table;                   // paged KV cache: [B, max_pages] or null
  int page_size, max_pages;
  long long wl, wr;
  float scale;        // scaleValue
  float scale_log2;   // scale * log2(e)
  const bf16* q;
  const bf16* k;      // K (or the shared KV)
  const bf16* v;      // V (or the shared KV)
  const bf16* cmpk;   // compressed KV (K = V)
  const int* ori_idx;
  const int* cmp_idx;
  const int* cu_q;
  const int* cu_kv;
  const int* cu_cmp;
  const int* ori_len;
  const int* cmp_len;
  const float* sinks;
  int* status;        // device status word (may be null)
  int f16;            // the 2-byte tensors (q, k, v, cmp_kv, O, dO, dQ, dK, dV) hold fp16, else bf16
};

struct Unit {
  int tq, g, b, t, ta, Lk, Lc, kv0, cmp0;
  int ori_mode, n_ori_slots, n_cmp_slots, lo, hi, tps;
  int n_ori_tiles, n_tiles;
};

__device__ __forceinline__ int find_batch(const int* cu, int B, int tq) {
  int lo = 0, hi = B - 1;  // largest b with cu[b] <= tq
  while (lo < hi) {
    int mid = (lo + hi + 1) >> 1;
    if (__ldg(cu + mid) <= tq) lo = mid; else hi = mid - 1;
  }
  return lo;
}

__device__ __forceinline__ Unit make_unit(const Prob& p, int tq, int g) {
  Unit u;
  u.tq = tq;
  u.g = g;
  int Lq;
  if (p.layout == kLayoutBSND) {
    u.b = tq / p.s_q;
    u.t = tq - u.b * p.s_q;
    Lq = p.s_q;
    u.Lk = p.s_kv;
    u.kv0 = u.b * p.s_kv;
    u.Lc = p.cmpk ? p.s_kv / p.ratio : 0;
    u.cmp0 = u.b * u.Lc;
  } else {
    // offsets are clamped to the packed extents, so inconsistent cu_seqlens can
    // shrink a sequence but never make a kernel read outside its tensors
    u.b = find_batch(p.cu_q, p.B, tq);
    int q0 = __ldg(p.cu_q + u.b);
    Lq = max(__ldg(p.cu_q + u.b + 1) - q0, 0);
    u.t = tq - q0;
    u.kv0 = min(max(__ldg(p.cu_kv + u.b), 0), p.Tkv);
    u.Lk = min(max(__ldg(p.cu_kv + u.b + 1), u.kv0), p.Tkv) - u.kv0;
    if (p.cmpk) {
      u.cmp0 = min(max(__ldg(p.cu_cmp + u.b), 0), p.Tcmp);
      u.Lc = min(max(__ldg(p.cu_cmp + u.b + 1), u.cmp0), p.Tcmp) - u.cmp0;
    } else {
      u.cmp0 = 0;
      u.Lc = 0;
    }
  }
  // the tokens that take part (sequsedQ / sequsedOriKv / sequsedCmpKv)
  if (p.used_q) Lq = min(Lq, max(0, __ldg(p.used_q + u.b)));
  if (p.used_kv) u.Lk = min(u.Lk, max(0, __ldg(p.used_kv + u.b)));
  if (p.used_cmp) u.Lc = min(u.Lc, max(0, __ldg(p.used_cmp + u.b)));
  const bool active = u.t < Lq;  // a row past sequsedQ selects nothing
  u.ta = u.t + u.Lk - Lq;
  const long long ug = (long long)tq * p.Hkv + g;
  u.tps = 1;
  u.lo = 0;
  u.hi = -1;
  if (p.topk > 0) {
    int n = p.topk;
    if (p.ori_len) n = min(n, max(0, __ldg(p.ori_len + ug)));
    u.n_ori_slots = n;
    if (p.bs > 1) {
      u.ori_mode = kOriBlock;
      u.tps = (p.bs + kTileRows - 1) / kTileRows;
      u.n_ori_tiles = n * u.tps;
    } else {
      u.ori_mode = kOriToken;
      u.n_ori_tiles = (n + kTileRows - 1) / kTileRows;
    }
  } else {
    u.ori_mode = kOriRange;
    u.n_ori_slots = 0;
    long long lo = 0, hi = (long long)u.Lk - 1;
    if (p.ori_mask == kMaskCausal) {
      hi = min(hi, (long long)u.ta);
    } else if (p.ori_mask == kMaskBand) {
      lo = max(lo, (long long)u.ta - p.wl);
      hi = min(hi, (long long)u.ta + p.wr);
    }
    if (hi < lo) { lo = 0; hi = -1; }
    u.lo = (int)lo;
    u.hi = (int)hi;
    u.n_ori_tiles = (int)((hi - lo + 1 + kTileRows - 1) / kTileRows);
  }
  if (p.cmp_topk > 0) {
    int n = p.cmp_topk;
    if (p.cmp_len) n = min(n, max(0, __ldg(p.cmp_len + ug)));
    u.n_cmp_slots = n;
  } else {
    // a compressed KV without indices (CFA): every compressed row, slot c = row c
    u.n_cmp_slots = p.cmpk ? u.Lc : 0;
  }
  u.n_tiles = u.n_ori_tiles + (u.n_cmp_slots + kTileRows - 1) / kTileRows;
  if (!active) {
    u.n_ori_slots = u.n_cmp_slots = 0;
    u.n_ori_tiles = u.n_tiles = 0;
    u.lo = 0;
    u.hi = -1;
  }
  return u;
}

// ---------------------------------------------------------------------------
// Block-level selection with 64-row blocks (aclnnSparseFlashAttentionGrad,
// "Formula": each of the selectBlockCount indices names 64 contiguous rows).
// The slot rule and the in-block row range below are the only definitions the
// block kernels, the key-stationary inverse index and the inspection entry
// point use, so what the inspection returns is what the kernels compute.
// A query row sits at sequence-local position ta (aligned bottom-right) over a
// key sequence of Lk rows; wl / wr are the BAND window (host-clamped to 2^40).
// ---------------------------------------------------------------------------

// Slot naming block x is usable: x >= 0, the block starts inside the sequence,
// and at least one of its rows survives the ori mask.
__device__ __forceinline__ bool blk_usable(int x, int Lk, int ta, int mask, long long wl, long long wr) {
  if (x < 0) return false;
  const long long first = (long long)x * kTileRows;
  if (first >= Lk) return false;
  if (mask == kMaskCausal) return first <= ta;
  if (mask == kMaskBand) {
    const long long last = min(first + kTileRows - 1, (long long)Lk - 1);
    return first <= (long long)ta + wr && last >= (long long)ta - wl;
  }
  return true;
}

// Visible rows of block x for the same query row, as offsets [*lo, *hi] within
// the block (0..63); *lo > *hi when none.  Non-empty whenever blk_usable holds.
__device__ __forceinline__ void blk_rows(int x, int Lk, int ta, int mask, long long wl, long long wr, int* lo,
                                         int* hi) {
  const long long first = (long long)x * kTileRows;
  long long l = 0, h = min((long long)kTileRows - 1, (long long)Lk - 1 - first);
  if (mask == kMaskCausal) {
    h = min(h, (long long)ta - first);
  } else if (mask == kMaskBand) {
    h = min(h, (long long)ta + wr - first);
    l = max(l, (long long)ta - wl - first);
  }
  if (h < l) {
    l = 0;
    h = -1;
  }
  *lo = (int)l;
  *hi = (int)h;
}

__device__ __forceinline__ bool ori_mask_ok(const Prob& p, const Unit& u, int r) {
  if (p.ori_mask == kMaskCausal) return r <= u.ta;
  if (p.ori_mask == kMaskBand) return (long long)r >= (long long)u.ta - p.wl && (long long)r <= (long long)u.ta + p.wr;
  return true;
}

// True when a tile (ori block slot) is empty before looking at its rows; lets
// callers skip whole slots cheaply.  Only used as a hint.
__device__ __forceinline__ bool tile_is_empty_slot(const Prob& p, const Unit& u, int tile) {
  if (tile < u.n_ori_tiles && u.ori_mode == kOriBlock) {
    int s = tile / u.tps;
    int x = __ldg(p.ori_idx + ((long long)u.tq * p.Hkv + u.g) * p.topk + s);
    return x < 0;
  }
  return false;
}

// The raw index row r (0..63) of tile `tile` of unit u reads: its slot's ori or
// cmp index, -1 for a slot past the unit's count, 0 for the window (range) mode,
// which reads none.  Split from resolve_row so that a kernel can issue the load
// early (the token-level kernels prefetch the next tile's indices).
__device__ __forceinline__ int slot_index(const Prob& p, const Unit& u, int tile, int r) {
  const long long ug = (long long)u.tq * p.Hkv + u.g;
  if (tile < u.n_ori_tiles) {
    if (u.ori_mode == kOriBlock) return __ldg(p.ori_idx + ug * p.topk + tile / u.tps);
    if (u.ori_mode == kOriToken) {
      const int s = tile * kTileRows + r;
      return s < u.n_ori_slots ? __ldg(p.ori_idx + ug * p.topk + s) : -1;
    }
    return 0;
  }
  const int s = (tile - u.n_ori_tiles) * kTileRows + r;
  if (s >= u.n_cmp_slots) return -1;
  return p.cmp_idx ? __ldg(p.cmp_idx + ug * p.cmp_topk + s) : s;
}

// Storage row code of sequence-local original-KV row `row` of unit u: contiguous
// from kv0, or through the block table of a paged cache (-1, with the index bit,
// for a page outside the cache).
__device__ __forceinline__ int kv_code(const Prob& p, const Unit& u, long long row) {
  if (!p.page_table) return u.kv0 + (int)row;
  const int page = __ldg(p.page_table + (long long)u.b * p.max_pages + (int)(row / p.page_size));
  const long long code = (long long)page * p.page_size + row % p.page_size;
  if (page < 0 || code >= p.Tkv) {
    if (p.status) atomicOr(p.status, kStatusIndexRange);
    return -1;
  }
  return (int)code;
}

// Resolve row r (0..63) of tile `tile` of unit u, whose slot holds index x (from
// slot_index), to a global row code, or -1.  An index past the end of its
// sequence selects nothing and raises the status word's index bit.
__device__ __forceinline__ int resolve_row_x(const Prob& p, const Unit& u, int tile, int r, int x) {
  if (tile < u.n_ori_tiles) {
    if (u.ori_mode == kOriBlock) {
      const int sub = tile - (tile / u.tps) * u.tps;
      if (x < 0) return -1;
      int within = sub * kTileRows + r;
      if (within >= p.bs) return -1;
      long long first = (long long)x * p.bs;
      if (first >= u.Lk) {
        if (p.status && r == 0 && sub == 0) atomicOr(p.status, kStatusIndexRange);
        return -1;
      }
      long long row = first + within;
      if (row >= u.Lk || !ori_mask_ok(p, u, (int)row)) return -1;
      return kv_code(p, u, row);
    } else if (u.ori_mode == kOriToken) {
      if (x < 0) return -1;
      if (x >= u.Lk) {
        if (p.status) atomicOr(p.status, kStatusIndexRange);
        return -1;
      }
      if (!ori_mask_ok(p, u, x)) return -1;
      return kv_code(p, u, x);
    } else {
      int row = u.lo + tile * kTileRows + r;
      if (row > u.hi) return -1;
      return kv_code(p, u, row);
    }
  }
  const int c = x;
  if (c < 0) return -1;
  if (c >= u.Lc) {
    if (p.status) atomicOr(p.status, kStatusIndexRange);
    return -1;
  }
  if (p.cmp_mask == kMaskCausal && (long long)(c + 1) * p.ratio - 1 > u.ta) return -1;
  return kCmpFlag | (u.cmp0 + c);
}

// Resolve row r (0..63) of tile `tile` of unit u to a global row code, or -1.
__device__ __forceinline__ int resolve_row(const Prob& p, const Unit& u, int tile, int r) {
  return resolve_row_x(p, u, tile, r, slot_index(p, u, tile, r));
}

// Element offsets of a row's K and V vectors (kv-head g) for a row code >= 0.
__device__ __forceinline__ const bf16* row_k_ptr(const Prob& p, int code, int g) {
  if (code & kCmpFlag) return p.cmpk + ((long long)(code & ~kCmpFlag) * p.Hkv + g) * p.dqk;
  return p.k + ((long long)code * p.Hkv + g) * p.dqk;
}
__device__ __forceinline__ const bf16* row_v_ptr(const Prob& p, int code, int g) {
  if (code & kCmpFlag) return p.cmpk + ((long long)(code & ~kCmpFlag) * p.Hkv + g) * p.dqk;
  if (p.shared) return p.k + ((long long)code * p.Hkv + g) * p.dqk;
  return p.v + ((long long)code * p.Hkv + g) * p.dv;
}

// ---------------------------------------------------------------------------
// shared-memory tiles: rows of D bf16 (D % 64 == 0), 16-byte chunks XOR-swizzled
// by (row & 7) so ldmatrix phases hit distinct banks.
// ---------------------------------------------------------------------------
template <int D>
__device__ __forceinline__ uint32_t swz(uint32_t base, int row, int chunk) {
  return base + (uint32_t)(row * D * 2) + (uint32_t)(((chunk ^ (row & 7))) << 4);
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool valid) {
  int n = valid ? 16 : 0;
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(dst), "l"(src), "r"(n));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;\n" ::); }

__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(addr));
}

__device__ __forceinline__ void mma16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// 2^x by the hardware approximation (ex2.approx.ftz.f32: a few ulp, results below
// the normal range flushed to 0, 2^-inf = 0): the softmax exponentials of the
// tensor-core kernels, whose scores are at most a few units above the row maximum.
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;\n" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// The element type of the 2-byte tensors for the mma.sync kernels: the tensors
// move as raw 16-bit data (the pointers are typed bf16 for storage only), and
// Elt<F16> supplies the arithmetic -- the m16n8k16 MMA on bf16 or fp16 operands
// (fp32 accumulation either way), two fp32 values rounded to nearest even into
// one 32-bit pair, and a pair widened to fp32.
template <bool F16>
struct Elt;
template <>
struct Elt<false> {
  static __device__ __forceinline__ void mma(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    mma16816(c, a, b0, b1);
  }
  static __device__ __forceinline__ uint32_t pack(float lo, float hi) { return pack_bf16(lo, hi); }
  static __device__ __forceinline__ float2 widen(uint32_t x) {
    return __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&x));
  }
};
template <>
struct Elt<true> {
  static __device__ __forceinline__ void mma(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};\n"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
  }
  static __device__ __forceinline__ uint32_t pack(float lo, float hi) {
    __half2 v = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
  }
  static __device__ __forceinline__ float2 widen(uint32_t x) {
    return __half22float2(*reinterpret_cast<const __half2*>(&x));
  }
};

// A fragment (16 x 16) at rows r0.., k-chunk kc (k0 = 8*kc) of a row-major swizzled tile.
template <int D>
__device__ __forceinline__ void load_a(uint32_t (&a)[4], uint32_t base, int r0, int kc, int lane) {
  ldsm_x4(a, swz<D>(base, r0 + (lane & 15), kc + (lane >> 4)));
}
// B fragments for two n-tiles (rows n0..n0+15 of a row-major [N][D] tile, B[k][n] = T[n][k]),
// k-chunk kc: b[0],b[1] -> n-tile n0; b[2],b[3] -> n-tile n0+8.
template <int D>
__device__ __forceinline__ void load_b_nk(uint32_t (&b)[4], uint32_t base, int n0, int kc, int lane) {
  ldsm_x4(b, swz<D>(base, n0 + (lane & 7) + ((lane >> 4) << 3), kc + ((lane >> 3) & 1)));
}
// B fragments for two n-tiles from a row-major [K][D] tile with B[k][n] = T[k][n]
// (k rows k0..k0+15, columns n-chunk nc and nc+1).
template <int D>
__device__ __forceinline__ void load_b_kn(uint32_t (&b)[4], uint32_t base, int k0, int nc, int lane) {
  ldsm_x4_t(b, swz<D>(base, k0 + (lane & 7) + (((lane >> 3) & 1) << 3), nc + (lane >> 4)));
}
// A fragment of the transpose: A[m][k] = T[k][m] from a row-major [K][D] tile,
// m rows from column-chunk mc (m0 = 8*mc), k rows k0..k0+15.
template <int D>
__device__ __forceinline__ void load_a_t(uint32_t (&a)[4], uint32_t base, int k0, int mc, int lane) {
  ldsm_x4_t(a, swz<D>(base, k0 + (lane & 7) + ((lane >> 4) << 3), mc + ((lane >> 3) & 1)));
}

__device__ __forceinline__ float warp_max4(float v) {
  v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 1));
  v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 2));
  return v;
}
__device__ __forceinline__ float warp_sum4(float v) {
  v += __shfl_xor_sync(0xffffffffu, v, 1);
  v += __shfl_xor_sync(0xffffffffu, v, 2);
  return v;
}

// Programmatic dependent launch.  A kernel launched with programmatic stream
// serialization may begin while the kernel before it on the stream is still
// running; pdl_wait() returns once that kernel has completed and its memory is
// visible (at once when there is no such predecessor), so everything before it
// may touch only this CTA's own shared memory and TMEM.  pdl_trigger() lets the
// next kernel on the stream start launching.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;\n" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory"); }

// Delta of one row: sum_d a[d] * b[d] over n 2-byte elements (bf16, or fp16 with
// F16; n a multiple of 8, 16-byte aligned rows) in fp32, by one warp; every lane
// returns the sum.
template <bool F16 = false>
__device__ __forceinline__ float warp_row_dot_bf16(const bf16* __restrict__ a, const bf16* __restrict__ b, int n,
                                                   int lane) {
  const uint4* a4 = reinterpret_cast<const uint4*>(a);
  const uint4* b4 = reinterpret_cast<const uint4*>(b);
  float acc = 0.f;
  for (int i = lane; i < n / 8; i += 32) {
    uint4 x = __ldg(a4 + i), y = __ldg(b4 + i);
    const uint32_t px[4] = {x.x, x.y, x.z, x.w}, py[4] = {y.x, y.y, y.z, y.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float2 fx = Elt<F16>::widen(px[j]), fy = Elt<F16>::widen(py[j]);
      acc = fmaf(fx.x, fy.x, acc);
      acc = fmaf(fx.y, fy.y, acc);
    }
  }
#pragma unroll
  for (int off = 16; off; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
  return acc;
}

}  // namespace sa
