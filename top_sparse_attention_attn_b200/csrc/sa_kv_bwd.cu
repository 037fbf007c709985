// sa_kv_bwd.cu -- key-stationary backward for block-level selection (BSND):
// dK and dV accumulate in TMEM per selected KV block, with no per-token
// scatter.
//
// aclnnSparseFlashAttentionGrad "Formula" Phases 1-3 (dV = P^T dO,
// dS = P o (dP - rowsum(dO o O)), dK = dS^T Q scale), restructured around
// the KV block: an inverse index lists, for every (batch, kv-head, block),
// the query tokens whose selection names the block; one CTA takes a chunk of
// that list and streams the tokens' query rows through the block in tiles of
// 128 rows (128 / RPT tokens: RPT = G for G = 1, 2, 4, rows copied one by one;
// else G rounded up to a multiple of 8, one TMA box per token).
//
// Per tile (tcgen05, bf16 operands, fp32 TMEM accumulators):
//   S   [128 x 64]  = Q K_j^T             (A = Q K-major, B = K_j K-major)
//   dP  [128 x 64]  = dO V_j^T            (A = dO K-major, B = V_j K-major)
//   P = exp2(S * scale * log2e - lse * log2e), dS = P o (dP - Delta)   (softmax warps)
//   dV^T [DV x 64] += dO^T P              (A = dO MN-major, B = P MN-major)
//   dK^T [DQK x 64] += Q^T dS             (A = Q MN-major, B = dS MN-major)
//   dQ  [128 x DQK] = dS K_j              (optional; A = dS K-major, B = K_j MN-major),
//                      added to an fp32 dQ accumulator with 16-byte atomics that a
//                      per-warp shared-memory slice makes contiguous (8 rows x 64 B).
// At the end dK^T / dV^T (scaled) pass through shared memory and are added to the
// fp32 dK / dV accumulators; blocks split into several chunks meet there.
//
// Warp roles: 0 = TMA producer, 1 = MMA issuer + TMEM owner, 2..5 = softmax /
// dK-dV epilogue (thread = query row = TMEM lane), 6..9 (with dQ) = dQ epilogue
// and, for G = 1, 2, 4, the row gather of the tiles' Q / dO rows.
// Every wait is bounded (sa_tc.cuh): on timeout the CTA raises the status
// word, skips the rest of its work, drains and frees TMEM.
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "sa_device.cuh"
#include "sa_kv_bwd.h"
#include "sa_launch.h"
#include "sa_tc.cuh"

namespace sa {

constexpr float kLog2eKv = 1.4426950408889634f;

template <int DQK, int DV, bool WITH_DQ>
struct KvPlan {
  static constexpr int NSQ = DQK / 64;             // 64-wide slabs of a Q row
  static constexpr int NSV = DV / 64;
  static constexpr int kQStage = NSQ * 128 * 128;  // 128 rows x 128 B per slab
  static constexpr int kDOStage = NSV * 128 * 128;
  static constexpr int oQ = 0;                     // 2 stages
  static constexpr int oDO = oQ + 2 * kQStage;     // 2 stages
  static constexpr int oK = oDO + 2 * kDOStage;    // NSQ slabs of 64 rows
  static constexpr int oV = oK + NSQ * 64 * 128;   // NSV slabs of 64 rows
  static constexpr int oPS = oV + NSV * 64 * 128;  // P, then dS: 128 rows x 128 B
  static constexpr int oTok = oPS + 128 * 128;     // bucketed mode: the chunk's token ids
  static constexpr int oDQS = oTok + kBucketMaxChunk * 4;  // dQ staging: 128 rows x 16 fp32
  static constexpr int kBytes = oDQS + 128 * 16 * 4;
  // the dynamic region starts right after the 1024-byte static region (KvBars padded
  // to the extern array's 1024-byte alignment): no slack, checked at run time
  static constexpr int kSmem = kBytes;
  static constexpr int NV = (DV + 127) / 128;      // M tiles of dV^T
  static constexpr int NK = (DQK + 127) / 128;     // M tiles of dK^T
  // d_qk = d_v = 64: dV^T and dK^T are both M = 64 accumulators (16 lanes of each
  // sub-partition), so they share columns at lane offsets 0 and 16 and the plan
  // fits 256 columns (two CTAs per SM)
  static constexpr bool kPack = DQK == 64 && DV == 64;
  static constexpr int kDkLane = kPack ? 16 : 0;
  static constexpr int cS = 0, cDP = 64, cDV = 128;
  static constexpr int cDK = kPack ? cDV : cDV + 64 * NV;
  static constexpr int cDQ = kPack ? cDV + 64 : cDK + 64 * NK;
  static constexpr int kCols = cDQ + (WITH_DQ ? DQK : 0);
  static constexpr uint32_t kAlloc = kCols <= 256 ? 256 : 512;
  static_assert(kCols <= 512, "TMEM plan too large");
  // epilogue staging of dV^T / dK^T as fp32 [key][dim] over the (then idle) Q / dO
  // stages; with packed accumulators the dK rows start 16 banks after the dV rows
  // so that the two lane halves of a warp store without bank conflicts
  static constexpr int oStV = oQ;
  static constexpr int oStK = oStV + 64 * DV * 4 + (kPack ? 64 : 0);
  static_assert(oStK + 64 * DQK * 4 <= oK, "epilogue staging does not fit the Q / dO stages");
  static_assert(kSmem + 1024 <= 227 * 1024, "shared memory plan too large");
};

// A CTA's work item: list L (-1 past the last item), chunk c of the list and its
// ntok tokens; bucketed mode also keeps where each bucket's part of the list
// starts (in rank order) and sits.
struct KvItem {
  int L, c, ntok;
  int bstart[kBucketMax];
  int boff[kBucketMax];
};

struct KvBars {
  uint64_t kv_full, q_full[2], q_empty[2], s_full, p_full, p_free, ds_full, tile_done, acc_done, dq_full, dq_free;
  uint32_t tmem_base;
  int abort_flag;
  KvItem item;
};

// The list that block x of one token's selections joins: (batch b, token window,
// kv-head g, block x), or -1 when the block is out of range or keeps no visible
// row for the token (offset ta within its sequence).  A is KvArgs or KvIndexArgs.
template <class A>
__device__ __forceinline__ int kv_block_list(const A& a, int x, int b, int ta, int g) {
  if (!blk_usable(x, a.S, ta, a.ori_mask, a.wl, a.wr)) return -1;
  // keyed by the token's window first, so that CTAs launched together add their dQ
  // contributions to a window of tokens whose fp32 accumulators stay in L2
  return ((b * a.nwin + ta / a.win_tokens) * a.Hkv + g) * a.nblk + x;
}

__device__ __forceinline__ void red_add_v4(float* addr, float a, float b, float c, float d) {
  asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};\n" ::"l"(addr), "f"(a), "f"(b), "f"(c), "f"(d)
               : "memory");
}

// Row gather of one tile by NT threads (t = 0 .. NT-1): rows r = u * G + h of the
// stage hold head head0 + h of token toks[u]; consecutive threads copy
// consecutive 16-byte pieces with cp.async into the 128-byte-swizzled slab
// layout the tensor core reads (64 columns per slab).
template <int D, int NT>
__device__ __forceinline__ void kv_gather_rows(uint32_t sbase, const bf16* __restrict__ src, const int* toks,
                                               int nrows, int lg, int Hq, int head0, int t) {
  constexpr int CPR = D / 8;  // 16-byte pieces per row
#pragma unroll 4
  for (int idx = t; idx < nrows * CPR; idx += NT) {
    const int r = idx / CPR, c = idx - r * CPR;
    const int tq = toks[r >> lg];
    const bf16* p = src + ((long long)tq * Hq + head0 + (r & ((1 << lg) - 1))) * D + c * 8;
    cp_async16(sbase + (c >> 3) * (128 * 128) + r * 128 + (((c & 7) ^ (r & 7)) << 4), p, true);
  }
}

// Work item w from the bucketed index (every thread of the CTA).  Warp 0 sums
// each list's counts over the buckets, turns them into chunk counts, finds the
// list and chunk of item w, and where each bucket's part of that list starts (in
// rank order) and sits; then the CTA gathers the chunk's token ids into `toks`.
// Fills `it` (it.L = -1 past the last item).
__device__ void kv_bucket_item(const KvArgs& a, int w, int* toks, KvItem& it) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nl = a.n_lists, nb = a.n_buckets;
  if (warp == 0) {
    // indices past their sequence, seen by the preparation launch, reach the status word
    if (w == 0 && lane < nb && __ldg(a.bucket_flag + lane) && a.status) atomicOr(a.status, kStatusIndexRange);
    int carry = 0, fL = -1, fc = 0, fn = 0;
    for (int l0 = 0; l0 < nl; l0 += 32) {
      const int L = l0 + lane;
      int cnt = 0;
      if (L < nl)
        for (int k = 0; k < nb; ++k) cnt += __ldg(a.bucket_cnt + k * nl + L);
      const int nk = (cnt + a.chunk_tokens - 1) / a.chunk_tokens;
      int incl = nk;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      const int excl = carry + incl - nk;
      const unsigned m = __ballot_sync(0xffffffffu, w >= excl && w < excl + nk);
      if (m) {
        const int src = __ffs(m) - 1;
        fL = __shfl_sync(0xffffffffu, L, src);
        fc = __shfl_sync(0xffffffffu, w - excl, src);
        fn = __shfl_sync(0xffffffffu, cnt, src);
      }
      carry += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) {
      it.L = fL;
      it.c = fc;
      it.ntok = fL >= 0 ? min(a.chunk_tokens, fn - fc * a.chunk_tokens) : 0;
    }
    if (fL >= 0) {
      const int v = lane < nb ? __ldg(a.bucket_cnt + lane * nl + fL) : 0;
      int incl = v;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      if (lane < nb) {
        it.bstart[lane] = incl - v;
        it.boff[lane] = __ldg(a.bucket_off + lane * nl + fL);
      }
    }
  }
  __syncthreads();
  if (it.L < 0) return;
  const int lo = it.c * a.chunk_tokens, n = it.ntok;
  for (int r = threadIdx.x; r < n; r += blockDim.x) {
    const int R = lo + r;
    int k = 0;  // the last bucket whose part starts at or before rank R
    for (int k2 = 1; k2 < nb; ++k2)
      if (it.bstart[k2] <= R) k = k2;
    toks[r] = __ldg(a.entries + k * kBucketSlots + it.boff[k] + (R - it.bstart[k]));
  }
}

// Work item w of either index (every thread of the CTA calls it): its token ids
// are returned (shared memory `toks_smem` in bucketed mode, the entries array
// otherwise) and `it` is filled by the time of the caller's next __syncthreads.
__device__ __forceinline__ const int* kv_get_item(const KvArgs& a, int w, int* toks_smem, KvItem& it) {
  if (a.n_buckets > 0) {
    kv_bucket_item(a, w, toks_smem, it);
    return toks_smem;
  }
  const int4 item = __ldg(a.items + w);  // in bounds (w < max_work); used only when w < work_count
  const int nwork = __ldg(a.work_count);
  if (threadIdx.x == 0) {
    it.L = w < nwork ? item.x : -1;
    it.c = 0;
    it.ntok = item.z;
  }
  return a.entries + item.y;
}

// List id = ((batch * nwin + window) * Hkv + kv-head) * nblk + block.
__device__ __forceinline__ void kv_list_decode(const KvArgs& a, int L, int* b, int* g, int* j) {
  *j = L % a.nblk;
  const int rest = L / a.nblk;
  *g = rest % a.Hkv;
  *b = (rest / a.Hkv) / a.nwin;
}

template <int DQK, int DV, bool WITH_DQ>
__global__ void __launch_bounds__(WITH_DQ ? 320 : 192, 1) kv_bwd_kernel(const __grid_constant__ CUtensorMap mapQ,
                                                        const __grid_constant__ CUtensorMap mapDO,
                                                        const __grid_constant__ CUtensorMap mapK,
                                                        const __grid_constant__ CUtensorMap mapV,
                                                        const KvArgs a) {
  using PL = KvPlan<DQK, DV, WITH_DQ>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  __shared__ KvBars bars;
  uint8_t* smem = smem_raw;
  if (smem_u32(smem_raw) & 1023) {  // the swizzled operand layouts need 1024-byte alignment
    pdl_wait();  // the status word is cleared by a preceding launch
    if (threadIdx.x == 0 && a.status) atomicOr(a.status, kStatusSmemAlign);
    return;
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  const uint32_t sQ = smem_u32(smem + PL::oQ), sDO = smem_u32(smem + PL::oDO);
  const uint32_t sK = smem_u32(smem + PL::oK), sV = smem_u32(smem + PL::oV);
  const uint32_t sPS = smem_u32(smem + PL::oPS);
  volatile int* abort_flag = &bars.abort_flag;

  const bool gather = WITH_DQ && a.gather_rows;  // Q / dO rows copied by the dQ role

  // ---- set-up on shared memory and TMEM only: may overlap the preceding kernel
  // zero the Q / dO stages once: rows no token fills stay finite (0)
  {
    uint4 z = make_uint4(0, 0, 0, 0);
    uint4* p = reinterpret_cast<uint4*>(smem + PL::oQ);
    const int n16 = (PL::oK - PL::oQ) / 16;
    for (int i = threadIdx.x; i < n16; i += blockDim.x) p[i] = z;
  }
  if (threadIdx.x == 0) {
    bars.abort_flag = 0;
    mbar_init(&bars.kv_full, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bars.q_full[s], gather ? 128 : 1);  // row gather: every dQ-role thread arrives
      mbar_init(&bars.q_empty[s], 1);
    }
    mbar_init(&bars.s_full, 1);
    mbar_init(&bars.p_full, 128);
    mbar_init(&bars.p_free, 1);
    mbar_init(&bars.ds_full, 128);
    mbar_init(&bars.tile_done, 1);
    mbar_init(&bars.acc_done, 1);
    mbar_init(&bars.dq_full, 1);
    mbar_init(&bars.dq_free, 128);
    mbar_fence_init();
    tma_prefetch_desc(&mapQ);
    tma_prefetch_desc(&mapDO);
    tma_prefetch_desc(&mapK);
    tma_prefetch_desc(&mapV);
  }
  if (warp == 1) tmem_alloc(&bars.tmem_base, PL::kAlloc);

  // ---- the work item {list, tokens}
  const int w = blockIdx.x;
  pdl_wait();  // the index, Delta and the cleared accumulators come from the preceding kernels
  const int* toks = kv_get_item(a, w, reinterpret_cast<int*>(smem + PL::oTok), bars.item);
  fence_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  pdl_trigger();
  const uint32_t tmem = bars.tmem_base;
  const int L = bars.item.L, ntok = bars.item.ntok;
  if (L < 0) {  // past the last work item (uniform over the CTA)
    if (warp == 1) {
      tmem_dealloc(tmem, PL::kAlloc);
      tmem_relinquish();
    }
    return;
  }
  int b, g, j;
  kv_list_decode(a, L, &b, &g, &j);
  const int TPT = a.TPT, RPT = a.RPT;
  const int ntiles = (ntok + TPT - 1) / TPT;
  if (threadIdx.x == 0) {
    const int row0 = b * a.S + 64 * j;  // first KV row of block j
    mbar_arrive_tx(&bars.kv_full, (uint32_t)(64 * (DQK + DV) * 2));
    for (int s = 0; s < DQK / 64; ++s) tma_load_2d(sK + s * 64 * 128, &mapK, g * DQK + 64 * s, row0, &bars.kv_full);
    for (int s = 0; s < DV / 64; ++s) tma_load_2d(sV + s * 64 * 128, &mapV, g * DV + 64 * s, row0, &bars.kv_full);
  }

  if (warp == 0) {
    // ------------------------------------------------------------ producer (whole warp)
    // lane u issues the TMA loads of token u of the tile; the next tile's token
    // ids are fetched while the current stage is being waited for.
    int issued = 0;
    if (gather && lane == 0) mbar_wait_drain(&bars.kv_full, 0);  // the dQ role copies Q / dO
    int tq_next = (!gather && lane < TPT && lane < ntok) ? toks[lane] : 0;
    for (int i = 0; !gather && i < ntiles; ++i) {
      const int st = i & 1;
      const int n = min(TPT, ntok - i * TPT);
      const int tq = tq_next;
      if (i + 1 < ntiles) {
        const int u2 = (i + 1) * TPT + lane;
        tq_next = (lane < TPT && u2 < ntok) ? toks[u2] : 0;
      }
      bool ok = true;
      if (lane == 0 && i >= 2) ok = mbar_wait(&bars.q_empty[st], ((i >> 1) - 1) & 1, abort_flag, a.status);
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      issued = i + 1;
      if (lane == 0) mbar_arrive_tx(&bars.q_full[st], (uint32_t)(n * a.G * (DQK + DV) * 2));
      __syncwarp();
      if (lane < n) {
        const int row = tq * a.Hq + g * a.G;
        const uint32_t off = (uint32_t)(lane * RPT * 128);
        for (int s = 0; s < DQK / 64; ++s)
          tma_load_2d(sQ + st * PL::kQStage + s * 128 * 128 + off, &mapQ, 64 * s, row, &bars.q_full[st]);
        for (int s = 0; s < DV / 64; ++s)
          tma_load_2d(sDO + st * PL::kDOStage + s * 128 * 128 + off, &mapDO, 64 * s, row, &bars.q_full[st]);
      }
      __syncwarp();
    }
    // drain: before the CTA can exit, every TMA load it issued must have landed
    // (on an abort some stages are never consumed)
    if (lane == 0 && !gather) {
      mbar_wait_drain(&bars.kv_full, 0);
      for (int st = 0; st < 2; ++st) {
        int last = -1;
        for (int i = st; i < issued; i += 2) last = i;
        if (last >= 0) mbar_wait_drain(&bars.q_full[st], (last >> 1) & 1);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idS = idesc_bf16(128, 64, false, false);
      constexpr uint32_t idQ = idesc_bf16(128, WITH_DQ ? DQK : 64, false, true);
      // operand descriptors at the buffers' starts (K-major "k", MN-major "n")
      const uint64_t dKk = sdesc(sK, 16, 1024), dVk = sdesc(sV, 16, 1024), dKn = sdesc(sK, 8192, 1024);
      const uint64_t dPSk = sdesc(sPS, 16, 1024), dPSn = sdesc(sPS, 16384, 1024);
      bool ok = mbar_wait(&bars.kv_full, 0, abort_flag, a.status);
      for (int i = 0; ok && i < ntiles; ++i) {
        const int st = i & 1;
        if (!mbar_wait(&bars.q_full[st], (i >> 1) & 1, abort_flag, a.status)) break;
        tc_fence_after();
        const uint32_t q = sQ + st * PL::kQStage, d = sDO + st * PL::kDOStage;
        const uint64_t dQk = sdesc(q, 16, 1024), dDOk = sdesc(d, 16, 1024);
        const uint64_t dQn = sdesc(q, 16384, 1024), dDOn = sdesc(d, 16384, 1024);
        // S = Q K^T, dP = dO V^T
#pragma unroll
        for (int kk = 0; kk < DQK / 16; ++kk)
          mma_bf16(tmem + PL::cS, desc_add(dQk, (kk >> 2) * 16384 + (kk & 3) * 32),
                   desc_add(dKk, (kk >> 2) * 8192 + (kk & 3) * 32), idS, kk > 0);
#pragma unroll
        for (int kk = 0; kk < DV / 16; ++kk)
          mma_bf16(tmem + PL::cDP, desc_add(dDOk, (kk >> 2) * 16384 + (kk & 3) * 32),
                   desc_add(dVk, (kk >> 2) * 8192 + (kk & 3) * 32), idS, kk > 0);
        mma_commit(&bars.s_full);
        if (!mbar_wait(&bars.p_full, i & 1, abort_flag, a.status)) break;
        tc_fence_after();
        // dV^T += dO^T P
#pragma unroll
        for (int t = 0; t < PL::NV; ++t) {
          const int M = min(128, DV - 128 * t);
          const uint32_t id = idesc_bf16(M, 64, true, true);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_bf16(tmem + PL::cDV + 64 * t, desc_add(dDOn, 2 * t * 16384 + kk * 2048), desc_add(dPSn, kk * 2048), id,
                     (i > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit(&bars.p_free);
        if (!mbar_wait(&bars.ds_full, i & 1, abort_flag, a.status)) break;
        tc_fence_after();
        // dK^T += Q^T dS
#pragma unroll
        for (int t = 0; t < PL::NK; ++t) {
          const int M = min(128, DQK - 128 * t);
          const uint32_t id = idesc_bf16(M, 64, true, true);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_bf16(tmem + ((uint32_t)PL::kDkLane << 16) + PL::cDK + 64 * t, desc_add(dQn, 2 * t * 16384 + kk * 2048),
                     desc_add(dPSn, kk * 2048), id, (i > 0 || kk > 0) ? 1u : 0u);
        }
        if (WITH_DQ) {
          if (i > 0 && !mbar_wait(&bars.dq_free, (i - 1) & 1, abort_flag, a.status)) break;
          tc_fence_after();
          // dQ = dS K_j  (K_j as an MN-major B: N = DQK columns in 64-wide slabs of 64 rows)
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_bf16(tmem + PL::cDQ, desc_add(dPSk, kk * 32), desc_add(dKn, kk * 2048), idQ, kk > 0);
        }
        mma_commit(&bars.q_empty[st]);
        mma_commit(&bars.tile_done);
        if (WITH_DQ) mma_commit(&bars.dq_full);
      }
      mma_commit(&bars.acc_done);
    }
  } else if (warp < 6) {
    // ------------------------------------------------------------ softmax / epilogue
    const int sub = warp & 3;
    const int r = 32 * sub + lane;  // query row of the tile = TMEM lane
    const uint32_t lane_base = tmem + ((uint32_t)(32 * sub) << 16);
    const int u = r / RPT, hh = r - u * RPT;
    bool ok = true;
    // row metadata of tile i (token, lse, Delta), fetched one tile ahead
    int tq_n = 0;
    float lse_n = INFINITY, dlt_n = 0.f;
    auto fetch = [&](int i2) {
      const int n2 = min(TPT, ntok - i2 * TPT);
      tq_n = 0;
      lse_n = INFINITY;
      dlt_n = 0.f;
      if (i2 < ntiles && u < n2 && hh < a.G) {
        tq_n = toks[i2 * TPT + u];
        const long long ih = (long long)tq_n * a.Hq + g * a.G + hh;
        lse_n = __ldg(a.lse + ih);
        dlt_n = __ldg(a.delta + ih);
      }
    };
    fetch(0);
    for (int i = 0; i < ntiles && ok; ++i) {
      const int n = min(TPT, ntok - i * TPT);
      const bool vrow = (u < n) && (hh < a.G);
      const int tq = tq_n;
      const int ta = tq - b * a.S;  // equal query / key lengths (BSND)
      const float lse2 = vrow ? lse_n * kLog2eKv : INFINITY;
      const float dlt = vrow ? dlt_n : 0.f;
      fetch(i + 1);
      // visible key rows of this block for this query row (blk_rows)
      int vlo = 0, vhi = -1;
      if (vrow) blk_rows(j, a.S, ta, a.ori_mask, a.wl, a.wr, &vlo, &vhi);
      if (!mbar_wait(&bars.s_full, i & 1, abort_flag, a.status)) { ok = false; break; }
      tc_fence_after();
      // The P / dS buffer is free once the previous tile's dK^T and dQ MMAs are
      // done; those were committed before this tile's S and dP, so after s_full
      // this wait returns at once.  P goes to shared memory as it is formed; only
      // dS (bf16 pairs) stays in registers until p_free.
      if (i > 0 && !mbar_wait(&bars.tile_done, (i - 1) & 1, abort_flag, a.status)) { ok = false; break; }
      const uint32_t rowaddr = sPS + r * 128;
      uint32_t dk[32];
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        uint32_t sr[2][16], dr[2][16];
#pragma unroll
        for (int c = 0; c < 2; ++c) tmem_ld16(lane_base + PL::cS + 32 * half + 16 * c, sr[c]);
#pragma unroll
        for (int c = 0; c < 2; ++c) tmem_ld16(lane_base + PL::cDP + 32 * half + 16 * c, dr[c]);
        tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          reg_dep16(sr[c]);
          reg_dep16(dr[c]);
        }
        uint32_t pk[16];
#pragma unroll
        for (int c = 0; c < 2; ++c)
#pragma unroll
          for (int e = 0; e < 16; e += 2) {
            float pv[2], dsv[2];
#pragma unroll
            for (int q2 = 0; q2 < 2; ++q2) {
              const int col = 32 * half + 16 * c + e + q2;
              const bool vis = col >= vlo && col <= vhi;
              const float p = vis ? ex2_approx(__uint_as_float(sr[c][e + q2]) * a.scale_log2 - lse2) : 0.f;
              pv[q2] = p;
              dsv[q2] = p * (__uint_as_float(dr[c][e + q2]) - dlt);
            }
            pk[(16 * c + e) >> 1] = pack_bf16(pv[0], pv[1]);
            dk[(32 * half + 16 * c + e) >> 1] = pack_bf16(dsv[0], dsv[1]);
          }
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) {
          const int cc = 4 * half + ch;
          asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};\n" ::"r"(rowaddr + ((cc ^ (r & 7)) << 4)),
                       "r"(pk[4 * ch]), "r"(pk[4 * ch + 1]), "r"(pk[4 * ch + 2]), "r"(pk[4 * ch + 3])
                       : "memory");
        }
      }
      tc_fence_before();
      fence_async_smem();
      mbar_arrive(&bars.p_full);
      if (!mbar_wait(&bars.p_free, i & 1, abort_flag, a.status)) { ok = false; break; }
#pragma unroll
      for (int ch = 0; ch < 8; ++ch)
        asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};\n" ::"r"(rowaddr + ((ch ^ (r & 7)) << 4)),
                     "r"(dk[4 * ch]), "r"(dk[4 * ch + 1]), "r"(dk[4 * ch + 2]), "r"(dk[4 * ch + 3])
                     : "memory");
      fence_async_smem();
      mbar_arrive(&bars.ds_full);
    }
    // ---- epilogue, part 1: dV^T and dK^T from TMEM into shared memory as fp32
    // [key][dim] rows (the Q / dO stages are idle once acc_done has fired)
    if (ok && mbar_wait(&bars.acc_done, 0, abort_flag, a.status)) {
      tc_fence_after();
      float* stV = reinterpret_cast<float*>(smem + PL::oStV);
      float* stK = reinterpret_cast<float*>(smem + PL::oStK);
      if constexpr (PL::kPack) {
        // one pass: lanes 0..15 hold dV^T rows, lanes 16..31 dK^T rows (lane offset 16)
        float* dst = (lane < 16 ? stV : stK) + 16 * sub + (lane & 15);
#pragma unroll
        for (int c = 0; c < 64; c += 16) {
          uint32_t v[16];
          tmem_ld16(lane_base + PL::cDV + c, v);
          tmem_wait_ld();
          reg_dep16(v);
#pragma unroll
          for (int e = 0; e < 16; ++e) dst[(c + e) * 64] = __uint_as_float(v[e]);
        }
      } else {
        for (int which = 0; which < 2; ++which) {
          const int D = which == 0 ? DV : DQK;
          const int ntile = which == 0 ? PL::NV : PL::NK;
          const int cbase = which == 0 ? PL::cDV : PL::cDK;
          float* st = which == 0 ? stV : stK;
          for (int t = 0; t < ntile; ++t) {
            const int M = min(128, D - 128 * t);
            int dim = -1;
            if (M == 128) dim = 128 * t + 32 * sub + lane;
            else if (lane < 16) dim = 128 * t + 16 * sub + lane;
#pragma unroll 1
            for (int c = 0; c < 64; c += 16) {
              uint32_t v[16];
              tmem_ld16(lane_base + cbase + 64 * t + c, v);
              tmem_wait_ld();
              reg_dep16(v);
              if (dim >= 0) {
#pragma unroll
                for (int e = 0; e < 16; ++e) st[(c + e) * D + dim] = __uint_as_float(v[e]);
              }
            }
          }
        }
      }
    }
    tc_fence_before();
  } else if (WITH_DQ) {
    // ------------------------------------------------------------ dQ epilogue (warps 6..9)
    // reads each tile's dQ partial from TMEM and adds it (scaled) to the fp32 dQ
    // accumulator with vector atomics, overlapping the next tile's softmax
    const int sub = warp & 3;
    const int r = 32 * sub + lane;
    const uint32_t lane_base = tmem + ((uint32_t)(32 * sub) << 16);
    // row gather: these threads also copy the tiles' Q / dO rows, two stages ahead;
    // a stage is announced (128 arrivals) once its copies have landed and are
    // fenced for the tensor core
    auto gather_tile = [&](int i2) {
      const int st = i2 & 1, rows = min(TPT, ntok - i2 * TPT) << a.log2_G;
      kv_gather_rows<DQK, 128>(sQ + st * PL::kQStage, a.q, toks + i2 * TPT, rows, a.log2_G, a.Hq, g * a.G, r);
      kv_gather_rows<DV, 128>(sDO + st * PL::kDOStage, a.d_o, toks + i2 * TPT, rows, a.log2_G, a.Hq, g * a.G, r);
      cp_async_commit();
    };
    auto announce = [&](int i2) {
      fence_async_smem();
      mbar_arrive(&bars.q_full[i2 & 1]);
    };
    if (gather) {
      if (ntiles > 0) gather_tile(0);
      if (ntiles > 1) {
        gather_tile(1);
        cp_async_wait_prev();
      } else {
        cp_async_wait_none();
      }
      if (ntiles > 0) announce(0);
      if (ntiles > 1) {
        cp_async_wait_none();
        announce(1);
      }
    }
    // The atomics go out coalesced: each 16-column slice of a warp's 32 rows passes
    // through shared memory, so that a reduction covers 8 rows x 64 contiguous bytes
    // instead of 32 rows x 16 bytes (a quarter of the L1 / L2 requests).  Lane l
    // stages its row, then adds 16-byte piece (l & 3) of the warp's rows (l >> 2) + 8 k.
    const uint32_t sq = smem_u32(smem + PL::oDQS) + sub * (32 * 64);
    const int pq = lane & 3;
    for (int i = 0; i < ntiles; ++i) {
      // the warp leaves together if any lane's wait gave up (the lanes exchange
      // data below)
      if (!__all_sync(0xffffffffu, mbar_wait(&bars.dq_full, i & 1, abort_flag, a.status))) break;
      tc_fence_after();
      const int n = min(TPT, ntok - i * TPT);
      // a CTA with one tile has no next tile to overlap: its lanes add their own rows
      // directly (shorter latency); otherwise the coalesced slices keep the memory
      // pipeline free for the next tile's softmax
      const bool staged = ntiles > 1;
      float* own = nullptr;
      {
        const int u0 = r / RPT, h0 = r - u0 * RPT;
        if (u0 < n && h0 < a.G) own = a.dq_acc + ((long long)toks[i * TPT + u0] * a.Hq + g * a.G + h0) * DQK;
      }
      float* rowp[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int rho = 32 * sub + (lane >> 2) + 8 * k, uu = rho / RPT, h2 = rho - uu * RPT;
        rowp[k] = (uu < n && h2 < a.G) ? a.dq_acc + ((long long)toks[i * TPT + uu] * a.Hq + g * a.G + h2) * DQK
                                       : nullptr;
      }
      // one 16-column slice: stage this lane's row, then add 16-byte pieces of four rows
      auto stage_and_add = [&](int c, const uint32_t (&v)[16]) {
        if (!staged) {
          if (own) {
#pragma unroll
            for (int e = 0; e < 16; e += 4)
              red_add_v4(own + c + e, __uint_as_float(v[e]) * a.scale, __uint_as_float(v[e + 1]) * a.scale,
                         __uint_as_float(v[e + 2]) * a.scale, __uint_as_float(v[e + 3]) * a.scale);
          }
          return;
        }
#pragma unroll
        for (int q2 = 0; q2 < 4; ++q2)
          asm volatile("st.shared.v4.f32 [%0], {%1, %2, %3, %4};\n" ::"r"(
                           sq + lane * 64 + ((q2 ^ ((lane >> 1) & 3)) << 4)),
                       "f"(__uint_as_float(v[4 * q2]) * a.scale), "f"(__uint_as_float(v[4 * q2 + 1]) * a.scale),
                       "f"(__uint_as_float(v[4 * q2 + 2]) * a.scale), "f"(__uint_as_float(v[4 * q2 + 3]) * a.scale)
                       : "memory");
        __syncwarp();
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const int rl = (lane >> 2) + 8 * k;  // row within the warp's 32
          float x0, x1, x2, x3;
          asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];\n"
                       : "=f"(x0), "=f"(x1), "=f"(x2), "=f"(x3)
                       : "r"(sq + rl * 64 + ((pq ^ ((rl >> 1) & 3)) << 4))
                       : "memory");
          if (rowp[k]) red_add_v4(rowp[k] + c + 4 * pq, x0, x1, x2, x3);
        }
        __syncwarp();
      };
      // TMEM reads run one slice ahead of the staging; the accumulator goes back to
      // the MMA warp as soon as its last slice is in registers
      uint32_t v0[16], v1[16];
      tmem_ld16(lane_base + PL::cDQ, v0);
#pragma unroll 1
      for (int c = 0; c < DQK; c += 32) {
        tmem_wait_ld();
        reg_dep16(v0);
        tmem_ld16(lane_base + PL::cDQ + c + 16, v1);
        stage_and_add(c, v0);
        tmem_wait_ld();
        reg_dep16(v1);
        if (c + 32 < DQK) {
          tmem_ld16(lane_base + PL::cDQ + c + 32, v0);
        } else {
          tc_fence_before();
          mbar_arrive(&bars.dq_free);
        }
        stage_and_add(c + 16, v1);
      }
      if (gather && i + 2 < ntiles) {
        // dq_full(i) came after every MMA of tile i: its stage is free
        gather_tile(i + 2);
        cp_async_wait_none();
        announce(i + 2);
      }
    }
    cp_async_wait_none();  // nothing in flight when the CTA leaves
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, PL::kAlloc);
    tmem_relinquish();
  }
  // ---- epilogue, part 2: every thread adds the staged dV^T / dK^T (scaled) to the
  // fp32 accumulators, four consecutive dims per vector reduction
  if (!bars.abort_flag) {
    // the item again (shared): keeps its fields out of registers through the roles above
    int b2, g2, j2;
    kv_list_decode(a, bars.item.L, &b2, &g2, &j2);
    const long long kv_row0 = (long long)b2 * a.S + 64 * j2;
    const int nrows = min(64, a.S - 64 * j2);
    const float4* stV = reinterpret_cast<const float4*>(smem + PL::oStV);
    const float4* stK = reinterpret_cast<const float4*>(smem + PL::oStK);
    for (int i = threadIdx.x; i < 16 * DV; i += blockDim.x) {
      const int key = i / (DV / 4), d4 = i - key * (DV / 4);
      if (key < nrows) {
        const float4 x = stV[i];
        red_add_v4(a.dv_acc + ((kv_row0 + key) * a.Hkv + g2) * DV + 4 * d4, x.x, x.y, x.z, x.w);
      }
    }
    for (int i = threadIdx.x; i < 16 * DQK; i += blockDim.x) {
      const int key = i / (DQK / 4), d4 = i - key * (DQK / 4);
      if (key < nrows) {
        const float4 x = stK[i];
        red_add_v4(a.dk_acc + ((kv_row0 + key) * a.Hkv + g2) * DQK + 4 * d4, x.x * a.scale, x.y * a.scale,
                   x.z * a.scale, x.w * a.scale);
      }
    }
  }
}

// ---------------------------------------------------------------------------
// inverse index: for every (batch, token window, kv-head, block) the tokens
// of the window that select the block
// ---------------------------------------------------------------------------
// The list that slot e joins (false when the slot is unusable); *oor is raised
// when the slot is usable by length but names a block past its sequence.
__device__ __forceinline__ bool kv_slot_list(const KvIndexArgs& a, long long e, int* list, int* tq_out, bool* oor) {
  int slot, tq, g;
  long long ug;
  if (a.n_slots <= 0x7fffffffll) {  // 32-bit index arithmetic when it fits
    const int e32 = (int)e, u32 = e32 / a.topk;
    slot = e32 - u32 * a.topk;
    tq = u32 / a.Hkv;
    g = u32 - tq * a.Hkv;
    ug = u32;
  } else {
    slot = (int)(e % a.topk);
    ug = e / a.topk;
    tq = (int)(ug / a.Hkv);
    g = (int)(ug - (long long)tq * a.Hkv);
  }
  if (a.ori_len && slot >= __ldg(a.ori_len + ug)) return false;
  const int b = tq / a.S;
  const int x = __ldg(a.ori_idx + e);
  if (x >= 0 && (long long)x * kTileRows >= a.S) *oor = true;
  const int L = kv_block_list(a, x, b, tq - b * a.S, g);
  if (L < 0) return false;
  *list = L;
  *tq_out = tq;
  return true;
}

// Small problems (fewer than 2^31 slots): the same with 32-bit index arithmetic only.
__device__ __forceinline__ int kv_slot_list32(const KvIndexArgs& a, int e, int* tq_out, bool* oor) {
  const int ug = e / a.topk, slot = e - ug * a.topk;
  const int tq = ug / a.Hkv, g = ug - tq * a.Hkv;
  if (a.ori_len && slot >= __ldg(a.ori_len + ug)) return -1;
  const int b = tq / a.S;
  *tq_out = tq;
  const int x = __ldg(a.ori_idx + e);
  if (x >= 0 && (long long)x * kTileRows >= a.S) *oor = true;
  return kv_block_list(a, x, b, tq - b * a.S, g);
}

__global__ void kv_count_kernel(const KvIndexArgs a) {
  pdl_wait();
  pdl_trigger();
  long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= a.n_slots) return;
  int list, tq;
  bool oor = false;
  if (kv_slot_list(a, e, &list, &tq, &oor)) atomicAdd(a.counts + list, 1);
  if (oor && a.status) atomicOr(a.status, kStatusIndexRange);
}

__global__ void kv_fill_kernel(const KvIndexArgs a) {
  pdl_wait();
  pdl_trigger();
  long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= a.n_slots) return;
  int list, tq;
  bool oor = false;
  if (kv_slot_list(a, e, &list, &tq, &oor)) {
    int pos = atomicAdd(a.cursor + list, 1);
    a.entries[__ldg(a.list_off + list) + pos] = tq;
  }
}

// Exclusive scans of the list counts -> list offsets, and of the lists' chunk
// counts -> the work-item table (one item per chunk of a list).  Run by a whole
// CTA of 1024 threads.
__device__ void kv_scan_lists(const KvIndexArgs& a, const int* counts) {
  __shared__ int warp_tot[2][32];
  __shared__ int carry[2];
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  if (tid == 0) carry[0] = carry[1] = 0;
  __syncthreads();
  for (int base = 0; base < a.n_lists; base += 1024) {
    const int i = base + tid;
    int c = i < a.n_lists ? counts[i] : 0;
    int k = (c + a.chunk_tokens - 1) / a.chunk_tokens;
    int xc = c, xk = k;  // inclusive warp scans
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int yc = __shfl_up_sync(0xffffffffu, xc, o), yk = __shfl_up_sync(0xffffffffu, xk, o);
      if (lane >= o) { xc += yc; xk += yk; }
    }
    if (lane == 31) { warp_tot[0][wid] = xc; warp_tot[1][wid] = xk; }
    __syncthreads();
    if (wid == 0) {
      int tc = warp_tot[0][lane], tk = warp_tot[1][lane];
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        int yc = __shfl_up_sync(0xffffffffu, tc, o), yk = __shfl_up_sync(0xffffffffu, tk, o);
        if (lane >= o) { tc += yc; tk += yk; }
      }
      warp_tot[0][lane] = tc;
      warp_tot[1][lane] = tk;
    }
    __syncthreads();
    const int pc = (wid ? warp_tot[0][wid - 1] : 0) + xc - c + carry[0];
    const int pk = (wid ? warp_tot[1][wid - 1] : 0) + xk - k + carry[1];
    if (i < a.n_lists) {
      a.list_off[i] = pc;
      // the list's work items: consecutive chunks of its entries
      for (int q = 0; q < k; ++q) {
        const int first = q * a.chunk_tokens;
        a.items[pk + q] = make_int4(i, pc + first, min(a.chunk_tokens, c - first), 0);
      }
    }
    __syncthreads();
    if (tid == 1023) { carry[0] = pc + c; carry[1] = pk + k; }
    __syncthreads();
  }
  if (tid == 0) {
    a.list_off[a.n_lists] = carry[0];
    *a.work_count = carry[1];
  }
}

__global__ void __launch_bounds__(1024) kv_scan_kernel(const KvIndexArgs a) {
  pdl_wait();
  pdl_trigger();
  kv_scan_lists(a, a.counts);
}

// Small problems: one launch builds the bucketed index, clears the workspace's
// accumulators and forms Delta = rowsum(dO o O).  CTA b < n_buckets takes slots
// [b * 512, (b + 1) * 512): it ranks each valid slot within its list in the
// bucket (shared-memory counters, one atomic per list and warp), lays the
// bucket's lists out back to back, and publishes their counts and offsets.
// The other CTAs clear and form Delta.
__global__ void __launch_bounds__(kBucketSlots) kv_prep_small_kernel(const KvIndexArgs a, const KvPrepArgs p) {
  pdl_wait();
  pdl_trigger();
  if ((int)blockIdx.x < a.n_buckets) {
    extern __shared__ int sh[];
    int* cnt = sh;             // [n_lists]
    int* off = sh + a.n_lists;  // [n_lists]
    const int nl = a.n_lists, bk = blockIdx.x, lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    for (int i = threadIdx.x; i < nl; i += blockDim.x) cnt[i] = 0;
    const int e = bk * kBucketSlots + threadIdx.x;
    int tq = 0;
    bool oor = false;
    const int L = e < a.n_slots ? kv_slot_list32(a, e, &tq, &oor) : -1;
    // the bucket's out-of-range flag, written whole every call (the status word itself
    // is cleared by CTA 0 below, so the main kernel folds the flags into it)
    const int any_oor = __syncthreads_or(oor);
    if (threadIdx.x == 0) a.bucket_flag[bk] = any_oor;
    const unsigned peers = __match_any_sync(0xffffffffu, L);
    const int leader = __ffs(peers) - 1;
    int rank = 0;
    if (L >= 0 && lane == leader) rank = atomicAdd(cnt + L, __popc(peers));
    rank = __shfl_sync(0xffffffffu, rank, leader) + __popc(peers & ((1u << lane) - 1));
    __syncthreads();
    if (warp == 0) {
      int carry = 0;
      for (int l0 = 0; l0 < nl; l0 += 32) {
        const int l = l0 + lane;
        const int c = l < nl ? cnt[l] : 0;
        int incl = c;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int y = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += y;
        }
        if (l < nl) {
          off[l] = carry + incl - c;
          a.bucket_cnt[bk * nl + l] = c;
          a.bucket_off[bk * nl + l] = carry + incl - c;
        }
        carry += __shfl_sync(0xffffffffu, incl, 31);
      }
    }
    __syncthreads();
    if (L >= 0) a.entries[bk * kBucketSlots + off[L] + rank] = tq;
    if (bk == 0 && threadIdx.x == 0) *p.status = 0;
    return;
  }
  const long long nthreads = (long long)(gridDim.x - a.n_buckets) * blockDim.x;
  const long long t0 = (long long)(blockIdx.x - a.n_buckets) * blockDim.x + threadIdx.x;
  for (long long i = t0; i < p.zero_n16; i += nthreads) p.zero[i] = make_float4(0.f, 0.f, 0.f, 0.f);
  const int lane = threadIdx.x & 31;
  for (long long row = t0 >> 5; row < p.rows; row += nthreads >> 5) {
    const float d = warp_row_dot_bf16(p.o + row * p.dv, p.d_o + row * p.dv, p.dv, lane);
    if (lane == 0) p.delta[row] = d;
  }
}

// Inspection: walks every work item exactly as kv_bwd_kernel does (kv_get_item,
// kv_list_decode) and records, per (item, token), the block and its visible row
// range (blk_rows): {token * Hkv + kv-head, block, lo, hi}.
__global__ void __launch_bounds__(128) kv_debug_walk_kernel(const KvArgs a, int4* rec, long long max_rec,
                                                            int* n_rec) {
  __shared__ KvItem item;
  __shared__ int toks_smem[kBucketMaxChunk];
  const int* toks = kv_get_item(a, blockIdx.x, toks_smem, item);
  __syncthreads();
  if (item.L < 0) return;
  int b, g, j;
  kv_list_decode(a, item.L, &b, &g, &j);
  for (int r = threadIdx.x; r < item.ntok; r += blockDim.x) {
    const int tq = toks[r];
    int lo, hi;
    blk_rows(j, a.S, tq - b * a.S, a.ori_mask, a.wl, a.wr, &lo, &hi);
    const int k = atomicAdd(n_rec, 1);
    if (k < max_rec) rec[k] = make_int4(tq * a.Hkv + g, j, lo, hi);
  }
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
bool kv_path_built(int dqk, int dv) {
  return (dqk == 64 && dv == 64) || (dqk == 128 && dv == 128) || (dqk == 192 && dv == 128);
}

template <int DQK, int DV, bool WITH_DQ>
static cudaError_t kv_launch_t(const KvLaunch& L, cudaStream_t st) {
  using PL = KvPlan<DQK, DV, WITH_DQ>;
  CUtensorMap mq, mdo, mk, mv;
  const KvArgs& a = L.args;
  if (!make_tmap_bf16(&mq, L.q, (uint64_t)L.Tq * a.Hq, DQK, (uint64_t)DQK * 2, a.G) ||
      !make_tmap_bf16(&mdo, L.d_o, (uint64_t)L.Tq * a.Hq, DV, (uint64_t)DV * 2, a.G) ||
      !make_tmap_bf16(&mk, L.k, (uint64_t)L.Tkv, (uint64_t)a.Hkv * DQK, (uint64_t)a.Hkv * DQK * 2, 64) ||
      !make_tmap_bf16(&mv, L.v, (uint64_t)L.Tkv, (uint64_t)a.Hkv * DV, (uint64_t)a.Hkv * DV * 2, 64))
    return cudaErrorInvalidValue;
  auto k = kv_bwd_kernel<DQK, DV, WITH_DQ>;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, PL::kSmem);
  if (e != cudaSuccess) return e;
  if (L.max_work == 0) return cudaSuccess;
  mark_begin(st, kTimeBwdKV);
  e = launch_pdl(k, (unsigned)L.max_work, WITH_DQ ? 320 : 192, PL::kSmem, st, mq, mdo, mk, mv, a);
  count_launch();
  mark_end(st, kTimeBwdKV);
  return e;
}

int kv_bucket_count(long long n_slots) { return (int)((n_slots + kBucketSlots - 1) / kBucketSlots); }

bool kv_bucketed_fits(long long n_slots, int n_lists, int chunk) {
  const long long nb = kv_bucket_count(n_slots);
  return nb >= 1 && nb <= kBucketMax && n_lists <= kBucketMaxLists && nb * n_lists <= kBucketMaxCells &&
         chunk <= kBucketMaxChunk;
}

cudaError_t launch_kv_prep_small(const KvIndexArgs& a, const KvPrepArgs& p, cudaStream_t st) {
  if (a.n_buckets < 1 || !kv_bucketed_fits(a.n_slots, a.n_lists, a.chunk_tokens)) return cudaErrorInvalidValue;
  long long work = (p.rows + kBucketSlots / 32 - 1) / (kBucketSlots / 32);  // one warp per Delta row
  long long zw = (p.zero_n16 + kBucketSlots - 1) / kBucketSlots;
  if (zw > work) work = zw;
  if (work < 1) work = 1;
  if (work > 148 - a.n_buckets) work = 148 - a.n_buckets;
  const size_t shm = sizeof(int) * 2 * (size_t)a.n_lists;
  cudaError_t e = launch_pdl(kv_prep_small_kernel, (unsigned)(a.n_buckets + work), kBucketSlots, shm, st, a, p);
  count_launch();
  return e;
}

cudaError_t launch_kv_index(const KvIndexArgs& a, cudaStream_t st) {
  // counts and cursor arrive zeroed (cleared with the rest of the workspace)
  cudaError_t e = cudaSuccess;
  if (a.n_slots > 0) {
    e = launch_pdl(kv_count_kernel, (unsigned)((a.n_slots + 255) / 256), 256, 0, st, a);
    count_launch();
    if (e != cudaSuccess) return e;
  }
  e = launch_pdl(kv_scan_kernel, 1, 1024, 0, st, a);
  count_launch();
  if (e != cudaSuccess) return e;
  if (a.n_slots > 0) {
    e = launch_pdl(kv_fill_kernel, (unsigned)((a.n_slots + 255) / 256), 256, 0, st, a);
    count_launch();
  }
  return e;
}

cudaError_t launch_kv_debug_walk(const KvArgs& a, long long max_work, int4* rec, long long max_rec, int* n_rec,
                                 cudaStream_t st) {
  if (max_work == 0) return cudaSuccess;
  kv_debug_walk_kernel<<<(unsigned)max_work, 128, 0, st>>>(a, rec, max_rec, n_rec);
  count_launch();
  return cudaGetLastError();
}

cudaError_t launch_kv_bwd(const KvLaunch& L, bool with_dq, cudaStream_t st) {
  const int dqk = L.dqk, dv = L.dv;
  if (dqk == 64 && dv == 64) return with_dq ? kv_launch_t<64, 64, true>(L, st) : kv_launch_t<64, 64, false>(L, st);
  if (dqk == 128 && dv == 128)
    return with_dq ? kv_launch_t<128, 128, true>(L, st) : kv_launch_t<128, 128, false>(L, st);
  if (dqk == 192 && dv == 128)
    return with_dq ? kv_launch_t<192, 128, true>(L, st) : kv_launch_t<192, 128, false>(L, st);
  return cudaErrorInvalidValue;
}

}  // namespace sa
