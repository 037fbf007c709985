// sa_kv_bwd.cu -- key-stationary backward for block-level selection (BSND):
// dK and dV accumulate in TMEM per selected KV block, with no per-token
// scatter.
//
// aclnnSparseFlashAttentionGrad "Formula" Phases 1-3 (dV = P^T dO,
// dS = P o (dP - rowsum(dO o O)), dK = dS^T Q scale), restructured around
// the KV block: an inverse index lists, for every (batch, kv-head, block),
// the query tokens whose selection names the block; one CTA takes a chunk of
// that list and streams the tokens' query rows through the block in tiles of
// 128 rows (128 / RPT tokens, RPT = G rounded up to a multiple of 8).
//
// Per tile (tcgen05, bf16 operands, fp32 TMEM accumulators):
//   S   [128 x 64]  = Q K_j^T             (A = Q K-major, B = K_j K-major)
//   dP  [128 x 64]  = dO V_j^T            (A = dO K-major, B = V_j K-major)
//   P = exp2(S * scale * log2e - lse * log2e), dS = P o (dP - Delta)   (softmax warps)
//   dV^T [DV x 64] += dO^T P              (A = dO MN-major, B = P MN-major)
//   dK^T [DQK x 64] += Q^T dS             (A = Q MN-major, B = dS MN-major)
//   dQ  [128 x DQK] = dS K_j              (optional; A = dS K-major, B = K_j MN-major),
//                      added to an fp32 dQ accumulator with vector atomics.
// At the end dK^T / dV^T (scaled) are added to the fp32 dK / dV accumulators;
// blocks split into several chunks meet there.
//
// Warp roles: 0 = TMA producer, 1 = MMA issuer + TMEM owner, 2..5 = softmax /
// dK-dV epilogue (thread = query row = TMEM lane), 6..9 (with dQ) = dQ epilogue.
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
  static constexpr int kBytes = oPS + 128 * 128;
  static constexpr int kSmem = kBytes + 1024;      // + alignment slack
  static constexpr int NV = (DV + 127) / 128;      // M tiles of dV^T
  static constexpr int NK = (DQK + 127) / 128;     // M tiles of dK^T
  static constexpr int cS = 0, cDP = 64, cDV = 128, cDK = cDV + 64 * NV, cDQ = cDK + 64 * NK;
  static constexpr int kCols = cDQ + (WITH_DQ ? DQK : 0);
  static constexpr uint32_t kAlloc = kCols <= 256 ? 256 : 512;
  static_assert(kCols <= 512, "TMEM plan too large");
  static_assert(kSmem <= 227 * 1024, "shared memory plan too large");
};

struct KvBars {
  uint64_t kv_full, q_full[2], q_empty[2], s_full, p_full, p_free, ds_full, tile_done, acc_done, dq_full, dq_free;
  uint32_t tmem_base;
  int abort_flag;
};

__device__ __forceinline__ void red_add_v4(float* addr, float a, float b, float c, float d) {
  asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};\n" ::"l"(addr), "f"(a), "f"(b), "f"(c), "f"(d)
               : "memory");
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
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // ---- which work item: (list, chunk) ----
  const int w = blockIdx.x;
  if (w >= *a.work_count) return;
  if (a.status && (*(volatile int*)a.status & kStatusTimeout)) return;  // another CTA gave up
  int lo = 0, hi = a.n_lists - 1;  // largest list L with chunk_off[L] <= w
  while (lo < hi) {
    int mid = (lo + hi + 1) >> 1;
    if (__ldg(a.chunk_off + mid) <= w) lo = mid; else hi = mid - 1;
  }
  const int L = lo;
  const int chunk = w - __ldg(a.chunk_off + L);
  // list id = ((batch * nwin + window) * Hkv + kv-head) * nblk + block
  const int j = L % a.nblk;
  const int rest = L / a.nblk;
  const int g = rest % a.Hkv, b = (rest / a.Hkv) / a.nwin;
  const int list_begin = __ldg(a.list_off + L), list_end = __ldg(a.list_off + L + 1);
  const int tok0 = list_begin + chunk * a.chunk_tokens;
  const int ntok = min(a.chunk_tokens, list_end - tok0);
  const int TPT = a.TPT, RPT = a.RPT;
  const int ntiles = (ntok + TPT - 1) / TPT;
  const int* toks = a.entries + tok0;

  const uint32_t sQ = smem_u32(smem + PL::oQ), sDO = smem_u32(smem + PL::oDO);
  const uint32_t sK = smem_u32(smem + PL::oK), sV = smem_u32(smem + PL::oV);
  const uint32_t sPS = smem_u32(smem + PL::oPS);
  volatile int* abort_flag = &bars.abort_flag;

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
      mbar_init(&bars.q_full[s], 1);
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
  }
  if (warp == 1) tmem_alloc(&bars.tmem_base, PL::kAlloc);
  fence_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars.tmem_base;

  if (warp == 0) {
    // ------------------------------------------------------------ producer (whole warp)
    // lane u issues the TMA loads of token u of the tile; the next tile's token
    // ids are fetched while the current stage is being waited for.
    const int row0 = b * a.S + 64 * j;
    if (lane == 0) {
      tma_prefetch_desc(&mapQ);
      tma_prefetch_desc(&mapDO);
      mbar_arrive_tx(&bars.kv_full, (uint32_t)(64 * (DQK + DV) * 2));
      for (int s = 0; s < DQK / 64; ++s) tma_load_2d(sK + s * 64 * 128, &mapK, g * DQK + 64 * s, row0, &bars.kv_full);
      for (int s = 0; s < DV / 64; ++s) tma_load_2d(sV + s * 64 * 128, &mapV, g * DV + 64 * s, row0, &bars.kv_full);
    }
    int issued = 0;
    int tq_next = (lane < TPT && lane < ntok) ? __ldg(toks + lane) : 0;
    for (int i = 0; i < ntiles; ++i) {
      const int st = i & 1;
      const int n = min(TPT, ntok - i * TPT);
      const int tq = tq_next;
      if (i + 1 < ntiles) {
        const int u2 = (i + 1) * TPT + lane;
        tq_next = (lane < TPT && u2 < ntok) ? __ldg(toks + u2) : 0;
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
    if (lane == 0) {
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
      bool ok = mbar_wait(&bars.kv_full, 0, abort_flag, a.status);
      for (int i = 0; ok && i < ntiles; ++i) {
        const int st = i & 1;
        if (!mbar_wait(&bars.q_full[st], (i >> 1) & 1, abort_flag, a.status)) break;
        tc_fence_after();
        const uint32_t q = sQ + st * PL::kQStage, d = sDO + st * PL::kDOStage;
        // S = Q K^T, dP = dO V^T
        for (int kk = 0; kk < DQK / 16; ++kk)
          mma_bf16(tmem + PL::cS, sdesc(q + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024),
                   sdesc(sK + (kk >> 2) * 8192 + (kk & 3) * 32, 16, 1024), idS, kk > 0);
        for (int kk = 0; kk < DV / 16; ++kk)
          mma_bf16(tmem + PL::cDP, sdesc(d + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024),
                   sdesc(sV + (kk >> 2) * 8192 + (kk & 3) * 32, 16, 1024), idS, kk > 0);
        mma_commit(&bars.s_full);
        if (!mbar_wait(&bars.p_full, i & 1, abort_flag, a.status)) break;
        tc_fence_after();
        // dV^T += dO^T P
        for (int t = 0; t < PL::NV; ++t) {
          const int M = min(128, DV - 128 * t);
          const uint32_t id = idesc_bf16(M, 64, true, true);
          for (int kk = 0; kk < 8; ++kk)
            mma_bf16(tmem + PL::cDV + 64 * t, sdesc(d + 2 * t * 16384 + kk * 2048, 16384, 1024),
                     sdesc(sPS + kk * 2048, 16384, 1024), id, (i > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit(&bars.p_free);
        if (!mbar_wait(&bars.ds_full, i & 1, abort_flag, a.status)) break;
        tc_fence_after();
        // dK^T += Q^T dS
        for (int t = 0; t < PL::NK; ++t) {
          const int M = min(128, DQK - 128 * t);
          const uint32_t id = idesc_bf16(M, 64, true, true);
          for (int kk = 0; kk < 8; ++kk)
            mma_bf16(tmem + PL::cDK + 64 * t, sdesc(q + 2 * t * 16384 + kk * 2048, 16384, 1024),
                     sdesc(sPS + kk * 2048, 16384, 1024), id, (i > 0 || kk > 0) ? 1u : 0u);
        }
        if (WITH_DQ) {
          if (i > 0 && !mbar_wait(&bars.dq_free, (i - 1) & 1, abort_flag, a.status)) break;
          tc_fence_after();
          // dQ = dS K_j  (K_j as an MN-major B: N = DQK columns in 64-wide slabs of 64 rows)
          for (int kk = 0; kk < 4; ++kk)
            mma_bf16(tmem + PL::cDQ, sdesc(sPS + kk * 32, 16, 1024), sdesc(sK + kk * 2048, 8192, 1024), idQ,
                     kk > 0);
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
    const int blk_row0 = 64 * j;
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
        tq_n = __ldg(toks + i2 * TPT + u);
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
      // visible key rows of this block for this query row
      int vlo = 0, vhi = -1;
      if (vrow) {
        vlo = 0;
        vhi = min(63, a.S - 1 - blk_row0);
        if (a.ori_mask == kMaskCausal) {
          vhi = min(vhi, ta - blk_row0);
        } else if (a.ori_mask == kMaskBand) {
          vhi = (int)min((long long)vhi, (long long)ta + a.wr - blk_row0);
          vlo = (int)max((long long)vlo, (long long)ta - a.wl - blk_row0);
        }
      }
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
              const float p = vis ? exp2f(__uint_as_float(sr[c][e + q2]) * a.scale_log2 - lse2) : 0.f;
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
    // ---- epilogue: dV^T and dK^T (scaled) into the fp32 accumulators
    if (ok && mbar_wait(&bars.acc_done, 0, abort_flag, a.status)) {
      tc_fence_after();
      const long long kv_row0 = (long long)b * a.S + blk_row0;
      const int nrows = min(64, a.S - blk_row0);
      for (int which = 0; which < 2; ++which) {
        const int D = which == 0 ? DV : DQK;
        const int ntile = which == 0 ? PL::NV : PL::NK;
        const int cbase = which == 0 ? PL::cDV : PL::cDK;
        float* acc = which == 0 ? a.dv_acc : a.dk_acc;
        const float mul = which == 0 ? 1.f : a.scale;
        for (int t = 0; t < ntile; ++t) {
          const int M = min(128, D - 128 * t);
          int dim = -1;
          if (M == 128) dim = 128 * t + 32 * sub + lane;
          else if (lane < 16) dim = 128 * t + 16 * sub + lane;
          for (int c = 0; c < 64; c += 16) {
            uint32_t v[16];
            tmem_ld16(lane_base + cbase + 64 * t + c, v);
            tmem_wait_ld();
            reg_dep16(v);
            if (dim >= 0) {
#pragma unroll
              for (int e = 0; e < 16; ++e) {
                if (c + e < nrows)
                  atomicAdd(acc + ((kv_row0 + c + e) * a.Hkv + g) * D + dim, __uint_as_float(v[e]) * mul);
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
    const int u = r / RPT, hh = r - u * RPT;
    int tq_n = (u < min(TPT, ntok) && hh < a.G) ? __ldg(toks + u) : -1;
    for (int i = 0; i < ntiles; ++i) {
      const int tq = tq_n;
      const int n2 = min(TPT, ntok - (i + 1) * TPT);
      tq_n = (i + 1 < ntiles && u < n2 && hh < a.G) ? __ldg(toks + (i + 1) * TPT + u) : -1;
      if (!mbar_wait(&bars.dq_full, i & 1, abort_flag, a.status)) break;
      tc_fence_after();
      float* dst = a.dq_acc + ((long long)(tq < 0 ? 0 : tq) * a.Hq + g * a.G + hh) * DQK;
#pragma unroll 1
      for (int c = 0; c < DQK; c += 16) {
        uint32_t v[16];
        tmem_ld16(lane_base + PL::cDQ + c, v);
        tmem_wait_ld();
        reg_dep16(v);
        if (tq >= 0) {
#pragma unroll
          for (int e = 0; e < 16; e += 4)
            red_add_v4(dst + c + e, __uint_as_float(v[e]) * a.scale, __uint_as_float(v[e + 1]) * a.scale,
                       __uint_as_float(v[e + 2]) * a.scale, __uint_as_float(v[e + 3]) * a.scale);
        }
      }
      tc_fence_before();
      mbar_arrive(&bars.dq_free);
    }
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, PL::kAlloc);
    tmem_relinquish();
  }
}

// ---------------------------------------------------------------------------
// inverse index: for every (batch, token window, kv-head, block) the tokens
// of the window that select the block
// ---------------------------------------------------------------------------
__device__ __forceinline__ bool kv_slot_list(const KvIndexArgs& a, long long e, int* list, int* tq_out) {
  const int slot = (int)(e % a.topk);
  const long long ug = e / a.topk;
  const int tq = (int)(ug / a.Hkv), g = (int)(ug - (long long)tq * a.Hkv);
  if (a.ori_len && slot >= __ldg(a.ori_len + ug)) return false;
  const int x = __ldg(a.ori_idx + e);
  if (x < 0) return false;
  const long long first = (long long)x * 64;
  if (first >= a.S) return false;
  const int b = tq / a.S;
  const int ta = tq - b * a.S;
  // the block must keep at least one visible row for this token
  if (a.ori_mask == kMaskCausal && first > ta) return false;
  if (a.ori_mask == kMaskBand) {
    long long last = min(first + 63, (long long)a.S - 1);
    if (first > (long long)ta + a.wr || last < (long long)ta - a.wl) return false;
  }
  // keyed by the token's window first, so that CTAs launched together add their dQ
  // contributions to a window of tokens whose fp32 accumulators stay in L2
  const int win = ta / a.win_tokens;
  *list = ((b * a.nwin + win) * a.Hkv + g) * a.nblk + x;
  *tq_out = tq;
  return true;
}

__global__ void kv_count_kernel(const KvIndexArgs a) {
  long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= a.n_slots) return;
  int list, tq;
  if (kv_slot_list(a, e, &list, &tq)) atomicAdd(a.counts + list, 1);
}

__global__ void kv_fill_kernel(const KvIndexArgs a) {
  long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= a.n_slots) return;
  int list, tq;
  if (kv_slot_list(a, e, &list, &tq)) {
    int pos = atomicAdd(a.cursor + list, 1);
    a.entries[__ldg(a.list_off + list) + pos] = tq;
  }
}

// exclusive scans of counts -> list_off, chunk counts -> chunk_off; one CTA of 1024
__global__ void __launch_bounds__(1024) kv_scan_kernel(const KvIndexArgs a) {
  __shared__ int warp_tot[2][32];
  __shared__ int carry[2];
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  if (tid == 0) carry[0] = carry[1] = 0;
  __syncthreads();
  for (int base = 0; base < a.n_lists; base += 1024) {
    const int i = base + tid;
    int c = i < a.n_lists ? a.counts[i] : 0;
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
      a.chunk_off[i] = pk;
    }
    __syncthreads();
    if (tid == 1023) { carry[0] = pc + c; carry[1] = pk + k; }
    __syncthreads();
  }
  if (tid == 0) {
    a.list_off[a.n_lists] = carry[0];
    a.chunk_off[a.n_lists] = carry[1];
    *a.work_count = carry[1];
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
  k<<<(unsigned)L.max_work, WITH_DQ ? 320 : 192, PL::kSmem, st>>>(mq, mdo, mk, mv, a);
  count_launch();
  mark_end(st, kTimeBwdKV);
  return cudaGetLastError();
}

cudaError_t launch_kv_index(const KvIndexArgs& a, cudaStream_t st) {
  // counts and cursor arrive zeroed (cleared with the rest of the workspace)
  if (a.n_slots > 0) {
    kv_count_kernel<<<(unsigned)((a.n_slots + 255) / 256), 256, 0, st>>>(a);
    count_launch();
  }
  kv_scan_kernel<<<1, 1024, 0, st>>>(a);
  count_launch();
  if (a.n_slots > 0) {
    kv_fill_kernel<<<(unsigned)((a.n_slots + 255) / 256), 256, 0, st>>>(a);
    count_launch();
  }
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
