// sa_tk_bwd.cu -- token-level backward over one shared latent KV head (K = V,
// d_qk = 576, d_v = 512) on tcgen05, query-stationary: one CTA takes one
// (token, kv-head) unit and 64 of its query heads, and streams the unit's
// selected KV rows through in tiles of 32 rows.
//
// SparseFlashMlaGrad "Computation formula" Stages 2-3 (P recomputed from lse,
// dP = dO V^T, dS = P o (dP - Delta), dQ = dS K scale, dKV = dS^T Q scale + P^T dO).
//
// Per 32-row tile (bf16 operands, fp32 TMEM accumulators; M = 64 heads):
//   S    [64 x 32]   = Q KV^T            lanes 0..15 of each sub-partition
//   dP   [64 x 32]   = dO V^T            lanes 16..31, the same columns
//   P, dS (scaled)                        softmax warps, to shared memory
//   dKV^T [576 x 32] = Q^T dS + dO^T P   (the P^T dO term on dims 0..511),
//                                          added to the fp32 dKV accumulator
//   dQ   [64 x 576] += dS KV              accumulated in TMEM over every tile
// TMEM columns: [0, 32) S / dP; [32, 288) dQ dims 0..255 (lanes 0..15) and
// 256..511 (lanes 16..31); [288, 352) dQ dims 512..575; [352, 480) dKV^T dims
// 0..511 as four M = 128 tiles; [480, 512) dKV^T dims 512..575 (M = 64).
//
// Warp roles: 0 = loader (Q / dO by TMA, KV rows by cp.async), 1 = MMA issuer
// + TMEM owner, 2..5 = softmax and the final dQ store, 6..9 = dKV reductions.
// Every wait is bounded (sa_tc.cuh).
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "sa_device.cuh"
#include "sa_launch.h"
#include "sa_tc.cuh"

namespace sa {

constexpr float kLog2eTk = 1.4426950408889634f;

struct TkPlan {
  static constexpr int DQK = 576, DV = 512;
  static constexpr int H = 64;     // query heads per CTA
  static constexpr int NK = 32;    // KV rows per tile
  static constexpr int NSQ = DQK / 64, NSV = DV / 64;
  static constexpr int oQ = 0;                           // Q: NSQ slabs of 64 rows x 128 B
  static constexpr int oDO = oQ + NSQ * H * 128;         // dO: NSV slabs of 64 rows
  static constexpr int kKVStage = NSQ * NK * 128;        // one KV tile: NSQ slabs of 32 rows
  static constexpr int oKV = oDO + NSV * H * 128;        // 2 stages
  // P and dS [64 heads][32 keys] bf16 in the 64-byte swizzle (rows of 64 B): a
  // K-major A for dQ (K = keys) and an MN-major B of one 32-wide atom for dKV
  static constexpr int oP = oKV + 2 * kKVStage;
  static constexpr int oDS = oP + H * 64;
  static constexpr int oCode = oDS + H * 64;             // row codes of the last 4 tiles
  static constexpr int kSmem = oCode + 4 * NK * 4;
  static_assert(kSmem + 1024 <= 227 * 1024, "shared memory plan too large");
  static_assert(oDO % 1024 == 0 && oKV % 1024 == 0 && kKVStage % 1024 == 0 && oP % 1024 == 0 && oDS % 1024 == 0,
                "swizzled operands need 1024-byte alignment");
  static constexpr int cS = 0, cDQ = 32, cDQR = 288, cKV = 352, cKVR = 480;
  static constexpr uint32_t kAlloc = 512;
};

struct TkBars {
  uint64_t q_full, kv_full[2], kv_empty[2], s_full, pds_full, pds_free, dkv_full, dkv_free, dq_done;
  uint64_t codes_full[4];  // a tile's row codes are in shared memory (ring of 4 tiles)
  uint32_t tmem_base;
  int abort_flag;
};

// 16-byte piece c (0..71) of a 576-wide bf16 row r of a 32-row KV tile
__device__ __forceinline__ uint32_t tk_kv_addr(uint32_t stage, int r, int c) {
  return stage + (c >> 3) * (TkPlan::NK * 128) + r * 128 + (((c & 7) ^ (r & 7)) << 4);
}

__global__ void __launch_bounds__(320, 1) tk_bwd_kernel(const __grid_constant__ CUtensorMap mapQ,
                                                         const __grid_constant__ CUtensorMap mapDO, const Prob p,
                                                         const float* __restrict__ LSE,
                                                         const float* __restrict__ Delta, BwdOut out) {
  using PL = TkPlan;
  extern __shared__ __align__(1024) uint8_t smem[];
  __shared__ TkBars bars;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (smem_u32(smem) & 1023) {
    if (threadIdx.x == 0 && p.status) atomicOr(p.status, kStatusSmemAlign);
    return;
  }
  const int nhs = p.G / PL::H;  // head slices per unit
  const int unit = blockIdx.x / nhs, hs = blockIdx.x - unit * nhs;
  const int tq = unit / p.Hkv, g = unit - tq * p.Hkv;
  const int head0 = g * p.G + hs * PL::H;  // first query head of the CTA
  const uint32_t sQ = smem_u32(smem + PL::oQ), sDO = smem_u32(smem + PL::oDO);
  const uint32_t sKV = smem_u32(smem + PL::oKV), sP = smem_u32(smem + PL::oP), sDS = smem_u32(smem + PL::oDS);
  int* codes = reinterpret_cast<int*>(smem + PL::oCode);
  volatile int* abort_flag = &bars.abort_flag;

  if (threadIdx.x == 0) {
    bars.abort_flag = 0;
    mbar_init(&bars.q_full, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bars.kv_full[s], 32);
      mbar_init(&bars.kv_empty[s], 1);
    }
    mbar_init(&bars.s_full, 1);
    mbar_init(&bars.pds_full, 128);
    mbar_init(&bars.pds_free, 1);
    mbar_init(&bars.dkv_full, 1);
    mbar_init(&bars.dkv_free, 128);
    mbar_init(&bars.dq_done, 1);
    for (int s = 0; s < 4; ++s) mbar_init(&bars.codes_full[s], 1);
    mbar_fence_init();
    tma_prefetch_desc(&mapQ);
    tma_prefetch_desc(&mapDO);
  }
  if (warp == 1) tmem_alloc(&bars.tmem_base, PL::kAlloc);
  pdl_wait();
  pdl_trigger();
  const Unit u = make_unit(p, tq, g);
  const int nsub = 2 * u.n_tiles;  // 32-row tiles
  fence_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars.tmem_base;

  if (warp == 0) {
    // ------------------------------------------------------------ loader
    if (lane == 0) {
      mbar_arrive_tx(&bars.q_full, (uint32_t)((PL::NSQ + PL::NSV) * PL::H * 128));
      const int row = tq * p.Hq + head0;
      for (int s = 0; s < PL::NSQ; ++s) tma_load_2d(sQ + s * PL::H * 128, &mapQ, 64 * s, row, &bars.q_full);
      for (int s = 0; s < PL::NSV; ++s) tma_load_2d(sDO + s * PL::H * 128, &mapDO, 64 * s, row, &bars.q_full);
    }
    for (int i = 0; i < nsub; ++i) {
      const int st = i & 1;
      bool ok = true;
      if (lane == 0 && i >= 2) ok = mbar_wait(&bars.kv_empty[st], ((i >> 1) - 1) & 1, abort_flag, p.status);
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      int* cd = codes + (i & 3) * PL::NK;
      cd[lane] = resolve_row(p, u, i >> 1, 32 * (i & 1) + lane);
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars.codes_full[i & 3]);
      const uint32_t stage = sKV + st * PL::kKVStage;
#pragma unroll 4
      for (int idx = lane; idx < PL::NK * (PL::DQK / 8); idx += 32) {
        const int r = idx / (PL::DQK / 8), c = idx - r * (PL::DQK / 8);
        const int code = cd[r];
        const bf16* src = code >= 0 ? row_k_ptr(p, code, g) + c * 8 : p.k;
        cp_async16(tk_kv_addr(stage, r, c), src, code >= 0);
      }
      cp_async_commit();
      cp_async_wait_none();
      fence_async_smem();
      mbar_arrive(&bars.kv_full[st]);
    }
    cp_async_wait_none();
    if (lane == 0) mbar_wait_drain(&bars.q_full, 0);
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idS = idesc_bf16(64, 32, false, false);
      constexpr uint32_t idKV = idesc_bf16(128, 32, true, true);
      constexpr uint32_t idKVR = idesc_bf16(64, 32, true, true);
      constexpr uint32_t idDQ = idesc_bf16(64, 256, false, true);
      constexpr uint32_t idDQR = idesc_bf16(64, 64, false, true);
      bool ok = mbar_wait(&bars.q_full, 0, abort_flag, p.status);
      for (int i = 0; ok && i < nsub; ++i) {
        const int st = i & 1;
        if (!mbar_wait(&bars.kv_full[st], (i >> 1) & 1, abort_flag, p.status)) break;
        tc_fence_after();
        const uint32_t kv = sKV + st * PL::kKVStage;
        // S = Q KV^T (lanes 0..15), dP = dO V^T (lanes 16..31)
        for (int kk = 0; kk < PL::DQK / 16; ++kk)
          mma_bf16(tmem + PL::cS, sdesc(sQ + (kk >> 2) * (PL::H * 128) + (kk & 3) * 32, 16, 1024),
                   sdesc(kv + (kk >> 2) * (PL::NK * 128) + (kk & 3) * 32, 16, 1024), idS, kk > 0);
        for (int kk = 0; kk < PL::DV / 16; ++kk)
          mma_bf16(tmem + (16u << 16) + PL::cS, sdesc(sDO + (kk >> 2) * (PL::H * 128) + (kk & 3) * 32, 16, 1024),
                   sdesc(kv + (kk >> 2) * (PL::NK * 128) + (kk & 3) * 32, 16, 1024), idS, kk > 0);
        mma_commit(&bars.s_full);
        if (!mbar_wait(&bars.pds_full, i & 1, abort_flag, p.status)) break;
        if (i > 0 && !mbar_wait(&bars.dkv_free, (i - 1) & 1, abort_flag, p.status)) break;
        tc_fence_after();
        // dKV^T = Q^T dS + dO^T P over the 64 heads (fresh for every tile)
        for (int t = 0; t < 4; ++t) {
          for (int kk = 0; kk < 4; ++kk)
            mma_bf16(tmem + PL::cKV + 32 * t, sdesc(sQ + 2 * t * (PL::H * 128) + kk * 2048, PL::H * 128, 1024),
                     sdesc64(sDS + kk * 1024, PL::H * 64, 512), idKV, kk > 0);
          for (int kk = 0; kk < 4; ++kk)
            mma_bf16(tmem + PL::cKV + 32 * t, sdesc(sDO + 2 * t * (PL::H * 128) + kk * 2048, PL::H * 128, 1024),
                     sdesc64(sP + kk * 1024, PL::H * 64, 512), idKV, 1u);
        }
        for (int kk = 0; kk < 4; ++kk)
          mma_bf16(tmem + PL::cKVR, sdesc(sQ + 8 * (PL::H * 128) + kk * 2048, PL::H * 128, 1024),
                   sdesc64(sDS + kk * 1024, PL::H * 64, 512), idKVR, kk > 0);
        mma_commit(&bars.dkv_full);
        // dQ += dS KV (KV as an MN-major B: N = dims in 64-wide slabs of 32 rows)
        for (int kk = 0; kk < PL::NK / 16; ++kk) {
          const uint32_t acc = (i > 0 || kk > 0) ? 1u : 0u;
          const uint64_t a = sdesc64(sDS + kk * 32, 16, 512);
          mma_bf16(tmem + PL::cDQ, a, sdesc(kv + kk * 2048, PL::NK * 128, 1024), idDQ, acc);
          mma_bf16(tmem + (16u << 16) + PL::cDQ, a, sdesc(kv + 4 * (PL::NK * 128) + kk * 2048, PL::NK * 128, 1024),
                   idDQ, acc);
          mma_bf16(tmem + PL::cDQR, a, sdesc(kv + 8 * (PL::NK * 128) + kk * 2048, PL::NK * 128, 1024), idDQR, acc);
        }
        mma_commit(&bars.kv_empty[st]);
        mma_commit(&bars.pds_free);
      }
      mma_commit(&bars.dq_done);
    }
  } else if (warp < 6) {
    // ------------------------------------------------------------ softmax, then dQ
    const int sub = warp & 3;
    const int h = 16 * sub + (lane & 15);  // head within the CTA
    const bool is_s = lane < 16;           // S row (else the dP row of the same head)
    const uint32_t lane_base = tmem + ((uint32_t)(32 * sub) << 16);
    const long long row = (long long)tq * p.Hq + head0 + h;
    const float lse = __ldg(LSE + row);
    const float lse2 = lse * kLog2eTk;
    const float dlt = __ldg(Delta + row);
    float psd = 0.f;  // sum_j P_j dP_j for dSinks
    bool ok = true;
    for (int i = 0; i < nsub; ++i) {
      if (!mbar_wait(&bars.s_full, i & 1, abort_flag, p.status)) { ok = false; break; }
      tc_fence_after();
      uint32_t v[2][16];
      tmem_ld16(lane_base + PL::cS, v[0]);
      tmem_ld16(lane_base + PL::cS + 16, v[1]);
      tmem_wait_ld();
      reg_dep16(v[0]);
      reg_dep16(v[1]);
      if (!mbar_wait(&bars.codes_full[i & 3], (i >> 2) & 1, abort_flag, p.status)) { ok = false; break; }
      const int* cd = codes + (i & 3) * PL::NK;
      float own[32], oth[32];
#pragma unroll
      for (int k = 0; k < 32; ++k) {
        const float x = __uint_as_float(v[k >> 4][k & 15]);
        own[k] = is_s ? (cd[k] >= 0 ? exp2f(x * p.scale_log2 - lse2) : 0.f) : x;  // P or dP
      }
#pragma unroll
      for (int k = 0; k < 32; ++k) oth[k] = __shfl_xor_sync(0xffffffffu, own[k], 16);
      // the P / dS buffers are free once the previous tile's dKV and dQ MMAs are done
      if (i > 0 && !mbar_wait(&bars.pds_free, (i - 1) & 1, abort_flag, p.status)) { ok = false; break; }
      uint32_t pk[16];
#pragma unroll
      for (int k = 0; k < 32; k += 2) {
        float a0, a1;
        if (is_s) {
          a0 = own[k];
          a1 = own[k + 1];
        } else {  // dS = P (dP - Delta), scaled: dQ and dKV both take scale * dS
          a0 = oth[k] * (own[k] - dlt) * p.scale;
          a1 = oth[k + 1] * (own[k + 1] - dlt) * p.scale;
          psd += oth[k] * own[k] + oth[k + 1] * own[k + 1];
        }
        pk[k >> 1] = pack_bf16(a0, a1);
      }
      const uint32_t rowaddr = (is_s ? sP : sDS) + h * 64;
#pragma unroll
      for (int c = 0; c < 4; ++c)
        asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};\n" ::"r"(rowaddr + ((c ^ ((h >> 1) & 3)) << 4)),
                     "r"(pk[4 * c]), "r"(pk[4 * c + 1]), "r"(pk[4 * c + 2]), "r"(pk[4 * c + 3])
                     : "memory");
      tc_fence_before();
      fence_async_smem();
      mbar_arrive(&bars.pds_full);
    }
    // dSinks: -P_sink * sum_j P_j dP_j per head (the dP lane holds the sum)
    if (ok && p.sinks && !is_s) {
      const float psink = exp2f(__ldg(p.sinks + head0 + h) * kLog2eTk - lse2);
      atomicAdd(out.dsinks + head0 + h, -psink * psd);
    }
    // dQ (already scaled through dS) to bf16: lanes 0..15 dims 0..255 and 512..575,
    // lanes 16..31 dims 256..511
    if (ok && (nsub == 0 || mbar_wait(&bars.dq_done, 0, abort_flag, p.status))) {
      tc_fence_after();
      bf16* dst = out.dq + row * PL::DQK + (is_s ? 0 : 256);
      for (int c = 0; c < 256 + 64; c += 16) {
        uint32_t v[16];
        tmem_ld16(lane_base + PL::cDQ + c, v);
        tmem_wait_ld();
        reg_dep16(v);
        if (c >= 256 && !is_s) continue;  // dims 512..575 live in lanes 0..15 only
        bf16* d = c < 256 ? dst + c : out.dq + row * PL::DQK + 512 + (c - 256);
        uint32_t w[8];
#pragma unroll
        for (int e = 0; e < 8; ++e)
          w[e] = nsub == 0 ? 0u : pack_bf16(__uint_as_float(v[2 * e]), __uint_as_float(v[2 * e + 1]));
        reinterpret_cast<uint4*>(d)[0] = make_uint4(w[0], w[1], w[2], w[3]);
        reinterpret_cast<uint4*>(d)[1] = make_uint4(w[4], w[5], w[6], w[7]);
      }
    }
    tc_fence_before();
  } else {
    // ------------------------------------------------------------ dKV reductions
    const int sub = warp & 3;
    const uint32_t lane_base = tmem + ((uint32_t)(32 * sub) << 16);
    for (int i = 0; i < nsub; ++i) {
      if (!mbar_wait(&bars.dkv_full, i & 1, abort_flag, p.status)) break;
      if (!mbar_wait(&bars.codes_full[i & 3], (i >> 2) & 1, abort_flag, p.status)) break;
      tc_fence_after();
      const int* cd = codes + (i & 3) * PL::NK;
      float* rowp[PL::NK];
#pragma unroll
      for (int k = 0; k < PL::NK; ++k) {
        const int code = cd[k];
        rowp[k] = code < 0 ? nullptr
                           : ((code & kCmpFlag) ? out.dcmp_acc + ((long long)(code & ~kCmpFlag) * p.Hkv + g) * PL::DQK
                                                : out.dk_acc + ((long long)code * p.Hkv + g) * PL::DQK);
      }
      // four M = 128 tiles (dims 128 t + 32 sub + lane) and the rope tile (dims
      // 512 + 16 sub + lane, lanes 0..15)
#pragma unroll 1
      for (int t = 0; t < 5; ++t) {
        uint32_t v[2][16];
        tmem_ld16(lane_base + PL::cKV + 32 * t, v[0]);
        tmem_ld16(lane_base + PL::cKV + 32 * t + 16, v[1]);
        tmem_wait_ld();
        reg_dep16(v[0]);
        reg_dep16(v[1]);
        if (t == 4) {
          tc_fence_before();
          mbar_arrive(&bars.dkv_free);  // the accumulators go back before the reductions
        }
        const int dim = t < 4 ? 128 * t + 32 * sub + lane : 512 + 16 * sub + lane;
        if (t == 4 && lane >= 16) continue;
#pragma unroll
        for (int k = 0; k < PL::NK; ++k)
          if (rowp[k]) atomicAdd(rowp[k] + dim, __uint_as_float(v[k >> 4][k & 15]));
      }
    }
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, PL::kAlloc);
    tmem_relinquish();
  }
}

bool tk_path_built(int dqk, int dv, int shared, int G) {
  return dqk == TkPlan::DQK && dv == TkPlan::DV && shared && G % TkPlan::H == 0;
}

cudaError_t launch_tk_bwd(const Prob& p, const float* lse, const float* delta, const bf16* d_o, const BwdOut& out,
                          cudaStream_t st) {
  using PL = TkPlan;
  if (!tk_path_built(p.dqk, p.dv, p.shared, p.G)) return cudaErrorInvalidValue;
  const long long grid = (long long)p.Tq * p.Hkv * (p.G / PL::H);
  if (grid == 0) return cudaSuccess;
  CUtensorMap mq, mdo;
  if (!make_tmap_bf16(&mq, p.q, (uint64_t)p.Tq * p.Hq, PL::DQK, (uint64_t)PL::DQK * 2, PL::H) ||
      !make_tmap_bf16(&mdo, d_o, (uint64_t)p.Tq * p.Hq, PL::DV, (uint64_t)PL::DV * 2, PL::H))
    return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(tk_bwd_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, PL::kSmem);
  if (e != cudaSuccess) return e;
  mark_begin(st, kTimeBwdKV);
  e = launch_pdl(tk_bwd_kernel, (unsigned)grid, 320, PL::kSmem, st, mq, mdo, p, lse, delta, out);
  count_launch();
  mark_end(st, kTimeBwdKV);
  return e;
}



// ---------------------------------------------------------------------------
// Token-level forward over one shared KV head (576 / 512) on tcgen05, the same
// unit and tile decomposition: one CTA per (token, kv-head, 64 heads).
//   S [64 x 32] = Q KV^T (lanes 0..15); online softmax in the softmax warps;
//   O [64 x 512] += P V: dims 0..255 in lanes 0..15 and 256..511 in lanes 16..31
//   of TMEM columns [32, 288).  The running maximum moves only when a tile's
//   maximum exceeds it by more than 8 (a factor of 256 in the exponentials): O and
//   the running sum are then rescaled once, after the previous P V has landed.
// Sinks start the running state (m = sink, l = 1).
// ---------------------------------------------------------------------------
struct TkFwdPlan {
  static constexpr int DQK = 576, DV = 512, H = 64, NK = 32;
  static constexpr int NSQ = DQK / 64;
  static constexpr int oQ = 0;
  static constexpr int kKVStage = NSQ * NK * 128;
  static constexpr int oKV = oQ + NSQ * H * 128;
  static constexpr int oP = oKV + 2 * kKVStage;  // P [64 heads][32 keys] bf16, 64-byte swizzle
  static constexpr int oCode = oP + H * 64;
  static constexpr int kSmem = oCode + 4 * NK * 4;
  static_assert(kSmem + 1024 <= 227 * 1024, "shared memory plan too large");
  static constexpr int cS = 0, cO = 32;
  static constexpr uint32_t kAlloc = 512;
};

struct TkFwdBars {
  uint64_t q_full, kv_full[2], kv_empty[2], s_full, p_full, pv_done;
  uint64_t codes_full[4];
  uint32_t tmem_base;
  int abort_flag;
};

__global__ void __launch_bounds__(192, 1) tk_fwd_kernel(const __grid_constant__ CUtensorMap mapQ, const Prob p,
                                                        bf16* __restrict__ O, float* __restrict__ LSE) {
  using PL = TkFwdPlan;
  extern __shared__ __align__(1024) uint8_t smem[];
  __shared__ TkFwdBars bars;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (smem_u32(smem) & 1023) {
    if (threadIdx.x == 0 && p.status) atomicOr(p.status, kStatusSmemAlign);
    return;
  }
  const int nhs = p.G / PL::H;
  const int unit = blockIdx.x / nhs, hs = blockIdx.x - unit * nhs;
  const int tq = unit / p.Hkv, g = unit - tq * p.Hkv;
  const int head0 = g * p.G + hs * PL::H;
  const uint32_t sQ = smem_u32(smem + PL::oQ), sKV = smem_u32(smem + PL::oKV), sP = smem_u32(smem + PL::oP);
  int* codes = reinterpret_cast<int*>(smem + PL::oCode);
  volatile int* abort_flag = &bars.abort_flag;
  if (threadIdx.x == 0) {
    bars.abort_flag = 0;
    mbar_init(&bars.q_full, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bars.kv_full[s], 32);
      mbar_init(&bars.kv_empty[s], 1);
    }
    mbar_init(&bars.s_full, 1);
    mbar_init(&bars.p_full, 128);
    mbar_init(&bars.pv_done, 1);
    for (int s = 0; s < 4; ++s) mbar_init(&bars.codes_full[s], 1);
    mbar_fence_init();
    tma_prefetch_desc(&mapQ);
  }
  if (warp == 1) tmem_alloc(&bars.tmem_base, PL::kAlloc);
  pdl_wait();
  pdl_trigger();
  const Unit u = make_unit(p, tq, g);
  const int nsub = 2 * u.n_tiles;
  fence_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars.tmem_base;

  if (warp == 0) {
    // ------------------------------------------------------------ loader
    if (lane == 0) {
      mbar_arrive_tx(&bars.q_full, (uint32_t)(PL::NSQ * PL::H * 128));
      for (int s = 0; s < PL::NSQ; ++s)
        tma_load_2d(sQ + s * PL::H * 128, &mapQ, 64 * s, tq * p.Hq + head0, &bars.q_full);
    }
    for (int i = 0; i < nsub; ++i) {
      const int st = i & 1;
      bool ok = true;
      if (lane == 0 && i >= 2) ok = mbar_wait(&bars.kv_empty[st], ((i >> 1) - 1) & 1, abort_flag, p.status);
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      int* cd = codes + (i & 3) * PL::NK;
      cd[lane] = resolve_row(p, u, i >> 1, 32 * (i & 1) + lane);
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars.codes_full[i & 3]);
      const uint32_t stage = sKV + st * PL::kKVStage;
#pragma unroll 4
      for (int idx = lane; idx < PL::NK * (PL::DQK / 8); idx += 32) {
        const int r = idx / (PL::DQK / 8), c = idx - r * (PL::DQK / 8);
        const int code = cd[r];
        const bf16* src = code >= 0 ? row_k_ptr(p, code, g) + c * 8 : p.k;
        cp_async16(tk_kv_addr(stage, r, c), src, code >= 0);
      }
      cp_async_commit();
      cp_async_wait_none();
      fence_async_smem();
      mbar_arrive(&bars.kv_full[st]);
    }
    cp_async_wait_none();
    if (lane == 0) mbar_wait_drain(&bars.q_full, 0);
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idS = idesc_bf16(64, 32, false, false);
      constexpr uint32_t idPV = idesc_bf16(64, 256, false, true);
      bool ok = mbar_wait(&bars.q_full, 0, abort_flag, p.status);
      for (int i = 0; ok && i < nsub; ++i) {
        const int st = i & 1;
        if (!mbar_wait(&bars.kv_full[st], (i >> 1) & 1, abort_flag, p.status)) break;
        tc_fence_after();
        const uint32_t kv = sKV + st * PL::kKVStage;
        for (int kk = 0; kk < PL::DQK / 16; ++kk)
          mma_bf16(tmem + PL::cS, sdesc(sQ + (kk >> 2) * (PL::H * 128) + (kk & 3) * 32, 16, 1024),
                   sdesc(kv + (kk >> 2) * (PL::NK * 128) + (kk & 3) * 32, 16, 1024), idS, kk > 0);
        mma_commit(&bars.s_full);
        if (!mbar_wait(&bars.p_full, i & 1, abort_flag, p.status)) break;
        tc_fence_after();
        // O += P V (V = the first 512 dims of the KV rows, an MN-major B)
        for (int kk = 0; kk < PL::NK / 16; ++kk) {
          const uint32_t acc = (i > 0 || kk > 0) ? 1u : 0u;
          const uint64_t a = sdesc64(sP + kk * 32, 16, 512);
          mma_bf16(tmem + PL::cO, a, sdesc(kv + kk * 2048, PL::NK * 128, 1024), idPV, acc);
          mma_bf16(tmem + (16u << 16) + PL::cO, a, sdesc(kv + 4 * (PL::NK * 128) + kk * 2048, PL::NK * 128, 1024),
                   idPV, acc);
        }
        mma_commit(&bars.kv_empty[st]);
        mma_commit(&bars.pv_done);
      }
    }
  } else {
    // ------------------------------------------------------------ softmax + O
    const int sub = warp & 3;
    const int h = 16 * sub + (lane & 15);
    const bool is_s = lane < 16;
    const uint32_t lane_base = tmem + ((uint32_t)(32 * sub) << 16);
    const long long row = (long long)tq * p.Hq + head0 + h;
    float m = -INFINITY, l = 0.f;  // running maximum (log2 units) and sum
    if (p.sinks) {
      m = __ldg(p.sinks + head0 + h) * kLog2eTk;
      l = 1.f;
    }
    bool ok = true;
    for (int i = 0; i < nsub; ++i) {
      if (!mbar_wait(&bars.s_full, i & 1, abort_flag, p.status)) { ok = false; break; }
      tc_fence_after();
      uint32_t v[2][16];
      tmem_ld16(lane_base + PL::cS, v[0]);
      tmem_ld16(lane_base + PL::cS + 16, v[1]);
      tmem_wait_ld();
      reg_dep16(v[0]);
      reg_dep16(v[1]);
      if (!mbar_wait(&bars.codes_full[i & 3], (i >> 2) & 1, abort_flag, p.status)) { ok = false; break; }
      const int* cd = codes + (i & 3) * PL::NK;
      float sc[32];
      float tmax = -INFINITY;
#pragma unroll
      for (int k = 0; k < 32; ++k) {
        sc[k] = cd[k] >= 0 ? __uint_as_float(v[k >> 4][k & 15]) * p.scale_log2 : -INFINITY;
        tmax = fmaxf(tmax, sc[k]);
      }
      tmax = __shfl_sync(0xffffffffu, tmax, lane & 15);  // the S lane's maximum for both halves
      // the previous P V has landed (P buffer free, O stable) before P or O changes
      if (i > 0 && !mbar_wait(&bars.pv_done, (i - 1) & 1, abort_flag, p.status)) { ok = false; break; }
      tc_fence_after();
      const bool grow = tmax > m + 8.f;  // the same decision in both lanes of a head
      if (__any_sync(0xffffffffu, grow)) {
        const float mn = grow ? tmax : m;
        const float f = (m == -INFINITY) ? 0.f : exp2f(m - mn);
        if (i > 0) {
          // rescale this lane's half of the head's O row (256 columns)
          for (int c = 0; c < 256; c += 16) {
            uint32_t w[16];
            tmem_ld16(lane_base + PL::cO + c, w);
            tmem_wait_ld();
            reg_dep16(w);
#pragma unroll
            for (int e = 0; e < 16; ++e) w[e] = __float_as_uint(__uint_as_float(w[e]) * f);
            tmem_st16(lane_base + PL::cO + c, w);
          }
          tmem_wait_st();
        }
        l *= f;
        m = mn;
      }
      if (is_s) {
        uint32_t pk[16];
#pragma unroll
        for (int k = 0; k < 32; k += 2) {
          const float a0 = exp2f(sc[k] - m), a1 = exp2f(sc[k + 1] - m);
          l += a0 + a1;
          pk[k >> 1] = pack_bf16(a0, a1);
        }
        const uint32_t rowaddr = sP + h * 64;
#pragma unroll
        for (int c = 0; c < 4; ++c)
          asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};\n" ::"r"(rowaddr + ((c ^ ((h >> 1) & 3)) << 4)),
                       "r"(pk[4 * c]), "r"(pk[4 * c + 1]), "r"(pk[4 * c + 2]), "r"(pk[4 * c + 3])
                       : "memory");
      }
      tc_fence_before();
      fence_async_smem();
      mbar_arrive(&bars.p_full);
    }
    l = __shfl_sync(0xffffffffu, l, lane & 15);  // the S lane holds the sum
    // O / l to bf16, lse = (m + log2 l) ln 2; a row with nothing visible gets O = 0, lse = +inf
    if (ok && (nsub == 0 || mbar_wait(&bars.pv_done, (nsub - 1) & 1, abort_flag, p.status))) {
      tc_fence_after();
      const float inv = l > 0.f ? 1.f / l : 0.f;
      bf16* dst = O + row * PL::DV + (is_s ? 0 : 256);
      for (int c = 0; c < 256; c += 16) {
        uint32_t w[16];
        tmem_ld16(lane_base + PL::cO + c, w);
        tmem_wait_ld();
        reg_dep16(w);
        uint32_t o8[8];
#pragma unroll
        for (int e = 0; e < 8; ++e)
          o8[e] = nsub == 0 ? 0u : pack_bf16(__uint_as_float(w[2 * e]) * inv, __uint_as_float(w[2 * e + 1]) * inv);
        reinterpret_cast<uint4*>(dst + c)[0] = make_uint4(o8[0], o8[1], o8[2], o8[3]);
        reinterpret_cast<uint4*>(dst + c)[1] = make_uint4(o8[4], o8[5], o8[6], o8[7]);
      }
      if (is_s) LSE[row] = l > 0.f ? (m + log2f(l)) * 0.6931471805599453f : INFINITY;
    }
    tc_fence_before();
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, PL::kAlloc);
    tmem_relinquish();
  }
}

cudaError_t launch_tk_fwd(const Prob& p, bf16* o, float* lse, cudaStream_t st) {
  using PL = TkFwdPlan;
  if (!tk_path_built(p.dqk, p.dv, p.shared, p.G)) return cudaErrorInvalidValue;
  const long long grid = (long long)p.Tq * p.Hkv * (p.G / PL::H);
  if (grid == 0) return cudaSuccess;
  CUtensorMap mq;
  if (!make_tmap_bf16(&mq, p.q, (uint64_t)p.Tq * p.Hq, PL::DQK, (uint64_t)PL::DQK * 2, PL::H))
    return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(tk_fwd_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, PL::kSmem);
  if (e != cudaSuccess) return e;
  mark_begin(st, kTimeFwd);
  e = launch_pdl(tk_fwd_kernel, (unsigned)grid, 192, PL::kSmem, st, mq, p, o, lse);
  count_launch();
  mark_end(st, kTimeFwd);
  return e;
}

}  // namespace sa
