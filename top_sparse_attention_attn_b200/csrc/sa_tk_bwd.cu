// sa_tk_bwd.cu -- token-level selection over one shared latent KV head (K = V,
// d_qk = 576, d_v = 512: the first 512 columns of each KV row are V) on tcgen05,
// query-stationary: one CTA takes one (query token, kv-head) unit and 64 of its
// query heads, and streams the unit's selected KV rows through in sub-tiles of
// 32 rows.
//
// Selection: SparseFlashMlaGrad "Computation formula" Stage 1 (ori rows through
// token indices or the sliding window, concatenated with gathered cmpKv rows),
// resolved row by row with resolve_row_x.  The rows of a sub-tile arrive by TMA
// row gathers (tile::gather4, four rows per copy) into 128-byte-swizzled shared
// memory; a lane of the loader warp resolves each row, and the next sub-tile's
// indices are loaded while the current one is issued.
//
// Forward (aclnnNsaSelectedAttentionInfer "Formula"; SparseFlashMlaGrad Stage 2
// for lse), per sub-tile i (bf16 operands, fp32 TMEM accumulators, M = 64 heads):
//   S_i [64 x 32] = Q KV_i^T               two TMEM buffers (lanes 0..15 of each
//                                           sub-partition)
//   online softmax in the softmax warps     P_i to one of two shared buffers
//   O   [64 x 512] += P_i V_i              dims 0..255 in lanes 0..15, 256..511 in
//                                           lanes 16..31
// The MMA warp issues S_{i+1} before P_i V_i, so the softmax of one sub-tile
// overlaps the tensor work of its neighbours (three KV stages in flight).  The
// running maximum moves only when a sub-tile's maximum exceeds it by more than 8
// (a factor of 256 in the exponentials): O and the running sum are then rescaled
// once, after the previous P V has landed.  Sinks start the running state.
// With 128 query heads per kv-head the two 64-head CTAs of a token run as a
// two-CTA cluster: each gathers half of every sub-tile and copies it into the
// other's stage over distributed shared memory (tk_load_rows, PAIR).
//
// Backward (SparseFlashMlaGrad Stages 2-3: P recomputed from lse, dP = dO V^T,
// dS = P o (dP - Delta), dQ = dS K scale, dKV = dS^T Q scale + P^T dO), per
// sub-tile:
//   S  [64 x 32] = Q KV^T   (lanes 0..15)   dP [64 x 32] = dO V^T (lanes 16..31)
//   P, dS (scaled) by the softmax warps, to shared memory
//   dKV^T [576 x 32] = Q^T dS + dO^T P      (the P^T dO term on dims 0..511);
//                                           the reduction warps stage it as fp32
//                                           key rows over the sub-tile's KV stage
//                                           (two passes of 288 dims) and add each
//                                           row to the fp32 dKV accumulator with
//                                           one TMA bulk reduction
//   dQ [64 x 576] += dS KV                  accumulated in TMEM over every sub-tile
//
// Warp roles: 0 = loader (Q / dO box loads, row codes, KV row gathers), 1 = MMA
// issuer + TMEM owner, 2..5 = softmax (and the final O or dQ store), 6..9
// (backward) = dKV reductions.  Every wait is bounded (sa_tc.cuh).
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "sa_device.cuh"
#include "sa_launch.h"
#include "sa_tc.cuh"

namespace sa {

constexpr float kLog2eTk = 1.4426950408889634f;

namespace tk {
constexpr int DQK = 576, DV = 512;
constexpr int H = 64;                    // query heads per CTA
constexpr int NK = 32;                   // KV rows per sub-tile
constexpr int NSQ = DQK / 64, NSV = DV / 64;
constexpr int kKVStage = NSQ * NK * 128; // one sub-tile: NSQ slabs of 32 rows x 128 B
constexpr int kQBytes = NSQ * H * 128;   // Q: NSQ slabs of 64 rows
constexpr int kDOBytes = NSV * H * 128;  // dO: NSV slabs of 64 rows
constexpr int kPBytes = H * 64;          // P or dS [64 heads][32 keys] bf16, 64-byte swizzle
}  // namespace tk

// 16-byte piece index XOR for a [64][32] bf16 operand in the 64-byte swizzle.
__device__ __forceinline__ uint32_t tk_p_addr(uint32_t base, int h, int c) {
  return base + h * 64 + ((c ^ ((h >> 1) & 3)) << 4);
}

// 16-byte piece c (0..71) of row r of a 32-row sub-tile stage: NSQ slabs of 32
// rows x 128 bytes, 128-byte swizzle (the layout a TMA box or gather writes).
__device__ __forceinline__ uint32_t tk_kv_addr(uint32_t stage, int r, int c) {
  return stage + (c >> 3) * (tk::NK * 128) + r * 128 + (((c & 7) ^ (r & 7)) << 4);
}

// Loader (warp 0, every lane): the row codes of each 32-row sub-tile (lane = row)
// into the 4-deep codes ring, then the rows themselves into stage i % NST.  The
// first TMA_SLABS 64-column slabs of every row arrive by TMA row gathers
// (tile::gather4, four rows per copy, 512 bytes each); the rest by 16-byte
// cp.async copies through the load/store path.  The TMA engine handles about one
// gather per 70 cycles, so splitting the slabs keeps both paths busy.  kv_full
// expects the gathered bytes (one arrival) plus one arrival per lane once its
// copies have landed (TMA_SLABS < NSQ).  The next sub-tile's indices are loaded
// while the current one is issued.  Stage reuse waits for kv_empty; on abort the
// warp stops issuing.  Before returning it waits (bounded) for every copy to land.
//
// PAIR: the two CTAs of a cluster (two head slices of one token) select the same
// rows.  Each gathers half of every sub-tile (rows 16 * rank .. + 15, 36 gathers)
// into its own stage, completing half_full; the copier warp of tk_fwd_kernel then
// copies that half into the same rows of the partner's stage.  kv_full needs both
// halves: the copier's arrival once this CTA's half has landed, and the partner's
// bytes (expected by the loader).  Before gathering into a stage again the loader
// waits for copy_done (the partner has received this CTA's previous half, so the
// copy has read it), then tells the partner through peer_ready that the stage may
// take the partner's half (its previous use has been consumed).  Every
// one of these barriers completes once per use of a stage (phase (i / NST) & 1).
template <int NST, int TMA_SLABS, bool PAIR = false>
__device__ void tk_load_rows(const Prob& p, const Unit& u, int g, int nsub, uint32_t sKV, int* codes,
                             const CUtensorMap* mapKV, const CUtensorMap* mapCmp, bool has_cmp, uint64_t* kv_full,
                             uint64_t* kv_empty, uint64_t* codes_full, volatile int* abort_flag, int lane,
                             uint64_t* half_full = nullptr, uint64_t* peer_ready = nullptr,
                             uint64_t* copy_done = nullptr, uint32_t crank = 0) {
  constexpr int CP_PIECES = (tk::NSQ - TMA_SLABS) * 8;  // 16-byte pieces of a row copied by cp.async
  static_assert(!PAIR || CP_PIECES == 0, "a pair gathers every slab by TMA");
  int x_next = nsub > 0 ? slot_index(p, u, 0, lane) : -1;
  int issued = 0;
  for (int i = 0; i < nsub; ++i) {
    const int st = i % NST, tile = i >> 1, r = 32 * (i & 1) + lane;
    const int x = x_next;
    if (i + 1 < nsub) x_next = slot_index(p, u, (i + 1) >> 1, 32 * ((i + 1) & 1) + lane);  // prefetch
    bool ok = true;
    if (lane == 0) {
      if (i >= NST) ok = mbar_wait(&kv_empty[st], ((i / NST) - 1) & 1, abort_flag, p.status);
      if (PAIR && ok && i >= NST) ok = mbar_wait_cluster(&copy_done[st], ((i / NST) - 1) & 1, abort_flag, p.status);
      // the partner's half may land (once signalled, the stage is armed below and drained on exit)
      if (PAIR && ok) mbar_arrive_remote(mapa_shared(smem_u32(&peer_ready[st]), crank ^ 1u));
    }
    ok = __shfl_sync(0xffffffffu, ok, 0);
    if (!ok) break;
    const int code = resolve_row_x(p, u, tile, r, x);
    codes[(i & 3) * tk::NK + lane] = code;
    __syncwarp();
    if (lane == 0) mbar_arrive(&codes_full[i & 3]);
    const uint32_t stage = sKV + st * tk::kKVStage;
    if (TMA_SLABS > 0) {
      const bool cmp_tile = tile >= u.n_ori_tiles && has_cmp;
      const int y = code >= 0 ? (code & ~kCmpFlag) : 0;  // invisible rows load row 0 (masked later)
      uint64_t* gbar = PAIR ? &half_full[st] : &kv_full[st];
      if (lane == 0) {
        if (PAIR) mbar_arrive_tx(&kv_full[st], (uint32_t)(TMA_SLABS * 16 * 128));  // the partner's half
        mbar_arrive_tx(gbar, (uint32_t)(TMA_SLABS * (PAIR ? 16 : tk::NK) * 128));
      }
      __syncwarp();
      const int q4 = lane & 7;
      const int y0 = __shfl_sync(0xffffffffu, y, 4 * q4), y1 = __shfl_sync(0xffffffffu, y, 4 * q4 + 1);
      const int y2 = __shfl_sync(0xffffffffu, y, 4 * q4 + 2), y3 = __shfl_sync(0xffffffffu, y, 4 * q4 + 3);
      if (lane < 8 && (!PAIR || (uint32_t)(lane >> 2) == crank)) {
        const CUtensorMap* map = cmp_tile ? mapCmp : mapKV;
        const uint32_t dst = stage + q4 * 4 * 128;
#pragma unroll
        for (int s = 0; s < TMA_SLABS; ++s)
          tma_gather4(dst + s * (tk::NK * 128), map, g * tk::DQK + 64 * s, y0, y1, y2, y3, gbar);
      }
    }
    if constexpr (CP_PIECES > 0) {
      // lanes take consecutive 16-byte pieces of one row; invisible rows are zero-filled
      const int* cd = codes + (i & 3) * tk::NK;
#pragma unroll 4
      for (int idx = lane; idx < tk::NK * CP_PIECES; idx += 32) {
        const int rr = idx / CP_PIECES, c = TMA_SLABS * 8 + (idx - rr * CP_PIECES);
        const int cr = cd[rr];
        const bf16* src = cr >= 0 ? row_k_ptr(p, cr, g) + c * 8 : p.k;
        cp_async16(tk_kv_addr(stage, rr, c), src, cr >= 0);
      }
      cp_async_commit();
      cp_async_wait_none();
      fence_async_smem();  // the copies -> visible to the tensor core
      mbar_arrive(&kv_full[st]);
    }
    issued = i + 1;
  }
  if (TMA_SLABS > 0 && lane == 0)
    for (int i = issued > NST ? issued - NST : 0; i < issued; ++i) {
      if (PAIR) mbar_wait_drain(&half_full[i % NST], (i / NST) & 1);
      mbar_wait_drain(&kv_full[i % NST], (i / NST) & 1);
    }
  if constexpr (CP_PIECES > 0) cp_async_wait_none();
}

// ===========================================================================
// backward
// ===========================================================================
struct TkBwdPlan {
  static constexpr int NST = 2;
  // slabs of each KV row by TMA gather (the rest by cp.async); the TMA engine also
  // carries the Q / dO boxes and the dKV bulk reductions
  static constexpr int kTmaSlabs = 9;
  static constexpr int oQ = 0;
  static constexpr int oDO = oQ + tk::kQBytes;
  static constexpr int oKV = oDO + tk::kDOBytes;
  static constexpr int oP = oKV + NST * tk::kKVStage;
  static constexpr int oDS = oP + tk::kPBytes;
  static constexpr int oCode = oDS + tk::kPBytes;  // row codes of the last 4 sub-tiles
  static constexpr int kSmem = oCode + 4 * tk::NK * 4;
  static_assert(kSmem + 1024 <= 227 * 1024, "shared memory plan too large");
  static_assert(oDO % 1024 == 0 && oKV % 1024 == 0 && tk::kKVStage % 1024 == 0 && oP % 1024 == 0 &&
                    oDS % 1024 == 0,
                "swizzled operands need 1024-byte alignment");
  // TMEM columns: [0, 32) S (lanes 0..15) / dP (lanes 16..31); [32, 288) dQ dims
  // 0..255 (lanes 0..15) and 256..511 (lanes 16..31); [288, 352) dQ dims 512..575
  // (lanes 0..15); [352, 480) dKV^T dims 0..511 as four M = 128 tiles; [480, 512)
  // dKV^T dims 512..575 (M = 64).
  static constexpr int cS = 0, cDQ = 32, cDQR = 288, cKV = 352, cKVR = 480;
  static constexpr uint32_t kAlloc = 512;
};

struct TkBwdBars {
  uint64_t q_full, kv_full[TkBwdPlan::NST], kv_empty[TkBwdPlan::NST], s_full, pds_full, pds_free, kvq_done,
      dkv_free, dq_done;
  uint64_t codes_full[4];  // a sub-tile's row codes are in shared memory (ring of 4)
  uint32_t tmem_base;
  int abort_flag;
};

__global__ void __launch_bounds__(320, 1) tk_bwd_kernel(const __grid_constant__ CUtensorMap mapQ,
                                                         const __grid_constant__ CUtensorMap mapDO,
                                                         const __grid_constant__ CUtensorMap mapKV,
                                                         const __grid_constant__ CUtensorMap mapCmp, const int has_cmp,
                                                         const Prob p, const float* __restrict__ LSE,
                                                         const float* __restrict__ Delta, BwdOut out) {
  using PL = TkBwdPlan;
  extern __shared__ __align__(1024) uint8_t smem[];
  __shared__ TkBwdBars bars;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (smem_u32(smem) & 1023) {
    pdl_wait();
    if (threadIdx.x == 0 && p.status) atomicOr(p.status, kStatusSmemAlign);
    return;
  }
  const int nhs = p.G / tk::H;  // head slices per unit
  const int unit = blockIdx.x / nhs, hs = blockIdx.x - unit * nhs;
  const int tq = unit / p.Hkv, g = unit - tq * p.Hkv;
  const int head0 = g * p.G + hs * tk::H;  // first query head of the CTA
  const uint32_t sQ = smem_u32(smem + PL::oQ), sDO = smem_u32(smem + PL::oDO);
  const uint32_t sKV = smem_u32(smem + PL::oKV), sP = smem_u32(smem + PL::oP), sDS = smem_u32(smem + PL::oDS);
  int* codes = reinterpret_cast<int*>(smem + PL::oCode);
  volatile int* abort_flag = &bars.abort_flag;

  if (threadIdx.x == 0) {
    bars.abort_flag = 0;
    mbar_init(&bars.q_full, 1);
    for (int s = 0; s < PL::NST; ++s) {
      mbar_init(&bars.kv_full[s], (PL::kTmaSlabs > 0 ? 1 : 0) + (PL::kTmaSlabs < tk::NSQ ? 32 : 0));
      mbar_init(&bars.kv_empty[s], 1);
    }
    mbar_init(&bars.s_full, 1);
    mbar_init(&bars.pds_full, 128);
    mbar_init(&bars.pds_free, 1);
    mbar_init(&bars.kvq_done, 1);
    mbar_init(&bars.dkv_free, 128);
    mbar_init(&bars.dq_done, 1);
    for (int s = 0; s < 4; ++s) mbar_init(&bars.codes_full[s], 1);
    mbar_fence_init();
    tma_prefetch_desc(&mapQ);
    tma_prefetch_desc(&mapDO);
    tma_prefetch_desc(&mapKV);
    tma_prefetch_desc(&mapCmp);
  }
  if (warp == 1) tmem_alloc(&bars.tmem_base, PL::kAlloc);
  pdl_wait();
  pdl_trigger();
  const Unit u = make_unit(p, tq, g);
  const int nsub = 2 * u.n_tiles;  // 32-row sub-tiles
  fence_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars.tmem_base;

  if (warp == 0) {
    // ------------------------------------------------------------ loader
    if (lane == 0) {
      mbar_arrive_tx(&bars.q_full, (uint32_t)(tk::kQBytes + tk::kDOBytes));
      const int row = tq * p.Hq + head0;
      for (int s = 0; s < tk::NSQ; ++s) tma_load_2d(sQ + s * tk::H * 128, &mapQ, 64 * s, row, &bars.q_full);
      for (int s = 0; s < tk::NSV; ++s) tma_load_2d(sDO + s * tk::H * 128, &mapDO, 64 * s, row, &bars.q_full);
    }
    tk_load_rows<PL::NST, PL::kTmaSlabs>(p, u, g, nsub, sKV, codes, &mapKV, &mapCmp, has_cmp != 0, bars.kv_full,
                                          bars.kv_empty, bars.codes_full, abort_flag, lane);
    if (lane == 0) mbar_wait_drain(&bars.q_full, 0);
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idS = idesc_bf16(64, 32, false, false);
      constexpr uint32_t idKV = idesc_bf16(128, 32, true, true);
      constexpr uint32_t idKVR = idesc_bf16(64, 32, true, true);
      constexpr uint32_t idDQ = idesc_bf16(64, 256, false, true);
      constexpr uint32_t idDQR = idesc_bf16(64, 64, false, true);
      // operand descriptors at the buffers' starts (K-major "k", MN-major "m" / "n")
      const uint64_t dQk = sdesc(sQ, 16, 1024), dDOk = sdesc(sDO, 16, 1024);
      const uint64_t dQm = sdesc(sQ, tk::H * 128, 1024), dDOm = sdesc(sDO, tk::H * 128, 1024);
      const uint64_t dDSn = sdesc64(sDS, tk::H * 64, 512), dPn = sdesc64(sP, tk::H * 64, 512);
      const uint64_t dDSk = sdesc64(sDS, 16, 512);
      bool ok = mbar_wait(&bars.q_full, 0, abort_flag, p.status);
      for (int i = 0; ok && i < nsub; ++i) {
        const int st = i % PL::NST;
        if (!mbar_wait(&bars.kv_full[st], (i / PL::NST) & 1, abort_flag, p.status)) break;
        tc_fence_after();
        const uint32_t kv = sKV + st * tk::kKVStage;
        const uint64_t dKVk = sdesc(kv, 16, 1024);
        // S = Q KV^T (lanes 0..15), dP = dO V^T (lanes 16..31)
#pragma unroll
        for (int kk = 0; kk < tk::DQK / 16; ++kk)
          mma_bf16(tmem + PL::cS, desc_add(dQk, (kk >> 2) * (tk::H * 128) + (kk & 3) * 32),
                   desc_add(dKVk, (kk >> 2) * (tk::NK * 128) + (kk & 3) * 32), idS, kk > 0);
#pragma unroll
        for (int kk = 0; kk < tk::DV / 16; ++kk)
          mma_bf16(tmem + (16u << 16) + PL::cS, desc_add(dDOk, (kk >> 2) * (tk::H * 128) + (kk & 3) * 32),
                   desc_add(dKVk, (kk >> 2) * (tk::NK * 128) + (kk & 3) * 32), idS, kk > 0);
        mma_commit(&bars.s_full);
        if (!mbar_wait(&bars.pds_full, i & 1, abort_flag, p.status)) break;
        if (i > 0 && !mbar_wait(&bars.dkv_free, (i - 1) & 1, abort_flag, p.status)) break;
        tc_fence_after();
        // dKV^T = Q^T dS + dO^T P over the 64 heads (fresh for every sub-tile)
#pragma unroll
        for (int t = 0; t < 4; ++t) {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_bf16(tmem + PL::cKV + 32 * t, desc_add(dQm, 2 * t * (tk::H * 128) + kk * 2048),
                     desc_add(dDSn, kk * 1024), idKV, kk > 0);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_bf16(tmem + PL::cKV + 32 * t, desc_add(dDOm, 2 * t * (tk::H * 128) + kk * 2048),
                     desc_add(dPn, kk * 1024), idKV, 1u);
        }
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_bf16(tmem + PL::cKVR, desc_add(dQm, 8 * (tk::H * 128) + kk * 2048), desc_add(dDSn, kk * 1024), idKVR,
                   kk > 0);
        // dQ += dS KV (KV as an MN-major B: N = dims in 64-wide slabs of 32 rows)
        const uint64_t dKVn = sdesc(kv, tk::NK * 128, 1024);
#pragma unroll
        for (int kk = 0; kk < tk::NK / 16; ++kk) {
          const uint32_t acc = (i > 0 || kk > 0) ? 1u : 0u;
          const uint64_t a = desc_add(dDSk, kk * 32);
          mma_bf16(tmem + PL::cDQ, a, desc_add(dKVn, kk * 2048), idDQ, acc);
          mma_bf16(tmem + (16u << 16) + PL::cDQ, a, desc_add(dKVn, 4 * (tk::NK * 128) + kk * 2048), idDQ, acc);
          mma_bf16(tmem + PL::cDQR, a, desc_add(dKVn, 8 * (tk::NK * 128) + kk * 2048), idDQR, acc);
        }
        // the stage is released by the reduction warps, which stage dKV^T in it once
        // every MMA of the sub-tile (dKV^T included) has completed
        mma_commit(&bars.kvq_done);
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
      // the sub-tile's visible keys as a bit mask (eight 16-byte reads of the codes)
      unsigned visk = 0;
      {
        const int4* cd4 = reinterpret_cast<const int4*>(codes + (i & 3) * tk::NK);
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const int4 c4 = cd4[q];
          visk |= (c4.x >= 0 ? 1u : 0u) << (4 * q);
          visk |= (c4.y >= 0 ? 1u : 0u) << (4 * q + 1);
          visk |= (c4.z >= 0 ? 1u : 0u) << (4 * q + 2);
          visk |= (c4.w >= 0 ? 1u : 0u) << (4 * q + 3);
        }
      }
      float own[32], oth[32];
#pragma unroll
      for (int k = 0; k < 32; ++k) {
        const float x = __uint_as_float(v[k >> 4][k & 15]);
        own[k] = is_s ? (((visk >> k) & 1u) ? ex2_approx(fmaf(x, p.scale_log2, -lse2)) : 0.f) : x;  // P or dP
      }
#pragma unroll
      for (int k = 0; k < 32; ++k) oth[k] = __shfl_xor_sync(0xffffffffu, own[k], 16);
      // the P / dS buffers are free once the previous sub-tile's dKV and dQ MMAs are done
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
      const uint32_t rb = is_s ? sP : sDS;
#pragma unroll
      for (int c = 0; c < 4; ++c)
        asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};\n" ::"r"(tk_p_addr(rb, h, c)), "r"(pk[4 * c]),
                     "r"(pk[4 * c + 1]), "r"(pk[4 * c + 2]), "r"(pk[4 * c + 3])
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
      bf16* dst = out.dq + row * tk::DQK + (is_s ? 0 : 256);
      for (int c = 0; c < 256 + 64; c += 16) {
        uint32_t v[16];
        tmem_ld16(lane_base + PL::cDQ + c, v);
        tmem_wait_ld();
        reg_dep16(v);
        if (c >= 256 && !is_s) continue;  // dims 512..575 live in lanes 0..15 only
        bf16* d = c < 256 ? dst + c : out.dq + row * tk::DQK + 512 + (c - 256);
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
    // dKV^T leaves through the TMA engine: once every MMA of sub-tile i is done (the
    // KV stage and dKV^T are then both free), the four warps copy dKV^T from TMEM
    // into the KV stage as fp32 [key][dim] rows, 288 dims at a time (a full stage),
    // and each warp's lane 0 adds eight of the key rows to the fp32 accumulator with
    // bulk reductions (cp.reduce.async.bulk ... .add.f32).  After
    // the last pass the stage goes back to the loader.  Bulk reductions keep many
    // bytes in flight per issuing thread, where per-thread atomics were limited by
    // the few warps issuing them.
    const int sub = warp & 3, rw = warp - 6;  // sub-partition; warp within the role (0..3)
    const uint32_t lane_base = tmem + ((uint32_t)(32 * sub) << 16);
    for (int i = 0; i < nsub; ++i) {
      const int st = i % PL::NST;
      bool ok = mbar_wait(&bars.kvq_done, i & 1, abort_flag, p.status) &&
                mbar_wait(&bars.codes_full[i & 3], (i >> 2) & 1, abort_flag, p.status);
      ok = __all_sync(0xffffffffu, ok);
      tc_fence_after();
      const int* cd = codes + (i & 3) * tk::NK;
      const uint32_t stage = sKV + st * tk::kKVStage;
#pragma unroll 1
      for (int pass = 0; pass < 2; ++pass) {
        // pass 0: dims 0..287 (tiles 0, 1 and the first 32 dims of tile 2); pass 1: dims
        // 288..575 (the rest of tile 2, tile 3 and the rope tile); rows of 288 fp32
        if (ok) {
#pragma unroll 1
          for (int t = 2 * pass; t < 2 * pass + 3; ++t) {
            uint32_t v[2][16];
            tmem_ld16(lane_base + PL::cKV + 32 * t, v[0]);
            tmem_ld16(lane_base + PL::cKV + 32 * t + 16, v[1]);
            tmem_wait_ld();
            reg_dep16(v[0]);
            reg_dep16(v[1]);
            // this lane's dim: M = 128 tiles 128 t + 32 sub + lane; the rope tile (M = 64)
            // 512 + 16 sub + lane for lanes 0..15
            const int dim = t < 4 ? 128 * t + 32 * sub + lane : (lane < 16 ? 512 + 16 * sub + lane : -1);
            const int dl = dim - 288 * pass;
            if (dl >= 0 && dl < 288) {
#pragma unroll
              for (int k = 0; k < tk::NK; ++k)
                asm volatile("st.shared.f32 [%0], %1;\n" ::"r"(stage + k * (288 * 4) + dl * 4),
                             "f"(__uint_as_float(v[k >> 4][k & 15]))
                             : "memory");
            }
          }
        }
        if (pass == 1) {
          tc_fence_before();
          mbar_arrive(&bars.dkv_free);  // dKV^T has been read out of TMEM
        }
        fence_async_smem();
        asm volatile("bar.sync 2, 128;\n" ::: "memory");
        if (ok && lane == 0) {
          for (int k = 8 * rw; k < 8 * rw + 8; ++k) {
            const int code = cd[k];
            if (code < 0) continue;
            float* rp = (code & kCmpFlag) ? out.dcmp_acc + ((long long)(code & ~kCmpFlag) * p.Hkv + g) * tk::DQK
                                          : out.dk_acc + ((long long)code * p.Hkv + g) * tk::DQK;
            bulk_reduce_add_f32(rp + 288 * pass, stage + k * (288 * 4), 288 * 4);
          }
          bulk_commit();
          bulk_wait_read_all();  // the stage may be overwritten once these reads are done
        }
        asm volatile("bar.sync 2, 128;\n" ::: "memory");
      }
      if (rw == 0 && lane == 0) mbar_arrive(&bars.kv_empty[st]);  // the stage goes back to the loader
    }
    if (lane == 0) bulk_wait_all();  // every bulk reduction complete before the CTA leaves
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, PL::kAlloc);
    tmem_relinquish();
  }
}

// ===========================================================================
// forward
// ===========================================================================
struct TkFwdPlan {
  static constexpr int NST = 3;
  static constexpr int kTmaSlabs = 9;  // every slab by TMA gather (measured faster than a cp.async share)
  static constexpr int oQ = 0;
  static constexpr int oKV = oQ + tk::kQBytes;
  static constexpr int oP = oKV + NST * tk::kKVStage;  // two P buffers
  static constexpr int oCode = oP + 2 * tk::kPBytes;
  static constexpr int kSmem = oCode + 4 * tk::NK * 4;
  static_assert(kSmem + 1024 <= 227 * 1024, "shared memory plan too large");
  static_assert(oKV % 1024 == 0 && oP % 1024 == 0, "swizzled operands need 1024-byte alignment");
  // TMEM columns: S buffers [0, 32) and [32, 64) (lanes 0..15); O [64, 320): dims
  // 0..255 in lanes 0..15, 256..511 in lanes 16..31.
  static constexpr int cS0 = 0, cO = 64;
  static constexpr uint32_t kAlloc = 512;
};

struct TkFwdBars {
  uint64_t q_full, kv_full[TkFwdPlan::NST], kv_empty[TkFwdPlan::NST], s_full[2], s_free[2], p_full[2],
      pv_done[2];
  uint64_t codes_full[4];
  // cluster pair: this CTA's half of a stage has landed / the partner's stage may
  // take this CTA's half / the partner has received this CTA's half
  uint64_t half_full[TkFwdPlan::NST], peer_ready[TkFwdPlan::NST], copy_done[TkFwdPlan::NST];
  uint32_t tmem_base;
  int abort_flag;
};

// PAIR: launched in clusters of two CTAs, the two 64-head slices of one token
// (G / 64 even), which share the row gathers (tk_load_rows); a seventh warp
// copies the half of each stage this CTA gathered into the partner's stage.
template <bool PAIR>
__global__ void __launch_bounds__(PAIR ? 224 : 192, 1) tk_fwd_kernel(const __grid_constant__ CUtensorMap mapQ,
                                                                     const __grid_constant__ CUtensorMap mapKV,
                                                                     const __grid_constant__ CUtensorMap mapCmp,
                                                                     const int has_cmp, const Prob p,
                                                                     bf16* __restrict__ O, float* __restrict__ LSE) {
  using PL = TkFwdPlan;
  extern __shared__ __align__(1024) uint8_t smem[];
  __shared__ TkFwdBars bars;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (smem_u32(smem) & 1023) {
    pdl_wait();
    if (threadIdx.x == 0 && p.status) atomicOr(p.status, kStatusSmemAlign);
    if (PAIR) cluster_sync();  // the same outcome in both CTAs
    return;
  }
  const uint32_t crank = PAIR ? cluster_ctarank() : 0u;
  const int nhs = p.G / tk::H;
  const int unit = blockIdx.x / nhs, hs = blockIdx.x - unit * nhs;
  const int tq = unit / p.Hkv, g = unit - tq * p.Hkv;
  const int head0 = g * p.G + hs * tk::H;
  const uint32_t sQ = smem_u32(smem + PL::oQ), sKV = smem_u32(smem + PL::oKV), sP = smem_u32(smem + PL::oP);
  int* codes = reinterpret_cast<int*>(smem + PL::oCode);
  volatile int* abort_flag = &bars.abort_flag;
  if (threadIdx.x == 0) {
    bars.abort_flag = 0;
    mbar_init(&bars.q_full, 1);
    for (int s = 0; s < PL::NST; ++s) {
      mbar_init(&bars.kv_full[s], PAIR ? 2 : (PL::kTmaSlabs > 0 ? 1 : 0) + (PL::kTmaSlabs < tk::NSQ ? 32 : 0));
      mbar_init(&bars.kv_empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&bars.s_full[b], 1);
      mbar_init(&bars.s_free[b], 128);
      mbar_init(&bars.p_full[b], 128);
      mbar_init(&bars.pv_done[b], 1);
    }
    for (int s = 0; s < 4; ++s) mbar_init(&bars.codes_full[s], 1);
    for (int s = 0; s < PL::NST; ++s) {
      mbar_init(&bars.half_full[s], 1);
      mbar_init(&bars.peer_ready[s], 1);
      mbar_init(&bars.copy_done[s], 1);
    }
    mbar_fence_init();
    tma_prefetch_desc(&mapQ);
    tma_prefetch_desc(&mapKV);
    tma_prefetch_desc(&mapCmp);
  }
  if (warp == 1) tmem_alloc(&bars.tmem_base, PL::kAlloc);
  pdl_wait();
  pdl_trigger();
  const Unit u = make_unit(p, tq, g);
  const int nsub = 2 * u.n_tiles;
  fence_async_smem();
  tc_fence_before();
  if (PAIR)
    cluster_sync();  // the partner's barriers are initialised before any remote arrive or copy
  else
    __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars.tmem_base;

  if (warp == 0) {
    // ------------------------------------------------------------ loader
    if (lane == 0) {
      mbar_arrive_tx(&bars.q_full, (uint32_t)tk::kQBytes);
      for (int s = 0; s < tk::NSQ; ++s)
        tma_load_2d(sQ + s * tk::H * 128, &mapQ, 64 * s, tq * p.Hq + head0, &bars.q_full);
    }
    tk_load_rows<PL::NST, PL::kTmaSlabs, PAIR>(p, u, g, nsub, sKV, codes, &mapKV, &mapCmp, has_cmp != 0,
                                                bars.kv_full, bars.kv_empty, bars.codes_full, abort_flag, lane,
                                                bars.half_full, bars.peer_ready, bars.copy_done, crank);
    if (lane == 0) mbar_wait_drain(&bars.q_full, 0);
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // order: S_0, then for each i: S_{i+1} (when it exists) before P_i V_i
    if (lane == 0) {
      constexpr uint32_t idS = idesc_bf16(64, 32, false, false);
      constexpr uint32_t idPV = idesc_bf16(64, 256, false, true);
      const uint64_t dQk = sdesc(sQ, 16, 1024);  // Q as the K-major A of S
      bool ok = mbar_wait(&bars.q_full, 0, abort_flag, p.status);
      for (int i = 0; ok && i <= nsub; ++i) {
        if (i < nsub) {
          const int st = i % PL::NST;
          if (!mbar_wait(&bars.kv_full[st], (i / PL::NST) & 1, abort_flag, p.status)) break;
          if (PAIR)  // the partner's half has landed: the partner may gather into that stage again
            mbar_arrive_remote(mapa_shared(smem_u32(&bars.copy_done[st]), crank ^ 1u));
          if (i >= 2 && !mbar_wait(&bars.s_free[i & 1], ((i - 2) >> 1) & 1, abort_flag, p.status)) break;
          tc_fence_after();
          const uint64_t dKVk = sdesc(sKV + st * tk::kKVStage, 16, 1024);
          const uint32_t dS = tmem + PL::cS0 + 32 * (i & 1);
#pragma unroll
          for (int kk = 0; kk < tk::DQK / 16; ++kk)
            mma_bf16(dS, desc_add(dQk, (kk >> 2) * (tk::H * 128) + (kk & 3) * 32),
                     desc_add(dKVk, (kk >> 2) * (tk::NK * 128) + (kk & 3) * 32), idS, kk > 0);
          mma_commit(&bars.s_full[i & 1]);
        }
        if (i >= 1) {
          const int j = i - 1, stj = j % PL::NST;
          if (!mbar_wait(&bars.p_full[j & 1], (j >> 1) & 1, abort_flag, p.status)) break;
          tc_fence_after();
          // O += P_j V_j (V = the first 512 dims of the KV rows, an MN-major B)
          const uint64_t dVn = sdesc(sKV + stj * tk::kKVStage, tk::NK * 128, 1024);
          const uint64_t dPk = sdesc64(sP + (j & 1) * tk::kPBytes, 16, 512);
#pragma unroll
          for (int kk = 0; kk < tk::NK / 16; ++kk) {
            const uint32_t acc = (j > 0 || kk > 0) ? 1u : 0u;
            const uint64_t a = desc_add(dPk, kk * 32);
            mma_bf16(tmem + PL::cO, a, desc_add(dVn, kk * 2048), idPV, acc);
            mma_bf16(tmem + (16u << 16) + PL::cO, a, desc_add(dVn, 4 * (tk::NK * 128) + kk * 2048), idPV, acc);
          }
          mma_commit(&bars.kv_empty[stj]);
          mma_commit(&bars.pv_done[j & 1]);
        }
      }
    }
  } else if (PAIR && warp == 6) {
    // ------------------------------------------------------------ copier
    // this CTA's half of each sub-tile, once landed, into the same rows of the
    // partner's stage (16 rows x 128 bytes = 2 KB per slab) as soon as the
    // partner's stage may take it
    if (lane == 0) {
      for (int i = 0; i < nsub; ++i) {
        const int st = i % PL::NST, ph = (i / PL::NST) & 1;
        if (!mbar_wait(&bars.half_full[st], ph, abort_flag, p.status)) break;
        mbar_arrive(&bars.kv_full[st]);  // this CTA's half is in
        if (!mbar_wait_cluster(&bars.peer_ready[st], ph, abort_flag, p.status)) break;
        const uint32_t half = sKV + st * tk::kKVStage + crank * (16 * 128);
        const uint32_t bar = mapa_shared(smem_u32(&bars.kv_full[st]), crank ^ 1u);
#pragma unroll
        for (int s = 0; s < tk::NSQ; ++s) {
          const uint32_t src = half + s * (tk::NK * 128);
          bulk_copy_to_peer(mapa_shared(src, crank ^ 1u), src, 16 * 128, bar);
        }
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
      if (!mbar_wait(&bars.s_full[i & 1], (i >> 1) & 1, abort_flag, p.status)) { ok = false; break; }
      tc_fence_after();
      uint32_t v[2][16];
      tmem_ld16(lane_base + PL::cS0 + 32 * (i & 1), v[0]);
      tmem_ld16(lane_base + PL::cS0 + 32 * (i & 1) + 16, v[1]);
      tmem_wait_ld();
      reg_dep16(v[0]);
      reg_dep16(v[1]);
      tc_fence_before();
      mbar_arrive(&bars.s_free[i & 1]);  // the S buffer may take S_{i+2}
      if (!mbar_wait(&bars.codes_full[i & 3], (i >> 2) & 1, abort_flag, p.status)) { ok = false; break; }
      const int* cd = codes + (i & 3) * tk::NK;
      float sc[32];
      float tmax = -INFINITY;
#pragma unroll
      for (int k = 0; k < 32; ++k) {
        sc[k] = cd[k] >= 0 ? __uint_as_float(v[k >> 4][k & 15]) * p.scale_log2 : -INFINITY;
        tmax = fmaxf(tmax, sc[k]);
      }
      tmax = __shfl_sync(0xffffffffu, tmax, lane & 15);  // the S lane's maximum for both halves
      // P buffer i & 1 is free once P_{i-2} V_{i-2} has landed
      if (i >= 2 && !mbar_wait(&bars.pv_done[i & 1], ((i - 2) >> 1) & 1, abort_flag, p.status)) { ok = false; break; }
      const bool grow = tmax > m + 8.f;  // the same decision in both lanes of a head
      if (__any_sync(0xffffffffu, grow)) {
        const float mn = grow ? tmax : m;
        const float f = (m == -INFINITY) ? 0.f : exp2f(m - mn);
        if (i >= 1) {
          // O must be stable: P_{i-1} V_{i-1} has landed (and no P V is in flight)
          if (!mbar_wait(&bars.pv_done[(i - 1) & 1], ((i - 1) >> 1) & 1, abort_flag, p.status)) { ok = false; }
          ok = __all_sync(0xffffffffu, ok);
          if (!ok) break;
          tc_fence_after();
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
          const float a0 = sc[k] == -INFINITY ? 0.f : ex2_approx(sc[k] - m);
          const float a1 = sc[k + 1] == -INFINITY ? 0.f : ex2_approx(sc[k + 1] - m);
          l += a0 + a1;
          pk[k >> 1] = pack_bf16(a0, a1);
        }
        const uint32_t pb = sP + (i & 1) * tk::kPBytes;
#pragma unroll
        for (int c = 0; c < 4; ++c)
          asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};\n" ::"r"(tk_p_addr(pb, h, c)), "r"(pk[4 * c]),
                       "r"(pk[4 * c + 1]), "r"(pk[4 * c + 2]), "r"(pk[4 * c + 3])
                       : "memory");
      }
      tc_fence_before();
      fence_async_smem();
      mbar_arrive(&bars.p_full[i & 1]);
    }
    l = __shfl_sync(0xffffffffu, l, lane & 15);  // the S lane holds the sum
    // O / l to bf16, lse = (m + log2 l) ln 2; a row with nothing visible gets O = 0, lse = +inf
    const int last = nsub - 1;
    if (ok && (nsub == 0 || mbar_wait(&bars.pv_done[last & 1], (last >> 1) & 1, abort_flag, p.status))) {
      tc_fence_after();
      const float inv = l > 0.f ? 1.f / l : 0.f;
      bf16* dst = O + row * tk::DV + (is_s ? 0 : 256);
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
  // no CTA leaves while its partner may still copy into it or arrive on its barriers
  if (PAIR) cluster_sync();
}

// ===========================================================================
// host side
// ===========================================================================
bool tk_path_built(int dqk, int dv, int shared, int G) {
  return dqk == tk::DQK && dv == tk::DV && shared && G % tk::H == 0;
}

// Row-gather maps over the shared KV and cmp_kv ([rows][Hkv * 576], boxes of one
// row x 64 columns); without compressed rows the cmp map repeats the KV map.
static bool tk_row_maps(const Prob& p, CUtensorMap* mkv, CUtensorMap* mcmp, int* has_cmp) {
  if (p.Tkv < 1) return false;
  if (!make_tmap_bf16(mkv, p.k, (uint64_t)p.Tkv, (uint64_t)p.Hkv * tk::DQK, (uint64_t)p.Hkv * tk::DQK * 2, 1))
    return false;
  *has_cmp = 0;
  *mcmp = *mkv;
  if (p.cmpk && p.Tcmp > 0) {
    if (!make_tmap_bf16(mcmp, p.cmpk, (uint64_t)p.Tcmp, (uint64_t)p.Hkv * tk::DQK, (uint64_t)p.Hkv * tk::DQK * 2, 1))
      return false;
    *has_cmp = 1;
  }
  return true;
}

cudaError_t launch_tk_bwd(const Prob& p, const float* lse, const float* delta, const bf16* d_o, const BwdOut& out,
                          cudaStream_t st) {
  using PL = TkBwdPlan;
  if (!tk_path_built(p.dqk, p.dv, p.shared, p.G)) return cudaErrorInvalidValue;
  const long long grid = (long long)p.Tq * p.Hkv * (p.G / tk::H);
  if (grid == 0) return cudaSuccess;
  CUtensorMap mq, mdo, mkv, mcmp;
  int has_cmp = 0;
  if (!make_tmap_bf16(&mq, p.q, (uint64_t)p.Tq * p.Hq, tk::DQK, (uint64_t)tk::DQK * 2, tk::H) ||
      !make_tmap_bf16(&mdo, d_o, (uint64_t)p.Tq * p.Hq, tk::DV, (uint64_t)tk::DV * 2, tk::H) ||
      !tk_row_maps(p, &mkv, &mcmp, &has_cmp))
    return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(tk_bwd_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, PL::kSmem);
  if (e != cudaSuccess) return e;
  mark_begin(st, kTimeBwdKV);
  e = launch_pdl(tk_bwd_kernel, (unsigned)grid, 320, PL::kSmem, st, mq, mdo, mkv, mcmp, has_cmp, p, lse, delta, out);
  count_launch();
  mark_end(st, kTimeBwdKV);
  return e;
}

cudaError_t launch_tk_fwd(const Prob& p, bf16* o, float* lse, bool pair, cudaStream_t st) {
  using PL = TkFwdPlan;
  if (!tk_path_built(p.dqk, p.dv, p.shared, p.G)) return cudaErrorInvalidValue;
  const long long grid = (long long)p.Tq * p.Hkv * (p.G / tk::H);
  if (grid == 0) return cudaSuccess;
  CUtensorMap mq, mkv, mcmp;
  int has_cmp = 0;
  if (!make_tmap_bf16(&mq, p.q, (uint64_t)p.Tq * p.Hq, tk::DQK, (uint64_t)tk::DQK * 2, tk::H) ||
      !tk_row_maps(p, &mkv, &mcmp, &has_cmp))
    return cudaErrorInvalidValue;
  // the two 64-head slices of a token are consecutive CTAs: pair them when every token has an even count
  pair = pair && (p.G / tk::H) % 2 == 0;
  cudaError_t e = pair ? cudaFuncSetAttribute(tk_fwd_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                              PL::kSmem)
                       : cudaFuncSetAttribute(tk_fwd_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                              PL::kSmem);
  if (e != cudaSuccess) return e;
  mark_begin(st, kTimeFwd);
  if (pair)
    e = launch_pdl_cluster(tk_fwd_kernel<true>, (unsigned)grid, 224, PL::kSmem, st, 2u, mq, mkv, mcmp, has_cmp, p,
                           o, lse);
  else
    e = launch_pdl(tk_fwd_kernel<false>, (unsigned)grid, 192, PL::kSmem, st, mq, mkv, mcmp, has_cmp, p, o, lse);
  count_launch();
  mark_end(st, kTimeFwd);
  return e;
}

}  // namespace sa
