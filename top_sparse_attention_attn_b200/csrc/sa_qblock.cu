// sa_qblock.cu -- query-stationary kernels for block-level selection with
// 64-row blocks: the forward (O, lse) and the dQ pass of the key-stationary
// backward.
//
// aclnnNsaSelectedAttentionInfer "Formula" (forward) and
// aclnnSparseFlashAttentionGrad "Formula" Phases 2-3 (dS, dQ = dS K scale).
//
// Persistent, warp-specialised CTAs (1 producer warp + 4 consumer warps).  A
// work item is (query token, kv-head, 16-head slice).  The producer walks the
// CTA's work items and streams each selected block (64 K rows and 64 V rows of
// one kv-head) into a ring of shared-memory stages with 2D TMA box loads
// (128-byte swizzle), running ahead across work items.  Consumer warp w owns
// rows [16w, 16w+16) of every block: it keeps its own online-softmax state
// (forward) or dQ partial sum (dQ pass) in registers, on mma.sync m16n8k16
// bf16 with fp32 accumulation, so blocks need no barrier between warps.  The
// four partial states are merged once per work item through shared memory.
#include <cuda.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "sa_device.cuh"
#include "sa_launch.h"
#include "sa_qblock.h"
#include "sa_tc.cuh"

namespace sa {

constexpr float kLog2eQb = 1.4426950408889634f;
constexpr float kLn2Qb = 0.6931471805599453f;

// NCTA = CTAs per SM the plan is sized for.  With two, the ring is two stages
// and the per-warp partials are merged in two column halves, so two CTAs (eight
// consumer warps) share an SM: the forward is bound by mma.sync dependency
// latency, which more resident warps hide.
template <int DQK, int DV, bool DQ, int NCTA>
struct QbPlan {
  static constexpr int kStage = 64 * (DQK + DV) * 2;  // K block + V block
  static constexpr int W = DQ ? DQK : DV;              // accumulator width
  static constexpr int NR = (NCTA > 1 && W > 64) ? 2 : 1;  // merge rounds
  static constexpr int WC = W / NR;                    // columns merged per round
  static constexpr int kComb = 4 * 16 * WC * 4 + 4 * 16 * 2 * 4;  // partials + (m, l)
  static constexpr int kStatic = 6 * 1024;             // static shared memory
  static constexpr int kBudget = (227 * 1024) / NCTA - 1024 - kComb - kStatic;
  // small stages (d <= 64): a short ring keeps the CTA small enough for two or
  // more per SM, which small problems need more than pipeline depth
  static constexpr int kMaxStages = NCTA > 1 ? 2 : (kStage <= 16384 ? 3 : 6);
  static constexpr int kStages = (kBudget / kStage) > kMaxStages ? kMaxStages : (kBudget / kStage);
  static constexpr int oRing = 0;
  static constexpr int oComb = kStages * kStage;
  static constexpr int kSmem = oComb + kComb + 1024;
  static_assert(kStages >= 2, "not enough shared memory for the ring");
};

// 16-byte chunk c of row r in a tile stored as slabs of rows_per_slab x 128 bytes (TMA 128-byte swizzle).
__device__ __forceinline__ uint32_t slab_addr(uint32_t base, int rows_per_slab, int r, int c) {
  return base + (uint32_t)((c >> 3) * rows_per_slab * 128 + r * 128 + ((((c & 7) ^ (r & 7))) << 4));
}

struct QbBars {
  uint64_t full[6], empty[6];
  int abort_flag;
};

// Warp-collective: the usable slots of a work item (blk_usable: valid, in range,
// not fully masked), in slot order, written to xs (shared, kQbMaxSlots entries);
// returns their number.  An index past the end of its sequence raises the
// status word's index bit.  The host routes only topk <= kQbMaxSlots here.
__device__ __forceinline__ int qb_slots(const QbArgs& a, const Unit& u, int* xs, int lane) {
  const long long ug = (long long)u.tq * a.Hkv + u.g;
  int n = a.topk;
  if (a.ori_len) n = min(n, max(0, __ldg(a.ori_len + ug)));
  int cnt = 0;
  for (int s0 = 0; s0 < n; s0 += 32) {
    const int s = s0 + lane;
    bool ok = false;
    int x = -1;
    if (s < n) {
      x = __ldg(a.ori_idx + ug * a.topk + s);
      ok = blk_usable(x, u.Lk, u.ta, a.ori_mask, a.wl, a.wr);
      if (x >= 0 && (long long)x * kTileRows >= u.Lk && a.status) atomicOr(a.status, kStatusIndexRange);
    }
    const unsigned m = __ballot_sync(0xffffffffu, ok);
    const int pos = cnt + __popc(m & ((1u << lane) - 1u));
    if (ok && pos < kQbMaxSlots) xs[pos] = x;
    cnt += __popc(m);
  }
  __syncwarp();
  return min(cnt, kQbMaxSlots);
}

__device__ __forceinline__ Unit qb_unit(const QbArgs& a, int tq, int g) {
  Prob p;
  p.layout = a.layout;
  p.B = a.B;
  p.s_q = a.s_q;
  p.s_kv = a.s_kv;
  p.Tkv = a.Tkv;
  p.Tcmp = 0;
  p.cu_q = a.cu_q;
  p.cu_kv = a.cu_kv;
  p.cu_cmp = nullptr;
  p.topk = 0;  // only the sequence geometry is needed here
  p.cmp_topk = 0;
  p.ori_mask = kMaskNone;
  p.ratio = 1;
  p.Hkv = a.Hkv;
  p.ori_len = nullptr;
  p.cmp_len = nullptr;
  p.wl = p.wr = 0;
  return make_unit(p, tq, g);
}

template <int DQK, int DV, bool DQ, int NCTA>
__global__ void __launch_bounds__(160, NCTA) qb_kernel(const __grid_constant__ CUtensorMap mapK,
                                                       const __grid_constant__ CUtensorMap mapV, const QbArgs a) {
  using PL = QbPlan<DQK, DV, DQ, NCTA>;
  constexpr int S = PL::kStages;
  constexpr int NQK = DQK / 16;  // k steps over d_qk
  constexpr int NV = DV / 16;    // k steps over d_v
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  __shared__ QbBars bars;
  __shared__ int slot_x[5][kQbMaxSlots];  // per warp: the current item's usable block indices
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t ring = smem_u32(smem + PL::oRing);
  float* comb = reinterpret_cast<float*>(smem + PL::oComb);
  volatile int* abort_flag = &bars.abort_flag;
  const int n_hsl = (a.G + 15) >> 4;
  const long long n_items = (long long)a.Tq * a.Hkv * n_hsl;

  if (threadIdx.x == 0) {
    bars.abort_flag = 0;
    for (int s = 0; s < S; ++s) {
      mbar_init(&bars.full[s], 1);
      mbar_init(&bars.empty[s], 4);
    }
    mbar_fence_init();
  }
  __syncthreads();

  if (warp == 4) {
    // ------------------------------------------------------------ producer
    int* xs = slot_x[4];
    long long t = 0;  // blocks streamed so far
    bool ok = true;
    if (lane == 0) {
      tma_prefetch_desc(&mapK);
      tma_prefetch_desc(&mapV);
    }
    for (long long it = blockIdx.x; ok && it < n_items; it += gridDim.x) {
      const int unit = (int)(it / n_hsl);
      const int tq = unit / a.Hkv, g = unit - tq * a.Hkv;
      const Unit u = qb_unit(a, tq, g);
      const int n = qb_slots(a, u, xs, lane);
      for (int i = 0; i < n; ++i, ++t) {
        const int st = (int)(t % S);
        if (lane == 0) {
          if (t >= S && !mbar_wait(&bars.empty[st], (uint32_t)(((t / S) - 1) & 1), abort_flag, a.status)) {
            ok = false;
          } else {
            const uint32_t sk = ring + st * PL::kStage, sv = sk + 64 * DQK * 2;
            const int row = u.kv0 + 64 * xs[i];
            mbar_arrive_tx(&bars.full[st], (uint32_t)PL::kStage);
            for (int s2 = 0; s2 < DQK / 64; ++s2)
              tma_load_2d(sk + s2 * 8192, &mapK, g * DQK + 64 * s2, row, &bars.full[st]);
            for (int s2 = 0; s2 < DV / 64; ++s2)
              tma_load_2d(sv + s2 * 8192, &mapV, g * DV + 64 * s2, row, &bars.full[st]);
          }
        }
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) break;
      }
      __syncwarp();
    }
    // drain: the last S stages must have landed before the CTA exits
    if (lane == 0)
      for (long long k = (t > S ? t - S : 0); k < t; ++k) mbar_wait_drain(&bars.full[k % S], (uint32_t)((k / S) & 1));
    return;
  }

  // ------------------------------------------------------------ consumers
  const int r0 = lane >> 2;
  const int cq = 2 * (lane & 3);
  long long t = 0;
  bool ok = true;
  for (long long it = blockIdx.x; it < n_items; it += gridDim.x) {
    const int unit = (int)(it / n_hsl), hsl = (int)(it - (long long)unit * n_hsl);
    const int tq = unit / a.Hkv, g = unit - tq * a.Hkv;
    const Unit u = qb_unit(a, tq, g);
    const int h0 = g * a.G + hsl * 16;
    const int nh = min(16, a.G - hsl * 16);
    int* xs = slot_x[warp];
    const int n = qb_slots(a, u, xs, lane);

    // query rows as A fragments (rows >= nh are zero)
    uint32_t qf[NQK][4];
    {
      const bf16* q0 = a.q + ((long long)tq * a.Hq + h0) * DQK;
#pragma unroll
      for (int k = 0; k < NQK; ++k)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int row = r0 + 8 * (j & 1), col = 16 * k + cq + 8 * (j >> 1);
          qf[k][j] = row < nh ? __ldg(reinterpret_cast<const uint32_t*>(q0 + (long long)row * DQK + col)) : 0u;
        }
    }
    float lse2[2] = {INFINITY, INFINITY}, dlt[2] = {0.f, 0.f};
    uint32_t df[DQ ? NV : 1][4];
    if (DQ) {
      const bf16* d0 = a.d_o + ((long long)tq * a.Hq + h0) * DV;
#pragma unroll
      for (int k = 0; k < (DQ ? NV : 1); ++k)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int row = r0 + 8 * (j & 1), col = 16 * k + cq + 8 * (j >> 1);
          df[k][j] = row < nh ? __ldg(reinterpret_cast<const uint32_t*>(d0 + (long long)row * DV + col)) : 0u;
        }
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        const int row = r0 + 8 * r;
        if (row < nh) {
          const long long ih = (long long)tq * a.Hq + h0 + row;
          lse2[r] = __ldg(a.lse + ih) * kLog2eQb;
          dlt[r] = __ldg(a.delta + ih);
        }
      }
    }
    constexpr int NACC = DQ ? DQK / 8 : DV / 8;  // 8-column n tiles of the accumulator
    float acc[NACC][4];
#pragma unroll
    for (int i = 0; i < NACC; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;
    float m[2] = {-INFINITY, -INFINITY}, l[2] = {0.f, 0.f};

    for (int i = 0; i < n; ++i, ++t) {
      const int st = (int)(t % S);
      if (ok && !mbar_wait(&bars.full[st], (uint32_t)((t / S) & 1), abort_flag, a.status)) ok = false;
      if (ok) {
        const uint32_t sk = ring + st * PL::kStage, sv = sk + 64 * DQK * 2;
        const int x = xs[i];
        // S_w = Q K_w^T: the warp's 16 block rows
        // two independent accumulation chains per n tile (even / odd k steps)
        float s[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
        float s2[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
        for (int k = 0; k < NQK; ++k) {
          uint32_t b[4];
          const int rr = 16 * warp + (lane & 7) + ((lane >> 4) << 3);
          ldsm_x4(b, slab_addr(sk, 64, rr, 2 * k + ((lane >> 3) & 1)));
          if (k & 1) {
            mma16816(s2[0], qf[k], b[0], b[1]);
            mma16816(s2[1], qf[k], b[2], b[3]);
          } else {
            mma16816(s[0], qf[k], b[0], b[1]);
            mma16816(s[1], qf[k], b[2], b[3]);
          }
        }
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
          for (int j = 0; j < 4; ++j) s[nt][j] += s2[nt][j];
        // visibility of the warp's block rows for this query token (blk_rows)
        int vlo, vhi;
        blk_rows(x, u.Lk, u.ta, a.ori_mask, a.wl, a.wr, &vlo, &vhi);
        bool vis[2][2];
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int off = 16 * warp + 8 * nt + cq + e;
            vis[nt][e] = off >= vlo && off <= vhi;
          }
        uint32_t pa[4];  // P (forward) or dS (dQ pass) as an A fragment over the 16 block rows
        if (!DQ) {
          float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
          for (int nt = 0; nt < 2; ++nt)
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const float v = vis[nt][j & 1] ? s[nt][j] * a.scale_log2 : -INFINITY;
              s[nt][j] = v;
              mx[j >> 1] = fmaxf(mx[j >> 1], v);
            }
          float alpha[2], muse[2];
#pragma unroll
          for (int r = 0; r < 2; ++r) {
            const float mn = fmaxf(m[r], warp_max4(mx[r]));
            muse[r] = mn == -INFINITY ? 0.f : mn;
            alpha[r] = exp2f(m[r] - muse[r]);
            m[r] = mn;
          }
          float ps[2] = {0.f, 0.f};
          float pv[2][4];
#pragma unroll
          for (int nt = 0; nt < 2; ++nt)
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              pv[nt][j] = exp2f(s[nt][j] - muse[j >> 1]);
              ps[j >> 1] += pv[nt][j];
            }
#pragma unroll
          for (int r = 0; r < 2; ++r) l[r] = l[r] * alpha[r] + warp_sum4(ps[r]);
#pragma unroll
          for (int c = 0; c < NACC; ++c) {
            acc[c][0] *= alpha[0];
            acc[c][1] *= alpha[0];
            acc[c][2] *= alpha[1];
            acc[c][3] *= alpha[1];
          }
          pa[0] = pack_bf16(pv[0][0], pv[0][1]);
          pa[1] = pack_bf16(pv[0][2], pv[0][3]);
          pa[2] = pack_bf16(pv[1][0], pv[1][1]);
          pa[3] = pack_bf16(pv[1][2], pv[1][3]);
          // O_w += P V_w
#pragma unroll
          for (int c = 0; c < DV / 16; ++c) {
            uint32_t b[4];
            const int rr = 16 * warp + (lane & 7) + (((lane >> 3) & 1) << 3);
            ldsm_x4_t(b, slab_addr(sv, 64, rr, 2 * c + (lane >> 4)));
            mma16816(acc[2 * c], pa, b[0], b[1]);
            mma16816(acc[2 * c + 1], pa, b[2], b[3]);
          }
        } else {
          // dP_w = dO V_w^T
          float dp[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
          for (int k = 0; k < NV; ++k) {
            uint32_t b[4];
            const int rr = 16 * warp + (lane & 7) + ((lane >> 4) << 3);
            ldsm_x4(b, slab_addr(sv, 64, rr, 2 * k + ((lane >> 3) & 1)));
            mma16816(dp[0], df[k], b[0], b[1]);
            mma16816(dp[1], df[k], b[2], b[3]);
          }
          float dsv[2][4];
#pragma unroll
          for (int nt = 0; nt < 2; ++nt)
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const float p = vis[nt][j & 1] ? exp2f(s[nt][j] * a.scale_log2 - lse2[j >> 1]) : 0.f;
              dsv[nt][j] = p * (dp[nt][j] - dlt[j >> 1]);
            }
          pa[0] = pack_bf16(dsv[0][0], dsv[0][1]);
          pa[1] = pack_bf16(dsv[0][2], dsv[0][3]);
          pa[2] = pack_bf16(dsv[1][0], dsv[1][1]);
          pa[3] = pack_bf16(dsv[1][2], dsv[1][3]);
          // dQ_w += dS K_w
#pragma unroll
          for (int c = 0; c < DQK / 16; ++c) {
            uint32_t b[4];
            const int rr = 16 * warp + (lane & 7) + (((lane >> 3) & 1) << 3);
            ldsm_x4_t(b, slab_addr(sk, 64, rr, 2 * c + (lane >> 4)));
            mma16816(acc[2 * c], pa, b[0], b[1]);
            mma16816(acc[2 * c + 1], pa, b[2], b[3]);
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars.empty[st]);
    }

    // ---- merge the four warps' partials (named barrier over the consumer warps),
    // PL::NR rounds of PL::WC columns
    constexpr int W = PL::W, WC = PL::WC;
    float* part = comb;                   // [4][16][WC]
    float* stat = comb + 4 * 16 * WC;     // [4][16][2]
    if (!DQ && (lane & 3) == 0) {
      stat[(warp * 16 + r0) * 2] = m[0];
      stat[(warp * 16 + r0) * 2 + 1] = l[0];
      stat[(warp * 16 + r0 + 8) * 2] = m[1];
      stat[(warp * 16 + r0 + 8) * 2 + 1] = l[1];
    }
    const int ct = threadIdx.x;  // 0..127: thread -> (row, column group of 8)
    const int row = ct >> 3, cg = ct & 7;
#pragma unroll
    for (int hr = 0; hr < PL::NR; ++hr) {
#pragma unroll
      for (int c = 0; c < NACC; ++c) {
        if (c / (WC / 8) != hr) continue;
        const int col = 8 * c + cq - hr * WC;
        *reinterpret_cast<float2*>(part + (warp * 16 + r0) * WC + col) = make_float2(acc[c][0], acc[c][1]);
        *reinterpret_cast<float2*>(part + (warp * 16 + r0 + 8) * WC + col) = make_float2(acc[c][2], acc[c][3]);
      }
      asm volatile("bar.sync 1, 128;\n" ::: "memory");
      if (row < nh) {
        const long long ih = (long long)tq * a.Hq + h0 + row;
        if (!DQ) {
          float M = a.sinks ? __ldg(a.sinks + h0 + row) * kLog2eQb : -INFINITY;
          for (int w2 = 0; w2 < 4; ++w2) M = fmaxf(M, stat[(w2 * 16 + row) * 2]);
          const float Mu = M == -INFINITY ? 0.f : M;
          float al[4], Lsum = a.sinks ? exp2f(__ldg(a.sinks + h0 + row) * kLog2eQb - Mu) : 0.f;
          for (int w2 = 0; w2 < 4; ++w2) {
            al[w2] = exp2f(stat[(w2 * 16 + row) * 2] - Mu);
            Lsum += al[w2] * stat[(w2 * 16 + row) * 2 + 1];
          }
          const float inv = Lsum > 0.f ? 1.f / Lsum : 0.f;
          bf16* orow = a.o + ih * DV + hr * WC;
          for (int c = cg * 8; c < WC; c += 64) {
            float v[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              float s2 = 0.f;
#pragma unroll
              for (int w2 = 0; w2 < 4; ++w2) s2 += al[w2] * part[(w2 * 16 + row) * WC + c + e];
              v[e] = s2 * inv;
            }
            uint4 pk;
            pk.x = pack_bf16(v[0], v[1]);
            pk.y = pack_bf16(v[2], v[3]);
            pk.z = pack_bf16(v[4], v[5]);
            pk.w = pack_bf16(v[6], v[7]);
            *reinterpret_cast<uint4*>(orow + c) = pk;
          }
          if (cg == 0 && hr == 0) a.lse[ih] = Lsum > 0.f ? (M + log2f(Lsum)) * kLn2Qb : INFINITY;
        } else {
          bf16* qrow = a.dq + ih * DQK + hr * WC;
          for (int c = cg * 8; c < WC; c += 64) {
            float v[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              float s2 = 0.f;
#pragma unroll
              for (int w2 = 0; w2 < 4; ++w2) s2 += part[(w2 * 16 + row) * WC + c + e];
              v[e] = s2 * a.scale;
            }
            uint4 pk;
            pk.x = pack_bf16(v[0], v[1]);
            pk.y = pack_bf16(v[2], v[3]);
            pk.z = pack_bf16(v[4], v[5]);
            pk.w = pack_bf16(v[6], v[7]);
            *reinterpret_cast<uint4*>(qrow + c) = pk;
          }
        }
      }
      asm volatile("bar.sync 1, 128;\n" ::: "memory");
    }
    (void)W;
  }
}

// Inspection: one warp per (token, kv-head) unit runs qb_unit / qb_slots /
// blk_rows exactly as qb_kernel does and records every usable slot as
// {unit, block, lo, hi}.
__global__ void __launch_bounds__(128) qb_debug_slots_kernel(const QbArgs a, int4* rec, long long max_rec,
                                                             int* n_rec) {
  __shared__ int xs_all[4][kQbMaxSlots];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long unit = (long long)blockIdx.x * 4 + warp;
  if (unit >= (long long)a.Tq * a.Hkv) return;  // whole warps leave together
  const int tq = (int)(unit / a.Hkv), g = (int)(unit - (long long)tq * a.Hkv);
  const Unit u = qb_unit(a, tq, g);
  int* xs = xs_all[warp];
  const int n = qb_slots(a, u, xs, lane);
  for (int i = lane; i < n; i += 32) {
    int lo, hi;
    blk_rows(xs[i], u.Lk, u.ta, a.ori_mask, a.wl, a.wr, &lo, &hi);
    const int k = atomicAdd(n_rec, 1);
    if (k < max_rec) rec[k] = make_int4((int)unit, xs[i], lo, hi);
  }
}

cudaError_t launch_qb_debug_slots(const QbArgs& a, int4* rec, long long max_rec, int* n_rec, cudaStream_t st) {
  const long long units = (long long)a.Tq * a.Hkv;
  if (units == 0) return cudaSuccess;
  qb_debug_slots_kernel<<<(unsigned)((units + 3) / 4), 128, 0, st>>>(a, rec, max_rec, n_rec);
  count_launch();
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
bool qb_path_built(int dqk, int dv) {
  return (dqk == 64 && dv == 64) || (dqk == 128 && dv == 128) || (dqk == 192 && dv == 128);
}

template <int DQK, int DV, bool DQ>
static cudaError_t qb_launch_t(const QbArgs& a, const void* k, const void* v, cudaStream_t st, int time_id) {
  constexpr int NCTA = DQ ? 1 : 2;  // the dQ pass needs more registers per thread
  using PL = QbPlan<DQK, DV, DQ, NCTA>;
  CUtensorMap mk, mv;
  if (!make_tmap_bf16(&mk, k, (uint64_t)a.Tkv, (uint64_t)a.Hkv * DQK, (uint64_t)a.Hkv * DQK * 2, 64) ||
      !make_tmap_bf16(&mv, v, (uint64_t)a.Tkv, (uint64_t)a.Hkv * DV, (uint64_t)a.Hkv * DV * 2, 64))
    return cudaErrorInvalidValue;
  auto kern = qb_kernel<DQK, DV, DQ, NCTA>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, PL::kSmem);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 148, per_sm = 1;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, 160, PL::kSmem) != cudaSuccess || per_sm < 1)
    per_sm = 1;
  const long long n_items = (long long)a.Tq * a.Hkv * ((a.G + 15) / 16);
  const long long slots = (long long)sms * per_sm;
  const long long grid = n_items < slots ? n_items : slots;
  if (grid == 0) return cudaSuccess;
  mark_begin(st, time_id);
  kern<<<(unsigned)grid, 160, PL::kSmem, st>>>(mk, mv, a);
  count_launch();
  mark_end(st, time_id);
  return cudaGetLastError();
}

cudaError_t launch_qb(const QbArgs& a, const void* k, const void* v, bool dq, cudaStream_t st) {
  const int tid = dq ? kTimeBwdDQ : kTimeFwd;
  if (a.dqk == 64 && a.dv == 64)
    return dq ? qb_launch_t<64, 64, true>(a, k, v, st, tid) : qb_launch_t<64, 64, false>(a, k, v, st, tid);
  if (a.dqk == 128 && a.dv == 128)
    return dq ? qb_launch_t<128, 128, true>(a, k, v, st, tid) : qb_launch_t<128, 128, false>(a, k, v, st, tid);
  if (a.dqk == 192 && a.dv == 128)
    return dq ? qb_launch_t<192, 128, true>(a, k, v, st, tid) : qb_launch_t<192, 128, false>(a, k, v, st, tid);
  return cudaErrorInvalidValue;
}

}  // namespace sa
