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
  Prob p = {};  // only the sequence geometry is set: no indices, no compressed KV
  p.layout = a.layout;
  p.B = a.B;
  p.s_q = a.s_q;
  p.s_kv = a.s_kv;
  p.Tkv = a.Tkv;
  p.Tcmp = 0;
  p.cu_q = a.cu_q;
  p.cu_kv = a.cu_kv;
  p.cu_cmp = nullptr;
  p.topk = 0;
  p.cmp_topk = 0;
  p.cmpk = nullptr;
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

// ---------------------------------------------------------------------------
// Forward for 64-row blocks on tcgen05 (aclnnNsaSelectedAttentionInfer,
// "Formula": O = Softmax(Q K_sel^T scale) V_sel, lse with the sink).
// Persistent: one CTA per SM walks work items (query token, kv-head, slice of
// up to 16 heads).  Transposed so that the tensor-core M dimension is keys or
// value dims, which a 16-head slice could not fill:
//   S_j^T [128 keys x 16 heads] = K_j Q^T  pair j of blocks (2j, 2j + 1) of a chunk
//                                          of up to 16 usable blocks, stacked in one
//                                          ring stage (M = 128; 128 columns per chunk,
//                                          two buffers)
//   softmax over the chunk's keys per head (cross-warp reductions of the
//   running maximum and sum; a later chunk of the same item rescales O^T)
//   O^T [d_v x 16] += V_b^T P_b^T          V_b as an MN-major A, P_b^T [16][64]
//                                          (two buffers, one per item in flight)
// The producer warp streams through one ring of TMA-loaded stages, in the order
// K(chunk c), V(chunk c - 1): the scores of a chunk are formed while the
// previous chunk's softmax runs, and the ring keeps loading across items.  An
// item without usable blocks flushes the pending V chunk (in the producer and
// the MMA warp alike), so a chunk's V never waits behind a later item.  The
// usable slots and each block's visible rows are qb_slots / blk_rows, as in every
// block kernel.
// ---------------------------------------------------------------------------
template <int DQK, int DV>
struct BqPlan {
  static constexpr int NH = 16;   // heads per item: the N of every MMA
  static constexpr int CH = 16;   // blocks per chunk: their scores fill 128 TMEM columns
  static constexpr int NIT = 3;   // item descriptors in flight
  static constexpr int kStage = 128 * (DQK > DV ? DQK : DV) * 2;  // a pair of blocks
  static constexpr int kQ = (DQK / 64) * NH * 128;              // one Q slice
  static constexpr int oQ = 0;                                  // two Q slices
  static constexpr int oP = (2 * kQ + 1023) / 1024 * 1024;      // CH blocks of P^T [16][64] bf16
  static constexpr int oRedM = oP + CH * NH * 128;              // [4 warps][16] maxima
  static constexpr int oRedL = oRedM + 4 * NH * 4;              // [4 warps][16] sums
  static constexpr int oInfo = oRedL + 4 * NH * 4;              // NIT x (count + usable block indices)
  static constexpr int kInfo = (1 + kQbMaxSlots) * 4;
  static constexpr int oRing = (oInfo + NIT * kInfo + 1023) / 1024 * 1024;
  static constexpr int kBudget = 225 * 1024;
  static constexpr int NST0 = (kBudget - oRing) / kStage;
  static constexpr int NST = NST0 > 8 ? 8 : NST0;
  static constexpr int kSmem = oRing + NST * kStage;
  static constexpr int cS = 0, cO = 256;                        // S: 2 x 128 columns; O: 2 x 16
  static constexpr uint32_t kAlloc = 512;
  static_assert(NST >= 3, "ring too small");
  static_assert(kStage % 1024 == 0 && oP % 1024 == 0 && oRing % 1024 == 0, "swizzle alignment");
  static_assert(kSmem + 1024 <= 227 * 1024, "shared memory plan too large");
};

struct BqBars {
  uint64_t info_full[3], info_free[3], q_full[2], q_empty[2], kv_full[8], kv_empty[8];
  uint64_t s_full[2], s_free[2], p_full, pv_done, o_full[2], o_free[2], stats_full[2];
  float stat_m[2][16], stat_l[2][16];  // an item's running maximum and sum per head, softmax -> epilogue
  uint32_t tmem_base;
  int abort_flag;
};

// The chunk walk shared by the three roles: item k's n usable blocks split into
// chunks of at most CH; an item with n = 0 has none.
struct BqWalk {
  int k, slot, n, nch, c_in;  // item (local index), its info slot, count, chunks, chunk within the item
};

template <int DQK, int DV>
__global__ void __launch_bounds__(320, 1) bq_fwd_kernel(const __grid_constant__ CUtensorMap mapQ,
                                                        const __grid_constant__ CUtensorMap mapK,
                                                        const __grid_constant__ CUtensorMap mapV, const QbArgs a) {
  using PL = BqPlan<DQK, DV>;
  constexpr int NST = PL::NST, CH = PL::CH, NIT = PL::NIT;
  extern __shared__ __align__(1024) uint8_t smem[];
  __shared__ BqBars bars;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (smem_u32(smem) & 1023) {
    if (threadIdx.x == 0 && a.status) atomicOr(a.status, kStatusSmemAlign);
    return;
  }
  const int n_hsl = (a.G + 15) >> 4;
  const long long n_items = (long long)a.Tq * a.Hkv * n_hsl;
  const uint32_t sQ = smem_u32(smem + PL::oQ), sRing = smem_u32(smem + PL::oRing), sP = smem_u32(smem + PL::oP);
  float* redm = reinterpret_cast<float*>(smem + PL::oRedM);
  float* redl = reinterpret_cast<float*>(smem + PL::oRedL);
  volatile int* abort_flag = &bars.abort_flag;
  auto info_n = [&](int slot) -> volatile int* { return reinterpret_cast<volatile int*>(smem + PL::oInfo + slot * PL::kInfo); };
  auto info_xs = [&](int slot) -> int* { return reinterpret_cast<int*>(smem + PL::oInfo + slot * PL::kInfo + 4); };
  // item k of this CTA -> (token, kv-head, first head, heads)
  auto item_of = [&](int k, int* tq, int* g, int* h0, int* nh) -> bool {
    const long long it = blockIdx.x + (long long)k * gridDim.x;
    if (it >= n_items) return false;
    const int unit = (int)(it / n_hsl), hsl = (int)(it - (long long)unit * n_hsl);
    *tq = unit / a.Hkv;
    *g = unit - *tq * a.Hkv;
    *h0 = *g * a.G + hsl * 16;
    *nh = min(16, a.G - hsl * 16);
    return true;
  };

  if (threadIdx.x == 0) {
    bars.abort_flag = 0;
    for (int s = 0; s < NIT; ++s) {
      mbar_init(&bars.info_full[s], 32);
      mbar_init(&bars.info_free[s], 1 + 128 + 128);  // MMA thread, softmax and epilogue warps
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bars.q_full[s], 1);
      mbar_init(&bars.q_empty[s], 1);
      mbar_init(&bars.s_full[s], 1);
      mbar_init(&bars.s_free[s], 128);
      mbar_init(&bars.o_full[s], 1);
      mbar_init(&bars.o_free[s], 128);
      mbar_init(&bars.stats_full[s], 128);
    }
    for (int s = 0; s < NST; ++s) {
      mbar_init(&bars.kv_full[s], 1);
      mbar_init(&bars.kv_empty[s], 1);
    }
    mbar_init(&bars.p_full, 128);
    mbar_init(&bars.pv_done, 1);
    mbar_fence_init();
    tma_prefetch_desc(&mapQ);
    tma_prefetch_desc(&mapK);
    tma_prefetch_desc(&mapV);
  }
  if (warp == 1) tmem_alloc(&bars.tmem_base, PL::kAlloc);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars.tmem_base;

  if (warp == 0) {
    // ------------------------------------------------------------ producer (whole warp)
    // items in order: the usable slots to the info ring, the Q slice, then the
    // blocks in the order K(chunk c), V(chunk c - 1)
    int t = 0, qk = 0;
    bool ok = true;
    int pv_slot = -1, pv_first = 0, pv_nb = 0, pv_row0 = 0, pv_g = 0;  // the chunk whose V is pending
    auto load_blocks = [&](bool is_v, int slot, int first, int nb, int kv0, int g) {
      // pairs of blocks: block 2j in rows 0..63 of the stage's slabs, 2j + 1 in rows 64..127
      for (int j = 0; ok && 2 * j < nb; ++j, ++t) {
        const int st = t % NST, nbp = min(2, nb - 2 * j);
        if (lane == 0) {
          if (t >= NST && !mbar_wait(&bars.kv_empty[st], ((t / NST) - 1) & 1, abort_flag, a.status)) {
            ok = false;
          } else {
            const uint32_t stage = sRing + st * PL::kStage;
            const int D = is_v ? DV : DQK;
            mbar_arrive_tx(&bars.kv_full[st], (uint32_t)(nbp * 64 * D * 2));
            for (int e = 0; e < nbp; ++e) {
              const int row = kv0 + 64 * info_xs(slot)[first + 2 * j + e];
              for (int s = 0; s < D / 64; ++s) {
                if (is_v)
                  tma_load_2d(stage + s * 16384 + e * 8192, &mapV, g * DV + 64 * s, row, &bars.kv_full[st]);
                else
                  tma_load_2d(stage + s * 16384 + e * 8192, &mapK, g * DQK + 64 * s, row, &bars.kv_full[st]);
              }
            }
          }
        }
        ok = __shfl_sync(0xffffffffu, ok, 0);
      }
    };
    for (int k = 0; ok; ++k) {
      int tq, g, h0, nh;
      const bool have = item_of(k, &tq, &g, &h0, &nh);
      const int slot = k % NIT;
      if (k >= NIT) {
        bool w = lane != 0 || mbar_wait(&bars.info_free[slot], ((k / NIT) - 1) & 1, abort_flag, a.status);
        ok = __shfl_sync(0xffffffffu, w, 0);
        if (!ok) break;
      }
      int n = -1;  // -1: no more items
      if (have) {
        const Unit u = qb_unit(a, tq, g);
        n = qb_slots(a, u, info_xs(slot), lane);
        if (lane == 0) *info_n(slot) = n;
        __syncwarp();
        mbar_arrive(&bars.info_full[slot]);
        if (n == 0 && pv_slot >= 0) {
          // an item without blocks: the pending V chunk goes now (the MMA warp issues its
          // P V at the same point), before its slot list can be reused
          load_blocks(true, pv_slot, pv_first, pv_nb, pv_row0, pv_g);
          pv_slot = -1;
        }
        if (n > 0) {
          const int qs = qk & 1;
          if (lane == 0) {
            if (qk >= 2 && !mbar_wait(&bars.q_empty[qs], ((qk >> 1) - 1) & 1, abort_flag, a.status)) {
              ok = false;
            } else {
              mbar_arrive_tx(&bars.q_full[qs], (uint32_t)(PL::NH * DQK * 2));
              for (int s = 0; s < DQK / 64; ++s)
                tma_load_2d(sQ + qs * PL::kQ + s * (PL::NH * 128), &mapQ, 64 * s, tq * a.Hq + h0, &bars.q_full[qs]);
            }
          }
          ok = __shfl_sync(0xffffffffu, ok, 0);
          ++qk;
          const int nch = (n + CH - 1) / CH;
          for (int c = 0; ok && c < nch; ++c) {
            const int nb = min(CH, n - c * CH);
            load_blocks(false, slot, c * CH, nb, u.kv0, g);
            if (pv_slot >= 0) load_blocks(true, pv_slot, pv_first, pv_nb, pv_row0, pv_g);
            pv_slot = slot;
            pv_first = c * CH;
            pv_nb = nb;
            pv_row0 = u.kv0;
            pv_g = g;
          }
        }
      } else {
        if (lane == 0) *info_n(slot) = -1;
        __syncwarp();
        mbar_arrive(&bars.info_full[slot]);
        break;
      }
    }
    if (ok && pv_slot >= 0) load_blocks(true, pv_slot, pv_first, pv_nb, pv_row0, pv_g);
    // drain: every issued load lands before the CTA exits
    if (lane == 0) {
      for (int k2 = t > NST ? t - NST : 0; k2 < t; ++k2) mbar_wait_drain(&bars.kv_full[k2 % NST], (k2 / NST) & 1);
      for (int q2 = qk > 2 ? qk - 2 : 0; q2 < qk; ++q2) mbar_wait_drain(&bars.q_full[q2 & 1], (q2 >> 1) & 1);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idS = idesc_bf16(128, PL::NH, false, false);
      constexpr uint32_t idO = idesc_bf16(DV >= 128 ? 128 : 64, PL::NH, true, false);
      int t = 0, c = 0, qk = 0, ok_items = 0;
      bool ok = true;
      // the chunk whose P V is pending: its chunk number, blocks, O buffer and whether it opens its item
      int pv_c = -1, pv_nb = 0, pv_ob = 0;
      bool pv_first = false, pv_last = false;
      auto issue_pv = [&]() {
        if (!mbar_wait(&bars.p_full, pv_c & 1, abort_flag, a.status)) { ok = false; return; }
        tc_fence_after();
        for (int j = 0; ok && 2 * j < pv_nb; ++j, ++t) {
          const int st = t % NST;
          if (!mbar_wait(&bars.kv_full[st], (t / NST) & 1, abort_flag, a.status)) { ok = false; break; }
          tc_fence_after();
          const uint32_t stage = sRing + st * PL::kStage;
          for (int e = 0; e < 2 && 2 * j + e < pv_nb; ++e) {
            const int b = 2 * j + e;
            for (int kk = 0; kk < 4; ++kk)
              mma_bf16(tmem + PL::cO + 16 * pv_ob, sdesc(stage + e * 8192 + kk * 2048, 16384, 1024),
                       sdesc(sP + b * 2048 + kk * 32, 16, 1024), idO, (!pv_first || b > 0 || kk > 0) ? 1u : 0u);
          }
          mma_commit(&bars.kv_empty[st]);
        }
        if (ok) {
          mma_commit(&bars.pv_done);
          if (pv_last) mma_commit(&bars.o_full[pv_ob]);  // the item's O^T is final
        }
      };
      for (int k = 0; ok; ++k) {
        const int slot = k % NIT;
        if (!mbar_wait(&bars.info_full[slot], (k / NIT) & 1, abort_flag, a.status)) break;
        const int n = *info_n(slot);
        mbar_arrive(&bars.info_free[slot]);
        if (n < 0) break;
        if (n == 0) {
          if (pv_c >= 0) issue_pv();  // mirrors the producer: the pending V chunk comes now
          pv_c = -1;
          continue;
        }
        const int qs = qk & 1, ob = ok_items & 1;
        if (!mbar_wait(&bars.q_full[qs], (qk >> 1) & 1, abort_flag, a.status)) break;
        // the O buffer of this item was read by the epilogue of item ok_items - 2
        if (ok_items >= 2 && !mbar_wait(&bars.o_free[ob], ((ok_items >> 1) - 1) & 1, abort_flag, a.status)) break;
        const int nch = (n + CH - 1) / CH;
        for (int cc = 0; ok && cc < nch; ++cc, ++c) {
          const int nb = min(CH, n - cc * CH);
          const int sb = c & 1;
          if (c >= 2 && !mbar_wait(&bars.s_free[sb], ((c >> 1) - 1) & 1, abort_flag, a.status)) { ok = false; break; }
          for (int j = 0; 2 * j < nb; ++j, ++t) {
            const int st = t % NST;
            if (!mbar_wait(&bars.kv_full[st], (t / NST) & 1, abort_flag, a.status)) { ok = false; break; }
            tc_fence_after();
            const uint32_t stage = sRing + st * PL::kStage;
            const uint32_t d = tmem + PL::cS + 128 * sb + 16 * j;
            for (int kk = 0; kk < DQK / 16; ++kk)
              mma_bf16(d, sdesc(stage + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024),
                       sdesc(sQ + qs * PL::kQ + (kk >> 2) * (PL::NH * 128) + (kk & 3) * 32, 16, 1024), idS, kk > 0);
            mma_commit(&bars.kv_empty[st]);
          }
          if (!ok) break;
          if (cc == nch - 1) mma_commit(&bars.q_empty[qs]);
          mma_commit(&bars.s_full[sb]);
          if (pv_c >= 0) issue_pv();
          pv_c = c;
          pv_nb = nb;
          pv_ob = ob;
          pv_first = cc == 0;
          pv_last = cc == nch - 1;
        }
        ++qk;
        ++ok_items;
      }
      if (ok && pv_c >= 0) issue_pv();
    }
  } else if (warp < 6) {
    // ------------------------------------------------------------ softmax
    // Every chunk runs both named barriers in all four warps, also after a wait gave
    // up (the work is skipped, the barriers are not), so no warp is left at one.
    const int sub = warp & 3;
    // TMEM lane 32 sub + lane holds key (32 sub + lane) of a pair: block 2j + par, key
    const int par = sub >> 1, key = 32 * (sub & 1) + lane;
    const uint32_t lane_base = tmem + ((uint32_t)(32 * sub) << 16);
    const int tid = threadIdx.x - 64;
    int c = 0, ok_items = 0;
    bool ok = true;
    for (int k = 0;; ++k) {
      const int slot = k % NIT;
      if (!mbar_wait(&bars.info_full[slot], (k / NIT) & 1, abort_flag, a.status)) break;
      const int n = *info_n(slot);
      if (n < 0) break;
      int tq, g, h0, nh;
      item_of(k, &tq, &g, &h0, &nh);
      const Unit u = qb_unit(a, tq, g);
      const int* xs = info_xs(slot);
      const int ob = ok_items & 1;
      float m[16], l[16];
#pragma unroll
      for (int h = 0; h < 16; ++h) {
        const bool sk = a.sinks && h < nh;
        m[h] = sk ? __ldg(a.sinks + h0 + h) * kLog2eQb : -INFINITY;
        l[h] = sk ? 1.f : 0.f;
      }
      const int nch = (n + CH - 1) / CH;
      for (int cc = 0; cc < nch; ++cc, ++c) {
        const int nb = min(CH, n - cc * CH);
        const int sb = c & 1;
        ok = __all_sync(0xffffffffu, ok && mbar_wait(&bars.s_full[sb], (c >> 1) & 1, abort_flag, a.status));
        tc_fence_after();
        unsigned vis = 0;  // bit j: this thread's key of block 2j + par is visible
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const int b = 2 * j + par;
          if (b < nb) {
            int lo, hi;
            blk_rows(xs[cc * CH + b], u.Lk, u.ta, a.ori_mask, a.wl, a.wr, &lo, &hi);
            if (key >= lo && key <= hi) vis |= 1u << j;
          }
        }
        // pass 1 over the scores (TMEM): the chunk's maximum per head
        float mx[16];
#pragma unroll
        for (int h = 0; h < 16; ++h) mx[h] = -INFINITY;
#pragma unroll 1
        for (int j = 0; ok && j < 8; ++j) {
          if (2 * j >= nb) break;  // uniform over the CTA
          uint32_t v[16];
          tmem_ld16(lane_base + PL::cS + 128 * sb + 16 * j, v);
          tmem_wait_ld();
          reg_dep16(v);
          if ((vis >> j) & 1u) {
#pragma unroll
            for (int h = 0; h < 16; ++h) mx[h] = fmaxf(mx[h], __uint_as_float(v[h]) * a.scale_log2);
          }
        }
#pragma unroll
        for (int h = 0; h < 16; ++h) {
#pragma unroll
          for (int o = 16; o; o >>= 1) mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xffffffffu, mx[h], o));
        }
        if (lane < 16) {
          float mine = mx[0];
#pragma unroll
          for (int h = 1; h < 16; ++h) mine = lane == h ? mx[h] : mine;
          redm[sub * 16 + lane] = mine;
        }
        asm volatile("bar.sync 1, 128;\n" ::: "memory");
        bool grow = false;
        float* f = mx;  // the rescale factors replace the maxima
#pragma unroll
        for (int h = 0; h < 16; ++h) {
          const float cm = fmaxf(fmaxf(redm[h], redm[16 + h]), fmaxf(redm[32 + h], redm[48 + h]));
          const float mn = fmaxf(m[h], cm);
          f[h] = (m[h] == -INFINITY) ? 0.f : exp2f(m[h] - mn);
          grow |= (cc > 0) && (mn > m[h]);
          m[h] = mn;
          l[h] *= f[h];
        }
        // the single P buffer and O^T: the previous chunk's P V has landed
        if (c >= 1) ok = __all_sync(0xffffffffu, ok && mbar_wait(&bars.pv_done, (c - 1) & 1, abort_flag, a.status));
        if (ok && __any_sync(0xffffffffu, grow)) {
          // a later chunk of the item raised a maximum: rescale O^T columns
          tc_fence_after();
          uint32_t w[16];
          tmem_ld16(lane_base + PL::cO + 16 * ob, w);
          tmem_wait_ld();
          reg_dep16(w);
#pragma unroll
          for (int h = 0; h < 16; ++h) w[h] = __float_as_uint(__uint_as_float(w[h]) * f[h]);
          tmem_st16(lane_base + PL::cO + 16 * ob, w);
          tmem_wait_st();
        }
        // pass 2: P = exp2(s - m) to the P^T buffers (row = head, 64 keys per block)
        float sm[16];
#pragma unroll
        for (int h = 0; h < 16; ++h) sm[h] = 0.f;
#pragma unroll 1
        for (int j = 0; ok && j < 8; ++j) {
          if (2 * j >= nb) break;
          uint32_t v[16];
          tmem_ld16(lane_base + PL::cS + 128 * sb + 16 * j, v);
          tmem_wait_ld();
          reg_dep16(v);
          const int b = 2 * j + par;
          if (b < nb) {
            const bool on = (vis >> j) & 1u;
            const uint32_t pb = sP + b * 2048 + (key & 7) * 2;
#pragma unroll
            for (int h = 0; h < 16; ++h) {
              const float pv = on ? ex2_approx(fmaf(__uint_as_float(v[h]), a.scale_log2, -m[h])) : 0.f;
              sm[h] += pv;
              const __nv_bfloat16 pbf = __float2bfloat16_rn(pv);
              const uint16_t bits = *reinterpret_cast<const uint16_t*>(&pbf);
              asm volatile("st.shared.b16 [%0], %1;\n" ::"r"(pb + h * 128 + ((((key >> 3) ^ h) & 7) << 4)),
                           "h"(bits)
                           : "memory");
            }
          }
        }
        tc_fence_before();
        mbar_arrive(&bars.s_free[sb]);
#pragma unroll
        for (int h = 0; h < 16; ++h) {
#pragma unroll
          for (int o = 16; o; o >>= 1) sm[h] += __shfl_xor_sync(0xffffffffu, sm[h], o);
        }
        if (lane < 16) {
          float mine = sm[0];
#pragma unroll
          for (int h = 1; h < 16; ++h) mine = lane == h ? sm[h] : mine;
          redl[sub * 16 + lane] = mine;
        }
        fence_async_smem();
        mbar_arrive(&bars.p_full);
        asm volatile("bar.sync 1, 128;\n" ::: "memory");
#pragma unroll
        for (int h = 0; h < 16; ++h) l[h] += (redl[h] + redl[16 + h]) + (redl[32 + h] + redl[48 + h]);
      }
      // the item's per-head maximum and sum go to the epilogue warps
      if (n > 0) {
        if (tid < 16) {
          float lt = l[0], mt = m[0];
#pragma unroll
          for (int h = 1; h < 16; ++h) {
            lt = tid == h ? l[h] : lt;
            mt = tid == h ? m[h] : mt;
          }
          bars.stat_m[ob][tid] = mt;
          bars.stat_l[ob][tid] = lt;
        }
        mbar_arrive(&bars.stats_full[ob]);
        ++ok_items;
      }
      mbar_arrive(&bars.info_free[slot]);
    }
    tc_fence_before();
  } else {
    // ------------------------------------------------------------ epilogue (warps 6..9)
    // O = O^T / l for this thread's value dim and every head, lse per head; items
    // without blocks get O = 0 and the sink-only lse.  Runs beside the softmax of the
    // next item.
    const int sub = warp & 3;
    const uint32_t lane_base = tmem + ((uint32_t)(32 * sub) << 16);
    const int tid = threadIdx.x - 192;
    // O^T rows: M = 128 puts value dim d in lane d; M = 64 puts it in lane (d % 16) + 32 (d / 16)
    const int dvi = DV >= 128 ? 32 * sub + lane : (lane < 16 ? 16 * sub + lane : -1);
    int ok_items = 0;
    bool ok = true;
    for (int k = 0;; ++k) {
      const int slot = k % NIT;
      if (!mbar_wait(&bars.info_full[slot], (k / NIT) & 1, abort_flag, a.status)) break;
      const int n = *info_n(slot);
      if (n < 0) break;
      int tq, g, h0, nh;
      item_of(k, &tq, &g, &h0, &nh);
      const int ob = ok_items & 1;
      float w[16], mt = -INFINITY, lt = 0.f;
      if (n > 0) {
        ok = __all_sync(0xffffffffu, ok && mbar_wait(&bars.o_full[ob], (ok_items >> 1) & 1, abort_flag, a.status) &&
                                         mbar_wait(&bars.stats_full[ob], (ok_items >> 1) & 1, abort_flag, a.status));
        if (ok) {
          tc_fence_after();
          uint32_t v[16];
          tmem_ld16(lane_base + PL::cO + 16 * ob, v);
          tmem_wait_ld();
          reg_dep16(v);
#pragma unroll
          for (int h = 0; h < 16; ++h) {
            const float lh = bars.stat_l[ob][h];
            w[h] = lh > 0.f ? __uint_as_float(v[h]) / lh : 0.f;
          }
          if (tid < nh) {
            mt = bars.stat_m[ob][tid];
            lt = bars.stat_l[ob][tid];
          }
        }
      } else {
#pragma unroll
        for (int h = 0; h < 16; ++h) w[h] = 0.f;
        if (tid < nh && a.sinks) {
          mt = __ldg(a.sinks + h0 + tid) * kLog2eQb;
          lt = 1.f;
        }
      }
      if (ok) {
        if (dvi >= 0) {
#pragma unroll
          for (int h = 0; h < 16; ++h)
            if (h < nh) a.o[((long long)tq * a.Hq + h0 + h) * DV + dvi] = __float2bfloat16_rn(w[h]);
        }
        if (tid < nh) a.lse[(long long)tq * a.Hq + h0 + tid] = lt > 0.f ? (mt + log2f(lt)) * kLn2Qb : INFINITY;
      }
      if (n > 0) {
        tc_fence_before();
        mbar_arrive(&bars.o_free[ob]);
        ++ok_items;
      }
      mbar_arrive(&bars.info_free[slot]);
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

template <int DQK, int DV>
static cudaError_t bq_launch_t(const QbArgs& a, const void* k, const void* v, cudaStream_t st) {
  using PL = BqPlan<DQK, DV>;
  CUtensorMap mq, mk, mv;
  if (!make_tmap_bf16(&mq, a.q, (uint64_t)a.Tq * a.Hq, DQK, (uint64_t)DQK * 2, PL::NH) ||
      !make_tmap_bf16(&mk, k, (uint64_t)a.Tkv, (uint64_t)a.Hkv * DQK, (uint64_t)a.Hkv * DQK * 2, 64) ||
      !make_tmap_bf16(&mv, v, (uint64_t)a.Tkv, (uint64_t)a.Hkv * DV, (uint64_t)a.Hkv * DV * 2, 64))
    return cudaErrorInvalidValue;
  auto kern = bq_fwd_kernel<DQK, DV>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, PL::kSmem);
  if (e != cudaSuccess) return e;
  const long long items = (long long)a.Tq * a.Hkv * ((a.G + 15) / 16);
  if (items == 0) return cudaSuccess;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const long long grid = items < sms ? items : sms;
  mark_begin(st, kTimeFwd);
  kern<<<(unsigned)grid, 320, PL::kSmem, st>>>(mq, mk, mv, a);
  count_launch();
  mark_end(st, kTimeFwd);
  return cudaGetLastError();
}

cudaError_t launch_bq_fwd(const QbArgs& a, const void* k, const void* v, cudaStream_t st) {
  if (a.dqk == 64 && a.dv == 64) return bq_launch_t<64, 64>(a, k, v, st);
  if (a.dqk == 128 && a.dv == 128) return bq_launch_t<128, 128>(a, k, v, st);
  if (a.dqk == 192 && a.dv == 128) return bq_launch_t<192, 128>(a, k, v, st);
  return cudaErrorInvalidValue;
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

// The forward (dq = false) or the separate dQ pass (dq = true).
cudaError_t launch_qb(const QbArgs& a, const void* k, const void* v, bool dq, cudaStream_t st) {
  if (dq) {
    if (a.dqk == 64 && a.dv == 64) return qb_launch_t<64, 64, true>(a, k, v, st, kTimeBwdDQ);
    if (a.dqk == 128 && a.dv == 128) return qb_launch_t<128, 128, true>(a, k, v, st, kTimeBwdDQ);
    if (a.dqk == 192 && a.dv == 128) return qb_launch_t<192, 128, true>(a, k, v, st, kTimeBwdDQ);
  } else {
    if (a.dqk == 64 && a.dv == 64) return qb_launch_t<64, 64, false>(a, k, v, st, kTimeFwd);
    if (a.dqk == 128 && a.dv == 128) return qb_launch_t<128, 128, false>(a, k, v, st, kTimeFwd);
    if (a.dqk == 192 && a.dv == 128) return qb_launch_t<192, 128, false>(a, k, v, st, kTimeFwd);
  }
  return cudaErrorInvalidValue;
}

}  // namespace sa
