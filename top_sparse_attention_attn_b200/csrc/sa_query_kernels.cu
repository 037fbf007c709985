// sa_query_kernels.cu -- query-stationary kernels: forward, fused backward
// (dQ in-CTA, dK/dV scatter-add), rowsum(dO o O), fp32 -> bf16 finalize,
// index check and the resolve inspection kernel.
//
// Work decomposition: one CTA (4 warps) per (query token, kv-head, 16-head
// slice of the G heads sharing that kv-head).  The unit's visible KV rows come
// in 64-row tiles (sa_device.cuh), gathered row by row with cp.async into
// XOR-swizzled shared memory, double-buffered.  Warp w owns tile rows
// [16w, 16w + 16) for the score block S = Q K^T and d-column slice w of the
// O / dQ accumulators; softmax statistics are exchanged through shared memory.
//
// Math (bf16 operands, fp32 accumulation, mma.sync m16n8k16):
//   forward   -- aclnnNsaSelectedAttentionInfer "Formula", online softmax with
//                the sink logit as an extra denominator term;
//   backward  -- SparseFlashMlaGrad "Computation formula" Stages 2-3 /
//                aclnnSparseFlashAttentionGrad "Formula" Phases 1-3.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "sa_device.cuh"
#include "sa_launch.h"

namespace sa {

cudaEvent_t g_ev_begin = nullptr, g_ev_end = nullptr;
int g_ev_which = -1;
long long g_launches = 0;

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

// ---------------------------------------------------------------------------
// shared-memory plan
// ---------------------------------------------------------------------------
template <int DQK, int DV, bool SHARED>
struct Plan {
  static constexpr int DVS = SHARED ? DQK : DV;        // row length of the V tile
  static constexpr int kK = kTileRows * DQK * 2;
  static constexpr int kV = SHARED ? 0 : kTileRows * DV * 2;
  static constexpr int kBuf = kK + kV;
  static constexpr int oBuf = 0;                        // 2 buffers
  static constexpr int oQ = 2 * kBuf;
  static constexpr int oDO = oQ + 16 * DQK * 2;
  static constexpr int oP = oDO + 16 * DV * 2;          // bf16 [16][64]
  static constexpr int oDS = oP + 16 * 64 * 2;          // bf16 [16][64]
  static constexpr int oRow = oDS + 16 * 64 * 2;        // int [3][64]
  static constexpr int oRed = oRow + 3 * 64 * 4;        // float [2][4][16]
  static constexpr int kBytes = oRed + 2 * 4 * 16 * 4;
  static_assert(DQK % 64 == 0 && DV % 64 == 0, "head dims must be multiples of 64");
  static_assert(kBytes <= 227 * 1024, "shared memory plan too large");
};

template <int DQK, int DV, bool SHARED>
__device__ __forceinline__ void issue_tile(const Prob& p, int g, const int* rc, uint32_t sK,
                                           uint32_t sV, int tid) {
  constexpr int KCH = DQK / 8;
  for (int i = tid; i < kTileRows * KCH; i += 128) {
    int r = i / KCH, c = i - r * KCH;
    int code = rc[r];
    const bf16* src = code >= 0 ? row_k_ptr(p, code, g) + c * 8 : p.q;
    cp_async16(swz<DQK>(sK, r, c), src, code >= 0);
  }
  if (!SHARED) {
    constexpr int VCH = DV / 8;
    for (int i = tid; i < kTileRows * VCH; i += 128) {
      int r = i / VCH, c = i - r * VCH;
      int code = rc[r];
      const bf16* src = code >= 0 ? row_v_ptr(p, code, g) + c * 8 : p.q;
      cp_async16(swz<DV>(sV, r, c), src, code >= 0);
    }
  }
}

// Load 16 rows (heads h0.., rows >= nh zero) of a [token, H, D] tensor into a swizzled tile.
template <int D>
__device__ __forceinline__ void load_rows16(const bf16* base, int nh, uint32_t dst, int tid) {
  constexpr int CH = D / 8;
  for (int i = tid; i < 16 * CH; i += 128) {
    int r = i / CH, c = i - r * CH;
    const bf16* src = base + (long long)min(r, nh - 1) * D + c * 8;
    cp_async16(swz<D>(dst, r, c), src, r < nh);
  }
}

// ---------------------------------------------------------------------------
// forward
// ---------------------------------------------------------------------------
template <int DQK, int DV, bool SHARED, bool F16>
__global__ void __launch_bounds__(128) fwd_kernel(const Prob p, bf16* __restrict__ O,
                                                  float* __restrict__ LSE) {
  using PL = Plan<DQK, DV, SHARED>;
  constexpr int DVS = PL::DVS;
  constexpr int NT = DV / 32;  // 8-col n-tiles per warp slice
  extern __shared__ __align__(1024) uint8_t smem[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int n_hsl = (p.G + 15) >> 4;
  const int unit = blockIdx.x / n_hsl, hsl = blockIdx.x - unit * n_hsl;
  const int tq = unit / p.Hkv, g = unit - tq * p.Hkv;
  const Unit u = make_unit(p, tq, g);
  const int h0 = g * p.G + hsl * 16;
  const int nh = min(16, p.G - hsl * 16);

  const uint32_t sbuf = smem_u32(smem + PL::oBuf);
  const uint32_t sQ = smem_u32(smem + PL::oQ);
  const uint32_t sP = smem_u32(smem + PL::oP);
  int* rowc = reinterpret_cast<int*>(smem + PL::oRow);
  float* smax = reinterpret_cast<float*>(smem + PL::oRed);
  float* ssum = smax + 64;

  load_rows16<DQK>(p.q + ((long long)tq * p.Hq + h0) * DQK, nh, sQ, tid);
  cp_async_commit();
  if (tid < 64 && u.n_tiles > 0) rowc[tid] = resolve_row(p, u, 0, tid);
  __syncthreads();
  if (u.n_tiles > 0) {
    issue_tile<DQK, DV, SHARED>(p, g, rowc, sbuf, sbuf + PL::kK, tid);
    cp_async_commit();
  }

  const int r0 = lane >> 2;  // rows r0 and r0 + 8
  float m[2], l[2];
  for (int r = 0; r < 2; ++r) {
    int row = r0 + 8 * r;
    if (p.sinks && row < nh) {
      m[r] = __ldg(p.sinks + h0 + row) * kLog2e;
      l[r] = 1.f;
    } else {
      m[r] = -INFINITY;
      l[r] = 0.f;
    }
  }
  float o[NT][4];
#pragma unroll
  for (int i = 0; i < NT; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;

  for (int it = 0; it < u.n_tiles; ++it) {
    const int cur = it % 3;
    const uint32_t bK = sbuf + (it & 1) * PL::kBuf;
    const uint32_t bV = SHARED ? bK : bK + PL::kK;
    if (tid < 64 && it + 1 < u.n_tiles) rowc[((it + 1) % 3) * 64 + tid] = resolve_row(p, u, it + 1, tid);
    cp_async_wait_all();
    __syncthreads();
    if (it + 1 < u.n_tiles) {
      const uint32_t nK = sbuf + ((it + 1) & 1) * PL::kBuf;
      issue_tile<DQK, DV, SHARED>(p, g, rowc + ((it + 1) % 3) * 64, nK, nK + PL::kK, tid);
      cp_async_commit();
    }
    // S_w = Q K_w^T over the warp's 16 tile rows
    float s[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll 4
    for (int kc = 0; kc < DQK / 8; kc += 2) {
      uint32_t a[4], b[4];
      load_a<DQK>(a, sQ, 0, kc, lane);
      load_b_nk<DQK>(b, bK, warp * 16, kc, lane);
      Elt<F16>::mma(s[0], a, b[0], b[1]);
      Elt<F16>::mma(s[1], a, b[2], b[3]);
    }
    const int* rc = rowc + cur * 64 + warp * 16;
    float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        int col = nt * 8 + 2 * (lane & 3) + (j & 1);
        float v = rc[col] >= 0 ? s[nt][j] * p.scale_log2 : -INFINITY;
        s[nt][j] = v;
        mx[j >> 1] = fmaxf(mx[j >> 1], v);
      }
    mx[0] = warp_max4(mx[0]);
    mx[1] = warp_max4(mx[1]);
    if ((lane & 3) == 0) {
      smax[warp * 16 + r0] = mx[0];
      smax[warp * 16 + r0 + 8] = mx[1];
    }
    __syncthreads();
    float mnew[2], muse[2], alpha[2], ps[2];
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      int row = r0 + 8 * r;
      float t = fmaxf(fmaxf(smax[row], smax[16 + row]), fmaxf(smax[32 + row], smax[48 + row]));
      mnew[r] = fmaxf(m[r], t);
      muse[r] = mnew[r] == -INFINITY ? 0.f : mnew[r];
      alpha[r] = exp2f(m[r] - muse[r]);
      ps[r] = 0.f;
    }
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
      float p0 = exp2f(s[nt][0] - muse[0]), p1 = exp2f(s[nt][1] - muse[0]);
      float p2 = exp2f(s[nt][2] - muse[1]), p3 = exp2f(s[nt][3] - muse[1]);
      ps[0] += p0 + p1;
      ps[1] += p2 + p3;
      const int chunk = warp * 2 + nt;
      uint32_t a0 = swz<64>(sP, r0, chunk) + (lane & 3) * 4;
      uint32_t a1 = swz<64>(sP, r0 + 8, chunk) + (lane & 3) * 4;
      asm volatile("st.shared.b32 [%0], %1;\n" ::"r"(a0), "r"(Elt<F16>::pack(p0, p1)));
      asm volatile("st.shared.b32 [%0], %1;\n" ::"r"(a1), "r"(Elt<F16>::pack(p2, p3)));
    }
    ps[0] = warp_sum4(ps[0]);
    ps[1] = warp_sum4(ps[1]);
    if ((lane & 3) == 0) {
      ssum[warp * 16 + r0] = ps[0];
      ssum[warp * 16 + r0 + 8] = ps[1];
    }
    __syncthreads();
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      int row = r0 + 8 * r;
      l[r] = l[r] * alpha[r] + (ssum[row] + ssum[16 + row] + ssum[32 + row] + ssum[48 + row]);
      m[r] = mnew[r];
    }
#pragma unroll
    for (int i = 0; i < NT; ++i) {
      o[i][0] *= alpha[0];
      o[i][1] *= alpha[0];
      o[i][2] *= alpha[1];
      o[i][3] *= alpha[1];
    }
    // O_w += P (16 x 64) V[:, slice w]
#pragma unroll
    for (int kc = 0; kc < 8; kc += 2) {
      uint32_t a[4];
      load_a<64>(a, sP, 0, kc, lane);
#pragma unroll
      for (int j = 0; j < NT / 2; ++j) {
        uint32_t b[4];
        load_b_kn<DVS>(b, bV, kc * 8, warp * (NT) + 2 * j, lane);
        Elt<F16>::mma(o[2 * j], a, b[0], b[1]);
        Elt<F16>::mma(o[2 * j + 1], a, b[2], b[3]);
      }
    }
  }
  cp_async_wait_all();

  // epilogue: O = o / l, lse = (m + log2 l) ln 2
  float inv[2];
#pragma unroll
  for (int r = 0; r < 2; ++r) inv[r] = l[r] > 0.f ? 1.f / l[r] : 0.f;
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    int row = r0 + 8 * r;
    if (row >= nh) continue;
    bf16* orow = O + ((long long)tq * p.Hq + h0 + row) * DV + warp * (DV / 4);
#pragma unroll
    for (int i = 0; i < NT; ++i) {
      int col = i * 8 + 2 * (lane & 3);
      *reinterpret_cast<uint32_t*>(orow + col) = Elt<F16>::pack(o[i][2 * r] * inv[r], o[i][2 * r + 1] * inv[r]);
    }
    if (warp == 0 && (lane & 3) == 0)
      LSE[(long long)tq * p.Hq + h0 + row] = l[r] > 0.f ? (m[r] + log2f(l[r])) * kLn2 : INFINITY;
  }
}

// ---------------------------------------------------------------------------
// SoftmaxL1Norm outputs (SparseFlashMlaGrad "Parameter Description":
// oriSoftmaxL1NormOptional / cmpSoftmaxL1NormOptional, the target distribution of
// aclnnSparseLightningIndexerGradKLLoss "Formula": attention probabilities summed
// over the heads, L1-normalised along the context).  The backward's P = exp(S -
// lse) is recomputed tile by tile as in the forward, summed over the CTA's heads
// for every tile row, and added to the row's slot of the unit's output (fp32
// atomics: the 16-head slices of a unit share its output row).  l1_norm_kernel
// then divides every output row by its sum.
// ---------------------------------------------------------------------------
template <int DQK>
__device__ __forceinline__ void issue_k_tile(const Prob& p, int g, const int* rc, uint32_t sK, int tid) {
  constexpr int KCH = DQK / 8;
  for (int i = tid; i < kTileRows * KCH; i += 128) {
    int r = i / KCH, c = i - r * KCH;
    int code = rc[r];
    const bf16* src = code >= 0 ? row_k_ptr(p, code, g) + c * 8 : p.q;
    cp_async16(swz<DQK>(sK, r, c), src, code >= 0);
  }
}

template <int DQK, int DV, bool SHARED, bool F16>
__global__ void __launch_bounds__(128) l1_sum_kernel(const Prob p, const float* __restrict__ LSE,
                                                     float* __restrict__ ori_out, float* __restrict__ cmp_out) {
  using PL = Plan<DQK, DV, SHARED>;
  extern __shared__ __align__(1024) uint8_t smem[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int n_hsl = (p.G + 15) >> 4;
  const int unit = blockIdx.x / n_hsl, hsl = blockIdx.x - unit * n_hsl;
  const int tq = unit / p.Hkv, g = unit - tq * p.Hkv;
  const Unit u = make_unit(p, tq, g);
  const int h0 = g * p.G + hsl * 16;
  const int nh = min(16, p.G - hsl * 16);
  const long long ug = (long long)tq * p.Hkv + g;
  const uint32_t sbuf = smem_u32(smem + PL::oBuf);
  const uint32_t sQ = smem_u32(smem + PL::oQ);
  int* rowc = reinterpret_cast<int*>(smem + PL::oRow);

  load_rows16<DQK>(p.q + ((long long)tq * p.Hq + h0) * DQK, nh, sQ, tid);
  cp_async_commit();
  if (tid < 64 && u.n_tiles > 0) rowc[tid] = resolve_row(p, u, 0, tid);
  __syncthreads();
  if (u.n_tiles > 0) {
    issue_k_tile<DQK>(p, g, rowc, sbuf, tid);
    cp_async_commit();
  }
  // this thread's score rows r0 and r0 + 8 are heads h0 + r0, h0 + r0 + 8
  const int r0 = lane >> 2;
  float lse2[2];
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    const int row = r0 + 8 * r;
    lse2[r] = row < nh ? __ldg(LSE + (long long)tq * p.Hq + h0 + row) * kLog2e : INFINITY;  // P = 0 past nh
  }
  for (int it = 0; it < u.n_tiles; ++it) {
    const int cur = it % 3;
    const uint32_t bK = sbuf + (it & 1) * PL::kBuf;
    if (tid < 64 && it + 1 < u.n_tiles) rowc[((it + 1) % 3) * 64 + tid] = resolve_row(p, u, it + 1, tid);
    cp_async_wait_all();
    __syncthreads();
    if (it + 1 < u.n_tiles) {
      issue_k_tile<DQK>(p, g, rowc + ((it + 1) % 3) * 64, sbuf + ((it + 1) & 1) * PL::kBuf, tid);
      cp_async_commit();
    }
    // S_w = Q K_w^T over the warp's 16 tile rows (columns of s)
    float s[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll 4
    for (int kc = 0; kc < DQK / 8; kc += 2) {
      uint32_t a[4], b[4];
      load_a<DQK>(a, sQ, 0, kc, lane);
      load_b_nk<DQK>(b, bK, warp * 16, kc, lane);
      Elt<F16>::mma(s[0], a, b[0], b[1]);
      Elt<F16>::mma(s[1], a, b[2], b[3]);
    }
    const int* rc = rowc + cur * 64 + warp * 16;
    // P summed over this thread's two heads, then over the 8 row groups of the warp
    float cs[2][2];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int col = nt * 8 + 2 * (lane & 3) + e;
        float v = 0.f;
        if (rc[col] >= 0) v = exp2f(fmaf(s[nt][e], p.scale_log2, -lse2[0])) + exp2f(fmaf(s[nt][2 + e], p.scale_log2, -lse2[1]));
        v += __shfl_xor_sync(0xffffffffu, v, 4);
        v += __shfl_xor_sync(0xffffffffu, v, 8);
        v += __shfl_xor_sync(0xffffffffu, v, 16);
        cs[nt][e] = v;
      }
    if (lane < 4) {
      if (it < u.n_ori_tiles) {
        if (ori_out && u.ori_mode == kOriToken) {
#pragma unroll
          for (int nt = 0; nt < 2; ++nt)
#pragma unroll
            for (int e = 0; e < 2; ++e) {
              const int col = nt * 8 + 2 * lane + e;
              if (rc[col] >= 0) atomicAdd(ori_out + ug * p.topk + it * kTileRows + warp * 16 + col, cs[nt][e]);
            }
        } else if (ori_out && u.ori_mode == kOriBlock) {
          // every row of the tile belongs to one slot
          const float t = (cs[0][0] + cs[0][1]) + (cs[1][0] + cs[1][1]);
          if (t != 0.f) atomicAdd(ori_out + ug * p.topk + it / u.tps, t);
        }
      } else if (cmp_out) {
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int col = nt * 8 + 2 * lane + e;
            if (rc[col] >= 0)
              atomicAdd(cmp_out + ug * p.cmp_topk + (it - u.n_ori_tiles) * kTileRows + warp * 16 + col, cs[nt][e]);
          }
      }
    }
  }
  cp_async_wait_all();
}

// Each of `rows` rows of `width` floats divided by its sum (left at zero when 0);
// one warp per row.
__global__ void __launch_bounds__(256) l1_norm_kernel(float* __restrict__ out, long long rows, int width) {
  const long long row = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  float* r = out + row * width;
  float sum = 0.f;
  for (int i = lane; i < width; i += 32) sum += r[i];
#pragma unroll
  for (int o = 16; o; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
  const float inv = sum > 0.f ? 1.f / sum : 0.f;
  for (int i = lane; i < width; i += 32) r[i] *= inv;
}

// ---------------------------------------------------------------------------
// fused backward: dQ accumulated in the CTA, dK / dV (dKV) scattered with
// fp32 vector atomics, dSinks partial sums
// ---------------------------------------------------------------------------
__device__ __forceinline__ void red_add2(float* addr, float a, float b) {
  atomicAdd(reinterpret_cast<float2*>(addr), make_float2(a, b));
}

template <int DQK, int DV, bool SHARED, bool SCATTER, bool F16>
__global__ void __launch_bounds__(128) bwd_kernel(const Prob p, const bf16* __restrict__ dO,
                                                  const float* __restrict__ LSE,
                                                  const float* __restrict__ Delta, BwdOut out) {
  using PL = Plan<DQK, DV, SHARED>;
  constexpr int DVS = PL::DVS;
  constexpr int NQ = DQK / 32;  // 8-col n-tiles of the warp's dQ slice
  extern __shared__ __align__(1024) uint8_t smem[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int n_hsl = (p.G + 15) >> 4;
  const int unit = blockIdx.x / n_hsl, hsl = blockIdx.x - unit * n_hsl;
  const int tq = unit / p.Hkv, g = unit - tq * p.Hkv;
  const Unit u = make_unit(p, tq, g);
  const int h0 = g * p.G + hsl * 16;
  const int nh = min(16, p.G - hsl * 16);

  const uint32_t sbuf = smem_u32(smem + PL::oBuf);
  const uint32_t sQ = smem_u32(smem + PL::oQ);
  const uint32_t sDO = smem_u32(smem + PL::oDO);
  const uint32_t sP = smem_u32(smem + PL::oP);
  const uint32_t sDS = smem_u32(smem + PL::oDS);
  int* rowc = reinterpret_cast<int*>(smem + PL::oRow);
  float* sred = reinterpret_cast<float*>(smem + PL::oRed);

  load_rows16<DQK>(p.q + ((long long)tq * p.Hq + h0) * DQK, nh, sQ, tid);
  load_rows16<DV>(dO + ((long long)tq * p.Hq + h0) * DV, nh, sDO, tid);
  cp_async_commit();
  if (tid < 64 && u.n_tiles > 0) rowc[tid] = resolve_row(p, u, 0, tid);
  __syncthreads();
  if (u.n_tiles > 0) {
    issue_tile<DQK, DV, SHARED>(p, g, rowc, sbuf, sbuf + PL::kK, tid);
    cp_async_commit();
  }

  const int r0 = lane >> 2;
  float lse2[2], dlt[2], psd[2] = {0.f, 0.f};
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    int row = r0 + 8 * r;
    if (row < nh) {
      long long idx = (long long)tq * p.Hq + h0 + row;
      lse2[r] = __ldg(LSE + idx) * kLog2e;
      dlt[r] = __ldg(Delta + idx);
    } else {
      lse2[r] = INFINITY;
      dlt[r] = 0.f;
    }
  }
  float dq[NQ][4];
#pragma unroll
  for (int i = 0; i < NQ; ++i) dq[i][0] = dq[i][1] = dq[i][2] = dq[i][3] = 0.f;

  for (int it = 0; it < u.n_tiles; ++it) {
    const int cur = it % 3;
    const uint32_t bK = sbuf + (it & 1) * PL::kBuf;
    const uint32_t bV = SHARED ? bK : bK + PL::kK;
    if (tid < 64 && it + 1 < u.n_tiles) rowc[((it + 1) % 3) * 64 + tid] = resolve_row(p, u, it + 1, tid);
    cp_async_wait_all();
    __syncthreads();
    if (it + 1 < u.n_tiles) {
      const uint32_t nK = sbuf + ((it + 1) & 1) * PL::kBuf;
      issue_tile<DQK, DV, SHARED>(p, g, rowc + ((it + 1) % 3) * 64, nK, nK + PL::kK, tid);
      cp_async_commit();
    }
    const int* rc = rowc + cur * 64 + warp * 16;
    // S_w and dP_w (16 heads x the warp's 16 tile rows)
    float s[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
    float dp[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll 4
    for (int kc = 0; kc < DQK / 8; kc += 2) {
      uint32_t a[4], b[4];
      load_a<DQK>(a, sQ, 0, kc, lane);
      load_b_nk<DQK>(b, bK, warp * 16, kc, lane);
      Elt<F16>::mma(s[0], a, b[0], b[1]);
      Elt<F16>::mma(s[1], a, b[2], b[3]);
    }
#pragma unroll 4
    for (int kc = 0; kc < DV / 8; kc += 2) {
      uint32_t a[4], b[4];
      load_a<DV>(a, sDO, 0, kc, lane);
      load_b_nk<DVS>(b, bV, warp * 16, kc, lane);
      Elt<F16>::mma(dp[0], a, b[0], b[1]);
      Elt<F16>::mma(dp[1], a, b[2], b[3]);
    }
    // P = exp(S - lse), dS = P (dP - Delta)
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
      float pv[4], dsv[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        int col = nt * 8 + 2 * (lane & 3) + (j & 1);
        int r = j >> 1;
        float pj = rc[col] >= 0 ? exp2f(s[nt][j] * p.scale_log2 - lse2[r]) : 0.f;
        pv[j] = pj;
        dsv[j] = pj * (dp[nt][j] - dlt[r]);
        psd[r] += pj * dp[nt][j];
      }
      const int chunk = warp * 2 + nt;
      uint32_t a0 = (lane & 3) * 4;
      asm volatile("st.shared.b32 [%0], %1;\n" ::"r"(swz<64>(sP, r0, chunk) + a0), "r"(Elt<F16>::pack(pv[0], pv[1])));
      asm volatile("st.shared.b32 [%0], %1;\n" ::"r"(swz<64>(sP, r0 + 8, chunk) + a0), "r"(Elt<F16>::pack(pv[2], pv[3])));
      asm volatile("st.shared.b32 [%0], %1;\n" ::"r"(swz<64>(sDS, r0, chunk) + a0), "r"(Elt<F16>::pack(dsv[0], dsv[1])));
      asm volatile("st.shared.b32 [%0], %1;\n" ::"r"(swz<64>(sDS, r0 + 8, chunk) + a0), "r"(Elt<F16>::pack(dsv[2], dsv[3])));
    }
    __syncwarp();
    // scatter: dK rows (the warp's 16 tile rows) = scale dS^T Q  [+ P^T dO on the V columns]
    const int code0 = rc[r0], code1 = rc[r0 + 8];
    float* kdst0 = nullptr;
    float* kdst1 = nullptr;
    if (code0 >= 0)
      kdst0 = (code0 & kCmpFlag) ? out.dcmp_acc + ((long long)(code0 & ~kCmpFlag) * p.Hkv + g) * DQK
                                 : out.dk_acc + ((long long)code0 * p.Hkv + g) * DQK;
    if (code1 >= 0)
      kdst1 = (code1 & kCmpFlag) ? out.dcmp_acc + ((long long)(code1 & ~kCmpFlag) * p.Hkv + g) * DQK
                                 : out.dk_acc + ((long long)code1 * p.Hkv + g) * DQK;
    if (SCATTER && __any_sync(0xffffffffu, code0 >= 0 || code1 >= 0)) {
      uint32_t adsT[4], apT[4];
      load_a_t<64>(adsT, sDS, 0, warp * 2, lane);
      load_a_t<64>(apT, sP, 0, warp * 2, lane);
#pragma unroll 1
      for (int nc0 = 0; nc0 < DQK / 8; nc0 += 8) {
        float acc[8][4];
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          uint32_t b[4];
          load_b_kn<DQK>(b, sQ, 0, nc0 + 2 * j, lane);
          Elt<F16>::mma(acc[2 * j], adsT, b[0], b[1]);
          Elt<F16>::mma(acc[2 * j + 1], adsT, b[2], b[3]);
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          acc[i][0] *= p.scale;
          acc[i][1] *= p.scale;
          acc[i][2] *= p.scale;
          acc[i][3] *= p.scale;
        }
        if (SHARED && nc0 * 8 < DV) {
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            uint32_t b[4];
            load_b_kn<DV>(b, sDO, 0, nc0 + 2 * j, lane);
            Elt<F16>::mma(acc[2 * j], apT, b[0], b[1]);
            Elt<F16>::mma(acc[2 * j + 1], apT, b[2], b[3]);
          }
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          int col = nc0 * 8 + i * 8 + 2 * (lane & 3);
          if (kdst0) red_add2(kdst0 + col, acc[i][0], acc[i][1]);
          if (kdst1) red_add2(kdst1 + col, acc[i][2], acc[i][3]);
        }
      }
      if (!SHARED) {
        float* vdst0 = code0 >= 0 ? out.dv_acc + ((long long)code0 * p.Hkv + g) * DV : nullptr;
        float* vdst1 = code1 >= 0 ? out.dv_acc + ((long long)code1 * p.Hkv + g) * DV : nullptr;
#pragma unroll 1
        for (int nc0 = 0; nc0 < DV / 8; nc0 += 8) {
          float acc[8][4];
#pragma unroll
          for (int i = 0; i < 8; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            uint32_t b[4];
            load_b_kn<DV>(b, sDO, 0, nc0 + 2 * j, lane);
            Elt<F16>::mma(acc[2 * j], apT, b[0], b[1]);
            Elt<F16>::mma(acc[2 * j + 1], apT, b[2], b[3]);
          }
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            int col = nc0 * 8 + i * 8 + 2 * (lane & 3);
            if (vdst0) red_add2(vdst0 + col, acc[i][0], acc[i][1]);
            if (vdst1) red_add2(vdst1 + col, acc[i][2], acc[i][3]);
          }
        }
      }
    }
    __syncthreads();  // every warp's dS columns are in shared memory
    // dQ_w += dS (16 x 64) K[:, slice w]
#pragma unroll
    for (int kc = 0; kc < 8; kc += 2) {
      uint32_t a[4];
      load_a<64>(a, sDS, 0, kc, lane);
#pragma unroll
      for (int j = 0; j < NQ / 2; ++j) {
        uint32_t b[4];
        load_b_kn<DQK>(b, bK, kc * 8, warp * NQ + 2 * j, lane);
        Elt<F16>::mma(dq[2 * j], a, b[0], b[1]);
        Elt<F16>::mma(dq[2 * j + 1], a, b[2], b[3]);
      }
    }
  }
  cp_async_wait_all();

  // dQ epilogue
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    int row = r0 + 8 * r;
    if (row >= nh) continue;
    bf16* qrow = out.dq + ((long long)tq * p.Hq + h0 + row) * DQK + warp * (DQK / 4);
#pragma unroll
    for (int i = 0; i < NQ; ++i) {
      int col = i * 8 + 2 * (lane & 3);
      *reinterpret_cast<uint32_t*>(qrow + col) =
          Elt<F16>::pack(dq[i][2 * r] * p.scale, dq[i][2 * r + 1] * p.scale);
    }
  }
  // dSinks: -P_sink * sum_j P_j dP_j summed over this CTA's rows
  if (p.sinks) {
    psd[0] = warp_sum4(psd[0]);
    psd[1] = warp_sum4(psd[1]);
    __syncthreads();
    if ((lane & 3) == 0) {
      sred[warp * 16 + r0] = psd[0];
      sred[warp * 16 + r0 + 8] = psd[1];
    }
    __syncthreads();
    if (tid < nh) {
      float tot = sred[tid] + sred[16 + tid] + sred[32 + tid] + sred[48 + tid];
      long long idx = (long long)tq * p.Hq + h0 + tid;
      float l2 = __ldg(LSE + idx) * kLog2e;
      float psink = exp2f(__ldg(p.sinks + h0 + tid) * kLog2e - l2);
      atomicAdd(out.dsinks + h0 + tid, -psink * tot);
    }
  }
}

// ---------------------------------------------------------------------------
// rowsum(dO o O), finalize, checks, inspection
// ---------------------------------------------------------------------------
template <bool F16>
__global__ void __launch_bounds__(256) delta_kernel(const bf16* __restrict__ O, const bf16* __restrict__ dO,
                                                    float* __restrict__ delta, long long rows, int dv) {
  pdl_wait();
  pdl_trigger();
  long long row = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
  int lane = threadIdx.x & 31;
  if (row >= rows) return;
  const float acc = warp_row_dot_bf16<F16>(O + row * dv, dO + row * dv, dv, lane);
  if (lane == 0) delta[row] = acc;
}

// fp32 -> the output element type (bf16, or fp16 with F16), eight at a time.
template <bool F16>
__global__ void __launch_bounds__(256) to_bf16_kernel(const float* __restrict__ src, bf16* __restrict__ dst,
                                                      long long n8) {
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n8;
       i += (long long)gridDim.x * blockDim.x) {
    float4 a = __ldg(reinterpret_cast<const float4*>(src) + 2 * i);
    float4 b = __ldg(reinterpret_cast<const float4*>(src) + 2 * i + 1);
    uint4 r;
    r.x = Elt<F16>::pack(a.x, a.y);
    r.y = Elt<F16>::pack(a.z, a.w);
    r.z = Elt<F16>::pack(b.x, b.y);
    r.w = Elt<F16>::pack(b.z, b.w);
    reinterpret_cast<uint4*>(dst)[i] = r;
  }
}

struct CvtJobs {
  Cvt job[4];
  long long end8[4];  // cumulative 8-element group counts
  int n;
};

template <bool F16>
__global__ void __launch_bounds__(256) to_bf16_multi_kernel(const CvtJobs J) {
  pdl_wait();
  pdl_trigger();
  const long long total = J.end8[J.n - 1];
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < total;
       i += (long long)gridDim.x * blockDim.x) {
    int k = 0;
    while (i >= J.end8[k]) ++k;
    const long long li = i - (k ? J.end8[k - 1] : 0);
    const float4* src = reinterpret_cast<const float4*>(J.job[k].src);
    float4 a = __ldg(src + 2 * li), b = __ldg(src + 2 * li + 1);
    uint4 r;
    r.x = Elt<F16>::pack(a.x, a.y);
    r.y = Elt<F16>::pack(a.z, a.w);
    r.z = Elt<F16>::pack(b.x, b.y);
    r.w = Elt<F16>::pack(b.z, b.w);
    reinterpret_cast<uint4*>(J.job[k].dst)[li] = r;
  }
}

__global__ void check_kernel(const Prob p) {
  long long ug = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (ug >= (long long)p.Tq * p.Hkv) return;
  int tq = (int)(ug / p.Hkv), g = (int)(ug - (long long)tq * p.Hkv);
  Unit u = make_unit(p, tq, g);
  bool bad = false;
  for (int s = 0; s < u.n_ori_slots; ++s) {
    int x = __ldg(p.ori_idx + ug * p.topk + s);
    if (x >= 0 && (long long)x * p.bs >= u.Lk) bad = true;
  }
  for (int s = 0; s < u.n_cmp_slots; ++s) {
    int c = __ldg(p.cmp_idx + ug * p.cmp_topk + s);
    if (c >= u.Lc) bad = true;
  }
  if (bad) atomicOr(p.status, kStatusIndexRange);
}

__global__ void debug_resolve_kernel(const Prob p, int* rows, int* counts, int max_rows) {
  long long ug = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (ug >= (long long)p.Tq * p.Hkv) return;
  int tq = (int)(ug / p.Hkv), g = (int)(ug - (long long)tq * p.Hkv);
  Unit u = make_unit(p, tq, g);
  int n = 0;
  for (int tile = 0; tile < u.n_tiles; ++tile) {
    for (int r = 0; r < kTileRows; ++r) {
      int code = resolve_row(p, u, tile, r);
      if (code < 0) continue;
      int local = (code & kCmpFlag) ? (kCmpFlag | ((code & ~kCmpFlag) - u.cmp0)) : code - u.kv0;
      if (n < max_rows) rows[ug * max_rows + n] = local;
      ++n;
    }
  }
  counts[ug] = n;
}

// ---------------------------------------------------------------------------
// launchers
// ---------------------------------------------------------------------------
#define SA_FOR_EACH_SHAPE(X) \
  X(64, 64, false)           \
  X(128, 128, false)         \
  X(192, 128, false)         \
  X(128, 128, true)          \
  X(576, 512, true)

bool kernels_built(int dqk, int dv, bool shared) {
#define X(A, B, C) \
  if (dqk == A && dv == B && shared == C) return true;
  SA_FOR_EACH_SHAPE(X)
#undef X
  return false;
}

template <int DQK, int DV, bool SHARED, bool F16>
static cudaError_t fwd_t(const Prob& p, bf16* o, float* lse, cudaStream_t st) {
  using PL = Plan<DQK, DV, SHARED>;
  auto k = fwd_kernel<DQK, DV, SHARED, F16>;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, PL::kBytes);
  if (e != cudaSuccess) return e;
  long long grid = (long long)p.Tq * p.Hkv * ((p.G + 15) / 16);
  mark_begin(st, kTimeFwd);
  k<<<(unsigned)grid, 128, PL::kBytes, st>>>(p, o, lse);
  count_launch();
  mark_end(st, kTimeFwd);
  return cudaGetLastError();
}

template <int DQK, int DV, bool SHARED, bool SCATTER, bool F16>
static cudaError_t bwd_t(const Prob& p, const bf16* d_o, const float* lse, const float* delta,
                         const BwdOut& out, cudaStream_t st) {
  using PL = Plan<DQK, DV, SHARED>;
  auto k = bwd_kernel<DQK, DV, SHARED, SCATTER, F16>;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, PL::kBytes);
  if (e != cudaSuccess) return e;
  long long grid = (long long)p.Tq * p.Hkv * ((p.G + 15) / 16);
  const int which = SCATTER ? kTimeBwdKV : kTimeBwdDQ;
  mark_begin(st, which);
  k<<<(unsigned)grid, 128, PL::kBytes, st>>>(p, d_o, lse, delta, out);
  count_launch();
  mark_end(st, which);
  return cudaGetLastError();
}

template <int DQK, int DV, bool SHARED, bool F16>
static cudaError_t l1_t(const Prob& p, const float* lse, float* ori_out, float* cmp_out, cudaStream_t st) {
  using PL = Plan<DQK, DV, SHARED>;
  auto k = l1_sum_kernel<DQK, DV, SHARED, F16>;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, PL::kBytes);
  if (e != cudaSuccess) return e;
  const long long units = (long long)p.Tq * p.Hkv;
  if (ori_out && cudaMemsetAsync(ori_out, 0, (size_t)units * p.topk * sizeof(float), st) != cudaSuccess)
    return cudaGetLastError();
  if (cmp_out && cudaMemsetAsync(cmp_out, 0, (size_t)units * p.cmp_topk * sizeof(float), st) != cudaSuccess)
    return cudaGetLastError();
  const long long grid = units * ((p.G + 15) / 16);
  k<<<(unsigned)grid, 128, PL::kBytes, st>>>(p, lse, ori_out, cmp_out);
  count_launch();
  const unsigned ng = (unsigned)((units + 7) / 8);
  if (ori_out) {
    l1_norm_kernel<<<ng, 256, 0, st>>>(ori_out, units, p.topk);
    count_launch();
  }
  if (cmp_out) {
    l1_norm_kernel<<<ng, 256, 0, st>>>(cmp_out, units, p.cmp_topk);
    count_launch();
  }
  return cudaGetLastError();
}

cudaError_t launch_softmax_l1norm(const Prob& p, const float* lse, float* ori_out, float* cmp_out, cudaStream_t st) {
#define X(A, B, C)                                                                                          \
  if (p.dqk == A && p.dv == B && (bool)p.shared == C)                                                       \
    return p.f16 ? l1_t<A, B, C, true>(p, lse, ori_out, cmp_out, st) : l1_t<A, B, C, false>(p, lse, ori_out, cmp_out, st);
  SA_FOR_EACH_SHAPE(X)
#undef X
  return cudaErrorInvalidValue;
}

cudaError_t launch_fwd(const Prob& p, bf16* o, float* lse, cudaStream_t st) {
#define X(A, B, C)                              \
  if (p.dqk == A && p.dv == B && (bool)p.shared == C) \
    return p.f16 ? fwd_t<A, B, C, true>(p, o, lse, st) : fwd_t<A, B, C, false>(p, o, lse, st);
  SA_FOR_EACH_SHAPE(X)
#undef X
  return cudaErrorInvalidValue;
}

cudaError_t launch_bwd(const Prob& p, const bf16* o, const bf16* d_o, const float* lse,
                       const float* delta, const BwdOut& out, cudaStream_t st) {
  (void)o;
#define X(A, B, C)                                                         \
  if (p.dqk == A && p.dv == B && (bool)p.shared == C)                          \
    return p.f16 ? bwd_t<A, B, C, true, true>(p, d_o, lse, delta, out, st)     \
                 : bwd_t<A, B, C, true, false>(p, d_o, lse, delta, out, st);
  SA_FOR_EACH_SHAPE(X)
#undef X
  return cudaErrorInvalidValue;
}

cudaError_t launch_bwd_dq(const Prob& p, const bf16* d_o, const float* lse, const float* delta,
                          const BwdOut& out, cudaStream_t st) {
  // dQ only (dK / dV come from the key-stationary kernel); dSinks needs no sinks here
  if (p.dqk == 64 && p.dv == 64 && !p.shared) return bwd_t<64, 64, false, false, false>(p, d_o, lse, delta, out, st);
  if (p.dqk == 128 && p.dv == 128 && !p.shared)
    return bwd_t<128, 128, false, false, false>(p, d_o, lse, delta, out, st);
  if (p.dqk == 192 && p.dv == 128 && !p.shared)
    return bwd_t<192, 128, false, false, false>(p, d_o, lse, delta, out, st);
  return cudaErrorInvalidValue;
}

cudaError_t launch_delta(const bf16* o, const bf16* d_o, float* delta, long long rows, int dv,
                         cudaStream_t st, bool f16) {
  if (rows == 0) return cudaSuccess;
  cudaError_t e = f16 ? launch_pdl(delta_kernel<true>, (unsigned)((rows + 7) / 8), 256, 0, st, o, d_o, delta, rows, dv)
                      : launch_pdl(delta_kernel<false>, (unsigned)((rows + 7) / 8), 256, 0, st, o, d_o, delta, rows, dv);
  count_launch();
  return e;
}

cudaError_t launch_to_bf16(const float* src, bf16* dst, long long n, cudaStream_t st, bool f16) {
  if (n == 0) return cudaSuccess;
  long long n8 = n / 8;  // every caller's n is a multiple of 64
  long long blocks = (n8 + 255) / 256;
  if (blocks > 148 * 16) blocks = 148 * 16;
  if (f16)
    to_bf16_kernel<true><<<(unsigned)blocks, 256, 0, st>>>(src, dst, n8);
  else
    to_bf16_kernel<false><<<(unsigned)blocks, 256, 0, st>>>(src, dst, n8);
  count_launch();
  return cudaGetLastError();
}

cudaError_t launch_to_bf16_multi(const Cvt* jobs, int njobs, cudaStream_t st, bool f16) {
  CvtJobs J;
  J.n = 0;
  long long acc = 0;
  for (int k = 0; k < njobs && k < 4; ++k) {
    if (jobs[k].n <= 0) continue;
    J.job[J.n] = jobs[k];
    acc += jobs[k].n / 8;
    J.end8[J.n] = acc;
    ++J.n;
  }
  if (J.n == 0) return cudaSuccess;
  long long blocks = (acc + 255) / 256;
  if (blocks > 148 * 16) blocks = 148 * 16;
  cudaError_t e = f16 ? launch_pdl(to_bf16_multi_kernel<true>, (unsigned)blocks, 256, 0, st, J)
                      : launch_pdl(to_bf16_multi_kernel<false>, (unsigned)blocks, 256, 0, st, J);
  count_launch();
  return e;
}

cudaError_t launch_check(const Prob& p, cudaStream_t st) {
  long long n = (long long)p.Tq * p.Hkv;
  if (n == 0) return cudaSuccess;
  check_kernel<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(p);
  count_launch();
  return cudaGetLastError();
}

cudaError_t launch_debug_resolve(const Prob& p, int* rows, int* counts, int max_rows, cudaStream_t st) {
  long long n = (long long)p.Tq * p.Hkv;
  if (n == 0) return cudaSuccess;
  debug_resolve_kernel<<<(unsigned)((n + 127) / 128), 128, 0, st>>>(p, rows, counts, max_rows);
  count_launch();
  return cudaGetLastError();
}

}  // namespace sa
