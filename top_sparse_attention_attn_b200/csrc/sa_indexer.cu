// sa_indexer.cu -- the lightning indexer's KL-loss backward
// (aclnnSparseLightningIndexerGradKLLoss, "Formula"):
//   I[t, j]  = sum_h W[t, h] ReLU(q[t, h] . K[j])   over token t's used slots j
//   L        = sum_t KL(p[t, :] || Softmax(I[t, :]))
//   dI       = Softmax(I) - p
//   dW[t, h] = sum_j ReLU(S[t, h, j]) dI[t, j]
//   dS       = W[t, h] (S > 0) dI[t, j],  dq[t] = dS K,  dK[j] += dS^T q[t]
// A slot is used when its index is >= 0, before the row's topk length, inside the
// sequence and not in the token's future (the page's K[:t, :]).
//
// One CTA (4 warps) per query token, two passes over the token's slots in tiles of
// 64 (key rows gathered with cp.async into swizzled shared memory, mma.sync tiles):
//   pass 1: S = q K^T (warp w: keys 16w..16w+15, every head), I per key by a head
//           reduction in registers and warp shuffles, into shared memory;
//   softmax over the used slots -> dI (in place) and the token's loss;
//   pass 2: S again, dS (bf16) to shared memory, then dq += dS K (warp w: dims
//           w D/4 .. (w + 1) D/4, in registers) and dK_tile = dS^T q (warp w: keys
//           16w..) added to an fp32 accumulator with vector atomics; dW per head in
//           registers, summed over the warps at the end.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "sa_device.cuh"
#include "sa_launch.h"

namespace sa {

template <int H, int D>
struct IxPlan {
  static constexpr int oQ = 0;                      // q [H][D] bf16
  static constexpr int oK = oQ + H * D * 2;         // two key tiles [64][D] bf16
  static constexpr int oDS = oK + 2 * 64 * D * 2;   // dS [H][64] bf16
  static constexpr int oDW = oDS + H * 64 * 2;      // [4 warps][H] fp32
  static constexpr int oRow = oDW + 4 * H * 4;      // key row codes [2][64]
  static constexpr int oRed = oRow + 2 * 64 * 4;    // [2][4] reduction scratch
  static constexpr int oI = oRed + 64;              // I / dI per slot (topk padded to 64)
  static int bytes(int topk_pad) { return oI + topk_pad * 4; }
};

// Key row code of slot s of token tq (global row of k), or -1 when the slot is unused.
__device__ __forceinline__ int ix_code(const IxArgs& a, long long tq, int s, int n, int ta, int Lk, int kv0) {
  if (s >= n) return -1;
  const int x = __ldg(a.idx + tq * a.topk + s);
  if (x < 0) return -1;
  if (x >= Lk) {
    if (a.status) atomicOr(a.status, kStatusIndexRange);
    return -1;
  }
  return x <= ta ? kv0 + x : -1;
}

template <int D>
__device__ __forceinline__ void ix_gather(const IxArgs& a, const int* rc, uint32_t sK, int tid) {
  constexpr int CH = D / 8;
  for (int i = tid; i < 64 * CH; i += 128) {
    const int r = i / CH, c = i - r * CH;
    const int code = rc[r];
    const bf16* src = code >= 0 ? a.k + (long long)code * D + c * 8 : a.k;
    cp_async16(swz<D>(sK, r, c), src, code >= 0);
  }
}

template <int H, int D>
__global__ void __launch_bounds__(128) ix_kl_kernel(const IxArgs a) {
  using PL = IxPlan<H, D>;
  constexpr int MT = H / 16;   // head m-tiles
  constexpr int NQ = D / 32;   // dq n-tiles (8 dims) per warp
  constexpr int NK = D / 8;    // dK n-tiles (8 dims)
  extern __shared__ __align__(1024) uint8_t smem[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const long long tq = blockIdx.x;
  // sequence geometry of the token
  int b, t, Lq, Lk, kv0;
  if (a.layout == kLayoutBSND) {
    b = (int)(tq / a.s_q);
    t = (int)(tq - (long long)b * a.s_q);
    Lq = a.s_q;
    Lk = a.s_kv;
    kv0 = b * a.s_kv;
  } else {
    b = find_batch(a.cu_q, a.B, (int)tq);
    const int q0 = __ldg(a.cu_q + b);
    Lq = max(__ldg(a.cu_q + b + 1) - q0, 0);
    t = (int)tq - q0;
    kv0 = min(max(__ldg(a.cu_kv + b), 0), a.Tkv);
    Lk = min(max(__ldg(a.cu_kv + b + 1), kv0), a.Tkv) - kv0;
  }
  const int ta = t + Lk - Lq;
  int n = a.topk;
  if (a.topk_len) n = min(n, max(0, __ldg(a.topk_len + tq)));
  const int ntiles = (a.topk + 63) / 64;
  const uint32_t sQ = smem_u32(smem + PL::oQ), sK = smem_u32(smem + PL::oK), sDS = smem_u32(smem + PL::oDS);
  float* sDW = reinterpret_cast<float*>(smem + PL::oDW);
  int* rowc = reinterpret_cast<int*>(smem + PL::oRow);
  float* red = reinterpret_cast<float*>(smem + PL::oRed);
  float* sI = reinterpret_cast<float*>(smem + PL::oI);

  // q of the token, and W of this thread's heads (rows r0 and r0 + 8 of each m-tile)
  {
    constexpr int CH = D / 8;
    for (int i = tid; i < H * CH; i += 128) {
      const int r = i / CH, c = i - r * CH;
      cp_async16(swz<D>(sQ, r, c), a.q + (tq * H + r) * D + c * 8, true);
    }
    cp_async_commit();
  }
  const int r0 = lane >> 2;
  float wv[MT][2];
#pragma unroll
  for (int mt = 0; mt < MT; ++mt)
#pragma unroll
    for (int r = 0; r < 2; ++r) wv[mt][r] = __ldg(a.w + tq * H + 16 * mt + r0 + 8 * r);

  // S = q K_tile^T for the warp's 16 keys: s[mt][nt][j], head 16 mt + r0 (+8 for j >= 2),
  // key 16 warp + 8 nt + 2 (lane & 3) + (j & 1)
  auto scores = [&](uint32_t bK, float (&s)[MT][2][4]) {
#pragma unroll
    for (int mt = 0; mt < MT; ++mt)
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) s[mt][nt][0] = s[mt][nt][1] = s[mt][nt][2] = s[mt][nt][3] = 0.f;
#pragma unroll
    for (int kc = 0; kc < D / 8; kc += 2) {
      uint32_t bb[4];
      load_b_nk<D>(bb, bK, warp * 16, kc, lane);
#pragma unroll
      for (int mt = 0; mt < MT; ++mt) {
        uint32_t aa[4];
        load_a<D>(aa, sQ, 16 * mt, kc, lane);
        mma16816(s[mt][0], aa, bb[0], bb[1]);
        mma16816(s[mt][1], aa, bb[2], bb[3]);
      }
    }
  };
  auto load_tile = [&](int it) {
    if (tid < 64) rowc[(it & 1) * 64 + tid] = ix_code(a, tq, it * 64 + tid, n, ta, Lk, kv0);
    __syncthreads();
    ix_gather<D>(a, rowc + (it & 1) * 64, sK + (it & 1) * (64 * D * 2), tid);
    cp_async_commit();
  };

  // ---------------- pass 1: I per slot
  if (ntiles > 0) load_tile(0);
  for (int it = 0; it < ntiles; ++it) {
    cp_async_wait_all();
    __syncthreads();
    if (it + 1 < ntiles) load_tile(it + 1);
    float s[MT][2][4];
    scores(sK + (it & 1) * (64 * D * 2), s);
    const int* rc = rowc + (it & 1) * 64;
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        float v = 0.f;
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) v += wv[mt][0] * fmaxf(s[mt][nt][e], 0.f) + wv[mt][1] * fmaxf(s[mt][nt][2 + e], 0.f);
        v += __shfl_xor_sync(0xffffffffu, v, 4);
        v += __shfl_xor_sync(0xffffffffu, v, 8);
        v += __shfl_xor_sync(0xffffffffu, v, 16);
        if (lane < 4) {
          const int key = warp * 16 + nt * 8 + 2 * lane + e;
          sI[it * 64 + key] = rc[key] >= 0 ? v : -INFINITY;
        }
      }
  }
  cp_async_wait_all();
  __syncthreads();

  // ---------------- softmax over the used slots: dI in place, the token's loss
  const int npad = ntiles * 64;
  float mx = -INFINITY;
  for (int s2 = tid; s2 < npad; s2 += 128) mx = fmaxf(mx, sI[s2]);
#pragma unroll
  for (int o = 16; o; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  if (lane == 0) red[warp] = mx;
  __syncthreads();
  mx = fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3]));
  float z = 0.f;
  if (mx > -INFINITY)
    for (int s2 = tid; s2 < npad; s2 += 128) z += __expf(sI[s2] - mx);
#pragma unroll
  for (int o = 16; o; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
  __syncthreads();
  if (lane == 0) red[4 + warp] = z;
  __syncthreads();
  z = (red[4] + red[5]) + (red[6] + red[7]);
  const float lz = mx + logf(z);  // log of the softmax denominator
  float loss = 0.f;
  for (int s2 = tid; s2 < npad; s2 += 128) {
    const float iv = sI[s2];
    float di = 0.f;
    if (iv > -INFINITY) {
      const float pt = __ldg(a.p + tq * a.topk + s2);
      di = __expf(iv - lz) - pt;
      if (pt > 0.f) loss += pt * (logf(pt) - (iv - lz));
    }
    sI[s2] = di;
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) loss += __shfl_xor_sync(0xffffffffu, loss, o);
  __syncthreads();
  if (lane == 0) red[warp] = loss;
  __syncthreads();
  if (tid == 0 && a.loss) a.loss[tq] = (red[0] + red[1]) + (red[2] + red[3]);

  // ---------------- pass 2: dS, dq, dK, dW
  float dq[MT][NQ][4];
#pragma unroll
  for (int mt = 0; mt < MT; ++mt)
#pragma unroll
    for (int j = 0; j < NQ; ++j) dq[mt][j][0] = dq[mt][j][1] = dq[mt][j][2] = dq[mt][j][3] = 0.f;
  float dw[MT][2];
#pragma unroll
  for (int mt = 0; mt < MT; ++mt) dw[mt][0] = dw[mt][1] = 0.f;
  if (ntiles > 0) load_tile(0);
  for (int it = 0; it < ntiles; ++it) {
    cp_async_wait_all();
    __syncthreads();
    if (it + 1 < ntiles) load_tile(it + 1);
    const uint32_t bK = sK + (it & 1) * (64 * D * 2);
    float s[MT][2][4];
    scores(bK, s);
    // dS = W (S > 0) dI to shared memory; dW += ReLU(S) dI
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
      const int key0 = warp * 16 + nt * 8 + 2 * (lane & 3);
      const float di0 = sI[it * 64 + key0], di1 = sI[it * 64 + key0 + 1];
#pragma unroll
      for (int mt = 0; mt < MT; ++mt)
#pragma unroll
        for (int r = 0; r < 2; ++r) {
          const float x0 = s[mt][nt][2 * r], x1 = s[mt][nt][2 * r + 1];
          dw[mt][r] += fmaxf(x0, 0.f) * di0 + fmaxf(x1, 0.f) * di1;
          const float d0 = x0 > 0.f ? wv[mt][r] * di0 : 0.f, d1 = x1 > 0.f ? wv[mt][r] * di1 : 0.f;
          const uint32_t addr = swz<64>(sDS, 16 * mt + r0 + 8 * r, warp * 2 + nt) + (lane & 3) * 4;
          asm volatile("st.shared.b32 [%0], %1;\n" ::"r"(addr), "r"(pack_bf16(d0, d1)) : "memory");
        }
    }
    __syncthreads();
    // dq[:, warp's dims] += dS K
#pragma unroll
    for (int kc = 0; kc < 8; kc += 2) {
#pragma unroll
      for (int mt = 0; mt < MT; ++mt) {
        uint32_t aa[4];
        load_a<64>(aa, sDS, 16 * mt, kc, lane);
#pragma unroll
        for (int j = 0; j < NQ / 2; ++j) {
          uint32_t bb[4];
          load_b_kn<D>(bb, bK, kc * 8, warp * (D / 32) + 2 * j, lane);
          mma16816(dq[mt][2 * j], aa, bb[0], bb[1]);
          mma16816(dq[mt][2 * j + 1], aa, bb[2], bb[3]);
        }
      }
    }
    // dK of the warp's 16 keys = dS^T q, added to the fp32 accumulator
    {
      float dk[NK][4];
#pragma unroll
      for (int j = 0; j < NK; ++j) dk[j][0] = dk[j][1] = dk[j][2] = dk[j][3] = 0.f;
#pragma unroll
      for (int kh = 0; kh < MT; ++kh) {
        uint32_t aa[4];
        load_a_t<64>(aa, sDS, 16 * kh, warp * 2, lane);
#pragma unroll
        for (int j = 0; j < NK / 2; ++j) {
          uint32_t bb[4];
          load_b_kn<D>(bb, sQ, 16 * kh, 2 * j, lane);
          mma16816(dk[2 * j], aa, bb[0], bb[1]);
          mma16816(dk[2 * j + 1], aa, bb[2], bb[3]);
        }
      }
      const int* rc = rowc + (it & 1) * 64;
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        const int code = rc[warp * 16 + r0 + 8 * r];
        if (code < 0) continue;
        float* row = a.dk_acc + (long long)code * D;
#pragma unroll
        for (int j = 0; j < NK; ++j) {
          const int col = j * 8 + 2 * (lane & 3);
          asm volatile("red.global.add.v2.f32 [%0], {%1, %2};\n" ::"l"(row + col), "f"(dk[j][2 * r]), "f"(dk[j][2 * r + 1])
                       : "memory");
        }
      }
    }
    __syncthreads();  // the dS buffer and this key tile are reused next
  }
  cp_async_wait_all();

  // dq (bf16; the token's own rows, no atomics)
#pragma unroll
  for (int mt = 0; mt < MT; ++mt)
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      const int h = 16 * mt + r0 + 8 * r;
      bf16* row = a.dq + (tq * H + h) * D + warp * (D / 4);
#pragma unroll
      for (int j = 0; j < NQ; ++j) {
        const int col = j * 8 + 2 * (lane & 3);
        *reinterpret_cast<uint32_t*>(row + col) = pack_bf16(dq[mt][j][2 * r], dq[mt][j][2 * r + 1]);
      }
    }
  // dW: over this thread's keys (lanes sharing r0), then over the warps
#pragma unroll
  for (int mt = 0; mt < MT; ++mt)
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      float v = dw[mt][r];
      v += __shfl_xor_sync(0xffffffffu, v, 1);
      v += __shfl_xor_sync(0xffffffffu, v, 2);
      if ((lane & 3) == 0) sDW[warp * H + 16 * mt + r0 + 8 * r] = v;
    }
  __syncthreads();
  if (tid < H) a.dw[tq * H + tid] = (sDW[tid] + sDW[H + tid]) + (sDW[2 * H + tid] + sDW[3 * H + tid]);
}

bool ix_built(int H, int D) { return (H == 16 || H == 32 || H == 64) && (D == 64 || D == 128); }

template <int H, int D>
static cudaError_t ix_t(const IxArgs& a, cudaStream_t st) {
  auto k = ix_kl_kernel<H, D>;
  const int topk_pad = (a.topk + 63) / 64 * 64;
  const int smem = IxPlan<H, D>::bytes(topk_pad);
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  k<<<(unsigned)a.Tq, 128, smem, st>>>(a);
  count_launch();
  return cudaGetLastError();
}

cudaError_t launch_indexer_kl(const IxArgs& a, cudaStream_t st) {
  if (a.Tq == 0) return cudaSuccess;
#define X(HH, DD) \
  if (a.H == HH && a.D == DD) return ix_t<HH, DD>(a, st);
  X(16, 64) X(32, 64) X(64, 64) X(16, 128) X(32, 128) X(64, 128)
#undef X
  return cudaErrorInvalidValue;
}

}  // namespace sa
