// sa_selftest.cu -- sa_selftest_mma: one CTA computes D = A * B through the
// same TMA loads, shared-memory matrix descriptors, tcgen05.mma and TMEM loads
// that the key-stationary backward kernel is built from, so that each operand
// orientation (K-major, MN-major) and each accumulator height (M = 64, 128)
// can be checked against a plain matmul.
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/sparse_attn.h"
#include "sa_launch.h"
#include "sa_tc.cuh"

namespace sa {

struct SelftestArgs {
  int M, N, K, a_mn, b_mn, box_rows, d_lane;
};

__global__ void __launch_bounds__(128) selftest_mma_kernel(const __grid_constant__ CUtensorMap mapA,
                                                           const __grid_constant__ CUtensorMap mapB,
                                                           const SelftestArgs a, float* __restrict__ D,
                                                           int* status) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // 1024-byte aligned operand area
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  __shared__ uint64_t bar_load, bar_mma;
  __shared__ uint32_t tmem_base;
  __shared__ int abort_flag;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t sA = smem_u32(smem);
  const uint32_t sB = sA + a.M * a.K * 2;
  const uint32_t ncols = a.N <= 64 ? 64 : (a.N <= 128 ? 128 : 256);

  if (threadIdx.x == 0) {
    abort_flag = 0;
    mbar_init(&bar_load, 1);
    mbar_init(&bar_mma, 1);
    mbar_fence_init();
  }
  if (warp == 0) tmem_alloc(&tmem_base, ncols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  if (threadIdx.x == 0) {
    // operand tiles: K-major -> slabs over K of [rows][64]; MN-major -> slabs over M/N of [K][64]
    mbar_arrive_tx(&bar_load, (uint32_t)((a.M + a.N) * a.K * 2));
    const int br = a.box_rows;
    if (!a.a_mn) {
      for (int s = 0; s < a.K / 64; ++s)
        for (int r = 0; r < a.M; r += br) tma_load_2d(sA + s * a.M * 128 + r * 128, &mapA, 64 * s, r, &bar_load);
    } else {
      for (int s = 0; s < a.M / 64; ++s)
        for (int r = 0; r < a.K; r += br) tma_load_2d(sA + s * a.K * 128 + r * 128, &mapA, 64 * s, r, &bar_load);
    }
    if (!a.b_mn) {
      for (int s = 0; s < a.K / 64; ++s)
        for (int r = 0; r < a.N; r += br) tma_load_2d(sB + s * a.N * 128 + r * 128, &mapB, 64 * s, r, &bar_load);
    } else {
      for (int s = 0; s < a.N / 64; ++s)
        for (int r = 0; r < a.K; r += br) tma_load_2d(sB + s * a.K * 128 + r * 128, &mapB, 64 * s, r, &bar_load);
    }
    if (mbar_wait(&bar_load, 0, &abort_flag, status)) {
      tc_fence_after();
      const uint32_t idesc = idesc_bf16(a.M, a.N, a.a_mn != 0, a.b_mn != 0);
      for (int kk = 0; kk < a.K / 16; ++kk) {
        uint64_t da = a.a_mn ? sdesc(sA + kk * 2048, a.K * 128, 1024)
                             : sdesc(sA + (kk >> 2) * a.M * 128 + (kk & 3) * 32, 16, 1024);
        uint64_t db = a.b_mn ? sdesc(sB + kk * 2048, a.K * 128, 1024)
                             : sdesc(sB + (kk >> 2) * a.N * 128 + (kk & 3) * 32, 16, 1024);
        mma_bf16(tmem_base + ((uint32_t)a.d_lane << 16), da, db, idesc, kk > 0 ? 1u : 0u);
      }
      mma_commit(&bar_mma);
    }
  }
  __syncwarp();
  bool ok = mbar_wait(&bar_mma, 0, &abort_flag, status);
  tc_fence_after();
  if (ok) {
    const int sub = warp & 3;
    int m = -1;
    if (a.M == 128) m = 32 * sub + lane;
    else if (lane >= a.d_lane && lane < a.d_lane + 16) m = 16 * sub + (lane - a.d_lane);
    for (int c = 0; c < a.N; c += 16) {
      uint32_t r[16];
      tmem_ld16(tmem_base + ((uint32_t)(32 * sub) << 16) + c, r);
      tmem_wait_ld();
      reg_dep16(r);
      if (m >= 0)
        for (int i = 0; i < 16; ++i) D[(long long)m * a.N + c + i] = __uint_as_float(r[i]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem_base, ncols);
    tmem_relinquish();
  }
}

// Operand layouts written in software: a matrix X[R][C] (R rows, C contiguous)
// in atoms of W = sw / 2 elements along C, rows of sw bytes, the 16-byte piece
// index XOR (r & 7) for the 128-byte swizzle or ((r >> 1) & 3) for the 64-byte one.
__device__ __forceinline__ uint32_t sw_offset(int r, int c, int R, int sw) {
  const int W = sw / 2;
  const int a = c / W, w = c - a * W;
  const int piece = (w * 2) >> 4, sub = (w * 2) & 15;
  const int x = sw == 128 ? (r & 7) : ((r >> 1) & 3);
  return (uint32_t)(a * (R * sw) + r * sw + ((piece ^ x) << 4) + sub);
}

struct Selftest2Args {
  int M, N, K, a_mn, b_mn, a_sw, b_sw, d_lane;
};

// D = A B with both operands copied into shared memory in software (any of the
// K-major / MN-major orientations, 128- or 64-byte swizzle), one CTA of 128.
__global__ void __launch_bounds__(128) selftest_mma2_kernel(const bf16* __restrict__ A, const bf16* __restrict__ B,
                                                            const Selftest2Args a, float* __restrict__ D,
                                                            int* status) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  __shared__ uint64_t bar_mma;
  __shared__ uint32_t tmem_base;
  __shared__ int abort_flag;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // A: K-major [M][K] (rows M) or MN-major [K][M] (rows K); B: K-major [N][K] or MN-major [K][N]
  const int aR = a.a_mn ? a.K : a.M, aC = a.a_mn ? a.M : a.K;
  const int bR = a.b_mn ? a.K : a.N, bC = a.b_mn ? a.N : a.K;
  const int aBytes = aR * aC * 2;
  uint8_t* sA = smem;
  uint8_t* sB = smem + ((aBytes + 1023) & ~1023);
  for (int i = threadIdx.x; i < aR * aC; i += blockDim.x) {
    const int r = i / aC, c = i - r * aC;
    *reinterpret_cast<bf16*>(sA + sw_offset(r, c, aR, a.a_sw)) = A[i];
  }
  for (int i = threadIdx.x; i < bR * bC; i += blockDim.x) {
    const int r = i / bC, c = i - r * bC;
    *reinterpret_cast<bf16*>(sB + sw_offset(r, c, bR, a.b_sw)) = B[i];
  }
  if (threadIdx.x == 0) {
    abort_flag = 0;
    mbar_init(&bar_mma, 1);
    mbar_fence_init();
  }
  const uint32_t ncols = a.N <= 32 ? 32 : (a.N <= 64 ? 64 : (a.N <= 128 ? 128 : 256));
  if (warp == 0) tmem_alloc(&tmem_base, ncols);
  fence_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t uA = smem_u32(sA), uB = smem_u32(sB);
  auto desc = [](uint32_t base, bool mn, int R, int sw, int kk) -> uint64_t {
    const int W = sw / 2;
    if (!mn) {  // K-major: a K step of 16 moves 32 bytes inside an atom
      const uint32_t addr = base + ((kk * 16) / W) * (R * sw) + ((kk * 16) % W) * 2;
      return sw == 128 ? sdesc(addr, 16, 1024) : sdesc64(addr, 16, 512);
    }
    // MN-major: a K step of 16 rows; atoms of W elements along M / N, R * sw bytes apart
    const uint32_t addr = base + kk * 16 * sw;
    return sw == 128 ? sdesc(addr, R * sw, 1024) : sdesc64(addr, R * sw, 512);
  };
  if (threadIdx.x == 0) {
    const uint32_t idesc = idesc_bf16(a.M, a.N, a.a_mn != 0, a.b_mn != 0);
    for (int kk = 0; kk < a.K / 16; ++kk)
      mma_bf16(tmem_base + ((uint32_t)a.d_lane << 16), desc(uA, a.a_mn != 0, aR, a.a_sw, kk),
               desc(uB, a.b_mn != 0, bR, a.b_sw, kk), idesc, kk > 0 ? 1u : 0u);
    mma_commit(&bar_mma);
  }
  __syncwarp();
  const bool ok = mbar_wait(&bar_mma, 0, &abort_flag, status);
  tc_fence_after();
  if (ok) {
    const int sub = warp & 3;
    int m = -1;
    if (a.M == 128) m = 32 * sub + lane;
    else if (lane >= a.d_lane && lane < a.d_lane + 16) m = 16 * sub + (lane - a.d_lane);
    for (int c = 0; c < a.N; c += 16) {
      uint32_t r[16];
      tmem_ld16(tmem_base + ((uint32_t)(32 * sub) << 16) + c, r);
      tmem_wait_ld();
      reg_dep16(r);
      if (m >= 0)
        for (int i = 0; i < 16; ++i) D[(long long)m * a.N + c + i] = __uint_as_float(r[i]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem_base, ncols);
    tmem_relinquish();
  }
}

// TMA row gather: n rows (n a multiple of 4, <= 32) of a [rows][cols] bf16 matrix
// (cols a multiple of 64, <= 576) named by row_idx land by tile::gather4 loads in
// shared memory as slabs of n rows x 128 bytes (128-byte swizzle), exactly where
// the token-level kernels read them; the CTA then writes them back un-swizzled
// to out [n][cols].
__global__ void __launch_bounds__(128) selftest_gather4_kernel(const __grid_constant__ CUtensorMap map,
                                                               const int* __restrict__ row_idx, int n, int cols,
                                                               bf16* __restrict__ out, int* status) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  const uint32_t base = smem_u32(smem);
  const int nslab = cols / 64;
  if (threadIdx.x == 0) {
    abort_flag = 0;
    mbar_init(&bar, 1);
    mbar_fence_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    mbar_arrive_tx(&bar, (uint32_t)(n * cols * 2));
    for (int q = 0; q < n / 4; ++q)
      for (int s = 0; s < nslab; ++s)
        tma_gather4(base + s * (n * 128) + q * 4 * 128, &map, 64 * s, __ldg(row_idx + 4 * q),
                    __ldg(row_idx + 4 * q + 1), __ldg(row_idx + 4 * q + 2), __ldg(row_idx + 4 * q + 3), &bar);
  }
  const bool ok = mbar_wait(&bar, 0, &abort_flag, status);
  if (!ok) {
    if (threadIdx.x == 0) mbar_wait_drain(&bar, 0);
    return;
  }
  for (int i = threadIdx.x; i < n * cols / 8; i += blockDim.x) {
    const int r = i / (cols / 8), c = i - r * (cols / 8);  // 16-byte piece c of row r
    const uint32_t a = base + (c >> 3) * (n * 128) + r * 128 + (((c & 7) ^ (r & 7)) << 4);
    uint4 v;
    asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];\n" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a));
    reinterpret_cast<uint4*>(out + (long long)r * cols)[c] = v;
  }
}

// Nothing ever arrives on `bar`: the bounded wait gives up and raises the status word.
__global__ void selftest_wait_kernel(int* status, int* waited) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    abort_flag = 0;
    mbar_init(&bar, 1);
    mbar_fence_init();
  }
  __syncthreads();
  const bool ok = mbar_wait(&bar, 0, &abort_flag, status);
  if (threadIdx.x == 0) *waited = ok ? 1 : 0;
}

}  // namespace sa

extern "C" sa_status sa_selftest_mma2(int32_t M, int32_t N, int32_t K, int32_t a_mn, int32_t b_mn, int32_t a_sw,
                                      int32_t b_sw, int32_t d_lane, const void* A, const void* B, float* D,
                                      int32_t* status, void* stream) {
  if (!A || !B || !D || !status) return SA_ERR_NULLPTR;
  if ((M != 64 && M != 128) || N < 16 || N > 256 || N % 16 || K < 16 || K > 256 || K % 16) return SA_ERR_PARAM;
  if ((a_sw != 64 && a_sw != 128) || (b_sw != 64 && b_sw != 128)) return SA_ERR_PARAM;
  if (d_lane != 0 && !(d_lane == 16 && M == 64)) return SA_ERR_PARAM;
  // every operand extent along its contiguous dimension must fill whole atoms
  const int aC = a_mn ? M : K, bC = b_mn ? N : K;
  if (aC % (a_sw / 2) || bC % (b_sw / 2)) return SA_ERR_PARAM;
  sa::Selftest2Args args{M, N, K, a_mn, b_mn, a_sw, b_sw, d_lane};
  const int smem = ((M * K * 2 + 1023) & ~1023) + N * K * 2 + 1024;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaFuncSetAttribute(sa::selftest_mma2_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
      cudaSuccess)
    return SA_ERR_CUDA;
  sa::selftest_mma2_kernel<<<1, 128, smem, st>>>(static_cast<const sa::bf16*>(A), static_cast<const sa::bf16*>(B), args,
                                                 D, status);
  sa::count_launch();
  return cudaGetLastError() == cudaSuccess ? SA_OK : SA_ERR_CUDA;
}

extern "C" sa_status sa_selftest_gather4(const void* src, int32_t rows, int32_t cols, const int32_t* row_idx,
                                         int32_t n, void* out, int32_t* status, void* stream) {
  if (!src || !row_idx || !out || !status) return SA_ERR_NULLPTR;
  if (rows < 1 || cols < 64 || cols > 576 || cols % 64 || n < 4 || n > 32 || n % 4) return SA_ERR_PARAM;
  CUtensorMap map;
  if (!sa::make_tmap_bf16(&map, src, (uint64_t)rows, (uint64_t)cols, (uint64_t)cols * 2, 1)) return SA_ERR_PARAM;
  const int smem = n * cols * 2 + 1024;
  if (cudaFuncSetAttribute(sa::selftest_gather4_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
      cudaSuccess)
    return SA_ERR_CUDA;
  sa::selftest_gather4_kernel<<<1, 128, smem, static_cast<cudaStream_t>(stream)>>>(
      map, row_idx, n, cols, static_cast<sa::bf16*>(out), status);
  sa::count_launch();
  return cudaGetLastError() == cudaSuccess ? SA_OK : SA_ERR_CUDA;
}

extern "C" sa_status sa_selftest_wait_timeout(int32_t* status, int32_t* waited, void* stream) {
  if (!status || !waited) return SA_ERR_NULLPTR;
  sa::selftest_wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(status, waited);
  sa::count_launch();
  return cudaGetLastError() == cudaSuccess ? SA_OK : SA_ERR_CUDA;
}

extern "C" sa_status sa_selftest_mma(int32_t M, int32_t N, int32_t K, int32_t a_mn, int32_t b_mn,
                                     int32_t box_rows, int32_t d_lane, const void* A, const void* B, float* D,
                                     int32_t* status, void* stream) {
  if (!A || !B || !D || !status) return SA_ERR_NULLPTR;
  if (d_lane != 0 && !(d_lane == 16 && M == 64)) return SA_ERR_PARAM;
  if ((M != 64 && M != 128) || N < 64 || N > 256 || N % 64 || K < 64 || K > 256 || K % 64) return SA_ERR_PARAM;
  if (box_rows != 8 && box_rows != 16 && box_rows != 32 && box_rows != 64) return SA_ERR_PARAM;
  CUtensorMap ma, mb;
  // A: K-major [M][K] or MN-major [K][M]; B: K-major [N][K] or MN-major [K][N]
  bool okA = a_mn ? sa::make_tmap_bf16(&ma, A, K, M, (uint64_t)M * 2, box_rows)
                  : sa::make_tmap_bf16(&ma, A, M, K, (uint64_t)K * 2, box_rows);
  bool okB = b_mn ? sa::make_tmap_bf16(&mb, B, K, N, (uint64_t)N * 2, box_rows)
                  : sa::make_tmap_bf16(&mb, B, N, K, (uint64_t)K * 2, box_rows);
  if (!okA || !okB) return SA_ERR_PARAM;
  sa::SelftestArgs args{M, N, K, a_mn, b_mn, box_rows, d_lane};
  const int smem = (M + N) * K * 2 + 1024;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaFuncSetAttribute(sa::selftest_mma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
      cudaSuccess)
    return SA_ERR_CUDA;
  sa::selftest_mma_kernel<<<1, 128, smem, st>>>(ma, mb, args, D, status);
  sa::count_launch();
  return cudaGetLastError() == cudaSuccess ? SA_OK : SA_ERR_CUDA;
}
