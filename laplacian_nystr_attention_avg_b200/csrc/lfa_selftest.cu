// Self-test kernels for the sm_100a building blocks used by the fused forward pass: each mode
// runs one tensor-core product or TMA load through the exact shared-memory layouts and
// descriptors the fused kernel uses, and returns the result for comparison on the host.
//
//   mode 0  bf16, K-major A [128 x 64] x K-major B^T [64 x 64]      (pass-2 product C M')
//   mode 1  bf16, MN-major A^T and B, K = 128, M = 64 accumulator    (pass-1 product C^T V)
//   mode 3  bf16, K-major A read at a row offset `param` (a multiple of 8: 8-row groups)
//   mode 4  TMA 3-D load of 128 x 64 bf16 rows (128-byte swizzle) starting at row `param`,
//           out-of-range rows zero-filled; read back through the software swizzle
//   mode 5  tf32 x1, K-major A [128 x 64] x K-major B^T [64 x 64]
//   mode 7  tf32 x3 split, A [128 x 64], B^T = rows 64..127 of A read K-major (Newton-Schulz)
#include <string.h>

#include "lfa_internal.h"
#include "lfa_sm100.cuh"
#include "lfa_tma_host.h"

namespace lfa {
namespace {

using namespace sm100;

constexpr int kSelfThreads = 128;

struct SelfSmem {
  alignas(1024) unsigned char a[2 * 32768];   // A (and A_lo for tf32)
  alignas(1024) unsigned char b[16384];
  uint64_t bar;
  uint32_t tmem;
};

__device__ void store_bf16_sw128(unsigned char* tile, int row, int col, float v) {
  const uint32_t off = sw128(row, col >> 3) + ((col & 7) << 1);
  *reinterpret_cast<__nv_bfloat16*>(tile + off) = __float2bfloat16_rn(v);
}

__device__ void store_f32_sw128(unsigned char* tile, int row, int col, float v) {
  // 2 K-halves of 32 fp32 per 128-byte row, 16 KB apart (128-row tiles)
  const int half = col >> 5, cc = col & 31;
  const uint32_t off = half * 16384 + sw128(row, cc >> 2) + ((cc & 3) << 2);
  *reinterpret_cast<float*>(tile + off) = v;
}

__global__ void __launch_bounds__(kSelfThreads) k_selftest(int mode, const float* A, const float* B, float* D,
                                                            int param, const __grid_constant__ CUtensorMap tmap,
                                                            int* status) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  // operand tiles must start on a 1024-byte boundary (128-byte swizzle pattern)
  const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
  SelfSmem& s = *reinterpret_cast<SelfSmem*>(smem_raw + pad);
  const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
  if (warp == 0) tmem_alloc(&s.tmem, 64);
  if (t == 0) {
    mbar_init(&s.bar, 1);
    mbar_init_fence();
  }
  memset(s.a + t * 512, 0, 512);     // 128 threads x 512 B = 64 KB
  memset(s.b + t * 128, 0, 128);     // 16 KB
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s.tmem;
  const uint32_t a0 = smem_u32(s.a), b0 = smem_u32(s.b);
  uint32_t parity = 0;

  if (mode == 4) {
    if (t == 0) {
      mbar_expect_tx(&s.bar, 128 * 128);
      tma_load_3d(s.a, &tmap, 0, param, 0, &s.bar);
    }
    mbar_wait(&s.bar, 0, status, kStatusTimeout);
    for (int e = t; e < 128 * 64; e += kSelfThreads) {
      const int r = e / 64, c = e % 64;
      const uint32_t off = sw128(r, c >> 3) + ((c & 7) << 1);
      D[e] = __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(s.a + off));
    }
  } else {
    // stage operands
    if (mode == 0 || mode == 3) {
      const int rows = mode == 3 ? 192 : 128;
      for (int e = t; e < rows * 64; e += kSelfThreads) store_bf16_sw128(s.a, e / 64, e % 64, A[e]);
      for (int e = t; e < 64 * 64; e += kSelfThreads) store_bf16_sw128(s.b, e / 64, e % 64, B[e]);
    } else if (mode == 1) {
      for (int e = t; e < 128 * 64; e += kSelfThreads) store_bf16_sw128(s.a, e / 64, e % 64, A[e]);
      for (int e = t; e < 128 * 64; e += kSelfThreads) store_bf16_sw128(s.a + 16384, e / 64, e % 64, B[e]);
    } else if (mode == 5) {
      for (int e = t; e < 128 * 64; e += kSelfThreads) store_f32_sw128(s.a, e / 64, e % 64, A[e]);
      for (int e = t; e < 64 * 64; e += kSelfThreads) {
        // 64-row tile: K-halves 8 KB apart
        const int r = e / 64, c = e % 64, half = c >> 5, cc = c & 31;
        *reinterpret_cast<float*>(s.b + half * 8192 + sw128(r, cc >> 2) + ((cc & 3) << 2)) = B[e];
      }
    } else if (mode == 7) {
      for (int e = t; e < 128 * 64; e += kSelfThreads) {
        const float x = A[e];
        const float hi = tf32_round(x);
        store_f32_sw128(s.a, e / 64, e % 64, hi);
        store_f32_sw128(s.a + 32768, e / 64, e % 64, x - hi);
      }
    }
    fence_async_smem();
    __syncthreads();
    if (t == 0) {
      tc_fence_after();
      if (mode == 0 || mode == 3) {
        const uint32_t id = idesc(1, 128, 64, 0, 0);
        const uint32_t abase = a0 + (mode == 3 ? param * 128 : 0);
        for (int kk = 0; kk < 4; ++kk)
          mma_bf16(tmem, desc_sw128(abase + kk * 32, 16, 1024), desc_sw128(b0 + kk * 32, 16, 1024), id, kk > 0);
      } else if (mode == 5) {
        const uint32_t id = idesc(2, 128, 64, 0, 0);
        for (int ks = 0; ks < 8; ++ks)
          mma_tf32(tmem, desc_sw128(a0 + (ks >> 2) * 16384 + (ks & 3) * 32, 16, 1024),
                   desc_sw128(b0 + (ks >> 2) * 8192 + (ks & 3) * 32, 16, 1024), id, ks > 0);
      } else if (mode == 7) {
        const uint32_t id = idesc(2, 128, 64, 0, 0);
        const uint32_t lo = a0 + 32768;
        for (int g = 0; g < 3; ++g) {
          const uint32_t ab = (g == 2) ? lo : a0;
          const uint32_t bb = (g == 1) ? lo : a0;
          for (int ks = 0; ks < 8; ++ks) {
            // B^T rows = A rows 64..127: same K-major layout, 8 KB into each 16 KB K-half
            const uint64_t ad = desc_sw128(ab + (ks >> 2) * 16384 + (ks & 3) * 32, 16, 1024);
            const uint64_t bd = desc_sw128(bb + 8192 + (ks >> 2) * 16384 + (ks & 3) * 32, 16, 1024);
            mma_tf32(tmem, ad, bd, id, (g > 0 || ks > 0) ? 1u : 0u);
          }
        }
      } else if (mode == 1) {
        const uint32_t id = idesc(1, 64, 64, 1, 1);
        for (int kk = 0; kk < 8; ++kk)
          mma_bf16(tmem, desc_sw128(a0 + kk * 2048, 8192, 1024), desc_sw128(a0 + 16384 + kk * 2048, 8192, 1024),
                   id, kk > 0);
      }
      mma_commit(&s.bar);
    }
    __syncwarp();
    mbar_wait(&s.bar, parity, status, kStatusTimeout);
    tc_fence_after();
    float v[32];
    const int M = (mode == 1) ? 64 : 128;
    for (int h = 0; h < 2; ++h) {
      tmem_ld32(tmem + ((uint32_t)(32 * warp) << 16) + 32 * h, v);
      int row = -1;
      if (M == 128) row = 32 * warp + lane;
      else if (lane < 16) row = 16 * warp + lane;     // M = 64: rows 16w..16w+15 in lanes 0..15
      if (row >= 0)
        for (int c = 0; c < 32; ++c) D[row * 64 + 32 * h + c] = v[c];
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 64);
    tmem_relinquish();
  }
}

}  // namespace

cudaError_t launch_selftest(int mode, const float* A, const float* B, float* D, int param, const void* tma_src,
                            int tma_rows, int* status, cudaStream_t st) {
  CUtensorMap map;
  memset(&map, 0, sizeof(map));
  if (mode == 4 && !make_tmap_rows_bf16(&map, tma_src, (uint64_t)tma_rows, 1, 128)) return cudaErrorInvalidValue;
  const size_t smem = sizeof(SelfSmem) + 1024;
  cudaError_t e = cudaFuncSetAttribute(k_selftest, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  k_selftest<<<1, kSelfThreads, smem, st>>>(mode, A, B, D, param, map, status);
  return cudaGetLastError();
}

}  // namespace lfa
