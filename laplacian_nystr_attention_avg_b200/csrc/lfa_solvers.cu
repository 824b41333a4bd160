// Linear solvers for the landmark system W Y = B outside the forward pass: conjugate gradients, the
// solver the LaplacianFormer note ablates against Newton-Schulz (papernotes.org, §关键设计 3 and the
// CG-vs-NS ablation), and the forward pass's own Newton-Schulz chain started from a given W. They
// exist to measure the two solvers on the same matrices (the note's robustness claim at kappa = 50).
//
// k_cg: one CTA per (unit, block of 32 right-hand sides), 256 threads; thread i owns row i (m <= 256)
// of the residual R and the iterate Y in registers, the search directions P live in shared memory.
// Every column runs its own Hestenes-Stiefel recursion from Y_0 = 0 for exactly `iters` steps:
//   WP = W P,  a = (r^T r) / (p^T W p) (0 when p^T W p <= 0),  Y += a P,  R -= a WP,
//   beta = (r'^T r') / (r^T r) (0 when r^T r = 0),  P = R + beta P,
// in fp32, with column sums in a fixed order (deterministic). W is read as W[j][i] for W[i][j]
// (coalesced along a row; W is symmetric).
#include "lfa_internal.h"

namespace lfa {
namespace {

constexpr int kCgThreads = 256;
constexpr int kCgCols = 32;
constexpr int kCgRs = kCgCols + 1;   // row stride of the product buffer (bank-conflict free columns)

// Column sums of v[i][c] over the 256 rows: rows 32 g .. 32 g + 31 by thread (g = t / 32, c = t % 32),
// then the 8 partials in order. buf is [256][kCgRs], part [8][32], out [32].
__device__ void column_sums(const float (&v)[kCgCols], float* buf, float* part, float* out) {
  const int t = threadIdx.x;
#pragma unroll
  for (int c = 0; c < kCgCols; ++c) buf[t * kCgRs + c] = v[c];
  __syncthreads();
  {
    const int g = t >> 5, c = t & 31;
    float s = 0.f;
    for (int r = 32 * g; r < 32 * g + 32; ++r) s += buf[r * kCgRs + c];
    part[g * 32 + c] = s;
  }
  __syncthreads();
  if (t < 32) {
    float s = 0.f;
    for (int g = 0; g < kCgThreads / 32; ++g) s += part[g * 32 + t];
    out[t] = s;
  }
  __syncthreads();
}

__global__ void __launch_bounds__(kCgThreads) k_cg(const float* W, const float* B, float* Y, int m, int nrhs,
                                                   int iters) {
  extern __shared__ float4 smem_f4[];
  float* P = reinterpret_cast<float*>(smem_f4);   // [256][32] search directions
  float* buf = P + kCgThreads * kCgCols;           // [256][33]
  float* part = buf + kCgThreads * kCgRs;          // [8][32]
  float* rr = part + 8 * 32;                       // [32] r^T r
  float* tmp = rr + 32;                            // [32] p^T W p, then r'^T r'
  float* coef = tmp + 32;                          // [32] a, then beta
  const int u = blockIdx.y, c0 = blockIdx.x * kCgCols, i = threadIdx.x;
  const int nc = min(kCgCols, nrhs - c0);
  const float* Wu = W + (size_t)u * m * m;
  const float* Bu = B + (size_t)u * m * nrhs;
  float r[kCgCols], y[kCgCols], v[kCgCols];
#pragma unroll
  for (int c = 0; c < kCgCols; ++c) {
    r[c] = (i < m && c < nc) ? Bu[(size_t)i * nrhs + c0 + c] : 0.f;
    y[c] = 0.f;
    P[i * kCgCols + c] = r[c];
    v[c] = r[c] * r[c];
  }
  column_sums(v, buf, part, rr);
  for (int it = 0; it < iters; ++it) {
    // WP row i = sum_j W[j][i] P[j][:]
    float wp[kCgCols];
#pragma unroll
    for (int c = 0; c < kCgCols; ++c) wp[c] = 0.f;
    if (i < m) {
      int j = 0;
      for (; j + 4 <= m; j += 4) {
        float w[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) w[q] = __ldg(Wu + (size_t)(j + q) * m + i);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float4* pr = reinterpret_cast<const float4*>(P + (j + q) * kCgCols);
#pragma unroll
          for (int c4 = 0; c4 < kCgCols / 4; ++c4) {
            const float4 pv = pr[c4];
            wp[4 * c4 + 0] = fmaf(w[q], pv.x, wp[4 * c4 + 0]);
            wp[4 * c4 + 1] = fmaf(w[q], pv.y, wp[4 * c4 + 1]);
            wp[4 * c4 + 2] = fmaf(w[q], pv.z, wp[4 * c4 + 2]);
            wp[4 * c4 + 3] = fmaf(w[q], pv.w, wp[4 * c4 + 3]);
          }
        }
      }
      for (; j < m; ++j) {
        const float w = __ldg(Wu + (size_t)j * m + i);
        const float4* pr = reinterpret_cast<const float4*>(P + j * kCgCols);
#pragma unroll
        for (int c4 = 0; c4 < kCgCols / 4; ++c4) {
          const float4 pv = pr[c4];
          wp[4 * c4 + 0] = fmaf(w, pv.x, wp[4 * c4 + 0]);
          wp[4 * c4 + 1] = fmaf(w, pv.y, wp[4 * c4 + 1]);
          wp[4 * c4 + 2] = fmaf(w, pv.z, wp[4 * c4 + 2]);
          wp[4 * c4 + 3] = fmaf(w, pv.w, wp[4 * c4 + 3]);
        }
      }
    }
#pragma unroll
    for (int c = 0; c < kCgCols; ++c) v[c] = P[i * kCgCols + c] * wp[c];
    column_sums(v, buf, part, tmp);
    if (i < kCgCols) coef[i] = tmp[i] > 0.f ? rr[i] / tmp[i] : 0.f;
    __syncthreads();
#pragma unroll
    for (int c = 0; c < kCgCols; ++c) {
      y[c] = fmaf(coef[c], P[i * kCgCols + c], y[c]);
      r[c] = fmaf(-coef[c], wp[c], r[c]);
      v[c] = r[c] * r[c];
    }
    column_sums(v, buf, part, tmp);
    if (i < kCgCols) {
      coef[i] = rr[i] > 0.f ? tmp[i] / rr[i] : 0.f;
      rr[i] = tmp[i];
    }
    __syncthreads();
#pragma unroll
    for (int c = 0; c < kCgCols; ++c) P[i * kCgCols + c] = fmaf(coef[c], P[i * kCgCols + c], r[c]);
    __syncthreads();
  }
  if (i < m) {
    float* Yu = Y + (size_t)u * m * nrhs + (size_t)i * nrhs + c0;
#pragma unroll
    for (int c = 0; c < kCgCols; ++c)
      if (c < nc) Yu[c] = y[c];
  }
}

size_t cg_smem() {
  return sizeof(float) * ((size_t)kCgThreads * kCgCols + (size_t)kCgThreads * kCgRs + 8 * 32 + 3 * 32);
}

}  // namespace

cudaError_t cg_set_attributes() {
  return cudaFuncSetAttribute(k_cg, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)cg_smem());
}

cudaError_t launch_cg(const float* W, const float* B, float* Y, int U, int m, int nrhs, int iters,
                      cudaStream_t st) {
  const dim3 grid((nrhs + kCgCols - 1) / kCgCols, U);
  k_cg<<<grid, kCgThreads, cg_smem(), st>>>(W, B, Y, m, nrhs, iters);
  return cudaGetLastError();
}

}  // namespace lfa
