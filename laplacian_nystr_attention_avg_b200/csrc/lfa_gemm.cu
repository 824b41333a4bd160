// Batched m x m FP32 products for the per-stage kernels (m <= 256): the Newton-Schulz steps of
// the forward pass (LaplacianFormer note, papernotes.org, §关键设计 3) when m > 64, and the
// iterates and reverse steps of the backward pass.
//
// Out = scale * op(A) op(B) + beta * Cin + add_diag * I per (job, unit); up to three independent
// jobs share one launch (grid z = job * U + unit). 64 x 64 output tile per CTA, 4 x 4 per
// thread, K in steps of 32: the next step's operands are loaded into registers while the current
// one is multiplied from shared memory (two buffers, one barrier per step).
#include "lfa_internal.h"

namespace lfa {
namespace {

constexpr int kTile = 64;
constexpr int kKStep = 32;
constexpr int kPad = kTile + 4;   // row stride (floats) of the k-major shared tiles

__global__ void __launch_bounds__(256) k_mm(int m, int U, MmJobs jobs) {
  __shared__ __align__(16) float As[2][kKStep][kPad];   // As[k][i] = op(A)(i0 + i, k0 + k)
  __shared__ __align__(16) float Bs[2][kKStep][kPad];   // Bs[k][j] = op(B)(k0 + k, j0 + j)
  const int jz = blockIdx.z / U, u = blockIdx.z % U;
  const MmJob J = jobs.job[jz];
  const float* A = J.A + u * J.a_stride;
  const float* B = J.B + u * J.b_stride;
  const float* Cin = J.C ? J.C + u * J.c_stride : nullptr;
  float* Out = J.O + u * J.o_stride;
  const int i0 = blockIdx.y * kTile, j0 = blockIdx.x * kTile;
  const int t = threadIdx.x, bi = t >> 4, bj = t & 15;
  float ra[8], rb[8];
  // element r of this thread's share of a K step: coalesced along the contiguous index of the
  // stored matrix (k for A row-major, i for A^T; j for B row-major, k for B^T)
  auto a_ik = [&](int e, int& i, int& k) {
    if (J.ta) { k = e >> 6; i = e & 63; } else { i = e >> 5; k = e & 31; }
  };
  auto b_kj = [&](int e, int& k, int& j) {
    if (J.tb) { j = e >> 5; k = e & 31; } else { k = e >> 6; j = e & 63; }
  };
  auto load = [&](int k0) {
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      const int e = t + 256 * r;
      int i, k, j, k2;
      a_ik(e, i, k);
      b_kj(e, k2, j);
      const int gi = i0 + i, gk = k0 + k, gk2 = k0 + k2, gj = j0 + j;
      ra[r] = (gi < m && gk < m) ? (J.ta ? A[(size_t)gk * m + gi] : A[(size_t)gi * m + gk]) : 0.f;
      rb[r] = (gk2 < m && gj < m) ? (J.tb ? B[(size_t)gj * m + gk2] : B[(size_t)gk2 * m + gj]) : 0.f;
    }
  };
  auto store = [&](int buf) {
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      const int e = t + 256 * r;
      int i, k, j, k2;
      a_ik(e, i, k);
      b_kj(e, k2, j);
      As[buf][k][i] = ra[r];
      Bs[buf][k2][j] = rb[r];
    }
  };
  float acc[4][4] = {};
  const int nk = (m + kKStep - 1) / kKStep;
  load(0);
  store(0);
  __syncthreads();
  for (int c = 0; c < nk; ++c) {
    if (c + 1 < nk) load((c + 1) * kKStep);
    const int buf = c & 1;
#pragma unroll 8
    for (int k = 0; k < kKStep; ++k) {
      const float4 a = *reinterpret_cast<const float4*>(&As[buf][k][4 * bi]);
      const float4 b = *reinterpret_cast<const float4*>(&Bs[buf][k][4 * bj]);
      const float av[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
      for (int x = 0; x < 4; ++x) {
        acc[x][0] = fmaf(av[x], b.x, acc[x][0]);
        acc[x][1] = fmaf(av[x], b.y, acc[x][1]);
        acc[x][2] = fmaf(av[x], b.z, acc[x][2]);
        acc[x][3] = fmaf(av[x], b.w, acc[x][3]);
      }
    }
    if (c + 1 < nk) store(buf ^ 1);
    __syncthreads();
  }
#pragma unroll
  for (int x = 0; x < 4; ++x)
#pragma unroll
    for (int y = 0; y < 4; ++y) {
      const int i = i0 + 4 * bi + x, j = j0 + 4 * bj + y;
      if (i < m && j < m) {
        float v = J.scale * acc[x][y] + (i == j ? J.add_diag : 0.f);
        if (Cin) v = fmaf(J.beta, Cin[(size_t)i * m + j], v);
        Out[(size_t)i * m + j] = v;
      }
    }
}

}  // namespace

cudaError_t launch_mm(const MmJob* jobs, int njobs, int m, int U, cudaStream_t st) {
  if (njobs < 1 || njobs > 3) return cudaErrorInvalidValue;
  MmJobs js{};
  for (int i = 0; i < njobs; ++i) js.job[i] = jobs[i];
  js.n = njobs;
  const dim3 g(ceil_div(m, kTile), ceil_div(m, kTile), U * njobs);
  k_mm<<<g, 256, 0, st>>>(m, U, js);
  return cudaGetLastError();
}

}  // namespace lfa
