// Batched m x m products for the per-stage kernels (m <= 256) on the tcgen05 tensor cores: the
// Newton-Schulz steps of the forward pass (LaplacianFormer note, papernotes.org, §关键设计 3) when the
// one-CTA chain does not apply, the iterates and the reverse steps of the backward pass, and the
// Reading-B products.
//
// Out = scale * op(A) op(B) + beta * Cin + add_diag * I per (job, unit); up to three independent jobs
// share one launch (grid z = job * U + unit). Each CTA forms a 128 x 64 output tile (M = 128 rows i,
// N = 64 columns j) in a TMEM accumulator, fp32-accurate by three TF32 products (hi*hi + hi*lo +
// lo*hi with hi = tf32(x), lo = x - hi: about 2^-21 relative per product). K advances in steps of 64
// (two 128-byte SW128 K-halves of fp32 per row). The operands of step c + 1 are already in registers
// while the 24 MMAs of step c run: they are split and stored into the other shared-memory stage, and
// the global loads of step c + 2 are issued right after, so one L2 latency overlaps each step.
#include "lfa_internal.h"
#include "lfa_sm100.cuh"

namespace lfa {
namespace {

using namespace sm100;

constexpr int kTM = 128, kTN = 64, kKS = 64;
constexpr int kGT = 256;                          // threads per CTA
constexpr uint32_t kAH = kTM * 128;               // bytes of one K-half of one A split tile
constexpr uint32_t kBH = kTN * 128;               // bytes of one K-half of one B split tile
// stage: A hi [2 halves], A lo [2], B hi [2], B lo [2]
constexpr uint32_t kOffAhi = 0, kOffAlo = 2 * kAH, kOffBhi = 4 * kAH, kOffBlo = 4 * kAH + 2 * kBH;
constexpr uint32_t kStage = 4 * kAH + 4 * kBH;    // 96 KB
constexpr uint32_t kGemmSmem = 2 * kStage + 1024 + 64;
constexpr int kAR = kTM * kKS / 4 / kGT;          // float4 groups of A per thread and step (8)
constexpr int kBR = kTN * kKS / 4 / kGT;          // of B (4)

// byte offset of (row, fp32 column k < 64) in a K-major split tile made of two SW128 K-halves
__device__ __forceinline__ uint32_t kofs(int row, int k, uint32_t half_bytes) {
  return (uint32_t)(k >> 5) * half_bytes + sw128(row, (k & 31) >> 2) + (k & 3) * 4;
}

struct Regs {
  float4 a[kAR];
  float4 b[kBR];
};

__global__ void __launch_bounds__(kGT) k_mm_tc(int m, int U, MmJobs jobs) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
  unsigned char* sm = smem_raw + pad;
  const uint32_t sbase = smem_u32(sm);
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + 2 * kStage);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + 2 * kStage + 32);
  __shared__ int status_dummy;
  const int jz = blockIdx.z / U, u = blockIdx.z % U;
  const MmJob J = jobs.job[jz];
  const float* A = J.A + u * J.a_stride;
  const float* B = J.B + u * J.b_stride;
  const float* Cin = J.C ? J.C + u * J.c_stride : nullptr;
  float* Out = J.O + u * J.o_stride;
  const int i0 = blockIdx.y * kTM, j0 = blockIdx.x * kTN;
  const int t = threadIdx.x, w = t >> 5, lane = t & 31;
  if (w == 0) {
    tmem_alloc(tmem_slot, 64);
    tmem_relinquish();
  }
  if (t == 0) {
    mbar_init(bars + 0, 1);
    mbar_init(bars + 1, 1);
    mbar_init_fence();
    status_dummy = 0;
  }
  const bool vec = (m & 3) == 0;   // rows start on 16-byte boundaries
  // Group e of a step covers 4 consecutive elements along the stored matrix's contiguous index:
  //   A untransposed: row i = e / 16, k = 4 (e % 16) .. ;  transposed: row k = e / 32, i = 4 (e % 32) ..
  //   B transposed:   row j = e / 16, k = 4 (e % 16) .. ;  untransposed: row k = e / 16, j = 4 (e % 16) ..
  auto ld4 = [&](const float* base, int row, int col, int nrow, int ncol) -> float4 {
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    if (row < nrow) {
      const float* src = base + (size_t)row * m + col;
      if (vec && col + 3 < ncol) v = *reinterpret_cast<const float4*>(src);
      else {
        v.x = col + 0 < ncol ? src[0] : 0.f;
        v.y = col + 1 < ncol ? src[1] : 0.f;
        v.z = col + 2 < ncol ? src[2] : 0.f;
        v.w = col + 3 < ncol ? src[3] : 0.f;
      }
    }
    return v;
  };
  auto load = [&](int c, Regs& r) {
    const int k0 = c * kKS;
#pragma unroll
    for (int x = 0; x < kAR; ++x) {
      const int e = t + kGT * x;
      r.a[x] = J.ta ? ld4(A, k0 + (e >> 5), i0 + 4 * (e & 31), m, m) : ld4(A, i0 + (e >> 4), k0 + 4 * (e & 15), m, m);
    }
#pragma unroll
    for (int x = 0; x < kBR; ++x) {
      const int e = t + kGT * x;
      r.b[x] = J.tb ? ld4(B, j0 + (e >> 4), k0 + 4 * (e & 15), m, m) : ld4(B, k0 + (e >> 4), j0 + 4 * (e & 15), m, m);
    }
  };
  auto put = [&](unsigned char* hi, unsigned char* lo, uint32_t off, float v) {
    const float h = tf32_round(v);
    *reinterpret_cast<float*>(hi + off) = h;
    *reinterpret_cast<float*>(lo + off) = v - h;
  };
  auto put4 = [&](unsigned char* hi, unsigned char* lo, uint32_t off, float4 v) {
    float4 h, l;
    h.x = tf32_round(v.x); l.x = v.x - h.x;
    h.y = tf32_round(v.y); l.y = v.y - h.y;
    h.z = tf32_round(v.z); l.z = v.z - h.z;
    h.w = tf32_round(v.w); l.w = v.w - h.w;
    *reinterpret_cast<float4*>(hi + off) = h;
    *reinterpret_cast<float4*>(lo + off) = l;
  };
  // split into tf32 hi / lo and store K-major: A rows i, B rows j, each row the step's 64 k
  auto store = [&](const Regs& r, int buf) {
    unsigned char* st = sm + buf * kStage;
#pragma unroll
    for (int x = 0; x < kAR; ++x) {
      const int e = t + kGT * x;
      if (!J.ta) {
        put4(st + kOffAhi, st + kOffAlo, kofs(e >> 4, 4 * (e & 15), kAH), r.a[x]);
      } else {
        const int k = e >> 5, i = 4 * (e & 31);
        put(st + kOffAhi, st + kOffAlo, kofs(i + 0, k, kAH), r.a[x].x);
        put(st + kOffAhi, st + kOffAlo, kofs(i + 1, k, kAH), r.a[x].y);
        put(st + kOffAhi, st + kOffAlo, kofs(i + 2, k, kAH), r.a[x].z);
        put(st + kOffAhi, st + kOffAlo, kofs(i + 3, k, kAH), r.a[x].w);
      }
    }
#pragma unroll
    for (int x = 0; x < kBR; ++x) {
      const int e = t + kGT * x;
      if (J.tb) {
        put4(st + kOffBhi, st + kOffBlo, kofs(e >> 4, 4 * (e & 15), kBH), r.b[x]);
      } else {
        const int k = e >> 4, j = 4 * (e & 15);
        put(st + kOffBhi, st + kOffBlo, kofs(j + 0, k, kBH), r.b[x].x);
        put(st + kOffBhi, st + kOffBlo, kofs(j + 1, k, kBH), r.b[x].y);
        put(st + kOffBhi, st + kOffBlo, kofs(j + 2, k, kBH), r.b[x].z);
        put(st + kOffBhi, st + kOffBlo, kofs(j + 3, k, kBH), r.b[x].w);
      }
    }
  };
  const int nk = (m + kKS - 1) / kKS;
  Regs r;
  load(0, r);
  store(r, 0);
  if (nk > 1) load(1, r);
  fence_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t id = idesc(2, kTM, kTN, 0, 0);
  for (int c = 0; c < nk; ++c) {
    const int buf = c & 1;
    if (t == 0) {
      tc_fence_after();
      const uint32_t sb = sbase + buf * kStage;
#pragma unroll
      for (int g = 0; g < 3; ++g) {
        const uint32_t ab = sb + ((g == 2) ? kOffAlo : kOffAhi);
        const uint32_t bb = sb + ((g == 1) ? kOffBlo : kOffBhi);
#pragma unroll
        for (int ks = 0; ks < kKS / 8; ++ks) {
          const uint64_t ad = desc_sw128(ab + (ks >> 2) * kAH, 16, 1024) + (uint64_t)((ks & 3) * 2);
          const uint64_t bd = desc_sw128(bb + (ks >> 2) * kBH, 16, 1024) + (uint64_t)((ks & 3) * 2);
          mma_tf32(tmem, ad, bd, id, (c > 0 || g > 0 || ks > 0) ? 1u : 0u);
        }
      }
      mma_commit(bars + buf);
    }
    if (c + 1 < nk) {
      // buffer buf ^ 1 was read by the products of step c - 1 (the ((c - 1) >> 1)-th commit on it)
      if (c >= 1) mbar_wait(bars + (buf ^ 1), ((c - 1) >> 1) & 1, &status_dummy, 1);
      store(r, buf ^ 1);
      if (c + 2 < nk) load(c + 2, r);
      fence_async_smem();
      tc_fence_before();
      __syncthreads();
    }
  }
  // the last commit covers every product issued before it
  mbar_wait(bars + ((nk - 1) & 1), ((nk - 1) >> 1) & 1, &status_dummy, 1);
  tc_fence_after();
  // epilogue: warp w reads TMEM lanes 32 (w % 4) .., columns 32 (w / 4) ..
  {
    const int q = w & 3, h = w >> 2;
    float v[32];
    tmem_ld32(tmem + ((uint32_t)(32 * q) << 16) + 32 * h, v);
    const int i = i0 + 32 * q + lane;
    if (i < m) {
#pragma unroll
      for (int x = 0; x < 32; ++x) {
        const int j = j0 + 32 * h + x;
        if (j < m) {
          float o = J.scale * v[x] + (i == j ? J.add_diag : 0.f);
          if (Cin) o = fmaf(J.beta, Cin[(size_t)i * m + j], o);
          Out[(size_t)i * m + j] = o;
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (w == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 64);
  }
}

}  // namespace

cudaError_t gemm_set_attributes() {
  return cudaFuncSetAttribute(k_mm_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kGemmSmem);
}

cudaError_t launch_mm(const MmJob* jobs, int njobs, int m, int U, cudaStream_t st) {
  if (njobs < 1 || njobs > 3) return cudaErrorInvalidValue;
  MmJobs js{};
  for (int i = 0; i < njobs; ++i) js.job[i] = jobs[i];
  js.n = njobs;
  const dim3 g(ceil_div(m, kTN), ceil_div(m, kTM), U * njobs);
  k_mm_tc<<<g, kGT, kGemmSmem, st>>>(m, U, js);
  return cudaGetLastError();
}

}  // namespace lfa
