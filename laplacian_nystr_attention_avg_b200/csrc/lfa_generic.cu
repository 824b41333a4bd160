// Generic forward path of Laplacian-kernel Nystrom attention: every shape and dtype the
// ABI accepts, CUDA cores only, two streaming passes over the tokens (C recomputed in
// pass 2, never stored in HBM).
//
// Steps (LaplacianFormer note, papernotes.org: §整体框架 flowchart, §关键设计 1-3):
//   k_pool          L = r x r average pool of Q                         (§关键设计 2)
//   (m <= 64: k_ns_tc in lfa_fused.cu: W, ||W||_2, alpha and the T steps on tcgen05, one CTA per unit)
//   k_gram / k_alpha / k_mm (lfa_gemm.cu) / k_ns_gemm   the same for 64 < m <= 256, spread over
//                   CTAs (§关键设计 3); k_ns_gemm forms the closing residual I - W X_T and its norm
//   k_pass1         C tiles in registers/smem, column sums of C and C^2, raw C^T V, sum V
//   k_combine_*     mu, var, s = 1/sqrt(var + eps); A = C~^T V by rank-1 folding; M = X A;
//                   M' = diag(s) M; bias b = (1/N 1 - s o mu)^T M               (§关键设计 1)
//   k_pass2         O = C M' + 1 b^T + DWC(V)                                  (§关键设计 1)
#include <math.h>

#include <algorithm>

#include "lfa_internal.h"

namespace lfa {
namespace {

__device__ __forceinline__ float to_f(float x) { return x; }
__device__ __forceinline__ float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }

// 4 consecutive elements -> float4 (16-byte / 8-byte aligned by the callers' layout)
__device__ __forceinline__ float4 load4(const float* g) { return *reinterpret_cast<const float4*>(g); }
__device__ __forceinline__ float4 load4(const __nv_bfloat16* g) {
  uint2 raw = *reinterpret_cast<const uint2*>(g);
  __nv_bfloat162 a = *reinterpret_cast<__nv_bfloat162*>(&raw.x);
  __nv_bfloat162 b = *reinterpret_cast<__nv_bfloat162*>(&raw.y);
  float2 fa = __bfloat1622float2(a), fb = __bfloat1622float2(b);
  return make_float4(fa.x, fa.y, fb.x, fb.y);
}
__device__ __forceinline__ void store4(float* g, float4 v) { *reinterpret_cast<float4*>(g) = v; }
__device__ __forceinline__ void store4(__nv_bfloat16* g, float4 v) {
  __nv_bfloat162 a = __floats2bfloat162_rn(v.x, v.y);
  __nv_bfloat162 b = __floats2bfloat162_rn(v.z, v.w);
  uint2 raw;
  raw.x = *reinterpret_cast<uint32_t*>(&a);
  raw.y = *reinterpret_cast<uint32_t*>(&b);
  *reinterpret_cast<uint2*>(g) = raw;
}

__device__ __forceinline__ float l1_4(float4 a, float4 b, float acc) {
  acc += fabsf(a.x - b.x);
  acc += fabsf(a.y - b.y);
  acc += fabsf(a.z - b.z);
  acc += fabsf(a.w - b.w);
  return acc;
}

// ---------------------------------------------------------------------------------------
// Landmark pooling: one warp per landmark. A token row is C16 = d * sizeof(T) / 16 chunks of 16 bytes
// (C16 in {4, 8, 16}); lane = (token group tg = lane / C16, chunk c = lane % C16), so one load
// instruction of the warp covers 32 / C16 window tokens in full rows. The token groups' sums meet by
// shuffles, in a fixed order. (Other d: one lane per channel.)
// ---------------------------------------------------------------------------------------
__device__ __forceinline__ int unpack16(const uint4& raw, float* f, const float*) {
  f[0] = __uint_as_float(raw.x); f[1] = __uint_as_float(raw.y); f[2] = __uint_as_float(raw.z); f[3] = __uint_as_float(raw.w);
  return 4;
}
__device__ __forceinline__ int unpack16(const uint4& raw, float* f, const __nv_bfloat16*) {
  const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
  }
  return 8;
}

template <typename T>
__global__ void __launch_bounds__(kThreads) k_pool(Params p) {
  if (blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x == 0) *p.status = 0;
  const int u = blockIdx.y;
  const int l = blockIdx.x * (kThreads / 32) + threadIdx.x / 32;
  const int lane = threadIdx.x & 31;
  if (l >= p.m) return;
  const int Wr = p.W / p.r;
  const int Y0 = (l / Wr) * p.r, X0 = (l % Wr) * p.r;
  const T* q = static_cast<const T*>(p.Q) + (size_t)u * p.N * p.d;
  const float inv = 1.0f / float(p.r * p.r);
  constexpr int kPer = 16 / (int)sizeof(T);   // values per 16-byte chunk
  const int C16 = p.d / kPer;
  if (p.d % kPer == 0 && (C16 == 4 || C16 == 8 || C16 == 16)) {
    const int TG = 32 / C16, tg = lane / C16, c = lane % C16, rr = p.r * p.r;
    float acc[kPer];
#pragma unroll
    for (int i = 0; i < kPer; ++i) acc[i] = 0.f;
#pragma unroll 4
    for (int t = tg; t < rr; t += TG) {
      // window rows outside this call's band of grid rows (sequence split) contribute nothing here
      const int yl = Y0 + t / p.r - p.y0;
      if (yl < 0 || yl >= p.H) continue;
      const uint4 raw = __ldg(reinterpret_cast<const uint4*>(q + ((size_t)yl * p.W + X0 + t % p.r) * p.d) + c);
      float f[kPer];
      unpack16(raw, f, q);
#pragma unroll
      for (int i = 0; i < kPer; ++i) acc[i] += f[i];
    }
    for (int o = C16; o < 32; o <<= 1)
#pragma unroll
      for (int i = 0; i < kPer; ++i) acc[i] += __shfl_xor_sync(0xffffffffu, acc[i], o);
    if (tg == 0) {
      float* dst = p.L + ((size_t)u * p.m + l) * p.d + c * kPer;
#pragma unroll
      for (int i = 0; i < kPer; i += 4)
        *reinterpret_cast<float4*>(dst + i) = make_float4(acc[i] * inv, acc[i + 1] * inv, acc[i + 2] * inv, acc[i + 3] * inv);
    }
    return;
  }
  for (int k = lane; k < p.d; k += 32) {
    float acc = 0.f;
    for (int dy = 0; dy < p.r; ++dy) {
      const int yl = Y0 + dy - p.y0;
      if (yl < 0 || yl >= p.H) continue;
      for (int dx = 0; dx < p.r; ++dx) acc += to_f(q[((size_t)yl * p.W + X0 + dx) * p.d + k]);
    }
    p.L[((size_t)u * p.m + l) * p.d + k] = acc * inv;
  }
}

// ---------------------------------------------------------------------------------------
// Small-m landmark kernel + alpha + Newton-Schulz, one CTA per unit, all in shared memory.
// ---------------------------------------------------------------------------------------
// Sum of v over the block (every thread gets the total; all threads must call it).
// ---------------------------------------------------------------------------------------
// Large-m Newton-Schulz (64 < m <= 256): W and X in global memory, one launch per product.
// ---------------------------------------------------------------------------------------
// dst[i * ds + c] = src[i * d + c] for i * d + c < n (ds = d for a plain copy), with eight loads in flight
// per thread
__device__ __forceinline__ void stage_floats(float* dst, const float* src, int n, int d, int ds) {
  const int nt = blockDim.x;
  int e = threadIdx.x;
  for (; e + 7 * nt < n; e += 8 * nt) {
    float r[8];
#pragma unroll
    for (int x = 0; x < 8; ++x) r[x] = __ldg(src + e + x * nt);
#pragma unroll
    for (int x = 0; x < 8; ++x) {
      const int f = e + x * nt;
      dst[(f / d) * ds + f % d] = r[x];
    }
  }
  for (; e < n; e += nt) dst[(e / d) * ds + e % d] = __ldg(src + e);
}

// W = exp(-||l_a - l_b||_1 / lambda) + eps I: the unit's landmarks staged in shared memory (row stride
// d + 1, conflict-free), rows a of this CTA's group of 16, thread = column b (m <= kThreads); the
// distance is summed over k in order, so W is exactly symmetric.
__global__ void __launch_bounds__(kThreads) k_gram(Params p) {
  extern __shared__ float4 smem_f4[];
  float* Ls = reinterpret_cast<float*>(smem_f4);   // [m][d + 1]
  const int u = blockIdx.y, m = p.m, d = p.d, ds = d + 1, t = threadIdx.x;
  stage_floats(Ls, p.L + (size_t)u * m * d, m * d, d, ds);
  __syncthreads();
  const int b = t;
  if (b >= m) return;
  for (int r = 0; r < 16; ++r) {
    const int a = blockIdx.x * 16 + r;
    if (a >= m) break;
    float acc = 0.f;
    for (int k = 0; k < d; ++k) acc += fabsf(Ls[a * ds + k] - Ls[b * ds + k]);
    p.Wm[((size_t)u * m + a) * m + b] = exp2f(acc * p.neg_log2e_over_lam) + (a == b ? p.eps : 0.f);
  }
}

// Power iteration for ||W||_2: one CTA of kAlphaThreads per unit, four groups of kAlphaCols threads.
// Thread t of group g owns column t (m <= kAlphaCols): W is symmetric, so (W v)_t is column t,
// sum_j W[j][t] v_j, and the threads of a warp read consecutive words of one row (conflict-free in
// shared memory, coalesced in L2). Group g sums a quarter of the rows j; the four partials meet in
// shared memory in a fixed order. The first alpha_rows(m) rows of W are staged in shared memory once,
// the rest (at most 56, for m = 256) in registers, kAlphaRegRows of them per group. The split keeps
// 32 warps per SM and a short dependent chain: a step's time is the shared-memory reads of W.
constexpr int kAlphaCols = 256;
constexpr int kAlphaGroups = 4;
constexpr int kAlphaThreads = kAlphaCols * kAlphaGroups;
__host__ __device__ constexpr int alpha_rows(int m) {
  return m < (200 * 1024) / (4 * (m > 0 ? m : 1)) ? m : (200 * 1024) / (4 * (m > 0 ? m : 1));
}
constexpr int kAlphaRegRows = 14;
static_assert(kMaxM - alpha_rows(kMaxM) <= kAlphaGroups * kAlphaRegRows, "rows of W beyond shared memory and registers");
static_assert(kMaxM <= kAlphaCols, "one thread per entry of the power-iteration vector");

__global__ void __launch_bounds__(kAlphaThreads, 1) k_alpha(Params p) {
  __shared__ __align__(16) float v[kMaxM];
  __shared__ float part[kAlphaGroups][kAlphaCols], red[2 * kAlphaCols / 32];
  extern __shared__ float4 smem_f4[];
  float* Ws = reinterpret_cast<float*>(smem_f4);   // [alpha_rows(m)][m]
  const int u = blockIdx.x, m = p.m;
  const int t = threadIdx.x % kAlphaCols, g = threadIdx.x / kAlphaCols;
  const float* Wg = p.Wm + (size_t)u * m * m;
  const int rs = alpha_rows(m);
  stage_floats(Ws, Wg, rs * m, m, m);
  // this group's rows: [j0, j1) of the staged ones (j0 a multiple of 4, so v[j0..] reads as float4),
  // then rows rg + q (q < kAlphaRegRows) from registers
  const int qrows = ((rs + 4 * kAlphaGroups - 1) / (4 * kAlphaGroups)) * 4;
  const int j0 = min(rs, g * qrows), j1 = min(rs, j0 + qrows);
  const int rg = rs + g * kAlphaRegRows;
  float wr[kAlphaRegRows];
#pragma unroll
  for (int q = 0; q < kAlphaRegRows; ++q) wr[q] = (t < m && rg + q < m) ? Wg[(size_t)(rg + q) * m + t] : 0.f;
  if (threadIdx.x < m) v[threadIdx.x] = rsqrtf(float(m));
  __syncthreads();
  float rq = 0.f;
  const int iters = 24;
  const int j4 = j0 + ((j1 - j0) & ~3);
  for (int it = 0; it <= iters; ++it) {
    if (t < m) {
      float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
      for (int j = j0; j < j4; j += 4) {
        const float4 vj = *reinterpret_cast<const float4*>(v + j);
        a0 = fmaf(Ws[(size_t)j * m + t], vj.x, a0);
        a1 = fmaf(Ws[(size_t)(j + 1) * m + t], vj.y, a1);
        a2 = fmaf(Ws[(size_t)(j + 2) * m + t], vj.z, a2);
        a3 = fmaf(Ws[(size_t)(j + 3) * m + t], vj.w, a3);
      }
      for (int j = j4; j < j1; ++j) a0 = fmaf(Ws[(size_t)j * m + t], v[j], a0);
      if (rg < m) {
#pragma unroll
        for (int q = 0; q < kAlphaRegRows; ++q) {
          if (rg + q >= m) break;
          if (q % 4 == 0) a1 = fmaf(wr[q], v[rg + q], a1);
          if (q % 4 == 1) a2 = fmaf(wr[q], v[rg + q], a2);
          if (q % 4 == 2) a3 = fmaf(wr[q], v[rg + q], a3);
          if (q % 4 == 3) a0 = fmaf(wr[q], v[rg + q], a0);
        }
      }
      part[g][t] = (a0 + a1) + (a2 + a3);
    }
    __syncthreads();
    // w = W v (the group partials in order), v^T w and ||w||^2 over the first group's warps
    float w = 0.f;
    if (g == 0) {
      float vw = 0.f, nn = 0.f;
      if (t < m) {
        w = (part[0][t] + part[1][t]) + (part[2][t] + part[3][t]);
        vw = w * v[t];
        nn = w * w;
      }
      for (int o = 16; o > 0; o >>= 1) {
        vw += __shfl_xor_sync(0xffffffffu, vw, o);
        nn += __shfl_xor_sync(0xffffffffu, nn, o);
      }
      if ((t & 31) == 0) {
        red[t >> 5] = vw;
        red[kAlphaCols / 32 + (t >> 5)] = nn;
      }
    }
    __syncthreads();
    float vw = 0.f, nn = 0.f;
#pragma unroll
    for (int i = 0; i < kAlphaCols / 32; ++i) {
      vw += red[i];
      nn += red[kAlphaCols / 32 + i];
    }
    rq = vw;
    if (it == iters) break;
    if (g == 0 && t < m) v[t] = w * rsqrtf(nn);
    __syncthreads();
  }
  const float lmax = rq;
  const float alpha_p = 2.f / lmax;
  const int fallback = (alpha_p * lmax * lmax < 2.f) ? 0 : 1;
  const float alpha = fallback ? 1.f / (lmax * lmax) : alpha_p;
  // X_0 = alpha W^T = alpha W (W symmetric), from the staged rows where they are
  float* Xg = p.X + (size_t)u * m * m;
  const int ns = rs * m;
  for (int e = threadIdx.x; e < m * m; e += blockDim.x) Xg[e] = alpha * (e < ns ? Ws[e] : Wg[e]);
  if (threadIdx.x == 0) {
    float* inf = p.info + (size_t)u * kInfoStride;
    inf[kInfoAlpha] = alpha;
    inf[kInfoLambdaMax] = lmax;
    inf[kInfoFallback] = float(fallback);
    inf[kInfoResidual] = 0.f;
    if (!isfinite(lmax)) atomicOr(p.status, kStatusNonFinite);
  }
}

// out = scale * (A B) + add_diag * I for m x m row-major matrices of unit blockIdx.z.
// 64 x 64 output tile per CTA, 16-wide K chunks staged in shared memory.
// mode 2 additionally accumulates ||out||_F^2 into info[residual].
__global__ void __launch_bounds__(kThreads) k_ns_gemm(Params p, const float* Ab, const float* Bb,
                                                      float* Ob, float scale, float add_diag,
                                                      int accumulate_norm) {
  __shared__ float As[64][17];
  __shared__ __align__(16) float Bs[16][64];
  const int u = blockIdx.z, m = p.m;
  const float* A = Ab + (size_t)u * m * m;
  const float* B = Bb + (size_t)u * m * m;
  float* Out = Ob + (size_t)u * m * m;
  const int i0 = blockIdx.y * 64, j0 = blockIdx.x * 64;
  const int t = threadIdx.x, bi = t / 16, bj = t % 16;
  float acc[4][4] = {};
  for (int k0 = 0; k0 < m; k0 += 16) {
    for (int e = t; e < 64 * 16; e += blockDim.x) {
      const int r = e / 16, c = e % 16;
      As[r][c] = (i0 + r < m && k0 + c < m) ? A[(size_t)(i0 + r) * m + k0 + c] : 0.f;
      const int r2 = e / 64, c2 = e % 64;
      Bs[r2][c2] = (k0 + r2 < m && j0 + c2 < m) ? B[(size_t)(k0 + r2) * m + j0 + c2] : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int l = 0; l < 16; ++l) {
      float a[4];
#pragma unroll
      for (int x = 0; x < 4; ++x) a[x] = As[4 * bi + x][l];
      float4 b = *reinterpret_cast<const float4*>(&Bs[l][4 * bj]);
#pragma unroll
      for (int x = 0; x < 4; ++x) {
        acc[x][0] = fmaf(a[x], b.x, acc[x][0]);
        acc[x][1] = fmaf(a[x], b.y, acc[x][1]);
        acc[x][2] = fmaf(a[x], b.z, acc[x][2]);
        acc[x][3] = fmaf(a[x], b.w, acc[x][3]);
      }
    }
    __syncthreads();
  }
  float sq = 0.f;
#pragma unroll
  for (int x = 0; x < 4; ++x)
#pragma unroll
    for (int y = 0; y < 4; ++y) {
      const int i = i0 + 4 * bi + x, j = j0 + 4 * bj + y;
      if (i < m && j < m) {
        const float v = scale * acc[x][y] + (i == j ? add_diag : 0.f);
        Out[(size_t)i * m + j] = v;
        sq += v * v;
      }
    }
  if (accumulate_norm) {
    for (int o = 16; o > 0; o >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, o);
    if ((t & 31) == 0) atomicAdd(p.info + (size_t)u * kInfoStride + kInfoResidual, sq);
  }
}

__global__ void k_residual_sqrt(Params p) {
  const int u = blockIdx.x * blockDim.x + threadIdx.x;
  if (u >= p.U) return;
  float* r = p.info + (size_t)u * kInfoStride + kInfoResidual;
  *r = sqrtf(*r);
  if (!isfinite(*r)) atomicOr(p.status, kStatusNonFinite);
}

// ---------------------------------------------------------------------------------------
// Cross-kernel tile: rows [0, 64) of Qs against landmarks [j0, j0 + 64) of Ls.
// 256 threads: thread (tr, tl) owns rows 4tr..4tr+3 and landmarks j0 + tl + 16 jj.
// ---------------------------------------------------------------------------------------
__device__ __forceinline__ void cross_tile(const float* Qs, const float* Ls, float* Cs, int d,
                                           int j0, int m, int cs_stride, float scale,
                                           int valid_rows) {
  const int t = threadIdx.x, tr = t >> 4, tl = t & 15;
  const int ds = d + 4;
  float acc[4][4] = {};
  for (int k = 0; k < d; k += 4) {
    float4 q[4], l[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) q[i] = *reinterpret_cast<const float4*>(&Qs[(4 * tr + i) * ds + k]);
#pragma unroll
    for (int j = 0; j < 4; ++j)
      l[j] = *reinterpret_cast<const float4*>(&Ls[(j0 + tl + 16 * j) * ds + k]);
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[i][j] = l1_4(q[i], l[j], acc[i][j]);
  }
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int row = 4 * tr + i, col = j0 + tl + 16 * j;
      Cs[row * cs_stride + col] = (col < m && row < valid_rows) ? exp2f(acc[i][j] * scale) : 0.f;
    }
}

// Stage a 64-row tile of a [N][d] token tensor into shared memory (fp32, row stride d + 4),
// zero-filling rows past `valid`.
template <typename T>
__device__ __forceinline__ void stage_rows(const T* g, float* s, int d, int valid) {
  const int ds = d + 4, q4 = d / 4;
  for (int e = threadIdx.x; e < kRowTile * q4; e += blockDim.x) {
    const int r = e / q4, c = (e % q4) * 4;
    float4 v = r < valid ? load4(g + (size_t)r * d + c) : make_float4(0.f, 0.f, 0.f, 0.f);
    *reinterpret_cast<float4*>(&s[r * ds + c]) = v;
  }
}

__device__ __forceinline__ void stage_landmarks(const float* Lg, float* Ls, int m, int mpl, int d) {
  const int ds = d + 4;
  for (int e = threadIdx.x; e < mpl * d; e += blockDim.x) {
    const int r = e / d, c = e % d;
    Ls[r * ds + c] = r < m ? Lg[(size_t)r * d + c] : 0.f;
  }
}

// ---------------------------------------------------------------------------------------
// Pass 1: per unit and CTA, sums over its rows of C, C^2, C^T V and V.
// ---------------------------------------------------------------------------------------
template <typename T, int BPT>
__global__ void __launch_bounds__(kThreads) k_pass1(Params p) {
  extern __shared__ float4 smem_f4[];
  float* sm = reinterpret_cast<float*>(smem_f4);
  const int m = p.m, d = p.d, ds = d + 4;
  const int mpl = round_up(m, 64), cs = mpl + 4;
  float* Ls = sm;                    // [mpl][ds]
  float* Qs = Ls + mpl * ds;         // [64][ds]
  float* Vs = Qs + kRowTile * ds;    // [64][ds]
  float* Cs = Vs + kRowTile * ds;    // [64][cs]
  const int u = blockIdx.y, pc = blockIdx.x, t = threadIdx.x;
  const T* Qg = static_cast<const T*>(p.Q) + (size_t)u * p.N * d;
  const T* Vg = static_cast<const T*>(p.V) + (size_t)u * p.N * d;
  stage_landmarks(p.L + (size_t)u * m * d, Ls, m, mpl, d);

  const int nbk = d / 4, nbj = round_up(m, 4) / 4, nb = nbj * nbk;
  float accP[BPT][4][4] = {};
  float s1 = 0.f, s2 = 0.f, sv = 0.f;
  const int tile0 = pc * p.tiles_per_cta;
  const int tile1 = min(tile0 + p.tiles_per_cta, p.n_tiles);
  for (int tile = tile0; tile < tile1; ++tile) {
    const int row0 = tile * kRowTile;
    const int valid = min(kRowTile, p.N - row0);
    __syncthreads();
    stage_rows(Qg + (size_t)row0 * d, Qs, d, valid);
    stage_rows(Vg + (size_t)row0 * d, Vs, d, valid);
    __syncthreads();
    for (int j0 = 0; j0 < mpl; j0 += 64) cross_tile(Qs, Ls, Cs, d, j0, m, cs, p.neg_log2e_over_lam, valid);
    __syncthreads();
    if (t < m) {
      for (int i = 0; i < kRowTile; ++i) {
        const float c = Cs[i * cs + t];
        s1 += c;
        s2 = fmaf(c, c, s2);
      }
    }
    if (t < d) {
      for (int i = 0; i < kRowTile; ++i) sv += Vs[i * ds + t];
    }
#pragma unroll
    for (int q = 0; q < BPT; ++q) {
      const int b = t + q * kThreads;
      if (b < nb) {
        const int jb = b / nbk, kb = b % nbk;
        for (int i = 0; i < kRowTile; ++i) {
          const float4 c = *reinterpret_cast<const float4*>(&Cs[i * cs + 4 * jb]);
          const float4 v = *reinterpret_cast<const float4*>(&Vs[i * ds + 4 * kb]);
          const float cc[4] = {c.x, c.y, c.z, c.w}, vv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
          for (int x = 0; x < 4; ++x)
#pragma unroll
            for (int y = 0; y < 4; ++y) accP[q][x][y] = fmaf(cc[x], vv[y], accP[q][x][y]);
        }
      }
    }
  }
  float* out = p.part + ((size_t)u * p.P + pc) * p.part_stride;
  if (t < m) {
    out[t] = s1;
    out[m + t] = s2;
  }
  if (t < d) out[2 * m + m * d + t] = sv;
#pragma unroll
  for (int q = 0; q < BPT; ++q) {
    const int b = t + q * kThreads;
    if (b < nb) {
      const int jb = b / nbk, kb = b % nbk;
#pragma unroll
      for (int x = 0; x < 4; ++x) {
        const int j = 4 * jb + x;
        if (j < m)
#pragma unroll
          for (int y = 0; y < 4; ++y) out[2 * m + j * d + 4 * kb + y] = accP[q][x][y];
      }
    }
  }
}

// ---------------------------------------------------------------------------------------
// Combine: reduce the pass-1 partials of a unit in fp64.
// ---------------------------------------------------------------------------------------
__global__ void __launch_bounds__(kThreads) k_combine_reduce(Params p) {
  const int u = blockIdx.y;
  const int e = blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= p.part_stride) return;
  double acc = 0.0;
  const float* src = p.part + (size_t)u * p.P * p.part_stride + e;
  for (int pc = 0; pc < p.P; ++pc) acc += (double)src[(size_t)pc * p.part_stride];
  p.red[(size_t)u * p.part_stride + e] = acc;
}

// Batch-pooled statistics (whiten = 2; the note's whitening statistics over a batch of
// similarity vectors, §关键设计 1): for each head and landmark column, the fp64 sums of C and
// C^2 of the B units u = b * heads + h are replaced in every one of them by their mean over b,
// so that the per-unit combine's sum / N becomes the pooled sum / (B N). One thread per (head,
// entry): it reads all B sums before writing any.
__global__ void __launch_bounds__(kThreads) k_pool_batch_stats(Params p) {
  const int h = blockIdx.y, e = blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= 2 * p.m) return;
  double acc = 0.0;
  for (int b = 0; b < p.B; ++b) acc += p.red[(size_t)(b * p.heads + h) * p.part_stride + e];
  acc /= (double)p.B;
  for (int b = 0; b < p.B; ++b) p.red[(size_t)(b * p.heads + h) * p.part_stride + e] = acc;
}

// mu, s, A (all landmarks), then M = X A, M' and bias partials for 16 landmark rows.
__host__ __device__ inline size_t combine_smem(int m, int d) {
  return 2 * sizeof(double) * (size_t)m + sizeof(float) * ((size_t)m * d + 2 * m + 16 * (size_t)m + 16 * (size_t)d);
}
__global__ void __launch_bounds__(kThreads) k_combine_finish(Params p) {
  extern __shared__ float4 smem_f4[];
  const int m = p.m, d = p.d, u = blockIdx.y, c = blockIdx.x, t = threadIdx.x;
  double* mud = reinterpret_cast<double*>(smem_f4);   // [m] fp64 mean and scale, formed once
  double* sd = mud + m;
  float* As = reinterpret_cast<float*>(sd + m);       // [m][d]
  float* mus = As + m * d;      // [m]
  float* ss = mus + m;          // [m]
  const double* red = p.red + (size_t)u * p.part_stride;
  const double invN = 1.0 / double(p.Ng);
  for (int j = t; j < m; j += blockDim.x) {
    const double mu = red[j] * invN;
    double var = red[m + j] * invN - mu * mu;
    if (var < 0.0) var = 0.0;
    const double s = 1.0 / sqrt(var + (double)p.eps);
    mud[j] = mu;
    sd[j] = s;
    mus[j] = (float)mu;
    ss[j] = (float)s;
    if (c == 0) {
      p.mu[(size_t)u * m + j] = (float)mu;
      p.s[(size_t)u * m + j] = (float)s;
    }
  }
  __syncthreads();
  const double* P = red + 2 * m;
  const double* SV = red + 2 * m + m * d;
  // eight entries of A per thread and step, their fp64 loads issued first
  const int md = m * d, nt = blockDim.x;
  for (int e0 = t; e0 < md; e0 += 8 * nt) {
    double pv[8], sv[8];
#pragma unroll
    for (int x = 0; x < 8; ++x) {
      const int e = e0 + x * nt;
      pv[x] = e < md ? __ldg(P + e) : 0.0;
      sv[x] = e < md ? __ldg(SV + e % d) : 0.0;
    }
#pragma unroll
    for (int x = 0; x < 8; ++x) {
      const int e = e0 + x * nt;
      if (e < md) {
        const int j = e / d;
        const double a = p.whiten ? sd[j] * (pv[x] - mud[j] * sv[x]) + sv[x] * invN : pv[x];
        As[e] = (float)a;
        if (c == 0) p.A[(size_t)u * m * d + e] = (float)a;
      }
    }
  }
  __syncthreads();
  // rows [16c, 16c + 16) of M = X A: the rows of X staged in shared memory, four output entries per
  // thread with their sums over l interleaved (each one still in l order); 16 d <= 4 kThreads because
  // the library accepts d = 32 and 64 only
  const float* Xg = p.X + (size_t)u * m * m;
  float* bp = p.bpart + ((size_t)u * p.n_chunks + c) * d;
  const int j0 = c * 16, nj = min(16, m - j0);
  float* Xs = ss + m;        // [16][m]
  float* Ms = Xs + 16 * m;   // [16][d]
  stage_floats(Xs, Xg + (size_t)j0 * m, nj * m, m, m);
  __syncthreads();
  {
    int jj[4], kk[4];
    bool ok[4];
#pragma unroll
    for (int x = 0; x < 4; ++x) {
      const int e = t + kThreads * x;
      jj[x] = e / d;
      kk[x] = e % d;
      ok[x] = e < 16 * d && jj[x] < nj;
    }
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    for (int l = 0; l < m; ++l) {
#pragma unroll
      for (int x = 0; x < 4; ++x)
        if (ok[x]) acc[x] = fmaf(Xs[jj[x] * m + l], As[l * d + kk[x]], acc[x]);
    }
#pragma unroll
    for (int x = 0; x < 4; ++x) {
      if (!ok[x]) continue;
      const int j = j0 + jj[x];
      p.M[((size_t)u * m + j) * d + kk[x]] = acc[x];
      p.Mp[((size_t)u * m + j) * d + kk[x]] = p.whiten ? ss[j] * acc[x] : acc[x];
      Ms[jj[x] * d + kk[x]] = acc[x];
    }
  }
  __syncthreads();
  // bias partial: b[k] = sum_j (1/N - s_j mu_j) M[j][k] over this chunk's rows
  for (int k = t; k < d; k += blockDim.x) {
    float acc = 0.f;
    if (p.whiten) {
      for (int jj = 0; jj < nj; ++jj) {
        const int j = j0 + jj;
        acc += (float)(invN - (double)ss[j] * (double)mus[j]) * Ms[jj * d + k];
      }
    }
    bp[k] = acc;
  }
}

// ---------------------------------------------------------------------------------------
// Reading B (whiten = 3): whitening of the columns of the whole Nystrom matrix
// G^ = C X C^T (LaplacianFormer note, §关键设计 1 applied to §关键设计 2's G^), one column per
// key token j, in factored form. With c- the column mean of C and S = cov(C) (population):
//   mean_i G^_ij = c-^T X c_j,  var_j = c_j^T K c_j with K = X^T S X,
//   O_attn = (C - 1 c-^T) X C^T D^-1/2 V + (1/N) 1 (1^T V),  D = diag(var_j + eps),
// so pass 2 runs unchanged with M' = X C^T D^-1/2 V and b = (1/N) sum_i v_i - M'^T c-.
// Steps: k_rb_gram (C^T C partials, into the tail of the pass-1 partial record, one 64 x 64 block
// pair of landmarks per CTA), the pass-1 reduction, k_rb_cov (S in fp64), K = X^T (S X) by two
// batched products, k_rb_pass (var_j per token with K streamed in 64 x 64 blocks, partials of
// C^T D^-1/2 V), k_rb_reduce, k_rb_finish (M', b). Any m up to the library's maximum.
// ---------------------------------------------------------------------------------------
constexpr int kRbKs = 64 + 4;   // row stride (floats) of a staged 64 x 64 block of K

// Upper-triangle block pair (bj <= bk) number `idx` of an nb x nb grid of 64 x 64 blocks.
__device__ __forceinline__ void block_pair(int idx, int nb, int& bj, int& bk) {
  bj = 0;
  while (idx >= nb - bj) {
    idx -= nb - bj;
    ++bj;
  }
  bk = bj + idx;
}

// C^T C over the CTA's rows (the same row partition as pass 1), one 64 x 64 block pair (bj, bk) per
// blockIdx.z: C is formed for those two landmark blocks only, and thread t owns the 4 x 4 block rows
// 64 bj + 4 (t / 16) .., columns 64 bk + 4 (t % 16) ..; the mirror block is written too.
template <typename T>
__global__ void __launch_bounds__(kThreads) k_rb_gram(Params p) {
  extern __shared__ float4 smem_f4[];
  float* sm = reinterpret_cast<float*>(smem_f4);
  const int m = p.m, d = p.d, ds = d + 4;
  const int mpl = round_up(m, 64), cs = mpl + 4, nb = mpl / 64;
  float* Ls = sm;                    // [mpl][ds]
  float* Qs = Ls + mpl * ds;         // [64][ds]
  float* Cs = Qs + kRowTile * ds;    // [64][cs]
  const int u = blockIdx.y, pc = blockIdx.x, t = threadIdx.x, jb = t >> 4, kb = t & 15;
  int bj, bk;
  block_pair(blockIdx.z, nb, bj, bk);
  const T* Qg = static_cast<const T*>(p.Q) + (size_t)u * p.N * d;
  stage_landmarks(p.L + (size_t)u * m * d, Ls, m, mpl, d);
  float acc[4][4] = {};
  const int tile0 = pc * p.tiles_per_cta;
  const int tile1 = min(tile0 + p.tiles_per_cta, p.n_tiles);
  for (int tile = tile0; tile < tile1; ++tile) {
    const int row0 = tile * kRowTile;
    const int valid = min(kRowTile, p.N - row0);
    __syncthreads();
    stage_rows(Qg + (size_t)row0 * d, Qs, d, valid);
    __syncthreads();
    cross_tile(Qs, Ls, Cs, d, 64 * bj, m, cs, p.neg_log2e_over_lam, valid);
    if (bk != bj) cross_tile(Qs, Ls, Cs, d, 64 * bk, m, cs, p.neg_log2e_over_lam, valid);
    __syncthreads();
    for (int i = 0; i < kRowTile; ++i) {
      const float4 a = *reinterpret_cast<const float4*>(&Cs[i * cs + 64 * bj + 4 * jb]);
      const float4 b = *reinterpret_cast<const float4*>(&Cs[i * cs + 64 * bk + 4 * kb]);
      const float av[4] = {a.x, a.y, a.z, a.w}, bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
      for (int x = 0; x < 4; ++x)
#pragma unroll
        for (int y = 0; y < 4; ++y) acc[x][y] = fmaf(av[x], bv[y], acc[x][y]);
    }
  }
  float* out = p.part + ((size_t)u * p.P + pc) * p.part_stride + (2 * m + m * d + d);
#pragma unroll
  for (int x = 0; x < 4; ++x)
#pragma unroll
    for (int y = 0; y < 4; ++y) {
      const int j = 64 * bj + 4 * jb + x, k = 64 * bk + 4 * kb + y;
      if (j < m && k < m) {
        out[j * m + k] = acc[x][y];
        if (bk != bj) out[k * m + j] = acc[x][y];
      }
    }
}

// S = C^T C / N - c- c-^T (fp64 from the reduced sums) into Y; mu = c-, s = 1 for inspection.
__global__ void __launch_bounds__(kThreads) k_rb_cov(Params p) {
  const int u = blockIdx.y, e = blockIdx.x * blockDim.x + threadIdx.x, m = p.m;
  if (e >= m * m) return;
  const double* red = p.red + (size_t)u * p.part_stride;
  const double invN = 1.0 / double(p.Ng);
  const int j = e / m, k = e % m;
  const double cj = red[j] * invN, ck = red[k] * invN;
  p.Y[(size_t)u * m * m + e] = (float)(red[2 * m + m * p.d + p.d + e] * invN - cj * ck);
  if (e < m) {
    p.mu[(size_t)u * m + e] = (float)(red[e] * invN);
    p.s[(size_t)u * m + e] = 1.f;
  }
}

// Per 64-row tile: C (all landmarks), var_i = c_i^T K c_i by a blocked product C K (K streamed in
// 64 x 64 blocks through shared memory; thread (t / 16, t % 16) owns a 4 x 4 block of each output
// block and keeps its share of sum_k C_ik (C K)_ik), w_i = 1 / sqrt(var_i + eps) (0 past the end), and
// C^T (w o V) into the P slot of the CTA's partial record (pass 1's records are already reduced):
// thread (t / (d / 4), t % (d / 4)) owns a 4 x 4 block of every 64-landmark block of the m x d sum.
template <typename T>
__global__ void __launch_bounds__(kThreads) k_rb_pass(Params p) {
  extern __shared__ float4 smem_f4[];
  float* sm = reinterpret_cast<float*>(smem_f4);
  const int m = p.m, d = p.d, ds = d + 4;
  const int mpl = round_up(m, 64), cs = mpl + 4, nb = mpl / 64;
  float* Ls = sm;                    // [mpl][ds]
  float* Qs = Ls + mpl * ds;         // [64][ds]
  float* Vs = Qs + kRowTile * ds;    // [64][ds]
  float* Cs = Vs + kRowTile * ds;    // [64][cs]
  float* Ks = Cs + kRowTile * cs;    // [64][kRbKs] one block of K
  float* wr = Ks + 64 * kRbKs;       // [64]
  const int u = blockIdx.y, pc = blockIdx.x, t = threadIdx.x;
  const T* Qg = static_cast<const T*>(p.Q) + (size_t)u * p.N * d;
  const T* Vg = static_cast<const T*>(p.V) + (size_t)u * p.N * d;
  const float* Kg = p.Y + (size_t)u * m * m;
  stage_landmarks(p.L + (size_t)u * m * d, Ls, m, mpl, d);
  const int ib = t >> 4, kk = t & 15;                     // C K blocks
  const int nbk = d / 4, nt = 16 * nbk;                   // C^T (w o V) blocks
  const int jb2 = t / nbk, kb2 = t % nbk;
  float acc2[4][4][4];
#pragma unroll
  for (int b = 0; b < 4; ++b)
#pragma unroll
    for (int x = 0; x < 4; ++x)
#pragma unroll
      for (int y = 0; y < 4; ++y) acc2[b][x][y] = 0.f;
  const int tile0 = pc * p.tiles_per_cta;
  const int tile1 = min(tile0 + p.tiles_per_cta, p.n_tiles);
  for (int tile = tile0; tile < tile1; ++tile) {
    const int row0 = tile * kRowTile;
    const int valid = min(kRowTile, p.N - row0);
    __syncthreads();
    stage_rows(Qg + (size_t)row0 * d, Qs, d, valid);
    stage_rows(Vg + (size_t)row0 * d, Vs, d, valid);
    __syncthreads();
    for (int j0 = 0; j0 < mpl; j0 += 64) cross_tile(Qs, Ls, Cs, d, j0, m, cs, p.neg_log2e_over_lam, valid);
    float vp[4] = {0.f, 0.f, 0.f, 0.f};
    for (int kbk = 0; kbk < nb; ++kbk) {
      float acc[4][4] = {};
      for (int jbk = 0; jbk < nb; ++jbk) {
        __syncthreads();   // C is complete; the previous K block is no longer read
        for (int e = t; e < 64 * 64; e += blockDim.x) {
          const int j = e >> 6, k = e & 63, gj = 64 * jbk + j, gk = 64 * kbk + k;
          Ks[j * kRbKs + k] = (gj < m && gk < m) ? Kg[(size_t)gj * m + gk] : 0.f;
        }
        __syncthreads();
        for (int j = 0; j < 64; ++j) {
          const float4 b = *reinterpret_cast<const float4*>(&Ks[j * kRbKs + 4 * kk]);
          const float bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
          for (int x = 0; x < 4; ++x) {
            const float a = Cs[(4 * ib + x) * cs + 64 * jbk + j];
#pragma unroll
            for (int y = 0; y < 4; ++y) acc[x][y] = fmaf(a, bv[y], acc[x][y]);
          }
        }
      }
#pragma unroll
      for (int x = 0; x < 4; ++x)
#pragma unroll
        for (int y = 0; y < 4; ++y) vp[x] = fmaf(Cs[(4 * ib + x) * cs + 64 * kbk + 4 * kk + y], acc[x][y], vp[x]);
    }
    // rows 4 ib .. are shared by the 16 threads with the same ib (consecutive lanes)
#pragma unroll
    for (int x = 0; x < 4; ++x)
      for (int o = 8; o > 0; o >>= 1) vp[x] += __shfl_xor_sync(0xffffffffu, vp[x], o);
    if (kk == 0) {
#pragma unroll
      for (int x = 0; x < 4; ++x) {
        const int i = 4 * ib + x;
        wr[i] = i < valid ? 1.f / sqrtf(vp[x] + p.eps) : 0.f;
      }
    }
    __syncthreads();
    for (int e = t; e < kRowTile * d; e += blockDim.x) {
      const int i = e / d, c = e % d;
      Vs[i * ds + c] *= wr[i];
    }
    __syncthreads();
    if (t < nt) {
      for (int i = 0; i < kRowTile; ++i) {
        const float4 v = *reinterpret_cast<const float4*>(&Vs[i * ds + 4 * kb2]);
        const float vv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int b = 0; b < 4; ++b) {
          if (b >= nb) break;
          const float4 c = *reinterpret_cast<const float4*>(&Cs[i * cs + 64 * b + 4 * jb2]);
          const float cc[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
          for (int x = 0; x < 4; ++x)
#pragma unroll
            for (int y = 0; y < 4; ++y) acc2[b][x][y] = fmaf(cc[x], vv[y], acc2[b][x][y]);
        }
      }
    }
  }
  if (t < nt) {
    float* out = p.part + ((size_t)u * p.P + pc) * p.part_stride + 2 * m;
#pragma unroll
    for (int b = 0; b < 4; ++b) {
      if (b >= nb) break;
#pragma unroll
      for (int x = 0; x < 4; ++x) {
        const int j = 64 * b + 4 * jb2 + x;
        if (j < m)
#pragma unroll
          for (int y = 0; y < 4; ++y) out[j * d + 4 * kb2 + y] = acc2[b][x][y];
      }
    }
  }
}

// A = C^T D^-1/2 V: the partials' P slots summed in fp64.
__global__ void __launch_bounds__(kThreads) k_rb_reduce(Params p) {
  const int u = blockIdx.y, e = blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= p.m * p.d) return;
  double acc = 0.0;
  const float* src = p.part + (size_t)u * p.P * p.part_stride + 2 * p.m + e;
  for (int pc = 0; pc < p.P; ++pc) acc += (double)src[(size_t)pc * p.part_stride];
  p.A[(size_t)u * p.m * p.d + e] = (float)acc;
}

// Rows [16c, 16c + 16) of M' = X A, and the bias partial -sum_j c-_j M'[j][k] over them; chunk 0
// adds (1/N) sum_i v_ik.
__global__ void __launch_bounds__(kThreads) k_rb_finish(Params p) {
  extern __shared__ float4 smem_f4[];
  float* As = reinterpret_cast<float*>(smem_f4);   // [m][d]
  const int m = p.m, d = p.d, u = blockIdx.y, c = blockIdx.x, t = threadIdx.x;
  for (int e = t; e < m * d; e += blockDim.x) As[e] = p.A[(size_t)u * m * d + e];
  __syncthreads();
  const double* red = p.red + (size_t)u * p.part_stride;
  const double invN = 1.0 / double(p.Ng);
  const float* Xg = p.X + (size_t)u * m * m;
  const int j0 = c * 16;
  for (int e = t; e < 16 * d; e += blockDim.x) {
    const int j = j0 + e / d, k = e % d;
    if (j < m) {
      float acc = 0.f;
      for (int l = 0; l < m; ++l) acc = fmaf(Xg[(size_t)j * m + l], As[l * d + k], acc);
      p.M[((size_t)u * m + j) * d + k] = acc;
      p.Mp[((size_t)u * m + j) * d + k] = acc;
    }
  }
  __syncthreads();
  float* bp = p.bpart + ((size_t)u * p.n_chunks + c) * d;
  for (int k = t; k < d; k += blockDim.x) {
    double acc = c == 0 ? red[2 * m + m * d + k] * invN : 0.0;
    for (int jj = 0; jj < 16; ++jj) {
      const int j = j0 + jj;
      if (j < m) acc -= red[j] * invN * (double)p.M[((size_t)u * m + j) * d + k];
    }
    bp[k] = (float)acc;
  }
}

// ---------------------------------------------------------------------------------------
// Pass 2: O = C M' + 1 b^T + DWC(V) over the CTA's 64-row tiles (the same row partition as
// pass 1); L and M' are staged once per CTA.
// ---------------------------------------------------------------------------------------
template <typename T>
__global__ void __launch_bounds__(kThreads) k_pass2(Params p) {
  extern __shared__ float4 smem_f4[];
  float* sm = reinterpret_cast<float*>(smem_f4);
  const int m = p.m, d = p.d, ds = d + 4;
  const int mpl = round_up(m, 64), cs = mpl + 4, m4 = round_up(m, 4);
  float* Ls = sm;                    // [mpl][ds]
  float* Ms = Ls + mpl * ds;         // [m4][ds] M'
  float* Qs = Ms + m4 * ds;          // [64][ds]
  float* Cs = Qs + kRowTile * ds;    // [64][cs]
  float* bs = Cs + kRowTile * cs;    // [d]
  const int u = blockIdx.y, pc = blockIdx.x, t = threadIdx.x;
  const T* Qg = static_cast<const T*>(p.Q) + (size_t)u * p.N * d;
  const T* Vg = static_cast<const T*>(p.V) + (size_t)u * p.N * d;
  stage_landmarks(p.L + (size_t)u * m * d, Ls, m, mpl, d);
  stage_landmarks(p.Mp + (size_t)u * m * d, Ms, m, m4, d);
  if (t < d) {
    float b = 0.f;
    for (int c = 0; c < p.n_chunks; ++c) b += p.bpart[((size_t)u * p.n_chunks + c) * d + t];
    bs[t] = b;
  }
  const int nbk = d / 4;
  const int ib = t / nbk, kb = t % nbk;
  const bool mapped = t < 16 * nbk;
  // DWC weights of this thread's 4 channels: w[h][k][a][b] multiplies V[y + a - 1][x + b - 1][k]
  const int h = u % p.heads;
  float wt[4][9];
#pragma unroll
  for (int y = 0; y < 4; ++y)
#pragma unroll
    for (int e = 0; e < 9; ++e) wt[y][e] = mapped ? p.dwc[((size_t)h * d + 4 * kb + y) * 9 + e] : 0.f;
  T* Og = static_cast<T*>(p.O) + (size_t)u * p.N * d;
  const int tile0 = pc * p.tiles_per_cta;
  const int tile1 = min(tile0 + p.tiles_per_cta, p.n_tiles);
  for (int tile = tile0; tile < tile1; ++tile) {
    const int row0 = tile * kRowTile, valid = min(kRowTile, p.N - row0);
    __syncthreads();   // the previous tile's readers of Qs and Cs are done
    stage_rows(Qg + (size_t)row0 * d, Qs, d, valid);
    __syncthreads();
    for (int j0 = 0; j0 < mpl; j0 += 64) cross_tile(Qs, Ls, Cs, d, j0, m, cs, p.neg_log2e_over_lam, valid);
    __syncthreads();
    if (mapped) {
      float acc[4][4] = {};
      for (int j = 0; j < m4; j += 4) {
        float4 c[4], mp[4];
#pragma unroll
        for (int x = 0; x < 4; ++x) c[x] = *reinterpret_cast<const float4*>(&Cs[(4 * ib + x) * cs + j]);
#pragma unroll
        for (int y = 0; y < 4; ++y) mp[y] = *reinterpret_cast<const float4*>(&Ms[(j + y) * ds + 4 * kb]);
#pragma unroll
        for (int x = 0; x < 4; ++x) {
          const float cc[4] = {c[x].x, c[x].y, c[x].z, c[x].w};
#pragma unroll
          for (int y = 0; y < 4; ++y) {
            acc[x][0] = fmaf(cc[y], mp[y].x, acc[x][0]);
            acc[x][1] = fmaf(cc[y], mp[y].y, acc[x][1]);
            acc[x][2] = fmaf(cc[y], mp[y].z, acc[x][2]);
            acc[x][3] = fmaf(cc[y], mp[y].w, acc[x][3]);
          }
        }
      }
#pragma unroll
      for (int x = 0; x < 4; ++x) {
        const int i = 4 * ib + x;
        if (i >= valid) continue;
        const int n = row0 + i, gy = n / p.W, gx = n % p.W;
        float o[4] = {acc[x][0] + bs[4 * kb], acc[x][1] + bs[4 * kb + 1], acc[x][2] + bs[4 * kb + 2],
                      acc[x][3] + bs[4 * kb + 3]};
#pragma unroll
        for (int a = 0; a < 3; ++a) {
          // local row yy, global row p.y0 + yy; the rows just outside a band come from the halo
          const int yy = gy + a - 1, yg = p.y0 + yy;
          if (yg < 0 || yg >= p.Hg) continue;
          const T* vrow = (yy >= 0 && yy < p.H)
                              ? Vg + (size_t)yy * p.W * d
                              : static_cast<const T*>(p.Vh) + ((size_t)u * 2 + (yy < 0 ? 0 : 1)) * p.W * d;
#pragma unroll
          for (int b = 0; b < 3; ++b) {
            const int xx = gx + b - 1;
            if (xx < 0 || xx >= p.W) continue;
            const float4 v = load4(vrow + (size_t)xx * d + 4 * kb);
            o[0] = fmaf(wt[0][a * 3 + b], v.x, o[0]);
            o[1] = fmaf(wt[1][a * 3 + b], v.y, o[1]);
            o[2] = fmaf(wt[2][a * 3 + b], v.z, o[2]);
            o[3] = fmaf(wt[3][a * 3 + b], v.w, o[3]);
          }
        }
        store4(Og + (size_t)n * d + 4 * kb, make_float4(o[0], o[1], o[2], o[3]));
      }
    }
  }
}

// C of one unit, [N][m] fp32, from the same tile code as the passes.
template <typename T>
__global__ void __launch_bounds__(kThreads) k_cross_out(Params p, int u, float* C_out) {
  extern __shared__ float4 smem_f4[];
  float* sm = reinterpret_cast<float*>(smem_f4);
  const int m = p.m, d = p.d, ds = d + 4;
  const int mpl = round_up(m, 64), cs = mpl + 4;
  float* Ls = sm;
  float* Qs = Ls + mpl * ds;
  float* Cs = Qs + kRowTile * ds;
  const int row0 = blockIdx.x * kRowTile, valid = min(kRowTile, p.N - row0);
  const T* Qg = static_cast<const T*>(p.Q) + (size_t)u * p.N * d;
  stage_landmarks(p.L + (size_t)u * m * d, Ls, m, mpl, d);
  stage_rows(Qg + (size_t)row0 * d, Qs, d, valid);
  __syncthreads();
  for (int j0 = 0; j0 < mpl; j0 += 64) cross_tile(Qs, Ls, Cs, d, j0, m, cs, p.neg_log2e_over_lam, valid);
  __syncthreads();
  for (int e = threadIdx.x; e < valid * m; e += blockDim.x) {
    const int i = e / m, j = e % m;
    C_out[(size_t)(row0 + i) * m + j] = Cs[i * cs + j];
  }
}

// Pass 1 over the tokens (sums of C, C^2, C^T V and V per CTA) and their fp64 reduction
// into p.red. With p.V pointing at another [N][d] tensor (dO) the same code forms C^T dO.
template <typename T>
void pass1_t(const Params& p, cudaStream_t st) {
  const int U = p.U, m = p.m, d = p.d;
  const int bpt = ceil_div((round_up(m, 4) / 4) * (d / 4), kThreads);
  const dim3 g1(p.P, U);
  const size_t s1 = generic_smem_pass1(m, d);
  if (bpt <= 1) k_pass1<T, 1><<<g1, kThreads, s1, st>>>(p);
  else if (bpt <= 2) k_pass1<T, 2><<<g1, kThreads, s1, st>>>(p);
  else k_pass1<T, 4><<<g1, kThreads, s1, st>>>(p);
}

// (bf16 tokens with d = 64 take the tcgen05 streaming pass, whose partial records come with their own
// count per unit)
template <typename T>
void pass1_reduce_t(const Params& p, cudaStream_t st) {
  Params q = p;
  const int P = stream_pass1(p, st);
  if (P > 0) q.P = P;
  else pass1_t<T>(p, st);
  k_combine_reduce<<<dim3(ceil_div(q.part_stride, kThreads), q.U), kThreads, 0, st>>>(q);
}

// pass 2: the tcgen05 streaming kernel for bf16 tokens with d = 64, else the CUDA-core one
template <typename T>
void pass2_t(const Params& p, cudaStream_t st) {
  if (!stream_pass2(p, st)) k_pass2<T><<<dim3(p.P, p.U), kThreads, generic_smem_pass2(p.m, p.d), st>>>(p);
}

size_t rb_gram_smem(int m, int d) {
  const int mpl = round_up(m, 64);
  return sizeof(float) * ((size_t)mpl * (d + 4) + 64 * (d + 4) + 64 * (size_t)(mpl + 4));
}
size_t rb_pass_smem(int m, int d) {
  const int mpl = round_up(m, 64);
  return sizeof(float) * ((size_t)mpl * (d + 4) + 2 * 64 * (d + 4) + 64 * (size_t)(mpl + 4) + 64 * kRbKs + 64);
}

// Reading B after the Newton-Schulz chain (the Y / Xb buffers are free once X is in p.X): every stage
// up to M' and b.
template <typename T>
void reading_b_t(const Params& p, cudaStream_t st) {
  const int U = p.U, m = p.m, d = p.d;
  const size_t mm = (size_t)m * m;
  pass1_t<T>(p, st);
  const int nb = round_up(m, 64) / 64;
  k_rb_gram<T><<<dim3(p.P, U, nb * (nb + 1) / 2), kThreads, rb_gram_smem(m, d), st>>>(p);
  k_combine_reduce<<<dim3(ceil_div(p.part_stride, kThreads), U), kThreads, 0, st>>>(p);
  k_rb_cov<<<dim3(ceil_div(m * m, kThreads), U), kThreads, 0, st>>>(p);
  const MmJob sx{p.Y, mm, p.X, mm, nullptr, 0, p.Xb, mm, 1.f, 0.f, 0.f, 0, 0};   // Xb = S X
  launch_mm(&sx, 1, m, U, st, p.status);
  const MmJob k{p.X, mm, p.Xb, mm, nullptr, 0, p.Y, mm, 1.f, 0.f, 0.f, 1, 0};     // Y = X^T (S X)
  launch_mm(&k, 1, m, U, st, p.status);
  k_rb_pass<T><<<dim3(p.P, U), kThreads, rb_pass_smem(m, d), st>>>(p);
  k_rb_reduce<<<dim3(ceil_div(m * d, kThreads), U), kThreads, 0, st>>>(p);
  k_rb_finish<<<dim3(p.n_chunks, U), kThreads, sizeof(float) * (size_t)m * d, st>>>(p);
}

// alpha (power iteration and the fallback rule) and X_0 = alpha W^T in p.X, from W in p.Wm
void ns_alpha(const Params& p, cudaStream_t st) {
  k_alpha<<<p.U, kAlphaThreads, sizeof(float) * (size_t)alpha_rows(p.m) * p.m, st>>>(p);
}

// the T Newton-Schulz steps X <- X (2I - W X) from X_0 in p.X as tcgen05 products (p.Y and p.Xb are
// scratch); X_T ends in p.X.
void ns_steps(const Params& p, cudaStream_t st) {
  const int U = p.U, m = p.m;
  float* x = p.X;
  float* xb = p.Xb;
  const size_t mm = (size_t)m * m;
  const NsChain c{p.Wm, mm, p.Y, mm, p.X, p.Xb, mm, 0, m, p.T, 0, p.status};
  if (launch_ns_chain(c, U, st)) {
    if (p.T & 1) { x = p.Xb; xb = p.X; }
  } else for (int k = 0; k < p.T; ++k) {
    const MmJob y{p.Wm, mm, x, mm, nullptr, 0, p.Y, mm, -1.f, 0.f, 2.f, 0, 0};   // Y = 2I - W X
    launch_mm(&y, 1, m, U, st, p.status);
    const MmJob xn{x, mm, p.Y, mm, nullptr, 0, xb, mm, 1.f, 0.f, 0.f, 0, 0};     // X' = X Y
    launch_mm(&xn, 1, m, U, st, p.status);
    float* tmp = x; x = xb; xb = tmp;
  }
  if (x != p.X) cudaMemcpyAsync(p.X, x, sizeof(float) * (size_t)U * m * m, cudaMemcpyDeviceToDevice, st);
}

// the closing residual ||I - W X_T||_F of each unit into its info record (p.Y is scratch)
void ns_residual(const Params& p, cudaStream_t st) {
  const int U = p.U, m = p.m;
  const dim3 g(ceil_div(m, 64), ceil_div(m, 64), U);
  k_ns_gemm<<<g, kThreads, 0, st>>>(p, p.Wm, p.X, p.Y, -1.f, 1.f, 1);  // I - W X, ||.||_F^2
  k_residual_sqrt<<<ceil_div(U, 128), 128, 0, st>>>(p);
}

void ns_from_w(const Params& p, cudaStream_t st) {
  ns_alpha(p, st);
  ns_steps(p, st);
  ns_residual(p, st);
}

// W, alpha and the Newton-Schulz chain from the landmarks in the workspace (X_T in p.X); the closing
// residual too unless with_residual is false (m > 64 only: the m <= 64 kernel always forms it).
void ns_t(const Params& p, cudaStream_t st, bool with_residual = true) {
  const int U = p.U, m = p.m;
  if (m <= kSmallM) {
    launch_ns_tc(p, st);
  } else {
    k_gram<<<dim3(ceil_div(m, 16), U), kThreads, sizeof(float) * (size_t)m * (p.d + 1), st>>>(p);
    if (with_residual) {
      ns_from_w(p, st);
    } else {
      ns_alpha(p, st);
      ns_steps(p, st);
    }
  }
}

// The chain-first schedule of context_t. Pass 1 (one block per SM) dispatched first leaves no whole
// group of SMs for the chain's clusters, so the two would run one after the other. Chain first: W and
// alpha before the fork, then the chain's U clusters of G blocks, and pass 1 beside it on the pa blocks
// per unit that the clusters leave, over the first ta tiles of each unit: as many as those blocks finish
// in about the chain's time. The other tiles, if any, run after the chain on pb blocks per unit (every
// SM). pa = 0: the concurrent order instead. Estimates: 2T chain products of about 9.5 us; a 64-token
// tile about 16 us per block at 256 landmark columns and d = 64, in proportion to both. Worth it when
// the chain takes longer than W and alpha (about 0.1 ms at m = 256) by a margin.
struct ChainFirst {
  int pa, ta, pb;
};

ChainFirst chain_first_plan(const Params& p, bool check_maps = true) {
  ChainFirst cf{0, 0, 0};
  if (p.m <= kSmallM || p.T <= 0 || !stream_eligible(p) || !ns_chain_fits(p.m)) return cf;
  if (check_maps && !stream_maps_ok(p)) return cf;
  if (!(p.aux_stream && p.ev_fork && p.ev_mid && p.ev_x && p.ev_join)) return cf;
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return cf;
  const int pa = std::min((sms - p.U * ns_chain_blocks(p.m)) / p.U, p.P);
  const double t_chain = 2.0 * p.T * 9.5e-6;
  if (pa < 1 || t_chain < 150e-6) return cf;
  const double t_tile = 16e-6 * (double)((p.m + 63) / 64) / 4.0 * ((double)p.d / 64.0);
  const int n = stream_tiles(p);
  const int ta = std::min(n, pa * std::max(1, (int)(t_chain / t_tile)));
  int pb = 0;
  if (ta < n) {
    pb = std::min(std::max(sms / p.U, 1), p.P - stream_range_blocks(0, ta, pa));
    if (pb < 1) return cf;
  }
  cf.pa = pa;
  cf.ta = ta;
  cf.pb = pb;
  return cf;
}

// Every forward stage before pass 2: L, W, alpha, X, the column statistics, A, M, M', b. The
// Newton-Schulz chain (W, alpha, X) and pass 1 (the column sums, C^T V) share no data: with an
// auxiliary stream they run concurrently, joined before the combine, in the chain-first schedule
// (chain_first_plan) where it applies. The closing residual of the chain (m > 64) only reports: it
// runs on the auxiliary stream beside the combine, joined after it.
template <typename T>
void context_t(const Params& p, cudaStream_t st) {
  const int U = p.U, m = p.m, d = p.d;
  k_pool<T><<<dim3(ceil_div(m, kThreads / 32), U), kThreads, 0, st>>>(p);
  if (p.whiten == 3) {
    ns_t(p, st);
    reading_b_t<T>(p, st);
    return;
  }
  auto pass1 = [&](cudaStream_t s) {
    pass1_reduce_t<T>(p, s);
    if (p.whiten == 2) k_pool_batch_stats<<<dim3(ceil_div(2 * m, kThreads), p.heads), kThreads, 0, s>>>(p);
  };
  auto combine = [&](cudaStream_t s) {
    k_combine_finish<<<dim3(p.n_chunks, U), kThreads, combine_smem(m, d), s>>>(p);
  };
  const ChainFirst cf = chain_first_plan(p);
  if (cf.pa > 0) {
    // main: W, alpha, the chain, the tiles after ta (if any) on every SM, then the combine; auxiliary:
    // pass 1 over the first ta tiles on pa blocks per unit once alpha is done, then the residual once X_T
    // (and the main stream's pass-1 tiles) are. The records are reduced after the last pass-1 launch.
    cudaStream_t aux = static_cast<cudaStream_t>(p.aux_stream);
    const int n = stream_tiles(p);
    const int ra = stream_range_blocks(0, cf.ta, cf.pa), rb = stream_range_blocks(cf.ta, n, cf.pb);
    Params q = p;
    q.P = ra + rb;   // the records of both launches, per unit
    auto reduce = [&](cudaStream_t s) {
      k_combine_reduce<<<dim3(ceil_div(q.part_stride, kThreads), q.U), kThreads, 0, s>>>(q);
      if (p.whiten == 2) k_pool_batch_stats<<<dim3(ceil_div(2 * m, kThreads), p.heads), kThreads, 0, s>>>(p);
    };
    k_gram<<<dim3(ceil_div(m, 16), U), kThreads, sizeof(float) * (size_t)m * (p.d + 1), st>>>(p);
    ns_alpha(p, st);
    cudaEventRecord(static_cast<cudaEvent_t>(p.ev_fork), st);
    ns_steps(p, st);
    if (rb > 0) stream_pass1_range(p, cf.ta, n, cf.pb, ra, q.P, st);
    cudaEventRecord(static_cast<cudaEvent_t>(p.ev_x), st);
    cudaStreamWaitEvent(aux, static_cast<cudaEvent_t>(p.ev_fork), 0);
    stream_pass1_range(p, 0, cf.ta, cf.pa, 0, q.P, aux);
    if (rb == 0) reduce(aux);
    cudaEventRecord(static_cast<cudaEvent_t>(p.ev_mid), aux);
    cudaStreamWaitEvent(aux, static_cast<cudaEvent_t>(p.ev_x), 0);
    ns_residual(p, aux);
    cudaEventRecord(static_cast<cudaEvent_t>(p.ev_join), aux);
    cudaStreamWaitEvent(st, static_cast<cudaEvent_t>(p.ev_mid), 0);
    if (rb > 0) reduce(st);
    combine(st);
    cudaStreamWaitEvent(st, static_cast<cudaEvent_t>(p.ev_join), 0);
    return;
  }
  if (m > kSmallM && p.aux_stream && p.ev_fork && p.ev_mid && p.ev_join) {
    cudaStream_t aux = static_cast<cudaStream_t>(p.aux_stream);
    cudaEventRecord(static_cast<cudaEvent_t>(p.ev_fork), st);
    cudaStreamWaitEvent(aux, static_cast<cudaEvent_t>(p.ev_fork), 0);
    ns_t(p, aux, false);
    cudaEventRecord(static_cast<cudaEvent_t>(p.ev_mid), aux);
    ns_residual(p, aux);
    cudaEventRecord(static_cast<cudaEvent_t>(p.ev_join), aux);
    pass1(st);
    cudaStreamWaitEvent(st, static_cast<cudaEvent_t>(p.ev_mid), 0);
    combine(st);
    cudaStreamWaitEvent(st, static_cast<cudaEvent_t>(p.ev_join), 0);
    return;
  }
  fork_join(p, st, pass1, [&](cudaStream_t s) { ns_t(p, s); });
  combine(st);
}

template <typename T>
cudaError_t forward_t(const Params& p, cudaStream_t st) {
  context_t<T>(p, st);
  if (p.ev_begin) cudaEventRecord(static_cast<cudaEvent_t>(p.ev_begin), st);
  pass2_t<T>(p, st);
  if (p.ev_end) cudaEventRecord(static_cast<cudaEvent_t>(p.ev_end), st);
  return cudaGetLastError();
}

}  // namespace

size_t generic_smem_pass1(int m, int d) {
  const int mpl = round_up(m, 64), ds = d + 4;
  return sizeof(float) * ((size_t)mpl * ds + 2 * kRowTile * ds + (size_t)kRowTile * (mpl + 4));
}

size_t generic_smem_pass2(int m, int d) {
  const int mpl = round_up(m, 64), ds = d + 4, m4 = round_up(m, 4);
  return sizeof(float) * ((size_t)mpl * ds + (size_t)m4 * ds + kRowTile * ds + (size_t)kRowTile * (mpl + 4) + d);
}

cudaError_t generic_set_attributes() {
  const int big = 227 * 1024;
  cudaError_t e = cudaSuccess;
#define LFA_ATTR(fn) \
  if (e == cudaSuccess) e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, big)
  LFA_ATTR((k_pass1<float, 1>));
  LFA_ATTR((k_pass1<float, 2>));
  LFA_ATTR((k_pass1<float, 4>));
  LFA_ATTR((k_pass1<__nv_bfloat16, 1>));
  LFA_ATTR((k_pass1<__nv_bfloat16, 2>));
  LFA_ATTR((k_pass1<__nv_bfloat16, 4>));
  LFA_ATTR(k_combine_finish);
  LFA_ATTR(k_gram);
  LFA_ATTR(k_rb_finish);
  LFA_ATTR(k_rb_gram<float>);
  LFA_ATTR(k_rb_gram<__nv_bfloat16>);
  LFA_ATTR(k_rb_pass<float>);
  LFA_ATTR(k_rb_pass<__nv_bfloat16>);
  LFA_ATTR(k_pass2<float>);
  LFA_ATTR(k_pass2<__nv_bfloat16>);
  LFA_ATTR(k_cross_out<float>);
  LFA_ATTR(k_cross_out<__nv_bfloat16>);
#undef LFA_ATTR
  // k_alpha also has static shared memory: its dynamic part stays below the per-block limit
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(k_alpha, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)(sizeof(float) * (size_t)alpha_rows(kMaxM) * kMaxM));
  return e;
}

int generic_launch_count(const Params& p) {
  // pool, Newton-Schulz chain, pass 1 (two launches when the chain-first schedule splits it), two
  // combine kernels (three with batch-pooled statistics), pass 2; the chain for m > 64 is gram, alpha,
  // the steps (one cluster launch, or two per step), the residual product and its square root
  const int ns = p.m <= kSmallM ? 1 : 2 + (p.T > 0 ? (ns_chain_fits(p.m) ? 1 : 2 * p.T) : 0) + 2;
  // Reading B: pass 1, C^T C, reduction, covariance, two products, token pass, reduction, finish
  if (p.whiten == 3) return 1 + ns + 9 + 1;
  const int split = chain_first_plan(p, false).pb > 0 ? 1 : 0;
  return 1 + ns + 1 + split + 2 + (p.whiten == 2 ? 1 : 0) + 1;
}

cudaError_t launch_generic_forward(const Params& p, cudaStream_t st) {
  return p.dtype == LFA_BF16 ? forward_t<__nv_bfloat16>(p, st) : forward_t<float>(p, st);
}

cudaError_t launch_generic_context(const Params& p, cudaStream_t st) {
  if (p.dtype == LFA_BF16) context_t<__nv_bfloat16>(p, st);
  else context_t<float>(p, st);
  return cudaGetLastError();
}

cudaError_t launch_generic_pass1_reduce(const Params& p, cudaStream_t st) {
  if (p.dtype == LFA_BF16) pass1_reduce_t<__nv_bfloat16>(p, st);
  else pass1_reduce_t<float>(p, st);
  return cudaGetLastError();
}

cudaError_t launch_generic_ns(const Params& p, cudaStream_t st) {
  ns_t(p, st);
  return cudaGetLastError();
}

cudaError_t launch_ns_from_w(const Params& p, cudaStream_t st) {
  ns_from_w(p, st);
  return cudaGetLastError();
}

// The combine from the fp64 totals in the workspace (mu, s, A, M, M', b), then pass 2.
cudaError_t launch_generic_finish(const Params& p, cudaStream_t st) {
  k_combine_finish<<<dim3(p.n_chunks, p.U), kThreads, combine_smem(p.m, p.d), st>>>(p);
  if (p.dtype == LFA_BF16) pass2_t<__nv_bfloat16>(p, st);
  else pass2_t<float>(p, st);
  return cudaGetLastError();
}

cudaError_t launch_pool(const Params& p, cudaStream_t st) {
  const dim3 g(ceil_div(p.m, kThreads / 32), p.U);
  if (p.dtype == LFA_BF16) k_pool<__nv_bfloat16><<<g, kThreads, 0, st>>>(p);
  else k_pool<float><<<g, kThreads, 0, st>>>(p);
  return cudaGetLastError();
}

// Condition number estimate of W + eps I for lfa_get_info (not part of the forward): ||X_T||_2 by
// power iteration on X_T, which approximates (W + eps I)^-1 (symmetric positive definite) once the
// Newton-Schulz chain has converged, times the forward's lambda_max = ||W||_2, i.e. lambda_max /
// lambda_min. One CTA of 256 threads per unit, a warp per matrix row, kKappaIters normalised steps
// from the ones vector and a final Rayleigh quotient.
constexpr int kKappaIters = 48;
__global__ void __launch_bounds__(kThreads) k_kappa(Params p) {
  __shared__ float v[2][kMaxM];
  __shared__ float red[2 * (kThreads / 32)];
  const int u = blockIdx.x, t = threadIdx.x, w = t >> 5, lane = t & 31, m = p.m;
  const float* X = p.X + (size_t)u * m * m;
  for (int i = t; i < kMaxM; i += kThreads) v[0][i] = i < m ? rsqrtf((float)m) : 0.f;
  __syncthreads();
  float rq = 0.f;
  for (int it = 0; it <= kKappaIters; ++it) {
    const float* vin = v[it & 1];
    float* vout = v[(it + 1) & 1];
    float num = 0.f, den = 0.f;
    for (int i = w; i < m; i += kThreads / 32) {
      float s = 0.f;
      for (int j = lane; j < m; j += 32) s = fmaf(X[(size_t)i * m + j], vin[j], s);
      for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
      if (lane == 0) vout[i] = s;
      num = fmaf(s, vin[i], num);   // lane-uniform: every lane adds the same terms
      den = fmaf(s, s, den);
    }
    if (lane == 0) {
      red[w] = num;
      red[kThreads / 32 + w] = den;
    }
    __syncthreads();
    float nsum = 0.f, dsum = 0.f;
    for (int k = 0; k < kThreads / 32; ++k) {
      nsum += red[k];
      dsum += red[kThreads / 32 + k];
    }
    rq = nsum;   // v^T X v with ||v|| = 1
    const float sc = dsum > 0.f ? rsqrtf(dsum) : 0.f;
    __syncthreads();
    for (int i = t; i < m; i += kThreads) vout[i] *= sc;
    __syncthreads();
  }
  if (t == 0) {
    float* inf = p.info + (size_t)u * kInfoStride;
    inf[kInfoKappa] = inf[kInfoLambdaMax] * rq;
  }
}

cudaError_t launch_kappa(const Params& p, cudaStream_t st) {
  k_kappa<<<p.U, kThreads, 0, st>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_cross_kernel(const Params& p, int unit, float* C_out, cudaStream_t st) {
  const size_t smem = generic_smem_pass2(p.m, p.d);
  if (p.dtype == LFA_BF16)
    k_cross_out<__nv_bfloat16><<<p.n_tiles, kThreads, smem, st>>>(p, unit, C_out);
  else
    k_cross_out<float><<<p.n_tiles, kThreads, smem, st>>>(p, unit, C_out);
  return cudaGetLastError();
}

}  // namespace lfa
