// Backward pass of Laplacian-kernel Nystrom attention for the loss <dO, O>: dQ and dV.
//
// Reverse mode through the forward of the LaplacianFormer note (papernotes.org,
// §整体框架, §关键设计 1-3), per (batch, head) unit, with O = C~ M + DWC(V),
// M = X A, A = C~^T V:
//   dM = C~^T dO                   pass 1 again with dO in place of V (C^T dO, sum dO),
//                                  then the rank-1 whitening fold
//   dX = dM A^T, dA = X^T dM       k_bwd_combine
//   dC~ = dO M^T + V dA^T, the whitening backward (population-variance batch-norm form)
//   and dD = -(1/lam) C o dC (the kernel gradient -(1/lam) sign(x - y) k of
//   §研究背景与动机 with the sign corrected; sign(0) = 0)
//   dQ_direct[i,k] = sum_l dD[i,l] sign(q_ik - l_lk),  dL[l,k] -= sum_i dD[i,l] sign(q_ik - l_lk),
//   dV = C~ dA + DWC^T(dO)         k_bwd_main (C recomputed tile by tile, never stored)
//   Newton-Schulz in reverse (§关键设计 3, alpha held constant): iterates X_k recomputed
//   from X_0 = alpha W^T, then for k = T-1..0
//     dW -= X_k^T G X_k^T,  G <- 2G - G X_k^T W^T - W^T X_k^T G;   dW += alpha G^T
//   dE = -(1/lam) W o dW (off the diagonal), dL += sum_b (dE_ab + dE_ba) sign(l_a - l_b)
//   dQ = dQ_direct + pool^T(dL) / r^2                                k_dq_final
#include <math.h>

#include "lfa_internal.h"

namespace lfa {
namespace {

constexpr int kLC = 64;          // landmarks per chunk of the main backward kernel
constexpr int kCS = kLC + 4;     // row stride (floats) of the chunk tiles

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

// sign(t) * x with sign(0) = 0
__device__ __forceinline__ float sgn_mul(float t, float x) { return t > 0.f ? x : (t < 0.f ? -x : 0.f); }

// acc + sign(t) x with sign(0) = 0: x with t's sign bit folded in (one logic instruction), kept where t != 0
__device__ __forceinline__ float add_sgn(float acc, float t, float x) {
  const float r = __int_as_float(__float_as_int(x) ^ (__float_as_int(t) & 0x80000000));
  return acc + (t != 0.f ? r : 0.f);
}

// acc - sign(t) x with sign(0) = 0 on the FMA pipe: sat(t 2^126) is 1 for t >= 2^-126 and 0 for t <= 0
// (and sat(-t 2^126) the other way round), so the two products add exactly -x, +x or nothing; the logic /
// compare pipe, which the other sign contraction keeps busy, is not used. (A nonzero |t| below 2^-126
// would give a fraction; t is a difference of a token entry and a landmark average.)
__device__ __forceinline__ float sub_sgn_fma(float acc, float t, float x) {
  const float sp = __saturatef(t * 0x1p126f), sn = __saturatef(t * -0x1p126f);
  return fmaf(x, sn, fmaf(-x, sp, acc));
}

// X_0 = alpha W^T with the alpha the forward chose (per-unit info slot).
__global__ void k_init_iterate(BwdParams b) {
  const Params& p = b.p;
  const int u = blockIdx.y, m = p.m;
  const int e = blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= m * m) return;
  const float alpha = p.info[(size_t)u * kInfoStride + kInfoAlpha];
  const int i = e / m, j = e % m;
  b.its[(size_t)u * p.T * m * m + e] = alpha * p.Wm[(size_t)u * m * m + (size_t)j * m + i];
}

// ---------------------------------------------------------------------------------------
// Combine of the backward statistics: dM, then rows [16c, 16c + 16) of dX = dM A^T and
// dA = X^T dM, the whitening-backward coefficients (for batch-pooled statistics their per-unit sums,
// pooled by k_bwd_pool_coef), Gm = s o M, Gd = s o dA and the bias partial of dV.
//   dC_il = s_l dC~_il + beta_l + gamma_l C_il with
//   a_l = mean_i dC~_il, e_l = sum_i dC~_il C_il, c_l = (s_l / N)(e_l - mu_l N a_l),
//   gamma_l = -s_l^2 c_l, beta_l = -s_l a_l - gamma_l mu_l.
// ---------------------------------------------------------------------------------------
__global__ void __launch_bounds__(kThreads) k_bwd_combine(BwdParams b) {
  extern __shared__ float4 smem_f4[];
  float* dMs = reinterpret_cast<float*>(smem_f4);   // [m][d]
  const Params& p = b.p;
  const int m = p.m, d = p.d, u = blockIdx.y, c = blockIdx.x, t = threadIdx.x;
  const double invN = 1.0 / double(p.N);
  const double* rf = p.red + (size_t)u * p.part_stride;    // forward: S1, S2, P = C^T V, sum V
  const double* rb = b.red2 + (size_t)u * p.part_stride;   // backward: -, -, C^T dO, sum dO
  const float* mu = p.mu + (size_t)u * m;
  const float* s = p.s + (size_t)u * m;
  for (int e = t; e < m * d; e += blockDim.x) {
    const int j = e / d, k = e % d;
    const double pd = rb[2 * m + e], sdo = rb[2 * m + m * d + k];
    const double v = p.whiten ? (double)s[j] * (pd - (double)mu[j] * sdo) + sdo * invN : pd;
    dMs[e] = (float)v;
  }
  __syncthreads();
  const float* A = p.A + (size_t)u * m * d;
  const float* X = p.X + (size_t)u * m * m;
  const float* M = p.M + (size_t)u * m * d;
  const int j0 = c * 16;
  // dX rows: dX[j][l] = sum_k dM[j][k] A[l][k]  (initial G of the reverse Newton-Schulz)
  for (int e = t; e < 16 * m; e += blockDim.x) {
    const int jj = e / m, l = e % m, j = j0 + jj;
    if (j >= m) continue;
    float acc = 0.f;
    for (int k = 0; k < d; ++k) acc = fmaf(dMs[j * d + k], A[(size_t)l * d + k], acc);
    b.G[((size_t)u * m + j) * m + l] = acc;
  }
  // dA rows: dA[j][k] = sum_l X[l][j] dM[l][k]
  for (int e = t; e < 16 * d; e += blockDim.x) {
    const int jj = e / d, k = e % d, j = j0 + jj;
    if (j >= m) continue;
    float acc = 0.f;
    for (int l = 0; l < m; ++l) acc = fmaf(X[(size_t)l * m + j], dMs[l * d + k], acc);
    b.dA[((size_t)u * m + j) * d + k] = acc;
  }
  __syncthreads();   // this CTA's dA rows are visible to its own threads
  // per landmark row: one warp, lanes over channels
  const int w = t >> 5, lane = t & 31;
  for (int jj = w; jj < 16; jj += kThreads / 32) {
    const int j = j0 + jj;
    if (j >= m) break;
    const float sj = p.whiten ? s[j] : 1.f;
    double sa = 0.0, se = 0.0;
    for (int k = lane; k < d; k += 32) {
      const size_t o = ((size_t)u * m + j) * d + k;
      const double Mjk = M[(size_t)j * d + k], dAjk = b.dA[o];
      sa += rb[2 * m + m * d + k] * Mjk + rf[2 * m + m * d + k] * dAjk;
      se += Mjk * rb[2 * m + (size_t)j * d + k] + dAjk * rf[2 * m + (size_t)j * d + k];
      b.Gm[o] = sj * (float)Mjk;
      b.Gd[o] = sj * (float)dAjk;
    }
    for (int o = 16; o > 0; o >>= 1) {
      sa += __shfl_xor_sync(0xffffffffu, sa, o);
      se += __shfl_xor_sync(0xffffffffu, se, o);
    }
    if (lane == 0) {
      if (p.whiten == 2) {
        // batch-pooled statistics: the sums go to the unused column-sum slots of this unit's dO
        // record; k_bwd_pool_coef adds them over the head's units and forms beta and gamma
        double* rbw = b.red2 + (size_t)u * p.part_stride;
        rbw[j] = sa;
        rbw[m + j] = se;
      } else {
        double beta = 0.0, gamma = 0.0;
        if (p.whiten) {
          const double a = sa * invN, sd = sj, mj = mu[j];
          const double cc = sd * invN * (se - mj * double(p.N) * a);
          gamma = -sd * sd * cc;
          beta = -sd * a - gamma * mj;
        }
        b.beta[(size_t)u * m + j] = (float)beta;
        b.gamma[(size_t)u * m + j] = (float)gamma;
      }
    }
  }
  // bias partial of dV: sum over this chunk's rows of (1/N - s_j mu_j) dA[j][k]
  for (int k = t; k < d; k += blockDim.x) {
    double acc = 0.0;
    if (p.whiten) {
      for (int jj = 0; jj < 16; ++jj) {
        const int j = j0 + jj;
        if (j < m) acc += (invN - (double)s[j] * (double)mu[j]) * (double)b.dA[((size_t)u * m + j) * d + k];
      }
    }
    b.bpart2[((size_t)u * p.n_chunks + c) * d + k] = (float)acc;
  }
}

// ---------------------------------------------------------------------------------------
// Whitening-backward coefficients for statistics pooled per head over the batch (whiten = 2): the
// means over the B N stacked rows of the head's units (batch b = 0 .. B-1 in order), with the
// shared mu and s: a_l = (sum_b sum_i dC~_il) / (B N), e_l = sum_b sum_i dC~_il C_il,
// c_l = (s_l / (B N)) (e_l - mu_l B N a_l), gamma_l = -s_l^2 c_l, beta_l = -s_l a_l - gamma_l mu_l,
// written to every unit of the head.
// ---------------------------------------------------------------------------------------
__global__ void __launch_bounds__(kThreads) k_bwd_pool_coef(BwdParams b) {
  const Params& p = b.p;
  const int m = p.m, h = blockIdx.y, j = blockIdx.x * blockDim.x + threadIdx.x;
  if (j >= m) return;
  double sa = 0.0, se = 0.0;
  for (int bb = 0; bb < p.B; ++bb) {
    const double* rb = b.red2 + (size_t)(bb * p.heads + h) * p.part_stride;
    sa += rb[j];
    se += rb[m + j];
  }
  // the per-unit formula's operation order with N -> B N (identical results at B = 1)
  const double BN = double(p.B) * double(p.N), invBN = 1.0 / BN;
  const double sj = p.s[(size_t)h * m + j], mj = p.mu[(size_t)h * m + j];
  const double a = sa * invBN;
  const double cc = sj * invBN * (se - mj * BN * a);
  const double gamma = -sj * sj * cc;
  const double beta = -sj * a - gamma * mj;
  for (int bb = 0; bb < p.B; ++bb) {
    const size_t o = (size_t)(bb * p.heads + h) * m + j;
    b.beta[o] = (float)beta;
    b.gamma[o] = (float)gamma;
  }
}

// ---------------------------------------------------------------------------------------
// Landmark-gram part of dL: dL[a][k] = sum_{b != a} (dE_ab + dE_ba) sign(l_ak - l_bk) with
// dE_xy = -(1/lam) W_xy (dW_xy + alpha G0_yx) off the diagonal. The diagonal (W = 1 + eps)
// meets sign(0) = 0 and drops out. Rows of 256 / d landmarks per CTA.
// ---------------------------------------------------------------------------------------
__global__ void __launch_bounds__(kThreads) k_dl_gram(BwdParams b) {
  __shared__ float S[kThreads / 32][kMaxM];
  const Params& p = b.p;
  const int m = p.m, d = p.d, u = blockIdx.y;
  const int rows = kThreads / d;
  const int a = blockIdx.x * rows + threadIdx.x / d, k = threadIdx.x % d, ra = threadIdx.x / d;
  const size_t mm = (size_t)m * m;
  const float* W = p.Wm + u * mm;
  const float* dW = b.dW + u * mm;
  const float* G0 = b.G + u * mm;
  const float alpha = p.info[(size_t)u * kInfoStride + kInfoAlpha];
  const float il = 1.f / p.lam;
  if (a < m) {
    for (int bb = k; bb < m; bb += d) {
      float v = 0.f;
      if (bb != a) {
        const float e_ab = -il * W[(size_t)a * m + bb] * (dW[(size_t)a * m + bb] + alpha * G0[(size_t)bb * m + a]);
        const float e_ba = -il * W[(size_t)bb * m + a] * (dW[(size_t)bb * m + a] + alpha * G0[(size_t)a * m + bb]);
        v = e_ab + e_ba;
      }
      S[ra][bb] = v;
    }
  }
  __syncthreads();
  if (a >= m) return;
  const float* L = p.L + (size_t)u * m * d;
  const float la = L[(size_t)a * d + k];
  float acc = 0.f;
  for (int bb = 0; bb < m; ++bb) acc += sgn_mul(la - L[(size_t)bb * d + k], S[ra][bb]);
  b.dLns[((size_t)u * m + a) * d + k] = acc;
}

// ---------------------------------------------------------------------------------------
// Main backward pass over 64-row tiles of one unit, landmarks in chunks of 64.
// Thread maps: (tr = t / 16, tl = t % 16) rows 4tr.. x landmarks tl + 16j for C and dD;
// (ib = t / nkb, kb = t % nkb) rows 4ib.. x channels 4kb.. for dQ, dV;
// (jb = t / nkb, kb) chunk landmarks 4jb.. x channels 4kb.. for the dL partials.
// ---------------------------------------------------------------------------------------
template <typename T, int NC>
__global__ void __launch_bounds__(kThreads) k_bwd_main(BwdParams b) {
  extern __shared__ float4 smem_f4[];
  const Params& p = b.p;
  const int m = p.m, d = p.d, ds = d + 4, nkb = d / 4;
  float* Qs = reinterpret_cast<float*>(smem_f4);   // [64][ds]
  float* Os = Qs + kRowTile * ds;                   // dO tile [64][ds]
  float* Vs = Os + kRowTile * ds;                   // [64][ds]
  float* Lc = Vs + kRowTile * ds;                   // chunk landmarks [64][ds]
  float* Gmc = Lc + kLC * ds;                       // [64][ds]
  float* Gdc = Gmc + kLC * ds;                      // [64][ds]
  float* Cs = Gdc + kLC * ds;                       // [64 rows][kCS]
  float* Ds = Cs + kRowTile * kCS;                  // [64 rows][kCS]
  float* bg = Ds + kRowTile * kCS;                  // beta [64], gamma [64], bias [d]
  const int u = blockIdx.y, pc = blockIdx.x, t = threadIdx.x;
  const size_t uoff = (size_t)u * p.N * d;
  const T* Qg = static_cast<const T*>(p.Q) + uoff;
  const T* Vg = static_cast<const T*>(p.V) + uoff;
  const T* dOg = static_cast<const T*>(b.dO) + uoff;
  const float il = 1.f / p.lam;
  const bool mapped = t < 16 * nkb;
  const int ib = t / nkb, kb = t % nkb;
  const int tr = t >> 4, tl = t & 15;
  if (t < d) {
    float acc = 0.f;
    for (int c = 0; c < p.n_chunks; ++c) acc += b.bpart2[((size_t)u * p.n_chunks + c) * d + t];
    bg[2 * kLC + t] = acc;
  }
  float accL[NC][4][4];
#pragma unroll
  for (int c = 0; c < NC; ++c)
#pragma unroll
    for (int x = 0; x < 4; ++x)
#pragma unroll
      for (int y = 0; y < 4; ++y) accL[c][x][y] = 0.f;
  const int h = u % p.heads;
  const int tile0 = pc * p.tiles_per_cta;
  const int tile1 = min(tile0 + p.tiles_per_cta, p.n_tiles);
  for (int tile = tile0; tile < tile1; ++tile) {
    const int row0 = tile * kRowTile;
    const int valid = min(kRowTile, p.N - row0);
    __syncthreads();
    for (int e = t; e < kRowTile * nkb; e += kThreads) {
      const int r = e / nkb, c4 = (e % nkb) * 4;
      const bool ok = r < valid;
      const size_t g = (size_t)(row0 + r) * d + c4;
      const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
      *reinterpret_cast<float4*>(&Qs[r * ds + c4]) = ok ? load4(Qg + g) : z;
      *reinterpret_cast<float4*>(&Os[r * ds + c4]) = ok ? load4(dOg + g) : z;
      *reinterpret_cast<float4*>(&Vs[r * ds + c4]) = ok ? load4(Vg + g) : z;
    }
    float accQ[4][4] = {}, accV[4][4] = {};
#pragma unroll
    for (int c = 0; c < NC; ++c) {
      const int j0 = c * kLC;
      __syncthreads();   // previous chunk's readers are done; the row tiles are staged
      for (int e = t; e < kLC * nkb; e += kThreads) {
        const int r = e / nkb, c4 = (e % nkb) * 4;
        const int j = j0 + r;
        const bool ok = j < m;
        const size_t g = ((size_t)u * m + j) * d + c4;
        const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
        *reinterpret_cast<float4*>(&Lc[r * ds + c4]) = ok ? load4(p.L + g) : z;
        *reinterpret_cast<float4*>(&Gmc[r * ds + c4]) = ok ? load4(b.Gm + g) : z;
        *reinterpret_cast<float4*>(&Gdc[r * ds + c4]) = ok ? load4(b.Gd + g) : z;
      }
      if (t < kLC) {
        const int j = j0 + t;
        bg[t] = j < m ? b.beta[(size_t)u * m + j] : 0.f;
        bg[kLC + t] = j < m ? b.gamma[(size_t)u * m + j] : 0.f;
      }
      __syncthreads();
      // C and dD for rows 4tr + i, chunk landmarks tl + 16 jj
      {
        float dist[4][4] = {}, g[4][4] = {};
        for (int k = 0; k < d; k += 4) {
          float4 q[4], o[4], v[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            q[i] = *reinterpret_cast<const float4*>(&Qs[(4 * tr + i) * ds + k]);
            o[i] = *reinterpret_cast<const float4*>(&Os[(4 * tr + i) * ds + k]);
            v[i] = *reinterpret_cast<const float4*>(&Vs[(4 * tr + i) * ds + k]);
          }
#pragma unroll
          for (int jj = 0; jj < 4; ++jj) {
            const int lr = tl + 16 * jj;
            const float4 l = *reinterpret_cast<const float4*>(&Lc[lr * ds + k]);
            const float4 gm = *reinterpret_cast<const float4*>(&Gmc[lr * ds + k]);
            const float4 gd = *reinterpret_cast<const float4*>(&Gdc[lr * ds + k]);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              dist[i][jj] += fabsf(q[i].x - l.x);
              dist[i][jj] += fabsf(q[i].y - l.y);
              dist[i][jj] += fabsf(q[i].z - l.z);
              dist[i][jj] += fabsf(q[i].w - l.w);
              float a = g[i][jj];
              a = fmaf(o[i].x, gm.x, a);
              a = fmaf(o[i].y, gm.y, a);
              a = fmaf(o[i].z, gm.z, a);
              a = fmaf(o[i].w, gm.w, a);
              a = fmaf(v[i].x, gd.x, a);
              a = fmaf(v[i].y, gd.y, a);
              a = fmaf(v[i].z, gd.z, a);
              a = fmaf(v[i].w, gd.w, a);
              g[i][jj] = a;
            }
          }
        }
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int jj = 0; jj < 4; ++jj) {
            const int row = 4 * tr + i, lr = tl + 16 * jj;
            const bool ok = row < valid && j0 + lr < m;
            const float cv = ok ? exp2f(dist[i][jj] * p.neg_log2e_over_lam) : 0.f;
            const float dc = g[i][jj] + bg[lr] + bg[kLC + lr] * cv;
            Cs[row * kCS + lr] = cv;
            Ds[row * kCS + lr] = ok ? -il * cv * dc : 0.f;
          }
      }
      __syncthreads();
      if (mapped) {
        // dQ_direct and dV over this chunk: rows 4ib.., channels 4kb..
        float qv[4][4];
#pragma unroll
        for (int x = 0; x < 4; ++x) {
          const float4 q = *reinterpret_cast<const float4*>(&Qs[(4 * ib + x) * ds + 4 * kb]);
          qv[x][0] = q.x; qv[x][1] = q.y; qv[x][2] = q.z; qv[x][3] = q.w;
        }
        for (int lr = 0; lr < kLC; ++lr) {
          const float4 l = *reinterpret_cast<const float4*>(&Lc[lr * ds + 4 * kb]);
          const float4 gd = *reinterpret_cast<const float4*>(&Gdc[lr * ds + 4 * kb]);
          const float lv[4] = {l.x, l.y, l.z, l.w}, gv[4] = {gd.x, gd.y, gd.z, gd.w};
#pragma unroll
          for (int x = 0; x < 4; ++x) {
            const float dd = Ds[(4 * ib + x) * kCS + lr], cv = Cs[(4 * ib + x) * kCS + lr];
#pragma unroll
            for (int y = 0; y < 4; ++y) {
              accQ[x][y] = add_sgn(accQ[x][y], qv[x][y] - lv[y], dd);
              accV[x][y] = fmaf(cv, gv[y], accV[x][y]);
            }
          }
        }
        // dL partials: chunk landmarks 4jb.. (jb = ib), channels 4kb..
        float lv[4][4];
#pragma unroll
        for (int x = 0; x < 4; ++x) {
          const float4 l = *reinterpret_cast<const float4*>(&Lc[(4 * ib + x) * ds + 4 * kb]);
          lv[x][0] = l.x; lv[x][1] = l.y; lv[x][2] = l.z; lv[x][3] = l.w;
        }
        for (int i = 0; i < valid; ++i) {
          const float4 q = *reinterpret_cast<const float4*>(&Qs[i * ds + 4 * kb]);
          const float4 dd4 = *reinterpret_cast<const float4*>(&Ds[i * kCS + 4 * ib]);
          const float qq[4] = {q.x, q.y, q.z, q.w}, dd[4] = {dd4.x, dd4.y, dd4.z, dd4.w};
#pragma unroll
          for (int x = 0; x < 4; ++x)
#pragma unroll
            for (int y = 0; y < 4; ++y) accL[c][x][y] = sub_sgn_fma(accL[c][x][y], qq[y] - lv[x][y], dd[x]);
        }
      }
    }
    // write dQ_direct (fp32) and dV = C~ dA + DWC^T(dO) for the tile's rows
    if (mapped) {
      float wt[4][9];
#pragma unroll
      for (int y = 0; y < 4; ++y)
#pragma unroll
        for (int e = 0; e < 9; ++e) wt[y][e] = p.dwc[((size_t)h * d + 4 * kb + y) * 9 + e];
      T* dVg = static_cast<T*>(b.dV) + uoff;
#pragma unroll
      for (int x = 0; x < 4; ++x) {
        const int i = 4 * ib + x;
        if (i >= valid) continue;
        const int n = row0 + i, gy = n / p.W, gx = n % p.W;
        *reinterpret_cast<float4*>(b.dQd + uoff + (size_t)n * d + 4 * kb) =
            make_float4(accQ[x][0], accQ[x][1], accQ[x][2], accQ[x][3]);
        float o[4];
#pragma unroll
        for (int y = 0; y < 4; ++y) o[y] = accV[x][y] + bg[2 * kLC + 4 * kb + y];
        // DWC^T: dV[y][x] += w[a][b] dO[y + 1 - a][x + 1 - b]
#pragma unroll
        for (int a = 0; a < 3; ++a) {
          const int yy = gy + 1 - a;
          if (yy < 0 || yy >= p.H) continue;
#pragma unroll
          for (int bb = 0; bb < 3; ++bb) {
            const int xx = gx + 1 - bb;
            if (xx < 0 || xx >= p.W) continue;
            const float4 g = load4(dOg + ((size_t)yy * p.W + xx) * d + 4 * kb);
            o[0] = fmaf(wt[0][a * 3 + bb], g.x, o[0]);
            o[1] = fmaf(wt[1][a * 3 + bb], g.y, o[1]);
            o[2] = fmaf(wt[2][a * 3 + bb], g.z, o[2]);
            o[3] = fmaf(wt[3][a * 3 + bb], g.w, o[3]);
          }
        }
        store4(dVg + (size_t)n * d + 4 * kb, make_float4(o[0], o[1], o[2], o[3]));
      }
    }
  }
  if (mapped) {
    float* out = b.dLpart + ((size_t)u * p.P + pc) * m * d;
#pragma unroll
    for (int c = 0; c < NC; ++c)
#pragma unroll
      for (int x = 0; x < 4; ++x) {
        const int j = c * kLC + 4 * ib + x;
        if (j < m)
          *reinterpret_cast<float4*>(out + (size_t)j * d + 4 * kb) =
              make_float4(accL[c][x][0], accL[c][x][1], accL[c][x][2], accL[c][x][3]);
      }
  }
}

// dL total / r^2: the main pass's partials (fp64 sum) plus the landmark-gram part.
__global__ void __launch_bounds__(kThreads) k_dl_reduce(BwdParams b) {
  const Params& p = b.p;
  const int u = blockIdx.y, md = p.m * p.d;
  const int e = blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= md) return;
  double acc = b.dLns[(size_t)u * md + e];
  const float* src = b.dLpart + (size_t)u * p.P * md + e;
  for (int pc = 0; pc < p.P; ++pc) acc += (double)src[(size_t)pc * md];
  b.dLpool[(size_t)u * md + e] = (float)(acc / double(p.r * p.r));
}

// dQ = dQ_direct + pool^T(dL) / r^2, in the storage dtype.
template <typename T>
__global__ void __launch_bounds__(kThreads) k_dq_final(BwdParams b) {
  const Params& p = b.p;
  const int u = blockIdx.y, d = p.d, q4 = d / 4;
  const int e = blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= p.N * q4) return;
  const int n = e / q4, c4 = (e % q4) * 4;
  const int gy = n / p.W, gx = n % p.W;
  const int l = (gy / p.r) * (p.W / p.r) + gx / p.r;
  const size_t o = (size_t)u * p.N * d + (size_t)n * d + c4;
  const float4 a = *reinterpret_cast<const float4*>(b.dQd + o);
  const float4 g = *reinterpret_cast<const float4*>(b.dLpool + ((size_t)u * p.m + l) * d + c4);
  store4(static_cast<T*>(b.dQ) + o, make_float4(a.x + g.x, a.y + g.y, a.z + g.z, a.w + g.w));
}

template <typename T, int NC>
void launch_main(const BwdParams& b, cudaStream_t st) {
  k_bwd_main<T, NC><<<dim3(b.p.P, b.p.U), kThreads, backward_smem_main(b.p.d), st>>>(b);
}

template <typename T>
cudaError_t backward_t(const BwdParams& b, cudaStream_t st) {
  const Params& p = b.p;
  const int U = p.U, m = p.m, d = p.d, T_ = p.T;
  const size_t mm = (size_t)m * m;
  // C^T dO and sum dO per unit: pass 1 with dO in the place of V
  Params p1 = p;
  p1.V = b.dO;
  p1.part = b.part2;
  p1.red = b.red2;
  // C^T dO, the combine and the Newton-Schulz iterates X_0 .. X_{T-1} ([U][T][m][m]) share no data:
  // with an auxiliary stream the iterates run concurrently with the other two
  const size_t its_stride = (size_t)T_ * mm;
  cudaError_t e = cudaSuccess;
  fork_join(p, st,
            [&](cudaStream_t s) {
              e = launch_generic_pass1_reduce(p1, s);
              k_bwd_combine<<<dim3(p.n_chunks, U), kThreads, (size_t)m * d * sizeof(float), s>>>(b);
              if (p.whiten == 2) k_bwd_pool_coef<<<dim3(ceil_div(m, kThreads), p.heads), kThreads, 0, s>>>(b);
            },
            [&](cudaStream_t s) {
              if (T_ == 0) return;
              k_init_iterate<<<dim3(ceil_div(m * m, kThreads), U), kThreads, 0, s>>>(b);
              const NsChain c{p.Wm, mm, p.Y, mm, b.its, nullptr, its_stride, mm, m, T_ - 1, 1, p.status};
              if (m > kSmallM && launch_ns_chain(c, U, s)) return;
              for (int k = 0; k + 1 < T_; ++k) {
                const float* Xk = b.its + k * mm;
                const MmJob y{p.Wm, mm, Xk, its_stride, nullptr, 0, p.Y, mm, -1.f, 0.f, 2.f, 0, 0};  // Y = 2I - W X_k
                launch_mm(&y, 1, m, U, s, p.status);
                const MmJob xn{Xk, its_stride, p.Y, mm, nullptr, 0, b.its + (k + 1) * mm, its_stride,  // X_{k+1} = X_k Y
                               1.f, 0.f, 0.f, 0, 0};
                launch_mm(&xn, 1, m, U, s, p.status);
              }
            });
  if (e != cudaSuccess) return e;
  // reverse steps; G starts as dX
  if (cudaMemsetAsync(b.dW, 0, sizeof(float) * U * mm, st) != cudaSuccess) return cudaErrorUnknown;
  float* G = b.G;
  float* Gn = b.Gn;
  for (int k = T_ - 1; k >= 0; --k) {
    const float* Xk = b.its + k * mm;
    const MmJob s1[3] = {
        {Xk, its_stride, G, mm, nullptr, 0, b.T1, mm, 1.f, 0.f, 0.f, 1, 0},      // T1 = X_k^T G
        {G, mm, Xk, its_stride, nullptr, 0, b.T2, mm, 1.f, 0.f, 0.f, 0, 1},      // T2 = G X_k^T
        {p.Wm, mm, Xk, its_stride, nullptr, 0, b.T3, mm, 1.f, 0.f, 0.f, 1, 1}};  // T3 = W^T X_k^T
    launch_mm(s1, 3, m, U, st, p.status);
    const MmJob s2[2] = {
        {b.T1, mm, Xk, its_stride, b.dW, mm, b.dW, mm, -1.f, 1.f, 0.f, 0, 1},    // dW -= T1 X_k^T
        {b.T2, mm, p.Wm, mm, G, mm, Gn, mm, -1.f, 2.f, 0.f, 0, 1}};              // Gn = 2G - T2 W^T
    launch_mm(s2, 2, m, U, st, p.status);
    const MmJob s3{b.T3, mm, G, mm, Gn, mm, Gn, mm, -1.f, 1.f, 0.f, 0, 0};      // Gn -= T3 G
    launch_mm(&s3, 1, m, U, st, p.status);
    float* tmp = G;
    G = Gn;
    Gn = tmp;
  }
  BwdParams b0 = b;
  b0.G = G;   // G_0
  const int rows = kThreads / d;
  k_dl_gram<<<dim3(ceil_div(m, rows), U), kThreads, 0, st>>>(b0);
  const int nc = ceil_div(m, kLC);
  if (nc == 1) launch_main<T, 1>(b, st);
  else if (nc == 2) launch_main<T, 2>(b, st);
  else if (nc == 3) launch_main<T, 3>(b, st);
  else launch_main<T, 4>(b, st);
  k_dl_reduce<<<dim3(ceil_div(m * d, kThreads), U), kThreads, 0, st>>>(b);
  k_dq_final<T><<<dim3(ceil_div(p.N * (d / 4), kThreads), U), kThreads, 0, st>>>(b);
  return cudaGetLastError();
}

}  // namespace

size_t backward_smem_main(int d) {
  const int ds = d + 4;
  return sizeof(float) * ((size_t)3 * kRowTile * ds + (size_t)3 * kLC * ds + (size_t)2 * kRowTile * kCS + 2 * kLC + d);
}

cudaError_t backward_set_attributes() {
  const int big = 227 * 1024;
  cudaError_t e = cudaSuccess;
#define LFA_ATTR(fn) \
  if (e == cudaSuccess) e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, big)
  LFA_ATTR(k_bwd_combine);
  LFA_ATTR((k_bwd_main<float, 1>));
  LFA_ATTR((k_bwd_main<float, 2>));
  LFA_ATTR((k_bwd_main<float, 3>));
  LFA_ATTR((k_bwd_main<float, 4>));
  LFA_ATTR((k_bwd_main<__nv_bfloat16, 1>));
  LFA_ATTR((k_bwd_main<__nv_bfloat16, 2>));
  LFA_ATTR((k_bwd_main<__nv_bfloat16, 3>));
  LFA_ATTR((k_bwd_main<__nv_bfloat16, 4>));
#undef LFA_ATTR
  return e;
}

int backward_launch_count(const Params& p) {
  // pass 1 + reduce, combine, iterates (1 + 2 (T - 1), or 1 + 1 as one cluster launch), 3 T reverse launches (6 products per step, batched), gram part of dL,
  // main pass, dL reduction, dQ
  const int its = p.T > 0 ? 1 + (p.m > kSmallM && ns_chain_fits(p.m) ? (p.T > 1 ? 1 : 0) : 2 * (p.T - 1)) : 0;
  return 2 + 1 + (p.whiten == 2 ? 1 : 0) + its + 3 * p.T + 1 + 1 + 1 + 1;
}

cudaError_t launch_backward(const BwdParams& b, cudaStream_t st) {
  return b.p.dtype == LFA_BF16 ? backward_t<__nv_bfloat16>(b, st) : backward_t<float>(b, st);
}

}  // namespace lfa
