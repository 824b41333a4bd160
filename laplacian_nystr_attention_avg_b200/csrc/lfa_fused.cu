// Fused single-launch forward pass for bf16 inputs, d = 64 and m <= 63 landmarks.
//
// One cooperative persistent kernel, one CTA per SM:
//   phase 0  all CTAs: landmark pooling L = r x r average pool of Q      (LaplacianFormer note,
//            §关键设计 2), then a grid-wide barrier.
//   phase 1a CTAs 0..U-1 ("solver CTAs"), one per (batch, head) unit: W = exp(-E/lam) + eps I,
//            ||W||_2 by power iteration, alpha (§关键设计 3, with the fallback), and the T
//            Newton-Schulz steps on tcgen05 tensor cores in 3xTF32 (fp32-accurate). The steps
//            are evaluated as X_{k+1} = X_k + X_k R_k, R_{k+1} = R_k^2 (R_k = I - W X_k, the
//            same iterates in exact arithmetic, one stacked [X;R] product per step) followed by
//            the printed product form X (2I - W X) for the last two steps, which re-anchors R to
//            I - W X. X is published with a release flag.
//   phase 1b the other CTAs ("row CTAs") split the U*N token rows evenly. For each 128-row chunk:
//            C = exp(-||q - l||_1 / lam) on CUDA cores (fp32, the dominant cost), kept in shared
//            memory as bf16 for the whole kernel (never written to HBM); per-landmark sums of C
//            and C^2 in registers; P += C^T V on tcgen05 (V chunk staged by TMA; a constant-1
//            landmark column yields sum_i v_i in the same product).
//   phase 2  per unit, every row CTA of that unit waits for the unit's partial records and X,
//            then forms mu, var, s = 1/sqrt(var + eps), A = C~^T V (rank-1 folding of the
//            whitening, §关键设计 1), M = X A, M' = diag(s) M, b = (1/N - s o mu)^T M.
//   phase 3  per chunk: O = C M' (tcgen05, accumulator in TMEM) + b + DWC(V), stored as bf16.
// Every cross-CTA wait is bounded; an expired wait sets the timeout bit of the status word.
#include <string.h>

#include "lfa_internal.h"
#include "lfa_sm100.cuh"
#include "lfa_tma_host.h"

namespace lfa {
namespace {

using namespace sm100;

constexpr int kFT = 256;                  // threads per CTA (8 warps)
constexpr int kChunk = 128;               // token rows per chunk
constexpr int kMaxChunks = 8;             // resident C chunks per row CTA
constexpr int kQS = 68;                   // fp32 row stride (floats) of the Q and L tiles
constexpr int kRec = 128 + 64 * 64;       // floats per partial record: S1[64], S2[64], P[64][64]
constexpr int kMaxGrid = 256;             // records are sized for up to this many CTAs
constexpr int kPowerIters = 8;

// shared-memory map (bytes from a 1024-aligned base)
constexpr uint32_t kOffC = 0;                                   // 8 x 16 KB C chunks (SW128 rows)
constexpr uint32_t kOffV = kOffC + kMaxChunks * 16384;          // 2 x 16 KB V stages (TMA, SW128)
constexpr uint32_t kOffQ = kOffV + 2 * 16384;                   // Q chunk, fp32 [128][68]
constexpr uint32_t kOffL = kOffQ + kChunk * kQS * 4;            // landmarks, fp32 [64][68]
constexpr uint32_t kOffMp = kOffL + 64 * kQS * 4;               // M'^T bf16 [64 ch][64 lm] (SW128)
constexpr uint32_t kOffBv = kOffMp + 8192;                      // b, fp32 [64]
constexpr uint32_t kOffWd = kOffBv + 256;                       // DWC weights fp32 [9][64]
constexpr uint32_t kOffBar = kOffWd + 9 * 64 * 4;               // mbarriers + TMEM address
constexpr uint32_t kOffCt = kOffBar + 128;                       // int [32] record offsets
constexpr uint32_t kSmemBytes = kOffCt + 128;
constexpr uint32_t kSmemAlloc = kSmemBytes + 1024;              // slack for 1024-byte alignment
// combine scratch (aliases V/Q/L, free once pass 1 is done); then the pass-2 V halo tile
constexpr uint32_t kOffAs = kOffV;                              // fp32 [64][68]  A (row l, col k)
constexpr uint32_t kOffXt = kOffAs + 64 * kQS * 4;              // fp32 [64][68]  X^T (row l, col j)
constexpr uint32_t kOffS1 = kOffXt + 64 * kQS * 4;              // double [64]
constexpr uint32_t kOffS2 = kOffS1 + 512;                       // double [64]
constexpr uint32_t kOffMu = kOffS2 + 512;                       // float [64]
constexpr uint32_t kOffSc = kOffMu + 256;                       // float [64]
constexpr uint32_t kOffSv = kOffSc + 256;                       // float [64]
constexpr uint32_t kOffBp = kOffSv + 256;                       // float [16][64]
constexpr uint32_t kOffHalo = kOffV;                            // V halo rows: fp32 [rows][68] or bf16 [rows][72]
constexpr uint32_t kHaloBytes = kOffMp - kOffHalo;
constexpr int kHaloItems = 12;                                  // 16-byte halo loads per thread
// solver scratch (aliases the C region: solver CTAs hold no C)
constexpr uint32_t kOffNsHi = 0;                                // tf32 hi [2 K-halves][128 rows][128 B]
constexpr uint32_t kOffNsLo = 32768;                            // tf32 lo
constexpr uint32_t kOffNsW = 65536;                             // fp32 [64][68]
constexpr uint32_t kOffNsX = kOffNsW + 64 * kQS * 4;            // fp32 [64][68]
constexpr uint32_t kOffNsL = kOffNsX + 64 * kQS * 4;            // fp32 [64][68]
constexpr uint32_t kOffNsVec = kOffNsL + 64 * kQS * 4;          // float [64] x 2, red [64]

static_assert(kSmemAlloc <= 232448, "shared memory over the sm_100 per-block limit");
static_assert(kOffBp + 16 * 64 * 4 <= kOffMp, "combine scratch overlaps M'");
static_assert(kOffNsVec + 1024 <= kOffV, "solver scratch overlaps V stages");

// mbarrier slots
constexpr int kBarV = 0;      // [2] V stage filled by TMA
constexpr int kBarP1 = 2;     // [2] pass-1 product done (stage free)
constexpr int kBarP2 = 4;     // [2] pass-2 product done (accumulator ready)
constexpr int kBarNs = 6;     // solver product done

struct FusedArgs {
  unsigned long long epoch;   // launch count of this handle (>= 1); flags compare against it
  int G;                      // CTAs in the grid
  int n1;                     // row CTAs (G - U)
  unsigned long long* gbar;   // grid barrier counter
  unsigned long long* cnt;    // [U] partial records published per unit
  unsigned long long* xready; // [U] X published (holds the epoch)
  float* rec;                 // [n1][2][kRec]
};

__device__ __forceinline__ void trace_mark(const Params& p, int slot) {
  if (p.trace != nullptr && threadIdx.x == 0) p.trace[(size_t)blockIdx.x * 16 + slot] = globaltimer();
}

__device__ __forceinline__ void trace_clock(const Params& p, int slot) {
  if (p.trace != nullptr && threadIdx.x == 0) p.trace[(size_t)blockIdx.x * 16 + slot] = (unsigned long long)clock64();
}

__device__ __forceinline__ int row_cta(long long R, int n1, long long T) {
  return (int)(((R + 1) * n1 + T - 1) / T) - 1;
}
__device__ __forceinline__ long long row_start(int j, int n1, long long T) { return (long long)j * T / n1; }

__device__ __forceinline__ float bf_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf_hi(uint32_t v) { return __uint_as_float(v & 0xffff0000u); }

__device__ __forceinline__ void block_reduce2(float& a, float& b, float* red) {
  for (int o = 16; o > 0; o >>= 1) {
    a += __shfl_xor_sync(0xffffffffu, a, o);
    b += __shfl_xor_sync(0xffffffffu, b, o);
  }
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  __syncthreads();
  if (lane == 0) {
    red[w] = a;
    red[8 + w] = b;
  }
  __syncthreads();
  a = 0.f;
  b = 0.f;
  for (int i = 0; i < kFT / 32; ++i) {
    a += red[i];
    b += red[8 + i];
  }
}

// L [m][64] fp32 (global, written by other CTAs of this launch) -> [64][kQS] shared, zero rows >= m.
// 1024 float4 per CTA, 4 per thread, all loads issued before the stores.
__device__ __forceinline__ void load_landmarks(const float* Lg, float* Ls, int m) {
  float4 v[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int e4 = threadIdx.x + kFT * i, r = e4 >> 4;
    v[i] = r < m ? __ldcg(reinterpret_cast<const float4*>(Lg) + e4) : make_float4(0.f, 0.f, 0.f, 0.f);
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int e4 = threadIdx.x + kFT * i;
    *reinterpret_cast<float4*>(Ls + (e4 >> 4) * kQS + 4 * (e4 & 15)) = v[i];
  }
}

// ---------------------------------------------------------------------------------------
// Solver CTA: W, alpha and the Newton-Schulz chain of one unit on tcgen05 (3xTF32).
// Thread (warp w, lane) owns row r = 32 (w % 4) + lane of the stacked 128 x 64 operand
// [top; bottom] and the column half h = w / 4 (columns 32h .. 32h + 31).
// ---------------------------------------------------------------------------------------
__device__ void ns_store(unsigned char* base, int r, int h, const float* v) {
#pragma unroll
  for (int c4 = 0; c4 < 8; ++c4) {
    float4 hi, lo;
    hi.x = tf32_round(v[4 * c4 + 0]);
    hi.y = tf32_round(v[4 * c4 + 1]);
    hi.z = tf32_round(v[4 * c4 + 2]);
    hi.w = tf32_round(v[4 * c4 + 3]);
    lo.x = v[4 * c4 + 0] - hi.x;
    lo.y = v[4 * c4 + 1] - hi.y;
    lo.z = v[4 * c4 + 2] - hi.z;
    lo.w = v[4 * c4 + 3] - hi.w;
    const uint32_t off = h * 16384 + sw128(r, c4);
    *reinterpret_cast<float4*>(base + kOffNsHi + off) = hi;
    *reinterpret_cast<float4*>(base + kOffNsLo + off) = lo;
  }
}

// D = [top; bottom] * bottom^T in 3xTF32 (hi*hi + hi*lo + lo*hi), then commit to the barrier.
__device__ void ns_issue(uint32_t sbase, uint32_t tmem, uint64_t* bar) {
  tc_fence_after();
  const uint32_t id = idesc(2, 128, 64, 0, 0);
  // descriptors of the 1024-aligned bases; a K step adds its byte offset / 16 to the address field
  const uint64_t dhi = desc_sw128(sbase + kOffNsHi, 16, 1024), dlo = desc_sw128(sbase + kOffNsLo, 16, 1024);
  const uint64_t bofs = 8192 >> 4;
#pragma unroll
  for (int g = 0; g < 3; ++g) {
    const uint64_t ab = (g == 2) ? dlo : dhi;
    const uint64_t bb = ((g == 1) ? dlo : dhi) + bofs;
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
      const uint64_t koff = (uint64_t)(((ks >> 2) * 16384 + (ks & 3) * 32) >> 4);
      mma_tf32(tmem, ab + koff, bb + koff, id, (g > 0 || ks > 0) ? 1u : 0u);
    }
  }
  mma_commit(bar);
}

__device__ void solver_cta(const Params& p, const FusedArgs& fa, unsigned char* sm, uint32_t sbase,
                           uint32_t tmem, uint64_t* bars, int u) {
  const int t = threadIdx.x, w = t >> 5, lane = t & 31;
  const int m = p.m;
  float* Ls = reinterpret_cast<float*>(sm + kOffNsL);
  float* Ws = reinterpret_cast<float*>(sm + kOffNsW);
  float* Xsm = reinterpret_cast<float*>(sm + kOffNsX);
  float* vec = reinterpret_cast<float*>(sm + kOffNsVec);
  float* red = vec + 128;
  load_landmarks(p.L + (size_t)u * m * 64, Ls, m);
  __syncthreads();
  for (int e = t; e < 64 * 64; e += kFT) {
    const int a = e >> 6, b = e & 63;
    float v = 0.f;
    if (a < m && b < m) {
      float acc = 0.f;
#pragma unroll 8
      for (int k = 0; k < 64; k += 4) {
        const float4 x = *reinterpret_cast<const float4*>(&Ls[a * kQS + k]);
        const float4 y = *reinterpret_cast<const float4*>(&Ls[b * kQS + k]);
        acc += fabsf(x.x - y.x);
        acc += fabsf(x.y - y.y);
        acc += fabsf(x.z - y.z);
        acc += fabsf(x.w - y.w);
      }
      v = exp2f(acc * p.neg_log2e_over_lam) + (a == b ? p.eps : 0.f);
    }
    Ws[a * kQS + b] = v;
  }
  if (t < 64) vec[t] = t < m ? rsqrtf((float)m) : 0.f;
  __syncthreads();
  trace_mark(p, 5);
  // ||W||_2 = lambda_max (W symmetric positive definite): power iteration, 4 threads per row
  float lmax = 0.f;
  {
    const int row = t >> 2, part = t & 3;
    for (int it = 0; it <= kPowerIters; ++it) {
      float wi = 0.f;
      if (row < m) {
#pragma unroll
        for (int j = 0; j < 16; ++j) wi = fmaf(Ws[row * kQS + 16 * part + j], vec[16 * part + j], wi);
      }
      wi += __shfl_xor_sync(0xffffffffu, wi, 1);
      wi += __shfl_xor_sync(0xffffffffu, wi, 2);
      float vw = (part == 0 && row < m) ? wi * vec[row] : 0.f;
      float nn = (part == 0 && row < m) ? wi * wi : 0.f;
      block_reduce2(vw, nn, red);
      lmax = vw;
      if (it == kPowerIters) break;
      const float inv = rsqrtf(nn);
      if (part == 0 && row < 64) vec[64 + row] = row < m ? wi * inv : 0.f;
      __syncthreads();
      if (t < 64) vec[t] = vec[64 + t];
      __syncthreads();
    }
  }
  // alpha = 2/||W||_2 as printed is kept only if ||I - alpha W W^T||_2 < 1, i.e. alpha lmax^2 < 2
  const float alpha_p = 2.f / lmax;
  const int fallback = (alpha_p * lmax * lmax < 2.f) ? 0 : 1;
  const float alpha = fallback ? 1.f / (lmax * lmax) : alpha_p;
  trace_mark(p, 3);

  const int q = w & 3, h = w >> 2;
  const int r = 32 * q + lane;         // stacked row 0..127
  const int i = r & 63;                // matrix row
  const bool top = r < 64;
  const uint32_t trow = tmem + ((uint32_t)(32 * q) << 16) + 32 * h;
  uint64_t* bar = bars + kBarNs;
  int round = 0;
  float st[32], d[32];

  auto run_round = [&]() {
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    if (round == 5) trace_mark(p, 8);
    if (t == 0) ns_issue(sbase, tmem, bar);
    if (round == 5) trace_mark(p, 9);
    __syncwarp();
    mbar_wait(bar, round & 1, p.status, kStatusTimeout);
    if (round == 5) trace_mark(p, 10);
    tc_fence_after();
    tmem_ld32(trow, d);
    if (round == 5) trace_mark(p, 11);
    if (round == 0) trace_mark(p, 6);
    if (round == 10) trace_mark(p, 7);
    ++round;
  };
  auto clean = [&](float* v) {
#pragma unroll
    for (int c = 0; c < 32; ++c)
      if (i >= m || 32 * h + c >= m) v[c] = 0.f;
  };
  auto load_w_row = [&](float* v) {
#pragma unroll
    for (int c = 0; c < 32; ++c) v[c] = Ws[i * kQS + 32 * h + c];
  };

  // round 0: D_bottom = W W^T = W^2; X_0 = alpha W^T (= alpha W), R_0 = I - alpha W^2
  {
    float v[32];
    if (top) {
#pragma unroll
      for (int c = 0; c < 32; ++c) v[c] = 0.f;
    } else {
      load_w_row(v);
    }
    ns_store(sm, r, h, v);
  }
  run_round();
  if (top) {
    load_w_row(st);
#pragma unroll
    for (int c = 0; c < 32; ++c) st[c] *= alpha;
  } else {
#pragma unroll
    for (int c = 0; c < 32; ++c) st[c] = (i == 32 * h + c ? 1.f : 0.f) - alpha * d[c];
  }
  clean(st);
  const int n_lit = p.T < 2 ? p.T : 2;
  const int n_res = p.T - n_lit;
  // residual steps: A = [X; R], D = [X R^T; R R^T]
  for (int k = 0; k < n_res; ++k) {
    ns_store(sm, r, h, st);
    run_round();
    if (top) {
#pragma unroll
      for (int c = 0; c < 32; ++c) st[c] += d[c];
    } else {
#pragma unroll
      for (int c = 0; c < 32; ++c) st[c] = d[c];
    }
    clean(st);
  }
  // printed product steps X <- X (2I - W X) = X + X (I - W X), two products each
  auto stage_w_over_x = [&]() {
    // A = [W; X]: top rows W, bottom rows X (from the top threads through shared memory)
    if (top) {
#pragma unroll
      for (int c = 0; c < 32; ++c) Xsm[i * kQS + 32 * h + c] = st[c];
    }
    __syncthreads();
    float v[32];
    if (top) {
      load_w_row(v);
    } else {
#pragma unroll
      for (int c = 0; c < 32; ++c) v[c] = Xsm[i * kQS + 32 * h + c];
    }
    ns_store(sm, r, h, v);
  };
  for (int k = 0; k < n_lit; ++k) {
    stage_w_over_x();
    run_round();                       // D_top = W X
    if (top) {
      float rb[32];
#pragma unroll
      for (int c = 0; c < 32; ++c) rb[c] = (i == 32 * h + c ? 1.f : 0.f) - d[c];
      clean(rb);
      ns_store(sm, r, h, st);          // A = [X; I - W X]
      ns_store(sm, r + 64, h, rb);
    }
    run_round();                       // D_top = X (I - W X)
    if (top) {
#pragma unroll
      for (int c = 0; c < 32; ++c) st[c] += d[c];
      clean(st);
    }
  }
  // publish X_T
  if (top && i < m) {
#pragma unroll
    for (int c = 0; c < 32; ++c)
      if (32 * h + c < m) p.X[((size_t)u * m + i) * m + 32 * h + c] = st[c];
  }
  __syncthreads();
  if (t == 0) {
    __threadfence();
    st_release_u64(fa.xready + u, fa.epoch);
  }
  trace_mark(p, 4);
  // diagnostics: ||I - W X_T||_F
  stage_w_over_x();
  run_round();
  float sq = 0.f, dummy = 0.f;
  if (top && i < m) {
#pragma unroll
    for (int c = 0; c < 32; ++c)
      if (32 * h + c < m) {
        const float e = (i == 32 * h + c ? 1.f : 0.f) - d[c];
        sq += e * e;
      }
  }
  block_reduce2(sq, dummy, red);
  if (t == 0) {
    float* inf = p.info + (size_t)u * kInfoStride;
    inf[kInfoAlpha] = alpha;
    inf[kInfoLambdaMax] = lmax;
    inf[kInfoFallback] = (float)fallback;
    inf[kInfoResidual] = sqrtf(sq);
    if (!isfinite(lmax) || !isfinite(sq)) atomicOr(p.status, kStatusNonFinite);
  }
}

// ---------------------------------------------------------------------------------------
// Row CTA pieces.
// ---------------------------------------------------------------------------------------
struct Seg {
  int u;            // unit
  int lo, hi;       // token rows [lo, hi) within the unit
  int first_chunk;  // global chunk index of its first chunk
  int nch;
};

// C for a 128-row chunk: this warp's landmarks [j0, j0 + LT), lane rows lane + 32 i.
template <int LT>
__device__ __forceinline__ void cross_chunk(const float* Qs, const float* Ls, unsigned char* cslot, int j0,
                                            int nrows, float scale, float (&s1)[8], float (&s2)[8]) {
  const int lane = threadIdx.x & 31;
  float acc[4][LT];
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int b = 0; b < LT; ++b) acc[a][b] = 0.f;
#pragma unroll 2
  for (int k = 0; k < 64; k += 4) {
    float4 q[4], l[LT];
#pragma unroll
    for (int a = 0; a < 4; ++a) q[a] = *reinterpret_cast<const float4*>(&Qs[(lane + 32 * a) * kQS + k]);
#pragma unroll
    for (int b = 0; b < LT; ++b) l[b] = *reinterpret_cast<const float4*>(&Ls[(j0 + b) * kQS + k]);
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
      for (int b = 0; b < LT; ++b) {
        float s = acc[a][b];
        s += fabsf(q[a].x - l[b].x);
        s += fabsf(q[a].y - l[b].y);
        s += fabsf(q[a].z - l[b].z);
        s += fabsf(q[a].w - l[b].w);
        acc[a][b] = s;
      }
  }
#pragma unroll
  for (int a = 0; a < 4; ++a) {
    const int row = lane + 32 * a;
    const bool valid = row < nrows;
#pragma unroll
    for (int b = 0; b < LT; ++b) {
      const int col = j0 + b;
      const float c = valid ? ex2_approx(acc[a][b] * scale) : 0.f;
      s1[b] += c;
      s2[b] = fmaf(c, c, s2[b]);
      *reinterpret_cast<__nv_bfloat16*>(cslot + sw128(row, col >> 3) + ((col & 7) << 1)) = __float2bfloat16_rn(c);
    }
  }
}

__device__ __forceinline__ void cross_dispatch(int lt, const float* Qs, const float* Ls, unsigned char* cslot,
                                               int j0, int nrows, float scale, float (&s1)[8], float (&s2)[8]) {
  switch (lt) {
    case 1: cross_chunk<1>(Qs, Ls, cslot, j0, nrows, scale, s1, s2); break;
    case 2: cross_chunk<2>(Qs, Ls, cslot, j0, nrows, scale, s1, s2); break;
    case 3: cross_chunk<3>(Qs, Ls, cslot, j0, nrows, scale, s1, s2); break;
    case 4: cross_chunk<4>(Qs, Ls, cslot, j0, nrows, scale, s1, s2); break;
    case 5: cross_chunk<5>(Qs, Ls, cslot, j0, nrows, scale, s1, s2); break;
    case 6: cross_chunk<6>(Qs, Ls, cslot, j0, nrows, scale, s1, s2); break;
    case 7: cross_chunk<7>(Qs, Ls, cslot, j0, nrows, scale, s1, s2); break;
    case 8: cross_chunk<8>(Qs, Ls, cslot, j0, nrows, scale, s1, s2); break;
    default: break;
  }
}

// Q rows of a chunk: thread t loads row t/2, 32 channels (t % 2) as 4 x 16 bytes.
__device__ __forceinline__ void q_fetch(const __nv_bfloat16* Qu, int lo, int nrows, uint4 (&qr)[4]) {
  const int t = threadIdx.x, row = t >> 1, half = t & 1;
#pragma unroll
  for (int k = 0; k < 4; ++k) qr[k] = make_uint4(0u, 0u, 0u, 0u);
  if (row < nrows) {
    const uint4* src = reinterpret_cast<const uint4*>(Qu + ((size_t)(lo + row)) * 64 + 32 * half);
#pragma unroll
    for (int k = 0; k < 4; ++k) qr[k] = __ldg(src + k);
  }
}

__device__ __forceinline__ void q_stage(float* Qs, const uint4 (&qr)[4]) {
  const int t = threadIdx.x, row = t >> 1, half = t & 1;
  float* dst = Qs + row * kQS + 32 * half;
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const uint4 v = qr[k];
    *reinterpret_cast<float4*>(dst + 8 * k) = make_float4(bf_lo(v.x), bf_hi(v.x), bf_lo(v.y), bf_hi(v.y));
    *reinterpret_cast<float4*>(dst + 8 * k + 4) = make_float4(bf_lo(v.z), bf_hi(v.z), bf_lo(v.w), bf_hi(v.w));
  }
}

__global__ void __launch_bounds__(kFT, 1) k_fused_forward(const Params p, const FusedArgs fa,
                                                           const __grid_constant__ CUtensorMap tmapV) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
  unsigned char* sm = smem_raw + pad;
  const uint32_t sbase = smem_u32(sm);
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + kOffBar);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + kOffBar + 64);
  const int t = threadIdx.x, w = t >> 5, lane = t & 31;
  const int g = blockIdx.x;
  const int U = p.U, N = p.N, m = p.m;

  trace_mark(p, 0);
  trace_clock(p, 13);
  if (w == 0) {
    tmem_alloc(tmem_slot, 256);
    tmem_relinquish();
  }
  if (t == 0) {
    for (int b = 0; b < 7; ++b) mbar_init(bars + b, 1);
    mbar_init_fence();
    if (g == 0) *p.status = 0;
  }
  if (t == 32) tma_prefetch_desc(&tmapV);

  // ---- phase 0: landmark pooling, one warp per landmark ----
  // lane = (token group tg = lane / 8, 8 channels c8 = lane % 8); each load instruction of the
  // warp covers 4 window tokens x 128 bytes, all loads of a window are issued before use.
  {
    const __nv_bfloat16* Q = static_cast<const __nv_bfloat16*>(p.Q);
    const int total = U * m, Wr = p.W / p.r, rr = p.r * p.r;
    const float inv = 1.f / (float)rr;
    const int tg = lane >> 3, c8 = lane & 7;
    for (int gl = g * (kFT / 32) + w; gl < total; gl += gridDim.x * (kFT / 32)) {
      const int u = gl / m, l = gl % m;
      const int y0 = (l / Wr) * p.r, x0 = (l % Wr) * p.r;
      const __nv_bfloat16* base = Q + ((size_t)u * N) * 64 + 8 * c8;
      float a[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      for (int k0 = 0; k0 < rr; k0 += 64) {
        uint4 v[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const int k = k0 + tg + 4 * i;
          v[i] = make_uint4(0u, 0u, 0u, 0u);
          if (k < rr) {
            const int dy = k / p.r, dx = k % p.r;
            v[i] = __ldg(reinterpret_cast<const uint4*>(base + ((size_t)(y0 + dy) * p.W + x0 + dx) * 64));
          }
        }
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          a[0] += bf_lo(v[i].x); a[1] += bf_hi(v[i].x); a[2] += bf_lo(v[i].y); a[3] += bf_hi(v[i].y);
          a[4] += bf_lo(v[i].z); a[5] += bf_hi(v[i].z); a[6] += bf_lo(v[i].w); a[7] += bf_hi(v[i].w);
        }
      }
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        a[e] += __shfl_xor_sync(0xffffffffu, a[e], 8);
        a[e] += __shfl_xor_sync(0xffffffffu, a[e], 16);
      }
      if (tg == 0) {
        float* dst = p.L + ((size_t)u * m + l) * 64 + 8 * c8;
        *reinterpret_cast<float4*>(dst) = make_float4(a[0] * inv, a[1] * inv, a[2] * inv, a[3] * inv);
        *reinterpret_cast<float4*>(dst + 4) = make_float4(a[4] * inv, a[5] * inv, a[6] * inv, a[7] * inv);
      }
    }
  }
  __syncthreads();
  trace_mark(p, 1);
  if (t == 0) {
    __threadfence();
    red_release_add_u64(fa.gbar, 1ull);
    spin_until_geq(fa.gbar, fa.epoch * (unsigned long long)gridDim.x, p.status, kStatusTimeout);
  }
  __syncthreads();
  trace_mark(p, 2);
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (g < U) {
    solver_cta(p, fa, sm, sbase, tmem, bars, g);
  } else {
    // ---- row CTA ----
    const int j = g - U, n1 = fa.n1;
    const long long Trows = (long long)U * N;
    const long long r0 = row_start(j, n1, Trows), r1 = row_start(j + 1, n1, Trows);
    Seg seg[2];
    int nseg = 0;
    {
      long long a = r0;
      int fc = 0;
      while (a < r1 && nseg < 2) {
        const int u = (int)(a / N);
        const long long e = ((long long)(u + 1) * N < r1) ? (long long)(u + 1) * N : r1;
        seg[nseg].u = u;
        seg[nseg].lo = (int)(a - (long long)u * N);
        seg[nseg].hi = (int)(e - (long long)u * N);
        seg[nseg].first_chunk = fc;
        seg[nseg].nch = (seg[nseg].hi - seg[nseg].lo + kChunk - 1) / kChunk;
        fc += seg[nseg].nch;
        ++nseg;
        a = e;
      }
    }
    const int nchunks = nseg ? seg[nseg - 1].first_chunk + seg[nseg - 1].nch : 0;
    float* Qs = reinterpret_cast<float*>(sm + kOffQ);
    float* Ls = reinterpret_cast<float*>(sm + kOffL);
    const __nv_bfloat16* Qg = static_cast<const __nv_bfloat16*>(p.Q);
    // landmark groups: warps 0..extra-1 take base+1 landmarks, the rest base
    const int lbase = m / 8, lextra = m % 8;
    const int lt = lbase + (w < lextra ? 1 : 0);
    const int j0 = w * lbase + (w < lextra ? w : lextra);
    const float scale = p.neg_log2e_over_lam;

    auto chunk_of = [&](int gc, int& s, int& lo, int& nrows) {
      s = (nseg > 1 && gc >= seg[1].first_chunk) ? 1 : 0;
      const int c = gc - seg[s].first_chunk;
      lo = seg[s].lo + c * kChunk;
      nrows = min(kChunk, seg[s].hi - lo);
    };
    auto issue_v = [&](int gc) {
      int s, lo, nrows;
      chunk_of(gc, s, lo, nrows);
      uint64_t* fb = bars + kBarV + (gc & 1);
      mbar_expect_tx(fb, 16384);
      tma_load_3d(sm + kOffV + (gc & 1) * 16384, &tmapV, 0, lo, seg[s].u, fb);
    };

    // ---- phase 1b: pass 1 over all chunks ----
    uint4 qr[4];
    if (nchunks > 0) {
      int s, lo, nrows;
      chunk_of(0, s, lo, nrows);
      q_fetch(Qg + (size_t)seg[s].u * N * 64, lo, nrows, qr);
      if (t == 0) issue_v(0);
    }
    float s1[8], s2[8];
    for (int gc = 0; gc < nchunks; ++gc) {
      int s, lo, nrows;
      chunk_of(gc, s, lo, nrows);
      const int u = seg[s].u;
      const bool seg_first = gc == seg[s].first_chunk;
      const bool seg_last = gc == seg[s].first_chunk + seg[s].nch - 1;
      unsigned char* cslot = sm + kOffC + gc * 16384;
      __syncthreads();     // previous chunk's readers of Qs / Ls are done
      if (seg_first) {
        load_landmarks(p.L + (size_t)u * m * 64, Ls, m);
#pragma unroll
        for (int b = 0; b < 8; ++b) {
          s1[b] = 0.f;
          s2[b] = 0.f;
        }
      }
      q_stage(Qs, qr);
      // padding landmark columns m..63: zero, except column 63 = 1 on valid rows (sum of V)
      for (int e = t; e < kChunk * (64 - m); e += kFT) {
        const int row = e / (64 - m), col = m + e % (64 - m);
        const float v = (col == 63 && row < nrows) ? 1.f : 0.f;
        *reinterpret_cast<__nv_bfloat16*>(cslot + sw128(row, col >> 3) + ((col & 7) << 1)) = __float2bfloat16_rn(v);
      }
      __syncthreads();
      if (gc + 1 < nchunks) {
        int s2i, lo2, nr2;
        chunk_of(gc + 1, s2i, lo2, nr2);
        q_fetch(Qg + (size_t)seg[s2i].u * N * 64, lo2, nr2, qr);
        if (t == 0) {
          // stage (gc+1)&1 was last read by chunk gc-1's product
          if (gc >= 1) mbar_wait(bars + kBarP1 + ((gc + 1) & 1), ((gc - 1) >> 1) & 1, p.status, kStatusTimeout);
          issue_v(gc + 1);
        }
      }
      if (gc == 0) trace_mark(p, 10);
      if (lt > 0) cross_dispatch(lt, Qs, Ls, cslot, j0, nrows, scale, s1, s2);
      fence_async_smem();
      tc_fence_before();
      __syncthreads();
      if (gc < 2) trace_mark(p, 11 + gc);
      if (t == 0) {
        mbar_wait(bars + kBarV + (gc & 1), (gc >> 1) & 1, p.status, kStatusTimeout);
        tc_fence_after();
        const uint32_t id = idesc(1, 64, 64, 1, 1);
        const uint32_t ca = sbase + kOffC + gc * 16384, va = sbase + kOffV + (gc & 1) * 16384;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_bf16(tmem + 64 * s, desc_sw128(ca + kk * 2048, 8192, 1024), desc_sw128(va + kk * 2048, 8192, 1024),
                   id, (!seg_first || kk > 0) ? 1u : 0u);
        mma_commit(bars + kBarP1 + (gc & 1));
      }
      if (seg_last) {
        // publish this CTA's record for unit u: S1, S2 (warp shuffles) and P (TMEM)
        float* rec = fa.rec + ((size_t)j * 2 + s) * kRec;
#pragma unroll
        for (int b = 0; b < 8; ++b) {
          float a1 = s1[b], a2 = s2[b];
          for (int o = 16; o > 0; o >>= 1) {
            a1 += __shfl_xor_sync(0xffffffffu, a1, o);
            a2 += __shfl_xor_sync(0xffffffffu, a2, o);
          }
          if (lane == 0 && b < lt) {
            rec[j0 + b] = a1;
            rec[64 + j0 + b] = a2;
          }
        }
        if (t < 64 && (t >= m)) {
          rec[t] = 0.f;
          rec[64 + t] = 0.f;
        }
        mbar_wait(bars + kBarP1 + (gc & 1), (gc >> 1) & 1, p.status, kStatusTimeout);
        tc_fence_after();
        if (w < 4) {
          float v[32];
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            tmem_ld32(tmem + 64 * s + ((uint32_t)(32 * w) << 16) + 32 * hh, v);
            if (lane < 16) {
              float* dst = rec + 128 + (16 * w + lane) * 64 + 32 * hh;
#pragma unroll
              for (int c = 0; c < 32; c += 4)
                *reinterpret_cast<float4*>(dst + c) = make_float4(v[c], v[c + 1], v[c + 2], v[c + 3]);
            }
          }
        }
        tc_fence_before();
        __syncthreads();
        if (t == 0) {
          __threadfence();
          red_release_add_u64(fa.cnt + u, 1ull);
        }
      }
    }

    trace_mark(p, 3);
    // ---- phases 2 + 3 per segment ----
    float* As = reinterpret_cast<float*>(sm + kOffAs);
    float* Xt = reinterpret_cast<float*>(sm + kOffXt);
    double* S1d = reinterpret_cast<double*>(sm + kOffS1);
    double* S2d = reinterpret_cast<double*>(sm + kOffS2);
    float* mus = reinterpret_cast<float*>(sm + kOffMu);
    float* scs = reinterpret_cast<float*>(sm + kOffSc);
    float* svs = reinterpret_cast<float*>(sm + kOffSv);
    float* bps = reinterpret_cast<float*>(sm + kOffBp);
    float* bvec = reinterpret_cast<float*>(sm + kOffBv);
    float* wd = reinterpret_cast<float*>(sm + kOffWd);
    int* ctr = reinterpret_cast<int*>(sm + kOffCt);
    const float invNf = 1.f / (float)N;
    const double invN = 1.0 / (double)N;
    const bool halo_f32 = (kChunk + 2 * p.W + 2) * kQS * 4 <= (int)kHaloBytes;
    int pc = 0;    // pass-2 chunk counter (accumulator buffer parity)
    for (int s = 0; s < nseg; ++s) {
      const int u = seg[s].u;
      const __nv_bfloat16* Vu = static_cast<const __nv_bfloat16*>(p.V) + (size_t)u * N * 64;
      __nv_bfloat16* Ou = static_cast<__nv_bfloat16*>(p.O) + (size_t)u * N * 64;
      // V rows needed by chunk c's 3x3 stencil: [hlo, hhi) of unit u
      auto halo_range = [&](int c, int& hlo, int& hhi) {
        const int lo = seg[s].lo + c * kChunk, nr = min(kChunk, seg[s].hi - lo);
        hlo = max(0, lo - p.W - 1);
        hhi = min(N, lo + nr + p.W + 1);
      };
      uint4 hv[kHaloItems];
      auto halo_fetch = [&](int c) {
        int hlo, hhi;
        halo_range(c, hlo, hhi);
        const int n16 = (hhi - hlo) * 8;
        const uint4* src = reinterpret_cast<const uint4*>(Vu + (size_t)hlo * 64);
#pragma unroll
        for (int i = 0; i < kHaloItems; ++i) {
          const int e = t + kFT * i;
          hv[i] = e < n16 ? __ldg(src + e) : make_uint4(0u, 0u, 0u, 0u);
        }
      };
      auto halo_store = [&](int c) {
        int hlo, hhi;
        halo_range(c, hlo, hhi);
        const int n16 = (hhi - hlo) * 8;
#pragma unroll
        for (int i = 0; i < kHaloItems; ++i) {
          const int e = t + kFT * i;
          if (e < n16) {
            const int row = e >> 3, c8 = e & 7;
            if (halo_f32) {
              float* dst = reinterpret_cast<float*>(sm + kOffHalo) + row * kQS + 8 * c8;
              *reinterpret_cast<float4*>(dst) =
                  make_float4(bf_lo(hv[i].x), bf_hi(hv[i].x), bf_lo(hv[i].y), bf_hi(hv[i].y));
              *reinterpret_cast<float4*>(dst + 4) =
                  make_float4(bf_lo(hv[i].z), bf_hi(hv[i].z), bf_lo(hv[i].w), bf_hi(hv[i].w));
            } else {
              *reinterpret_cast<uint4*>(sm + kOffHalo + row * 144 + 16 * c8) = hv[i];
            }
          }
        }
      };
      halo_fetch(0);

      const int jf = row_cta((long long)u * N, n1, Trows);
      const int jl = row_cta((long long)(u + 1) * N - 1, n1, Trows);
      const int nct = jl - jf + 1;
      __syncthreads();
      if (t == 0) {
        spin_until_geq(fa.cnt + u, fa.epoch * (unsigned long long)nct, p.status, kStatusTimeout);
        spin_until_geq(fa.xready + u, fa.epoch, p.status, kStatusTimeout);
      }
      if (t < nct && t < 32) {
        const int jj = jf + t;
        const int sj = row_start(jj, n1, Trows) < (long long)u * N ? 1 : 0;
        ctr[t] = (jj * 2 + sj) * kRec;
      }
      __syncthreads();
      trace_mark(p, 4 + 3 * s);
      // sum the unit's records: S1, S2 in fp64, P in fp32 (float4)
      if (t < 128) {
        double acc = 0.0;
        for (int c = 0; c < nct; ++c) acc += (double)__ldcg(fa.rec + ctr[c] + t);
        if (t < 64) S1d[t] = acc;
        else S2d[t - 64] = acc;
      }
      for (int e4 = t; e4 < 1024; e4 += kFT) {
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int c = 0; c < nct; ++c) {
          const float4 v = __ldcg(reinterpret_cast<const float4*>(fa.rec + ctr[c] + 128) + e4);
          acc.x += v.x;
          acc.y += v.y;
          acc.z += v.z;
          acc.w += v.w;
        }
        *reinterpret_cast<float4*>(As + (e4 >> 4) * kQS + 4 * (e4 & 15)) = acc;
      }
      for (int e0 = t; e0 < 64 * 64; e0 += 4 * kFT) {
        float xv[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int e = e0 + kFT * i, jr = e >> 6, l = e & 63;
          xv[i] = (jr < m && l < m) ? __ldcg(p.X + ((size_t)u * m + jr) * m + l) : 0.f;
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int e = e0 + kFT * i;
          Xt[(e & 63) * kQS + (e >> 6)] = xv[i];
        }
      }
      const int head = u % p.heads;
      for (int e = t; e < 9 * 64; e += kFT) {
        const int tap = e >> 6, k = e & 63;
        wd[e] = __ldg(p.dwc + ((size_t)head * 64 + k) * 9 + tap);
      }
      __syncthreads();
      if (t < 64) {
        const double mu = S1d[t] * invN;
        double var = S2d[t] * invN - mu * mu;
        if (var < 0.0) var = 0.0;
        const double sc = 1.0 / sqrt(var + (double)p.eps);
        mus[t] = t < m ? (float)mu : 0.f;
        scs[t] = t < m ? (float)sc : 0.f;
        svs[t] = As[63 * kQS + t];       // landmark column 63 holds sum_i v_i
        if (j == jf && t < m) {
          p.mu[(size_t)u * m + t] = (float)mu;
          p.s[(size_t)u * m + t] = (float)sc;
        }
      }
      __syncthreads();
      for (int e = t; e < 64 * 64; e += kFT) {
        const int a = e >> 6, k = e & 63;
        float v = 0.f;
        if (a < m) {
          const float P = As[a * kQS + k];
          v = p.whiten ? scs[a] * (P - mus[a] * svs[k]) + svs[k] * invNf : P;
        }
        As[a * kQS + k] = v;
      }
      __syncthreads();
      {
        // M = X A with a 4 x 4 register tile per thread; M' = diag(s) M (bf16, K-major B of pass 2)
        const int jb = t >> 4, kb = t & 15;
        float acc[4][4] = {};
        for (int l = 0; l < m; ++l) {
          const float4 x4 = *reinterpret_cast<const float4*>(Xt + l * kQS + 4 * jb);
          const float4 a4 = *reinterpret_cast<const float4*>(As + l * kQS + 4 * kb);
          const float xv[4] = {x4.x, x4.y, x4.z, x4.w}, av[4] = {a4.x, a4.y, a4.z, a4.w};
#pragma unroll
          for (int x = 0; x < 4; ++x)
#pragma unroll
            for (int y = 0; y < 4; ++y) acc[x][y] = fmaf(xv[x], av[y], acc[x][y]);
        }
        unsigned char* mp = sm + kOffMp;
        float bp[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int x = 0; x < 4; ++x) {
          const int jr = 4 * jb + x;
#pragma unroll
          for (int y = 0; y < 4; ++y) {
            const int k = 4 * kb + y;
            float v = 0.f;
            if (jr < m) {
              v = p.whiten ? scs[jr] * acc[x][y] : acc[x][y];
              if (p.whiten) bp[y] += (invNf - scs[jr] * mus[jr]) * acc[x][y];
            }
            *reinterpret_cast<__nv_bfloat16*>(mp + sw128(k, jr >> 3) + ((jr & 7) << 1)) = __float2bfloat16_rn(v);
          }
        }
#pragma unroll
        for (int y = 0; y < 4; ++y) bps[jb * 64 + 4 * kb + y] = bp[y];
      }
      __syncthreads();
      if (t < 64) {
        float b = 0.f;
#pragma unroll
        for (int q = 0; q < 16; ++q) b += bps[q * 64 + t];
        bvec[t] = b;
      }
      fence_async_smem();
      tc_fence_before();
      __syncthreads();
      trace_mark(p, 5 + 3 * s);

      // phase 3: O = C M' + b + DWC(V)
      auto issue_o = [&](int gcc, int pcc) {
        tc_fence_after();
        const uint32_t id = idesc(1, 128, 64, 0, 0);
        const uint32_t ca = sbase + kOffC + gcc * 16384, mb = sbase + kOffMp;
        const uint32_t dt = tmem + 128 + 64 * (pcc & 1);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_bf16(dt, desc_sw128(ca + kk * 32, 16, 1024), desc_sw128(mb + kk * 32, 16, 1024), id, kk > 0 ? 1u : 0u);
        mma_commit(bars + kBarP2 + (pcc & 1));
      };
      if (t == 0) issue_o(seg[s].first_chunk, pc);
      for (int c = 0; c < seg[s].nch; ++c) {
        const int gc = seg[s].first_chunk + c;
        int hlo, hhi;
        halo_range(c, hlo, hhi);
        halo_store(c);
        __syncthreads();
        if (c + 1 < seg[s].nch) {
          halo_fetch(c + 1);
          if (t == 0) issue_o(gc + 1, pc + 1);
        }
        __syncwarp();
        mbar_wait(bars + kBarP2 + (pc & 1), (pc >> 1) & 1, p.status, kStatusTimeout);
        tc_fence_after();
        const int q = w & 3, h = w >> 2;
        float v[32];
        tmem_ld32(tmem + 128 + 64 * (pc & 1) + ((uint32_t)(32 * q) << 16) + 32 * h, v);
        const int lo = seg[s].lo + c * kChunk;
        const int nrows = min(kChunk, seg[s].hi - lo);
        const int row = 32 * q + lane;
        if (row < nrows) {
          const int n = lo + row, y = n / p.W, x = n % p.W;
#pragma unroll
          for (int cc = 0; cc < 32; cc += 4) {
            const float4 b4 = *reinterpret_cast<const float4*>(bvec + 32 * h + cc);
            v[cc] += b4.x;
            v[cc + 1] += b4.y;
            v[cc + 2] += b4.z;
            v[cc + 3] += b4.w;
          }
#pragma unroll
          for (int a = 0; a < 3; ++a) {
            const int yy = y + a - 1;
            if (yy < 0 || yy >= p.H) continue;
#pragma unroll
            for (int b = 0; b < 3; ++b) {
              const int xx = x + b - 1;
              if (xx < 0 || xx >= p.W) continue;
              const int hr = yy * p.W + xx - hlo;
              const float* wt = wd + (a * 3 + b) * 64 + 32 * h;
              if (halo_f32) {
                const float* vr = reinterpret_cast<const float*>(sm + kOffHalo) + hr * kQS + 32 * h;
#pragma unroll
                for (int c4 = 0; c4 < 32; c4 += 4) {
                  const float4 vv = *reinterpret_cast<const float4*>(vr + c4);
                  const float4 ww = *reinterpret_cast<const float4*>(wt + c4);
                  v[c4] = fmaf(ww.x, vv.x, v[c4]);
                  v[c4 + 1] = fmaf(ww.y, vv.y, v[c4 + 1]);
                  v[c4 + 2] = fmaf(ww.z, vv.z, v[c4 + 2]);
                  v[c4 + 3] = fmaf(ww.w, vv.w, v[c4 + 3]);
                }
              } else {
                const uint4* vr = reinterpret_cast<const uint4*>(sm + kOffHalo + hr * 144 + 64 * h);
#pragma unroll
                for (int k4 = 0; k4 < 4; ++k4) {
                  const uint4 vv = vr[k4];
                  const uint32_t wv[4] = {vv.x, vv.y, vv.z, vv.w};
#pragma unroll
                  for (int e = 0; e < 4; ++e) {
                    v[8 * k4 + 2 * e] = fmaf(wt[8 * k4 + 2 * e], bf_lo(wv[e]), v[8 * k4 + 2 * e]);
                    v[8 * k4 + 2 * e + 1] = fmaf(wt[8 * k4 + 2 * e + 1], bf_hi(wv[e]), v[8 * k4 + 2 * e + 1]);
                  }
                }
              }
            }
          }
          uint4* dst = reinterpret_cast<uint4*>(Ou + (size_t)n * 64 + 32 * h);
#pragma unroll
          for (int k4 = 0; k4 < 4; ++k4) {
            uint32_t o[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              __nv_bfloat162 pr = __floats2bfloat162_rn(v[8 * k4 + 2 * e], v[8 * k4 + 2 * e + 1]);
              o[e] = *reinterpret_cast<uint32_t*>(&pr);
            }
            dst[k4] = make_uint4(o[0], o[1], o[2], o[3]);
          }
        }
        tc_fence_before();
        __syncthreads();
        ++pc;
      }
      trace_mark(p, 6 + 3 * s);
    }
  }
  trace_mark(p, 15);
  trace_clock(p, 14);
  __syncthreads();
  if (w == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

}  // namespace

size_t fused_workspace_bytes(int U) {
  const size_t flags = 256 + 2 * 256 * (size_t)((U * 8 + 255) / 256);
  return flags + sizeof(float) * (size_t)kMaxGrid * 2 * kRec;
}

// Decide whether the fused kernel serves this shape on the current device; returns the grid size
// (0 if not eligible).
int fused_grid(const Params& p) {
  if (p.dtype != LFA_BF16 || p.d != 64 || p.m > 63 || p.m < 1) return 0;
  int dev = 0, sms = 0, coop = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  if (cudaDeviceGetAttribute(&coop, cudaDevAttrCooperativeLaunch, dev) != cudaSuccess || !coop) return 0;
  int major = 0;
  cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
  if (major != 10) return 0;
  const int G = sms < kMaxGrid ? sms : kMaxGrid;
  if (2 * p.U > G) return 0;
  if ((kChunk + 2 * p.W + 2) * 8 > kHaloItems * kFT) return 0;   // V halo of one chunk fits the prefetch
  const int n1 = G - p.U;
  const long long T = (long long)p.U * p.N;
  const long long rpc = (T + n1 - 1) / n1;
  if (rpc > (long long)(kMaxChunks - 1) * kChunk || rpc > p.N) return 0;
  if (p.N / (T / n1) + 2 > 32) return 0;     // contributors of one unit fit the offset table
  if (cudaFuncSetAttribute(k_fused_forward, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemAlloc) !=
      cudaSuccess)
    return 0;
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k_fused_forward, kFT, kSmemAlloc) != cudaSuccess ||
      per_sm < 1)
    return 0;
  return G;
}

cudaError_t launch_fused_forward(const Params& p, int G, unsigned char* fused_ws, unsigned long long epoch,
                                 cudaStream_t st) {
  if (epoch == 1) {
    const cudaError_t e = cudaMemsetAsync(fused_ws, 0, 256 + 2 * 256 * (size_t)((p.U * 8 + 255) / 256), st);
    if (e != cudaSuccess) return e;
  }
  CUtensorMap tmap;
  if (!make_tmap_rows_bf16(&tmap, p.V, (uint64_t)p.N, (uint64_t)p.U, kChunk)) return cudaErrorInvalidValue;
  FusedArgs fa;
  fa.epoch = epoch;
  fa.G = G;
  fa.n1 = G - p.U;
  fa.gbar = reinterpret_cast<unsigned long long*>(fused_ws);
  const size_t flag_stride = 256 * (size_t)((p.U * 8 + 255) / 256);
  fa.cnt = reinterpret_cast<unsigned long long*>(fused_ws + 256);
  fa.xready = reinterpret_cast<unsigned long long*>(fused_ws + 256 + flag_stride);
  fa.rec = reinterpret_cast<float*>(fused_ws + 256 + 2 * flag_stride);
  Params pp = p;
  void* args[] = {(void*)&pp, (void*)&fa, (void*)&tmap};
  if (p.ev_begin) cudaEventRecord(static_cast<cudaEvent_t>(p.ev_begin), st);
  cudaError_t e = cudaLaunchCooperativeKernel((const void*)k_fused_forward, dim3(G), dim3(kFT), args, kSmemAlloc, st);
  if (p.ev_end) cudaEventRecord(static_cast<cudaEvent_t>(p.ev_end), st);
  return e;
}

}  // namespace lfa
