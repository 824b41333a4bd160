// Fused single-launch forward pass for bf16 inputs, d = 64 and m <= 63 landmarks.
//
// One cooperative persistent kernel, one CTA per SM. Token rows of all U = B*heads units are
// split into contiguous per-CTA ranges (cut at unit boundaries into at most two segments,
// processed in 128-row chunks); CTAs 0..U-1 are the units' solver CTAs and own no rows.
//   phase 0  all CTAs: landmark pooling L = r x r average pool of Q (LaplacianFormer note,
//            §关键设计 2); arrive on a grid-wide barrier.
//   phase 1  solver CTA of unit u: W = exp(-E/lam) + eps I, ||W||_2 by power iteration, alpha
//            (§关键设计 3 with the fallback), and the T Newton-Schulz steps on tcgen05 in 3xTF32
//            (fp32-accurate): X_{k+1} = X_k + X_k R_k, R_{k+1} = R_k R_k^T (R_k = I - W X_k; the
//            same iterates in exact arithmetic, one stacked [X; R] product per step), then the
//            printed product form X (2I - W X) for the last two steps, which re-anchors R to
//            I - W X.
//   phase 2  row CTAs, pass 1 per chunk (Q rows by TMA): C = exp(-||q - l||_1 / lam) on CUDA cores
//            in fp32 (the dominant cost), kept in shared memory as bf16 for the whole kernel (never
//            in HBM);
//            per-landmark sums of C and C^2 in registers; P += C^T V on tcgen05 (V chunk staged
//            by TMA; a constant-1 landmark column 63 yields sum_i v_i in the same product).
//            Each CTA publishes one partial record per segment.
//   phase 3  solver CTA of unit u, once the unit's records are out: mu, var, s = 1/sqrt(var +
//            eps), A = C~^T V by rank-1 folding (§关键设计 1), M = X A, M' = diag(s) M,
//            b = (1/N - s o mu)^T M; M'^T (bf16, in the shared-memory image pass 2 consumes) and
//            b are published with a release flag; then the solve's diagnostics, off the
//            critical path.
//   phase 3b row CTAs, while M' is formed: DWC(V) (§关键设计 1 "ZV + DWC(V)", 3 x 3 depthwise,
//            zero padding) of every chunk from a TMA-staged V tile with a one-grid-row halo,
//            rounded to bf16 and written into the chunk's TMEM accumulator.
//   phase 4  row CTAs: O = DWC + C M' (tcgen05 accumulating onto the DWC values; all chunks'
//            products at once, one TMEM accumulator each) + b, stored once as bf16.
// Every cross-CTA wait is bounded; an expired wait sets the timeout bit of the status word.
#include <stdlib.h>
#include <string.h>

#include <mutex>

#include "lfa_internal.h"
#include "lfa_sm100.cuh"
#include "lfa_tma_host.h"

namespace lfa {
namespace {

using namespace sm100;

constexpr int kFT = 512;                  // threads per CTA (16 warps, at most 128 registers each)
constexpr int kWarps = kFT / 32;
constexpr int kV1Thread = 12 * 32;        // pass 1: issues the V chunk loads (warp 12, scheduler 0)
constexpr int kChunk = 128;               // token rows per chunk
constexpr int kMaxChunks = 8;             // resident C chunks per CTA
constexpr int kQS = 68;                   // fp32 row stride (floats) of the Q, L and halo tiles
constexpr int kRec = 128 + 64 * 64;       // floats per partial record: S1[64], S2[64], P[64][64]
constexpr int kMaxGrid = 256;             // records are sized for up to this many CTAs
constexpr int kMaxContrib = 32;           // CTAs contributing to one unit
constexpr int kPowerIters = 8;

// shared-memory map (bytes from a 1024-aligned base)
constexpr uint32_t kOffC = 0;                                   // 8 x 16 KB C chunks (SW128 rows)
constexpr uint32_t kOffV = kOffC + kMaxChunks * 16384;          // 3 x 16 KB V stages (TMA, SW128)
constexpr uint32_t kOffQ = kOffV + 2 * 16384;                   // third V stage + 18 KB spare in pass 1
constexpr uint32_t kOffL = kOffQ + kChunk * kQS * 4;            // landmarks, fp32 [64][68]
constexpr uint32_t kOffMp = kOffL + 64 * kQS * 4;               // M'^T bf16 [64 ch][64 lm] (SW128)
constexpr uint32_t kOffBv = kOffMp + 8192;                      // b, fp32 [segment][64]
constexpr uint32_t kOffBar = kOffBv + 512;                      // mbarriers + TMEM address
constexpr uint32_t kOffCt = kOffBar + 256;                      // int [32] record offsets
constexpr uint32_t kOffSr = kOffCt + 128;                       // pass-1 column sums [segment][row half][128]
constexpr uint32_t kOffRows = kOffSr + 2 * 256 * 4;            // this CTA's row plan (struct Rows)
constexpr uint32_t kSmemBytes = kOffRows + 64;
constexpr uint32_t kSmemAlloc = kSmemBytes + 1024;              // slack for 1024-byte alignment
// pass-2 scratch: V rows of one chunk with a one-grid-row halo on each side, SW128 (TMA boxes of
// 128 rows), one or two buffers in the region of the V stages, Q and L (free after pass 1)
constexpr uint32_t kOffHb = kOffV;
constexpr uint32_t kHaloSpace = kOffMp - kOffV;
constexpr int kImgBytes = 8192 + 256;                           // published M' image + b per unit
// combine scratch (aliases V/Q/L, free once pass 1 is done)
constexpr uint32_t kOffAs = kOffV;                              // fp32 [64][68]  A (row l, col k)
constexpr uint32_t kOffXt = kOffAs + 64 * kQS * 4;              // fp32 [64][68]  X^T (row l, col j)
constexpr uint32_t kOffS1 = kOffXt + 64 * kQS * 4;              // double [64]
constexpr uint32_t kOffS2 = kOffS1 + 512;                       // double [64]
constexpr uint32_t kOffMu = kOffS2 + 512;                       // float [64]
constexpr uint32_t kOffSc = kOffMu + 256;                       // float [64]
constexpr uint32_t kOffSv = kOffSc + 256;                       // float [64]
constexpr uint32_t kOffBp = kOffSv + 256;                       // float [16][64]
// solver scratch (aliases the C region: the solver runs before this CTA's pass 1)
constexpr uint32_t kOffNsHi = 0;                                // tf32 hi [2 K-halves][128 rows][128 B]
constexpr uint32_t kOffNsLo = 32768;                            // tf32 lo
constexpr uint32_t kOffNsW = 65536;                             // fp32 [64][68]
constexpr uint32_t kOffNsX = kOffNsW + 64 * kQS * 4;            // fp32 [64][68]
constexpr uint32_t kOffNsL = kOffNsX + 64 * kQS * 4;            // fp32 [64][68]
constexpr uint32_t kOffNsVec = kOffNsL + 64 * kQS * 4;          // float [2][64] + reduction [16]

static_assert(kSmemAlloc <= 232448, "shared memory over the sm_100 per-block limit");
static_assert(kOffBp + (kFT / 16) * 64 * 4 <= kOffMp, "combine scratch overlaps M'");
static_assert(kOffNsVec + 1024 <= kOffV, "solver scratch overlaps V stages");

// mbarrier slots
constexpr int kBarV = 0;      // [3] V stage filled by TMA
constexpr int kBarP1 = 3;     // [2] pass-1 product done
constexpr int kBarP2 = 5;     // [kMaxChunks] pass-2 product of chunk gc done (one use per launch)
constexpr int kBarNs = 13;    // solver product done
constexpr int kBarH = 14;     // [2] DWC V halo tile landed (TMA)
constexpr int kBarQ = 16;     // all of the CTA's pass-1 Q chunks landed (TMA)
constexpr int kBarDiag = kBarP2;       // solver CTAs (which run no pass 2): the diagnostics product
constexpr int kBarComb = kBarP2 + 1;   // solver CTAs: the combine's M = X A product
constexpr int kBarDw = 17;    // [2] DWC transfer product of staging buffer b done
constexpr int kNumBars = kBarDw + 2;
constexpr uint32_t kTmemSlot = 248;  // byte offset of the TMEM address within the barrier area
constexpr uint32_t kTmemCols = 512;  // whole TMEM: pass 2 gives every chunk its own accumulator
static_assert(kNumBars * 8 <= (int)kTmemSlot && kTmemSlot + 4 <= 256, "mbarriers overlap the TMEM address slot");

struct FusedArgs {
  unsigned long long epoch;   // launch count of this handle (>= 1); flags compare against it
  unsigned long long* gbar;   // grid barrier counter
  unsigned long long* cnt;    // [U] partial records published per unit
  unsigned long long* xready; // [U] X published (holds the epoch)
  unsigned long long* mready; // [U] M' image and b published (holds the epoch)
  float* rec;                 // [G][2][kRec]
  unsigned char* mimg;        // [U][kImgBytes] M'^T bf16 (SW128 image of the pass-2 B operand), b fp32
  // pass-1 warp plan: warp w computes landmarks [wj0[w], wj0[w] + wlt[w]) of row half w / 8;
  // warp padw[h] writes the padding columns of row half h
  unsigned char wj0[kWarps], wlt[kWarps], padw[2];
};

__device__ __forceinline__ void trace_mark(const Params& p, int slot) {
  if (p.trace != nullptr && threadIdx.x == 0) p.trace[(size_t)blockIdx.x * 32 + slot] = globaltimer();
}
__device__ __forceinline__ void trace_clock(const Params& p, int slot) {
  if (p.trace != nullptr && threadIdx.x == 0) p.trace[(size_t)blockIdx.x * 32 + slot] = (unsigned long long)clock64();
}

// Row partition. Each unit's rows are cut into nchu 128-row chunks (the last one may be short);
// the T = U nchu chunks of all units, in unit order, are dealt out evenly to the P = G - U row
// CTAs: row CTA k = g - U starts at chunk floor(T k / P). Solver CTAs (g < U) take no rows: they
// run the Newton-Schulz chain while the others compute C. No CTA gets a partial chunk mid-unit.
// 32-bit arithmetic: on the shapes the fused kernel accepts (at most kMaxChunks - 1 chunks per row
// CTA, at most kMaxGrid CTAs) T P stays below 7 kMaxGrid^2 and every row index below
// 7 kMaxGrid kChunk. (64-bit division is a long software sequence on the GPU.)
static_assert((long long)(kMaxChunks - 1) * kMaxGrid * kMaxGrid * 2 < (1ll << 31),
              "partition arithmetic overflows 32 bits");
// first global row (u N + row) of CTA g
__host__ __device__ __forceinline__ int part_start(int g, int U, int N, int G) {
  const int nchu = (N + kChunk - 1) / kChunk, T = U * nchu, P = G - U;
  const int ci = g <= U ? 0 : T * (g - U) / P;
  return (ci / nchu) * N + (ci % nchu) * kChunk;
}
__device__ __forceinline__ int cta_start(int g, const Params& p) { return part_start(g, p.U, p.N, gridDim.x); }
// CTA whose range holds global chunk C: the largest k with floor(T k / P) <= C, i.e. T k < (C + 1) P
__device__ __forceinline__ int chunk_owner(int C, const Params& p) {
  const int nchu = (p.N + kChunk - 1) / kChunk, T = p.U * nchu, P = (int)gridDim.x - p.U;
  return p.U + ((C + 1) * P - 1) / T;
}

__device__ __forceinline__ float bf_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf_hi(uint32_t v) { return __uint_as_float(v & 0xffff0000u); }
__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
  __nv_bfloat162 pr = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&pr);
}

__device__ __forceinline__ void block_reduce2(float& a, float& b, float* red) {
  for (int o = 16; o > 0; o >>= 1) {
    a += __shfl_xor_sync(0xffffffffu, a, o);
    b += __shfl_xor_sync(0xffffffffu, b, o);
  }
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  __syncthreads();
  if (lane == 0) {
    red[w] = a;
    red[kWarps + w] = b;
  }
  __syncthreads();
  a = 0.f;
  b = 0.f;
  for (int i = 0; i < kWarps; ++i) {
    a += red[i];
    b += red[kWarps + i];
  }
}

// L [m][64] fp32 (global, written by other CTAs of this launch) -> [64][kQS] shared, zero rows >= m.
__device__ __forceinline__ void load_landmarks(const float* Lg, float* Ls, int m) {
  constexpr int kN4 = 1024 / kFT;   // float4 of the [64][64] block per thread
  float4 v[kN4];
#pragma unroll
  for (int i = 0; i < kN4; ++i) {
    const int e4 = threadIdx.x + kFT * i, r = e4 >> 4;
    v[i] = r < m ? __ldcg(reinterpret_cast<const float4*>(Lg) + e4) : make_float4(0.f, 0.f, 0.f, 0.f);
  }
#pragma unroll
  for (int i = 0; i < kN4; ++i) {
    const int e4 = threadIdx.x + kFT * i;
    *reinterpret_cast<float4*>(Ls + (e4 >> 4) * kQS + 4 * (e4 & 15)) = v[i];
  }
}

struct Seg {
  int u;            // unit
  int lo, hi;       // token rows [lo, hi) within the unit
  int first_chunk;  // CTA-local index of its first chunk
  int nch;
};

struct Rows {
  Seg seg[2];
  int nseg;
  int nchunks;
  __device__ void chunk(int gc, int& s, int& lo, int& nrows) const {
    s = (nseg > 1 && gc >= seg[1].first_chunk) ? 1 : 0;
    lo = seg[s].lo + (gc - seg[s].first_chunk) * kChunk;
    nrows = min(kChunk, seg[s].hi - lo);
  }
};

__device__ Rows cta_rows(int g, const Params& p) {
  Rows R;
  const int r0 = cta_start(g, p), r1 = cta_start(g + 1, p);
  R.nseg = 0;
  int a = r0;
  int fc = 0;
  while (a < r1 && R.nseg < 2) {
    const int u = a / p.N;
    const int e = (u + 1) * p.N < r1 ? (u + 1) * p.N : r1;
    Seg& s = R.seg[R.nseg];
    s.u = u;
    s.lo = a - u * p.N;
    s.hi = e - u * p.N;
    s.first_chunk = fc;
    s.nch = (s.hi - s.lo + kChunk - 1) / kChunk;
    fc += s.nch;
    ++R.nseg;
    a = e;
  }
  R.nchunks = fc;
  return R;
}

// ---------------------------------------------------------------------------------------
// Phase 1: solver of one unit. Thread (warp w, lane) owns row r = 32 (w % 4) + lane of the
// stacked 128 x 64 operand [top; bottom] and the column quarter h = w / 4 (16 columns).
// ---------------------------------------------------------------------------------------
// The operand is stored as two K-halves of 32 fp32 columns (128-byte SW128 rows), split into
// tf32 hi and lo parts.
__device__ void ns_store(unsigned char* base, int r, int h, const float* v) {
#pragma unroll
  for (int c4 = 0; c4 < 4; ++c4) {
    float4 hi, lo;
    hi.x = tf32_round(v[4 * c4 + 0]);
    hi.y = tf32_round(v[4 * c4 + 1]);
    hi.z = tf32_round(v[4 * c4 + 2]);
    hi.w = tf32_round(v[4 * c4 + 3]);
    lo.x = v[4 * c4 + 0] - hi.x;
    lo.y = v[4 * c4 + 1] - hi.y;
    lo.z = v[4 * c4 + 2] - hi.z;
    lo.w = v[4 * c4 + 3] - hi.w;
    const uint32_t off = (h >> 1) * 16384 + sw128(r, (h & 1) * 4 + c4);
    *reinterpret_cast<float4*>(base + kOffNsHi + off) = hi;
    *reinterpret_cast<float4*>(base + kOffNsLo + off) = lo;
  }
}

// D = [top; bottom] * bottom^T over the first 8 * NKS columns, 3xTF32 (hi*hi + hi*lo + lo*hi).
template <int NKS>
__device__ __forceinline__ void ns_issue_k(uint32_t sbase, uint32_t tmem, uint64_t* bar) {
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
    for (int ks = 0; ks < NKS; ++ks) {
      const uint64_t koff = (uint64_t)(((ks >> 2) * 16384 + (ks & 3) * 32) >> 4);
      mma_tf32(tmem, ab + koff, bb + koff, id, (g > 0 || ks > 0) ? 1u : 0u);
    }
  }
  mma_commit(bar);
}

__device__ void ns_issue(uint32_t sbase, uint32_t tmem, uint64_t* bar, int nks) {
  switch (nks) {
    case 1: ns_issue_k<1>(sbase, tmem, bar); break;
    case 2: ns_issue_k<2>(sbase, tmem, bar); break;
    case 3: ns_issue_k<3>(sbase, tmem, bar); break;
    case 4: ns_issue_k<4>(sbase, tmem, bar); break;
    case 5: ns_issue_k<5>(sbase, tmem, bar); break;
    case 6: ns_issue_k<6>(sbase, tmem, bar); break;
    case 7: ns_issue_k<7>(sbase, tmem, bar); break;
    default: ns_issue_k<8>(sbase, tmem, bar); break;
  }
}

// Scalars of the solver that its diagnostics report after the combine.
struct SolverInfo {
  float alpha, lmax;
  int fallback;
};

__device__ SolverInfo solver_cta(const Params& p, const FusedArgs& fa, unsigned char* sm, uint32_t sbase,
                                 uint32_t tmem, uint64_t* bars, int u) {
  const int t = threadIdx.x, w = t >> 5, lane = t & 31;
  const int m = p.m;
  float* Ls = reinterpret_cast<float*>(sm + kOffNsL);
  float* Ws = reinterpret_cast<float*>(sm + kOffNsW);
  float* Xsm = reinterpret_cast<float*>(sm + kOffNsX);
  float* vec = reinterpret_cast<float*>(sm + kOffNsVec);
  float* red = vec + 128;
  load_landmarks(p.L + (size_t)u * m * 64, Ls, m);
  if (t < 128) vec[t] = (t & 63) < m ? 1.f : 0.f;
  __syncthreads();
  // W (symmetric): upper triangle, mirrored
  for (int e = t; e < 64 * 64; e += kFT) {
    const int a = e >> 6, b = e & 63;
    if (a > b) continue;
    float v = 0.f;
    if (b < m) {
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
      v = exp2f(acc * p.neg_log2e_over_lam);
    }
    Ws[a * kQS + b] = v + (a == b && a < m ? p.eps : 0.f);
    Ws[b * kQS + a] = v + (a == b && a < m ? p.eps : 0.f);
  }
  __syncthreads();
  trace_mark(p, 16);
  // lambda_max = ||W||_2 (W symmetric positive definite): power iteration from the ones vector,
  // scaled by 1/m per step (the Rayleigh quotient is scale free), one barrier per step
  float lmax;
  {
    const int row = t >> 3, part = t & 7;
    const float sc = 1.f / (float)m;
    float wi = 0.f;
    for (int it = 0; it <= kPowerIters; ++it) {
      const float* vin = vec + 64 * (it & 1);
      wi = 0.f;
      if (row < m) {
#pragma unroll
        for (int j = 0; j < 8; ++j) wi = fmaf(Ws[row * kQS + 8 * part + j], vin[8 * part + j], wi);
      }
      wi += __shfl_xor_sync(0xffffffffu, wi, 1);
      wi += __shfl_xor_sync(0xffffffffu, wi, 2);
      wi += __shfl_xor_sync(0xffffffffu, wi, 4);
      if (it == kPowerIters) break;
      if (part == 0) vec[64 * ((it + 1) & 1) + row] = row < m ? wi * sc : 0.f;
      __syncthreads();
    }
    const float* vl = vec + 64 * (kPowerIters & 1);
    float vw = (part == 0 && row < m) ? wi * vl[row] : 0.f;
    float vv = (part == 0 && row < m) ? vl[row] * vl[row] : 0.f;
    block_reduce2(vw, vv, red);
    lmax = vw / vv;
  }
  // alpha = 2/||W||_2 as printed is kept only if ||I - alpha W W^T||_2 < 1, i.e. alpha lmax^2 < 2
  const float alpha_p = 2.f / lmax;
  const int fallback = (alpha_p * lmax * lmax < 2.f) ? 0 : 1;
  const float alpha = fallback ? 1.f / (lmax * lmax) : alpha_p;
  trace_mark(p, 17);

  const int q = w & 3, h = w >> 2;
  const int r = 32 * q + lane;         // stacked row 0..127
  const int i = r & 63;                // matrix row
  const bool top = r < 64;
  const int nks = (m + 7) >> 3;        // K steps of 8 covering the m landmarks
  const uint32_t trow = tmem + ((uint32_t)(32 * q) << 16) + 16 * h;
  uint64_t* bar = bars + kBarNs;
  int round = 0;
  float st[16], d[16], wrow[16];
#pragma unroll
  for (int c = 0; c < 16; ++c) wrow[c] = Ws[i * kQS + 16 * h + c];

  auto run_round = [&]() {
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    if (round == 5) trace_mark(p, 20);
    if (t == 0) ns_issue(sbase, tmem, bar, nks);
    if (round == 5) trace_mark(p, 21);
    __syncwarp();
    mbar_wait(bar, round & 1, p.status, kStatusTimeout);
    if (round == 5) trace_mark(p, 22);
    tc_fence_after();
    tmem_ld16(trow, d);
    if (round == 5) trace_mark(p, 23);
    if (round == 0) trace_mark(p, 18);
    if (round == 10) trace_mark(p, 19);
    ++round;
  };
  auto clean = [&](float* v) {
#pragma unroll
    for (int c = 0; c < 16; ++c)
      if (i >= m || 16 * h + c >= m) v[c] = 0.f;
  };

  // round 0: D_bottom = W W^T = W^2; X_0 = alpha W^T (= alpha W), R_0 = I - alpha W^2
  {
    float v[16];
#pragma unroll
    for (int c = 0; c < 16; ++c) v[c] = top ? 0.f : wrow[c];
    ns_store(sm, r, h, v);
  }
  run_round();
  if (top) {
#pragma unroll
    for (int c = 0; c < 16; ++c) st[c] = alpha * wrow[c];
  } else {
#pragma unroll
    for (int c = 0; c < 16; ++c) st[c] = (i == 16 * h + c ? 1.f : 0.f) - alpha * d[c];
  }
  clean(st);
  const int n_lit = p.T < 2 ? p.T : 2;
  const int n_res = p.T - n_lit;
  // residual steps: A = [X; R], D = [X R^T; R R^T]
  for (int k = 0; k < n_res; ++k) {
    // R_k exactly zero: every remaining residual step is the identity in floating point
    // (X + X 0 = X, 0 0^T = 0), so the chain continues with the printed steps below
    bool rnz = false;
    if (!top) {
#pragma unroll
      for (int c = 0; c < 16; ++c) rnz |= st[c] != 0.f;
    }
    if (!__syncthreads_or(rnz)) break;
    ns_store(sm, r, h, st);
    run_round();
    if (top) {
#pragma unroll
      for (int c = 0; c < 16; ++c) st[c] += d[c];
    } else {
#pragma unroll
      for (int c = 0; c < 16; ++c) st[c] = d[c];
    }
    clean(st);
  }
  // printed product steps X <- X (2I - W X) = X + X (I - W X), two products each
  auto stage_w_over_x = [&]() {
    // A = [W; X]: top rows W, bottom rows X (from the top threads through shared memory)
    if (top) {
#pragma unroll
      for (int c = 0; c < 16; ++c) Xsm[i * kQS + 16 * h + c] = st[c];
    }
    __syncthreads();
    float v[16];
#pragma unroll
    for (int c = 0; c < 16; ++c) v[c] = top ? wrow[c] : Xsm[i * kQS + 16 * h + c];
    ns_store(sm, r, h, v);
  };
  for (int k = 0; k < n_lit; ++k) {
    stage_w_over_x();
    run_round();                       // D_top = W X
    if (top) {
      float rb[16];
#pragma unroll
      for (int c = 0; c < 16; ++c) rb[c] = (i == 16 * h + c ? 1.f : 0.f) - d[c];
      clean(rb);
      ns_store(sm, r, h, st);          // A = [X; I - W X]
      ns_store(sm, r + 64, h, rb);
    }
    run_round();                       // D_top = X (I - W X)
    if (top) {
#pragma unroll
      for (int c = 0; c < 16; ++c) st[c] += d[c];
      clean(st);
    }
  }
  // publish X_T; its transpose, zero outside m x m, stays in shared memory for the combine
  {
    float* Xt = reinterpret_cast<float*>(sm + kOffXt);
#pragma unroll
    for (int c = 0; c < 16; ++c) {
      const bool in = top && i < m && 16 * h + c < m;
      if (in) p.X[((size_t)u * m + i) * m + 16 * h + c] = st[c];
      if (top) Xt[(16 * h + c) * kQS + i] = in ? st[c] : 0.f;
    }
  }
  __syncthreads();
  if (t == 0) {
    __threadfence();
    st_release_u64(fa.xready + u, fa.epoch);
  }
  trace_mark(p, 24);
  tc_fence_before();
  __syncthreads();
  return SolverInfo{alpha, lmax, fallback};
}

// Diagnostics of the unit's solve, ||I - W X_T||_F, by one more product of the same kind as the
// Newton-Schulz steps ([W; X_T] times X_T^T, 3xTF32). It runs after M' is published, off the
// critical path: W is still in the solver's scratch, X_T^T in the combine's (the combine leaves
// both unchanged).
__device__ void solver_diagnostics(const Params& p, unsigned char* sm, uint32_t sbase, uint32_t tmem,
                                   uint64_t* bars, int u, const SolverInfo& si) {
  const int t = threadIdx.x, w = t >> 5, lane = t & 31;
  const int m = p.m;
  const float* Ws = reinterpret_cast<const float*>(sm + kOffNsW);
  const float* Xt = reinterpret_cast<const float*>(sm + kOffXt);
  float* red = reinterpret_cast<float*>(sm + kOffNsVec) + 128;
  const int q = w & 3, h = w >> 2;
  const int r = 32 * q + lane, i = r & 63;
  const bool top = r < 64;
  float v[16];
#pragma unroll
  for (int c = 0; c < 16; ++c) v[c] = top ? Ws[i * kQS + 16 * h + c] : Xt[(16 * h + c) * kQS + i];
  ns_store(sm, r, h, v);
  fence_async_smem();
  tc_fence_before();
  __syncthreads();
  if (t == 0) ns_issue(sbase, tmem, bars + kBarDiag, (m + 7) >> 3);
  __syncwarp();
  mbar_wait(bars + kBarDiag, 0, p.status, kStatusTimeout);
  tc_fence_after();
  float d[16];
  tmem_ld16(tmem + ((uint32_t)(32 * q) << 16) + 16 * h, d);
  float sq = 0.f, dummy = 0.f;
  if (top && i < m) {
#pragma unroll
    for (int c = 0; c < 16; ++c)
      if (16 * h + c < m) {
        const float e = (i == 16 * h + c ? 1.f : 0.f) - d[c];
        sq += e * e;
      }
  }
  block_reduce2(sq, dummy, red);
  if (t == 0) {
    float* inf = p.info + (size_t)u * kInfoStride;
    inf[kInfoAlpha] = si.alpha;
    inf[kInfoLambdaMax] = si.lmax;
    inf[kInfoFallback] = (float)si.fallback;
    inf[kInfoResidual] = sqrtf(sq);
    if (!isfinite(si.lmax) || !isfinite(sq)) atomicOr(p.status, kStatusNonFinite);
  }
  tc_fence_before();
  __syncthreads();
}

// ---------------------------------------------------------------------------------------
// Phase 3: C for a 128-row chunk: this warp's landmarks [j0, j0 + LT), lane rows lane + 32 a.
// ---------------------------------------------------------------------------------------
// Q rows come from a bf16 SW128 tile (TMA): one 16-byte read gives 8 channels of a row, and the
// lanes' rows spread the reads over all banks.
template <int LT>
__device__ __forceinline__ void cross_chunk(const unsigned char* qb, const float* Ls, unsigned char* cslot, int j0,
                                            int rb, int nrows, float scale, float (&s1)[8], float (&s2)[8]) {
  const int lane = threadIdx.x & 31;
  float acc[2][LT];
#pragma unroll
  for (int a = 0; a < 2; ++a)
#pragma unroll
    for (int b = 0; b < LT; ++b) acc[a][b] = 0.f;
#pragma unroll 2
  for (int k8 = 0; k8 < 8; ++k8) {
    float q[2][8];
#pragma unroll
    for (int a = 0; a < 2; ++a) {
      const int r = rb + lane + 32 * a;
      const uint4 raw = *reinterpret_cast<const uint4*>(qb + sw128(r, k8));
      q[a][0] = bf_lo(raw.x); q[a][1] = bf_hi(raw.x); q[a][2] = bf_lo(raw.y); q[a][3] = bf_hi(raw.y);
      q[a][4] = bf_lo(raw.z); q[a][5] = bf_hi(raw.z); q[a][6] = bf_lo(raw.w); q[a][7] = bf_hi(raw.w);
    }
#pragma unroll
    for (int h4 = 0; h4 < 2; ++h4) {
      float4 l[LT];
#pragma unroll
      for (int b = 0; b < LT; ++b) l[b] = *reinterpret_cast<const float4*>(&Ls[(j0 + b) * kQS + 8 * k8 + 4 * h4]);
#pragma unroll
      for (int a = 0; a < 2; ++a)
#pragma unroll
        for (int b = 0; b < LT; ++b) {
          float s = acc[a][b];
          s += fabsf(q[a][4 * h4 + 0] - l[b].x);
          s += fabsf(q[a][4 * h4 + 1] - l[b].y);
          s += fabsf(q[a][4 * h4 + 2] - l[b].z);
          s += fabsf(q[a][4 * h4 + 3] - l[b].w);
          acc[a][b] = s;
        }
    }
  }
  const bool even = (j0 & 1) == 0;
#pragma unroll
  for (int a = 0; a < 2; ++a) {
    const int row = rb + lane + 32 * a;
    const bool valid = row < nrows;
    float c[LT];
#pragma unroll
    for (int b = 0; b < LT; ++b) {
      c[b] = valid ? ex2_approx(acc[a][b] * scale) : 0.f;
      s1[b] += c[b];
      s2[b] = fmaf(c[b], c[b], s2[b]);
    }
    // bf16 stores, paired into 4-byte words where the landmark index is even
    if (even) {
#pragma unroll
      for (int b = 0; b < LT; b += 2) {
        const int col = j0 + b;
        unsigned char* dst = cslot + sw128(row, col >> 3) + ((col & 7) << 1);
        if (b + 1 < LT) *reinterpret_cast<uint32_t*>(dst) = pack_bf16(c[b], c[b + 1]);
        else *reinterpret_cast<__nv_bfloat16*>(dst) = __float2bfloat16_rn(c[b]);
      }
    } else {
#pragma unroll
      for (int b = 0; b < LT; ++b) {
        const int col = j0 + b;
        *reinterpret_cast<__nv_bfloat16*>(cslot + sw128(row, col >> 3) + ((col & 7) << 1)) = __float2bfloat16_rn(c[b]);
      }
    }
  }
}

// Padding columns m..63 of the rows rb + lane, rb + lane + 32: zero, except column 63 = 1 on valid
// rows (it yields sum_i v_i in the C^T V product). Whole 16-byte column groups are written at once;
// only the group that holds landmark m - 1 is written column by column.
__device__ __forceinline__ void write_padding(unsigned char* cslot, int rb, int nrows, int m) {
  const int lane = threadIdx.x & 31;
  const uint32_t one = 0x3f80u;   // bf16 1.0
#pragma unroll
  for (int a = 0; a < 2; ++a) {
    const int row = rb + lane + 32 * a;
    const bool valid = row < nrows;
    int col = m;
    for (; col < 64 && (col & 7) != 0; ++col)
      *reinterpret_cast<uint16_t*>(cslot + sw128(row, col >> 3) + ((col & 7) << 1)) =
          (col == 63 && valid) ? (uint16_t)one : (uint16_t)0;
    for (int c8 = col >> 3; c8 < 8; ++c8)
      *reinterpret_cast<uint4*>(cslot + sw128(row, c8)) = make_uint4(0u, 0u, 0u, (c8 == 7 && valid) ? (one << 16) : 0u);
  }
}

__device__ __forceinline__ void cross_dispatch(int lt, const unsigned char* Qs, const float* Ls, unsigned char* cslot,
                                               int j0, int rb, int nrows, float scale, float (&s1)[8],
                                               float (&s2)[8]) {
  switch (lt) {
    case 1: cross_chunk<1>(Qs, Ls, cslot, j0, rb, nrows, scale, s1, s2); break;
    case 2: cross_chunk<2>(Qs, Ls, cslot, j0, rb, nrows, scale, s1, s2); break;
    case 3: cross_chunk<3>(Qs, Ls, cslot, j0, rb, nrows, scale, s1, s2); break;
    case 4: cross_chunk<4>(Qs, Ls, cslot, j0, rb, nrows, scale, s1, s2); break;
    case 5: cross_chunk<5>(Qs, Ls, cslot, j0, rb, nrows, scale, s1, s2); break;
    case 6: cross_chunk<6>(Qs, Ls, cslot, j0, rb, nrows, scale, s1, s2); break;
    case 7: cross_chunk<7>(Qs, Ls, cslot, j0, rb, nrows, scale, s1, s2); break;
    case 8: cross_chunk<8>(Qs, Ls, cslot, j0, rb, nrows, scale, s1, s2); break;
    default: break;
  }
}

// Pass-1 inputs, issued by one thread while the SM is otherwise idle: every Q chunk of this CTA
// (bf16, SW128) goes to C slot gc + 1 (chunk gc writes its C tile into slot gc, which held the
// previous chunk's rows), one barrier for all of them; the first two V chunks go to stages 0, 1.
__device__ void pass1_prefetch(const Rows& R, unsigned char* sm, uint64_t* bars, const CUtensorMap* tmapV,
                               const CUtensorMap* tmapQ) {
  const int nch = R.nchunks;
  if (nch == 0) return;
  mbar_expect_tx(bars + kBarQ, (uint32_t)nch * 16384u);
  for (int gc = 0; gc < nch; ++gc) {
    int s, lo, nrows;
    R.chunk(gc, s, lo, nrows);
    tma_load_3d(sm + kOffC + (gc + 1) * 16384, tmapQ, 0, lo, R.seg[s].u, bars + kBarQ);
  }
  for (int gc = 0; gc < nch && gc < 2; ++gc) {
    int s, lo, nrows;
    R.chunk(gc, s, lo, nrows);
    mbar_expect_tx(bars + kBarV + gc, 16384);
    tma_load_3d(sm + kOffV + gc * 16384, tmapV, 0, lo, R.seg[s].u, bars + kBarV + gc);
  }
}

__device__ void pass1(const Params& p, const FusedArgs& fa, const Rows& R, unsigned char* sm, uint32_t sbase,
                      uint32_t tmem, uint64_t* bars, const CUtensorMap* tmapV) {
  const int t = threadIdx.x, w = t >> 5, lane = t & 31, g = blockIdx.x;
  const int m = p.m, nch = R.nchunks;
  float* Ls = reinterpret_cast<float*>(sm + kOffL);
  float* sred = reinterpret_cast<float*>(sm + kOffSr);   // [segment][row half][S1 64 | S2 64]
  // (constant indices only: a variable index into the parameter arrays would copy them to the stack)
  const int rh = w >> 3;
  int lt = 0, j0 = 0;
#pragma unroll
  for (int k = 0; k < kWarps; ++k)
    if (k == w) {
      lt = fa.wlt[k];
      j0 = fa.wj0[k];
    }
  const bool padder = w == (rh ? fa.padw[1] : fa.padw[0]);
  const float scale = p.neg_log2e_over_lam;
  // V chunk gc -> stage gc % 3 (its (gc / 3)-th fill)
  auto issue_v = [&](int gc) {
    int s, lo, nrows;
    R.chunk(gc, s, lo, nrows);
    uint64_t* fb = bars + kBarV + gc % 3;
    mbar_expect_tx(fb, 16384);
    tma_load_3d(sm + kOffV + (gc % 3) * 16384, tmapV, 0, lo, R.seg[s].u, fb);
  };
  // P_s += C^T V for chunk gc (M = 64 landmarks, N = 64 channels, K = 128 rows)
  auto issue_mma = [&](int gc) {
    int s, lo, nrows;
    R.chunk(gc, s, lo, nrows);
    const bool first = gc == R.seg[s].first_chunk;
    mbar_wait(bars + kBarV + gc % 3, (gc / 3) & 1, p.status, kStatusTimeout);
    tc_fence_after();
    const uint32_t id = idesc(1, 64, 64, 1, 1);
    const uint64_t ca = desc_sw128(sbase + kOffC + gc * 16384, 8192, 1024);
    const uint64_t va = desc_sw128(sbase + kOffV + (gc % 3) * 16384, 8192, 1024);
#pragma unroll
    for (int kk = 0; kk < 8; ++kk)
      mma_bf16(tmem + 64 * s, ca + (uint64_t)(kk * 2048 >> 4), va + (uint64_t)(kk * 2048 >> 4), id,
               (!first || kk > 0) ? 1u : 0u);
    mma_commit(bars + kBarP1 + (gc & 1));
  };
  // product gc done (commit gc on slot gc & 1 is that slot's (gc >> 1)-th completion)
  auto wait_mma = [&](int gc) {
    mbar_wait(bars + kBarP1 + (gc & 1), (gc >> 1) & 1, p.status, kStatusTimeout);
  };
  trace_mark(p, 28);
  float s1[8], s2[8];
  for (int gc = 0; gc < nch; ++gc) {
    int s, lo, nrows;
    R.chunk(gc, s, lo, nrows);
    const int u = R.seg[s].u;
    const bool seg_first = gc == R.seg[s].first_chunk;
    const bool seg_last = gc == R.seg[s].first_chunk + R.seg[s].nch - 1;
    unsigned char* cslot = sm + kOffC + gc * 16384;
    // products run two chunks behind: tile gc - 2 is complete and its V stage has had a chunk
    if (t == 0 && gc >= 2) issue_mma(gc - 2);
    // Ls was last read before the previous chunk's closing barrier
    if (seg_first) {
      load_landmarks(p.L + (size_t)u * m * 64, Ls, m);
#pragma unroll
      for (int b = 0; b < 8; ++b) {
        s1[b] = 0.f;
        s2[b] = 0.f;
      }
      __syncthreads();
    }
    if (gc == 0) mbar_wait(bars + kBarQ, 0, p.status, kStatusTimeout);
    if (gc < 2) trace_mark(p, 10 + 11 * gc);
    if (lt > 0) cross_dispatch(lt, sm + kOffC + (gc + 1) * 16384, Ls, cslot, j0, 64 * rh, nrows, scale, s1, s2);
    if (padder) write_padding(cslot, 64 * rh, nrows, m);
    if (gc == 1) trace_mark(p, 22);
    if (seg_last) {
      // this segment's column sums of C and C^2, per row half
#pragma unroll
      for (int b = 0; b < 8; ++b) {
        float a1 = s1[b], a2 = s2[b];
        for (int o = 16; o > 0; o >>= 1) {
          a1 += __shfl_xor_sync(0xffffffffu, a1, o);
          a2 += __shfl_xor_sync(0xffffffffu, a2, o);
        }
        if (lane == 0 && b < lt) {
          sred[256 * s + 128 * rh + j0 + b] = a1;
          sred[256 * s + 128 * rh + 64 + j0 + b] = a2;
        }
      }
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    if (gc < 2) trace_mark(p, 11 + gc);
    // the next V chunk, issued after the barrier so that this thread's proxy fence above does not
    // wait for it: stage (gc + 1) % 3 last held chunk gc - 2, whose product went out at this
    // chunk's start. Warp 12 issues it (warp 0, which issues the products, starts its distances
    // late; the other warps of its scheduler finish early).
    if (t == kV1Thread && gc >= 1 && gc + 1 < nch) {
      if (gc >= 2) wait_mma(gc - 2);
      issue_v(gc + 1);
    }
  }
  // the last two products, each waited before the next one on its commit slot goes out
  if (t == 0) {
    if (nch >= 2) issue_mma(nch - 2);
    if (nch >= 3) wait_mma(nch - 3);
    issue_mma(nch - 1);
    if (nch >= 2) wait_mma(nch - 2);
  }
  wait_mma(nch - 1);
  tc_fence_after();
  // records: S1, S2 and P (TMEM columns 64 s) per segment
  for (int s = 0; s < R.nseg; ++s) {
    float* rec = fa.rec + ((size_t)g * 2 + s) * kRec;
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
    if (t < 128) rec[t] = (t & 63) < m ? sred[256 * s + t] + sred[256 * s + 128 + t] : 0.f;
  }
  tc_fence_before();
  __syncthreads();
  if (t == 0) {
    __threadfence();
    for (int s = 0; s < R.nseg; ++s) red_release_add_u64(fa.cnt + R.seg[s].u, 1ull);
  }
}

// ---------------------------------------------------------------------------------------
// Phase 4, on the unit's solver CTA once X is known: sum the unit's records and form mu, var,
// s = 1/sqrt(var + eps), A = C~^T V by rank-1 folding (§关键设计 1), M = X A, M' = diag(s) M and
// b = (1/N - s o mu)^T M. M'^T is written as the bf16 SW128 image of pass 2's B operand and
// published with b under a release flag.
// ---------------------------------------------------------------------------------------
__device__ void solver_combine(const Params& p, const FusedArgs& fa, unsigned char* sm, uint32_t sbase,
                               uint32_t tmem, uint64_t* bars, int u) {
  const int t = threadIdx.x;
  const int m = p.m, N = p.N;
  float* As = reinterpret_cast<float*>(sm + kOffAs);
  float* Xt = reinterpret_cast<float*>(sm + kOffXt);
  double* S1d = reinterpret_cast<double*>(sm + kOffS1);
  double* S2d = reinterpret_cast<double*>(sm + kOffS2);
  float* mus = reinterpret_cast<float*>(sm + kOffMu);
  float* scs = reinterpret_cast<float*>(sm + kOffSc);
  float* svs = reinterpret_cast<float*>(sm + kOffSv);
  float* bps = reinterpret_cast<float*>(sm + kOffBp);
  int* ctr = reinterpret_cast<int*>(sm + kOffCt);
  const float invNf = 1.f / (float)N;
  const double invN = 1.0 / (double)N;
  // candidates gf..gl; CTAs with an empty range (possible when there are fewer chunks than
  // CTAs) publish nothing and are dropped from the contributor table
  const int nchu = (N + kChunk - 1) / kChunk;
  const int gf = chunk_owner(u * nchu, p);
  const int gl = chunk_owner(u * nchu + nchu - 1, p);
  const int ncand = gl - gf + 1;
  // X^T of this unit is in shared memory (written by solver_cta at publication)
  int* wcount = reinterpret_cast<int*>(sm + kOffBp);
  bool nonempty = false;
  int rec_off = 0;
  if (t < ncand) {
    const int gg = gf + t;
    const int a = cta_start(gg, p);
    nonempty = cta_start(gg + 1, p) > a;
    rec_off = (gg * 2 + (a < u * N ? 1 : 0)) * kRec;
  }
  const unsigned bal = __ballot_sync(0xffffffffu, nonempty);
  if ((t & 31) == 0) wcount[t >> 5] = __popc(bal);
  __syncthreads();
  int before = __popc(bal & ((1u << (t & 31)) - 1u)), nct = 0;
  for (int i = 0; i < kWarps; ++i) {
    if (i < (t >> 5)) before += wcount[i];
    nct += wcount[i];
  }
  if (nonempty && before < kMaxContrib) ctr[before] = rec_off;
  nct = nct < kMaxContrib ? nct : kMaxContrib;
  __syncthreads();
  if (t == 0) spin_until_geq(fa.cnt + u, fa.epoch * (unsigned long long)nct, p.status, kStatusTimeout);
  __syncthreads();
  trace_mark(p, 26);
  // sum the unit's records: S1, S2 in fp64, P in fp32. Every load of a batch of 8 records
  // (4 float4 of P per thread, plus one S value for threads < 128) is issued before any use.
  {
    constexpr int kNP = 1024 / kFT;   // float4 of P per thread
    double sacc = 0.0;
    float4 pacc[kNP];
#pragma unroll
    for (int i = 0; i < kNP; ++i) pacc[i] = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int c0 = 0; c0 < nct; c0 += 8) {
      float sv[8];
      float4 pv[8][kNP];
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        const bool ok = c0 + c < nct;
        const float* r = fa.rec + (ok ? ctr[c0 + c] : 0);
        sv[c] = (ok && t < 128) ? __ldcg(r + t) : 0.f;
#pragma unroll
        for (int i = 0; i < kNP; ++i) {
          pv[c][i] = make_float4(0.f, 0.f, 0.f, 0.f);
          if (ok) {
            const uint4 raw = ld_cg_v4_ordered(reinterpret_cast<const float4*>(r + 128) + t + kFT * i);
            pv[c][i] = make_float4(__uint_as_float(raw.x), __uint_as_float(raw.y), __uint_as_float(raw.z),
                                   __uint_as_float(raw.w));
          }
        }
      }
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        sacc += (double)sv[c];
#pragma unroll
        for (int i = 0; i < kNP; ++i) {
          pacc[i].x += pv[c][i].x;
          pacc[i].y += pv[c][i].y;
          pacc[i].z += pv[c][i].z;
          pacc[i].w += pv[c][i].w;
        }
      }
    }
    if (t < 64) S1d[t] = sacc;
    else if (t < 128) S2d[t - 64] = sacc;
    trace_mark(p, 28);
#pragma unroll
    for (int i = 0; i < kNP; ++i) {
      const int e4 = t + kFT * i;
      *reinterpret_cast<float4*>(As + (e4 >> 4) * kQS + 4 * (e4 & 15)) = pacc[i];
    }
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
    if (t < m) {
      p.mu[(size_t)u * m + t] = (float)mu;
      p.s[(size_t)u * m + t] = (float)sc;
    }
  }
  __syncthreads();
  trace_mark(p, 29);
  {
    // M = X A on tcgen05 in 3xTF32, as one product of the Newton-Schulz kind: stacked rows
    // [X; A^T] times A (its bottom half, transposed), so D_top = X A. A is folded on the fly:
    // A[l][k] = s_l (P[l][k] - mu_l sum_i v_ik) + sum_i v_ik / N. Thread (w, lane) stages row
    // r = 32 (w % 4) + lane, columns 16 (w / 4) ..
    const int w = t >> 5, lane = t & 31, q = w & 3, h = w >> 2, r = 32 * q + lane, i = r & 63;
    const bool top = r < 64;
    float v[16];
#pragma unroll
    for (int c = 0; c < 16; ++c) {
      const int l = 16 * h + c;
      if (top) {
        v[c] = Xt[l * kQS + i];
      } else {
        float a = 0.f;
        if (l < m) {
          const float P = As[l * kQS + i];
          a = p.whiten ? scs[l] * (P - mus[l] * svs[i]) + svs[i] * invNf : P;
        }
        v[c] = a;
      }
    }
    ns_store(sm, r, h, v);
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    if (t == 0) ns_issue(sbase, tmem, bars + kBarComb, (m + 7) >> 3);
    __syncwarp();
    mbar_wait(bars + kBarComb, 0, p.status, kStatusTimeout);
    tc_fence_after();
    float d[16];
    tmem_ld16(tmem + ((uint32_t)(32 * q) << 16) + 16 * h, d);
    if (top) {
      // M' = diag(s) M as bf16 (K-major B of pass 2: image row k = channel, column i = landmark,
      // zero for i >= m); b = (1/N - s o mu)^T M, reduced over the 64 rows
      const bool in = i < m;
      const float sc = in ? (p.whiten ? scs[i] : 1.f) : 0.f;
      const float wb = (in && p.whiten) ? invNf - scs[i] * mus[i] : 0.f;
      unsigned char* mp = sm + kOffMp;
      float bp[16];
#pragma unroll
      for (int c = 0; c < 16; ++c) {
        *reinterpret_cast<__nv_bfloat16*>(mp + sw128(16 * h + c, i >> 3) + ((i & 7) << 1)) =
            __float2bfloat16_rn(sc * d[c]);
        bp[c] = wb * d[c];
      }
#pragma unroll
      for (int c = 0; c < 16; ++c)
        for (int o = 16; o > 0; o >>= 1) bp[c] += __shfl_xor_sync(0xffffffffu, bp[c], o);
      if (lane == 0) {
#pragma unroll
        for (int c = 0; c < 16; ++c) bps[q * 64 + 16 * h + c] = bp[c];
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  trace_mark(p, 30);
  unsigned char* img = fa.mimg + (size_t)u * kImgBytes;
  if (t < 64) {
    float b = 0.f;
#pragma unroll
    for (int q = 0; q < 2; ++q) b += bps[q * 64 + t];
    reinterpret_cast<float*>(img + 8192)[t] = b;
  }
  for (int e = t; e < 512; e += kFT)
    reinterpret_cast<uint4*>(img)[e] = reinterpret_cast<const uint4*>(sm + kOffMp)[e];
  __syncthreads();
  if (t == 0) {
    __threadfence();
    st_release_u64(fa.mready + u, fa.epoch);
  }
  trace_mark(p, 27);
}

// ---------------------------------------------------------------------------------------
// Phase 3b (row CTAs, while the unit's M' is being formed): DWC(V) of every chunk, the 3 x 3
// depthwise taps (§关键设计 1 "ZV + DWC(V)", zero padding 1), rounded to bf16 and placed in the
// chunk's pass-2 TMEM accumulator (columns 64 gc), on which pass 2's product then accumulates.
// The chunk's V rows with a one-grid-row halo on each side arrive by TMA (SW128, boxes of 128
// rows, rows outside the unit read as zero), two chunks in flight where both tiles fit. Thread t
// owns 4 consecutive tokens of one grid row (W % 4 == 0, so a group never wraps) and 4 channels
// (t % 16), weights in registers, and slides the 3 x 6 input window along the group. The results
// go to a bf16 staging tile (SW128 rows, two alternating buffers), which one tcgen05 product with a
// 64 x 64 identity (exact: every product is by 1 or 0, summed in fp32) copies into the chunk's TMEM
// accumulator.
// ---------------------------------------------------------------------------------------
__device__ void dwc_all(const Params& p, const Rows& R, unsigned char* sm, uint32_t sbase, uint32_t tmem,
                        uint64_t* bars, const CUtensorMap* tmapV) {
  const int t = threadIdx.x, W = p.W;
  const int nbox = (kChunk + 2 * (W + 1) + kChunk - 1) / kChunk;
  const uint32_t hbytes = (uint32_t)nbox * 16384u;
  const int nbuf = 2 * hbytes + 16384 <= kHaloSpace ? 2 : 1;
  const int nch = R.nchunks;
  // staging buffers: C slot kMaxChunks - 1 (free: a CTA has at most kMaxChunks - 1 chunks, and the
  // Q tile that slot held is consumed) and the halo region after the halo buffers
  unsigned char* stg[2] = {sm + kOffC + (kMaxChunks - 1) * 16384, sm + kOffHb + nbuf * hbytes};
  auto issue = [&](int gc) {
    int s, lo, nrows;
    R.chunk(gc, s, lo, nrows);
    const int bi = gc % nbuf;
    uint64_t* hb = bars + kBarH + bi;
    mbar_expect_tx(hb, hbytes);
    for (int b = 0; b < nbox; ++b)
      tma_load_3d(sm + kOffHb + bi * hbytes + b * 16384, tmapV, 0, lo - (W + 1) + kChunk * b, R.seg[s].u, hb);
  };
  // staged chunk gc -> its TMEM accumulator (columns 64 gc): D = S I over K = 64 channels, the
  // identity (K-major B) in the M' area, which pass 2 fills only later
  auto transfer = [&](int gc) {
    tc_fence_after();
    const uint32_t id = idesc(1, 128, 64, 0, 0);
    const uint64_t sa = desc_sw128(sbase + (uint32_t)(stg[gc & 1] - sm), 16, 1024);
    const uint64_t ib = desc_sw128(sbase + kOffMp, 16, 1024);
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) mma_bf16(tmem + 64 * gc, sa + (uint64_t)(kk * 2), ib + (uint64_t)(kk * 2), id, kk > 0 ? 1u : 0u);
    mma_commit(bars + kBarDw + (gc & 1));
  };
  // transfer gc (the (gc >> 1)-th completion of its buffer's barrier) done
  auto wait_transfer = [&](int gc) {
    mbar_wait(bars + kBarDw + (gc & 1), (gc >> 1) & 1, p.status, kStatusTimeout);
  };
  __syncthreads();   // pass 1 is done with the V stages, Q and L (the halo region), and with TMEM
  if (t == 0) {
    issue(0);
    if (nbuf == 2 && nch > 1) issue(1);
  }
  // the 64 x 64 bf16 identity, SW128 rows (row n, column k): 512 16-byte groups
  for (int e = t; e < 512; e += kFT) {
    const int n = e >> 3, c8 = e & 7;
    const uint32_t one = 0x3f80u << (16 * (n & 1));
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if ((n >> 3) == c8) {
      const int word = (n & 7) >> 1;
      if (word == 0) v.x = one;
      else if (word == 1) v.y = one;
      else if (word == 2) v.z = one;
      else v.w = one;
    }
    *reinterpret_cast<uint4*>(sm + kOffMp + sw128(n, c8)) = v;
  }
  const int grp = t >> 4, c4 = t & 15;   // tokens 4 grp .. 4 grp + 3 of the chunk, channels 4 c4 ..
  float wt[9][4];
  int head = -1;
  for (int gc = 0; gc < nch; ++gc) {
    int s, lo, nrows;
    R.chunk(gc, s, lo, nrows);
    const int u = R.seg[s].u;
    if (u % p.heads != head) {
      head = u % p.heads;
#pragma unroll
      for (int tap = 0; tap < 9; ++tap)
#pragma unroll
        for (int e = 0; e < 4; ++e) wt[tap][e] = __ldg(p.dwc + ((size_t)head * 64 + 4 * c4 + e) * 9 + tap);
    }
    const int bi = gc % nbuf;
    mbar_wait(bars + kBarH + bi, (gc / nbuf) & 1, p.status, kStatusTimeout);   // fill gc / nbuf of buffer bi
    const int r0 = 4 * grp;                // chunk row of the group's first token
    float acc[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[i][e] = 0.f;
    if (r0 < nrows) {
      const int n0 = lo + r0, x0 = n0 % W;
      const unsigned char* hbuf = sm + kOffHb + bi * hbytes;
#pragma unroll
      for (int a = 0; a < 3; ++a) {
        // tile rows of tokens x0 - 1 .. x0 + 4 on grid row y + a - 1: r0 + a W + j, j = 0..5
        float v[6][4];
#pragma unroll
        for (int j = 0; j < 6; ++j) {
          const int tr = r0 + a * W + j;
          const bool inside = (j > 0 || x0 > 0) && (j < 5 || x0 + 4 < W);
          uint2 raw = make_uint2(0u, 0u);
          if (inside)
            raw = *reinterpret_cast<const uint2*>(hbuf + tr * 128 + ((((c4 >> 1) ^ (tr & 7))) << 4) + (c4 & 1) * 8);
          v[j][0] = bf_lo(raw.x);
          v[j][1] = bf_hi(raw.x);
          v[j][2] = bf_lo(raw.y);
          v[j][3] = bf_hi(raw.y);
        }
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int b = 0; b < 3; ++b)
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[i][e] = fmaf(wt[a * 3 + b][e], v[i + b][e], acc[i][e]);
      }
    }
    // rows past the chunk's end stage zeros (their accumulator rows are never stored); staging
    // buffer gc & 1 was last read by transfer gc - 2
    if (gc >= 2) wait_transfer(gc - 2);
    unsigned char* st = stg[gc & 1];
#pragma unroll
    for (int i = 0; i < 4; ++i)
      *reinterpret_cast<uint2*>(st + sw128(r0 + i, c4 >> 1) + (c4 & 1) * 8) =
          make_uint2(pack_bf16(acc[i][0], acc[i][1]), pack_bf16(acc[i][2], acc[i][3]));
    fence_async_smem();
    __syncthreads();   // staging gc written (and, at gc = 0, the identity), halo buffer bi read
    // two issuing threads in different warps, so that neither warp's chunk is late by both
    if (t == 0) transfer(gc);
    if (t == 32 && gc + nbuf < nch) issue(gc + nbuf);
  }
  // the last transfers (earlier ones were waited before their buffer was reused)
  if (nch >= 2) wait_transfer(nch - 2);
  if (nch >= 1) wait_transfer(nch - 1);
  tc_fence_before();
  __syncthreads();
  trace_mark(p, 25);
}

// ---------------------------------------------------------------------------------------
// Phase 4: O = C M' + b + DWC(V) for every chunk. M'^T and b of each segment's unit come from
// its solver CTA (segment 0's image in the M' area, segment 1's in the free halo region). Each
// chunk's product accumulates onto the DWC values already in its TMEM accumulator (phase 3b); all
// products are issued at once, each with its own barrier, and the epilogues (+ b, bf16) follow
// chunk by chunk. The bf16 rows are staged in the chunk's C slot (free once its product is done)
// and leave by TMA stores of 32-row quarters: warps w, w + 4, w + 8, w + 12 hold the same 32 rows
// (16 channels each) and meet on named barrier 1 + w % 4 before warp w % 4 issues the quarter's
// store.
// ---------------------------------------------------------------------------------------
__device__ void pass2_all(const Params& p, const FusedArgs& fa, const Rows& R, unsigned char* sm, uint32_t sbase,
                          uint32_t tmem, uint64_t* bars, const CUtensorMap* tmapO) {
  const int t = threadIdx.x, w = t >> 5, lane = t & 31;
  const int nch = R.nchunks;
  float* bvec = reinterpret_cast<float*>(sm + kOffBv);
  auto img_off = [](int s) -> uint32_t { return s == 0 ? kOffMp : kOffV; };
  if (t == 0)
    for (int s = 0; s < R.nseg; ++s) spin_until_geq(fa.mready + R.seg[s].u, fa.epoch, p.status, kStatusTimeout);
  __syncthreads();
  trace_mark(p, 4);
  for (int s = 0; s < R.nseg; ++s) {
    const unsigned char* img = fa.mimg + (size_t)R.seg[s].u * kImgBytes;
    for (int e = t; e < 512; e += kFT)
      reinterpret_cast<uint4*>(sm + img_off(s))[e] = __ldcg(reinterpret_cast<const uint4*>(img) + e);
    if (t < 64) bvec[64 * s + t] = __ldcg(reinterpret_cast<const float*>(img + 8192) + t);
  }
  fence_async_smem();
  tc_fence_before();
  __syncthreads();
  trace_mark(p, 5);
  // one thread (in warp 15, which issues no stores) issues the products in chunk order, each
  // chunk's four followed by its commit, so the epilogues can start while later chunks are issued
  if (t == kFT - 32) {
    tc_fence_after();
    const uint32_t id = idesc(1, 128, 64, 0, 0);
    for (int gc = 0; gc < nch; ++gc) {
      int s, lo, nrows;
      R.chunk(gc, s, lo, nrows);
      const uint64_t ca = desc_sw128(sbase + kOffC + gc * 16384, 16, 1024);
      const uint64_t mb = desc_sw128(sbase + img_off(s), 16, 1024);
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
        mma_bf16(tmem + 64 * gc, ca + (uint64_t)(kk * 2), mb + (uint64_t)(kk * 2), id, 1u);
      mma_commit(bars + kBarP2 + gc);
    }
  }
  const int q = w & 3, h = w >> 2, row = 32 * q + lane;
  for (int gc = 0; gc < nch; ++gc) {
    int s, lo, nrows;
    R.chunk(gc, s, lo, nrows);
    mbar_wait(bars + kBarP2 + gc, 0, p.status, kStatusTimeout);
    if (gc == 0) trace_mark(p, 29);
    tc_fence_after();
    float v[16];
    tmem_ld16(tmem + 64 * gc + ((uint32_t)(32 * q) << 16) + 16 * h, v);
    unsigned char* ob = sm + kOffC + gc * 16384;
    const float* bs = bvec + 64 * s + 16 * h;
#pragma unroll
    for (int k4 = 0; k4 < 2; ++k4) {
      uint32_t o[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int cc = 8 * k4 + 2 * e;
        o[e] = pack_bf16(v[cc] + bs[cc], v[cc + 1] + bs[cc + 1]);
      }
      *reinterpret_cast<uint4*>(ob + sw128(row, 2 * h + k4)) = make_uint4(o[0], o[1], o[2], o[3]);
    }
    fence_async_smem();
    named_bar_sync(1 + q, 128);
    // rows past the unit's end (a short last chunk) fall outside the tensor and are not written
    if (h == 0 && lane == 0 && 32 * q < nrows) {
      tma_store_3d(tmapO, 0, lo + 32 * q, R.seg[s].u, ob + 4096 * q);
      bulk_commit_group();
    }
    if (gc < 2) trace_mark(p, 30 + gc);
  }
  if (h == 0 && lane == 0) bulk_wait_all();
  tc_fence_before();
  __syncthreads();
  trace_mark(p, 6);
}

__global__ void __launch_bounds__(kFT, 1) k_fused_forward(const Params p, const FusedArgs fa,
                                                           const __grid_constant__ CUtensorMap tmapV,
                                                           const __grid_constant__ CUtensorMap tmapQ,
                                                           const __grid_constant__ CUtensorMap tmapO) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
  unsigned char* sm = smem_raw + pad;
  const uint32_t sbase = smem_u32(sm);
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + kOffBar);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + kOffBar + kTmemSlot);
  const int t = threadIdx.x, w = t >> 5, lane = t & 31;
  const int g = blockIdx.x;
  const int U = p.U, N = p.N, m = p.m;

  trace_mark(p, 0);
  trace_clock(p, 13);
  if (w == 0) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  // the row plan lives in shared memory: it is read at every chunk boundary by every thread
  Rows* Rsm = reinterpret_cast<Rows*>(sm + kOffRows);
  if (t == 0) *Rsm = cta_rows(g, p);
  const Rows& R = *Rsm;
  const bool solver = g < U;
  if (t == 0) {
    for (int b = 0; b < kNumBars; ++b) mbar_init(bars + b, 1);
    mbar_init_fence();
    if (g == 0) *p.status = 0;
    if (!solver) pass1_prefetch(R, sm, bars, &tmapV, &tmapQ);
  }
  if (t == 32) {
    tma_prefetch_desc(&tmapV);
    tma_prefetch_desc(&tmapQ);
    tma_prefetch_desc(&tmapO);
  }

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
  }
  if (t == 0) spin_until_geq(fa.gbar, fa.epoch * (unsigned long long)gridDim.x, p.status, kStatusTimeout);
  __syncthreads();
  trace_mark(p, 2);
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  // solver CTAs take no rows (R.nchunks == 0): solve, combine, then the diagnostics
  if (solver) {
    const SolverInfo si = solver_cta(p, fa, sm, sbase, tmem, bars, g);
    trace_mark(p, 3);
    solver_combine(p, fa, sm, sbase, tmem, bars, g);
    solver_diagnostics(p, sm, sbase, tmem, bars, g, si);
  }
  if (R.nchunks > 0) pass1(p, fa, R, sm, sbase, tmem, bars, &tmapV);
  if (!solver) trace_mark(p, 3);
  if (R.nchunks > 0) dwc_all(p, R, sm, sbase, tmem, bars, &tmapV);
  if (R.nchunks > 0) pass2_all(p, fa, R, sm, sbase, tmem, bars, &tmapO);
  __syncthreads();
  trace_mark(p, 15);
  trace_clock(p, 14);
  if (w == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace

// Flag area: grid barrier (256 B), then three [U] flag arrays (cnt, xready, mready), each padded
// to 256 B; then the per-CTA records and the per-unit M' images.
static size_t flag_stride(int U) { return 256 * (size_t)((U * 8 + 255) / 256); }
static size_t flag_bytes(int U) { return 256 + 3 * flag_stride(U); }

size_t fused_workspace_bytes(int U) {
  return flag_bytes(U) + sizeof(float) * (size_t)kMaxGrid * 2 * kRec + (size_t)U * kImgBytes;
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
  // chunks of a row CTA: resident C capacity, and at most two units (segments) per CTA
  const long long nchu = (p.N + kChunk - 1) / kChunk;
  const long long cpc = ((long long)p.U * nchu + (G - p.U) - 1) / (G - p.U);
  if (cpc > kMaxChunks - 1 || cpc > nchu) return 0;   // one C slot stays free for the Q chunk
  // the DWC phase's token groups of 4 stay on one grid row
  if (p.W % 4 != 0) return 0;
  // its V halo tile (a chunk plus one grid row on each side, in boxes of 128 rows) and one DWC
  // staging tile must fit the halo region
  if ((long long)((kChunk + 2 * (p.W + 1) + kChunk - 1) / kChunk) * 16384 + 16384 > (long long)kHaloSpace) return 0;
  // replay the row partition: contributors of every unit must fit the offset table
  {
    int worst = 0, cur_u = -1, cur = 0;
    for (int g = 0; g < G; ++g) {
      const int r0 = part_start(g, p.U, p.N, G);
      const int r1 = part_start(g + 1, p.U, p.N, G);
      if (r1 <= r0) continue;
      for (int u = r0 / p.N; u <= (r1 - 1) / p.N; ++u) {
        if ((int)u != cur_u) {
          cur_u = (int)u;
          cur = 0;
        }
        if (++cur > worst) worst = cur;
      }
    }
    if (worst > kMaxContrib) return 0;
  }
  if (cudaFuncSetAttribute(k_fused_forward, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemAlloc) !=
      cudaSuccess)
    return 0;
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k_fused_forward, kFT, kSmemAlloc) != cudaSuccess ||
      per_sm < 1)
    return 0;
  return G;
}

// Tensor maps of recently used V pointers (host side; encoding costs a driver call).
constexpr int kTmapCache = 32;   // Q, V and O maps of a few rotating buffer sets
struct TmapCache {
  const void* ptr[kTmapCache];
  int N[kTmapCache], U[kTmapCache], sw[kTmapCache], box[kTmapCache];
  CUtensorMap map[kTmapCache];
  int next;
};
static TmapCache g_tmaps;
static std::mutex g_tmaps_mu;

// [U][N][64] bf16 viewed as {64, N, U}, boxes of box_rows rows; 128-byte swizzle or plain rows
static bool tmap_for(const void* X, int N, int U, int box_rows, bool swizzle, CUtensorMap* out) {
  std::lock_guard<std::mutex> lk(g_tmaps_mu);
  for (int i = 0; i < kTmapCache; ++i)
    if (g_tmaps.ptr[i] == X && g_tmaps.N[i] == N && g_tmaps.U[i] == U && g_tmaps.sw[i] == (int)swizzle &&
        g_tmaps.box[i] == box_rows) {
      *out = g_tmaps.map[i];
      return true;
    }
  CUtensorMap m;
  if (!make_tmap_rows_bf16(&m, X, (uint64_t)N, (uint64_t)U, (uint32_t)box_rows, swizzle)) return false;
  const int i = g_tmaps.next;
  g_tmaps.next = (i + 1) % kTmapCache;
  g_tmaps.ptr[i] = X;
  g_tmaps.N[i] = N;
  g_tmaps.U[i] = U;
  g_tmaps.sw[i] = (int)swizzle;
  g_tmaps.box[i] = box_rows;
  g_tmaps.map[i] = m;
  *out = m;
  return true;
}

// Pass-1 warp plan. Each row half's m landmarks are cut into 8 contiguous ranges, one per warp of
// that half (warps 0-7 take rows 0-63, warps 8-15 rows 64-127); warp w issues on scheduler w % 4,
// which therefore serves four ranges. Every range gets b = m / 8 landmarks; the e = m % 8 ranges of
// each half that take one more go to the least-loaded scheduler, scheduler 0 counted one landmark
// heavier because its warp 0 also issues the chunk products. Each half's padding columns go to
// scheduler 0's other warp of that half (warps 4 and 8): warp 0 starts its distances late while it
// issues the products, so the other warps of its scheduler finish first.
static void plan_pass1_warps(int m, FusedArgs& fa) {
  const int b = m / 8, e = m % 8;
  int sz[kWarps], load[4] = {1, 0, 0, 0};
  for (int w = 0; w < kWarps; ++w) {
    sz[w] = b;
    load[w % 4] += b;
  }
  for (int i = 0; i < 2 * e; ++i) {
    const int half = i % 2;
    int best = -1;
    for (int k = 0; k < 8; ++k) {
      const int w = 8 * half + k;
      if (sz[w] != b || w == 0) continue;
      if (best < 0 || load[w % 4] < load[best % 4]) best = w;
    }
    if (best < 0) best = 0;   // only when every other warp of half 0 already has b + 1
    ++sz[best];
    ++load[best % 4];
  }
  for (int half = 0; half < 2; ++half) {
    int j = 0;
    for (int k = 0; k < 8; ++k) {
      const int w = 8 * half + k;
      fa.wj0[w] = (unsigned char)j;
      fa.wlt[w] = (unsigned char)sz[w];
      j += sz[w];
    }
    fa.padw[half] = (unsigned char)(half == 0 ? 4 : 8);
  }
}

cudaError_t launch_fused_forward(const Params& p, int G, unsigned char* fused_ws, unsigned long long epoch,
                                 cudaStream_t st) {
  if (epoch == 1) {
    const cudaError_t e = cudaMemsetAsync(fused_ws, 0, flag_bytes(p.U), st);
    if (e != cudaSuccess) return e;
  }
  CUtensorMap tmap, tmapq, tmapo;
  if (!tmap_for(p.V, p.N, p.U, kChunk, true, &tmap)) return cudaErrorInvalidValue;
  if (!tmap_for(p.Q, p.N, p.U, kChunk, true, &tmapq)) return cudaErrorInvalidValue;
  if (!tmap_for(p.O, p.N, p.U, 32, true, &tmapo)) return cudaErrorInvalidValue;
  FusedArgs fa;
  fa.epoch = epoch;
  fa.gbar = reinterpret_cast<unsigned long long*>(fused_ws);
  const size_t fs = flag_stride(p.U);
  fa.cnt = reinterpret_cast<unsigned long long*>(fused_ws + 256);
  fa.xready = reinterpret_cast<unsigned long long*>(fused_ws + 256 + fs);
  fa.mready = reinterpret_cast<unsigned long long*>(fused_ws + 256 + 2 * fs);
  fa.rec = reinterpret_cast<float*>(fused_ws + flag_bytes(p.U));
  fa.mimg = fused_ws + flag_bytes(p.U) + sizeof(float) * (size_t)kMaxGrid * 2 * kRec;
  plan_pass1_warps(p.m, fa);
  Params pp = p;
  void* args[] = {(void*)&pp, (void*)&fa, (void*)&tmap, (void*)&tmapq, (void*)&tmapo};
  if (p.ev_begin) cudaEventRecord(static_cast<cudaEvent_t>(p.ev_begin), st);
  cudaError_t e = cudaLaunchCooperativeKernel((const void*)k_fused_forward, dim3(G), dim3(kFT), args, kSmemAlloc, st);
  if (p.ev_end) cudaEventRecord(static_cast<cudaEvent_t>(p.ev_end), st);
  return e;
}

}  // namespace lfa
