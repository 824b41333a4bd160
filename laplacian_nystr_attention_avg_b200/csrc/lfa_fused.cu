// Fused single-launch forward pass for bf16 inputs, d = 64 and m <= 63 landmarks.
//
// One cooperative persistent kernel, one CTA per SM. Token rows of all U = B*heads units are
// split into contiguous per-CTA ranges (cut at unit boundaries into at most two segments,
// processed in 128-row chunks).
//   phase 0  all CTAs: landmark pooling L = r x r average pool of Q (LaplacianFormer note,
//            §关键设计 2); arrive on a grid-wide barrier.
//   phase 1  while the barrier completes: DWC(V) of the CTA's own rows (3x3 depthwise, zero
//            padding; §关键设计 1 "ZV + DWC(V)") written to O as bf16.
//   phase 2  CTAs 0..U-1 first run one unit's solver each: W = exp(-E/lam) + eps I, ||W||_2 by
//            power iteration, alpha (§关键设计 3 with the fallback), and the T Newton-Schulz
//            steps on tcgen05 in 3xTF32 (fp32-accurate): X_{k+1} = X_k + X_k R_k,
//            R_{k+1} = R_k R_k^T (R_k = I - W X_k; the same iterates in exact arithmetic, one
//            stacked [X; R] product per step), then the printed product form X (2I - W X) for
//            the last two steps, which re-anchors R to I - W X. X is published with a release
//            flag. (These CTAs own a smaller row share and do their DWC afterwards.)
//   phase 3  pass 1 per chunk: C = exp(-||q - l||_1 / lam) on CUDA cores in fp32 (the dominant
//            cost), kept in shared memory as bf16 for the whole kernel (never in HBM);
//            per-landmark sums of C and C^2 in registers; P += C^T V on tcgen05 (V chunk staged
//            by TMA; a constant-1 landmark column 63 yields sum_i v_i in the same product).
//            Each CTA publishes one partial record per segment.
//   phase 4  per unit, every CTA of the unit sums the unit's records and forms mu, var,
//            s = 1/sqrt(var + eps), A = C~^T V by rank-1 folding (§关键设计 1), M = X A,
//            M' = diag(s) M, b = (1/N - s o mu)^T M.
//   phase 5  per chunk: O = C M' (tcgen05, TMEM accumulator) + b + DWC(V) (read back), bf16.
// Every cross-CTA wait is bounded; an expired wait sets the timeout bit of the status word.
#include <stdlib.h>
#include <string.h>

#include "lfa_internal.h"
#include "lfa_sm100.cuh"
#include "lfa_tma_host.h"

namespace lfa {
namespace {

using namespace sm100;

constexpr int kFT = 256;                  // threads per CTA (8 warps)
constexpr int kChunk = 128;               // token rows per chunk
constexpr int kMaxChunks = 8;             // resident C chunks per CTA
constexpr int kQS = 68;                   // fp32 row stride (floats) of the Q, L and halo tiles
constexpr int kRec = 128 + 64 * 64;       // floats per partial record: S1[64], S2[64], P[64][64]
constexpr int kMaxGrid = 256;             // records are sized for up to this many CTAs
constexpr int kMaxContrib = 32;           // CTAs contributing to one unit
constexpr int kPowerIters = 8;

// shared-memory map (bytes from a 1024-aligned base)
constexpr uint32_t kOffC = 0;                                   // 8 x 16 KB C chunks (SW128 rows)
constexpr uint32_t kOffV = kOffC + kMaxChunks * 16384;          // 2 x 16 KB V stages (TMA, SW128)
constexpr uint32_t kOffQ = kOffV + 2 * 16384;                   // Q chunk, fp32 [128][68]
constexpr uint32_t kOffL = kOffQ + kChunk * kQS * 4;            // landmarks, fp32 [64][68]
constexpr uint32_t kOffMp = kOffL + 64 * kQS * 4;               // M'^T bf16 [64 ch][64 lm] (SW128)
constexpr uint32_t kOffBv = kOffMp + 8192;                      // b, fp32 [64]
constexpr uint32_t kOffBar = kOffBv + 256;                      // mbarriers + TMEM address
constexpr uint32_t kOffCt = kOffBar + 128;                      // int [32] record offsets
constexpr uint32_t kSmemBytes = kOffCt + 128;
constexpr uint32_t kSmemAlloc = kSmemBytes + 1024;              // slack for 1024-byte alignment
// phase-1 scratch: the V rows (with a one-grid-row halo) of this CTA's segments, bf16 [rows][64]
// (plain 128-byte rows, TMA without swizzle), in the region below M' that pass 1 fills later
constexpr uint32_t kOffHalo = kOffC;
constexpr int kHaloRows = (int)(kOffMp / 128);
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
static_assert(kOffBp + 16 * 64 * 4 <= kOffMp, "combine scratch overlaps M'");
static_assert(kOffNsVec + 1024 <= kOffV, "solver scratch overlaps V stages");

// mbarrier slots
constexpr int kBarV = 0;      // [2] V stage filled by TMA
constexpr int kBarP1 = 2;     // [2] pass-1 product done (stage free)
constexpr int kBarP2 = 4;     // [2] pass-2 product done (accumulator ready)
constexpr int kBarNs = 6;     // solver product done
constexpr int kBarDwc = 7;    // DWC halo rows landed (TMA)

struct FusedArgs {
  unsigned long long epoch;   // launch count of this handle (>= 1); flags compare against it
  int ws16;                   // row share of a solver CTA in 1/16 of a plain CTA's share
  int totw16;                 // ws16 * U + 16 * (G - U)
  unsigned long long* gbar;   // grid barrier counter
  unsigned long long* cnt;    // [U] partial records published per unit
  unsigned long long* xready; // [U] X published (holds the epoch)
  float* rec;                 // [G][2][kRec]
};

__device__ __forceinline__ void trace_mark(const Params& p, int slot) {
  if (p.trace != nullptr && threadIdx.x == 0) p.trace[(size_t)blockIdx.x * 32 + slot] = globaltimer();
}
__device__ __forceinline__ void trace_clock(const Params& p, int slot) {
  if (p.trace != nullptr && threadIdx.x == 0) p.trace[(size_t)blockIdx.x * 32 + slot] = (unsigned long long)clock64();
}

// first global row of CTA g (rows weighted: solver CTAs ws16/16 of a plain CTA)
__device__ __forceinline__ long long cta_start(int g, int U, const FusedArgs& fa, long long T) {
  const long long cw = g <= U ? (long long)fa.ws16 * g : (long long)fa.ws16 * U + 16ll * (g - U);
  return T * cw / fa.totw16;
}
// CTA whose range holds global row R
__device__ __forceinline__ int cta_of_row(long long R, int U, int G, const FusedArgs& fa, long long T) {
  int lo = 0, hi = G - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (cta_start(mid, U, fa, T) <= R) lo = mid;
    else hi = mid - 1;
  }
  return lo;
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

__device__ Rows cta_rows(int g, const Params& p, const FusedArgs& fa) {
  Rows R;
  const long long T = (long long)p.U * p.N;
  const long long r0 = cta_start(g, p.U, fa, T), r1 = cta_start(g + 1, p.U, fa, T);
  R.nseg = 0;
  long long a = r0;
  int fc = 0;
  while (a < r1 && R.nseg < 2) {
    const int u = (int)(a / p.N);
    const long long e = ((long long)(u + 1) * p.N < r1) ? (long long)(u + 1) * p.N : r1;
    Seg& s = R.seg[R.nseg];
    s.u = u;
    s.lo = (int)(a - (long long)u * p.N);
    s.hi = (int)(e - (long long)u * p.N);
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
// Phase 1: DWC(V) of this CTA's rows -> O (bf16). The V rows of each segment, with a
// one-grid-row halo, are brought in by TMA (plain rows) in one batch; each thread then owns
// 4 consecutive tokens of a grid row x 4 channels (weights in registers) and slides a
// 3 x 6 window over the tile.
// ---------------------------------------------------------------------------------------
struct HaloPlan {
  int hlo[2];    // first unit row of each segment's halo range
  int hhi[2];
  int base[2];   // tile row holding row hlo
  int rows;      // tile rows in use
};

__device__ __forceinline__ HaloPlan halo_plan(const Params& p, const Rows& R) {
  HaloPlan h;
  int base = 0;
  for (int s = 0; s < 2; ++s) {
    h.hlo[s] = h.hhi[s] = h.base[s] = 0;
    if (s >= R.nseg) continue;
    h.hlo[s] = max(0, R.seg[s].lo - p.W - 1);
    h.hhi[s] = min(p.N, R.seg[s].hi + p.W + 1);
    h.base[s] = base;
    base += (h.hhi[s] - h.hlo[s] + kChunk - 1) / kChunk * kChunk;
  }
  h.rows = base;
  return h;
}

// one thread: TMA loads of every segment's halo rows into the tile, completing on kBarDwc
__device__ void dwc_issue(const Params& p, const Rows& R, const HaloPlan& h, unsigned char* sm, uint64_t* bars,
                          const CUtensorMap* tmapVp) {
  if (h.rows == 0) return;
  fence_async_smem();
  mbar_expect_tx(bars + kBarDwc, (uint32_t)h.rows * 128u);
  for (int s = 0; s < R.nseg; ++s) {
    const int nb = (h.hhi[s] - h.hlo[s] + kChunk - 1) / kChunk;
    for (int b = 0; b < nb; ++b)
      tma_load_3d(sm + kOffHalo + (size_t)(h.base[s] + b * kChunk) * 128, tmapVp, 0, h.hlo[s] + b * kChunk, R.seg[s].u,
                  bars + kBarDwc);
  }
}

__device__ void dwc_compute(const Params& p, const Rows& R, const HaloPlan& h, const unsigned char* sm) {
  const int t = threadIdx.x, cq = t & 15, slot = t >> 4;
  const int W = p.W, H = p.H;
  const int runs = (W + 3) >> 2;
  __nv_bfloat16* O = static_cast<__nv_bfloat16*>(p.O);
  float wt[9][4];
  int head = -1;
  for (int s = 0; s < R.nseg; ++s) {
    const int u = R.seg[s].u, lo = R.seg[s].lo, hi = R.seg[s].hi;
    const int hlo = h.hlo[s], hhi = h.hhi[s], base = h.base[s];
    if (u % p.heads != head) {
      head = u % p.heads;
#pragma unroll
      for (int tap = 0; tap < 9; ++tap)
#pragma unroll
        for (int e = 0; e < 4; ++e) wt[tap][e] = __ldg(p.dwc + ((size_t)head * 64 + 4 * cq + e) * 9 + tap);
    }
    const int ylo = lo / W, yhi = (hi - 1) / W;
    const int nitems = (yhi - ylo + 1) * runs;
    __nv_bfloat16* Ou = O + (size_t)u * p.N * 64 + 4 * cq;
    for (int item = slot; item < nitems; item += kFT / 16) {
      const int y = ylo + item / runs, x0 = (item % runs) * 4;
      float v[3][6][4];
#pragma unroll
      for (int a = 0; a < 3; ++a) {
        const int yy = y + a - 1;
        const bool rv = yy >= 0 && yy < H;
#pragma unroll
        for (int b = 0; b < 6; ++b) {
          const int xx = x0 + b - 1;
          const int n2 = yy * W + xx;
          float4 f = make_float4(0.f, 0.f, 0.f, 0.f);
          if (rv && xx >= 0 && xx < W && n2 >= hlo && n2 < hhi) {
            const uint2 raw = *reinterpret_cast<const uint2*>(sm + kOffHalo + (size_t)(n2 - hlo + base) * 128 + 8 * cq);
            f = make_float4(bf_lo(raw.x), bf_hi(raw.x), bf_lo(raw.y), bf_hi(raw.y));
          }
          v[a][b][0] = f.x;
          v[a][b][1] = f.y;
          v[a][b][2] = f.z;
          v[a][b][3] = f.w;
        }
      }
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int x = x0 + j, n = y * W + x;
        if (x >= W || n < lo || n >= hi) continue;
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int a = 0; a < 3; ++a)
#pragma unroll
          for (int b = 0; b < 3; ++b)
#pragma unroll
            for (int c = 0; c < 4; ++c) acc[c] = fmaf(wt[a * 3 + b][c], v[a][j + b][c], acc[c]);
        *reinterpret_cast<uint2*>(Ou + (size_t)n * 64) = make_uint2(pack_bf16(acc[0], acc[1]), pack_bf16(acc[2], acc[3]));
      }
    }
  }
}

// ---------------------------------------------------------------------------------------
// Phase 2: solver of one unit. Thread (warp w, lane) owns row r = 32 (w % 4) + lane of the
// stacked 128 x 64 operand [top; bottom] and the column half h = w / 4.
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
    const int row = t >> 2, part = t & 3;
    const float sc = 1.f / (float)m;
    float wi = 0.f;
    for (int it = 0; it <= kPowerIters; ++it) {
      const float* vin = vec + 64 * (it & 1);
      wi = 0.f;
      if (row < m) {
#pragma unroll
        for (int j = 0; j < 16; ++j) wi = fmaf(Ws[row * kQS + 16 * part + j], vin[16 * part + j], wi);
      }
      wi += __shfl_xor_sync(0xffffffffu, wi, 1);
      wi += __shfl_xor_sync(0xffffffffu, wi, 2);
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
  const uint32_t trow = tmem + ((uint32_t)(32 * q) << 16) + 32 * h;
  uint64_t* bar = bars + kBarNs;
  int round = 0;
  float st[32], d[32], wrow[32];
#pragma unroll
  for (int c = 0; c < 32; ++c) wrow[c] = Ws[i * kQS + 32 * h + c];

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
    tmem_ld32(trow, d);
    if (round == 5) trace_mark(p, 23);
    if (round == 0) trace_mark(p, 18);
    if (round == 10) trace_mark(p, 19);
    ++round;
  };
  auto clean = [&](float* v) {
#pragma unroll
    for (int c = 0; c < 32; ++c)
      if (i >= m || 32 * h + c >= m) v[c] = 0.f;
  };

  // round 0: D_bottom = W W^T = W^2; X_0 = alpha W^T (= alpha W), R_0 = I - alpha W^2
  {
    float v[32];
#pragma unroll
    for (int c = 0; c < 32; ++c) v[c] = top ? 0.f : wrow[c];
    ns_store(sm, r, h, v);
  }
  run_round();
  if (top) {
#pragma unroll
    for (int c = 0; c < 32; ++c) st[c] = alpha * wrow[c];
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
#pragma unroll
    for (int c = 0; c < 32; ++c) v[c] = top ? wrow[c] : Xsm[i * kQS + 32 * h + c];
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
  trace_mark(p, 24);
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
  tc_fence_before();
  __syncthreads();
}

// ---------------------------------------------------------------------------------------
// Phase 3: C for a 128-row chunk: this warp's landmarks [j0, j0 + LT), lane rows lane + 32 a.
// ---------------------------------------------------------------------------------------
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
  const bool even = (j0 & 1) == 0;
#pragma unroll
  for (int a = 0; a < 4; ++a) {
    const int row = lane + 32 * a;
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

__device__ void pass1(const Params& p, const FusedArgs& fa, const Rows& R, unsigned char* sm, uint32_t sbase,
                      uint32_t tmem, uint64_t* bars, const CUtensorMap* tmapV) {
  const int t = threadIdx.x, w = t >> 5, lane = t & 31, g = blockIdx.x;
  const int m = p.m, N = p.N;
  float* Qs = reinterpret_cast<float*>(sm + kOffQ);
  float* Ls = reinterpret_cast<float*>(sm + kOffL);
  const __nv_bfloat16* Qg = static_cast<const __nv_bfloat16*>(p.Q);
  // landmark groups: 8 warps, the m % 8 larger groups last so that every group starts at an
  // even landmark when m / 8 is even (paired C stores)
  const int lbase = m / 8, lextra = m % 8;
  const int big = 8 - lextra;           // warps >= big take lbase + 1 landmarks
  const int lt = lbase + (w >= big ? 1 : 0);
  const int j0 = w * lbase + (w > big ? w - big : 0);
  const float scale = p.neg_log2e_over_lam;
  auto issue_v = [&](int gc) {
    int s, lo, nrows;
    R.chunk(gc, s, lo, nrows);
    uint64_t* fb = bars + kBarV + (gc & 1);
    mbar_expect_tx(fb, 16384);
    tma_load_3d(sm + kOffV + (gc & 1) * 16384, tmapV, 0, lo, R.seg[s].u, fb);
  };
  uint4 qr[4];
  {
    int s, lo, nrows;
    R.chunk(0, s, lo, nrows);
    q_fetch(Qg + (size_t)R.seg[s].u * N * 64, lo, nrows, qr);
    if (t == 0) {
      fence_async_smem();     // the V stages were read by generic loads (DWC tile) before
      issue_v(0);
    }
  }
  float s1[8], s2[8];
  for (int gc = 0; gc < R.nchunks; ++gc) {
    int s, lo, nrows;
    R.chunk(gc, s, lo, nrows);
    const int u = R.seg[s].u;
    const bool seg_first = gc == R.seg[s].first_chunk;
    const bool seg_last = gc == R.seg[s].first_chunk + R.seg[s].nch - 1;
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
    if (gc + 1 < R.nchunks) {
      int s2i, lo2, nr2;
      R.chunk(gc + 1, s2i, lo2, nr2);
      q_fetch(Qg + (size_t)R.seg[s2i].u * N * 64, lo2, nr2, qr);
    }
    if (gc == 0) trace_mark(p, 10);
    if (lt > 0) cross_dispatch(lt, Qs, Ls, cslot, j0, nrows, scale, s1, s2);
    // the other V stage was last read by chunk gc-1's product, committed long before here
    if (t == 0 && gc + 1 < R.nchunks) {
      if (gc >= 1) mbar_wait(bars + kBarP1 + ((gc + 1) & 1), ((gc - 1) >> 1) & 1, p.status, kStatusTimeout);
      issue_v(gc + 1);
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    if (gc < 2) trace_mark(p, 11 + gc);
    if (t == 0) {
      mbar_wait(bars + kBarV + (gc & 1), (gc >> 1) & 1, p.status, kStatusTimeout);
      tc_fence_after();
      const uint32_t id = idesc(1, 64, 64, 1, 1);
      const uint64_t ca = desc_sw128(sbase + kOffC + gc * 16384, 8192, 1024);
      const uint64_t va = desc_sw128(sbase + kOffV + (gc & 1) * 16384, 8192, 1024);
#pragma unroll
      for (int kk = 0; kk < 8; ++kk)
        mma_bf16(tmem + 64 * s, ca + (uint64_t)(kk * 2048 >> 4), va + (uint64_t)(kk * 2048 >> 4), id,
                 (!seg_first || kk > 0) ? 1u : 0u);
      mma_commit(bars + kBarP1 + (gc & 1));
    }
    if (seg_last) {
      // publish this CTA's record for unit u: S1, S2 (warp shuffles) and P (TMEM)
      float* rec = fa.rec + ((size_t)g * 2 + s) * kRec;
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
      if (t < 64 && t >= m) {
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
}

// ---------------------------------------------------------------------------------------
// Phases 4 + 5 for one segment: combine the unit's records, then O = C M' + b + DWC.
// ---------------------------------------------------------------------------------------
__device__ void combine_and_pass2(const Params& p, const FusedArgs& fa, const Rows& R, int s, int& pc,
                                  unsigned char* sm, uint32_t sbase, uint32_t tmem, uint64_t* bars) {
  const int t = threadIdx.x, w = t >> 5, lane = t & 31, g = blockIdx.x;
  const int m = p.m, N = p.N, U = p.U, G = gridDim.x;
  const long long Trows = (long long)U * N;
  float* As = reinterpret_cast<float*>(sm + kOffAs);
  float* Xt = reinterpret_cast<float*>(sm + kOffXt);
  double* S1d = reinterpret_cast<double*>(sm + kOffS1);
  double* S2d = reinterpret_cast<double*>(sm + kOffS2);
  float* mus = reinterpret_cast<float*>(sm + kOffMu);
  float* scs = reinterpret_cast<float*>(sm + kOffSc);
  float* svs = reinterpret_cast<float*>(sm + kOffSv);
  float* bps = reinterpret_cast<float*>(sm + kOffBp);
  float* bvec = reinterpret_cast<float*>(sm + kOffBv);
  int* ctr = reinterpret_cast<int*>(sm + kOffCt);
  const float invNf = 1.f / (float)N;
  const double invN = 1.0 / (double)N;
  const int u = R.seg[s].u;
  const int gf = cta_of_row((long long)u * N, U, G, fa, Trows);
  const int gl = cta_of_row((long long)(u + 1) * N - 1, U, G, fa, Trows);
  const int nct = gl - gf + 1;
  __syncthreads();
  if (t == 0) {
    spin_until_geq(fa.cnt + u, fa.epoch * (unsigned long long)nct, p.status, kStatusTimeout);
    spin_until_geq(fa.xready + u, fa.epoch, p.status, kStatusTimeout);
  }
  if (t < nct && t < kMaxContrib) {
    const int gg = gf + t;
    const int sj = cta_start(gg, U, fa, Trows) < (long long)u * N ? 1 : 0;
    ctr[t] = (gg * 2 + sj) * kRec;
  }
  __syncthreads();
  trace_mark(p, 4 + 3 * s);
  // sum the unit's records: S1, S2 in fp64, P in fp32 (float4), eight records in flight
  if (t < 128) {
    double acc = 0.0;
    for (int c0 = 0; c0 < nct; c0 += 8) {
      float v[8];
#pragma unroll
      for (int c = 0; c < 8; ++c) v[c] = c0 + c < nct ? __ldcg(fa.rec + ctr[c0 + c] + t) : 0.f;
#pragma unroll
      for (int c = 0; c < 8; ++c) acc += (double)v[c];
    }
    if (t < 64) S1d[t] = acc;
    else S2d[t - 64] = acc;
  }
  for (int e4 = t; e4 < 1024; e4 += kFT) {
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int c0 = 0; c0 < nct; c0 += 8) {
      float4 v[8];
#pragma unroll
      for (int c = 0; c < 8; ++c)
        v[c] = c0 + c < nct ? __ldcg(reinterpret_cast<const float4*>(fa.rec + ctr[c0 + c] + 128) + e4)
                            : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        acc.x += v[c].x;
        acc.y += v[c].y;
        acc.z += v[c].z;
        acc.w += v[c].w;
      }
    }
    *reinterpret_cast<float4*>(As + (e4 >> 4) * kQS + 4 * (e4 & 15)) = acc;
  }
  {
    float xv[16];
#pragma unroll
    for (int i2 = 0; i2 < 16; ++i2) {
      const int e = t + kFT * i2, jr = e >> 6, l = e & 63;
      xv[i2] = (jr < m && l < m) ? __ldcg(p.X + ((size_t)u * m + jr) * m + l) : 0.f;
    }
#pragma unroll
    for (int i2 = 0; i2 < 16; ++i2) {
      const int e = t + kFT * i2;
      Xt[(e & 63) * kQS + (e >> 6)] = xv[i2];
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
    if (g == gf && t < m) {
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

  // phase 5: O = C M' + b + DWC(V); the DWC values are in O already (phase 1)
  __nv_bfloat16* Ou = static_cast<__nv_bfloat16*>(p.O) + (size_t)u * N * 64;
  auto issue_o = [&](int gcc, int pcc) {
    tc_fence_after();
    const uint32_t id = idesc(1, 128, 64, 0, 0);
    const uint64_t ca = desc_sw128(sbase + kOffC + gcc * 16384, 16, 1024);
    const uint64_t mb = desc_sw128(sbase + kOffMp, 16, 1024);
    const uint32_t dt = tmem + 128 + 64 * (pcc & 1);
#pragma unroll
    for (int kk = 0; kk < 4; ++kk)
      mma_bf16(dt, ca + (uint64_t)(kk * 2), mb + (uint64_t)(kk * 2), id, kk > 0 ? 1u : 0u);
    mma_commit(bars + kBarP2 + (pcc & 1));
  };
  const int q = w & 3, h = w >> 2, row = 32 * q + lane;
  if (t == 0) issue_o(R.seg[s].first_chunk, pc);
  for (int c = 0; c < R.seg[s].nch; ++c) {
    const int gc = R.seg[s].first_chunk + c;
    const int lo = R.seg[s].lo + c * kChunk;
    const int nrows = min(kChunk, R.seg[s].hi - lo);
    if (t == 0 && c + 1 < R.seg[s].nch) issue_o(gc + 1, pc + 1);
    uint4 dw[4];
    uint4* orow = reinterpret_cast<uint4*>(Ou + (size_t)(lo + row) * 64 + 32 * h);
#pragma unroll
    for (int k4 = 0; k4 < 4; ++k4) dw[k4] = row < nrows ? orow[k4] : make_uint4(0u, 0u, 0u, 0u);
    __syncwarp();
    mbar_wait(bars + kBarP2 + (pc & 1), (pc >> 1) & 1, p.status, kStatusTimeout);
    tc_fence_after();
    float v[32];
    tmem_ld32(tmem + 128 + 64 * (pc & 1) + ((uint32_t)(32 * q) << 16) + 32 * h, v);
    if (row < nrows) {
#pragma unroll
      for (int k4 = 0; k4 < 4; ++k4) {
        const uint32_t wv[4] = {dw[k4].x, dw[k4].y, dw[k4].z, dw[k4].w};
        uint32_t o[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int cc = 8 * k4 + 2 * e;
          o[e] = pack_bf16(v[cc] + bvec[32 * h + cc] + bf_lo(wv[e]), v[cc + 1] + bvec[32 * h + cc + 1] + bf_hi(wv[e]));
        }
        orow[k4] = make_uint4(o[0], o[1], o[2], o[3]);
      }
    }
    tc_fence_before();
    __syncthreads();
    ++pc;
  }
  trace_mark(p, 6 + 3 * s);
}

__global__ void __launch_bounds__(kFT, 1) k_fused_forward(const Params p, const FusedArgs fa,
                                                           const __grid_constant__ CUtensorMap tmapV,
                                                           const __grid_constant__ CUtensorMap tmapVp) {
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
  const Rows R = cta_rows(g, p, fa);
  const bool solver = g < U;
  const HaloPlan hp = halo_plan(p, R);
  if (t == 0) {
    for (int b = 0; b < 8; ++b) mbar_init(bars + b, 1);
    mbar_init_fence();
    if (g == 0) *p.status = 0;
    // V rows for this CTA's DWC: in flight while pooling runs (solver CTAs: after their solver)
    if (!solver) dwc_issue(p, R, hp, sm, bars, &tmapVp);
  }
  if (t == 32) {
    tma_prefetch_desc(&tmapV);
    tma_prefetch_desc(&tmapVp);
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
  // ---- phase 1: DWC of this CTA's rows while the barrier completes (solver CTAs: later) ----
  if (!solver && hp.rows > 0) {
    mbar_wait(bars + kBarDwc, 0, p.status, kStatusTimeout);
    dwc_compute(p, R, hp, sm);
  }
  trace_mark(p, 25);
  if (t == 0) spin_until_geq(fa.gbar, fa.epoch * (unsigned long long)gridDim.x, p.status, kStatusTimeout);
  __syncthreads();
  trace_mark(p, 2);
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (solver) {
    solver_cta(p, fa, sm, sbase, tmem, bars, g);
    if (hp.rows > 0) {
      if (t == 0) dwc_issue(p, R, hp, sm, bars, &tmapVp);
      mbar_wait(bars + kBarDwc, 0, p.status, kStatusTimeout);
      dwc_compute(p, R, hp, sm);
    }
  }
  __syncthreads();
  if (R.nchunks > 0) pass1(p, fa, R, sm, sbase, tmem, bars, &tmapV);
  trace_mark(p, 3);
  int pc = 0;
  for (int s = 0; s < R.nseg; ++s) combine_and_pass2(p, fa, R, s, pc, sm, sbase, tmem, bars);
  __syncthreads();
  trace_mark(p, 15);
  trace_clock(p, 14);
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

// Row share of a solver CTA (in 1/16 of a plain CTA's share): they start their rows only after
// the Newton-Schulz chain. LFA_SOLVER_ROW_SHARE (0..16) overrides the default.
static int solver_share16() {
  const char* e = getenv("LFA_SOLVER_ROW_SHARE");
  if (e) {
    const int v = atoi(e);
    if (v >= 0 && v <= 16) return v;
  }
  return 0;
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
  const int ws16 = solver_share16();
  const long long totw16 = (long long)ws16 * p.U + 16ll * (G - p.U);
  const long long T = (long long)p.U * p.N;
  const long long rpc = (T * 16 + totw16 - 1) / totw16;           // rows of a plain CTA (rounded up)
  if (rpc > (long long)(kMaxChunks - 1) * kChunk || rpc > p.N) return 0;
  // replay the row partition: contributors of every unit must fit the offset table and every
  // CTA's DWC rows (segments plus one-grid-row halos, rounded to TMA boxes) must fit the tile
  {
    int worst = 0, cur_u = -1, cur = 0;
    for (int g = 0; g < G; ++g) {
      const long long cw0 = g <= p.U ? (long long)ws16 * g : (long long)ws16 * p.U + 16ll * (g - p.U);
      const long long cw1 = g + 1 <= p.U ? (long long)ws16 * (g + 1) : (long long)ws16 * p.U + 16ll * (g + 1 - p.U);
      const long long r0 = T * cw0 / totw16, r1 = T * cw1 / totw16;
      if (r1 <= r0) continue;
      long long halo_rows = 0;
      for (long long u = r0 / p.N; u <= (r1 - 1) / p.N; ++u) {
        if ((int)u != cur_u) {
          cur_u = (int)u;
          cur = 0;
        }
        if (++cur > worst) worst = cur;
        const long long lo = (r0 > u * p.N ? r0 : u * p.N) - u * p.N;
        const long long hi = (r1 < (u + 1) * p.N ? r1 : (u + 1) * p.N) - u * p.N;
        const long long hlo = lo - p.W - 1 > 0 ? lo - p.W - 1 : 0;
        const long long hhi = hi + p.W + 1 < p.N ? hi + p.W + 1 : p.N;
        halo_rows += (hhi - hlo + kChunk - 1) / kChunk * kChunk;
      }
      if (halo_rows > kHaloRows) return 0;
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
struct TmapCache {
  const void* ptr[8];
  int N[8], U[8];
  CUtensorMap map[8], plain[8];
  int next;
};
static TmapCache g_tmaps;

static bool tmap_for(const void* V, int N, int U, CUtensorMap* out, CUtensorMap* out_plain) {
  for (int i = 0; i < 8; ++i)
    if (g_tmaps.ptr[i] == V && g_tmaps.N[i] == N && g_tmaps.U[i] == U) {
      *out = g_tmaps.map[i];
      *out_plain = g_tmaps.plain[i];
      return true;
    }
  CUtensorMap m, mp;
  if (!make_tmap_rows_bf16(&m, V, (uint64_t)N, (uint64_t)U, kChunk, true)) return false;
  if (!make_tmap_rows_bf16(&mp, V, (uint64_t)N, (uint64_t)U, kChunk, false)) return false;
  const int i = g_tmaps.next;
  g_tmaps.next = (i + 1) & 7;
  g_tmaps.ptr[i] = V;
  g_tmaps.N[i] = N;
  g_tmaps.U[i] = U;
  g_tmaps.map[i] = m;
  g_tmaps.plain[i] = mp;
  *out = m;
  *out_plain = mp;
  return true;
}

cudaError_t launch_fused_forward(const Params& p, int G, unsigned char* fused_ws, unsigned long long epoch,
                                 cudaStream_t st) {
  if (epoch == 1) {
    const cudaError_t e = cudaMemsetAsync(fused_ws, 0, 256 + 2 * 256 * (size_t)((p.U * 8 + 255) / 256), st);
    if (e != cudaSuccess) return e;
  }
  CUtensorMap tmap, tmapp;
  if (!tmap_for(p.V, p.N, p.U, &tmap, &tmapp)) return cudaErrorInvalidValue;
  FusedArgs fa;
  fa.epoch = epoch;
  fa.ws16 = solver_share16();
  fa.totw16 = fa.ws16 * p.U + 16 * (G - p.U);
  fa.gbar = reinterpret_cast<unsigned long long*>(fused_ws);
  const size_t flag_stride = 256 * (size_t)((p.U * 8 + 255) / 256);
  fa.cnt = reinterpret_cast<unsigned long long*>(fused_ws + 256);
  fa.xready = reinterpret_cast<unsigned long long*>(fused_ws + 256 + flag_stride);
  fa.rec = reinterpret_cast<float*>(fused_ws + 256 + 2 * flag_stride);
  Params pp = p;
  void* args[] = {(void*)&pp, (void*)&fa, (void*)&tmap, (void*)&tmapp};
  if (p.ev_begin) cudaEventRecord(static_cast<cudaEvent_t>(p.ev_begin), st);
  cudaError_t e = cudaLaunchCooperativeKernel((const void*)k_fused_forward, dim3(G), dim3(kFT), args, kSmemAlloc, st);
  if (p.ev_end) cudaEventRecord(static_cast<cudaEvent_t>(p.ev_end), st);
  return e;
}

}  // namespace lfa
