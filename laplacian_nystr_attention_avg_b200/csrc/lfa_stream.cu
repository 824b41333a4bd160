// Streaming passes of the per-stage forward on tcgen05, for bf16 tokens with d = 64 and any m up to
// 256 landmarks (LaplacianFormer note, papernotes.org: §关键设计 1-3). The fused kernel covers m <= 63
// in one launch; these two kernels serve every other bf16 shape, and pass 1 also forms C^T dO for the
// backward pass.
//
// Both passes walk a CTA's run of 64-token tiles of one unit; Q (and, in pass 1, V) tiles arrive by TMA
// in a three-deep ring. The 16 warps compute a tile's cross kernel C = exp(-||q - l||_1 / lam) on CUDA
// cores in fp32: warp w owns a range of about m / 16 landmarks for all 64 rows of the tile (two rows
// per lane), so the statistics of a landmark column never leave its warp. C enters the tensor cores as
// bf16 of a shifted value C - c_l, which keeps the rounding relative to the column's spread instead of
// to C itself:
//   pass 1 (k_stream_pass1): c_l = the mean of C over the CTA's first tile. The warps keep the sums of
//          C - c and (C - c)^2 in registers; one thread issues P += (C - c)^T V per tile (M = 64
//          landmarks of one panel, N = 64 channels, K = 64 tokens; one TMEM accumulator per
//          64-landmark panel); sum V on CUDA cores. The CTA's record is rebased to no shift:
//          S1 = sum(C - c) + n c, S2 = sum((C - c)^2) + 2 c sum(C - c) + n c^2, C^T V = P + c (sum V)^T,
//          which is the generic pass-1 record.
//   pass 2 (k_stream_pass2): c_l = mu_l, the column mean from the combine. O = (C - mu) M' +
//          (b + mu^T M') + DWC(V), by the identity C M' + b = (C - mu) M' + mu^T M' + b. (C - mu) M' is
//          one tcgen05 product per tile (M = 64 tokens, N = 64 channels, K = m landmarks; M' in bf16,
//          K-major, staged once per CTA) into one of two TMEM accumulators. A tile's epilogue (bias,
//          the 3 x 3 depthwise DWC read from global V, bf16 store) runs after the next tile's distances,
//          while that tile's product runs.
// Every wait is a bounded mbarrier wait (an expired one sets the timeout bit of the status word).
#include <math.h>

#include "lfa_internal.h"
#include "lfa_sm100.cuh"
#include "lfa_tma_host.h"

namespace lfa {
namespace {

using namespace sm100;

constexpr int kST = 512;                         // threads per CTA (16 warps)
constexpr int kSTile = 64;                       // tokens per tile
constexpr int kPanel = 8192;                     // bytes of a 64-token x 64-landmark bf16 SW128 panel
constexpr int kPanels = kMaxM / 64;              // landmark panels of the largest m
constexpr int kCbBytes = kPanels * kPanel;       // one tile of C - c
constexpr int kStageBytes = 16384;               // Q tile, then V tile (pass 1)
constexpr int kOffCb = 0;                        // two C tiles
constexpr int kOffStage = kOffCb + 2 * kCbBytes; // three ring stages
constexpr int kOffMimg = kOffStage + 3 * kStageBytes;   // pass 2: M'^T, bf16, K-major panels
constexpr int kOffL = kOffMimg + kCbBytes;       // landmarks, fp32 [m][64]
constexpr int kOffSh = kOffL + kMaxM * 64 * 4;   // column shifts c, fp32 [m]
constexpr int kOffAux = kOffSh + kMaxM * 4;      // pass 1: sum-V partials; pass 2: bias, DWC taps
constexpr int kAuxFloats = 64 + 9 * 64 + 8 * 64;   // pass 2: bias, DWC taps, bias partials
constexpr int kOffBar = kOffAux + kAuxFloats * 4;
constexpr int kBarFull = 0, kBarMma = 3, kNumBars = 5;
constexpr int kOffTmem = kOffBar + 64;
constexpr int kStreamSmem = kOffTmem + 64 + 1024;   // + alignment of the dynamic base to 1024
static_assert(kStreamSmem <= 232448, "shared memory over the sm_100 per-block limit");
static_assert(kOffStage % 1024 == 0 && kOffMimg % 1024 == 0 && kStageBytes % 1024 == 0, "SW128 tiles need 1024-byte alignment");
static_assert(kNumBars * 8 <= 64, "mbarriers overlap the TMEM address slot");

struct StreamArgs {
  int P;         // CTAs per unit
  int tpc;       // tiles per CTA
  int n_tiles;   // end (exclusive) of this launch's tiles of a unit
  int t0;        // pass 1: first tile of this launch (its CTA c takes tiles t0 + c tpc ..)
  int rec0;      // pass 1: record of this launch's CTA 0 in the unit's records
  int rec_n;     // pass 1: records per unit in p.part
};

__device__ __forceinline__ float bflo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bfhi(uint32_t v) { return __uint_as_float(v & 0xffff0000u); }
__device__ __forceinline__ uint32_t pack2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// Landmark range of warp w: m / 16 landmarks, one more for the m % 16 warps whose rank 13 w mod 16 is
// below m % 16 (ranks 0, 1, 2, ... are warps 0, 5, 10, 15, 4, ..., one per scheduler in turn).
__device__ __forceinline__ void warp_range(int m, int w, int& j0, int& n) {
  const int base = m >> 4, e = m & 15;
  j0 = 0;
  for (int k = 0; k < w; ++k) j0 += base + (((13 * k) & 15) < e ? 1 : 0);
  n = base + (((13 * w) & 15) < e ? 1 : 0);
}

// address of (token row, landmark j) in a C tile: panel j / 64, SW128 row of 64 landmarks
__device__ __forceinline__ unsigned char* c_at(unsigned char* cb, int row, int j) {
  return cb + (j >> 6) * kPanel + sw128(row, (j & 63) >> 3) + ((j & 7) << 1);
}

// Tokens lane and lane + 32 of the tile against landmarks j0 .. j0 + LT - 1: L1 distance in fp32,
// C = exp2(D * scale), z = C - c (zero on rows past the unit's end) stored as bf16 into the C tile.
// Pass 1 (P1) adds z and z^2 into s1 / s2 [OFF + b]; on the CTA's first tile it forms the shift c of
// each landmark as the mean of C over the tile's valid rows (each lane holds the warp-wide sum) and
// records it in shs. Optionally copies bf16(z) + c of one unit to dbg ([N][m] fp32).
template <int LT, int OFF, bool P1>
__device__ __forceinline__ void dist_group(const unsigned char* qt, const float* Ls, float* shs, unsigned char* cb,
                                           int j0, int nvalid, bool first, float scale, float (&s1)[16],
                                           float (&s2)[16], float* dbg, int m) {
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
      const uint4 raw = *reinterpret_cast<const uint4*>(qt + sw128(lane + 32 * a, k8));
      q[a][0] = bflo(raw.x); q[a][1] = bfhi(raw.x); q[a][2] = bflo(raw.y); q[a][3] = bfhi(raw.y);
      q[a][4] = bflo(raw.z); q[a][5] = bfhi(raw.z); q[a][6] = bflo(raw.w); q[a][7] = bfhi(raw.w);
    }
#pragma unroll
    for (int h4 = 0; h4 < 2; ++h4) {
      float4 l[LT];
#pragma unroll
      for (int b = 0; b < LT; ++b) l[b] = *reinterpret_cast<const float4*>(&Ls[(j0 + b) * 64 + 8 * k8 + 4 * h4]);
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
  const bool v0 = lane < nvalid, v1 = lane + 32 < nvalid;
#pragma unroll
  for (int b = 0; b < LT; ++b) {
    const float c0 = ex2_approx(acc[0][b] * scale), c1 = ex2_approx(acc[1][b] * scale);
    float sh;
    if (P1 && first) {
      float x = (v0 ? c0 : 0.f) + (v1 ? c1 : 0.f);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
      sh = x / (float)nvalid;
      if (lane == 0) shs[j0 + b] = sh;
    } else {
      sh = shs[j0 + b];
    }
    acc[0][b] = v0 ? c0 - sh : 0.f;
    acc[1][b] = v1 ? c1 - sh : 0.f;
    if (P1) {
      s1[OFF + b] += acc[0][b] + acc[1][b];
      s2[OFF + b] = fmaf(acc[0][b], acc[0][b], fmaf(acc[1][b], acc[1][b], s2[OFF + b]));
    }
  }
  // bf16 stores, two landmarks per 4-byte word from an even landmark index on
#pragma unroll
  for (int a = 0; a < 2; ++a) {
    const int row = lane + 32 * a;
    if ((j0 & 1) == 0) {
#pragma unroll
      for (int b = 0; b + 1 < LT; b += 2)
        *reinterpret_cast<uint32_t*>(c_at(cb, row, j0 + b)) = pack2(acc[a][b], acc[a][b + 1]);
      if (LT & 1) *reinterpret_cast<__nv_bfloat16*>(c_at(cb, row, j0 + LT - 1)) = __float2bfloat16_rn(acc[a][LT - 1]);
    } else {
      *reinterpret_cast<__nv_bfloat16*>(c_at(cb, row, j0)) = __float2bfloat16_rn(acc[a][0]);
#pragma unroll
      for (int b = 1; b + 1 < LT; b += 2)
        *reinterpret_cast<uint32_t*>(c_at(cb, row, j0 + b)) = pack2(acc[a][b], acc[a][b + 1]);
      if (!(LT & 1)) *reinterpret_cast<__nv_bfloat16*>(c_at(cb, row, j0 + LT - 1)) = __float2bfloat16_rn(acc[a][LT - 1]);
    }
    if (dbg != nullptr && row < nvalid) {
#pragma unroll
      for (int b = 0; b < LT; ++b)
        dbg[(size_t)row * m + j0 + b] = __bfloat162float(__float2bfloat16_rn(acc[a][b])) + shs[j0 + b];
    }
  }
}

// The warp's landmark range as one group (n <= 8) or two (n <= 16), kept in registers s1 / s2 [0, 8)
// and [8, 16).
template <bool P1>
__device__ __forceinline__ void dist_warp(const unsigned char* qt, const float* Ls, float* shs, unsigned char* cb,
                                          int j0, int g0, int g1, int nvalid, bool first, float scale,
                                          float (&s1)[16], float (&s2)[16], float* dbg, int m) {
#define LFA_G(LT, OFF, J)                                                                          \
  dist_group<LT, OFF, P1>(qt, Ls, shs, cb, J, nvalid, first, scale, s1, s2, dbg, m)
  switch (g0) {
    case 1: LFA_G(1, 0, j0); break;
    case 2: LFA_G(2, 0, j0); break;
    case 3: LFA_G(3, 0, j0); break;
    case 4: LFA_G(4, 0, j0); break;
    case 5: LFA_G(5, 0, j0); break;
    case 6: LFA_G(6, 0, j0); break;
    case 7: LFA_G(7, 0, j0); break;
    case 8: LFA_G(8, 0, j0); break;
    default: break;
  }
  switch (g1) {
    case 1: LFA_G(1, 8, j0 + g0); break;
    case 2: LFA_G(2, 8, j0 + g0); break;
    case 3: LFA_G(3, 8, j0 + g0); break;
    case 4: LFA_G(4, 8, j0 + g0); break;
    case 5: LFA_G(5, 8, j0 + g0); break;
    case 6: LFA_G(6, 8, j0 + g0); break;
    case 7: LFA_G(7, 8, j0 + g0); break;
    case 8: LFA_G(8, 8, j0 + g0); break;
    default: break;
  }
#undef LFA_G
}

// Pass-1 column sums of one group, reduced over the warp and rebased to no shift.
template <int LT, int OFF>
__device__ __forceinline__ void group_sums(const float (&s1)[16], const float (&s2)[16], const float* shs, float* out,
                                           int m, int j0, int n_rows) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int b = 0; b < LT; ++b) {
    float a1 = s1[OFF + b], a2 = s2[OFF + b];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      a1 += __shfl_xor_sync(0xffffffffu, a1, o);
      a2 += __shfl_xor_sync(0xffffffffu, a2, o);
    }
    if (lane == 0) {
      const double c = shs[j0 + b], n = n_rows;
      out[j0 + b] = (float)((double)a1 + n * c);
      out[m + j0 + b] = (float)((double)a2 + 2.0 * c * (double)a1 + n * c * c);
    }
  }
}

__device__ __forceinline__ void warp_sums(const float (&s1)[16], const float (&s2)[16], const float* shs, float* out,
                                          int m, int j0, int g0, int g1, int n_rows) {
#define LFA_S(LT, OFF, J) group_sums<LT, OFF>(s1, s2, shs, out, m, J, n_rows)
  switch (g0) {
    case 1: LFA_S(1, 0, j0); break;
    case 2: LFA_S(2, 0, j0); break;
    case 3: LFA_S(3, 0, j0); break;
    case 4: LFA_S(4, 0, j0); break;
    case 5: LFA_S(5, 0, j0); break;
    case 6: LFA_S(6, 0, j0); break;
    case 7: LFA_S(7, 0, j0); break;
    case 8: LFA_S(8, 0, j0); break;
    default: break;
  }
  switch (g1) {
    case 1: LFA_S(1, 8, j0 + g0); break;
    case 2: LFA_S(2, 8, j0 + g0); break;
    case 3: LFA_S(3, 8, j0 + g0); break;
    case 4: LFA_S(4, 8, j0 + g0); break;
    case 5: LFA_S(5, 8, j0 + g0); break;
    case 6: LFA_S(6, 8, j0 + g0); break;
    case 7: LFA_S(7, 8, j0 + g0); break;
    case 8: LFA_S(8, 8, j0 + g0); break;
    default: break;
  }
#undef LFA_S
}

__device__ __forceinline__ void warp_groups(int m, int w, int& j0, int& g0, int& g1) {
  int n;
  warp_range(m, w, j0, n);
  g0 = n <= 8 ? n : (n + 1) / 2;
  g1 = n - g0;
}

// Common start of both passes: TMEM, barriers, both C tiles zeroed (the landmark padding of the last
// panel stays zero), the landmarks of unit u in shared memory.
__device__ __forceinline__ uint32_t stream_setup(const Params& p, unsigned char* sm, uint32_t ncols, int u) {
  const int t = threadIdx.x, w = t >> 5;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + kOffBar);
  uint32_t* tslot = reinterpret_cast<uint32_t*>(sm + kOffTmem);
  if (w == 0) {
    tmem_alloc(tslot, ncols);
    tmem_relinquish();
  }
  if (t == 0) {
    for (int b = 0; b < kNumBars; ++b) mbar_init(bars + b, 1);
    mbar_init_fence();
  }
  for (int e = t; e < 2 * kCbBytes / 16; e += kST) reinterpret_cast<uint4*>(sm + kOffCb)[e] = make_uint4(0u, 0u, 0u, 0u);
  const float4* Lg = reinterpret_cast<const float4*>(p.L + (size_t)u * p.m * 64);
  float4* Ld = reinterpret_cast<float4*>(sm + kOffL);
  int e = t;
  for (; e + 3 * kST < p.m * 16; e += 4 * kST) {   // four loads in flight per thread
    float4 r[4];
#pragma unroll
    for (int x = 0; x < 4; ++x) r[x] = __ldg(Lg + e + x * kST);
#pragma unroll
    for (int x = 0; x < 4; ++x) Ld[e + x * kST] = r[x];
  }
  for (; e < p.m * 16; e += kST) Ld[e] = __ldg(Lg + e);
  fence_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  return *tslot;
}

__device__ __forceinline__ void stream_teardown(unsigned char* sm, uint32_t tmem, uint32_t ncols) {
  tc_fence_before();
  __syncthreads();
  if ((threadIdx.x >> 5) == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, ncols);
  }
}

__global__ void __launch_bounds__(kST, 1) k_stream_pass1(const Params p, const StreamArgs sa,
                                                         const __grid_constant__ CUtensorMap tmQ,
                                                         const __grid_constant__ CUtensorMap tmV) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
  unsigned char* sm = smem_raw + pad;
  const uint32_t sbase = smem_u32(sm);
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + kOffBar);
  const float* Ls = reinterpret_cast<const float*>(sm + kOffL);
  float* shs = reinterpret_cast<float*>(sm + kOffSh);
  float* aux = reinterpret_cast<float*>(sm + kOffAux);
  const int t = threadIdx.x, w = t >> 5, lane = t & 31;
  const int u = blockIdx.y, pc = blockIdx.x, m = p.m;
  const int tile0 = sa.t0 + pc * sa.tpc;
  const int tile1 = min(tile0 + sa.tpc, sa.n_tiles);
  const int ntl = tile1 - tile0;
  float* out = p.part + ((size_t)u * sa.rec_n + sa.rec0 + pc) * p.part_stride;
  if (ntl <= 0) {   // (the host's plan gives every CTA a tile)
    for (int e = t; e < p.part_stride; e += kST) out[e] = 0.f;
    return;
  }
  const int npan = (m + 63) >> 6;
  const uint32_t ncols = npan == 1 ? 64u : (npan == 2 ? 128u : 256u);
  if (t == 32) {
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmV);
  }
  const uint32_t tmem = stream_setup(p, sm, ncols, u);
  auto issue = [&](int i) {
    const int s = i % 3;
    uint64_t* fb = bars + kBarFull + s;
    mbar_expect_tx(fb, kStageBytes);
    tma_load_3d(sm + kOffStage + s * kStageBytes, &tmQ, 0, (tile0 + i) * kSTile, u, fb);
    tma_load_3d(sm + kOffStage + s * kStageBytes + 8192, &tmV, 0, (tile0 + i) * kSTile, u, fb);
  };
  if (t == 0) {
    issue(0);
    if (ntl > 1) issue(1);
  }
  int wj0, g0, g1;
  warp_groups(m, w, wj0, g0, g1);
  float s1[16], s2[16];
#pragma unroll
  for (int b = 0; b < 16; ++b) {
    s1[b] = 0.f;
    s2[b] = 0.f;
  }
  float sv = 0.f;
  const int svc = t & 63, svr = (t >> 6) * 8;
  const float scale = p.neg_log2e_over_lam;
  for (int i = 0; i < ntl; ++i) {
    const int s = i % 3;
    const int row0 = (tile0 + i) * kSTile;
    const int nvalid = min(kSTile, p.N - row0);
    const unsigned char* stg = sm + kOffStage + s * kStageBytes;
    mbar_wait(bars + kBarFull + s, (i / 3) & 1, p.status, kStatusTimeout);
    unsigned char* cb = sm + kOffCb + (i & 1) * kCbBytes;
    dist_warp<true>(stg, Ls, shs, cb, wj0, g0, g1, nvalid, i == 0, scale, s1, s2, nullptr, m);
    // sum V: channel svc over rows svr .. svr + 7 (rows past the unit's end were filled with zeros)
#pragma unroll
    for (int r = 0; r < 8; ++r)
      sv += __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(stg + 8192 + sw128(svr + r, svc >> 3) + ((svc & 7) << 1)));
    // the previous tile's product is done: its C tile and ring stage are free after the barrier
    if (t == 0 && i >= 1) mbar_wait(bars + kBarMma + ((i - 1) & 1), ((i - 1) >> 1) & 1, p.status, kStatusTimeout);
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    if (t == 0) {
      if (i + 2 < ntl) issue(i + 2);
      tc_fence_after();
      const uint32_t id = idesc(1, 64, 64, 1, 1);
      const uint64_t vd = desc_sw128(sbase + kOffStage + s * kStageBytes + 8192, 8192, 1024);
      for (int pn = 0; pn < npan; ++pn) {
        const uint64_t cd = desc_sw128(sbase + kOffCb + (i & 1) * kCbBytes + pn * kPanel, 8192, 1024);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_bf16(tmem + 64 * pn, cd + (uint64_t)(kk * 2048 >> 4), vd + (uint64_t)(kk * 2048 >> 4), id,
                   (i > 0 || kk > 0) ? 1u : 0u);
      }
      mma_commit(bars + kBarMma + (i & 1));
    }
  }
  if (t == 0) mbar_wait(bars + kBarMma + ((ntl - 1) & 1), ((ntl - 1) >> 1) & 1, p.status, kStatusTimeout);
  aux[(t >> 6) * 64 + svc] = sv;
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const int n_rows = min(p.N, tile1 * kSTile) - tile0 * kSTile;
  if (t < 64) {
    float a = 0.f;
#pragma unroll
    for (int r = 0; r < 8; ++r) a += aux[r * 64 + t];
    out[2 * m + m * 64 + t] = a;
    aux[512 + t] = a;
  }
  warp_sums(s1, s2, shs, out, m, wj0, g0, g1, n_rows);
  __syncthreads();
  // C^T V = P + c (sum V)^T: panel pn holds landmark 64 pn + 16 q + lane (lane < 16) in TMEM lane
  // 32 q + lane; warp w reads channels 16 h .. 16 h + 15
  {
    const int q = w & 3, h = w >> 2;
    for (int pn = 0; pn < npan; ++pn) {
      float v[16];
      tmem_ld16(tmem + 64 * pn + 16 * h + ((uint32_t)(32 * q) << 16), v);
      const int j = 64 * pn + 16 * q + lane;
      if (lane < 16 && j < m) {
        const float c = shs[j];
        float* dst = out + 2 * m + (size_t)j * 64 + 16 * h;
#pragma unroll
        for (int x = 0; x < 16; ++x) dst[x] = fmaf(c, aux[512 + 16 * h + x], v[x]);
      }
    }
  }
  stream_teardown(sm, tmem, ncols);
}

__global__ void __launch_bounds__(kST, 1) k_stream_pass2(const Params p, const StreamArgs sa,
                                                         const __grid_constant__ CUtensorMap tmQ) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
  unsigned char* sm = smem_raw + pad;
  const uint32_t sbase = smem_u32(sm);
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + kOffBar);
  const float* Ls = reinterpret_cast<const float*>(sm + kOffL);
  float* shs = reinterpret_cast<float*>(sm + kOffSh);
  float* bias = reinterpret_cast<float*>(sm + kOffAux);        // [64]
  float* taps = bias + 64;                                     // [9][64]
  const int t = threadIdx.x, w = t >> 5, lane = t & 31;
  const int u = blockIdx.y, pc = blockIdx.x, m = p.m;
  const int tile0 = pc * sa.tpc;
  const int tile1 = min(tile0 + sa.tpc, sa.n_tiles);
  const int ntl = tile1 - tile0;
  if (ntl <= 0) return;
  const int npan = (m + 63) >> 6, nks = (m + 15) >> 4;
  if (t == 32) tma_prefetch_desc(&tmQ);
  // shift mu = the column mean of C (fp64 sums of the combine), M'^T as bf16 K-major panels (zero past
  // m), the DWC taps of this unit's head
  const double* red = p.red + (size_t)u * p.part_stride;
  for (int j = t; j < m; j += kST) shs[j] = (float)(red[j] / (double)p.Ng);
  __syncthreads();
  // thread t takes channel k = t % 64 and landmark pairs (t / 64) + 8 i: it also sums mu_j M'[j][k] over
  // its landmarks for the bias (the eight partial sums of a channel meet in aux below)
  const float* Mp = p.Mp + (size_t)u * m * 64;
  float bmu = 0.f;
#pragma unroll 4
  for (int e = t; e < npan * 32 * 64; e += kST) {
    const int k = e & 63, j = 2 * (e >> 6);
    const float lo = j < m ? __ldg(Mp + (size_t)j * 64 + k) : 0.f;
    const float hi = j + 1 < m ? __ldg(Mp + (size_t)(j + 1) * 64 + k) : 0.f;
    if (j < m) bmu = fmaf(shs[j], lo, bmu);
    if (j + 1 < m) bmu = fmaf(shs[j + 1], hi, bmu);
    *reinterpret_cast<uint32_t*>(sm + kOffMimg + (j >> 6) * kPanel + sw128(k, (j & 63) >> 3) + ((j & 7) << 1)) =
        pack2(lo, hi);
  }
  float* bpartial = taps + 9 * 64;   // [8][64]
  bpartial[(t >> 6) * 64 + (t & 63)] = bmu;
  const int hd = u % p.heads;
  for (int e = t; e < 9 * 64; e += kST) {
    const int tap = e >> 6, k = e & 63;
    taps[e] = p.dwc[((size_t)hd * 64 + k) * 9 + tap];
  }
  const uint32_t tmem = stream_setup(p, sm, 128, u);   // (its barrier also publishes M'^T, taps, partials)
  if (t < 64) {
    float b = 0.f;
    for (int c = 0; c < p.n_chunks; ++c) b += __ldg(p.bpart + ((size_t)u * p.n_chunks + c) * 64 + t);
#pragma unroll
    for (int r = 0; r < 8; ++r) b += bpartial[r * 64 + t];
    bias[t] = b;
  }
  auto issue = [&](int i) {
    const int s = i % 3;
    uint64_t* fb = bars + kBarFull + s;
    mbar_expect_tx(fb, 8192);
    tma_load_3d(sm + kOffStage + s * kStageBytes, &tmQ, 0, (tile0 + i) * kSTile, u, fb);
  };
  if (t == 0) {
    issue(0);
    if (ntl > 1) issue(1);
  }
  __syncthreads();   // bias
  int wj0, g0, g1;
  warp_groups(m, w, wj0, g0, g1);
  float s1[16], s2[16];   // (unused in pass 2)
  const float scale = p.neg_log2e_over_lam;
  const __nv_bfloat16* Vg = static_cast<const __nv_bfloat16*>(p.V) + (size_t)u * p.N * 64;
  __nv_bfloat16* Og = static_cast<__nv_bfloat16*>(p.O) + (size_t)u * p.N * 64;
  const int q = w & 3, h = w >> 2;
  // epilogue of tile j: TMEM lane 32 q + lane (lane < 16) holds token 16 q + lane; warp w takes
  // channels 16 h .. 16 h + 15
  auto epilogue = [&](int j) {
    mbar_wait(bars + kBarMma + (j & 1), (j >> 1) & 1, p.status, kStatusTimeout);
    tc_fence_after();
    float v[16];
    tmem_ld16(tmem + 64 * (j & 1) + 16 * h + ((uint32_t)(32 * q) << 16), v);
    const int n = (tile0 + j) * kSTile + 16 * q + lane;
    if (lane < 16 && n < p.N) {
      float o[16];
#pragma unroll
      for (int x = 0; x < 16; ++x) o[x] = v[x] + bias[16 * h + x];
      const int gy = n / p.W, gx = n % p.W;
#pragma unroll
      for (int a = 0; a < 3; ++a) {
        // local row yy, global row y0 + yy; rows just outside a band come from the halo
        const int yy = gy + a - 1, yg = p.y0 + yy;
        if (yg < 0 || yg >= p.Hg) continue;
        const __nv_bfloat16* vrow = (yy >= 0 && yy < p.H)
                                        ? Vg + (size_t)yy * p.W * 64
                                        : static_cast<const __nv_bfloat16*>(p.Vh) + ((size_t)u * 2 + (yy < 0 ? 0 : 1)) * p.W * 64;
#pragma unroll
        for (int b = 0; b < 3; ++b) {
          const int xx = gx + b - 1;
          if (xx < 0 || xx >= p.W) continue;
          const uint4* src = reinterpret_cast<const uint4*>(vrow + (size_t)xx * 64 + 16 * h);
          const uint4 r0 = __ldg(src), r1 = __ldg(src + 1);
          const uint32_t rv[8] = {r0.x, r0.y, r0.z, r0.w, r1.x, r1.y, r1.z, r1.w};
          const float* tp = taps + (a * 3 + b) * 64 + 16 * h;
#pragma unroll
          for (int x = 0; x < 8; ++x) {
            o[2 * x] = fmaf(tp[2 * x], bflo(rv[x]), o[2 * x]);
            o[2 * x + 1] = fmaf(tp[2 * x + 1], bfhi(rv[x]), o[2 * x + 1]);
          }
        }
      }
      uint4* dst = reinterpret_cast<uint4*>(Og + (size_t)n * 64 + 16 * h);
      dst[0] = make_uint4(pack2(o[0], o[1]), pack2(o[2], o[3]), pack2(o[4], o[5]), pack2(o[6], o[7]));
      dst[1] = make_uint4(pack2(o[8], o[9]), pack2(o[10], o[11]), pack2(o[12], o[13]), pack2(o[14], o[15]));
    }
  };
  const bool cap = p.dbgC != nullptr && u == p.dbg_unit;
  for (int i = 0; i < ntl; ++i) {
    const int s = i % 3;
    const int row0 = (tile0 + i) * kSTile;
    const int nvalid = min(kSTile, p.N - row0);
    mbar_wait(bars + kBarFull + s, (i / 3) & 1, p.status, kStatusTimeout);
    unsigned char* cb = sm + kOffCb + (i & 1) * kCbBytes;
    dist_warp<false>(sm + kOffStage + s * kStageBytes, Ls, shs, cb, wj0, g0, g1, nvalid, false, scale, s1, s2,
                     cap ? p.dbgC + (size_t)row0 * m : nullptr, m);
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    if (t == 0) {
      if (i + 2 < ntl) issue(i + 2);
      tc_fence_after();
      const uint32_t id = idesc(1, 64, 64, 0, 0);
      for (int ks = 0; ks < nks; ++ks) {
        const int pn = ks >> 2, kk = ks & 3;
        const uint64_t ad = desc_sw128(sbase + kOffCb + (i & 1) * kCbBytes + pn * kPanel, 16, 1024) + (uint64_t)(kk * 2);
        const uint64_t bd = desc_sw128(sbase + kOffMimg + pn * kPanel, 16, 1024) + (uint64_t)(kk * 2);
        mma_bf16(tmem + 64 * (i & 1), ad, bd, id, ks > 0 ? 1u : 0u);
      }
      mma_commit(bars + kBarMma + (i & 1));
    }
    if (i >= 1) epilogue(i - 1);
  }
  epilogue(ntl - 1);
  if (cap && p.dbgS != nullptr) {
    for (int e = t; e < (tile1 - tile0) * kSTile * m; e += kST) {
      const int row = tile0 * kSTile + e / m;
      if (row < p.N) p.dbgS[(size_t)row * m + e % m] = shs[e % m];
    }
  }
  stream_teardown(sm, tmem, 128);
}

// One CTA per SM at most (the kernels hold about 213 KB of shared memory): P CTAs per unit with P U
// within the SM count where the tiles allow, and never more than the generic plan's P (whose partial
// records the workspace holds).
StreamArgs stream_plan(const Params& p) {
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  StreamArgs sa;
  sa.n_tiles = ceil_div(p.N, kSTile);
  int P = sms / p.U;
  if (P < 1) P = 1;
  if (P > p.P) P = p.P;
  if (P > sa.n_tiles) P = sa.n_tiles;
  sa.tpc = ceil_div(sa.n_tiles, P);
  sa.P = ceil_div(sa.n_tiles, sa.tpc);
  sa.t0 = 0;
  sa.rec0 = 0;
  sa.rec_n = sa.P;
  return sa;
}

// pass 1 over the tiles [t_begin, t_end) of every unit with at most P CTAs per unit
StreamArgs stream_range_plan(int t_begin, int t_end, int P) {
  StreamArgs sa;
  const int nt = t_end - t_begin;
  if (P > nt) P = nt;
  if (P < 1) P = 1;
  sa.tpc = ceil_div(nt, P);
  sa.P = ceil_div(nt, sa.tpc);
  sa.n_tiles = t_end;
  sa.t0 = t_begin;
  sa.rec0 = 0;
  sa.rec_n = sa.P;
  return sa;
}

}  // namespace

bool stream_eligible(const Params& p) { return p.dtype == LFA_BF16 && p.d == 64 && p.m >= 1 && p.m <= kMaxM; }

cudaError_t stream_set_attributes() {
  cudaError_t e = cudaFuncSetAttribute(k_stream_pass1, cudaFuncAttributeMaxDynamicSharedMemorySize, kStreamSmem);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(k_stream_pass2, cudaFuncAttributeMaxDynamicSharedMemorySize, kStreamSmem);
  return e;
}

int stream_pass1(const Params& p, cudaStream_t st) {
  if (!stream_eligible(p)) return 0;
  const StreamArgs sa = stream_plan(p);
  CUtensorMap tq, tv;
  if (!make_tmap_rows_bf16(&tq, p.Q, (uint64_t)p.N, (uint64_t)p.U, kSTile) ||
      !make_tmap_rows_bf16(&tv, p.V, (uint64_t)p.N, (uint64_t)p.U, kSTile))
    return 0;
  k_stream_pass1<<<dim3(sa.P, p.U), kST, kStreamSmem, st>>>(p, sa, tq, tv);
  return sa.P;
}

int stream_tiles(const Params& p) { return ceil_div(p.N, kSTile); }

bool stream_maps_ok(const Params& p) {
  CUtensorMap tq, tv;
  return stream_eligible(p) && make_tmap_rows_bf16(&tq, p.Q, (uint64_t)p.N, (uint64_t)p.U, kSTile) &&
         make_tmap_rows_bf16(&tv, p.V, (uint64_t)p.N, (uint64_t)p.U, kSTile);
}

int stream_range_blocks(int t_begin, int t_end, int P) {
  return t_end > t_begin ? stream_range_plan(t_begin, t_end, P).P : 0;
}

bool stream_pass1_range(const Params& p, int t_begin, int t_end, int P, int rec0, int rec_n, cudaStream_t st) {
  if (!stream_eligible(p) || t_begin < 0 || t_end > stream_tiles(p) || t_end <= t_begin) return false;
  StreamArgs sa = stream_range_plan(t_begin, t_end, P);
  if (rec0 < 0 || rec0 + sa.P > rec_n || rec_n > p.P) return false;
  sa.rec0 = rec0;
  sa.rec_n = rec_n;
  CUtensorMap tq, tv;
  if (!make_tmap_rows_bf16(&tq, p.Q, (uint64_t)p.N, (uint64_t)p.U, kSTile) ||
      !make_tmap_rows_bf16(&tv, p.V, (uint64_t)p.N, (uint64_t)p.U, kSTile))
    return false;
  k_stream_pass1<<<dim3(sa.P, p.U), kST, kStreamSmem, st>>>(p, sa, tq, tv);
  return true;
}

bool stream_pass2(const Params& p, cudaStream_t st) {
  if (!stream_eligible(p)) return false;
  const StreamArgs sa = stream_plan(p);
  CUtensorMap tq;
  if (!make_tmap_rows_bf16(&tq, p.Q, (uint64_t)p.N, (uint64_t)p.U, kSTile)) return false;
  k_stream_pass2<<<dim3(sa.P, p.U), kST, kStreamSmem, st>>>(p, sa, tq);
  return true;
}

}  // namespace lfa
