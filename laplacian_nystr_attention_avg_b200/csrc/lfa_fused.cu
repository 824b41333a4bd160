// Fused single-launch forward pass for bf16 inputs, d = 64 and m <= 63 landmarks.
//
// One cooperative persistent kernel, one CTA per SM. Token rows of all U = B*heads units are cut into
// 128-row chunks dealt out to the row CTAs (at most two units, "segments", per CTA); CTAs 0..U-1 are
// the units' solver CTAs and own no rows. CTAs meet only through per-unit flags in global memory
// (epoch-stamped counters, bounded waits); there is no grid-wide barrier.
//   phase 0  all CTAs: landmark pooling L = r x r average pool of Q (LaplacianFormer note,
//            §关键设计 2); each landmark raises its unit's landmark counter.
//   phase 1  solver CTA of unit u: W = exp(-E/lam) + eps I, ||W||_2 by power iteration, alpha
//            (§关键设计 3 with the fallback), and the T Newton-Schulz steps on tcgen05 in 3xTF32
//            (fp32-accurate): X_{k+1} = X_k + X_k R_k, R_{k+1} = R_k R_k^T (R_k = I - W X_k; the
//            same iterates in exact arithmetic, one stacked [X; R] product per step), then the
//            printed product form X (2I - W X) for the last step, which re-anchors R to I - W X;
//            the diagnostic ||I - W X_T||_F; then its share of the unit's DWC.
//   phase 2  row CTAs, pass 1 per chunk (Q rows by TMA): C = exp(-||q - l||_1 / lam) on CUDA cores
//            in fp32 (the dominant cost), kept in shared memory as bf16(C - c), c a per-column shift
//            of the segment, for the whole kernel (never in HBM); per-landmark sums of C - c and
//            (C - c)^2 in registers; P += (C - c)^T V on tcgen05 (V chunk staged by TMA; a constant-1
//            landmark column 63 yields sum_i v_i in the same product). One record per segment.
//   phase 3  solver CTA of unit u, once the unit's records are out: sums them rebased to no shift,
//            mu, var, s = 1/sqrt(var + eps), A = C~^T V by rank-1 folding (§关键设计 1), M = X A,
//            M' = diag(s) M, b0 = (1/N - s o mu)^T M; publishes M'^T (bf16, the shared-memory image
//            pass 2 consumes) and each contributor's bias b0 + c_k^T M' with a release flag.
//   phase 3b row CTAs, meanwhile: DWC(V) (§关键设计 1 "ZV + DWC(V)", 3 x 3 depthwise, zero padding)
//            of their other chunks from TMA-staged V tiles with a one-grid-row halo, bf16 into O.
//   phase 4  row CTAs: O += (C - c) M' + bias by tcgen05 products (one TMEM accumulator per chunk) and
//            TMA bf16 reduce-adds of the epilogue rows onto the DWC values in O.
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
// floats per partial record: S1'[64], S2'[64], P'[64][64] (sums of the shifted C - c), c[64], the
// segment's row count n (padded to 64 floats), and the pass-2 bias b[64] for this record's shift,
// which the unit's solver CTA fills in
constexpr int kRec = 128 + 64 * 64 + 128 + 64;
constexpr int kRecC = 128 + 64 * 64;      // offset of c
constexpr int kRecN = kRecC + 64;         // offset of n
constexpr int kRecF = kRecN + 2;          // offset of the record's 64-bit published flag (holds the epoch)
constexpr int kRecB = kRecN + 64;         // offset of b
constexpr int kMaxGrid = 256;             // records are sized for up to this many CTAs
constexpr int kMaxContrib = 32;           // CTAs contributing to one unit
constexpr int kPowerIters = 8;

// shared-memory map (bytes from a 1024-aligned base)
constexpr uint32_t kOffC = 0;                                   // 8 x 16 KB C chunks (SW128 rows)
constexpr uint32_t kOffV = kOffC + kMaxChunks * 16384;          // 3 x 16 KB V stages (TMA, SW128)
constexpr uint32_t kOffQ = kOffV + 2 * 16384;                   // third V stage + 18 KB spare in pass 1
constexpr uint32_t kOffL = kOffQ + kChunk * kQS * 4;            // landmarks, fp32 [64][68]
constexpr uint32_t kOffL2 = kOffQ + 16384;                      // pass 1: segment 1's landmarks [64][68]
constexpr uint32_t kOffMp = kOffL + 64 * kQS * 4;               // M'^T bf16 [64 ch][64 lm] (SW128)
constexpr uint32_t kOffBv = kOffMp + 8192;                      // b, fp32 [segment][64]
constexpr uint32_t kOffBar = kOffBv + 512;                      // mbarriers + TMEM address
// the solver's DWC chunk list lives in the b area: a count and at most 127 chunks, enough for the
// first 3 chunks of each of kMaxContrib row CTAs (the host caps dwc_take at 3)
constexpr int kDwcListCap = 127;
constexpr int kMaxDwcTake = 3;
static_assert(kMaxDwcTake * kMaxContrib <= kDwcListCap && (1 + kDwcListCap) * 4 <= 512, "DWC list overflows");
constexpr uint32_t kOffCt = kOffBar + 256;                      // int [32] record offsets
constexpr uint32_t kOffSr = kOffCt + 128;                       // pass-1 column sums [segment][row half][128]
constexpr uint32_t kOffRows = kOffSr + 2 * 256 * 4;            // this CTA's row plan (struct Rows)
constexpr uint32_t kOffSh = kOffRows + 64;                      // per-segment column shift of C, fp32 [2][64]
constexpr uint32_t kSmemBytes = kOffSh + 2 * 64 * 4;
constexpr uint32_t kSmemAlloc = kSmemBytes + 1024;              // slack for 1024-byte alignment
// After pass 1 the region of the V stages, Q and L (kOffV .. kOffMp) is free. It holds the combine
// scratch: A [64][68] and X^T [64][68] fp32, the column statistics, the contributor table and the
// partial sums of b; then the second segment's M'^T image (the first segment's is at kOffMp).
constexpr uint32_t kOffAs = kOffV;                              // fp32 [64][68]  A (row l, col k)
constexpr uint32_t kOffXt = kOffAs + 64 * kQS * 4;              // fp32 [64][68]  X^T (row j, col l)
constexpr uint32_t kOffS1 = kOffXt + 64 * kQS * 4;              // double [64]
constexpr uint32_t kOffS2 = kOffS1 + 512;                       // double [64]
constexpr uint32_t kOffMu = kOffS2 + 512;                       // float [64]
constexpr uint32_t kOffSc = kOffMu + 256;                       // float [64]
constexpr uint32_t kOffSv = kOffSc + 256;                       // float [64]
constexpr uint32_t kOffMt = kOffSv + 256;                       // float [64] unshifted column mean
constexpr uint32_t kOffBp = kOffMt + 256;                       // float [kWarps][8] partial b
constexpr uint32_t kOffWc = kOffBp + kWarps * 8 * 4;            // int [kWarps] contributor counts
constexpr uint32_t kOffImg1 = (kOffWc + kWarps * 4 + 1023) / 1024 * 1024;   // M'^T of segment 1
// row CTAs' DWC tiles after pass 1: C slot kMaxChunks - 1 and the V / Q / L region, contiguous
constexpr uint32_t kOffDwcTiles = kOffC + (kMaxChunks - 1) * 16384;
// solver combine only (no pass 2 there): M' fp32 [64][68], after the image
constexpr uint32_t kOffMpf = kOffImg1 + 8192;
// solver combine: the contributors' column shifts and the size of the current batch of records, in the
// DWC tile area (free once the solver's DWC is done)
constexpr uint32_t kOffCks = 0;                                 // float [kMaxContrib][64]
constexpr uint32_t kOffBatch = kOffCks + kMaxContrib * 64 * 4;  // int
constexpr int kRecBatch = 6;                                    // records per bulk-copy batch
constexpr uint32_t kRecBytes = kRec * 4;
constexpr uint32_t kOffRecBuf = 16384;                          // kRecBatch records, copied whole
// solver scratch (aliases the C region: the solver runs before this CTA's pass 1)
constexpr uint32_t kOffNsHi = 0;                                // tf32 hi [2 K-halves][128 rows][128 B]
constexpr uint32_t kOffNsLo = 32768;                            // tf32 lo
constexpr uint32_t kOffNsW = 65536;                             // fp32 [64][68]
constexpr uint32_t kOffNsX = kOffNsW + 64 * kQS * 4;            // fp32 [64][68]
constexpr uint32_t kOffNsL = kOffNsX + 64 * kQS * 4;            // fp32 [64][68]
constexpr uint32_t kOffNsVec = kOffNsL + 64 * kQS * 4;          // float [2][64] + reduction [16]

static_assert(kSmemAlloc <= 232448, "shared memory over the sm_100 per-block limit");
static_assert(kOffImg1 + 8192 <= kOffMp, "post-pass-1 scratch overlaps M'");
static_assert(kOffDwcTiles + 6 * 16384 <= kOffMp, "DWC tiles overlap M'");
static_assert(kOffL2 + 64 * kQS * 4 <= kOffL, "segment 1's landmarks overlap the L area");
static_assert(kOffV == kOffDwcTiles + 16384, "the DWC tile region is not contiguous");
static_assert(kOffMpf + 64 * kQS * 4 <= kOffBar, "solver combine scratch overlaps the barriers");
static_assert(kOffRecBuf + kRecBatch * kRecBytes <= kOffAs && kRecBytes % 16 == 0 && kOffBatch + 4 <= kOffRecBuf,
              "combine record buffers overlap the combine scratch");
static_assert(kOffNsVec + 1024 <= kOffV, "solver scratch overlaps V stages");

// mbarrier slots
constexpr int kBarV = 0;      // [3] V stage filled by TMA
constexpr int kBarP1 = 3;     // [2] pass-1 product done
constexpr int kBarP2 = 5;     // [kMaxChunks] pass-2 product of chunk gc done (one use per launch)
constexpr int kBarNs = 13;    // solver product done
constexpr int kBarDiag = 14;  // the solver's diagnostics product done
constexpr int kBarQ = 16;     // all of the CTA's pass-1 Q chunks landed (TMA)
constexpr int kBarDrain = 17; // every tcgen05 operation of the issuing threads done (count kDrainCount)
constexpr int kBarH = 18;     // [4] DWC halo tile landed (TMA)
constexpr int kBarRec = kBarV;  // solver CTAs (which have no V stages): a batch of records copied in
constexpr int kNumBars = kBarH + 4;
// pass 2: lane 0 of warp kP2Warp0 + gc issues chunk gc's products (each chunk has its own accumulator,
// so the issuers need no order among themselves); with thread 0 they make up the drain count
constexpr int kP2Warp0 = 8;
constexpr int kDrainCount = 1 + (kMaxChunks - 1);
static_assert(kP2Warp0 + kMaxChunks - 1 <= kWarps, "pass-2 issuers beyond the last warp");
constexpr uint32_t kTmemSlot = 248;  // byte offset of the TMEM address within the barrier area
constexpr uint32_t kTmemCols = 512;  // whole TMEM: pass 2 gives every chunk its own accumulator
static_assert(kNumBars * 8 <= (int)kTmemSlot && kTmemSlot + 4 <= 256, "mbarriers overlap the TMEM address slot");

struct FusedArgs {
  unsigned long long epoch;   // launch count of this handle (>= 1); flags compare against it
  unsigned long long* lready; // [U] landmarks of the unit pooled (counts landmarks, m per launch)
  unsigned long long* xready; // [U] X published (holds the epoch)
  unsigned long long* mready; // [U] M' image, the contributors' biases and the solver's DWC chunks
                              // published (holds the epoch)
  int dwc_take;               // DWC of the first dwc_take chunks of every row CTA's part of a unit: by
                              // the unit's solver CTA
  unsigned char* mimg;        // [U][8192] M'^T bf16, the SW128 image of the pass-2 B operand
  float* rec;                 // [G][2][kRec]
  // pass-1 warp plan: warp w computes landmarks [wj0[w], wj0[w] + wlt[w]) of row half w / 8;
  // warp padw[h] writes the padding columns of row half h
  unsigned char wj0[kWarps], wlt[kWarps], padw[2];
};

// Phase timeline stamps (compiled in only with -DLFA_PHASE_TRACE; lfa_debug_trace arms them).
#ifdef LFA_PHASE_TRACE
__device__ __forceinline__ void trace_mark(const Params& p, int slot) {
  if (p.trace != nullptr && threadIdx.x == 0) p.trace[(size_t)blockIdx.x * 32 + slot] = globaltimer();
}
__device__ __forceinline__ void trace_clock(const Params& p, int slot) {
  if (p.trace != nullptr && threadIdx.x == 0) p.trace[(size_t)blockIdx.x * 32 + slot] = (unsigned long long)clock64();
}
__device__ __forceinline__ void trace_mark_by(const Params& p, int slot, int thread) {
  if (p.trace != nullptr && (int)threadIdx.x == thread) p.trace[(size_t)blockIdx.x * 32 + slot] = globaltimer();
}
#else
__device__ __forceinline__ void trace_mark(const Params&, int) {}
__device__ __forceinline__ void trace_clock(const Params&, int) {}
__device__ __forceinline__ void trace_mark_by(const Params&, int, int) {}
#endif

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
// first global chunk of CTA g (the row CTAs' ranges; G for the end of the last one)
__device__ __forceinline__ int cta_chunk0(int g, const Params& p) {
  const int nchu = (p.N + kChunk - 1) / kChunk, T = p.U * nchu, P = (int)gridDim.x - p.U;
  return g <= p.U ? 0 : T * (g - p.U) / P;
}
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

// L [m][d] fp32 (global, written by other CTAs of this launch) -> [64][kQS] shared, zero outside m x d
// (zero columns add nothing to an L1 distance, so d = 32 landmarks work in the same 64-wide layout).
__device__ __forceinline__ void load_landmarks(const float* Lg, float* Ls, int m, int d = 64) {
  constexpr int kN4 = 1024 / kFT;   // float4 of the [64][64] block per thread
  float4 v[kN4];
#pragma unroll
  for (int i = 0; i < kN4; ++i) {
    const int e4 = threadIdx.x + kFT * i, r = e4 >> 4, c = 4 * (e4 & 15);
    v[i] = (r < m && c < d) ? __ldcg(reinterpret_cast<const float4*>(Lg + (size_t)r * d + c))
                            : make_float4(0.f, 0.f, 0.f, 0.f);
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

// One thread issues; out of line, so that the unrolled bodies exist once in the kernel's code
// (it is called from several places).
__device__ __noinline__ void ns_issue(uint32_t sbase, uint32_t tmem, uint64_t* bar, int nks) {
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
  load_landmarks(p.L + (size_t)u * m * p.d, Ls, m, p.d);
  __syncthreads();
  // W (symmetric): entries a <= b < m of the upper triangle, dealt out evenly (entry e -> (a, b)
  // in row-major triangle order), mirrored; padding rows and columns are zero
  {
    const int ntri = m * (m + 1) / 2;
    for (int e = t; e < 64 * 64; e += kFT) Ws[(e >> 6) * kQS + (e & 63)] = 0.f;
    __syncthreads();
    for (int e = t; e < ntri; e += kFT) {
      // row a holds entries [a m - a (a - 1) / 2, ...): invert with a float estimate, then fix up
      int a = (int)((2.f * m + 1.f - sqrtf((2.f * m + 1.f) * (2.f * m + 1.f) - 8.f * (float)e)) * 0.5f);
      a = a < 0 ? 0 : (a >= m ? m - 1 : a);
      while (a > 0 && a * m - a * (a - 1) / 2 > e) --a;
      while ((a + 1) * m - (a + 1) * a / 2 <= e) ++a;
      const int b = a + (e - (a * m - a * (a - 1) / 2));
      float acc0 = 0.f, acc1 = 0.f;
#pragma unroll 4
      for (int k = 0; k < 64; k += 8) {
        const float4 x0 = *reinterpret_cast<const float4*>(&Ls[a * kQS + k]);
        const float4 y0 = *reinterpret_cast<const float4*>(&Ls[b * kQS + k]);
        const float4 x1 = *reinterpret_cast<const float4*>(&Ls[a * kQS + k + 4]);
        const float4 y1 = *reinterpret_cast<const float4*>(&Ls[b * kQS + k + 4]);
        acc0 += fabsf(x0.x - y0.x);
        acc1 += fabsf(x1.x - y1.x);
        acc0 += fabsf(x0.y - y0.y);
        acc1 += fabsf(x1.y - y1.y);
        acc0 += fabsf(x0.z - y0.z);
        acc1 += fabsf(x1.z - y1.z);
        acc0 += fabsf(x0.w - y0.w);
        acc1 += fabsf(x1.w - y1.w);
      }
      const float v = exp2f((acc0 + acc1) * p.neg_log2e_over_lam) + (a == b ? p.eps : 0.f);
      Ws[a * kQS + b] = v;
      Ws[b * kQS + a] = v;
    }
  }
  __syncthreads();
  trace_mark(p, 16);
  // W + eps I for the backward pass, which reads the forward's context from the workspace
  for (int e = t; e < m * m; e += kFT) p.Wm[(size_t)u * m * m + e] = Ws[(e / m) * kQS + e % m];

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

  auto issue_round = [&]() {
    if (t == 0) ns_issue(sbase, tmem, bar, nks);
    __syncwarp();
  };
  auto finish_round = [&]() {
    mbar_wait(bar, round & 1, p.status, kStatusTimeout);
    tc_fence_after();
    tmem_ld16(trow, d);
    ++round;
  };
  auto run_round = [&]() {
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    issue_round();
    finish_round();
  };
  auto clean = [&](float* v) {
#pragma unroll
    for (int c = 0; c < 16; ++c)
      if (i >= m || 16 * h + c >= m) v[c] = 0.f;
  };

  // round 0: D_bottom = W W^T = W^2, which does not depend on alpha; while the tensor cores run it,
  // warps 2-3 (one W row per thread; warp 0 is busy issuing the product) find lambda_max = ||W||_2
  // (W symmetric positive definite) by power iteration from the ones vector, scaled by 1/m per
  // step (the Rayleigh quotient is scale free), synchronising on named barrier 1 only
  {
    float v[16];
#pragma unroll
    for (int c = 0; c < 16; ++c) v[c] = top ? 0.f : wrow[c];
    ns_store(sm, r, h, v);
  }
  fence_async_smem();
  tc_fence_before();
  __syncthreads();
  issue_round();
  if (w == 2 || w == 3) {
    const int row = t - 64;
    const float sc = 1.f / (float)m;
    float* v0 = vec;          // [2][64] ping-pong
    v0[row] = row < m ? 1.f : 0.f;
    named_bar_sync(1, 64);
    float wi = 0.f;
    for (int it = 0; it <= kPowerIters; ++it) {
      const float* vin = v0 + 64 * (it & 1);
      float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
#pragma unroll
      for (int j = 0; j < 64; j += 4) {
        const float4 wv = *reinterpret_cast<const float4*>(&Ws[row * kQS + j]);
        const float4 xv = *reinterpret_cast<const float4*>(&vin[j]);
        a0 = fmaf(wv.x, xv.x, a0);
        a1 = fmaf(wv.y, xv.y, a1);
        a2 = fmaf(wv.z, xv.z, a2);
        a3 = fmaf(wv.w, xv.w, a3);
      }
      wi = (a0 + a1) + (a2 + a3);
      if (it == kPowerIters) break;
      v0[64 * ((it + 1) & 1) + row] = wi * sc;
      named_bar_sync(1, 64);
    }
    const float vl = v0[64 * (kPowerIters & 1) + row];
    float vw = wi * vl, vv = vl * vl;
    for (int o = 16; o > 0; o >>= 1) {
      vw += __shfl_xor_sync(0xffffffffu, vw, o);
      vv += __shfl_xor_sync(0xffffffffu, vv, o);
    }
    if (lane == 0) {
      red[2 * (w - 2)] = vw;
      red[2 * (w - 2) + 1] = vv;
    }
  }
  __syncthreads();
  const float lmax = (red[0] + red[2]) / (red[1] + red[3]);
  // alpha = 2/||W||_2 as printed is kept only if ||I - alpha W W^T||_2 < 1, i.e. alpha lmax^2 < 2
  const float alpha_p = 2.f / lmax;
  const int fallback = (alpha_p * lmax * lmax < 2.f) ? 0 : 1;
  const float alpha = fallback ? 1.f / (lmax * lmax) : alpha_p;
  trace_mark(p, 17);
  finish_round();
  // X_0 = alpha W^T (= alpha W), R_0 = I - alpha W^2
  if (top) {
#pragma unroll
    for (int c = 0; c < 16; ++c) st[c] = alpha * wrow[c];
  } else {
#pragma unroll
    for (int c = 0; c < 16; ++c) st[c] = (i == 16 * h + c ? 1.f : 0.f) - alpha * d[c];
  }
  clean(st);
  trace_mark(p, 18);
  const int n_lit = p.T < 1 ? p.T : 1;
  const int n_res = p.T - n_lit;
  // residual steps: A = [X; R], D = [X R^T; R R^T]. Once every |R_k| entry is at most 2^-30, X R_k
  // and all later corrections (R squares at each step) are below 64 * 2^-30 = 2^-24 of max |X|, under
  // one fp32 rounding of X's largest entries: the chain moves on to the printed step, which
  // re-anchors R to I - W X. The test shares the barrier before the product's issue.
  for (int k = 0; k < n_res; ++k) {
    bool big = false;
    if (!top) {
#pragma unroll
      for (int c = 0; c < 16; ++c) big |= fabsf(st[c]) > 0x1p-30f;
    }
    ns_store(sm, r, h, st);
    fence_async_smem();
    tc_fence_before();
    if (!__syncthreads_or(big)) break;
    issue_round();
    finish_round();
    if (top) {
#pragma unroll
      for (int c = 0; c < 16; ++c) st[c] += d[c];
    } else {
#pragma unroll
      for (int c = 0; c < 16; ++c) st[c] = d[c];
    }
    clean(st);
  }
  trace_mark(p, 19);
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
  if (t == 0 && fa.xready != nullptr) {
    __threadfence();
    st_release_u64(fa.xready + u, fa.epoch);
  }
  trace_mark(p, 24);
  tc_fence_before();
  __syncthreads();
  return SolverInfo{alpha, lmax, fallback};
}

// Diagnostics of the unit's solve, ||I - W X_T||_F, by one more product of the same kind as the
// Newton-Schulz steps ([W; X_T] times X_T^T, 3xTF32). It runs right after the chain, while the row
// CTAs are still in pass 1 (the solver waits for their records anyway): W is still in the solver's
// scratch and X_T^T where the chain left it.
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
// Phase 2 (pass 1): C for a 128-row chunk: this warp's landmarks [j0, j0 + LT), lane rows lane + 32 a.
// ---------------------------------------------------------------------------------------
// Q rows come from a bf16 SW128 tile (TMA): one 16-byte read gives 8 channels of a row, and the
// lanes' rows spread the reads over all banks.
template <int LT>
__device__ __forceinline__ void cross_chunk(const unsigned char* qb, const float* Ls, unsigned char* cslot, int j0,
                                            int rb, int nrows, float scale, const float (&sh)[8], float (&s1)[8],
                                            float (&s2)[8]) {
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
      c[b] = valid ? ex2_approx(acc[a][b] * scale) - sh[b] : 0.f;
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
                                               int j0, int rb, int nrows, float scale, const float (&sh)[8],
                                               float (&s1)[8], float (&s2)[8]) {
  switch (lt) {
    case 1: cross_chunk<1>(Qs, Ls, cslot, j0, rb, nrows, scale, sh, s1, s2); break;
    case 2: cross_chunk<2>(Qs, Ls, cslot, j0, rb, nrows, scale, sh, s1, s2); break;
    case 3: cross_chunk<3>(Qs, Ls, cslot, j0, rb, nrows, scale, sh, s1, s2); break;
    case 4: cross_chunk<4>(Qs, Ls, cslot, j0, rb, nrows, scale, sh, s1, s2); break;
    case 5: cross_chunk<5>(Qs, Ls, cslot, j0, rb, nrows, scale, sh, s1, s2); break;
    case 6: cross_chunk<6>(Qs, Ls, cslot, j0, rb, nrows, scale, sh, s1, s2); break;
    case 7: cross_chunk<7>(Qs, Ls, cslot, j0, rb, nrows, scale, sh, s1, s2); break;
    case 8: cross_chunk<8>(Qs, Ls, cslot, j0, rb, nrows, scale, sh, s1, s2); break;
    default: break;
  }
}

// Column shift of C for one segment of this CTA: c_l = the mean of C over the first min(16, rows)
// tokens of the segment's first chunk, from its resident Q tile (bf16 SW128), in the pass-1
// arithmetic. Pass 1 keeps bf16(C - c) on chip instead of bf16(C), so the rounding error of a
// resident entry is relative to |C - c|, of the order of the column's spread, not to C: once
// whitening divides by that spread, the error stays at the bf16 level whatever mu / sigma is (large
// lambda). The segment's record carries c and its row count; the combine rebases every record of the
// unit to this CTA's own c, and pass 2's bias adds c back. Warp w takes token w, lane the landmarks
// lane and lane + 32; red is [16][64] fp32 scratch.
__device__ void segment_shift(const Params& p, const unsigned char* qtile, int nrows, const float* Ls, float* red,
                              float* shift) {
  const int t = threadIdx.x, w = t >> 5, lane = t & 31, m = p.m;
  const int nr = nrows < 16 ? nrows : 16;
  if (w < nr) {
    float acc0 = 0.f, acc1 = 0.f;
    const int l0 = lane, l1 = lane + 32 < m ? lane + 32 : lane;
#pragma unroll
    for (int k8 = 0; k8 < 8; ++k8) {
      const uint4 qv = *reinterpret_cast<const uint4*>(qtile + sw128(w, k8));
      const float q[8] = {bf_lo(qv.x), bf_hi(qv.x), bf_lo(qv.y), bf_hi(qv.y),
                          bf_lo(qv.z), bf_hi(qv.z), bf_lo(qv.w), bf_hi(qv.w)};
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        acc0 += fabsf(q[e] - Ls[l0 * kQS + 8 * k8 + e]);
        acc1 += fabsf(q[e] - Ls[l1 * kQS + 8 * k8 + e]);
      }
    }
    const float scale = p.neg_log2e_over_lam;
    red[w * 64 + lane] = lane < m ? ex2_approx(acc0 * scale) : 0.f;
    red[w * 64 + lane + 32] = lane + 32 < m ? ex2_approx(acc1 * scale) : 0.f;
  }
  __syncthreads();
  if (t < 64) {
    float c = 0.f;
    for (int r = 0; r < nr; ++r) c += red[r * 64 + t];
    shift[t] = t < m ? c / (float)nr : 0.f;
  }
  __syncthreads();
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
  float* Ls = reinterpret_cast<float*>(sm + kOffL);     // segment 0's landmarks
  float* Ls2 = reinterpret_cast<float*>(sm + kOffL2);   // segment 1's landmarks
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
  float* shift = reinterpret_cast<float*>(sm + kOffSh);   // [segment][landmark]
  float sh[8];
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
  // Both segments' landmarks and column shifts before the first chunk: segment 0's landmarks go to
  // the L area, segment 1's to the spare area after the third V stage; the shifts need each segment's
  // first Q chunk (all of them have landed once kBarQ completes) and scratch in C slot 0 (free until
  // chunk 0's C tile).
  mbar_wait(bars + kBarQ, 0, p.status, kStatusTimeout);
  for (int s = 0; s < R.nseg; ++s) {
    if (t == 0)
      spin_until_geq(fa.lready + R.seg[s].u, fa.epoch * (unsigned long long)m + (p.spin_test ? 1 : 0), p.status,
                     kStatusTimeout, p.spin_budget);
    __syncthreads();
    float* L = s ? Ls2 : Ls;
    load_landmarks(p.L + (size_t)R.seg[s].u * m * 64, L, m);
    __syncthreads();
    int s_, lo, nrows;
    R.chunk(R.seg[s].first_chunk, s_, lo, nrows);
    segment_shift(p, sm + kOffC + (R.seg[s].first_chunk + 1) * 16384, nrows, L, reinterpret_cast<float*>(sm + kOffC),
                  shift + 64 * s);
  }
  trace_mark(p, 2);
  float s1[8], s2[8];
  for (int gc = 0; gc < nch; ++gc) {
    int s, lo, nrows;
    R.chunk(gc, s, lo, nrows);
    const bool seg_first = gc == R.seg[s].first_chunk;
    const bool seg_last = gc == R.seg[s].first_chunk + R.seg[s].nch - 1;
    unsigned char* cslot = sm + kOffC + gc * 16384;
    // products run two chunks behind: tile gc - 2 is complete and its V stage has had a chunk
    if (t == 0 && gc >= 2) issue_mma(gc - 2);
    if (seg_first) {
#pragma unroll
      for (int b = 0; b < 8; ++b) {
        s1[b] = 0.f;
        s2[b] = 0.f;
        sh[b] = b < lt ? shift[64 * s + j0 + b] : 0.f;
      }
    }
    if (gc < 2) trace_mark(p, 10 + 11 * gc);
    if (lt > 0)
      cross_dispatch(lt, sm + kOffC + (gc + 1) * 16384, s ? Ls2 : Ls, cslot, j0, 64 * rh, nrows, scale, sh, s1, s2);
    if (padder) write_padding(cslot, 64 * rh, nrows, m);
    if (gc == 1) trace_mark(p, 22);
    if (gc == 3) {
      trace_mark_by(p, 23, 5 * 32);
      trace_mark_by(p, 26, 10 * 32);
      trace_mark_by(p, 27, 15 * 32);
    }
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
    if (gc >= 2 && gc < 7) trace_mark(p, gc == 6 ? 24 : 14 + gc);
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
  // inspection copy (lfa_debug_capture_cross): the resident bf16 tiles of C minus the column shift of
  // one unit, widened to fp32 [N][m] with the shift added back: the C that pass 2 effectively uses
  if (p.dbgC != nullptr) {
    for (int gc = 0; gc < nch; ++gc) {
      int s, lo, nrows;
      R.chunk(gc, s, lo, nrows);
      if (R.seg[s].u != p.dbg_unit) continue;
      const unsigned char* cs = sm + kOffC + gc * 16384;
      for (int e = t; e < nrows * m; e += kFT) {
        const int row = e / m, col = e % m;
        const uint32_t raw = *reinterpret_cast<const uint16_t*>(cs + sw128(row, col >> 3) + ((col & 7) << 1));
        p.dbgC[(size_t)(lo + row) * m + col] = __uint_as_float(raw << 16) + shift[64 * s + col];
        if (p.dbgS != nullptr) p.dbgS[(size_t)(lo + row) * m + col] = shift[64 * s + col];
      }
    }
  }
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
    if (t < 64) rec[kRecC + t] = shift[64 * s + t];
    if (t == 64) rec[kRecN] = (float)(R.seg[s].hi - R.seg[s].lo);
  }
  tc_fence_before();
  __syncthreads();
  if (t == 0) {
    __threadfence();
    for (int s = 0; s < R.nseg; ++s)
      st_release_u64(reinterpret_cast<unsigned long long*>(fa.rec + ((size_t)g * 2 + s) * kRec + kRecF), fa.epoch);
  }
}

// ---------------------------------------------------------------------------------------
// Row CTAs, after pass 1: DWC(V) of every chunk (§关键设计 1 "ZV + DWC(V)", 3 x 3 depthwise taps, zero
// padding 1), written to O as bf16; pass 2 then adds C M' + b onto it with TMA reduces. Chunk gc (rows
// [lo, lo + 128) of its unit) comes in as a V tile with a halo, in plain 128-byte rows (no swizzle):
// rows [lo - top, lo - top + 128 nbox) with top = 64, nbox = 2 when one grid row (W + 1 tokens) fits in
// 64 rows, else top = 128, nbox = 3; rows outside the unit read as zero. Three (two) tiles are in
// flight. Thread
// t owns 4 consecutive tokens of one grid row (4 (t / 16) .. of the chunk; W % 4 == 0, so a group never
// wraps) and 4 channels (t % 16), with the head's weights in registers as channel pairs; the products
// run as paired fp32 FMAs (two channels per instruction, each rounded as fmaf).
// ---------------------------------------------------------------------------------------
__device__ __forceinline__ uint64_t f32x2(float lo, float hi) {
  return (uint64_t)__float_as_uint(lo) | ((uint64_t)__float_as_uint(hi) << 32);
}
// two bf16 (low half: even channel) -> the fp32 pair
__device__ __forceinline__ uint64_t bf16x2_to_f32x2(uint32_t v) {
  return (uint64_t)(v << 16) | ((uint64_t)(v & 0xffff0000u) << 32);
}
__device__ __forceinline__ void ffma2(uint64_t& acc, uint64_t a, uint64_t b) {
  asm("fma.rn.f32x2 %0, %1, %2, %0;" : "+l"(acc) : "l"(a), "l"(b));
}
__device__ __forceinline__ uint32_t pack_f32x2_bf16(uint64_t v) {
  return pack_bf16(__uint_as_float((uint32_t)v), __uint_as_float((uint32_t)(v >> 32)));
}

// DWC of `count` chunks, chunk i = (unit, first row) from get(i) (a callable), from V tiles with a
// halo in `nbuf` contiguous buffers at `tiles` (barriers kBarH ..), results to O as bf16.
template <typename Get>
__device__ void dwc_chunks(const Params& p, unsigned char* tiles, int nbuf, uint64_t* bars,
                           const CUtensorMap* tmapVp, int count, Get get) {
  const int t = threadIdx.x, W = p.W, H = p.H, N = p.N;
  const int nbox = (W + 1 <= 64) ? 2 : 3, top = (nbox == 2) ? 64 : 128;
  const uint32_t tbytes = (uint32_t)nbox * 16384u;
  auto issue = [&](int i) {
    int u, lo;
    get(i, u, lo);
    const int b = i % nbuf;
    mbar_expect_tx(bars + kBarH + b, tbytes);
    for (int k = 0; k < nbox; ++k)
      tma_load_3d(tiles + b * tbytes + k * 16384, tmapVp, 0, lo - top + kChunk * k, u, bars + kBarH + b);
  };
  if (t == 0)
    for (int i = 0; i < count && i < nbuf; ++i) issue(i);
  const int grp = t >> 4, c4 = t & 15, r0 = 4 * grp;
  uint64_t wt[9][2];   // tap, channel pair (4 c4, 4 c4 + 1), (4 c4 + 2, 4 c4 + 3)
  int head = -1;
#pragma unroll 1
  for (int i = 0; i < count; ++i) {
    int u, lo;
    get(i, u, lo);
    const int nrows = min(kChunk, N - lo);
    if (u % p.heads != head) {
      head = u % p.heads;
      const float* wp = p.dwc + (size_t)head * 64 * 9;
#pragma unroll
      for (int tap = 0; tap < 9; ++tap)
#pragma unroll
        for (int e = 0; e < 2; ++e)
          wt[tap][e] = f32x2(__ldg(wp + (4 * c4 + 2 * e) * 9 + tap), __ldg(wp + (4 * c4 + 2 * e + 1) * 9 + tap));
    }
    const int b = i % nbuf;
    mbar_wait(bars + kBarH + b, (i / nbuf) & 1, p.status, kStatusTimeout);
    if (r0 < nrows) {
      __nv_bfloat16* O = static_cast<__nv_bfloat16*>(p.O) + (size_t)u * N * 64;
      const int n0 = lo + r0, y = n0 / W, x0 = n0 - y * W;
      const bool xl = x0 > 0, xr = x0 + 4 < W;
      // tile row of token (y - 1, x0 - 1): (n0 - W - 1) - (lo - top); grid row y + a - 1 is W rows on
      const unsigned char* base = tiles + b * tbytes + (size_t)(r0 - W - 1 + top) * 128 + 8 * c4;
      uint64_t acc[4][2];
#pragma unroll
      for (int k = 0; k < 4; ++k) acc[k][0] = acc[k][1] = 0ull;
#pragma unroll
      for (int a = 0; a < 3; ++a) {
        const int yy = y + a - 1;
        if (yy < 0 || yy >= H) continue;
        const unsigned char* rowp = base + (size_t)a * W * 128;
        uint64_t x[6][2];
#pragma unroll
        for (int j = 0; j < 6; ++j) {
          uint2 raw = make_uint2(0u, 0u);
          if ((j > 0 || xl) && (j < 5 || xr)) raw = *reinterpret_cast<const uint2*>(rowp + j * 128);
          x[j][0] = bf16x2_to_f32x2(raw.x);
          x[j][1] = bf16x2_to_f32x2(raw.y);
        }
#pragma unroll
        for (int bb = 0; bb < 3; ++bb)
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            ffma2(acc[k][0], wt[a * 3 + bb][0], x[k + bb][0]);
            ffma2(acc[k][1], wt[a * 3 + bb][1], x[k + bb][1]);
          }
      }
      uint2* op = reinterpret_cast<uint2*>(O + (size_t)n0 * 64 + 4 * c4);
#pragma unroll
      for (int k = 0; k < 4; ++k)
        if (r0 + k < nrows) op[16 * k] = make_uint2(pack_f32x2_bf16(acc[k][0]), pack_f32x2_bf16(acc[k][1]));
    }
    __syncthreads();   // tile b read by every thread
    if (t == 0 && i + nbuf < count) issue(i + nbuf);
  }
  // the DWC values in O (generic-proxy stores) come before any TMA reduce onto them
  asm volatile("fence.proxy.async.global;" ::: "memory");
}

// Row CTAs, after pass 1: DWC of this CTA's chunks, except the first dwc_take chunks of each segment,
// which the segment's unit's solver CTA computes while it waits for the pass-1 records (so every row
// CTA hands over the same share). The tile buffers are contiguous from C slot kMaxChunks - 1 (free: a
// CTA has at most kMaxChunks - 1 chunks, and the Q tile that slot held is consumed) through the V
// stages, Q and L (free after pass 1): three of two boxes or two of three.
__device__ void row_dwc(const Params& p, const FusedArgs& fa, const Rows& R, unsigned char* sm, uint64_t* bars,
                        const CUtensorMap* tmapVp) {
  const int nbuf = (p.W + 1 <= 64) ? 3 : 2;
  int list[kMaxChunks];
  int n = 0;
  for (int gc = 0; gc < R.nchunks; ++gc) {
    const int s = (R.nseg > 1 && gc >= R.seg[1].first_chunk) ? 1 : 0;
    if (gc - R.seg[s].first_chunk >= fa.dwc_take) list[n++] = gc;
  }
  __syncthreads();   // pass 1 is done with the V stages, Q and L
  dwc_chunks(p, sm + kOffDwcTiles, nbuf, bars, tmapVp, n, [&](int i, int& u, int& lo) {
    int s, nrows;
    R.chunk(list[i], s, lo, nrows);
    u = R.seg[s].u;
  });
  __syncthreads();
  trace_mark(p, 25);
}

// Solver CTA of unit u, after its chain and diagnostics: its share of the unit's DWC, the first
// dwc_take chunks of each row CTA's part of the unit. Thread 0 lists them (chunk indices in the unit, in
// row order) in the b area, free until the combine; the tiles go to the free scratch from offset 0
// (four buffers of two boxes or two of three).
__device__ void solver_dwc(const Params& p, const FusedArgs& fa, unsigned char* sm, uint64_t* bars, int u,
                           const CUtensorMap* tmapVp) {
  int* list = reinterpret_cast<int*>(sm + kOffBv);   // [0] count, then the chunks
  if (threadIdx.x == 0) {
    const int nchu = (p.N + kChunk - 1) / kChunk, lo = u * nchu, hi = lo + nchu;
    int n = 0;
    for (int gg = chunk_owner(lo, p); gg <= chunk_owner(hi - 1, p); ++gg) {
      const int a = max(cta_chunk0(gg, p), lo), b = min(cta_chunk0(gg + 1, p), hi);
      for (int c = a; c < b && c < a + fa.dwc_take && n < kDwcListCap; ++c) list[1 + n++] = c - lo;
    }
    list[0] = n;
  }
  __syncthreads();   // the list is out; the chain's scratch is no longer read
  dwc_chunks(p, sm, (p.W + 1 <= 64) ? 4 : 2, bars, tmapVp, list[0], [&](int i, int& uu, int& lo) {
    uu = u;
    lo = kChunk * list[1 + i];
  });
  __syncthreads();
}

// ---------------------------------------------------------------------------------------
// Phase 3, on the unit's solver CTA as the contributors' pass-1 records come out (X is its own):
// sum the records (each rebased from its column shift c_k to none: S1 += S1'_k + n_k c_k, S2 += S2'_k +
// 2 c_k S1'_k + n_k c_k^2 in fp64, P += P'_k + c_k (sum_i v_i)_k^T in fp32), form mu, var,
// s = 1/sqrt(var + eps), A = C~^T V by rank-1 folding (§关键设计 1), M = X A (fp32 FMA), M' = diag(s) M
// and b0 = (1/N - s o mu)^T M. M'^T goes out as the bf16 SW128 image of pass 2's B operand (row k =
// channel, column l = landmark, zero for l >= m), and each contributor's record gets its pass-2 bias
// b_k = b0 + c_k^T M' (its resident tiles hold C - c_k, so C M' = (C - c_k) M' + 1 c_k^T M'), in fp32
// from the unrounded M'. Then a release flag.
// ---------------------------------------------------------------------------------------
__device__ void solver_combine(const Params& p, const FusedArgs& fa, unsigned char* sm, int u) {
  const int t = threadIdx.x, w = t >> 5, lane = t & 31;
  const int m = p.m, N = p.N;
  float* As = reinterpret_cast<float*>(sm + kOffAs);
  float* Xt = reinterpret_cast<float*>(sm + kOffXt);
  double* S1d = reinterpret_cast<double*>(sm + kOffS1);
  double* S2d = reinterpret_cast<double*>(sm + kOffS2);
  float* mus = reinterpret_cast<float*>(sm + kOffMu);
  float* scs = reinterpret_cast<float*>(sm + kOffSc);
  float* svs = reinterpret_cast<float*>(sm + kOffSv);
  int* wcount = reinterpret_cast<int*>(sm + kOffWc);
  int* ctr = reinterpret_cast<int*>(sm + kOffCt);
  const float invNf = 1.f / (float)N;
  const double invN = 1.0 / (double)N;
  // contributors: candidates gf..gl (the owners of the unit's first and last chunks); CTAs with an
  // empty range (possible when there are fewer chunks than CTAs) publish nothing and are dropped
  const int nchu = (N + kChunk - 1) / kChunk;
  const int gf = chunk_owner(u * nchu, p);
  const int gl = chunk_owner(u * nchu + nchu - 1, p);
  const int ncand = gl - gf + 1;
  bool nonempty = false;
  int rec_off = 0;
  if (t < ncand) {
    const int gg = gf + t;
    const int a = cta_start(gg, p);
    nonempty = cta_start(gg + 1, p) > a;
    rec_off = (gg * 2 + (a < u * N ? 1 : 0)) * kRec;
  }
  const unsigned bal = __ballot_sync(0xffffffffu, nonempty);
  if (lane == 0) wcount[w] = __popc(bal);
  __syncthreads();
  int before = __popc(bal & ((1u << lane) - 1u)), nct = 0;
  for (int k = 0; k < kWarps; ++k) {
    if (k < w) before += wcount[k];
    nct += wcount[k];
  }
  if (nonempty && before < kMaxContrib) ctr[before] = rec_off;
  nct = nct < kMaxContrib ? nct : kMaxContrib;
  __syncthreads();   // the contributor table
  float* Mp = reinterpret_cast<float*>(sm + kOffMpf);   // M' fp32 [64][68] (row l)
  unsigned char* img = sm + kOffMp;
  // X^T (row j, column l), zero outside m x m (X is this CTA's own): the product below reads it along l
  {
    constexpr int kNX = 64 * 64 / kFT;   // X entries per thread, all loads issued first
    float xv[kNX];
#pragma unroll
    for (int k = 0; k < kNX; ++k) {
      const int e = t + kFT * k, l = e >> 6, j = e & 63;
      xv[k] = 0.f;
      if (l < m && j < m) xv[k] = ld_cg_f32_ordered(p.X + ((size_t)u * m + l) * m + j);
    }
#pragma unroll
    for (int k = 0; k < kNX; ++k) {
      const int e = t + kFT * k, l = e >> 6, j = e & 63;
      Xt[j * kQS + l] = xv[k];
    }
  }
  // Sum the unit's records in contributor order as they are published, each rebased from its own
  // column shift c_k to none:
  //   S1 += S1'_k + n_k c_k,  S2 += S2'_k + 2 c_k S1'_k + n_k c_k^2   (fp64),
  //   P  += P'_k, then P += c_k (sum_i v_i)_k^T                       (fp32; row 63 of P'_k holds sum_i v_i)
  // Thread 0 waits for the next record's flag, takes every consecutive record already out (at most
  // kRecBatch) as one batch and copies them whole into shared memory by bulk copies on one mbarrier;
  // then all threads add them in order. The additions follow the contributor order whatever the batches
  // are, so the result does not depend on timing. Each record's c_k also goes to cks for the biases.
  float* cks = reinterpret_cast<float*>(sm + kOffCks);   // [kMaxContrib][64] the contributors' shifts
  int* batch = reinterpret_cast<int*>(sm + kOffBatch);  // records in the current batch
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + kOffBar);
  {
    constexpr int kNP = 1024 / kFT;   // float4 of P per thread: rows (t >> 4) + 32 k, columns 4 (t & 15)
    const int col4 = t & 15;
    double a1 = 0.0, a2 = 0.0;
    float4 pacc[kNP];
#pragma unroll
    for (int k = 0; k < kNP; ++k) pacc[k] = make_float4(0.f, 0.f, 0.f, 0.f);
    auto flag = [&](int c) {
      return reinterpret_cast<const unsigned long long*>(fa.rec + ctr[c] + kRecF);
    };
    int nbatch = 0;
    for (int c0 = 0; c0 < nct;) {
      if (t == 0) {
        spin_until_geq(flag(c0), fa.epoch, p.status, kStatusTimeout, p.spin_budget);
        int nb = 1;
        while (c0 + nb < nct && nb < kRecBatch && ld_acquire_u64(flag(c0 + nb)) >= fa.epoch) ++nb;
        *batch = nb;
        // the records are generic-proxy stores of other CTAs, released with their flags; the buffers
        // were last read (and the DWC tiles before them written) through the generic proxy
        asm volatile("fence.proxy.async.global;" ::: "memory");
        fence_async_smem();
        mbar_expect_tx(bars + kBarRec, (uint32_t)nb * kRecBytes);
        for (int c = 0; c < nb; ++c)
          bulk_load(sm + kOffRecBuf + c * kRecBytes, fa.rec + ctr[c0 + c], kRecBytes, bars + kBarRec);
      }
      __syncthreads();
      if (nbatch == 0) trace_mark(p, 7);
      const int nb = *batch;
      mbar_wait(bars + kBarRec, nbatch & 1, p.status, kStatusTimeout);
      for (int c = 0; c < nb; ++c) {
        const float* r = reinterpret_cast<const float*>(sm + kOffRecBuf + c * kRecBytes);
        if (t < 64) {
          const double cc = (double)r[kRecC + t], nk = (double)r[kRecN];
          const double s1 = (double)r[t];
          a1 += s1 + nk * cc;
          a2 += (double)r[64 + t] + 2.0 * cc * s1 + nk * cc * cc;
          cks[(c0 + c) * 64 + t] = r[kRecC + t];
        }
        const float4 sv = *reinterpret_cast<const float4*>(r + 128 + 63 * 64 + 4 * col4);
#pragma unroll
        for (int k = 0; k < kNP; ++k) {
          const float4 pv = reinterpret_cast<const float4*>(r + 128)[t + kFT * k];
          const float ck = r[kRecC + (t >> 4) + 32 * k];
          pacc[k].x = fmaf(ck, sv.x, pacc[k].x + pv.x);
          pacc[k].y = fmaf(ck, sv.y, pacc[k].y + pv.y);
          pacc[k].z = fmaf(ck, sv.z, pacc[k].z + pv.z);
          pacc[k].w = fmaf(ck, sv.w, pacc[k].w + pv.w);
        }
      }
      c0 += nb;
      ++nbatch;
      __syncthreads();   // the buffers and the batch size are rewritten by the next batch
    }
    if (t < 64) {
      S1d[t] = a1;
      S2d[t] = a2;
    }
#pragma unroll
    for (int k = 0; k < kNP; ++k) {
      const int e4 = t + kFT * k;
      *reinterpret_cast<float4*>(As + (e4 >> 4) * kQS + 4 * (e4 & 15)) = pacc[k];
    }
  }
  __syncthreads();
  trace_mark(p, 8);
  // mu, var and s from the totals (fp64)
  if (t < 64) {
    const double mup = S1d[t] * invN;
    double var = S2d[t] * invN - mup * mup;
    if (var < 0.0) var = 0.0;
    const double sc = 1.0 / sqrt(var + (double)p.eps);
    mus[t] = t < m ? (float)mup : 0.f;
    scs[t] = t < m ? (float)sc : 0.f;
    svs[t] = As[63 * kQS + t];       // landmark column 63 holds sum_i v_i
    if (t < m) {
      p.mu[(size_t)u * m + t] = (float)mup;
      p.s[(size_t)u * m + t] = (float)sc;
    }
  }
  __syncthreads();
  // A = C~^T V from P = C^T V by the rank-1 fold, in place (whitened: C~ = (C - mu) s + 1/N, so
  // A[l][k] = s_l (P[l][k] - mu_l sum_i v_ik) + sum_i v_ik / N; raw: A = P). Zero for l >= m.
  for (int e = t; e < 64 * 64; e += kFT) {
    const int l = e >> 6, k = e & 63;
    float a = 0.f;
    if (l < m) {
      const float P = As[l * kQS + k];
      a = p.whiten ? scs[l] * (P - mus[l] * svs[k]) + svs[k] * invNf : P;
    }
    As[l * kQS + k] = a;
  }
  __syncthreads();
  trace_mark(p, 9);
  // M = X A on all threads: thread (k0 = 4 (t / 32), l0 = 2 (t % 32)) forms M[l0 .. l0 + 1][k0 .. k0 + 3].
  // A warp shares k0 (the A reads are broadcasts) and takes the 64 landmarks in pairs (conflict-free
  // X^T reads and image stores). Four steps j per iteration, alternating between two accumulator sets
  // (rows j >= m of X^T and A are zero, so the steps run to a multiple of 4).
  float* bvec = reinterpret_cast<float*>(sm + kOffBv);
  {
    const int l0 = 2 * (t & 31), k0 = 4 * (t >> 5);
    float acc[2][4], acc2[2][4];
#pragma unroll
    for (int r = 0; r < 2; ++r)
#pragma unroll
      for (int c = 0; c < 4; ++c) acc[r][c] = acc2[r][c] = 0.f;
    const int m4 = (m + 3) & ~3;
#pragma unroll 1
    for (int j0 = 0; j0 < m4; j0 += 4) {
      float2 x[4];
      float4 a[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        x[q] = *reinterpret_cast<const float2*>(&Xt[(j0 + q) * kQS + l0]);
        a[q] = *reinterpret_cast<const float4*>(&As[(j0 + q) * kQS + k0]);
      }
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        float(&ac)[2][4] = (q & 1) ? acc2 : acc;
        const float av[4] = {a[q].x, a[q].y, a[q].z, a[q].w};
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          ac[0][c] = fmaf(x[q].x, av[c], ac[0][c]);
          ac[1][c] = fmaf(x[q].y, av[c], ac[1][c]);
        }
      }
    }
#pragma unroll
    for (int r = 0; r < 2; ++r)
#pragma unroll
      for (int c = 0; c < 4; ++c) acc[r][c] += acc2[r][c];
    // M' = diag(s) M (raw: M), as fp32 rows for the bias and as the bf16 image; b0 = sum_l
    // (1/N - s_l mu_l) M[l] (raw: 0)
    float sc[2], coef[2];
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      const int l = l0 + r;
      const bool in = l < m;
      sc[r] = in ? (p.whiten ? scs[l] : 1.f) : 0.f;
      coef[r] = (in && p.whiten) ? invNf - scs[l] * mus[l] : 0.f;
    }
    float bp[4];
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const float m0 = sc[0] * acc[0][c], m1 = sc[1] * acc[1][c];
      Mp[l0 * kQS + k0 + c] = m0;
      Mp[(l0 + 1) * kQS + k0 + c] = m1;
      *reinterpret_cast<uint32_t*>(img + sw128(k0 + c, l0 >> 3) + ((l0 & 7) << 1)) = pack_bf16(m0, m1);
      bp[c] = coef[0] * acc[0][c] + coef[1] * acc[1][c];
    }
#pragma unroll
    for (int c = 0; c < 4; ++c)
      for (int o = 16; o > 0; o >>= 1) bp[c] += __shfl_xor_sync(0xffffffffu, bp[c], o);
    if (lane == 0) {
#pragma unroll
      for (int c = 0; c < 4; ++c) bvec[k0 + c] = bp[c];
    }
  }
  __syncthreads();
  trace_mark(p, 20);
  // the contributors' biases b_k = b0 + c_k^T M', and the image, out before the flag
  for (int e = t; e < nct * 64; e += kFT) {
    const int k = e >> 6, jc = e & 63;
    float b0 = 0.f, b1 = 0.f;   // two chains over the landmarks
    int l = 0;
    for (; l + 1 < m; l += 2) {
      b0 = fmaf(cks[k * 64 + l], Mp[l * kQS + jc], b0);
      b1 = fmaf(cks[k * 64 + l + 1], Mp[(l + 1) * kQS + jc], b1);
    }
    if (l < m) b0 = fmaf(cks[k * 64 + l], Mp[l * kQS + jc], b0);
    fa.rec[ctr[k] + kRecB + jc] = bvec[jc] + (b0 + b1);
  }
  for (int e = t; e < 512; e += kFT)
    reinterpret_cast<uint4*>(fa.mimg + (size_t)u * 8192)[e] = reinterpret_cast<const uint4*>(img)[e];
  __syncthreads();
  if (t == 0) {
    __threadfence();
    st_release_u64(fa.mready + u, fa.epoch);
  }
  trace_mark(p, 21);
}

// ---------------------------------------------------------------------------------------
// Phase 4: O += (C - c) M' + b_k for every chunk, onto the DWC values already in O (from this CTA's
// row_dwc or from the unit's solver). M'^T of each segment's unit is the image its solver CTA published
// (copied to the M' area for segment 0, to kOffImg1 for segment 1); b_k is the bias that solver wrote
// into this CTA's record for its column shift. Each chunk's products are issued by their own thread
// with their own barrier, and the epilogues (+ b_k, bf16) follow chunk by chunk. The bf16 rows are
// staged in the chunk's C slot (free once its product is done) and leave by TMA reduce-adds of 32-row
// quarters onto O: warps w, w + 4, w + 8, w + 12 hold the same 32 rows (16 channels each) and meet on
// named barrier 1 + w % 4 before warp w % 4 issues the quarter's reduce.
// ---------------------------------------------------------------------------------------
__device__ void pass2_all(const Params& p, const FusedArgs& fa, const Rows& R, unsigned char* sm, uint32_t sbase,
                          uint32_t tmem, uint64_t* bars, const CUtensorMap* tmapO) {
  const int t = threadIdx.x, w = t >> 5, lane = t & 31;
  const int nch = R.nchunks;
  float* bvec = reinterpret_cast<float*>(sm + kOffBv);
  auto img_off = [](int s) -> uint32_t { return s == 0 ? kOffMp : kOffImg1; };
  // each segment's M'^T image from its unit's solver CTA, and the pass-2 bias that CTA computed for
  // this CTA's record (its column shift)
  if (t == 0)
    for (int s = 0; s < R.nseg; ++s)
      spin_until_geq(fa.mready + R.seg[s].u, fa.epoch, p.status, kStatusTimeout, p.spin_budget);
  __syncthreads();
  // the solver CTAs' DWC values in O (generic-proxy stores, released with mready) come before this
  // CTA's TMA reduces onto them
  asm volatile("fence.proxy.async.global;" ::: "memory");
  trace_mark(p, 4);
  for (int s = 0; s < R.nseg; ++s) {
    const unsigned char* img = fa.mimg + (size_t)R.seg[s].u * 8192;
    for (int e = t; e < 512; e += kFT)
      reinterpret_cast<uint4*>(sm + img_off(s))[e] = __ldcg(reinterpret_cast<const uint4*>(img) + e);
    if (t < 64) bvec[64 * s + t] = __ldcg(fa.rec + ((size_t)blockIdx.x * 2 + s) * kRec + kRecB + t);
  }
  fence_async_smem();
  tc_fence_before();
  __syncthreads();
  trace_mark(p, 5);
  // each chunk's four products and its commit come from its own thread (lane 0 of warp kP2Warp0 + gc,
  // warps that issue no reduces), so the issues of different chunks overlap
  {
    const int gc = w - kP2Warp0;
    if (lane == 0 && gc >= 0 && gc < nch) {
      tc_fence_after();
      const uint32_t id = idesc(1, 128, 64, 0, 0);
      int s, lo, nrows;
      R.chunk(gc, s, lo, nrows);
      const uint64_t ca = desc_sw128(sbase + kOffC + gc * 16384, 16, 1024);
      const uint64_t mb = desc_sw128(sbase + img_off(s), 16, 1024);
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
        mma_bf16(tmem + 64 * gc, ca + (uint64_t)(kk * 2), mb + (uint64_t)(kk * 2), id, kk > 0 ? 1u : 0u);
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
    // rows past the unit's end (a short last chunk) fall outside the tensor and are skipped
    if (h == 0 && lane == 0 && 32 * q < nrows) {
      tma_reduce_add_3d(tmapO, 0, lo + 32 * q, R.seg[s].u, ob + 4096 * q);
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
                                                           const __grid_constant__ CUtensorMap tmapO,
                                                           const __grid_constant__ CUtensorMap tmapVp) {
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
    for (int b = 0; b < kNumBars; ++b) mbar_init(bars + b, b == kBarDrain ? kDrainCount : 1);
    mbar_init_fence();
    if (g == 0) *p.status = 0;
    if (!solver) pass1_prefetch(R, sm, bars, &tmapV, &tmapQ);
  }
  if (t == 32) {
    tma_prefetch_desc(&tmapV);
    tma_prefetch_desc(&tmapQ);
    tma_prefetch_desc(&tmapO);
    tma_prefetch_desc(&tmapVp);
  }

  // ---- phase 0: landmark pooling ----
  // A landmark's r x r window is pooled by `span` warps of one CTA (1 for windows of at most 64 tokens,
  // up to 4 for larger ones), each summing its share of the window's tokens in steps of 64; the partial
  // sums meet in shared memory (C slot 0, free until the first chunk) and the group's first warp adds
  // them in warp order. lane = (token group tg = lane / 8, 8 channels c8 = lane % 8); each load
  // instruction of a warp covers 4 window tokens x 128 bytes, all loads of a step are issued before use.
  {
    const __nv_bfloat16* Q = static_cast<const __nv_bfloat16*>(p.Q);
    const int total = U * m, Wr = p.W / p.r, rr = p.r * p.r;
    const int span = rr >= 256 ? 4 : (rr >= 128 ? 2 : 1);
    const int groups = kWarps / span, grp = w / span, part = w % span;
    const float inv = 1.f / (float)rr;
    const int tg = lane >> 3, c8 = lane & 7;
    float* psum = reinterpret_cast<float*>(sm + kOffC);   // [kWarps][64] partial sums
    for (int gl0 = g * groups; gl0 < total; gl0 += gridDim.x * groups) {
      const int gl = gl0 + grp;   // the group's landmark (the whole CTA takes the same loop trips)
      float a[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      const int u = gl < total ? gl / m : 0, l = gl % m;
      if (gl < total) {
        const int y0 = (l / Wr) * p.r, x0 = (l % Wr) * p.r;
        const __nv_bfloat16* base = Q + ((size_t)u * N) * 64 + 8 * c8;
        for (int k0 = 64 * part; k0 < rr; k0 += 64 * span) {
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
      }
      if (span > 1) {
        if (tg == 0) {
#pragma unroll
          for (int e = 0; e < 8; ++e) psum[w * 64 + 8 * c8 + e] = a[e];
        }
        named_bar_sync(1 + grp, 32 * span);
        if (part == 0 && tg == 0) {
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            float acc = a[e];
            for (int q = 1; q < span; ++q) acc += psum[(w + q) * 64 + 8 * c8 + e];
            a[e] = acc;
          }
        }
        named_bar_sync(1 + grp, 32 * span);   // psum is rewritten by the next trip
      }
      if (gl < total && part == 0) {
        if (tg == 0) {
          float* dst = p.L + ((size_t)u * m + l) * 64 + 8 * c8;
          *reinterpret_cast<float4*>(dst) = make_float4(a[0] * inv, a[1] * inv, a[2] * inv, a[3] * inv);
          *reinterpret_cast<float4*>(dst + 4) = make_float4(a[4] * inv, a[5] * inv, a[6] * inv, a[7] * inv);
        }
        // one landmark of unit u is out: the unit's consumers wait for m of them (no grid barrier)
        __syncwarp();
        if (lane == 0) {
          __threadfence();
          red_release_add_u64(fa.lready + u, 1ull);
        }
      }
    }
  }
  trace_mark(p, 1);
  __syncthreads();   // the TMEM address, the mbarrier initialisation and the row plan are visible
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  // solver CTAs take no rows (R.nchunks == 0): the unit's chain, then its diagnostics; the row
  // CTAs of the unit pick up X for their own combine
  if (solver) {
    if (t == 0) spin_until_geq(fa.lready + g, fa.epoch * (unsigned long long)m + (p.spin_test ? 1 : 0), p.status,
                               kStatusTimeout, p.spin_budget);
    __syncthreads();
    trace_mark(p, 2);
    const SolverInfo si = solver_cta(p, fa, sm, sbase, tmem, bars, g);
    trace_mark(p, 3);
    solver_diagnostics(p, sm, sbase, tmem, bars, g, si);
    solver_dwc(p, fa, sm, bars, g, &tmapVp);
    solver_combine(p, fa, sm, g);
  }
  if (R.nchunks > 0) {
    pass1(p, fa, R, sm, sbase, tmem, bars, &tmapV);
    trace_mark(p, 3);
    row_dwc(p, fa, R, sm, bars, &tmapVp);
    pass2_all(p, fa, R, sm, sbase, tmem, bars, &tmapO);
  }
  // drain: the tcgen05 operations of every issuing thread (thread 0: solver and pass-1 products;
  // lane 0 of warps kP2Warp0 .. kP2Warp0 + 6: pass-2 products) have completed before TMEM is released.
  // In a normal run each was waited already; after an expired wait this bounds the wait for any still
  // running. (A commit with nothing outstanding arrives at once.)
  if (t == 0 || (lane == 0 && w >= kP2Warp0 && w < kP2Warp0 + kMaxChunks - 1)) mma_commit(bars + kBarDrain);
  if (t == 0) mbar_wait(bars + kBarDrain, 0, p.status, kStatusTimeout);
  __syncthreads();
  trace_mark(p, 15);
  trace_clock(p, 14);
  if (w == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace

// The Newton-Schulz chain of the fused kernel as a kernel of its own, one CTA per (batch, head) unit,
// for the per-stage path (any dtype, d = 32 or 64, m <= 64): W, alpha, the T steps on tcgen05 in
// 3xTF32 and the diagnostics, from landmarks already pooled into the workspace; X and W go to the
// workspace (the per-stage passes and the backward read them there).
__global__ void __launch_bounds__(kFT, 1) k_ns_tc(const Params p) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
  unsigned char* sm = smem_raw + pad;
  const uint32_t sbase = smem_u32(sm);
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + kOffBar);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + kOffBar + kTmemSlot);
  const int t = threadIdx.x, w = t >> 5;
  if (w == 0) {
    tmem_alloc(tmem_slot, 64);
    tmem_relinquish();
  }
  if (t == 0) {
    mbar_init(bars + kBarNs, 1);
    mbar_init(bars + kBarDiag, 1);
    mbar_init_fence();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  FusedArgs fa;
  memset(&fa, 0, sizeof(fa));
  fa.epoch = 1;
  const SolverInfo si = solver_cta(p, fa, sm, sbase, tmem, bars, blockIdx.x);
  solver_diagnostics(p, sm, sbase, tmem, bars, blockIdx.x, si);
  tc_fence_before();
  __syncthreads();
  if (w == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 64);
  }
}

// Flag area: three [U] flag arrays (lready, xready, mready), each padded to 256 B; then the
// per-CTA pass-1 records and the per-unit M' images.
static size_t flag_stride(int U) { return 256 * (size_t)((U * 8 + 255) / 256); }
static size_t flag_bytes(int U) { return 3 * flag_stride(U); }

size_t fused_workspace_bytes(int U) {
  return flag_bytes(U) + sizeof(float) * (size_t)kMaxGrid * 2 * kRec + (size_t)U * 8192;
}

cudaError_t ns_tc_set_attributes() {
  return cudaFuncSetAttribute(k_ns_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemAlloc);
}

cudaError_t launch_ns_tc(const Params& p, cudaStream_t st) {
  k_ns_tc<<<p.U, kFT, kSmemAlloc, st>>>(p);
  return cudaGetLastError();
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
  // the DWC phase's token groups of 4 stay on one grid row, and one grid row plus a token fits in the
  // 128-row halo above and below a chunk
  if (p.W % 4 != 0 || p.W > 127) return 0;
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
constexpr int kTmapCache = 48;   // Q, V (two layouts) and O maps of a few rotating buffer sets
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
    // the flags and the records (whose published flags hold epochs of earlier launches)
    const cudaError_t e = cudaMemsetAsync(fused_ws, 0, flag_bytes(p.U) + sizeof(float) * (size_t)kMaxGrid * 2 * kRec, st);
    if (e != cudaSuccess) return e;
  }
  CUtensorMap tmap, tmapq, tmapo, tmapvp;
  if (!tmap_for(p.V, p.N, p.U, kChunk, true, &tmap)) return cudaErrorInvalidValue;
  if (!tmap_for(p.V, p.N, p.U, kChunk, false, &tmapvp)) return cudaErrorInvalidValue;
  if (!tmap_for(p.Q, p.N, p.U, kChunk, true, &tmapq)) return cudaErrorInvalidValue;
  if (!tmap_for(p.O, p.N, p.U, 32, true, &tmapo)) return cudaErrorInvalidValue;
  FusedArgs fa;
  fa.epoch = epoch;
  const size_t fs = flag_stride(p.U);
  fa.lready = reinterpret_cast<unsigned long long*>(fused_ws);
  fa.xready = reinterpret_cast<unsigned long long*>(fused_ws + fs);
  fa.mready = reinterpret_cast<unsigned long long*>(fused_ws + 2 * fs);
  fa.mimg = fused_ws + flag_bytes(p.U) + sizeof(float) * (size_t)kMaxGrid * 2 * kRec;
  fa.rec = reinterpret_cast<float*>(fused_ws + flag_bytes(p.U));
  plan_pass1_warps(p.m, fa);
  // The solver CTAs wait, after their chain, for the pass-1 records; they spend that time on the DWC
  // of the first chunks of each row CTA's part of their unit. Rough model: a chunk of pass 1 takes
  // about 6.8 us, the chain with its diagnostics about 34 us, a chunk of DWC about 1.5 us, so a
  // solver has room for k = (6.8 cpc - 34) / 1.5 chunks (cpc the chunks of a row CTA), shared by the
  // about nchu / cpc + 1 row CTAs of a unit: take = k cpc / (nchu + cpc), rounded.
  {
    const int nchu = (p.N + kChunk - 1) / kChunk;
    const int cpc = (p.U * nchu + (G - p.U) - 1) / (G - p.U);
    int k = (68 * cpc - 340) / 15;
    k = k < 0 ? 0 : k;
    int take = (2 * k * cpc + (nchu + cpc)) / (2 * (nchu + cpc));
    take = take > cpc ? cpc : take;
    take = take > kMaxDwcTake ? kMaxDwcTake : take;
    fa.dwc_take = take;
  }
  Params pp = p;
  void* args[] = {(void*)&pp, (void*)&fa, (void*)&tmap, (void*)&tmapq, (void*)&tmapo, (void*)&tmapvp};
  if (p.ev_begin) cudaEventRecord(static_cast<cudaEvent_t>(p.ev_begin), st);
  cudaError_t e = cudaLaunchCooperativeKernel((const void*)k_fused_forward, dim3(G), dim3(kFT), args, kSmemAlloc, st);
  if (p.ev_end) cudaEventRecord(static_cast<cudaEvent_t>(p.ev_end), st);
  return e;
}

}  // namespace lfa
