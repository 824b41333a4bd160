// Batched m x m products for the per-stage kernels (m <= 256) on the tcgen05 tensor cores: the
// Newton-Schulz steps of the forward pass (LaplacianFormer note, papernotes.org, §关键设计 3) when the
// one-CTA chain does not apply, the iterates and the reverse steps of the backward pass, and the
// Reading-B products.
//
// Out = scale * op(A) op(B) + beta * Cin + add_diag * I per (job, unit); up to three independent jobs
// share one launch (grid z = job * U + unit). Each CTA (512 threads) forms a 128 x 64 output tile
// (M = 128 rows i, N = 64 columns j) in a TMEM accumulator, fp32-accurate by three TF32 products
// (hi*hi + hi*lo + lo*hi with hi = tf32(x), lo = x - hi: about 2^-21 relative per product). Two tile
// bodies, each compiled per transpose combination:
//   * m % 4 == 0 (mm_tile_async): K in steps of 32; the operands arrive by cp.async in a three-slot
//     ring in the layout the tensor cores read (K- or MN-major, no transposing stores), fifteen warps
//     split each step in place while one lane of the last warp issues the products of the step before;
//   * other m (mm_tile): K in steps of 64; the operands of step c + 1 wait in registers while the 24
//     MMAs of step c run, then are split and stored (transposes element by element) into the other of
//     two stages, and the loads of step c + 2 go out right after.
// The epilogue stages the tile through shared memory and writes whole rows.
//
// The Newton-Schulz chains (the forward's X_{k+1} = X_k (2I - W X_k), k < T, and the backward's
// iterates X_1 .. X_{T-1}) also run as ONE launch, k_ns_chain: a thread-block cluster per unit whose
// blocks each own one 128 x 64 output tile of every product and meet at a cluster barrier between
// products (operands through L2, loads that bypass L1). This removes the per-product launch and the
// cold instruction fetch that dominated it.
#include <mutex>

#include "lfa_internal.h"
#include "lfa_sm100.cuh"

namespace lfa {
namespace {

using namespace sm100;

constexpr int kTM = 128, kTN = 64, kKS = 64;
constexpr int kGT = 512;                          // threads per CTA
constexpr uint32_t kAH = kTM * 128;               // bytes of one K-half of one A split tile
constexpr uint32_t kBH = kTN * 128;               // bytes of one K-half of one B split tile
// stage: A hi [2 halves], A lo [2], B hi [2], B lo [2]
constexpr uint32_t kOffAhi = 0, kOffAlo = 2 * kAH, kOffBhi = 4 * kAH, kOffBlo = 4 * kAH + 2 * kBH;
constexpr uint32_t kStage = 4 * kAH + 4 * kBH;    // 96 KB
constexpr uint32_t kGemmSmem = 2 * kStage + 1024 + 64;
constexpr int kAR = kTM * kKS / 4 / kGT;          // float4 groups of A per thread and step (4)
constexpr int kBR = kTN * kKS / 4 / kGT;          // of B (2)

// byte offset of (row, fp32 column k < 64) in a K-major split tile made of two SW128 K-halves
__device__ __forceinline__ uint32_t kofs(int row, int k, uint32_t half_bytes) {
  return (uint32_t)(k >> 5) * half_bytes + sw128(row, (k & 31) >> 2) + (k & 3) * 4;
}

struct Regs {
  float4 a[kAR];
  float4 b[kBR];
};

__device__ __forceinline__ void tile_epilogue(const MmJob& J, int m, int u, int i0, int j0, unsigned char* sm,
                                              uint32_t tmem);

// One 128 x 64 output tile (rows i0.., columns j0..) of job J for unit u. The two shared-memory stages
// and their commit barriers continue across calls: step c of this tile is global step gs + c, staged in
// buffer (gs + c) & 1 and committed on that buffer's barrier as its ((gs + c) >> 1)-th completion; gs
// advances by the tile's step count. Every commit is waited before the call returns, so the stages
// and the TMEM accumulator are free for the next call. Operands are read through L2 (ld.global.cg):
// in a chain they were written by other thread blocks since the previous product. TA / TB: the job's
// transposes (J.ta, J.tb), fixed at compile time so that each variant's code holds only its own paths.
template <int TA, int TB>
__device__ __noinline__ void mm_tile(const MmJob& J, int m, int u, int i0, int j0, unsigned char* sm, uint32_t sbase, uint32_t tmem,
                        uint64_t* bars, int* status, int& gs) {
  const float* A = J.A + u * J.a_stride;
  const float* B = J.B + u * J.b_stride;
  const int t = threadIdx.x;
  const bool vec = (m & 3) == 0;   // rows start on 16-byte boundaries
  // Group e of a step covers 4 consecutive elements along the stored matrix's contiguous index:
  //   A untransposed: row i = e / 16, k = 4 (e % 16) .. ;  transposed: row k = e / 32, i = 4 (e % 32) ..
  //   B transposed:   row j = e / 16, k = 4 (e % 16) .. ;  untransposed: row k = e / 16, j = 4 (e % 16) ..
  auto ld4 = [&](const float* base, int row, int col, int nrow, int ncol) -> float4 {
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    if (row < nrow) {
      const float* src = base + (size_t)row * m + col;
      if (vec && col + 3 < ncol) v = __ldcg(reinterpret_cast<const float4*>(src));
      else {
        v.x = col + 0 < ncol ? __ldcg(src + 0) : 0.f;
        v.y = col + 1 < ncol ? __ldcg(src + 1) : 0.f;
        v.z = col + 2 < ncol ? __ldcg(src + 2) : 0.f;
        v.w = col + 3 < ncol ? __ldcg(src + 3) : 0.f;
      }
    }
    return v;
  };
  auto load = [&](int c, Regs& r) {
    const int k0 = c * kKS;
#pragma unroll
    for (int x = 0; x < kAR; ++x) {
      const int e = t + kGT * x;
      r.a[x] = TA ? ld4(A, k0 + (e >> 5), i0 + 4 * (e & 31), m, m) : ld4(A, i0 + (e >> 4), k0 + 4 * (e & 15), m, m);
    }
#pragma unroll
    for (int x = 0; x < kBR; ++x) {
      const int e = t + kGT * x;
      r.b[x] = TB ? ld4(B, j0 + (e >> 4), k0 + 4 * (e & 15), m, m) : ld4(B, k0 + (e >> 4), j0 + 4 * (e & 15), m, m);
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
      if constexpr (!TA) {
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
      if constexpr (TB) {
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
  store(r, gs & 1);
  if (nk > 1) load(1, r);
  fence_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t id = idesc(2, kTM, kTN, 0, 0);
  for (int c = 0; c < nk; ++c) {
    const int g = gs + c, buf = g & 1;
    if (t == 0) {
      tc_fence_after();
      const uint32_t sb = sbase + buf * kStage;
#pragma unroll
      for (int pr = 0; pr < 3; ++pr) {
        const uint32_t ab = sb + ((pr == 2) ? kOffAlo : kOffAhi);
        const uint32_t bb = sb + ((pr == 1) ? kOffBlo : kOffBhi);
#pragma unroll
        for (int ks = 0; ks < kKS / 8; ++ks) {
          const uint64_t ad = desc_sw128(ab + (ks >> 2) * kAH, 16, 1024) + (uint64_t)((ks & 3) * 2);
          const uint64_t bd = desc_sw128(bb + (ks >> 2) * kBH, 16, 1024) + (uint64_t)((ks & 3) * 2);
          mma_tf32(tmem, ad, bd, id, (c > 0 || pr > 0 || ks > 0) ? 1u : 0u);
        }
      }
      mma_commit(bars + buf);
    }
    if (c + 1 < nk) {
      // buffer buf ^ 1 was read by the products of global step g - 1 (its ((g - 1) >> 1)-th commit);
      // at c = 0 that step belongs to an earlier tile, whose last wait covered it
      if (c >= 1) mbar_wait(bars + (buf ^ 1), ((g - 1) >> 1) & 1, status, kStatusTimeout);
      store(r, buf ^ 1);
      if (c + 2 < nk) load(c + 2, r);
      fence_async_smem();
      tc_fence_before();
      __syncthreads();
    }
  }
  // the last commit covers every product issued before it (and completes the earlier commits that
  // were not waited: the step before it on the other buffer)
  {
    const int g = gs + nk - 1;
    mbar_wait(bars + (g & 1), (g >> 1) & 1, status, kStatusTimeout);
    if (nk >= 2) mbar_wait(bars + ((g - 1) & 1), ((g - 1) >> 1) & 1, status, kStatusTimeout);
  }
  gs += nk;
  tc_fence_after();
  tile_epilogue(J, m, u, i0, j0, sm, tmem);
}

// Epilogue of a tile whose products are complete: warp w reads TMEM lanes 32 (w % 4) .., columns
// 16 (w / 4) .. into a [128][65] fp32 staging tile at sm (free), then the rows go out coalesced as
// Out = scale * acc + beta * Cin + add_diag * I.
__device__ __forceinline__ void tile_epilogue(const MmJob& J, int m, int u, int i0, int j0, unsigned char* sm,
                                              uint32_t tmem) {
  const float* Cin = J.C ? J.C + u * J.c_stride : nullptr;
  float* Out = J.O + u * J.o_stride;
  const float scale = J.scale, beta = J.beta, add_diag = J.add_diag;
  const int t = threadIdx.x, w = t >> 5, lane = t & 31;
  float* stg = reinterpret_cast<float*>(sm);
  {
    const int q = w & 3, h = w >> 2;
    float v[16];
    tmem_ld16(tmem + ((uint32_t)(32 * q) << 16) + 16 * h, v);
    const int il = 32 * q + lane;
#pragma unroll
    for (int x = 0; x < 16; ++x) stg[il * 65 + 16 * h + x] = v[x];
  }
  __syncthreads();
  if ((m & 3) == 0) {
    // four columns per store (rows start on 16-byte boundaries; j < m covers j + 3 < m)
    for (int e = t; e < kTM * kTN / 4; e += kGT) {
      const int il = e >> 4, jl = 4 * (e & 15), i = i0 + il, j = j0 + jl;
      if (i < m && j < m) {
        const float* sr = stg + il * 65 + jl;
        float4 o = make_float4(scale * sr[0] + (i == j ? add_diag : 0.f), scale * sr[1] + (i == j + 1 ? add_diag : 0.f),
                               scale * sr[2] + (i == j + 2 ? add_diag : 0.f), scale * sr[3] + (i == j + 3 ? add_diag : 0.f));
        if (Cin) {
          const float4 c = __ldcg(reinterpret_cast<const float4*>(Cin + (size_t)i * m + j));
          o.x = fmaf(beta, c.x, o.x);
          o.y = fmaf(beta, c.y, o.y);
          o.z = fmaf(beta, c.z, o.z);
          o.w = fmaf(beta, c.w, o.w);
        }
        *reinterpret_cast<float4*>(Out + (size_t)i * m + j) = o;
      }
    }
  } else {
    for (int e = t; e < kTM * kTN; e += kGT) {
      const int il = e >> 6, jl = e & 63, i = i0 + il, j = j0 + jl;
      if (i < m && j < m) {
        float o = scale * stg[il * 65 + jl] + (i == j ? add_diag : 0.f);
        if (Cin) o = fmaf(beta, __ldcg(Cin + (size_t)i * m + j), o);
        Out[(size_t)i * m + j] = o;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
}

// ---- asynchronous-copy variant (m % 4 == 0: every matrix row starts on a 16-byte boundary) -------
// K advances in steps of 32. The raw fp32 operand tiles of a step land by cp.async (16-byte chunks
// through L2, zero-filled past m) in one of three ring slots, already in the layout the tensor cores
// read, so no transpose is needed:
//   A untransposed (rows i, k contiguous): K-major, one SW128 K-half of 128 rows;
//   A transposed (stored [k][i]): MN-major, four 4 KB blocks of 32 i, one 128-byte line per k;
//   B untransposed (stored [k][j]): MN-major, two 4 KB blocks of 32 j, one line per k;
//   B transposed (rows j, k contiguous): K-major, one SW128 K-half of 64 rows.
// MN-major 32-bit operands use the 128-byte swizzle with 32-byte granules (descriptor layout type
// 1): the granule g < 4 of line k sits at position g ^ (k % 4); LBO = 4096 (next 32-element block
// along M / N), SBO = 512 (next group of 4 lines along K); one K = 8 product step is 8 lines, 1024
// bytes. A step is split in place (hi = tf32(x) over x, lo = x - hi beside it); its products then
// run while the next step is split, and the copies of step c + 2 go out once the products of step
// c - 1 have released their slot.
constexpr int kKS2 = 32;
constexpr uint32_t kQA = 16384, kQB = 8192;                                  // hi (raw) tiles
constexpr uint32_t kSlotHiA = 0, kSlotHiB = kQA, kSlotLoA = kQA + kQB, kSlotLoB = 2 * kQA + kQB;
constexpr uint32_t kSlot = 2 * (kQA + kQB);                                  // 48 KB
static_assert(3 * kSlot <= 2 * kStage, "ring slots beyond the tile's shared memory");

__device__ __forceinline__ void cp_async16(uint32_t dst, const float* src, bool valid) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(valid ? 16 : 0)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// byte offset of (line, 16-byte chunk c < 8) in an MN-major block of 128-byte lines (32-byte granules
// swizzled by line % 4)
__device__ __forceinline__ uint32_t mnofs(int line, int c) {
  return (uint32_t)(line * 128 + ((((c >> 1) ^ (line & 3)) << 5) | ((c & 1) << 4)));
}

// descriptor of an MN-major 32-bit operand in that layout, blocks of 32 elements 4096 bytes apart
__device__ __forceinline__ uint64_t desc_mn32(uint32_t saddr) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFF);
  d |= (uint64_t)((4096u >> 4) & 0x3FFF) << 16;       // LBO
  d |= (uint64_t)((512u >> 4) & 0x3FFF) << 32;        // SBO
  d |= (uint64_t)1 << 46;                             // descriptor version (sm_100)
  d |= (uint64_t)1 << 61;                             // 128-byte swizzle, 32-byte atomicity
  return d;
}

// Ring slot and barrier of global step g: slot g % 3, committed on bars[g % 3] as that barrier's
// (g / 3)-th completion; every commit is waited once, in order. Warps 0-14 copy and split; lane 0 of
// warp 15 issues the products, so a step's split overlaps the products of the step before. Step c's
// hand-over from the splitters to the issuer is named barrier 2 + (c & 1) (the splitters arrive, the
// issuer warp waits): before the splitters arrive at step c + 2 they have waited (at step c + 1) for
// the products of step c, which the issuer issues only after its wait at step c, so an instance of a
// barrier never collects arrivals of two steps.
constexpr int kSplitters = kGT - 32;
template <int TA, int TB>
__device__ __noinline__ void mm_tile_async(const MmJob& J, int m, int u, int i0, int j0, unsigned char* sm,
                                           uint32_t sbase, uint32_t tmem, uint64_t* bars, int* status, int& gs) {
  const float* A = J.A + u * J.a_stride;
  const float* B = J.B + u * J.b_stride;
  const int t = threadIdx.x;
  const bool issuer = t >= kSplitters;
  const int nk = (m + kKS2 - 1) / kKS2;
  // This thread's copy items, fixed for the tile: up to three 16-byte chunks of A (1024 per step) and
  // two of B (512), each with its shared-memory offset inside a slot, its source at k0 = 0, the position
  // along K that bounds it (k0 + kpos < m) and whether its row / column lies inside the matrix. A step
  // advances K-major sources by k0 elements and MN-major ones by k0 rows.
  struct Item {
    const float* base;
    uint32_t dst;
    int kpos;
    bool in;
  };
  Item ia[3], ib[2];
#pragma unroll
  for (int x = 0; x < 3; ++x) {
    const int e = t + kSplitters * x;
    Item it{A, 0u, 0, false};
    if (e < 1024) {
      if constexpr (!TA) {
        const int row = e >> 3, kc = e & 7;
        it = Item{A + (size_t)(i0 + row) * m + 4 * kc, kSlotHiA + sw128(row, kc), 4 * kc, i0 + row < m};
      } else {
        const int kl = e >> 5, ic = e & 31;
        it = Item{A + (size_t)kl * m + i0 + 4 * ic, kSlotHiA + (ic >> 3) * 4096 + mnofs(kl, ic & 7), kl, i0 + 4 * ic < m};
      }
    }
    ia[x] = it;
  }
#pragma unroll
  for (int x = 0; x < 2; ++x) {
    const int e = t + kSplitters * x;
    Item it{B, 0u, 0, false};
    if (e < 512) {
      if constexpr (!TB) {
        const int kl = e >> 4, jc = e & 15;
        it = Item{B + (size_t)kl * m + j0 + 4 * jc, kSlotHiB + (jc >> 3) * 4096 + mnofs(kl, jc & 7), kl, j0 + 4 * jc < m};
      } else {
        const int jl = e >> 3, kc = e & 7;
        it = Item{B + (size_t)(j0 + jl) * m + 4 * kc, kSlotHiB + sw128(jl, kc), 4 * kc, j0 + jl < m};
      }
    }
    ib[x] = it;
  }
  const bool has_a[3] = {t < 1024, t + kSplitters < 1024, t + 2 * kSplitters < 1024};
  const bool has_b[2] = {t < 512, t + kSplitters < 512};
  auto issue = [&](int c) {
    const int k0 = c * kKS2;
    const uint32_t sl = sbase + ((gs + c) % 3) * kSlot;
    const size_t sa = TA ? (size_t)k0 * m : (size_t)k0, sb = TB ? (size_t)k0 : (size_t)k0 * m;
#pragma unroll
    for (int x = 0; x < 3; ++x)
      if (has_a[x]) {
        const bool ok = ia[x].in && k0 + ia[x].kpos < m;
        cp_async16(sl + ia[x].dst, ok ? ia[x].base + sa : A, ok);
      }
#pragma unroll
    for (int x = 0; x < 2; ++x)
      if (has_b[x]) {
        const bool ok = ib[x].in && k0 + ib[x].kpos < m;
        cp_async16(sl + ib[x].dst, ok ? ib[x].base + sb : B, ok);
      }
    cp_async_commit();
  };
  // a step's split: up to four float4 per thread, all loaded before any is converted (in place: hi over
  // the raw value, lo beside it)
  uint32_t so_hi[4], so_lo[4];
  bool so_ok[4];
#pragma unroll
  for (int x = 0; x < 4; ++x) {
    const int e = t + kSplitters * x;
    so_ok[x] = e < 1536;
    const uint32_t o = 16u * (e < 1024 ? e : e - 1024);
    so_hi[x] = (e < 1024 ? kSlotHiA : kSlotHiB) + o;
    so_lo[x] = (e < 1024 ? kSlotLoA : kSlotLoB) + o;
  }
  auto split_step = [&](uint32_t slot) {
    float4 v[4];
#pragma unroll
    for (int x = 0; x < 4; ++x)
      if (so_ok[x]) v[x] = *reinterpret_cast<const float4*>(sm + slot + so_hi[x]);
#pragma unroll
    for (int x = 0; x < 4; ++x)
      if (so_ok[x]) {
        float4 h, l;
        h.x = tf32_round(v[x].x); l.x = v[x].x - h.x;
        h.y = tf32_round(v[x].y); l.y = v[x].y - h.y;
        h.z = tf32_round(v[x].z); l.z = v[x].z - h.z;
        h.w = tf32_round(v[x].w); l.w = v[x].w - h.w;
        *reinterpret_cast<float4*>(sm + slot + so_hi[x]) = h;
        *reinterpret_cast<float4*>(sm + slot + so_lo[x]) = l;
      }
  };
  if (!issuer) {
    issue(0);
    if (nk > 1) issue(1);
    for (int c = 0; c < nk; ++c) {
      const int g = gs + c;
      const uint32_t slot = (g % 3) * kSlot;
      // this thread's copies of step c are in (those of step c + 1 may still be in flight)
      if (c + 1 < nk) cp_async_wait<1>();
      else cp_async_wait<0>();
      named_bar_sync(1, kSplitters);
      split_step(slot);
      fence_async_smem();
      named_bar_arrive(2 + (c & 1), kGT);
      // the products of step c - 1 are complete: their slot takes the copies of step c + 2
      if (c >= 1) mbar_wait(bars + (g - 1) % 3, ((g - 1) / 3) & 1, status, kStatusTimeout);
      if (c + 2 < nk) issue(c + 2);
    }
  } else {
    const uint32_t id = idesc(2, kTM, kTN, TA, TB ? 0 : 1);
    for (int c = 0; c < nk; ++c) {
      const int g = gs + c;
      named_bar_sync(2 + (c & 1), kGT);
      if (t == kSplitters) {
        tc_fence_after();
        const uint32_t sl = sbase + (g % 3) * kSlot;
#pragma unroll
        for (int pr = 0; pr < 3; ++pr) {
          const uint32_t ab = sl + ((pr == 2) ? kSlotLoA : kSlotHiA);
          const uint32_t bb = sl + ((pr == 1) ? kSlotLoB : kSlotHiB);
#pragma unroll
          for (int ks = 0; ks < kKS2 / 8; ++ks) {
            const uint64_t ad = TA ? desc_mn32(ab + ks * 1024) : desc_sw128(ab, 16, 1024) + (uint64_t)(ks * 2);
            const uint64_t bd = TB ? desc_sw128(bb, 16, 1024) + (uint64_t)(ks * 2) : desc_mn32(bb + ks * 1024);
            mma_tf32(tmem, ad, bd, id, (c > 0 || pr > 0 || ks > 0) ? 1u : 0u);
          }
        }
        mma_commit(bars + g % 3);
      }
      __syncwarp();
    }
  }
  {
    const int g = gs + nk - 1;
    mbar_wait(bars + g % 3, (g / 3) & 1, status, kStatusTimeout);
  }
  gs += nk;
  tc_fence_after();
  __syncthreads();
  tile_epilogue(J, m, u, i0, j0, sm, tmem);
}

// job J (transposes read at run time) by its compile-time variant; the asynchronous-copy tile when
// every row is 16-byte aligned
__device__ __forceinline__ void mm_tile_any(const MmJob& J, int m, int u, int i0, int j0, unsigned char* sm,
                                            uint32_t sbase, uint32_t tmem, uint64_t* bars, int* status, int& gs) {
  if ((m & 3) == 0) {
    if (J.ta) {
      if (J.tb) mm_tile_async<1, 1>(J, m, u, i0, j0, sm, sbase, tmem, bars, status, gs);
      else mm_tile_async<1, 0>(J, m, u, i0, j0, sm, sbase, tmem, bars, status, gs);
    } else {
      if (J.tb) mm_tile_async<0, 1>(J, m, u, i0, j0, sm, sbase, tmem, bars, status, gs);
      else mm_tile_async<0, 0>(J, m, u, i0, j0, sm, sbase, tmem, bars, status, gs);
    }
    return;
  }
  if (J.ta) {
    if (J.tb) mm_tile<1, 1>(J, m, u, i0, j0, sm, sbase, tmem, bars, status, gs);
    else mm_tile<1, 0>(J, m, u, i0, j0, sm, sbase, tmem, bars, status, gs);
  } else {
    if (J.tb) mm_tile<0, 1>(J, m, u, i0, j0, sm, sbase, tmem, bars, status, gs);
    else mm_tile<0, 0>(J, m, u, i0, j0, sm, sbase, tmem, bars, status, gs);
  }
}

__device__ __forceinline__ uint32_t gemm_setup(unsigned char* sm) {
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + 2 * kStage);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + 2 * kStage + 32);
  const int t = threadIdx.x;
  if ((t >> 5) == 0) {
    tmem_alloc(tmem_slot, 64);
    tmem_relinquish();
  }
  if (t == 0) {
    mbar_init(bars + 0, 1);
    mbar_init(bars + 1, 1);
    mbar_init(bars + 2, 1);
    mbar_init_fence();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  return *tmem_slot;
}

__device__ __forceinline__ void gemm_teardown(uint32_t tmem) {
  tc_fence_before();
  __syncthreads();
  if ((threadIdx.x >> 5) == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 64);
  }
}

__global__ void __launch_bounds__(kGT) k_mm_tc(int m, int U, MmJobs jobs, int* status) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
  unsigned char* sm = smem_raw + pad;
  const uint32_t tmem = gemm_setup(sm);
  const int jz = blockIdx.z / U, u = blockIdx.z % U;
  int gs = 0;
  mm_tile_any(jobs.job[jz], m, u, blockIdx.y * kTM, blockIdx.x * kTN, sm, smem_u32(sm),
              tmem, reinterpret_cast<uint64_t*>(sm + 2 * kStage), status, gs);
  gemm_teardown(tmem);
}

__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Newton-Schulz chain of unit blockIdx.y: for k < steps, Y = 2I - W X_k, X_{k+1} = X_k Y. Cluster
// (gridDim.x blocks, one per 128 x 64 output tile) per unit; the cluster barrier after each product
// publishes its tiles (release / acquire at cluster scope) before any block reads them. X_k is at
// xa + (k & 1 ? xb - xa : 0) (ping-pong, seq = 0) or xa + k step (seq = 1).
__global__ void __launch_bounds__(kGT) k_ns_chain(const NsChain c) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
  unsigned char* sm = smem_raw + pad;
  const uint32_t tmem = gemm_setup(sm);
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + 2 * kStage);
  const int m = c.m, u = blockIdx.y, nj = (m + kTN - 1) / kTN;
  const int i0 = (blockIdx.x / nj) * kTM, j0 = (blockIdx.x % nj) * kTN;
  const bool vec = (m & 3) == 0;
  int gs = 0;
  for (int k = 0; k < c.steps; ++k) {
    float* xk = c.seq ? c.xa + (size_t)k * c.step : ((k & 1) ? c.xb : c.xa);
    float* xn = c.seq ? c.xa + (size_t)(k + 1) * c.step : ((k & 1) ? c.xa : c.xb);
    const MmJob y{c.W, c.w_stride, xk, c.x_stride, nullptr, 0, c.Y, c.y_stride, -1.f, 0.f, 2.f, 0, 0};   // Y = 2I - W X_k
    if (vec) mm_tile_async<0, 0>(y, m, u, i0, j0, sm, smem_u32(sm), tmem, bars, c.status, gs);
    else mm_tile<0, 0>(y, m, u, i0, j0, sm, smem_u32(sm), tmem, bars, c.status, gs);
    cluster_sync_all();
    const MmJob x{xk, c.x_stride, c.Y, c.y_stride, nullptr, 0, xn, c.x_stride, 1.f, 0.f, 0.f, 0, 0};      // X_{k+1} = X_k Y
    if (vec) mm_tile_async<0, 0>(x, m, u, i0, j0, sm, smem_u32(sm), tmem, bars, c.status, gs);
    else mm_tile<0, 0>(x, m, u, i0, j0, sm, smem_u32(sm), tmem, bars, c.status, gs);
    cluster_sync_all();
  }
  gemm_teardown(tmem);
}

}  // namespace

cudaError_t gemm_set_attributes() {
  cudaError_t e = cudaFuncSetAttribute(k_mm_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kGemmSmem);
  if (e == cudaSuccess) e = cudaFuncSetAttribute(k_ns_chain, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kGemmSmem);
  return e;
}

namespace {

// launch configuration of the chain for m: G blocks per unit, one cluster of G per unit
int chain_blocks(int m) { return ((m + kTM - 1) / kTM) * ((m + kTN - 1) / kTN); }

void chain_config(cudaLaunchConfig_t& cfg, cudaLaunchAttribute* attr, int G, int U, cudaStream_t st) {
  cfg = {};
  cfg.gridDim = dim3(G, U, 1);
  cfg.blockDim = dim3(kGT, 1, 1);
  cfg.dynamicSmemBytes = kGemmSmem;
  cfg.stream = st;
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = G;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
}

}  // namespace

int ns_chain_blocks(int m) { return chain_blocks(m); }

// A cluster of the unit's G tiles (G <= 8, the portable cluster size: m <= 256) must fit on the device
// (one block per SM at this shared-memory size). Cached per (device, m).
bool ns_chain_fits(int m) {
  const int G = chain_blocks(m);
  if (m < 1 || m > kMaxM || G < 1 || G > 8) return false;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev >= 64) return false;
  static std::mutex mu;
  static signed char fits[64][kMaxM + 1];   // 0 unknown, 1 yes, -1 no
  std::lock_guard<std::mutex> lk(mu);
  if (fits[dev][m] == 0) {
    cudaLaunchConfig_t cfg;
    cudaLaunchAttribute attr[1];
    chain_config(cfg, attr, G, 1, 0);
    int n = 0;
    const bool ok = cudaOccupancyMaxActiveClusters(&n, k_ns_chain, &cfg) == cudaSuccess && n >= 1;
    if (!ok) cudaGetLastError();
    fits[dev][m] = ok ? 1 : -1;
  }
  return fits[dev][m] > 0;
}

// One launch for the whole chain when the unit's cluster fits; otherwise (returns false, nothing
// launched) the caller runs the products one launch each.
bool launch_ns_chain(const NsChain& c, int U, cudaStream_t st) {
  if (c.steps <= 0) return true;
  if (!ns_chain_fits(c.m)) return false;
  cudaLaunchConfig_t cfg;
  cudaLaunchAttribute attr[1];
  chain_config(cfg, attr, chain_blocks(c.m), U, st);
  return cudaLaunchKernelEx(&cfg, k_ns_chain, c) == cudaSuccess;
}

cudaError_t launch_mm(const MmJob* jobs, int njobs, int m, int U, cudaStream_t st, int* status) {
  if (njobs < 1 || njobs > 3) return cudaErrorInvalidValue;
  MmJobs js{};
  for (int i = 0; i < njobs; ++i) js.job[i] = jobs[i];
  js.n = njobs;
  const dim3 g(ceil_div(m, kTN), ceil_div(m, kTM), U * njobs);
  k_mm_tc<<<g, kGT, kGemmSmem, st>>>(m, U, js, status);
  return cudaGetLastError();
}

}  // namespace lfa
