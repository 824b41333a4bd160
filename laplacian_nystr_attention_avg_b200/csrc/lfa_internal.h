// Internal declarations shared by the host entry points and the kernels of liblfa.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "lfa.h"

namespace lfa {

constexpr int kMaxM = 256;        // largest landmark count supported
constexpr int kMaxT = 64;         // largest Newton-Schulz step count accepted
constexpr int kRowTile = 64;      // token rows per tile in the generic kernels
constexpr int kThreads = 256;     // threads per CTA in the generic kernels
constexpr int kSmallM = 64;       // m <= kSmallM: one CTA solves a unit's Newton-Schulz chain

// default bound (SM clock cycles, about 1 s) on the fused kernel's waits for flags of other CTAs
constexpr long long kFlagSpinBudget = 1ll << 31;

// status-word bits (device side); lfa_get_info maps them to lfa_status
constexpr int kStatusTimeout = 1;
constexpr int kStatusNonFinite = 2;

// per-unit diagnostics slots (floats) in the workspace
constexpr int kInfoAlpha = 0, kInfoLambdaMax = 1, kInfoFallback = 2, kInfoResidual = 3, kInfoKappa = 4;
constexpr int kInfoStride = 5;

__host__ __device__ inline int round_up(int a, int b) { return (a + b - 1) / b * b; }
__host__ __device__ inline int ceil_div(int a, int b) { return (a + b - 1) / b; }

// Byte offsets of every buffer carved from the caller's workspace.
struct Layout {
  size_t status, info, L, Wm, X, Xb, Y, part, red, mu, s, A, M, Mp, bpart;
  size_t fused;    // scratch of the fused forward (per-CTA partials, barriers)
  size_t bwd;      // backward-pass buffers (start of the region)
  size_t b_its, b_G, b_Gn, b_T1, b_T2, b_T3, b_dW, b_part2, b_red2, b_dA, b_Gm, b_Gd, b_beta, b_gamma,
      b_bpart2, b_dLpart, b_dLns, b_dLpool, b_dQd;
  size_t total;
};

// Everything a kernel needs, passed by value.
struct Params {
  // shape
  int B, heads, H, W, N, d, r, m, T, whiten, dtype, U;
  float lam, eps;
  float neg_log2e_over_lam;  // C = exp2(D * neg_log2e_over_lam)
  // generic pass-1 decomposition
  int P;             // pass-1 CTAs per unit
  int tiles_per_cta; // 64-row tiles per pass-1 CTA
  int n_tiles;       // 64-row tiles per unit
  int part_stride;   // floats per partial record: S1[m], S2[m], P[m][d], SV[d]
  int n_chunks;      // combine row chunks of 16 landmarks (bias partials)
  // tensors
  const void* Q;
  const void* V;
  void* O;
  const float* dwc;
  // workspace views
  int* status;
  float* info;
  float* L;      // [U][m][d]
  float* Wm;     // [U][m][m] (W + eps I)
  float* X;      // [U][m][m]
  float* Xb;     // [U][m][m] ping-pong buffer of the multi-CTA Newton-Schulz
  float* Y;      // [U][m][m]
  float* part;   // [U][P][part_stride]
  double* red;   // [U][part_stride]
  float* mu;     // [U][m]
  float* s;      // [U][m]
  float* A;      // [U][m][d]
  float* M;      // [U][m][d]
  float* Mp;     // [U][m][d]
  float* bpart;  // [U][n_chunks][d]
  // optional timing events bracketing the dominant kernel (cudaEvent_t or null)
  void* ev_begin;
  void* ev_end;
  // optional second stream and fork / join events (cudaStream_t, cudaEvent_t, or null): the
  // per-stage kernels run the Newton-Schulz chain there, concurrently with pass 1 (they share no data);
  // ev_mid and ev_x mark pass 1 done and X_T ready, so that the closing residual runs beside the combine
  void* aux_stream;
  void* ev_fork;
  void* ev_mid;
  void* ev_x;
  void* ev_join;
  // optional per-CTA phase timestamps (%globaltimer, ns) of the fused kernel: [grid][16]
  unsigned long long* trace;
  // optional copy of the cross kernel C of unit dbg_unit as computed by this forward, fp32 [N][m]
  float* dbgC;
  float* dbgS;   // optional: the column shift subtracted before bf16 rounding, per entry, fp32 [N][m]
  int dbg_unit;
  // sequence split (per-stage kernels only): this call holds grid rows [y0, y0 + H) of every unit's
  // Hg x W grid (Ng = Hg W tokens enter the column statistics); Vh, when not null, holds the V rows
  // y0 - 1 and y0 + H of every unit ([U][2][W][d], zero rows outside the grid) for DWC
  int y0, Hg, Ng;
  const void* Vh;
  // fused kernel: bound (SM cycles) on its waits for flags that other CTAs set; with spin_test the
  // landmark waits look for one landmark more than exist, so every one of them runs out (tests)
  long long spin_budget;
  int spin_test;
};

// Backward-pass tensors and workspace views (with the forward's Params).
struct BwdParams {
  Params p;
  const void* dO;
  void* dQ;
  void* dV;
  float* its;      // [U][T][m][m] Newton-Schulz iterates X_0 .. X_{T-1}
  float* G;        // [U][m][m] adjoint of the current iterate (starts as dX)
  float* Gn;       // [U][m][m]
  float* T1;       // [U][m][m] products of the reverse step
  float* T2;
  float* T3;
  float* dW;       // [U][m][m]
  float* part2;    // [U][P][part_stride] pass-1 partials with dO in the place of V
  double* red2;    // [U][part_stride]
  float* dA;       // [U][m][d]
  float* Gm;       // [U][m][d] s o M
  float* Gd;       // [U][m][d] s o dA
  float* beta;     // [U][m] whitening-backward coefficients
  float* gamma;    // [U][m]
  float* bpart2;   // [U][n_chunks][d] bias partials of dV
  float* dLpart;   // [U][P][m][d] main-pass partials of dL
  float* dLns;     // [U][m][d] landmark-gram part of dL
  float* dLpool;   // [U][m][d] dL / r^2
  float* dQd;      // [U][N][d] fp32 direct part of dQ
};

// One batched m x m product: Out[u] = scale * op(A[u]) op(B[u]) + beta * C[u] + add_diag * I
// (op = transpose when ta / tb is set; C may be null and may alias Out; A and B must not).
struct MmJob {
  const float* A;
  size_t a_stride;   // floats between consecutive units' matrices
  const float* B;
  size_t b_stride;
  const float* C;
  size_t c_stride;
  float* O;
  size_t o_stride;
  float scale, beta, add_diag;
  int ta, tb;
};
struct MmJobs {
  MmJob job[3];
  int n;
};

// A Newton-Schulz chain for k < steps: Y = 2I - W X_k, X_{k+1} = X_k Y, per unit (strides in floats
// between units' matrices). X_k: seq = 0 ping-pongs between xa (k even) and xb (k odd); seq = 1 reads
// X_k at xa + k step and writes X_{k+1} at xa + (k + 1) step. status: the device status word (timeout
// bit of the bounded waits).
struct NsChain {
  const float* W;
  size_t w_stride;
  float* Y;
  size_t y_stride;
  float* xa;
  float* xb;
  size_t x_stride;
  size_t step;
  int m, steps, seq;
  int* status;
};

// host helpers implemented in lfa_generic.cu / lfa_fused.cu / lfa_backward.cu / lfa_gemm.cu
// Up to three independent jobs (none reads another's output) in one launch; status as above.
cudaError_t launch_mm(const MmJob* jobs, int njobs, int m, int U, cudaStream_t st, int* status);
// the whole chain in one launch (a thread-block cluster per unit); false: not launched (no cluster of
// the needed size fits), the caller runs the products with launch_mm
bool launch_ns_chain(const NsChain& c, int U, cudaStream_t st);
// whether launch_ns_chain runs for this m on the current device
bool ns_chain_fits(int m);
// blocks (one per SM) of one unit's cluster in launch_ns_chain
int ns_chain_blocks(int m);
cudaError_t gemm_set_attributes();
cudaError_t ns_tc_set_attributes();
cudaError_t launch_ns_tc(const Params& p, cudaStream_t st);
cudaError_t launch_generic_forward(const Params& p, cudaStream_t st);
cudaError_t launch_generic_context(const Params& p, cudaStream_t st);
cudaError_t launch_generic_pass1_reduce(const Params& p, cudaStream_t st);
cudaError_t launch_generic_ns(const Params& p, cudaStream_t st);
// alpha, the Newton-Schulz steps and the closing residual from W in p.Wm (p.X out, p.Xb / p.Y scratch;
// uses p.U, p.m, p.T, p.info, p.status)
cudaError_t launch_ns_from_w(const Params& p, cudaStream_t st);
// conjugate gradients for U systems W Y = B (lfa_solvers.cu)
cudaError_t cg_set_attributes();
cudaError_t launch_cg(const float* W, const float* B, float* Y, int U, int m, int nrhs, int iters,
                      cudaStream_t st);
cudaError_t launch_generic_finish(const Params& p, cudaStream_t st);
cudaError_t launch_backward(const BwdParams& b, cudaStream_t st);

// on_main(st) and on_aux(s) with s = p.aux_stream, concurrently: s waits for st's work so far, and
// st waits for s's before it continues. Without an auxiliary stream both run on st, on_aux first.
template <typename FMain, typename FAux>
void fork_join(const Params& p, cudaStream_t st, FMain on_main, FAux on_aux) {
  if (p.aux_stream && p.ev_fork && p.ev_join) {
    cudaStream_t aux = static_cast<cudaStream_t>(p.aux_stream);
    cudaEventRecord(static_cast<cudaEvent_t>(p.ev_fork), st);
    cudaStreamWaitEvent(aux, static_cast<cudaEvent_t>(p.ev_fork), 0);
    on_aux(aux);
    cudaEventRecord(static_cast<cudaEvent_t>(p.ev_join), aux);
    on_main(st);
    cudaStreamWaitEvent(st, static_cast<cudaEvent_t>(p.ev_join), 0);
  } else {
    on_aux(st);
    on_main(st);
  }
}
size_t backward_smem_main(int d);
cudaError_t backward_set_attributes();
int backward_launch_count(const Params& p);
cudaError_t launch_pool(const Params& p, cudaStream_t st);
cudaError_t launch_cross_kernel(const Params& p, int unit, float* C_out, cudaStream_t st);
cudaError_t launch_kappa(const Params& p, cudaStream_t st);
size_t generic_smem_pass1(int m, int d);
size_t generic_smem_pass2(int m, int d);
cudaError_t generic_set_attributes();
int generic_launch_count(const Params& p);
// tcgen05 streaming passes for bf16 tokens, d = 64, m <= 256 (lfa_stream.cu): pass 1 writes its
// partial records with its own CTA count per unit, which it returns (0: not launched); pass 2 returns
// false when it does not apply
bool stream_eligible(const Params& p);
cudaError_t stream_set_attributes();
int stream_pass1(const Params& p, cudaStream_t st);
// pass 1 split over launches: tiles (64 tokens) per unit; the CTAs per unit one launch over the tiles
// [t_begin, t_end) takes with at most P; that launch, its records rec0 .. of rec_n per unit (rec_n <= p.P),
// false when it does not apply
int stream_tiles(const Params& p);
bool stream_maps_ok(const Params& p);
int stream_range_blocks(int t_begin, int t_end, int P);
bool stream_pass1_range(const Params& p, int t_begin, int t_end, int P, int rec0, int rec_n, cudaStream_t st);
bool stream_pass2(const Params& p, cudaStream_t st);
size_t fused_workspace_bytes(int U);
int fused_grid(const Params& p);
cudaError_t launch_fused_forward(const Params& p, int G, unsigned char* fused_ws, unsigned long long epoch,
                                 cudaStream_t st);
cudaError_t launch_selftest(int mode, const float* A, const float* B, float* D, int param, const void* tma_src,
                            int tma_rows, int* status, cudaStream_t st);

}  // namespace lfa
