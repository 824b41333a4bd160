/*
 * lfa.h -- C ABI of the Laplacian-kernel Nystrom attention library (liblfa.so),
 * built for NVIDIA B200 (sm_100a).
 *
 * What one call computes, per (batch b, head h) unit with tokens Q, V in
 * R^{N x d} on an H x W grid (token n = y*W + x):
 *   L   = r x r average pool of the query map, m = (H/r)(W/r) landmarks
 *         [LaplacianFormer note (papernotes.org), §关键设计 2: landmarks from
 *          average-pooling the reshaped query tensor, as in PVTv2];
 *   C   = exp(-||q_i - l_l||_1 / lambda)       (N x m cross kernel)
 *   W   = exp(-||l_a - l_b||_1 / lambda) + eps I   (m x m landmark kernel)
 *         [same note, §研究背景与动机 (核心 idea) for the kernel, §关键设计 2 for C and W,
 *          §关键设计 3 for the eps I shift];
 *   X   = Newton-Schulz pseudo-inverse of W, X_0 = alpha W^T,
 *         X_{k+1} = X_k (2I - W X_k), exactly T steps [§关键设计 3]. alpha = 2/||W||_2 as
 *         printed is kept only if ||I - alpha W W^T||_2 < 1; otherwise (always, since W
 *         has unit diagonal) alpha = 1/||W||_2^2 and the fallback is reported;
 *   C~  = (C - mu) / sqrt(var + eps) + 1/N, per-landmark-column mean and population
 *         variance over the unit's N rows [§关键设计 1, diagonal whitening];
 *   O   = C~ (X (C~^T V)) + DWC(V), DWC = 3x3 depthwise cross-correlation, zero
 *         padding 1, weights [heads][d][3][3] [§关键设计 1 output "ZV + DWC(V)";
 *         §整体框架 flowchart]. With whiten = 0 the raw C is used on both sides.
 *
 * Conventions for every entry point:
 *   - Tensors Q, V, O, dO, dQ, dV are contiguous [B][heads][N][d] in the config's
 *     dtype (fp32 or bf16). Device pointers must be 16-byte aligned.
 *     Arithmetic: distances, exponentials, sums and the whitening statistics are fp32 (the
 *     statistics' cross-CTA reductions fp64). The m x m Newton-Schulz products (and, in the
 *     fused kernel, M = X A) are split-TF32 tensor-core products (hi*hi + hi*lo + lo*hi, fp32
 *     accumulation). For bf16 tokens with d = 64 (the fused kernel, lfa_forward_path "fused",
 *     and the per-stage streaming passes) C^T V and C M' are bf16-operand tensor-core products
 *     with fp32 accumulation, taken on bf16(C - c) with c a per-column shift; for fp32 tokens and
 *     d = 32 the per-stage kernels run those two products in fp32 on CUDA cores.
 *   - The DWC weight is fp32 [heads][d][3][3] on the device.
 *   - All device memory is owned by the caller. The handle owns host state only and
 *     keeps the weight and workspace pointers it was created with; the weight is read
 *     at every call, not copied.
 *   - `stream` is a cudaStream_t (NULL = legacy default stream). Forward and
 *     backward only enqueue work: they never synchronise the host. The per-stage
 *     kernels also use the handle's own auxiliary stream (the landmark solver beside
 *     pass 1): that work waits for what `stream` held at the call and `stream` waits
 *     for it before the call's last kernels, so every call stays ordered on `stream`
 *     (and captures into a CUDA graph begun on `stream`).
 *   - Errors are returned as lfa_status; nothing is thrown across the ABI and the
 *     library never exits the process. Argument errors are detected on the host
 *     before any launch. Device-side conditions (a bounded wait that expired, a
 *     non-finite landmark kernel) set a status word in the workspace that
 *     lfa_get_info returns.
 *   - A handle must not be used by two host threads at once; calls on one handle
 *     that overlap on the GPU (different streams without ordering) race on its
 *     workspace.
 */
#ifndef LFA_H_
#define LFA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  LFA_OK = 0,
  LFA_ERR_INVALID_ARG = 1,   /* null pointer, bad size, misalignment, H%r or W%r != 0 ... */
  LFA_ERR_UNSUPPORTED = 2,   /* d not in {32, 64}, m > 256, unknown dtype; backward with
                                whiten = 3 */
  LFA_ERR_CUDA = 3,          /* a CUDA runtime call failed (launch, copy, attribute) */
  LFA_ERR_STATE = 4,         /* backward without a matching forward on this handle */
  LFA_ERR_TIMEOUT = 5,       /* a bounded device-side wait expired (reported by lfa_get_info) */
  LFA_ERR_NONFINITE = 6,     /* the landmark kernel or its norm was not finite */
  LFA_ERR_SCRATCH_LIMIT = 7  /* lfa_forward_noalloc: cfg needs more than LFA_NOALLOC_SCRATCH_BYTES */
} lfa_status;

typedef enum { LFA_F32 = 0, LFA_BF16 = 1 } lfa_dtype;

typedef struct {
  int B;          /* batch */
  int heads;      /* heads; units = B * heads */
  int H, W;       /* token grid, N = H * W */
  int d;          /* channels per head: 32 or 64 */
  int r;          /* pooling window; H % r == 0 and W % r == 0; m = (H/r)(W/r) <= 256 */
  float lambda;   /* Laplacian kernel scale, > 0 */
  float eps;      /* W regulariser and whitening epsilon, >= 0 */
  int T;          /* Newton-Schulz steps, 0 <= T <= 64 */
  int dtype;      /* lfa_dtype of Q, V, O, dO, dQ, dV */
  int whiten;     /* 1: whitened C~ on both sides (default); 0: raw C; 2: whitened, with mu and
                     var of each landmark column pooled per head over the B*N rows of all batch
                     elements (the note's statistics "over a batch", §关键设计 1; C~ keeps the
                     1/N of one unit). 3 ("Reading B"): the columns of the whole Nystrom matrix
                     G^ = C X C^T are whitened instead of those of C, O_attn = G~ V, in the
                     factored form (C - 1 c-^T) X C^T D^-1/2 V + (1/N) 1 1^T V with
                     D = diag(c_j^T X^T cov(C) X c_j + eps) over key tokens j; any m.
                     whiten = 2 and 3 run the per-stage kernels; whiten = 3 is forward only. */
} lfa_config;

/* Per-unit diagnostics of the most recent forward call. */
typedef struct {
  int alpha_fallback;    /* 1 when 2/||W||_2 failed ||I - alpha W W^T||_2 < 1 */
  float alpha;           /* alpha used for X_0 */
  float lambda_max;      /* estimate of ||W||_2 (power iteration; W is SPD) */
  float ns_residual_fro; /* ||I - W X_T||_F after the last step */
  float kappa;           /* estimate of the condition number of W + eps I: lambda_max times
                            ||X_T||_2 (power iteration; X_T approximates (W + eps I)^-1 once the
                            chain has converged), computed by lfa_get_info itself */
} lfa_unit_info;

typedef struct lfa_ctx* lfa_handle;

/* Bytes of device workspace a handle needs for `cfg` (0 if cfg is invalid). The
 * workspace holds the per-unit landmarks, W, X, whitening statistics, reduction
 * partials, the forward context that backward reuses, and the status word. */
size_t lfa_workspace_size(const lfa_config* cfg);

/* Validate cfg and build a handle. dwc_weight: device fp32 [heads][d][3][3].
 * workspace: device, >= lfa_workspace_size(cfg) bytes, 256-byte aligned, caller
 * owned for the handle's lifetime. No launch happens here; the handle creates its
 * auxiliary stream and four events, which lfa_destroy releases (without them the
 * per-stage kernels run one after the other on `stream`). */
lfa_status lfa_create(const lfa_config* cfg, const float* dwc_weight, void* workspace,
                      size_t workspace_bytes, lfa_handle* out);

/* Forward pass (see the file comment). Q, V: device inputs; O: device output, all
 * [B][heads][N][d] in cfg.dtype. Enqueued on `stream`. */
lfa_status lfa_forward(lfa_handle h, const void* Q, const void* V, void* O, void* stream);

/* Size of the static device scratch area behind lfa_forward_noalloc (16 MiB). */
#define LFA_NOALLOC_SCRATCH_BYTES (16u << 20)

/* Forward pass without a handle and without allocating anything: the same result as
 * lfa_forward (computed by the per-stage kernels that lfa_forward_path reports as
 * "generic"), with the intermediate data in one static device array of
 * LFA_NOALLOC_SCRATCH_BYTES inside the library instead of a caller workspace. This
 * entry point is a deployment convenience with no counterpart in the method's
 * description. It is meant for callers that may not allocate device memory: an
 * operator inside a host framework that owns the device memory pool and gives it no
 * allocator, or a latency-critical caller that cannot take the device-wide
 * synchronisation of cudaMalloc / cudaFree.
 *   cfg, dwc_weight, Q, V, O, stream: as for lfa_create and lfa_forward.
 *   Setup: every call looks up the device address of the scratch array on the current device
 *   (cudaGetSymbolAddress, a host-side query; nothing is cached across calls). The first call on a
 *   device may also load the library's device code there, so make that first call before any
 *   stream capture begins.
 *   Zeroing: nothing has to start at zero. Every scratch byte a call reads is written
 *   earlier by the same call; its status word is cleared by the call's first kernel.
 *   Limit: the scratch a config needs grows with B*heads and m (about
 *   B*heads*(16 m^2 + 24 m d + 4 P (m d + 2 m + d)) bytes with
 *   P <= min(ceil(296 / (B*heads)), ceil(N / 64)) row partitions); a config that needs more than LFA_NOALLOC_SCRATCH_BYTES is
 *   rejected with LFA_ERR_SCRATCH_LIMIT before any device work. B*heads = 32 on a
 *   56 x 56 grid with m = 49, d = 64 needs about 7.6 MiB; B*heads = 8 on a 112 x 112
 *   grid with m = 196 needs about 20 MiB and is rejected.
 *   Concurrency: there is one scratch array per device, shared by every call on that
 *   device. Calls that overlap on the GPU (two streams without ordering, or two host
 *   threads) race on it and give wrong results; order them on one stream.
 *   Diagnostics (lfa_get_info) are not available for these calls. */
lfa_status lfa_forward_noalloc(const lfa_config* cfg, const float* dwc_weight, const void* Q,
                               const void* V, void* O, void* stream);

/* Forward pass from and to HOST buffers: copies Q, V (host, [B][heads][N][d] in
 * cfg.dtype; pinned memory gives asynchronous copies) into the caller's device
 * buffers Q_dev, V_dev, runs lfa_forward into O_dev and copies O back to O_host.
 * Synchronises `stream` before returning, so O_host is ready on LFA_OK. */
lfa_status lfa_forward_host(lfa_handle h, const void* Q_host, const void* V_host, void* O_host,
                            void* Q_dev, void* V_dev, void* O_dev, void* stream);

/* lfa_forward_host without the final synchronisation: the two copies in, the forward and the copy out
 * are only enqueued on `stream`. O_host is ready, and the host and device buffers may be reused or
 * freed, once the caller has synchronised `stream` (or waited on an event recorded after the call).
 * With pinned host buffers, calls on two streams (two handles: a handle's workspace serves one call
 * at a time) overlap one call's copies with the other's forward and copies. Same arguments and argument
 * errors as lfa_forward_host. */
lfa_status lfa_forward_host_async(lfa_handle h, const void* Q_host, const void* V_host, void* O_host,
                                  void* Q_dev, void* V_dev, void* O_dev, void* stream);

/* Backward pass for the loss <dO, O>: writes dQ and dV ([B][heads][N][d], cfg.dtype).
 * Reuses the context saved by the most recent lfa_forward on this handle, which
 * must have been called with the same Q and V pointers (else LFA_ERR_STATE).
 * With batch-pooled statistics (whiten = 2) the whitening's reverse mode pools its two column
 * means over the B N rows of each head, as the forward pools mu and var. Reading B (whiten = 3)
 * has no backward: LFA_ERR_UNSUPPORTED.
 * The kernel gradient is -(1/lambda) sign(q - l) k with sign(0) = 0 [the note's
 * §研究背景与动机 prints the opposite sign]; alpha is held constant; the DWC
 * weight gets no gradient. */
lfa_status lfa_backward(lfa_handle h, const void* Q, const void* V, const void* dO,
                        void* dQ, void* dV, void* stream);

/* Copy per-unit diagnostics of the last forward into host_out[0..n_units-1]
 * (n_units must equal B * heads; the kappa estimate comes from one small kernel this call
 * launches on `stream`) and return the device status word
 * (LFA_OK, LFA_ERR_TIMEOUT or LFA_ERR_NONFINITE). Synchronises `stream`. After a
 * timeout the outputs of that call are invalid; the handle resets its cross-CTA flags
 * on the next forward. */
lfa_status lfa_get_info(lfa_handle h, lfa_unit_info* host_out, int n_units, void* stream);

/* Release the handle (host memory only; device memory stays the caller's). */
lfa_status lfa_destroy(lfa_handle h);

/* Static, human-readable name of a status code. */
const char* lfa_status_string(lfa_status s);

/* ---- sequence split over several devices ---------------------------------- *
 * One unit's N tokens can be split over devices in bands of whole grid rows (the note's 实验关键数据
 * and 局限 sections: memory grows linearly with the sequence, long sequences are the target). A
 * band handle holds grid rows [y0, y0 + ny) of every unit (its Q, V and O tensors are
 * [B][heads][ny * W][d] in cfg.dtype, token n = (y - y0) W + x). One forward is three exchanges of the
 * caller's choosing (all-reduce, neighbour send/receive), between four calls:
 *   1. lfa_sp_pool: this band's share of every landmark, L_partial [B*heads][m][d] fp32 (the sum over
 *      the window's tokens inside the band, divided by r^2); the SUM over all bands is L.
 *   2. lfa_sp_pass1(L): W, alpha and the Newton-Schulz chain from the full L (the same on every band),
 *      and this band's pass-1 sums, partial [B*heads][S] fp64 with S = lfa_sp_partial_size: column
 *      sums of C and C^2 [m] each, C^T V [m][d] and sum V [d]; the SUM over all bands is the unit's.
 *   3. lfa_sp_pass2(totals, halo): the combine from the summed partials (statistics over all H W
 *      tokens), then pass 2 and DWC for this band's rows. V_halo [B*heads][2][W][d] in cfg.dtype holds
 *      the V rows y0 - 1 and y0 + ny (from the neighbouring bands; any values where the row is outside
 *      the grid); it may be NULL when the band is the whole grid.
 * The result equals lfa_forward's on the whole grid up to the order of the sums. whiten = 0 or 1 only
 * (LFA_ERR_UNSUPPORTED otherwise); per-stage kernels; no backward. Band handles are rejected by
 * lfa_forward and lfa_backward (LFA_ERR_INVALID_ARG). Argument conventions as for lfa_create. */
size_t lfa_sp_workspace_size(const lfa_config* cfg, int y0, int ny);
lfa_status lfa_sp_create(const lfa_config* cfg, int y0, int ny, const float* dwc_weight, void* workspace,
                         size_t workspace_bytes, lfa_handle* out);
int lfa_sp_partial_size(lfa_handle h);
lfa_status lfa_sp_pool(lfa_handle h, const void* Q_local, float* L_partial, void* stream);
lfa_status lfa_sp_pass1(lfa_handle h, const void* Q_local, const void* V_local, const float* L_full,
                        double* partial_out, void* stream);
lfa_status lfa_sp_pass2(lfa_handle h, const void* Q_local, const void* V_local, const void* V_halo,
                        const double* partial_total, void* O_local, void* stream);

/* ---- solvers for the landmark system W Y = B -------------------------------------------------
 * The note solves with W by Newton-Schulz and ablates conjugate gradients against it, reporting
 * that CG degrades on ill-conditioned systems (condition number 50) while Newton-Schulz stays
 * stable (LaplacianFormer note, §关键设计 3 and the solver ablation). These two calls run both
 * solvers on caller-supplied matrices so the claim can be measured on the device; the forward
 * pass itself always uses Newton-Schulz. W: U symmetric positive-definite m x m matrices, fp32
 * row-major [U][m][m], 1 <= m <= 256; device pointers, 16-byte aligned, owned by the caller. */

/* Bytes of device workspace lfa_ns_solve needs for U systems of size m (0 for invalid sizes). */
size_t lfa_solver_workspace_size(int U, int m);

/* X [U][m][m] = the T-step Newton-Schulz approximation of W^-1 the forward pass computes:
 * alpha = 2 / ||W||_2 (power iteration; W must be symmetric, the iteration forms W v as the
 * columns' sums), or 1 / ||W||_2^2 when the printed condition
 * ||I - alpha W W^T||_2 < 1 fails; X_0 = alpha W^T; X <- X (2I - W X), each product on tcgen05 in
 * split TF32 (hi*hi + hi*lo + lo*hi, about 2^-21 relative). workspace: lfa_solver_workspace_size
 * bytes, 256-byte aligned, overwritten. host_out (optional, U entries): alpha, lambda_max,
 * the fallback flag and ||I - W X_T||_F per system (kappa = 0); with it the call synchronizes the
 * stream and returns LFA_ERR_NONFINITE if a value is not finite. LFA_ERR_INVALID_ARG for NULL or
 * misaligned pointers, sizes outside the bounds or T outside [0, 64]. */
lfa_status lfa_ns_solve(const float* W, float* X, int U, int m, int T, void* workspace, size_t workspace_bytes,
                        lfa_unit_info* host_out, void* stream);

/* Y [U][m][nrhs] = conjugate gradients for W Y = B (B [U][m][nrhs], fp32 row-major): for every
 * column an independent Hestenes-Stiefel recursion from Y_0 = 0, exactly `iters` iterations,
 * a = r^T r / p^T W p (0 when p^T W p <= 0), beta = r'^T r' / r^T r (0 when r^T r = 0), all in
 * fp32 with column sums in a fixed order (deterministic). W must be symmetric: the kernel reads
 * W[j][i] for W[i][j]. 1 <= nrhs <= 4096, 0 <= iters <= 4096; LFA_ERR_INVALID_ARG otherwise or
 * for NULL / misaligned pointers. Asynchronous on `stream`. */
lfa_status lfa_cg_solve(const float* W, const float* B, float* Y, int U, int m, int nrhs, int iters, void* stream);

/* ---- inspection entry points used by the parity tests ---------------------- */

/* Cross kernel C = exp(-||q_i - l_l||_1 / lambda) of one unit [the note's §关键设计 2],
 * written as fp32 [N][m] to the device buffer C_out by the per-stage kernels' tile code
 * (fp32 distance and exp2f), after pooling Q's landmarks into the handle's workspace. That
 * pooling replaces the saved forward context: lfa_backward then needs a new lfa_forward
 * (LFA_ERR_STATE until then). For the C that a forward itself multiplies (the fused kernel, or the
 * tensor-core pass 2 of the per-stage path), see lfa_debug_capture_cross. */
lfa_status lfa_debug_cross_kernel(lfa_handle h, const void* Q, int unit, float* C_out,
                                  void* stream);

/* Test of the bounded waits (no device fault, no hang): the NEXT lfa_forward on this handle waits
 * for one pooled landmark more than any unit has (a flag value that nothing sets), and every wait of
 * that call for a flag that other thread blocks set is bounded by budget_cycles SM clock cycles
 * instead of about one second. Those waits run out, the call sets the timeout bit of the status
 * word and still completes (its outputs are invalid); lfa_get_info then returns LFA_ERR_TIMEOUT and
 * re-arms the flags, so the forward after it is a normal one. Waits on the thread block's own
 * tensor-core and TMA operations keep their usual bound. Fused path only (LFA_ERR_UNSUPPORTED on the
 * per-stage path, which has no cross-block waits); LFA_ERR_INVALID_ARG for a negative budget. */
lfa_status lfa_debug_spin_test(lfa_handle h, long long budget_cycles);

/* Arm a one-shot copy of the cross kernel C of `unit` as the NEXT lfa_forward on this handle
 * computes it, written as fp32 [N][m] to the device buffer C_out (at least N*m floats, owned by the
 * caller, untouched until that forward runs). On the fused path the forward keeps bf16(C - c) on chip
 * and multiplies it in pass 2, with c a per-column shift that each thread block takes from the mean
 * of C over the first 16 tokens of its rows of the unit (the bias of pass 2 adds c back exactly); C
 * is computed by ex2.approx from the fp32 distance sum. The copy is that bf16 value widened to fp32
 * plus c, and shift_out (NULL, or a device buffer of N*m floats) receives c for every entry. On the
 * per-stage path with bf16 tokens and d = 64, pass 2 multiplies bf16(C - mu) on the tensor cores (mu the
 * column mean, C again by ex2.approx from the fp32 distance sum) and copies that value widened plus mu,
 * with mu in shift_out. On the other per-stage shapes (fp32 tokens, d != 64) the forward's CUDA-core tile
 * code computes C again for the copy, in fp32, and shift_out is zeroed. Host-only; LFA_ERR_INVALID_ARG
 * for a bad unit or a NULL C_out. */
lfa_status lfa_debug_capture_cross(lfa_handle h, int unit, float* C_out, float* shift_out);

/* Copy the forward context of one unit (device -> device, fp32): landmarks L [m][d],
 * Newton-Schulz result X [m][m], whitening mean mu [m] and scale s [m]. Any output
 * pointer may be NULL. Valid after lfa_forward on this handle. */
lfa_status lfa_debug_context(lfa_handle h, int unit, float* L_out, float* X_out, float* mu_out,
                             float* s_out, void* stream);

/* Self-test of the tensor-core and TMA building blocks of the fused forward pass (no
 * handle needed). modes 0, 1, 3, 5, 7 run one tcgen05 product on fp32 inputs A, B (device, row-major;
 * shapes documented beside each mode in the library source) and write the fp32 result to D
 * (device, [128][64]); mode 4 loads 128 rows of the bf16 [tma_rows][64] device tensor
 * tma_src starting at row `param` through TMA and writes them to D as fp32 (rows outside
 * the tensor read as zero). status: device int, set non-zero if a bounded wait expired. */
lfa_status lfa_debug_selftest(int mode, const float* A, const float* B, float* D, int param,
                              const void* tma_src, int tma_rows, int* status, void* stream);

/* Benchmark timing hook: with non-NULL ev_begin / ev_end (each a cudaEvent_t created by
 * the caller), every later lfa_forward on this handle records ev_begin on its stream
 * immediately before launching the forward's dominant kernel and ev_end immediately after
 * it, so the caller can time that one kernel with cudaEventElapsedTime. NULL, NULL turns
 * the hook off. Host-only; returns LFA_ERR_INVALID_ARG if exactly one event is NULL. */
lfa_status lfa_set_profile_events(lfa_handle h, void* ev_begin, void* ev_end);

/* Diagnostic timeline of the fused kernel, present only in a library built with
 * -DLFA_PHASE_TRACE (python -m laplacian_nystr_attention_avg_b200.build --phase-trace); the
 * default build returns LFA_ERR_UNSUPPORTED and its kernels carry no stamp code. With a non-NULL
 * device buffer of grid * 32 uint64 entries, later forwards on this handle record %globaltimer
 * (ns) stamps at phase boundaries of every CTA (slot 0 start, 1 landmarks pooled, then per role;
 * 15 end; 13 / 14 the SM clock64 at start / end). NULL turns it off. Host-only. */
lfa_status lfa_debug_trace(lfa_handle h, unsigned long long* dev_buf);

/* Name of the kernel the timing hook brackets for this handle's config (static string). */
const char* lfa_dominant_kernel(lfa_handle h);

/* CTAs of the fused kernel for this handle (0 when the generic path serves it). */
int lfa_fused_grid(lfa_handle h);

/* Number of kernels one lfa_forward launches for this handle's config (0 if h is NULL). */
int lfa_launches_per_forward(lfa_handle h);

/* Name of the forward implementation chosen for this handle's config, static string:
 * "fused" (one cooperative kernel: bf16, d = 64, m <= 56, W % 4 == 0, B*heads <= SMs/2, rows
 * per CTA within its on-chip C capacity) or "generic" (every other accepted shape). Setting the
 * environment variable LFA_FORWARD_PATH=generic before lfa_create forces the generic path. */
const char* lfa_forward_path(lfa_handle h);

#ifdef __cplusplus
}
#endif

#endif /* LFA_H_ */
