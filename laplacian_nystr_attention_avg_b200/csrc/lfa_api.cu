// C-ABI entry points of liblfa (declared in include/lfa.h): validation, workspace
// carve-up, launch sequencing and diagnostics read-back. No compute happens here.
#include <math.h>
#include <stdlib.h>
#include <string.h>

#include <mutex>
#include <new>
#include <vector>

#include "lfa_internal.h"

using lfa::Layout;
using lfa::Params;

struct lfa_ctx {
  lfa_config cfg;
  Params p;
  Layout lay;
  unsigned char* ws;
  size_t ws_bytes;
  const void* last_Q;
  const void* last_V;
  int have_forward;
  int path;   // 0 = generic, 1 = fused
  int grid;   // CTAs of the fused kernel
  unsigned long long epoch;   // forward calls issued (the fused kernel's flag generation)
  float* cap_C;   // armed by lfa_debug_capture_cross: the next forward copies C of cap_unit here
  float* cap_S;   // and, if set, the column shift of each entry
  int cap_unit;
  int sp;   // sequence-split handle (lfa_sp_create): per-stage kernels over a band of grid rows
  long long spin_test_budget;   // armed by lfa_debug_spin_test (>= 0): the next forward's flag waits
};

namespace {

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

bool aligned16(const void* ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 15u) == 0; }

lfa_status validate(const lfa_config* c) {
  if (!c) return LFA_ERR_INVALID_ARG;
  if (c->B < 1 || c->heads < 1 || c->H < 1 || c->W < 1 || c->r < 1) return LFA_ERR_INVALID_ARG;
  if (c->H % c->r != 0 || c->W % c->r != 0) return LFA_ERR_INVALID_ARG;
  if (!(c->lambda > 0.f) || !isfinite(c->lambda)) return LFA_ERR_INVALID_ARG;
  if (!(c->eps >= 0.f) || !isfinite(c->eps)) return LFA_ERR_INVALID_ARG;
  if (c->T < 0 || c->T > lfa::kMaxT) return LFA_ERR_INVALID_ARG;
  if (c->whiten < 0 || c->whiten > 3) return LFA_ERR_INVALID_ARG;
  if (c->d != 32 && c->d != 64) return LFA_ERR_UNSUPPORTED;
  if (c->dtype != LFA_F32 && c->dtype != LFA_BF16) return LFA_ERR_UNSUPPORTED;
  const long long m = (long long)(c->H / c->r) * (c->W / c->r);
  if (m > lfa::kMaxM) return LFA_ERR_UNSUPPORTED;
  const long long rows = (long long)c->B * c->heads * c->H * c->W;
  if (rows * c->d >= (1ll << 31)) return LFA_ERR_UNSUPPORTED;   // element index fits int32
  return LFA_OK;
}

// Shape-derived parameters and workspace offsets (no pointers yet).
void plan(const lfa_config* c, Params* p, Layout* L) {
  memset(p, 0, sizeof(*p));
  p->B = c->B;
  p->heads = c->heads;
  p->H = c->H;
  p->W = c->W;
  p->N = c->H * c->W;
  p->d = c->d;
  p->r = c->r;
  p->m = (c->H / c->r) * (c->W / c->r);
  p->T = c->T;
  p->whiten = c->whiten;
  p->dtype = c->dtype;
  p->U = c->B * c->heads;
  p->lam = c->lambda;
  p->eps = c->eps;
  p->neg_log2e_over_lam = (float)(-1.4426950408889634 / (double)c->lambda);
  p->spin_budget = lfa::kFlagSpinBudget;
  p->y0 = 0;
  p->Hg = c->H;
  p->Ng = c->H * c->W;
  p->Vh = nullptr;
  p->n_tiles = lfa::ceil_div(p->N, lfa::kRowTile);
  // about two pass-1 CTAs per SM of a 148-SM part
  const int want = lfa::ceil_div(296, p->U);
  int P = want < p->n_tiles ? want : p->n_tiles;
  if (P < 1) P = 1;
  p->tiles_per_cta = lfa::ceil_div(p->n_tiles, P);
  p->P = lfa::ceil_div(p->n_tiles, p->tiles_per_cta);
  // pass-1 partial record: S1 [m], S2 [m], C^T V [m][d], sum V [d]; Reading B adds C^T C [m][m]
  p->part_stride = 2 * p->m + p->m * p->d + p->d + (c->whiten == 3 ? p->m * p->m : 0);
  p->n_chunks = lfa::ceil_div(p->m, 16);

  const size_t U = p->U, m = p->m, d = p->d;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    size_t o = off;
    off = align256(off + bytes);
    return o;
  };
  L->status = take(64);
  L->info = take(sizeof(float) * U * lfa::kInfoStride);
  L->L = take(sizeof(float) * U * m * d);
  L->Wm = take(sizeof(float) * U * m * m);
  L->X = take(sizeof(float) * U * m * m);
  L->Xb = take(sizeof(float) * U * m * m);
  L->Y = take(sizeof(float) * U * m * m);
  L->part = take(sizeof(float) * U * p->P * p->part_stride);
  L->red = take(sizeof(double) * U * p->part_stride);
  L->mu = take(sizeof(float) * U * m);
  L->s = take(sizeof(float) * U * m);
  L->A = take(sizeof(float) * U * m * d);
  L->M = take(sizeof(float) * U * m * d);
  L->Mp = take(sizeof(float) * U * m * d);
  L->bpart = take(sizeof(float) * U * p->n_chunks * d);
  const bool fusable = c->dtype == LFA_BF16 && c->d == 64 && p->m <= 63;
  L->fused = take(fusable ? lfa::fused_workspace_bytes(p->U) : 0);
  // backward: Newton-Schulz iterates and reverse-step matrices, partials, dQ in fp32
  const size_t mm = m * m, T = p->T > 0 ? p->T : 1;
  L->bwd = off;
  L->b_its = take(sizeof(float) * U * T * mm);
  L->b_G = take(sizeof(float) * U * mm);
  L->b_Gn = take(sizeof(float) * U * mm);
  L->b_T1 = take(sizeof(float) * U * mm);
  L->b_T2 = take(sizeof(float) * U * mm);
  L->b_T3 = take(sizeof(float) * U * mm);
  L->b_dW = take(sizeof(float) * U * mm);
  L->b_part2 = take(sizeof(float) * U * p->P * p->part_stride);
  L->b_red2 = take(sizeof(double) * U * p->part_stride);
  L->b_dA = take(sizeof(float) * U * m * d);
  L->b_Gm = take(sizeof(float) * U * m * d);
  L->b_Gd = take(sizeof(float) * U * m * d);
  L->b_beta = take(sizeof(float) * U * m);
  L->b_gamma = take(sizeof(float) * U * m);
  L->b_bpart2 = take(sizeof(float) * U * p->n_chunks * d);
  L->b_dLpart = take(sizeof(float) * U * p->P * m * d);
  L->b_dLns = take(sizeof(float) * U * m * d);
  L->b_dLpool = take(sizeof(float) * U * m * d);
  L->b_dQd = take(sizeof(float) * U * (size_t)p->N * d);
  L->total = off;
}

void bind(Params* p, const Layout& L, unsigned char* ws) {
  p->status = reinterpret_cast<int*>(ws + L.status);
  p->info = reinterpret_cast<float*>(ws + L.info);
  p->L = reinterpret_cast<float*>(ws + L.L);
  p->Wm = reinterpret_cast<float*>(ws + L.Wm);
  p->X = reinterpret_cast<float*>(ws + L.X);
  p->Xb = reinterpret_cast<float*>(ws + L.Xb);
  p->Y = reinterpret_cast<float*>(ws + L.Y);
  p->part = reinterpret_cast<float*>(ws + L.part);
  p->red = reinterpret_cast<double*>(ws + L.red);
  p->mu = reinterpret_cast<float*>(ws + L.mu);
  p->s = reinterpret_cast<float*>(ws + L.s);
  p->A = reinterpret_cast<float*>(ws + L.A);
  p->M = reinterpret_cast<float*>(ws + L.M);
  p->Mp = reinterpret_cast<float*>(ws + L.Mp);
  p->bpart = reinterpret_cast<float*>(ws + L.bpart);
}

void bind_backward(lfa::BwdParams* b, const Params& p, const Layout& L, unsigned char* ws) {
  memset(b, 0, sizeof(*b));
  b->p = p;
  auto f = [&](size_t off) { return reinterpret_cast<float*>(ws + off); };
  b->its = f(L.b_its);
  b->G = f(L.b_G);
  b->Gn = f(L.b_Gn);
  b->T1 = f(L.b_T1);
  b->T2 = f(L.b_T2);
  b->T3 = f(L.b_T3);
  b->dW = f(L.b_dW);
  b->part2 = f(L.b_part2);
  b->red2 = reinterpret_cast<double*>(ws + L.b_red2);
  b->dA = f(L.b_dA);
  b->Gm = f(L.b_Gm);
  b->Gd = f(L.b_Gd);
  b->beta = f(L.b_beta);
  b->gamma = f(L.b_gamma);
  b->bpart2 = f(L.b_bpart2);
  b->dLpart = f(L.b_dLpart);
  b->dLns = f(L.b_dLns);
  b->dLpool = f(L.b_dLpool);
  b->dQd = f(L.b_dQd);
}

// Fused forwards on one device run one at a time, in the order they were enqueued, whatever their
// stream: each waits for the previous one's completion event and records its own. (Its thread blocks wait
// on flags of the same launch, so a launch should not share the SMs with another one; host-buffer calls
// on two streams still overlap their copies with each other's forwards.)
std::mutex g_fused_mu;
cudaEvent_t g_fused_ev[64] = {};

cudaError_t launch_fused_in_order(const Params& p, int grid, unsigned char* ws, unsigned long long epoch,
                                  cudaStream_t st) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev >= 64) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lk(g_fused_mu);
  if (!g_fused_ev[dev]) {
    const cudaError_t e = cudaEventCreateWithFlags(&g_fused_ev[dev], cudaEventDisableTiming);
    if (e != cudaSuccess) return e;
  } else if (cudaStreamWaitEvent(st, g_fused_ev[dev], 0) != cudaSuccess) {
    // an event of an earlier context (the device was reset since): start the order afresh
    cudaGetLastError();
    const cudaError_t e = cudaEventCreateWithFlags(&g_fused_ev[dev], cudaEventDisableTiming);
    if (e != cudaSuccess) return e;
  }
  const cudaError_t e = lfa::launch_fused_forward(p, grid, ws, epoch, st);
  if (e != cudaSuccess) return e;
  return cudaEventRecord(g_fused_ev[dev], st);
}

// Kernel attributes (dynamic shared memory opt-in) are per device; set them once each.
std::mutex g_attr_mu;
unsigned long long g_attr_done = 0;

lfa_status ensure_attributes() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return LFA_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_attr_mu);
  if (dev < 64 && (g_attr_done >> dev) & 1ull) return LFA_OK;
  if (lfa::generic_set_attributes() != cudaSuccess) return LFA_ERR_CUDA;
  if (lfa::backward_set_attributes() != cudaSuccess) return LFA_ERR_CUDA;
  if (lfa::gemm_set_attributes() != cudaSuccess) return LFA_ERR_CUDA;
  if (lfa::ns_tc_set_attributes() != cudaSuccess) return LFA_ERR_CUDA;
  if (lfa::cg_set_attributes() != cudaSuccess) return LFA_ERR_CUDA;
  if (lfa::stream_set_attributes() != cudaSuccess) return LFA_ERR_CUDA;
  if (dev < 64) g_attr_done |= 1ull << dev;
  return LFA_OK;
}

size_t elem_bytes(const lfa_config& c) { return c.dtype == LFA_BF16 ? 2 : 4; }

}  // namespace

extern "C" {

const char* lfa_status_string(lfa_status s) {
  switch (s) {
    case LFA_OK: return "ok";
    case LFA_ERR_INVALID_ARG: return "invalid argument";
    case LFA_ERR_UNSUPPORTED: return "unsupported configuration";
    case LFA_ERR_CUDA: return "CUDA runtime error";
    case LFA_ERR_STATE: return "backward without a matching forward";
    case LFA_ERR_TIMEOUT: return "device wait timed out";
    case LFA_ERR_NONFINITE: return "non-finite landmark kernel";
    case LFA_ERR_SCRATCH_LIMIT: return "configuration needs more scratch than the static no-alloc area holds";
  }
  return "unknown status";
}

size_t lfa_workspace_size(const lfa_config* cfg) {
  if (validate(cfg) != LFA_OK) return 0;
  Params p;
  Layout L;
  plan(cfg, &p, &L);
  return L.total;
}

// the handle's auxiliary stream and fork / join events (the per-stage kernels overlap the Newton-Schulz
// chain with pass 1 on it); released by lfa_destroy
void free_aux(lfa_ctx* h) {
  if (h->p.ev_fork) cudaEventDestroy(static_cast<cudaEvent_t>(h->p.ev_fork));
  if (h->p.ev_mid) cudaEventDestroy(static_cast<cudaEvent_t>(h->p.ev_mid));
  if (h->p.ev_x) cudaEventDestroy(static_cast<cudaEvent_t>(h->p.ev_x));
  if (h->p.ev_join) cudaEventDestroy(static_cast<cudaEvent_t>(h->p.ev_join));
  if (h->p.aux_stream) cudaStreamDestroy(static_cast<cudaStream_t>(h->p.aux_stream));
  h->p.ev_fork = h->p.ev_mid = h->p.ev_x = h->p.ev_join = h->p.aux_stream = nullptr;
}
bool make_aux(lfa_ctx* h) {
  cudaStream_t s = nullptr;
  cudaEvent_t a = nullptr, b = nullptr, c = nullptr, x = nullptr;
  const bool ok = cudaStreamCreateWithFlags(&s, cudaStreamNonBlocking) == cudaSuccess &&
                  cudaEventCreateWithFlags(&a, cudaEventDisableTiming) == cudaSuccess &&
                  cudaEventCreateWithFlags(&b, cudaEventDisableTiming) == cudaSuccess &&
                  cudaEventCreateWithFlags(&c, cudaEventDisableTiming) == cudaSuccess &&
                  cudaEventCreateWithFlags(&x, cudaEventDisableTiming) == cudaSuccess;
  h->p.aux_stream = s;
  h->p.ev_fork = a;
  h->p.ev_join = b;
  h->p.ev_mid = c;
  h->p.ev_x = x;
  if (!ok) {
    free_aux(h);
    cudaGetLastError();
  }
  return ok;
}

lfa_status lfa_create(const lfa_config* cfg, const float* dwc_weight, void* workspace,
                      size_t workspace_bytes, lfa_handle* out) {
  if (!out) return LFA_ERR_INVALID_ARG;
  *out = nullptr;
  lfa_status st = validate(cfg);
  if (st != LFA_OK) return st;
  if (!dwc_weight || !workspace) return LFA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0 || !aligned16(dwc_weight))
    return LFA_ERR_INVALID_ARG;
  lfa_ctx* h = new (std::nothrow) lfa_ctx;
  if (!h) return LFA_ERR_INVALID_ARG;
  memset(h, 0, sizeof(*h));
  h->cfg = *cfg;
  plan(cfg, &h->p, &h->lay);
  if (workspace_bytes < h->lay.total) {
    delete h;
    return LFA_ERR_INVALID_ARG;
  }
  st = ensure_attributes();
  if (st != LFA_OK) {
    delete h;
    return st;
  }
  h->ws = static_cast<unsigned char*>(workspace);
  h->ws_bytes = workspace_bytes;
  h->spin_test_budget = -1;
  bind(&h->p, h->lay, h->ws);
  h->p.dwc = dwc_weight;
  if (!make_aux(h)) {
    delete h;
    return LFA_ERR_CUDA;
  }
  h->path = 0;
  const char* force = getenv("LFA_FORWARD_PATH");
  const bool want_generic = force && strcmp(force, "generic") == 0;
  // batch-pooled statistics need every unit's column sums before any unit's combine, and
  // Reading B needs two more token passes: both run on the per-stage kernels
  if (!want_generic && h->p.whiten <= 1 && h->lay.fused != h->lay.bwd) {
    h->grid = lfa::fused_grid(h->p);
    if (h->grid > 0) h->path = 1;
  }
  cudaGetLastError();   // an ineligible probe must not leave a sticky error behind
  *out = h;
  return LFA_OK;
}

lfa_status lfa_destroy(lfa_handle h) {
  if (!h) return LFA_ERR_INVALID_ARG;
  free_aux(h);
  delete h;
  return LFA_OK;
}

lfa_status lfa_forward(lfa_handle h, const void* Q, const void* V, void* O, void* stream) {
  if (!h || !Q || !V || !O || h->sp) return LFA_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(V) || !aligned16(O)) return LFA_ERR_INVALID_ARG;
  Params p = h->p;
  p.Q = Q;
  p.V = V;
  p.O = O;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  float* cap = h->cap_C;
  float* cap_s = h->cap_S;
  h->cap_C = nullptr;   // one-shot
  h->cap_S = nullptr;
  if (h->path == 1) {
    const unsigned long long epoch = h->epoch + 1;
    p.dbgC = cap;
    p.dbgS = cap ? cap_s : nullptr;
    p.dbg_unit = h->cap_unit;
    if (h->spin_test_budget >= 0) {
      p.spin_test = 1;
      p.spin_budget = h->spin_test_budget;
      h->spin_test_budget = -1;   // one-shot
    }
    if (launch_fused_in_order(p, h->grid, h->ws + h->lay.fused, epoch, st) != cudaSuccess) return LFA_ERR_CUDA;
    h->epoch = epoch;
  } else {
    // the tcgen05 pass 2 copies the C it multiplies (bf16(C - mu) widened, mu added back) as it goes;
    // the CUDA-core passes keep C in registers: their tile code runs once more for the copy
    const bool in_pass = cap && lfa::stream_eligible(p);
    if (in_pass) {
      p.dbgC = cap;
      p.dbgS = cap_s;
      p.dbg_unit = h->cap_unit;
    }
    if (lfa::launch_generic_forward(p, st) != cudaSuccess) return LFA_ERR_CUDA;
    if (cap && !in_pass && lfa::launch_cross_kernel(p, h->cap_unit, cap, st) != cudaSuccess) return LFA_ERR_CUDA;
    if (cap && !in_pass && cap_s &&
        cudaMemsetAsync(cap_s, 0, sizeof(float) * (size_t)h->p.N * h->p.m, st) != cudaSuccess)
      return LFA_ERR_CUDA;
  }
  h->last_Q = Q;
  h->last_V = V;
  h->have_forward = 1;
  return LFA_OK;
}

}  // extern "C"

// Static scratch of lfa_forward_noalloc: one array per device, placed by module load.
static __device__ __align__(256) unsigned char g_noalloc_scratch[LFA_NOALLOC_SCRATCH_BYTES];

namespace {

// Address of the scratch array on the current device. Resolved at every call (a host-side query):
// a cached address would go stale if the device's context were torn down and re-created, since the
// module, and with it the array, is then loaded again at a new address.
lfa_status noalloc_scratch(unsigned char** out) {
  void* ptr = nullptr;
  if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || !ptr) return LFA_ERR_CUDA;
  *out = static_cast<unsigned char*>(ptr);
  return LFA_OK;
}

}  // namespace

extern "C" {

lfa_status lfa_forward_noalloc(const lfa_config* cfg, const float* dwc_weight, const void* Q,
                               const void* V, void* O, void* stream) {
  lfa_status st = validate(cfg);
  if (st != LFA_OK) return st;
  if (!dwc_weight || !Q || !V || !O) return LFA_ERR_INVALID_ARG;
  if (!aligned16(dwc_weight) || !aligned16(Q) || !aligned16(V) || !aligned16(O)) return LFA_ERR_INVALID_ARG;
  Params p;
  Layout lay;
  plan(cfg, &p, &lay);
  // the per-stage kernels use the layout up to the fused kernel's area
  if (lay.fused > (size_t)LFA_NOALLOC_SCRATCH_BYTES) return LFA_ERR_SCRATCH_LIMIT;
  st = ensure_attributes();
  if (st != LFA_OK) return st;
  unsigned char* ws = nullptr;
  st = noalloc_scratch(&ws);
  if (st != LFA_OK) return st;
  bind(&p, lay, ws);
  p.dwc = dwc_weight;
  p.Q = Q;
  p.V = V;
  p.O = O;
  return lfa::launch_generic_forward(p, static_cast<cudaStream_t>(stream)) == cudaSuccess ? LFA_OK
                                                                                           : LFA_ERR_CUDA;
}

lfa_status lfa_forward_host_async(lfa_handle h, const void* Q_host, const void* V_host, void* O_host,
                                  void* Q_dev, void* V_dev, void* O_dev, void* stream) {
  if (!h || !Q_host || !V_host || !O_host || !Q_dev || !V_dev || !O_dev) return LFA_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const size_t bytes = (size_t)h->p.U * h->p.N * h->p.d * elem_bytes(h->cfg);
  if (cudaMemcpyAsync(Q_dev, Q_host, bytes, cudaMemcpyHostToDevice, st) != cudaSuccess) return LFA_ERR_CUDA;
  if (cudaMemcpyAsync(V_dev, V_host, bytes, cudaMemcpyHostToDevice, st) != cudaSuccess) return LFA_ERR_CUDA;
  lfa_status s = lfa_forward(h, Q_dev, V_dev, O_dev, stream);
  if (s != LFA_OK) return s;
  if (cudaMemcpyAsync(O_host, O_dev, bytes, cudaMemcpyDeviceToHost, st) != cudaSuccess) return LFA_ERR_CUDA;
  return LFA_OK;
}

lfa_status lfa_forward_host(lfa_handle h, const void* Q_host, const void* V_host, void* O_host,
                            void* Q_dev, void* V_dev, void* O_dev, void* stream) {
  const lfa_status s = lfa_forward_host_async(h, Q_host, V_host, O_host, Q_dev, V_dev, O_dev, stream);
  if (s != LFA_OK) return s;
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return LFA_ERR_CUDA;
  return LFA_OK;
}

lfa_status lfa_backward(lfa_handle h, const void* Q, const void* V, const void* dO, void* dQ,
                        void* dV, void* stream) {
  if (!h || !Q || !V || !dO || !dQ || !dV || h->sp) return LFA_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(V) || !aligned16(dO) || !aligned16(dQ) || !aligned16(dV))
    return LFA_ERR_INVALID_ARG;
  if (h->p.whiten == 3) return LFA_ERR_UNSUPPORTED;   // Reading B: forward only
  if (!h->have_forward || h->last_Q != Q || h->last_V != V) return LFA_ERR_STATE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  Params p = h->p;
  p.Q = Q;
  p.V = V;
  p.O = nullptr;
  p.ev_begin = nullptr;
  p.ev_end = nullptr;
  p.trace = nullptr;
  // the fused forward keeps its intermediates on chip: rebuild the per-stage context
  if (h->path == 1 && lfa::launch_generic_context(p, st) != cudaSuccess) return LFA_ERR_CUDA;
  lfa::BwdParams b;
  bind_backward(&b, p, h->lay, h->ws);
  b.dO = dO;
  b.dQ = dQ;
  b.dV = dV;
  return lfa::launch_backward(b, st) == cudaSuccess ? LFA_OK : LFA_ERR_CUDA;
}

lfa_status lfa_get_info(lfa_handle h, lfa_unit_info* host_out, int n_units, void* stream) {
  if (!h || !host_out || n_units != h->p.U) return LFA_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const size_t n = (size_t)h->p.U * lfa::kInfoStride;
  float* tmp = static_cast<float*>(malloc(n * sizeof(float)));
  if (!tmp) return LFA_ERR_INVALID_ARG;
  int status = 0;
  lfa_status ret = LFA_OK;
  // the condition-number estimate is computed here, outside the forward
  if (h->have_forward && lfa::launch_kappa(h->p, st) != cudaSuccess) {
    free(tmp);
    return LFA_ERR_CUDA;
  }
  if (cudaMemcpyAsync(tmp, h->p.info, n * sizeof(float), cudaMemcpyDeviceToHost, st) != cudaSuccess ||
      cudaMemcpyAsync(&status, h->p.status, sizeof(int), cudaMemcpyDeviceToHost, st) != cudaSuccess ||
      cudaStreamSynchronize(st) != cudaSuccess) {
    ret = LFA_ERR_CUDA;
  } else {
    for (int u = 0; u < h->p.U; ++u) {
      const float* f = tmp + (size_t)u * lfa::kInfoStride;
      host_out[u].alpha = f[lfa::kInfoAlpha];
      host_out[u].lambda_max = f[lfa::kInfoLambdaMax];
      host_out[u].alpha_fallback = f[lfa::kInfoFallback] != 0.f;
      host_out[u].ns_residual_fro = f[lfa::kInfoResidual];
      host_out[u].kappa = h->have_forward ? f[lfa::kInfoKappa] : 0.f;
    }
    if (status & lfa::kStatusTimeout) {
      ret = LFA_ERR_TIMEOUT;
      h->epoch = 0;   // flags may be inconsistent: the next fused forward re-zeroes them
    }
    else if (status & lfa::kStatusNonFinite) ret = LFA_ERR_NONFINITE;
  }
  free(tmp);
  return ret;
}

lfa_status lfa_debug_cross_kernel(lfa_handle h, const void* Q, int unit, float* C_out, void* stream) {
  if (!h || !Q || !C_out || unit < 0 || unit >= h->p.U || !aligned16(Q)) return LFA_ERR_INVALID_ARG;
  Params p = h->p;
  p.Q = Q;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // the landmarks are pooled into the handle's workspace, replacing the forward context there
  h->have_forward = 0;
  if (lfa::launch_pool(p, st) != cudaSuccess) return LFA_ERR_CUDA;
  if (lfa::launch_cross_kernel(p, unit, C_out, st) != cudaSuccess) return LFA_ERR_CUDA;
  return LFA_OK;
}

// ---- solvers for W Y = B outside the forward pass -------------------------------------------

namespace {
// Newton-Schulz scratch: X_b and Y (U m^2 fp32 each), the per-unit info and the status word
struct SolverLayout {
  size_t xb, y, info, status, total;
};
SolverLayout solver_layout(int U, int m) {
  SolverLayout l;
  const size_t mm = (size_t)U * m * m * sizeof(float);
  l.xb = 0;
  l.y = align256(mm);
  l.info = l.y + align256(mm);
  l.status = l.info + align256((size_t)U * lfa::kInfoStride * sizeof(float));
  l.total = l.status + 256;
  return l;
}
bool solver_sizes_ok(int U, int m) { return U >= 1 && m >= 1 && m <= lfa::kMaxM && (size_t)U * m * m < (1ull << 31); }
}  // namespace

size_t lfa_solver_workspace_size(int U, int m) {
  if (!solver_sizes_ok(U, m)) return 0;
  return solver_layout(U, m).total;
}

lfa_status lfa_ns_solve(const float* W, float* X, int U, int m, int T, void* workspace, size_t workspace_bytes,
                        lfa_unit_info* host_out, void* stream) {
  if (!W || !X || !workspace || !solver_sizes_ok(U, m) || T < 0 || T > 64) return LFA_ERR_INVALID_ARG;
  if (!aligned16(W) || !aligned16(X) || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return LFA_ERR_INVALID_ARG;
  const SolverLayout l = solver_layout(U, m);
  if (workspace_bytes < l.total) return LFA_ERR_INVALID_ARG;
  const lfa_status st_attr = ensure_attributes();
  if (st_attr != LFA_OK) return st_attr;
  unsigned char* ws = static_cast<unsigned char*>(workspace);
  lfa::Params p;
  memset(&p, 0, sizeof(p));
  p.U = U;
  p.m = m;
  p.T = T;
  p.Wm = const_cast<float*>(W);   // read only on this path
  p.X = X;
  p.Xb = reinterpret_cast<float*>(ws + l.xb);
  p.Y = reinterpret_cast<float*>(ws + l.y);
  p.info = reinterpret_cast<float*>(ws + l.info);
  p.status = reinterpret_cast<int*>(ws + l.status);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(p.status, 0, sizeof(int), st) != cudaSuccess) return LFA_ERR_CUDA;
  if (lfa::launch_ns_from_w(p, st) != cudaSuccess) return LFA_ERR_CUDA;
  if (!host_out) return LFA_OK;
  std::vector<float> tmp((size_t)U * lfa::kInfoStride);
  int status = 0;
  if (cudaMemcpyAsync(tmp.data(), p.info, tmp.size() * sizeof(float), cudaMemcpyDeviceToHost, st) != cudaSuccess ||
      cudaMemcpyAsync(&status, p.status, sizeof(int), cudaMemcpyDeviceToHost, st) != cudaSuccess ||
      cudaStreamSynchronize(st) != cudaSuccess)
    return LFA_ERR_CUDA;
  for (int u = 0; u < U; ++u) {
    const float* f = tmp.data() + (size_t)u * lfa::kInfoStride;
    host_out[u].alpha = f[lfa::kInfoAlpha];
    host_out[u].lambda_max = f[lfa::kInfoLambdaMax];
    host_out[u].alpha_fallback = f[lfa::kInfoFallback] != 0.f;
    host_out[u].ns_residual_fro = f[lfa::kInfoResidual];
    host_out[u].kappa = 0.f;
  }
  return (status & lfa::kStatusNonFinite) ? LFA_ERR_NONFINITE : LFA_OK;
}

lfa_status lfa_cg_solve(const float* W, const float* B, float* Y, int U, int m, int nrhs, int iters, void* stream) {
  if (!W || !B || !Y || !solver_sizes_ok(U, m) || nrhs < 1 || nrhs > 4096 || iters < 0 || iters > 4096)
    return LFA_ERR_INVALID_ARG;
  if (!aligned16(W) || !aligned16(B) || !aligned16(Y)) return LFA_ERR_INVALID_ARG;
  if ((size_t)U * m * nrhs >= (1ull << 31)) return LFA_ERR_INVALID_ARG;
  const lfa_status st_attr = ensure_attributes();
  if (st_attr != LFA_OK) return st_attr;
  if (lfa::launch_cg(W, B, Y, U, m, nrhs, iters, static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return LFA_ERR_CUDA;
  return LFA_OK;
}

lfa_status lfa_debug_spin_test(lfa_handle h, long long budget_cycles) {
  if (!h || budget_cycles < 0) return LFA_ERR_INVALID_ARG;
  if (h->path != 1) return LFA_ERR_UNSUPPORTED;
  h->spin_test_budget = budget_cycles;
  return LFA_OK;
}

lfa_status lfa_debug_capture_cross(lfa_handle h, int unit, float* C_out, float* shift_out) {
  if (!h || unit < 0 || unit >= h->p.U || !C_out) return LFA_ERR_INVALID_ARG;
  h->cap_C = C_out;
  h->cap_S = shift_out;
  h->cap_unit = unit;
  return LFA_OK;
}

lfa_status lfa_debug_context(lfa_handle h, int unit, float* L_out, float* X_out, float* mu_out,
                             float* s_out, void* stream) {
  if (!h || unit < 0 || unit >= h->p.U) return LFA_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const size_t m = h->p.m, d = h->p.d;
  struct { float* dst; const float* src; size_t n; } cp[4] = {
      {L_out, h->p.L + unit * m * d, m * d},
      {X_out, h->p.X + unit * m * m, m * m},
      {mu_out, h->p.mu + unit * m, m},
      {s_out, h->p.s + unit * m, m}};
  for (auto& c : cp) {
    if (!c.dst) continue;
    if (cudaMemcpyAsync(c.dst, c.src, c.n * sizeof(float), cudaMemcpyDeviceToDevice, st) != cudaSuccess)
      return LFA_ERR_CUDA;
  }
  return LFA_OK;
}

lfa_status lfa_debug_selftest(int mode, const float* A, const float* B, float* D, int param,
                              const void* tma_src, int tma_rows, int* status, void* stream) {
  if (!(mode == 0 || mode == 1 || mode == 3 || mode == 4 || mode == 5 || mode == 7) || !D || !status)
    return LFA_ERR_INVALID_ARG;
  if (mode != 4 && (!A || !B)) return LFA_ERR_INVALID_ARG;
  if (mode == 3 && (param < 0 || param > 64 || param % 8 != 0)) return LFA_ERR_INVALID_ARG;
  if (mode == 4 && (!tma_src || tma_rows < 1 || !aligned16(tma_src))) return LFA_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  return lfa::launch_selftest(mode, A, B, D, param, tma_src, tma_rows, status, st) == cudaSuccess
             ? LFA_OK
             : LFA_ERR_CUDA;
}

lfa_status lfa_set_profile_events(lfa_handle h, void* ev_begin, void* ev_end) {
  if (!h || ((ev_begin == nullptr) != (ev_end == nullptr))) return LFA_ERR_INVALID_ARG;
  h->p.ev_begin = ev_begin;
  h->p.ev_end = ev_end;
  return LFA_OK;
}

lfa_status lfa_debug_trace(lfa_handle h, unsigned long long* dev_buf) {
  if (!h) return LFA_ERR_INVALID_ARG;
#ifdef LFA_PHASE_TRACE
  h->p.trace = dev_buf;
  return LFA_OK;
#else
  (void)dev_buf;
  return LFA_ERR_UNSUPPORTED;
#endif
}

const char* lfa_dominant_kernel(lfa_handle h) {
  if (!h) return "invalid";
  if (h->path == 1) return "k_fused_forward";
  return lfa::stream_eligible(h->p) ? "k_stream_pass2" : "k_pass2";
}

int lfa_fused_grid(lfa_handle h) { return h ? h->grid : 0; }

int lfa_launches_per_forward(lfa_handle h) {
  if (!h) return 0;
  return h->path == 1 ? 1 : lfa::generic_launch_count(h->p);
}

const char* lfa_forward_path(lfa_handle h) {
  if (!h) return "invalid";
  return h->path == 1 ? "fused" : "generic";
}

// ---- sequence split -------------------------------------------------------------------------

}  // extern "C"

namespace {

// The global plan (workspace sized for the whole grid, so any band fits), then the band's shape
// for the passes: grid rows [y0, y0 + ny), the pass-1 decomposition over the band's tokens.
lfa_status sp_plan(const lfa_config* c, int y0, int ny, Params* p, Layout* L) {
  lfa_status st = validate(c);
  if (st != LFA_OK) return st;
  if (c->whiten != 0 && c->whiten != 1) return LFA_ERR_UNSUPPORTED;
  if (y0 < 0 || ny < 1 || y0 + ny > c->H) return LFA_ERR_INVALID_ARG;
  plan(c, p, L);
  p->y0 = y0;
  p->H = ny;
  p->N = ny * c->W;
  p->n_tiles = lfa::ceil_div(p->N, lfa::kRowTile);
  const int want = lfa::ceil_div(296, p->U);
  int P = want < p->n_tiles ? want : p->n_tiles;
  if (P < 1) P = 1;
  p->tiles_per_cta = lfa::ceil_div(p->n_tiles, P);
  p->P = lfa::ceil_div(p->n_tiles, p->tiles_per_cta);
  return LFA_OK;
}

}  // namespace

extern "C" {

size_t lfa_sp_workspace_size(const lfa_config* cfg, int y0, int ny) {
  Params p;
  Layout L;
  if (sp_plan(cfg, y0, ny, &p, &L) != LFA_OK) return 0;
  return L.total;
}

lfa_status lfa_sp_create(const lfa_config* cfg, int y0, int ny, const float* dwc_weight, void* workspace,
                         size_t workspace_bytes, lfa_handle* out) {
  if (!out) return LFA_ERR_INVALID_ARG;
  *out = nullptr;
  Params p;
  Layout lay;
  lfa_status st = sp_plan(cfg, y0, ny, &p, &lay);
  if (st != LFA_OK) return st;
  if (!dwc_weight || !workspace || workspace_bytes < lay.total) return LFA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0 || !aligned16(dwc_weight)) return LFA_ERR_INVALID_ARG;
  st = ensure_attributes();
  if (st != LFA_OK) return st;
  lfa_ctx* h = new (std::nothrow) lfa_ctx;
  if (!h) return LFA_ERR_INVALID_ARG;
  memset(h, 0, sizeof(*h));
  h->cfg = *cfg;
  h->p = p;
  h->lay = lay;
  h->ws = static_cast<unsigned char*>(workspace);
  h->ws_bytes = workspace_bytes;
  h->spin_test_budget = -1;
  bind(&h->p, h->lay, h->ws);
  h->p.dwc = dwc_weight;
  if (!make_aux(h)) {
    delete h;
    return LFA_ERR_CUDA;
  }
  h->path = 0;
  h->sp = 1;
  *out = h;
  return LFA_OK;
}

int lfa_sp_partial_size(lfa_handle h) { return (h && h->sp) ? h->p.part_stride : 0; }

lfa_status lfa_sp_pool(lfa_handle h, const void* Q_local, float* L_partial, void* stream) {
  if (!h || !h->sp || !Q_local || !L_partial || !aligned16(Q_local) || !aligned16(L_partial))
    return LFA_ERR_INVALID_ARG;
  Params p = h->p;
  p.Q = Q_local;
  p.L = L_partial;
  return lfa::launch_pool(p, static_cast<cudaStream_t>(stream)) == cudaSuccess ? LFA_OK : LFA_ERR_CUDA;
}

lfa_status lfa_sp_pass1(lfa_handle h, const void* Q_local, const void* V_local, const float* L_full,
                        double* partial_out, void* stream) {
  if (!h || !h->sp || !Q_local || !V_local || !L_full || !partial_out) return LFA_ERR_INVALID_ARG;
  if (!aligned16(Q_local) || !aligned16(V_local) || !aligned16(L_full) || !aligned16(partial_out))
    return LFA_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  Params p = h->p;
  p.Q = Q_local;
  p.V = V_local;
  const size_t nL = (size_t)p.U * p.m * p.d;
  if (cudaMemsetAsync(p.status, 0, sizeof(int), st) != cudaSuccess) return LFA_ERR_CUDA;
  if (cudaMemcpyAsync(p.L, L_full, nL * sizeof(float), cudaMemcpyDeviceToDevice, st) != cudaSuccess)
    return LFA_ERR_CUDA;
  if (lfa::launch_generic_ns(p, st) != cudaSuccess) return LFA_ERR_CUDA;
  if (lfa::launch_generic_pass1_reduce(p, st) != cudaSuccess) return LFA_ERR_CUDA;
  if (cudaMemcpyAsync(partial_out, p.red, sizeof(double) * (size_t)p.U * p.part_stride, cudaMemcpyDeviceToDevice,
                      st) != cudaSuccess)
    return LFA_ERR_CUDA;
  h->have_forward = 0;   // the band's context is not a whole forward: no backward from it
  return LFA_OK;
}

lfa_status lfa_sp_pass2(lfa_handle h, const void* Q_local, const void* V_local, const void* V_halo,
                        const double* partial_total, void* O_local, void* stream) {
  if (!h || !h->sp || !Q_local || !V_local || !partial_total || !O_local) return LFA_ERR_INVALID_ARG;
  const bool need_halo = h->p.y0 > 0 || h->p.y0 + h->p.H < h->p.Hg;
  if (need_halo && !V_halo) return LFA_ERR_INVALID_ARG;
  if (!aligned16(Q_local) || !aligned16(V_local) || !aligned16(O_local) || !aligned16(partial_total) ||
      (V_halo && !aligned16(V_halo)))
    return LFA_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  Params p = h->p;
  p.Q = Q_local;
  p.V = V_local;
  p.O = O_local;
  p.Vh = V_halo;
  if (cudaMemcpyAsync(p.red, partial_total, sizeof(double) * (size_t)p.U * p.part_stride, cudaMemcpyDeviceToDevice,
                      st) != cudaSuccess)
    return LFA_ERR_CUDA;
  return lfa::launch_generic_finish(p, st) == cudaSuccess ? LFA_OK : LFA_ERR_CUDA;
}

}  // extern "C"
