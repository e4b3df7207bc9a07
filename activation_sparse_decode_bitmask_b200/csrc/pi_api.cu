// The C ABI: argument validation, library-owned layer and workspace objects, and the
// launches of the fused kernel for pi_predict / pi_sparse_ffn / pi_decode_stack.
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <new>

#include "pi_internal.h"
#include "pi_layout.h"

using namespace pi;

namespace {

constexpr long long kDefaultWaitNs = 1000LL * 1000 * 1000;   // 1 s: any legitimate wait is far shorter
static_assert(sizeof(FusedParams) <= 4000, "kernel parameter block too large");

int family_of(const pi_layer_desc& d) {
  if (d.w_dtype == PI_F32 && d.x_dtype == PI_F32 && d.p_dtype == PI_F32) return FAM_F32;
  if (d.w_dtype == PI_F16 && d.x_dtype == PI_F16 && d.p_dtype == PI_F16) return FAM_F16;
  if (d.w_dtype == PI_Q4_0 && d.x_dtype == PI_F16 && d.p_dtype == PI_F16) return FAM_Q4;
  return -1;
}
int wbytes(int fam) { return fam == FAM_F32 ? 4 : 2; }   // fp element size (weights / predictor)
int x_elem(const pi_layer_desc& d) { return d.x_dtype == PI_F32 ? 4 : 2; }
int round16(long long v) { return (int)((v + 15) / 16 * 16); }

int sm_count(int dev) {
  int n = 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  return n;
}
int smem_optin(int dev) {
  int n = 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess) return 0;
  return n;
}

pi_status check_desc(const pi_layer_desc& d) {
  if (d.act != PI_RELU && d.act != PI_REGLU && d.act != PI_RELU2) return PI_ERR_ARG;
  if ((unsigned)d.w_dtype > PI_Q4_0 || (unsigned)d.x_dtype > PI_Q4_0 || (unsigned)d.p_dtype > PI_Q4_0) return PI_ERR_ARG;
  if (d.d_model <= 0 || d.d_ff < 32 || d.rank <= 0) return PI_ERR_ARG;
  if (d.d_ff % 32 || d.d_model % 64 || d.rank % 8 || d.rank > d.d_model) return PI_ERR_ARG;
  const int fam = family_of(d);
  if (fam < 0) return PI_ERR_UNSUPPORTED;
  if (fam == FAM_Q4 && d.d_model % 256) return PI_ERR_ARG;
  return PI_OK;
}

pi_status cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return PI_OK;
  if (e == cudaErrorMemoryAllocation) { cudaGetLastError(); return PI_ERR_OOM; }
  cudaGetLastError();
  return PI_ERR_CUDA;
}

#define PI_TRY(expr)                              \
  do {                                            \
    pi_status _s = cuda_status(expr);             \
    if (_s != PI_OK) return _s;                   \
  } while (0)

template <typename T>
cudaError_t dmalloc(T** p, size_t bytes) {
  return cudaMalloc(reinterpret_cast<void**>(p), bytes ? bytes : 16);
}

void free_layer_buffers(pi_layer* L) {
  cudaFree(L->rec); cudaFree(L->p1t); cudaFree(L->p2o); cudaFree(L->bias);
  cudaFree(L->thresh); cudaFree(L->perm); cudaFree(L->freq_sorted);
  delete[] L->freq_host;
  L->freq_host = nullptr;
}

// Bytes of bulk copies each block of the fused kernel keeps in flight: enough to keep its
// share of HBM busy (about the SM's share of bandwidth times the unloaded latency), and no
// more, since every byte beyond that only lengthens the queue the exchange words wait in.
// PI_FUSED_INFLIGHT_KB in the environment (read once) overrides the default of 128 KB.
int inflight_budget_bytes() {
  static const int v = [] {
    const char* e = std::getenv("PI_FUSED_INFLIGHT_KB");
    const int kb = e ? std::atoi(e) : 0;
    return (kb > 0 && kb <= 4096 ? kb : 128) * 1024;
  }();
  return v;
}

// Geometry of the fused kernel for one layer shape.
// r_max: the largest predictor rank of the launch's layers (the layer's own when <= 0).
pi_status plan_fused(const pi_layer* L, int B, const pi_workspace* ws, FusedParams& p, size_t& smem, int r_max = 0) {
  const pi_layer_desc& d = L->desc;
  std::memset(&p, 0, sizeof(p));
  p.B = B; p.d = d.d_model; p.f = d.d_ff; p.r = r_max > 0 ? r_max : d.rank;
  if (p.r > 3072) return PI_ERR_UNSUPPORTED;   // the u exchange polls at most 3072 words per token
  p.grid = ws->grid;
  p.row_bytes = L->row_bytes; p.rec_stride = L->rec_stride;
  p.gate_off = L->gate_off; p.up_off = L->up_off; p.bias_off = L->bias_off;
  p.dn_stride = L->dn_stride; p.dn_off = (long long)L->dn_off;
  p.p1_row = L->p1_row; p.p2_stride = p2_stride_of(p.r, L->family == FAM_F32 ? 4 : 2);
  p.nown_max = L->nown_max;
  p.act_square = d.act == PI_RELU2;
  if (L->G != ws->grid) return PI_ERR_ARG;   // layer laid out for another device
  if (L->nown_max > kMaxOwn) return PI_ERR_UNSUPPORTED;
  if (!fused_supported(L->family, B, d.d_model)) return PI_ERR_UNSUPPORTED;
  if (!fused_plan_smem(p, L->family, (size_t)smem_optin(ws->device), smem)) return PI_ERR_UNSUPPORTED;
  // ws fields
  p.ux = ws->ux; p.mx = ws->mx; p.hx = ws->hx; p.vx = ws->vx; p.yx = ws->yx;
  p.bar = ws->bar; p.err = ws->err; p.active_total = ws->active_total;
  p.layer_count = nullptr;
  p.barrier_timeout_ns = kDefaultWaitNs;
  p.wait_cycles = kDefaultWaitNs * 3;   // cycles at up to 3 GHz: at least the nominal budget
  p.barrier_extra = 0;
  p.poll_ns = 256;         // back-off between exchange polling rounds (a round costs ~1 us anyway)
  p.inflight_budget = inflight_budget_bytes();
  return PI_OK;
}

pi_status check_ws(const pi_workspace* ws, const pi_layer_desc& d, int B, int L) {
  if (!ws) return PI_ERR_ARG;
  if (d.d_model > ws->d_max || d.d_ff > ws->f_max || d.rank > ws->r_max || B > ws->B_max || L > ws->L_max)
    return PI_ERR_ARG;
  return PI_OK;
}

BatchedLayer bview(const pi_layer* L) {
  BatchedLayer b;
  b.d = L->desc.d_model; b.f = L->desc.d_ff; b.r = L->desc.rank; b.G = L->G; b.nown_max = L->nown_max;
  b.rec = L->rec; b.rec_stride = L->rec_stride; b.up_off = L->up_off; b.gate_off = L->gate_off;
  b.dn = L->rec + L->dn_off; b.dn_stride = L->dn_stride;
  b.p1t = L->p1t; b.p1_row = L->p1_row; b.p2o = L->p2o; b.p2_stride = L->p2_stride;
  b.thresh = L->thresh; b.bias = L->bias;
  b.act_square = L->desc.act == PI_RELU2;
  return b;
}
// Calls the fused kernel does not serve take the batched path: more than 4 tokens, or
// 2 to 4 tokens with a d_model beyond the fused kernel's registers for that many tokens.
bool use_batched(const pi_layer* L, int B) {
  if (B > 4) return true;
  return !fused_supported(L->family, B, L->desc.d_model) &&
         batched_supported(L->family, B, L->desc.d_model, L->desc.rank);
}

// pi_decode_stack for more than 4 tokens: per layer, the predictor (mask words), the
// compaction of the union, the gate/up rows and the down columns of the active neurons,
// and the stack glue, as consecutive launches on the stream.
pi_status decode_stack_batched(pi_layer* const* layers, int Lc, void* x_inout, int B, const pi_trace* trace,
                               pi_workspace* ws, cudaStream_t stream) {
  const pi_layer* L0 = layers[0];
  const int d = L0->desc.d_model, f = L0->desc.d_ff, words = f / 32;
  for (int l = 0; l < Lc; ++l)
    if (!batched_supported(L0->family, B, d, layers[l]->desc.rank) || !ws->u_hi) return PI_ERR_UNSUPPORTED;
  if (trace && (trace->idx || trace->count) && !(trace->idx && trace->count && trace->mask)) return PI_ERR_ARG;
  PI_TRY(cudaMemsetAsync(ws->layer_count, 0, (size_t)Lc * 4, stream));
  if (trace && trace->x)
    PI_TRY(cudaMemcpyAsync(trace->x, x_inout, (size_t)B * d * 2, cudaMemcpyDeviceToDevice, stream));
  for (int l = 0; l < Lc; ++l) {
    const BatchedLayer bl = bview(layers[l]);
    uint32_t* mask = (trace && trace->mask) ? trace->mask + (size_t)l * B * words : ws->bmask;
    int32_t* idx = (trace && trace->idx) ? trace->idx + (size_t)l * f : ws->bidx;
    int32_t* count = (trace && trace->count) ? trace->count + l : ws->bcount;
    float* logits = (trace && trace->logits) ? trace->logits + (size_t)l * B * f : nullptr;
    float* y = (trace && trace->y) ? trace->y + (size_t)l * B * d : ws->by;
    void* tx = (trace && trace->x) ? static_cast<uint8_t*>(trace->x) + (size_t)(l + 1) * B * d * 2 : nullptr;
    PI_TRY(cudaMemsetAsync(mask, 0, (size_t)B * words * 4, stream));
    PI_TRY(batched_predict(bl, x_inout, B, mask, logits, ws->u_hi, ws->u_lo, ws->bpart, ws->bpart_floats, stream));
    PI_TRY(launch_compact(mask, B, f, idx, count, stream));
    PI_TRY(batched_count(count, ws->active_total, ws->layer_count + l, stream));
    PI_TRY(batched_ffn(bl, x_inout, B, mask, idx, count, ws->bh, y, ws->bpart, ws->bpart_floats, ws->bypart, ws->err,
                       stream));
    PI_TRY(batched_glue(x_inout, y, B, d, x_inout, tx, stream));
  }
  return PI_OK;
}

// Per-batch keep floors from the firing frequencies of the reorder: a share of the
// expected active records per block at batch B.  Every block keeps that many of its own
// active neurons whatever the counts say, so their records are fetched while the mask
// exchange runs.  Below the balanced target (the mean count) the floor does not change
// the assignment, so it sits just under the expected mean.
constexpr double kKeepShare = 0.85;
void set_batch_tables(pi_layer* L) {
  for (int B = 1; B <= 4; ++B) {
    double expect = 0.0;
    for (int i = 0; i < L->desc.d_ff; ++i) expect += 1.0 - std::pow(1.0 - (double)L->freq_host[i], (double)B);
    L->keep_floor[B - 1] = (int)(kKeepShare * expect / L->G);
  }
}

LayerDev dev_view(const pi_layer* L, int B = 0) {
  return LayerDev{L->rec, L->p1t, L->p2o, B > 0 ? L->keep_floor[std::min(B, 4) - 1] : 0, L->desc.rank};
}

// Layers of one stack share everything but the predictor rank, which may differ per layer.
bool same_desc_but_rank(const pi_layer_desc& a, const pi_layer_desc& b) {
  return a.d_model == b.d_model && a.d_ff == b.d_ff && a.act == b.act && a.w_dtype == b.w_dtype &&
         a.x_dtype == b.x_dtype && a.p_dtype == b.p_dtype;
}

}  // namespace

namespace pi {
std::atomic<uint64_t>& launch_counter() {
  static std::atomic<uint64_t> n{0};
  return n;
}
void note_launch() { launch_counter().fetch_add(1, std::memory_order_relaxed); }
}  // namespace pi

extern "C" {

int pi_abi_version(void) { return 10000; }

uint64_t pi_kernel_launches(void) { return pi::launch_counter().load(std::memory_order_relaxed); }

const char* pi_status_str(pi_status s) {
  switch (s) {
    case PI_OK: return "ok";
    case PI_ERR_ARG: return "invalid argument";
    case PI_ERR_UNSUPPORTED: return "unsupported shape, batch or dtype combination";
    case PI_ERR_OOM: return "device allocation failed";
    case PI_ERR_CUDA: return "CUDA runtime error";
    case PI_ERR_TIMEOUT: return "a device-side wait timed out";
    case PI_ERR_DEVICE: return "a device-side check failed";
  }
  return "unknown status";
}

// ------------------------------------------------------------------ layers
pi_status pi_load_layer(const pi_layer_desc* desc, const pi_layer_weights* w, cudaStream_t stream,
                        pi_layer** out) {
  if (!desc || !w || !out) return PI_ERR_ARG;
  *out = nullptr;
  pi_status st = check_desc(*desc);
  if (st != PI_OK) return st;
  const pi_layer_desc& d = *desc;
  const int fam = family_of(d);
  const bool reglu = d.act == PI_REGLU;
  if (!w->w_up || !w->w_down || !w->bias || !w->p1 || !w->p2 || !w->thresh) return PI_ERR_ARG;
  if (reglu != (w->w_gate != nullptr)) return PI_ERR_ARG;
  if (fam == FAM_Q4 && (!w->s_up || !w->s_down || (reglu && !w->s_gate))) return PI_ERR_ARG;
  if (fam != FAM_Q4 && (w->s_up || w->s_gate || w->s_down)) return PI_ERR_ARG;

  pi_layer* L = new (std::nothrow) pi_layer;
  if (!L) return PI_ERR_OOM;
  std::memset(L, 0, sizeof(*L));
  L->desc = d;
  L->family = fam;
  L->hot_count = -1;
  cudaGetDevice(&L->device);
  const int D = d.d_model, F = d.d_ff, R = d.rank;
  const int pb = wbytes(fam == FAM_Q4 ? FAM_F16 : fam);
  L->row_bytes = fam == FAM_Q4 ? round16((long long)D / 2 + D / 16) : D * wbytes(fam);
  L->rec_stride = L->row_bytes * (reglu ? 2 : 1) + 16;   // gate?, up, then a 16-byte header with the bias
  L->gate_off = reglu ? 0 : -1;
  L->up_off = reglu ? L->row_bytes : 0;
  L->bias_off = L->up_off + L->row_bytes;
  L->dn_stride = L->row_bytes;
  L->dn_off = (size_t)d.d_ff * L->rec_stride;
  L->p1_row = D * pb;
  L->p2_stride = round16((long long)R * pb + 8);
  L->G = sm_count(L->device);
  if (L->G <= 0) { delete L; return PI_ERR_CUDA; }
  L->nown_max = (F + L->G - 1) / L->G;

  auto fail = [&](pi_status s) { free_layer_buffers(L); delete L; return s; };
  const size_t rec_bytes = L->dn_off + (size_t)F * L->dn_stride;
  if (dmalloc(&L->rec, rec_bytes) != cudaSuccess) return fail(PI_ERR_OOM);
  if (dmalloc(&L->p1t, (size_t)R * L->p1_row) != cudaSuccess) return fail(PI_ERR_OOM);
  if (dmalloc(&L->p2o, (size_t)L->G * L->nown_max * L->p2_stride) != cudaSuccess) return fail(PI_ERR_OOM);
  if (dmalloc(&L->bias, (size_t)F * 4) != cudaSuccess) return fail(PI_ERR_OOM);
  if (dmalloc(&L->thresh, (size_t)F * 4) != cudaSuccess) return fail(PI_ERR_OOM);
  if (dmalloc(&L->perm, (size_t)F * 4) != cudaSuccess) return fail(PI_ERR_OOM);

  cudaError_t e = cudaSuccess;
  auto step = [&](cudaError_t r) { if (e == cudaSuccess) e = r; };
  step(cudaMemsetAsync(L->rec, 0, rec_bytes, stream));
  step(cudaMemsetAsync(L->p2o, 0, (size_t)L->G * L->nown_max * L->p2_stride, stream));
  if (fam == FAM_Q4) {
    const int nb = D / 32;
    const void* nib[3] = {w->w_gate, w->w_up, w->w_down};
    const void* scl[3] = {w->s_gate, w->s_up, w->s_down};
    uint8_t* const base[3] = {L->rec, L->rec, L->rec + L->dn_off};
    const int stride[3] = {L->rec_stride, L->rec_stride, L->dn_stride};
    const int off[3] = {L->gate_off, L->up_off, 0};
    for (int m = reglu ? 0 : 1; m < 3; ++m) {
      step(relayout_copy_rows(nib[m], nb * 16, 0, base[m], stride[m], off[m], F, nb * 16, nullptr, stream));
      step(relayout_copy_rows(scl[m], nb * 2, 0, base[m], stride[m], off[m] + D / 2, F, nb * 2, nullptr, stream));
    }
  } else {
    const int wb = wbytes(fam);
    if (reglu) step(relayout_copy_rows(w->w_gate, (long long)D * wb, 0, L->rec, L->rec_stride, L->gate_off, F, D * wb, nullptr, stream));
    step(relayout_copy_rows(w->w_up, (long long)D * wb, 0, L->rec, L->rec_stride, L->up_off, F, D * wb, nullptr, stream));
    // down: caller's [d x f] row-major -> neuron-major rows
    step(relayout_transpose(w->w_down, wb, D, F, F, L->rec + L->dn_off, L->dn_stride, 0, stream));
  }
  // P1 [d x r] -> P1^T [r x d];  P2 [r x f] -> per-neuron rows [f][r] + (t, b)
  step(relayout_transpose(w->p1, pb, D, R, R, L->p1t, L->p1_row, 0, stream));
  step(relayout_transpose(w->p2, pb, R, F, F, L->p2o, L->p2_stride, 0, stream, L->G, L->nown_max));
  step(relayout_p2_header(w->thresh, w->bias, F, L->p2o, L->p2_stride, R * pb, L->G, L->nown_max, stream));
  step(relayout_row_scalar(w->bias, F, L->rec, L->rec_stride, L->bias_off, stream));
  step(cudaMemcpyAsync(L->bias, w->bias, (size_t)F * 4, cudaMemcpyDeviceToDevice, stream));
  step(cudaMemcpyAsync(L->thresh, w->thresh, (size_t)F * 4, cudaMemcpyDeviceToDevice, stream));
  step(iota_i32(L->perm, F, stream));
  step(cudaStreamSynchronize(stream));
  if (e != cudaSuccess) return fail(cuda_status(e));
  *out = L;
  return PI_OK;
}

void pi_free_layer(pi_layer* L) {
  if (!L) return;
  free_layer_buffers(L);
  delete L;
}

pi_status pi_layer_get_desc(const pi_layer* L, pi_layer_desc* out) {
  if (!L || !out) return PI_ERR_ARG;
  *out = L->desc;
  return PI_OK;
}

pi_status pi_get_perm(const pi_layer* L, int32_t* perm_out, cudaStream_t stream) {
  if (!L || !perm_out) return PI_ERR_ARG;
  return cuda_status(cudaMemcpyAsync(perm_out, L->perm, (size_t)L->desc.d_ff * 4, cudaMemcpyDeviceToDevice, stream));
}

pi_status pi_reorder_hot_prefix(pi_layer* L, const float* freq, int hot_count, cudaStream_t stream) {
  if (!L || !freq) return PI_ERR_ARG;
  const int F = L->desc.d_ff;
  if (hot_count < -1 || hot_count > F) return PI_ERR_ARG;
  int32_t* order = nullptr;
  int* bad = nullptr;
  uint8_t *rec = nullptr, *p2o = nullptr;
  const size_t p2_bytes = (size_t)L->G * L->nown_max * L->p2_stride;
  float *bias = nullptr, *thresh = nullptr, *fs = nullptr;
  int32_t* perm = nullptr;
  auto cleanup = [&]() {
    cudaFree(order); cudaFree(bad); cudaFree(rec); cudaFree(p2o); cudaFree(bias); cudaFree(thresh);
    cudaFree(fs); cudaFree(perm);
  };
  const size_t rec_bytes = L->dn_off + (size_t)F * L->dn_stride;
  if (dmalloc(&order, (size_t)F * 4) || dmalloc(&bad, 4) || dmalloc(&rec, rec_bytes) ||
      dmalloc(&p2o, p2_bytes) || dmalloc(&bias, (size_t)F * 4) || dmalloc(&thresh, (size_t)F * 4) ||
      dmalloc(&fs, (size_t)F * 4) || dmalloc(&perm, (size_t)F * 4)) {
    cleanup();
    return PI_ERR_OOM;
  }
  cudaError_t e = cudaSuccess;
  auto step = [&](cudaError_t r) { if (e == cudaSuccess) e = r; };
  step(cudaMemsetAsync(bad, 0, 4, stream));
  step(hot_order(freq, F, order, bad, stream));
  int hbad = 0;
  step(cudaMemcpyAsync(&hbad, bad, 4, cudaMemcpyDeviceToHost, stream));
  step(cudaStreamSynchronize(stream));
  if (e != cudaSuccess) { cleanup(); return cuda_status(e); }
  if (hbad) { cleanup(); return PI_ERR_ARG; }
  step(relayout_copy_rows(L->rec, L->rec_stride, 0, rec, L->rec_stride, 0, F, L->rec_stride, order, stream));
  step(relayout_copy_rows(L->rec + L->dn_off, L->dn_stride, 0, rec + L->dn_off, L->dn_stride, 0, F, L->dn_stride, order,
                          stream));
  step(cudaMemsetAsync(p2o, 0, p2_bytes, stream));
  step(gather_owner_rows(L->p2o, p2o, order, F, L->G, L->nown_max, L->p2_stride, stream));
  step(gather_f32(L->bias, order, F, bias, stream));
  step(gather_f32(L->thresh, order, F, thresh, stream));
  step(gather_f32(freq, order, F, fs, stream));
  step(gather_i32(L->perm, order, F, perm, stream));
  step(cudaStreamSynchronize(stream));
  if (e != cudaSuccess) { cleanup(); return cuda_status(e); }
  std::swap(L->rec, rec);
  std::swap(L->p2o, p2o);
  std::swap(L->bias, bias);
  std::swap(L->thresh, thresh);
  std::swap(L->freq_sorted, fs);
  std::swap(L->perm, perm);
  L->hot_count = hot_count;
  float* fh = new (std::nothrow) float[F];
  if (fh && cudaMemcpy(fh, L->freq_sorted, (size_t)F * 4, cudaMemcpyDeviceToHost) == cudaSuccess) {
    delete[] L->freq_host;
    L->freq_host = fh;
    set_batch_tables(L);
  } else {
    delete[] fh;
  }
  cleanup();   // frees the old buffers now held in the temporaries
  return PI_OK;
}

// ------------------------------------------------------------------ workspace
pi_status pi_workspace_create(int d_max, int f_max, int r_max, int B_max, int L_max, pi_workspace** out) {
  if (!out) return PI_ERR_ARG;
  *out = nullptr;
  if (d_max <= 0 || f_max <= 0 || r_max <= 0 || B_max < 1 || B_max > PI_MAX_BATCH || L_max < 1 || L_max > kMaxLayers)
    return PI_ERR_ARG;
  if (d_max % 64 || f_max % 32) return PI_ERR_ARG;
  pi_workspace* ws = new (std::nothrow) pi_workspace;
  if (!ws) return PI_ERR_OOM;
  std::memset(ws, 0, sizeof(*ws));
  ws->d_max = d_max; ws->f_max = f_max; ws->r_max = r_max; ws->B_max = B_max; ws->L_max = L_max;
  cudaGetDevice(&ws->device);
  ws->grid = sm_count(ws->device);
  if (ws->grid <= 0) { delete ws; return PI_ERR_CUDA; }
  if (ws->grid > kMaxGrid) { delete ws; return PI_ERR_UNSUPPORTED; }
  const size_t G = ws->grid, Bm = B_max;
  const size_t mx_bytes = G * 4 * kMaxOwnWords * 8, hx_bytes = ((size_t)f_max + G) * Bm * 8;
  bool ok = dmalloc(&ws->ux, Bm * r_max * 8) == cudaSuccess &&
            dmalloc(&ws->mx, mx_bytes) == cudaSuccess &&
            dmalloc(&ws->hx, hx_bytes) == cudaSuccess &&
            dmalloc(&ws->vx, (Bm * d_max + 2 * Bm * G) * 8) == cudaSuccess &&
            dmalloc(&ws->yx, G * (size_t)d_max * 8) == cudaSuccess &&
            dmalloc(&ws->bar, 64) == cudaSuccess &&
            dmalloc(&ws->err, 16) == cudaSuccess &&
            dmalloc(&ws->active_total, 16) == cudaSuccess &&
            dmalloc(&ws->layer_count, (size_t)L_max * 4) == cudaSuccess &&
            dmalloc(&ws->x_dev, Bm * d_max * 4) == cudaSuccess;
  if (ok && B_max > 1) {   // batched path buffers (more than one token)
    ok = dmalloc(&ws->u_hi, (size_t)32 * r_max * 2) == cudaSuccess && dmalloc(&ws->u_lo, (size_t)32 * r_max * 2) == cudaSuccess &&
         dmalloc(&ws->bmask, (size_t)32 * (f_max / 32) * 4) == cudaSuccess && dmalloc(&ws->bidx, (size_t)f_max * 4) == cudaSuccess &&
         dmalloc(&ws->bcount, 16) == cudaSuccess && dmalloc(&ws->bh, (size_t)f_max * 32 * 4) == cudaSuccess &&
         dmalloc(&ws->by, (size_t)32 * d_max * 4) == cudaSuccess;
    ws->bpart_floats = batched_part_floats(d_max, f_max, r_max);
    ok = ok && dmalloc(&ws->bpart, ws->bpart_floats * 4) == cudaSuccess &&
         dmalloc(&ws->bypart, batched_ypart_floats(d_max) * 4) == cudaSuccess;
  }
  if (ok) {
    // tagged words start with tag 0; launch epochs start at 1, so no stale word matches
    const uint32_t bar0[4] = {0u, 0u, 1u, 0u};
    ok = cudaMemset(ws->ux, 0, Bm * r_max * 8) == cudaSuccess && cudaMemset(ws->mx, 0, mx_bytes) == cudaSuccess &&
         cudaMemset(ws->hx, 0, hx_bytes) == cudaSuccess &&
         cudaMemset(ws->vx, 0, (Bm * d_max + 2 * Bm * G) * 8) == cudaSuccess &&
         cudaMemset(ws->yx, 0, G * (size_t)d_max * 8) == cudaSuccess &&
         cudaMemset(ws->bar, 0, 64) == cudaSuccess &&
         cudaMemcpy(ws->bar, bar0, sizeof(bar0), cudaMemcpyHostToDevice) == cudaSuccess &&
         cudaMemset(ws->err, 0, 16) == cudaSuccess && cudaMemset(ws->active_total, 0, 16) == cudaSuccess &&
         cudaMemset(ws->layer_count, 0, (size_t)L_max * 4) == cudaSuccess && cudaDeviceSynchronize() == cudaSuccess;
  }
  if (!ok) {
    cudaGetLastError();
    pi_workspace_free(ws);
    return PI_ERR_OOM;
  }
  *out = ws;
  return PI_OK;
}

void pi_workspace_free(pi_workspace* ws) {
  if (!ws) return;
  cudaFree(ws->ux); cudaFree(ws->mx); cudaFree(ws->hx); cudaFree(ws->vx); cudaFree(ws->yx);
  cudaFree(ws->bar); cudaFree(ws->err); cudaFree(ws->active_total);
  cudaFree(ws->layer_count); cudaFree(ws->x_dev); cudaFree(ws->phase_clk);
  cudaFree(ws->u_hi); cudaFree(ws->u_lo); cudaFree(ws->bmask); cudaFree(ws->bidx); cudaFree(ws->bcount);
  cudaFree(ws->bh); cudaFree(ws->by); cudaFree(ws->bpart); cudaFree(ws->bypart);
  delete ws;
}

pi_status pi_stream_status(pi_workspace* ws, cudaStream_t stream) {
  if (!ws) return PI_ERR_ARG;
  PI_TRY(cudaStreamSynchronize(stream));
  int err = 0;
  PI_TRY(cudaMemcpy(&err, ws->err, 4, cudaMemcpyDeviceToHost));
  if (err == 0) return PI_OK;
  uint32_t bar[4];
  PI_TRY(cudaMemcpy(bar, ws->bar, sizeof(bar), cudaMemcpyDeviceToHost));
  bar[0] = 0u;
  bar[1] = 0u;
  bar[2] = next_launch_epoch(bar[2]);   // fresh tags: nothing an aborted launch left behind can match
  PI_TRY(cudaMemcpy(ws->bar, bar, sizeof(bar), cudaMemcpyHostToDevice));
  PI_TRY(cudaMemset(ws->err, 0, 16));
  PI_TRY(cudaDeviceSynchronize());
  return (err == DEV_ERR_GRID_TIMEOUT || err == DEV_ERR_RING_TIMEOUT) ? PI_ERR_TIMEOUT : PI_ERR_DEVICE;
}

pi_status pi_workspace_active_total(pi_workspace* ws, unsigned long long* out) {
  if (!ws || !out) return PI_ERR_ARG;
  PI_TRY(cudaMemcpy(out, ws->active_total, 8, cudaMemcpyDeviceToHost));
  return PI_OK;
}

pi_status pi_workspace_layer_counts(pi_workspace* ws, int32_t* host_out, int L) {
  if (!ws || !host_out || L < 1 || L > ws->L_max) return PI_ERR_ARG;
  PI_TRY(cudaMemcpy(host_out, ws->layer_count, (size_t)L * 4, cudaMemcpyDeviceToHost));
  return PI_OK;
}

// ------------------------------------------------------------------ hot path
pi_status pi_predict(const pi_layer* L, const void* x, int B, uint32_t* mask, float* logits, pi_workspace* ws,
                     cudaStream_t stream) {
  if (!L || !x || !mask || B < 1 || B > PI_MAX_BATCH) return PI_ERR_ARG;
  pi_status st = check_ws(ws, L->desc, B, 1);
  if (st != PI_OK) return st;
  if (use_batched(L, B)) {
    if (!batched_supported(L->family, B, L->desc.d_model, L->desc.rank) || !ws->u_hi) return PI_ERR_UNSUPPORTED;
    PI_TRY(cudaMemsetAsync(mask, 0, (size_t)B * (L->desc.d_ff / 32) * 4, stream));
    PI_TRY(batched_predict(bview(L), x, B, mask, logits, ws->u_hi, ws->u_lo, ws->bpart, ws->bpart_floats, stream));
    return PI_OK;
  }
  FusedParams p;
  size_t smem = 0;
  st = plan_fused(L, B, ws, p, smem);
  if (st != PI_OK) return st;
  p.mode = MODE_PREDICT;
  p.L = 1;
  p.layers[0] = dev_view(L);
  p.x_in = x;
  p.mask_out = mask;
  p.logits_out = logits;
  PI_TRY(cudaMemsetAsync(mask, 0, (size_t)B * (L->desc.d_ff / 32) * 4, stream));   // bits are OR-ed in
  PI_TRY(launch_fused(L->family, L->desc.act, B, p, smem, stream));
  note_launch();
  return PI_OK;
}

pi_status pi_compact_active(const uint32_t* mask, int B, int d_ff, int32_t* idx, int32_t* count, cudaStream_t stream) {
  if (!mask || !idx || !count || B < 1 || B > PI_MAX_BATCH || d_ff < 32 || d_ff % 32) return PI_ERR_ARG;
  PI_TRY(launch_compact(mask, B, d_ff, idx, count, stream));
  return PI_OK;
}

pi_status pi_sparse_ffn(const pi_layer* L, const void* x, int B, const uint32_t* mask, const int32_t* idx,
                        const int32_t* count, float* y, pi_workspace* ws, cudaStream_t stream) {
  if (!L || !x || !mask || !idx || !count || !y || B < 1 || B > PI_MAX_BATCH) return PI_ERR_ARG;
  pi_status st = check_ws(ws, L->desc, B, 1);
  if (st != PI_OK) return st;
  if (use_batched(L, B)) {
    if (!batched_supported(L->family, B, L->desc.d_model, L->desc.rank) || !ws->u_hi) return PI_ERR_UNSUPPORTED;
    PI_TRY(batched_ffn(bview(L), x, B, mask, idx, count, ws->bh, y, ws->bpart, ws->bpart_floats, ws->bypart, ws->err,
                       stream));
    return PI_OK;
  }
  FusedParams p;
  size_t smem = 0;
  st = plan_fused(L, B, ws, p, smem);
  if (st != PI_OK) return st;
  if ((L->desc.d_ff + ws->grid - 1) / ws->grid > kMaxList) return PI_ERR_UNSUPPORTED;
  p.mode = MODE_FFN;
  p.L = 1;
  p.layers[0] = dev_view(L);
  p.x_in = x;
  p.mask_in = mask;
  p.idx_in = idx;
  p.count_in = count;
  p.y_out = y;
  PI_TRY(launch_fused(L->family, L->desc.act, B, p, smem, stream));
  note_launch();
  return PI_OK;
}

pi_status pi_decode_stack(pi_layer* const* layers, int Lc, void* x_inout, int B, const pi_trace* trace,
                          pi_workspace* ws, cudaStream_t stream) {
  if (!layers || Lc < 1 || Lc > kMaxLayers || !x_inout || B < 1 || B > PI_MAX_BATCH) return PI_ERR_ARG;
  int r_max = 0;
  for (int l = 0; l < Lc; ++l) {
    if (!layers[l]) return PI_ERR_ARG;
    if (!same_desc_but_rank(layers[l]->desc, layers[0]->desc)) return PI_ERR_ARG;
    r_max = std::max(r_max, layers[l]->desc.rank);
  }
  const pi_layer* L0 = layers[0];
  pi_status st = check_ws(ws, L0->desc, B, Lc);
  if (st != PI_OK) return st;
  if (r_max > ws->r_max) return PI_ERR_ARG;
  if (use_batched(L0, B)) return decode_stack_batched(layers, Lc, x_inout, B, trace, ws, stream);
  FusedParams p;
  size_t smem = 0;
  st = plan_fused(L0, B, ws, p, smem, r_max);
  if (st != PI_OK) return st;
  p.mode = MODE_PREDICT | MODE_FFN | MODE_GLUE;
  p.L = Lc;
  for (int l = 0; l < Lc; ++l) p.layers[l] = dev_view(layers[l], B);
  p.x_in = x_inout;
  p.x_out = x_inout;
  const int words = L0->desc.d_ff / 32;
  if (trace) {
    // idx and count are the compaction of the layer's mask, so they come with it
    if ((trace->idx || trace->count) && !(trace->idx && trace->count && trace->mask)) return PI_ERR_ARG;
    p.trace = *trace;
    p.trace.idx = nullptr;
    p.trace.count = nullptr;
  }
  p.layer_count = ws->layer_count;
  p.phase_clk = ws->phase_clk;
  p.phase_global = ws->phase_global;
  PI_TRY(cudaMemsetAsync(ws->layer_count, 0, (size_t)Lc * 4, stream));
  if (trace && trace->mask) PI_TRY(cudaMemsetAsync(trace->mask, 0, (size_t)Lc * B * words * 4, stream));
  PI_TRY(launch_fused(L0->family, L0->desc.act, B, p, smem, stream));
  note_launch();
  if (trace && trace->idx)
    for (int l = 0; l < Lc; ++l)
      PI_TRY(launch_compact(trace->mask + (size_t)l * B * words, B, L0->desc.d_ff, trace->idx + (size_t)l * L0->desc.d_ff,
                            trace->count + l, stream));
  return PI_OK;
}

pi_status pi_decode_stack_host(pi_layer* const* layers, int Lc, const void* x_host, void* x_out_host, int B,
                               pi_workspace* ws, cudaStream_t stream) {
  if (!layers || Lc < 1 || !layers[0] || !x_host || !x_out_host || !ws || B < 1 || B > ws->B_max) return PI_ERR_ARG;
  const size_t bytes = (size_t)B * layers[0]->desc.d_model * x_elem(layers[0]->desc);
  if (layers[0]->desc.d_model > ws->d_max) return PI_ERR_ARG;
  PI_TRY(cudaMemcpyAsync(ws->x_dev, x_host, bytes, cudaMemcpyHostToDevice, stream));
  pi_status st = pi_decode_stack(layers, Lc, ws->x_dev, B, nullptr, ws, stream);
  if (st != PI_OK) return st;
  PI_TRY(cudaMemcpyAsync(x_out_host, ws->x_dev, bytes, cudaMemcpyDeviceToHost, stream));
  return pi_stream_status(ws, stream);
}

pi_status pi_diag_phase_clocks_enable(pi_workspace* ws, int on) {
  if (!ws) return PI_ERR_ARG;
  if (!on) {
    cudaFree(ws->phase_clk);
    ws->phase_clk = nullptr;
    return PI_OK;
  }
  ws->phase_global = on == 2;
  if (ws->phase_clk) return PI_OK;
  const size_t n = (size_t)ws->grid * ws->L_max * kDiagSlots;
  if (dmalloc(&ws->phase_clk, n * sizeof(long long)) != cudaSuccess) return PI_ERR_OOM;
  PI_TRY(cudaMemset(ws->phase_clk, 0, n * sizeof(long long)));
  return PI_OK;
}

pi_status pi_diag_phase_clocks_read(pi_workspace* ws, long long* host_out, size_t n) {
  if (!ws || !host_out || !ws->phase_clk) return PI_ERR_ARG;
  const size_t total = (size_t)ws->grid * ws->L_max * kDiagSlots;
  if (n > total) return PI_ERR_ARG;
  PI_TRY(cudaMemcpy(host_out, ws->phase_clk, n * sizeof(long long), cudaMemcpyDeviceToHost));
  return PI_OK;
}

int pi_device_grid(pi_workspace* ws) { return ws ? ws->grid : 0; }

pi_status pi_diag_barrier_timeout(pi_workspace* ws, long long timeout_ns, cudaStream_t stream) {
  if (!ws || timeout_ns <= 0) return PI_ERR_ARG;
  FusedParams p;
  std::memset(&p, 0, sizeof(p));
  p.grid = ws->grid;
  p.bar = ws->bar;
  p.err = ws->err;
  p.barrier_timeout_ns = timeout_ns;
  p.wait_cycles = timeout_ns * 2;   // SM cycles, about 2 per ns
  p.barrier_extra = 1;   // one arrival more than the grid has: no wait can complete
  PI_TRY(launch_barrier_probe(p, 2, stream));
  note_launch();
  return PI_OK;
}

}  // extern "C"

// ------------------------------------------------------------------ predictor without a workspace
// pi_predict_noalloc runs the predictor launch of pi_predict with its cross-block
// scratch in one static device array instead of a workspace. It exists for callers that
// cannot allocate device memory when they call it: a serving loop that has already
// handed all free HBM to its weights and KV cache, and a plug-in that sees only a stream
// and plain pointers and so has nowhere to keep a workspace between calls.
// Layout of the array: [0, 64) launch words (probe count, exit count, epoch),
// [64, 128) error word, [128, 256) active-list total, then the tagged u words
// (B * rank * 8 bytes).
namespace {

constexpr size_t kNoallocCtlBytes = 256;
constexpr int kNoallocMaxDevices = 64;

static __device__ __align__(256) unsigned char g_noalloc_scratch[PI_NOALLOC_SCRATCH_BYTES];

std::mutex g_noalloc_mu;
unsigned char* g_noalloc_base[kNoallocMaxDevices];   // per device, set once

size_t round256(size_t v) { return (v + 255) / 256 * 256; }

// Launch words start as {0, 0, 1}: counts at zero, epoch 1, so that no zeroed tagged
// word matches a live tag.
__global__ void noalloc_init_kernel(uint32_t* ctl) { ctl[2] = 1u; }

// After the predictor launch: report its error word and, if it aborted, leave the
// scratch as a fresh workspace would be (counts at zero, a new epoch, error cleared).
__global__ void noalloc_status_kernel(uint32_t* ctl, int* err, int32_t* status) {
  const int e = *err;
  *status = e == 0 ? PI_OK
                   : (e == DEV_ERR_GRID_TIMEOUT || e == DEV_ERR_RING_TIMEOUT) ? PI_ERR_TIMEOUT : PI_ERR_DEVICE;
  if (e != 0) {
    ctl[0] = 0u;
    ctl[1] = 0u;
    ctl[2] = next_launch_epoch(ctl[2]);
    *err = 0;
  }
}

// The scratch of the current device: on its first use the symbol's address is taken,
// the array cleared and the epoch set, and `stream` synchronised so that any stream
// may make the next call.
pi_status noalloc_scratch(int dev, cudaStream_t stream, unsigned char** out) {
  if (dev < 0 || dev >= kNoallocMaxDevices) return PI_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (!g_noalloc_base[dev]) {
    void* ptr = nullptr;
    PI_TRY(cudaGetSymbolAddress(&ptr, g_noalloc_scratch));
    PI_TRY(cudaMemsetAsync(ptr, 0, PI_NOALLOC_SCRATCH_BYTES, stream));
    note_launch();
    noalloc_init_kernel<<<1, 1, 0, stream>>>(static_cast<uint32_t*>(ptr));
    PI_TRY(cudaGetLastError());
    PI_TRY(cudaStreamSynchronize(stream));
    g_noalloc_base[dev] = static_cast<unsigned char*>(ptr);
  }
  *out = g_noalloc_base[dev];
  return PI_OK;
}

}  // namespace

extern "C" {

pi_status pi_predict_noalloc(const pi_layer* L, const void* x, int B, uint32_t* mask, float* logits,
                             int32_t* status, cudaStream_t stream) {
  if (!L || !x || !mask || !status || B < 1 || B > PI_MAX_BATCH) return PI_ERR_ARG;
  int dev = -1;
  PI_TRY(cudaGetDevice(&dev));
  const int G = sm_count(dev);
  if (G <= 0) return PI_ERR_CUDA;
  if (L->G != G) return PI_ERR_ARG;   // layer laid out for another device
  const size_t u_bytes = round256((size_t)B * L->desc.rank * 8);
  if (kNoallocCtlBytes + u_bytes > PI_NOALLOC_SCRATCH_BYTES) return PI_ERR_UNSUPPORTED;
  pi_workspace w;   // a view of the static scratch; nothing is allocated
  std::memset(&w, 0, sizeof(w));
  w.d_max = L->desc.d_model; w.f_max = L->desc.d_ff; w.r_max = L->desc.rank; w.B_max = B; w.L_max = 1;
  w.grid = G;
  w.device = dev;
  // the shape check comes first: a refused shape enqueues nothing, not even the set-up
  FusedParams p;
  size_t smem = 0;
  pi_status st = plan_fused(L, B, &w, p, smem);
  if (st != PI_OK) return st;
  unsigned char* s = nullptr;
  st = noalloc_scratch(dev, stream, &s);
  if (st != PI_OK) return st;
  p.bar = reinterpret_cast<uint32_t*>(s);
  p.err = reinterpret_cast<int*>(s + 64);
  p.active_total = reinterpret_cast<unsigned long long*>(s + 128);
  p.ux = reinterpret_cast<uint64_t*>(s + kNoallocCtlBytes);
  p.mode = MODE_PREDICT;
  p.L = 1;
  p.layers[0] = dev_view(L);
  p.x_in = x;
  p.mask_out = mask;
  p.logits_out = logits;
  PI_TRY(cudaMemsetAsync(mask, 0, (size_t)B * (L->desc.d_ff / 32) * 4, stream));   // bits are OR-ed in
  PI_TRY(launch_fused(L->family, L->desc.act, B, p, smem, stream));
  note_launch();

  note_launch();
  noalloc_status_kernel<<<1, 1, 0, stream>>>(p.bar, p.err, status);
  PI_TRY(cudaGetLastError());
  return PI_OK;
}

}  // extern "C"
