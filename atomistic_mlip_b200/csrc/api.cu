// C ABI of libe2f (declared in include/e2f.h): argument validation,
// dispatch to the kernels, the library's memory pool, diagnostics.
#include <math.h>
#include <stdio.h>
#include <string.h>

#include <mutex>
#include <vector>

#include "common.cuh"
#include "wigner.cuh"

namespace e2f {

std::atomic<int64_t> g_launches{0};
static thread_local char t_last_err[256] = "no CUDA error";

void set_cuda_error(cudaError_t e, const char *where) {
  snprintf(t_last_err, sizeof(t_last_err), "%s: %s", where, cudaGetErrorString(e));
}

// ---- per-device state: memory pool and error flag ---------------------------
// One slot per device in a fixed array: a pointer to a slot stays valid for
// the life of the process, whatever device another thread initialises.  The
// error flag is per device, shared by every stream of that device (see
// e2f_stream_status).
constexpr int MAX_DEVICES = 64;
struct DeviceState {
  cudaMemPool_t pool = nullptr;
  int *err_flag = nullptr;
};
static std::mutex g_mu;
static DeviceState g_dev[MAX_DEVICES];

static DeviceState *device_state() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return nullptr;
  if (dev < 0 || dev >= MAX_DEVICES) return nullptr;
  std::lock_guard<std::mutex> lk(g_mu);
  DeviceState &d = g_dev[dev];
  if (!d.pool) {
    cudaMemPoolProps props;
    memset(&props, 0, sizeof(props));
    props.allocType = cudaMemAllocationTypePinned;
    props.handleTypes = cudaMemHandleTypeNone;
    props.location.type = cudaMemLocationTypeDevice;
    props.location.id = dev;
    if (cudaMemPoolCreate(&d.pool, &props) != cudaSuccess) { d.pool = nullptr; return nullptr; }
    uint64_t thr = UINT64_MAX;   // keep freed blocks for reuse by later calls
    cudaMemPoolSetAttribute(d.pool, cudaMemPoolAttrReleaseThreshold, &thr);
  }
  if (!d.err_flag) {
    if (cudaMalloc(&d.err_flag, sizeof(int)) != cudaSuccess) { d.err_flag = nullptr; return nullptr; }
    if (cudaMemset(d.err_flag, 0, sizeof(int)) != cudaSuccess) return nullptr;
  }
  return &d;
}

cudaError_t pool_alloc(void **p, size_t bytes, cudaStream_t s) {
  DeviceState *d = device_state();
  if (!d) return cudaErrorInitializationError;
  return cudaMallocFromPoolAsync(p, bytes, d->pool, s);
}

int *device_error_flag() {
  DeviceState *d = device_state();
  return d ? d->err_flag : nullptr;
}

// ---- profiling of the dominant kernel ------------------------------------------
static std::atomic<bool> g_prof_on{false};
static std::mutex g_prof_mu;
static std::vector<std::pair<cudaEvent_t, cudaEvent_t>> g_prof_events;

static void prof_events(cudaEvent_t *a, cudaEvent_t *b) {
  *a = *b = nullptr;
  if (!g_prof_on.load()) return;
  if (cudaEventCreate(a) != cudaSuccess || cudaEventCreate(b) != cudaSuccess) { *a = *b = nullptr; return; }
  std::lock_guard<std::mutex> lk(g_prof_mu);
  g_prof_events.emplace_back(*a, *b);
}

// kernels (other translation units)
e2f_status build_neighbors_impl(const float *, int64_t, const float *, float, int32_t *, int32_t *, int64_t,
                                int64_t *, cudaStream_t);
e2f_status project_impl(const void *, int64_t, const e2f_weights *, void *, void *, void *, cudaStream_t);
template <typename T>
e2f_status attention_simt_impl(const T *, const T *, const T *, const float *, const e2f_csr *,
                               const e2f_weights *, float *, cudaStream_t, cudaEvent_t, cudaEvent_t);
e2f_status attention_tc_available(const e2f_weights *w);
e2f_status attention_tc_impl(const void *q, const void *k, const void *v, const float *pos, const e2f_csr *csr,
                             const e2f_weights *w, float *out, cudaStream_t s, cudaEvent_t ev0, cudaEvent_t ev1,
                             int F, const float *focus_a);

__global__ void wigner_kernel(const float *__restrict__ R, int64_t n, int L, float *__restrict__ D) {
  const int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= n) return;
  float Rl[9];
  for (int k = 0; k < 9; ++k) Rl[k] = R[e * 9 + k];
  wig_all_serial(Rl, L, D + e * wig_size(L));
}

// Feature rows and weight matrices are read and written as 16-byte vectors.
static bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

static e2f_status validate_weights(const e2f_weights *w) {
  if (!w) return E2F_ERR_INVALID_ARG;
  if (w->L_max < 0 || w->L_max > E2F_MAX_L || w->C < 1 || w->H < 1) return E2F_ERR_INVALID_ARG;
  if (w->C % w->H != 0) return E2F_ERR_UNSUPPORTED;
  if (w->dtype != E2F_F32 && w->dtype != E2F_BF16) return E2F_ERR_UNSUPPORTED;
  for (int l = 0; l <= w->L_max; ++l)
    if (!w->Wq[l] || !w->Wk[l] || !w->Wv[l]) return E2F_ERR_INVALID_ARG;
  if (!w->W0 || !w->rad_W1 || !w->rad_W2) return E2F_ERR_INVALID_ARG;
  for (int m = 1; m <= w->L_max; ++m)
    if (!w->Wr[m] || !w->Wi[m]) return E2F_ERR_INVALID_ARG;
  for (int l = 0; l <= w->L_max; ++l)
    if (!aligned16(w->Wq[l]) || !aligned16(w->Wk[l]) || !aligned16(w->Wv[l])) return E2F_ERR_INVALID_ARG;
  if (!aligned16(w->W0)) return E2F_ERR_INVALID_ARG;
  for (int m = 1; m <= w->L_max; ++m)
    if (!aligned16(w->Wr[m]) || !aligned16(w->Wi[m])) return E2F_ERR_INVALID_ARG;
  return E2F_OK;
}

static e2f_status validate_csr(const e2f_csr *csr) {
  if (!csr || csr->n_nodes < 0 || csr->n_edges < 0 || !(csr->r_c > 0.f)) return E2F_ERR_INVALID_ARG;
  if (csr->n_nodes > 0 && (!csr->row_ptr || (csr->n_edges > 0 && !csr->col_idx))) return E2F_ERR_INVALID_ARG;
  for (int k = 0; k < 3; ++k)
    if (csr->box[k] > 0.f && !(csr->r_c < 0.5f * csr->box[k])) return E2F_ERR_CUTOFF_TOO_LARGE;
  return E2F_OK;
}

e2f_status block_forward_impl(const float *x, const float *pos, const e2f_csr *csr, const e2f_block_weights *w,
                              float *out, cudaStream_t s);
int64_t cg_num_paths(int L);
e2f_status cg_conv_impl(const void *x, int dtype, const float *pos, const e2f_csr *csr, int L, int C,
                        const float *W, float *out, cudaStream_t s);
e2f_status attention_backward_impl(const void *x, const float *pos, const e2f_csr *csr, const e2f_weights *w,
                                   const float *G, float *dx, float *dpos, cudaStream_t s);

// q, k, v (library scratch), then the fused attention kernel; arguments
// already validated.
e2f_status attention_forward_impl(const void *x, const float *pos, const e2f_csr *csr, const e2f_weights *w,
                                  float *out, cudaStream_t s, int F = 1, const float *focus_a = nullptr) {
  const int64_t N = csr->n_nodes;
  if (N == 0) return E2F_OK;
  const size_t Q = (size_t)(w->L_max + 1) * (w->L_max + 1);
  const size_t esz = w->dtype == E2F_F32 ? 4 : 2;
  const size_t feat = (size_t)N * Q * w->C * esz;
  Scratch qkv;
  E2F_CUDA_TRY(qkv.alloc(3 * feat, s));
  char *base = qkv.as<char>();
  void *q = base, *k = base + feat, *v = base + 2 * feat;
  e2f_status st = project_impl(x, N, w, q, k, v, s);
  if (st != E2F_OK) return st;
  cudaEvent_t ev0, ev1;
  prof_events(&ev0, &ev1);
  if (F > 1) {   // multi-focus: the tensor-core kernel only (checked by the caller)
    return attention_tc_impl(q, k, v, pos, csr, w, out, s, ev0, ev1, F, focus_a);
  }
  if (w->dtype == E2F_BF16 && attention_tc_available(w) == E2F_OK)
    return attention_tc_impl(q, k, v, pos, csr, w, out, s, ev0, ev1, 1, nullptr);
  if (w->dtype == E2F_F32)
    return attention_simt_impl<float>((const float *)q, (const float *)k, (const float *)v, pos, csr, w, out, s,
                                      ev0, ev1);
  return attention_simt_impl<__nv_bfloat16>((const __nv_bfloat16 *)q, (const __nv_bfloat16 *)k,
                                            (const __nv_bfloat16 *)v, pos, csr, w, out, s, ev0, ev1);
}

}  // namespace e2f

using namespace e2f;

extern "C" {

const char *e2f_status_string(e2f_status s) {
  switch (s) {
    case E2F_OK: return "ok";
    case E2F_ERR_INVALID_ARG: return "invalid argument";
    case E2F_ERR_CUTOFF_TOO_LARGE: return "cutoff >= half the periodic box";
    case E2F_ERR_CAPACITY: return "col_idx capacity too small";
    case E2F_ERR_UNSUPPORTED: return "unsupported shape or dtype";
    case E2F_ERR_CUDA: return "CUDA error";
    case E2F_ERR_TIMEOUT: return "bounded device wait timed out";
    case E2F_ERR_DOMAIN: return "coordinate outside the periodic box";
    case E2F_ERR_SCRATCH_LIMIT: return "input exceeds the fixed scratch of a no-allocation entry point";
    default: return "unknown status";
  }
}

const char *e2f_last_cuda_error(void) { return t_last_err; }

e2f_status e2f_build_neighbors(const float *pos, int64_t N, const float *box, float r_c, int32_t *row_ptr,
                               int32_t *col_idx, int64_t capacity, int64_t *n_edges, e2f_csr *out_csr,
                               void *stream) {
  if (N < 0 || N > INT32_MAX - 1 || !n_edges || !row_ptr || capacity < 0) return E2F_ERR_INVALID_ARG;
  if (N > 0 && !pos) return E2F_ERR_INVALID_ARG;
  if (capacity > 0 && !col_idx) return E2F_ERR_INVALID_ARG;
  if (!(r_c > 0.f) || !(r_c < INFINITY)) return E2F_ERR_INVALID_ARG;
  if (box) {
    for (int k = 0; k < 3; ++k) {
      if (!(box[k] >= 0.f) || !(box[k] < INFINITY)) return E2F_ERR_INVALID_ARG;
      if (box[k] > 0.f && !(r_c < 0.5f * box[k])) return E2F_ERR_CUTOFF_TOO_LARGE;
    }
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  e2f_status st = build_neighbors_impl(pos, N, box, r_c, row_ptr, col_idx, capacity, n_edges, s);
  if (st != E2F_OK && st != E2F_ERR_CAPACITY) return st;
  if (out_csr) {
    out_csr->row_ptr = row_ptr;
    out_csr->col_idx = col_idx;
    out_csr->n_nodes = N;
    out_csr->n_edges = *n_edges;
    for (int k = 0; k < 3; ++k) out_csr->box[k] = box ? box[k] : 0.f;
    out_csr->r_c = r_c;
  }
  return st;
}

e2f_status e2f_project_qkv(const void *x, int64_t N, const e2f_weights *w, void *q, void *k, void *v,
                           void *stream) {
  e2f_status st = validate_weights(w);
  if (st != E2F_OK) return st;
  if (N < 0) return E2F_ERR_INVALID_ARG;
  if (N > 0 && (!x || !q || !k || !v)) return E2F_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(q) || !aligned16(k) || !aligned16(v)) return E2F_ERR_INVALID_ARG;
  return project_impl(x, N, w, q, k, v, static_cast<cudaStream_t>(stream));
}

e2f_status e2f_attention_forward(const void *x, const float *pos, const e2f_csr *csr, const e2f_weights *w,
                                 float *out, void *stream) {
  e2f_status st = validate_weights(w);
  if (st != E2F_OK) return st;
  st = validate_csr(csr);
  if (st != E2F_OK) return st;
  if (csr->n_nodes == 0) return E2F_OK;
  if (!x || !pos || !out) return E2F_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(out)) return E2F_ERR_INVALID_ARG;
  return attention_forward_impl(x, pos, csr, w, out, static_cast<cudaStream_t>(stream));
}

e2f_status e2f_attention_backward(const void *x, const float *pos, const e2f_csr *csr, const e2f_weights *w,
                                  const float *grad_out, float *grad_x, float *grad_pos, void *stream) {
  e2f_status st = validate_weights(w);
  if (st != E2F_OK) return st;
  st = validate_csr(csr);
  if (st != E2F_OK) return st;
  if (w->H > 16) return E2F_ERR_UNSUPPORTED;
  if (csr->n_nodes == 0) return E2F_OK;
  if (!x || !pos || !grad_out || !grad_x || !grad_pos) return E2F_ERR_INVALID_ARG;
  if (!aligned16(x)) return E2F_ERR_INVALID_ARG;
  return attention_backward_impl(x, pos, csr, w, grad_out, grad_x, grad_pos, static_cast<cudaStream_t>(stream));
}

e2f_status e2f_block_forward(const float *x, const float *pos, const e2f_csr *csr, const e2f_block_weights *w,
                             float *out, void *stream) {
  if (!w) return E2F_ERR_INVALID_ARG;
  e2f_status st = validate_weights(&w->attn);
  if (st != E2F_OK) return st;
  st = validate_csr(csr);
  if (st != E2F_OK) return st;
  const int L = w->attn.L_max;
  if (w->hidden < 1 || !w->gamma1 || !w->gamma2 || !w->Wa || !aligned16(w->Wa)) return E2F_ERR_INVALID_ARG;
  for (int l = 0; l <= L; ++l)
    if (!w->Wb[l] || !w->Wd[l] || !aligned16(w->Wb[l]) || !aligned16(w->Wd[l])) return E2F_ERR_INVALID_ARG;
  if (csr->n_nodes == 0) return E2F_OK;
  if (!x || !pos || !out || x == out) return E2F_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(out)) return E2F_ERR_INVALID_ARG;
  return block_forward_impl(x, pos, csr, w, out, static_cast<cudaStream_t>(stream));
}

e2f_status e2f_attention_forward_multifocus(const void *x, const float *pos, const e2f_csr *csr, const e2f_weights *w,
                                            int32_t F, const float *focus_a, float *out, void *stream) {
  e2f_status st = validate_weights(w);
  if (st != E2F_OK) return st;
  st = validate_csr(csr);
  if (st != E2F_OK) return st;
  if (F != 1 && F != 2 && F != 4 && F != 8) return E2F_ERR_INVALID_ARG;
  if (F > 1) {
    if (attention_tc_available(w) != E2F_OK || (w->L_max != 2 && w->L_max != 4)) return E2F_ERR_UNSUPPORTED;
    if (!focus_a || !aligned16(focus_a)) return E2F_ERR_INVALID_ARG;
  }
  if (csr->n_nodes == 0) return E2F_OK;
  if (!x || !pos || !out) return E2F_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(out)) return E2F_ERR_INVALID_ARG;
  return attention_forward_impl(x, pos, csr, w, out, static_cast<cudaStream_t>(stream), F, focus_a);
}

int64_t e2f_cg_num_paths(int32_t L) {
  if (L < 0 || L > E2F_MAX_L) return -1;
  return cg_num_paths(L);
}

e2f_status e2f_cg_conv_forward(const void *x, int32_t dtype, const float *pos, const e2f_csr *csr, int32_t L,
                               int32_t C, const float *W, float *out, void *stream) {
  e2f_status st = validate_csr(csr);
  if (st != E2F_OK) return st;
  if (L < 0 || L > E2F_MAX_L) return E2F_ERR_UNSUPPORTED;
  if (dtype != E2F_F32 && dtype != E2F_BF16) return E2F_ERR_UNSUPPORTED;
  if (C < 2 || C > 256 || (C & 1)) return E2F_ERR_INVALID_ARG;
  if (csr->n_nodes == 0) return E2F_OK;
  if (!x || !pos || !W || !out) return E2F_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(out)) return E2F_ERR_INVALID_ARG;
  return cg_conv_impl(x, dtype, pos, csr, L, C, W, out, static_cast<cudaStream_t>(stream));
}

e2f_status e2f_stream_status(void *stream) {
  E2F_CUDA_TRY(cudaStreamSynchronize(static_cast<cudaStream_t>(stream)));
  int *flag = device_error_flag();
  if (!flag) return E2F_ERR_CUDA;
  int h = 0;
  E2F_CUDA_TRY(cudaMemcpy(&h, flag, sizeof(int), cudaMemcpyDeviceToHost));
  if (h) {
    E2F_CUDA_TRY(cudaMemset(flag, 0, sizeof(int)));
    return h;
  }
  return E2F_OK;
}

e2f_status e2f_wigner_d(const float *R, int64_t n, int32_t L, float *D, void *stream) {
  if (n < 0 || L < 0 || L > E2F_MAX_L) return E2F_ERR_INVALID_ARG;
  if (n == 0) return E2F_OK;
  if (!R || !D) return E2F_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  E2F_LAUNCH(wigner_kernel, (unsigned)((n + 127) / 128), 128, 0, s, R, n, L, D);
  return E2F_OK;
}

int64_t e2f_kernel_launches(void) { return g_launches.load(); }

e2f_status e2f_profile_enable(int32_t on) {
  g_prof_on = on != 0;
  return E2F_OK;
}

e2f_status e2f_profile_read(int64_t *launches, double *total_ms) {
  if (!launches || !total_ms) return E2F_ERR_INVALID_ARG;
  double tot = 0.0;
  int64_t n = 0;
  e2f_status st = E2F_OK;
  std::lock_guard<std::mutex> lk(g_prof_mu);
  for (auto &pr : g_prof_events) {
    float ms = 0.f;
    if (cudaEventSynchronize(pr.second) != cudaSuccess || cudaEventElapsedTime(&ms, pr.first, pr.second) != cudaSuccess)
      st = E2F_ERR_CUDA;
    tot += ms;
    ++n;
    cudaEventDestroy(pr.first);
    cudaEventDestroy(pr.second);
  }
  g_prof_events.clear();
  *launches = n;
  *total_ms = tot;
  return st;
}

e2f_status e2f_scratch_high_water(int64_t *bytes, int32_t reset) {
  if (!bytes) return E2F_ERR_INVALID_ARG;
  DeviceState *d = device_state();
  if (!d) return E2F_ERR_CUDA;
  uint64_t v = 0;
  E2F_CUDA_TRY(cudaMemPoolGetAttribute(d->pool, cudaMemPoolAttrUsedMemHigh, &v));
  *bytes = (int64_t)v;
  if (reset) {
    uint64_t z = 0;
    E2F_CUDA_TRY(cudaMemPoolSetAttribute(d->pool, cudaMemPoolAttrUsedMemHigh, &z));
  }
  return E2F_OK;
}

}  // extern "C"
