// Node projections q, k, v = per-degree C x C linear maps of x (the Q/K/V
// projections of E2Former-V2's node-centric factorisation, "E2Former-V2
// ...", §2.2; Eq. 6 is not printed, the per-degree map shared by all m is
// the reading used here).  x, q, k, v: [N][Q][C]; W[l]: [C][C] out x in.
//
// SIMT kernel: one block per (node chunk, degree l, which of q/k/v);
// W[l]^T is staged in shared memory, each thread produces outputs of one
// channel for several rows; fp32 accumulation, rounded once to T.
#include <algorithm>

#include "common.cuh"

namespace e2f {

struct ProjArgs {
  const void *W[3][E2F_MAX_L + 1];
  void *out[3];
};

constexpr int PROJ_THREADS = 256;
constexpr int PROJ_ROWS = 32;   // rows (node, m) per block pass

template <typename T>
__global__ void __launch_bounds__(PROJ_THREADS)
project_simt_kernel(const T *__restrict__ x, int N, int L, int C, ProjArgs a) {
  extern __shared__ float sm[];
  const int l = blockIdx.y, which = blockIdx.z;
  const int Q = (L + 1) * (L + 1);
  const int w = 2 * l + 1;
  float *WT = sm;                 // [C][C]: WT[ci][co]
  float *xs = sm + C * C;         // [PROJ_ROWS][C]
  const T *W = static_cast<const T *>(a.W[which][l]);
  T *out = static_cast<T *>(a.out[which]);
  for (int idx = threadIdx.x; idx < C * C; idx += PROJ_THREADS) {
    const int co = idx / C, ci = idx % C;
    WT[ci * C + co] = to_f(W[idx]);
  }
  const long long rows_total = (long long)N * w;
  const long long rows_per_block = ((rows_total + gridDim.x - 1) / gridDim.x + PROJ_ROWS - 1) / PROJ_ROWS * PROJ_ROWS;
  const long long r_begin = (long long)blockIdx.x * rows_per_block;
  const long long r_end = rows_total < r_begin + rows_per_block ? rows_total : r_begin + rows_per_block;
  for (long long r0 = r_begin; r0 < r_end; r0 += PROJ_ROWS) {
    const int nr = (int)(r_end - r0 < PROJ_ROWS ? r_end - r0 : PROJ_ROWS);
    __syncthreads();
    for (int idx = threadIdx.x; idx < nr * C; idx += PROJ_THREADS) {
      const long long r = r0 + idx / C;
      const int c = idx % C;
      const long long node = r / w;
      const int m = (int)(r % w);
      xs[idx] = to_f(x[(node * Q + l * l + m) * C + c]);
    }
    __syncthreads();
    for (int idx = threadIdx.x; idx < nr * C; idx += PROJ_THREADS) {
      const int rr = idx / C, co = idx % C;
      const float *xr = xs + rr * C;
      float acc = 0.f;
      for (int ci = 0; ci < C; ++ci) acc = fmaf(WT[ci * C + co], xr[ci], acc);
      const long long r = r0 + rr;
      const long long node = r / w;
      const int m = (int)(r % w);
      out[(node * Q + l * l + m) * C + co] = from_f<T>(acc);
    }
  }
}

e2f_status project_impl(const void *x, int64_t N, const e2f_weights *w, void *q, void *k, void *v,
                        cudaStream_t s) {
  if (N == 0) return E2F_OK;
  ProjArgs a;
  for (int l = 0; l <= E2F_MAX_L; ++l) {
    a.W[0][l] = l <= w->L_max ? w->Wq[l] : nullptr;
    a.W[1][l] = l <= w->L_max ? w->Wk[l] : nullptr;
    a.W[2][l] = l <= w->L_max ? w->Wv[l] : nullptr;
  }
  a.out[0] = q; a.out[1] = k; a.out[2] = v;
  const int C = w->C, L = w->L_max;
  const size_t smem = sizeof(float) * ((size_t)C * C + (size_t)PROJ_ROWS * C);
  long long rows_max = N * (2LL * L + 1);
  int gx = (int)std::min<long long>(std::max<long long>(1, rows_max / (4 * PROJ_ROWS)), 2048);
  dim3 grid(gx, L + 1, 3);
  if (w->dtype == E2F_F32) {
    E2F_CUDA_TRY(cudaFuncSetAttribute(project_simt_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
    E2F_LAUNCH(project_simt_kernel<float>, grid, PROJ_THREADS, smem, s, (const float *)x, (int)N, L, C, a);
  } else {
    E2F_CUDA_TRY(cudaFuncSetAttribute(project_simt_kernel<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
    E2F_LAUNCH(project_simt_kernel<__nv_bfloat16>, grid, PROJ_THREADS, smem, s, (const __nv_bfloat16 *)x, (int)N, L, C, a);
  }
  return E2F_OK;
}

}  // namespace e2f
