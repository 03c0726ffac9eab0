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
#include "tc_common.cuh"

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

// ---------------------------------------------------------------------------
// Tensor-core path (bf16, C = 128): one CTA per (128-row tile of one degree,
// which of q / k / v).  Rows (node, m) of degree l are gathered from x into a
// K-major core-matrix tile in shared memory; W[l] (out x in, already K-major)
// is the B operand; one tcgen05.mma chain M = 128, N = 128, K = 128 into a
// 128-column TMEM accumulator; the epilogue rounds to bf16 and scatters the
// rows back to [N][Q][C].
// ---------------------------------------------------------------------------
namespace ptc {
constexpr int CH = 128, TR = 128;
constexpr size_t SMEM = 2 * (size_t)TR * CH * 2 + 16;

__global__ void __launch_bounds__(128) project_tc_kernel(const __nv_bfloat16 *__restrict__ x, int N, int L,
                                                          ProjArgs a, int *err) {
  using namespace tc;
  extern __shared__ __align__(1024) uint8_t smem[];
  uint8_t *sA = smem, *sB = smem + TR * CH * 2;
  uint64_t *bar = reinterpret_cast<uint64_t *>(smem + 2 * TR * CH * 2);
  __shared__ uint32_t tslot;
  const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
  const int Q = (L + 1) * (L + 1);
  // decode (degree, tile) from the flat tile index
  int l = 0;
  long long tile = blockIdx.x;
  for (;; ++l) {
    const long long nt = ((long long)N * (2 * l + 1) + TR - 1) / TR;
    if (tile < nt || l == L) break;
    tile -= nt;
  }
  const int w = 2 * l + 1;
  const long long rows = (long long)N * w;
  const int which = blockIdx.y;
  const __nv_bfloat16 *W = static_cast<const __nv_bfloat16 *>(a.W[which][l]);
  __nv_bfloat16 *out = static_cast<__nv_bfloat16 *>(a.out[which]);
  // gather: thread t owns row t of A and row t of B
  const long long r = tile * TR + t;
  const bool valid = r < rows;
  long long off = 0;
  if (valid) {
    const long long node = r / w;
    off = (node * Q + l * l + (r - node * w)) * CH;
  }
#pragma unroll
  for (int c = 0; c < CH / 8; ++c) {
    uint4 va = make_uint4(0, 0, 0, 0);
    if (valid) va = *reinterpret_cast<const uint4 *>(x + off + 8 * c);
    *reinterpret_cast<uint4 *>(sA + kmajor_off(t, 8 * c, CH)) = va;
    *reinterpret_cast<uint4 *>(sB + kmajor_off(t, 8 * c, CH)) =
        *reinterpret_cast<const uint4 *>(W + (size_t)t * CH + 8 * c);
  }
  if (t == 0) { mbar_init(bar, 1); mbar_fence_init(); }
  fence_async_smem();
  __syncthreads();
  if (warp == 0) { tmem_alloc(&tslot, 128); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tb = tslot;
  if (t == 0) {
    constexpr uint32_t id = idesc_bf16(128, 128, 0, 0);
    const uint32_t a0 = smem_addr(sA), b0 = smem_addr(sB);
#pragma unroll
    for (int kk = 0; kk < CH / 16; ++kk)
      mma_bf16_ss(tb, smem_desc(a0 + kmajor_off(0, 16 * kk, CH), 128, CH * 16),
                  smem_desc(b0 + kmajor_off(0, 16 * kk, CH), 128, CH * 16), id, kk > 0);
    mma_commit(bar);
  }
  __syncwarp();
  const bool ok = mbar_wait(bar, 0, 1u << 26);
  if (!ok && lane == 0) atomicExch(err, E2F_ERR_TIMEOUT);
  tc_fence_after();
  if (ok) {
#pragma unroll 1
    for (int c0 = 0; c0 < CH; c0 += 16) {
      float v[16];
      tmem_ld_32x32b_x16(tb + ((uint32_t)(32 * warp) << 16) + c0, v);
      tmem_ld_wait();
      if (valid) {
        __align__(16) __nv_bfloat16 o[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) o[i] = __float2bfloat16_rn(v[i]);
        *reinterpret_cast<uint4 *>(out + off + c0) = *reinterpret_cast<const uint4 *>(&o[0]);
        *reinterpret_cast<uint4 *>(out + off + c0 + 8) = *reinterpret_cast<const uint4 *>(&o[8]);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tb, 128);
}
}  // namespace ptc

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
  } else if (C == ptc::CH) {
    long long tiles = 0;
    for (int l = 0; l <= L; ++l) tiles += (N * (2LL * l + 1) + ptc::TR - 1) / ptc::TR;
    int *err = device_error_flag();
    if (!err) return E2F_ERR_CUDA;
    E2F_CUDA_TRY(cudaFuncSetAttribute(ptc::project_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      (int)ptc::SMEM));
    E2F_LAUNCH(ptc::project_tc_kernel, dim3((unsigned)tiles, 3), 128, ptc::SMEM, s, (const __nv_bfloat16 *)x,
               (int)N, L, a, err);
  } else {
    E2F_CUDA_TRY(cudaFuncSetAttribute(project_simt_kernel<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
    E2F_LAUNCH(project_simt_kernel<__nv_bfloat16>, grid, PROJ_THREADS, smem, s, (const __nv_bfloat16 *)x, (int)N, L, C, a);
  }
  return E2F_OK;
}

}  // namespace e2f
