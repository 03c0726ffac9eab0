// Shared helpers of libe2f: status plumbing, launch accounting, the
// library-owned stream-ordered memory pool and small device utilities.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>

#include "../../include/e2f.h"

namespace e2f {

// ---- host-side bookkeeping (defined in api.cu) -----------------------------
extern std::atomic<int64_t> g_launches;
void set_cuda_error(cudaError_t e, const char *where);
cudaError_t pool_alloc(void **p, size_t bytes, cudaStream_t s);
int *device_error_flag();   // per-device int latched by kernels, or nullptr

#define E2F_CUDA_TRY(expr)                                 \
  do {                                                     \
    cudaError_t e2f_err_ = (expr);                         \
    if (e2f_err_ != cudaSuccess) {                         \
      ::e2f::set_cuda_error(e2f_err_, #expr);              \
      return E2F_ERR_CUDA;                                 \
    }                                                      \
  } while (0)

// Launch + count + check the launch error.
#define E2F_LAUNCH(kernel, grid, block, smem, stream, ...)                 \
  do {                                                                     \
    kernel<<<(grid), (block), (smem), (stream)>>>(__VA_ARGS__);            \
    ::e2f::g_launches.fetch_add(1, std::memory_order_relaxed);             \
    const cudaError_t e2f_lerr_ = cudaGetLastError();                      \
    if (e2f_lerr_ != cudaSuccess) {                                        \
      ::e2f::set_cuda_error(e2f_lerr_, "launch of " #kernel);              \
      return E2F_ERR_CUDA;                                                 \
    }                                                                      \
  } while (0)

// Stream-ordered scratch buffer released (in stream order) on scope exit.
struct Scratch {
  void *p = nullptr;
  cudaStream_t s = nullptr;
  Scratch() = default;
  Scratch(const Scratch &) = delete;
  Scratch &operator=(const Scratch &) = delete;
  cudaError_t alloc(size_t bytes, cudaStream_t st) {
    s = st;
    if (bytes == 0) bytes = 256;
    return pool_alloc(&p, bytes, st);
  }
  template <typename T> T *as() const { return static_cast<T *>(p); }
  ~Scratch() {
    if (p) cudaFreeAsync(p, s);
  }
};

// ---- device utilities ---------------------------------------------------------
__device__ __forceinline__ float to_f(float v) { return v; }
__device__ __forceinline__ float to_f(__nv_bfloat16 v) { return __bfloat162float(v); }
template <typename T> __device__ __forceinline__ T from_f(float v);
template <> __device__ __forceinline__ float from_f<float>(float v) { return v; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float v) {
  return __float2bfloat16_rn(v);
}

// Word i of a 16-byte vector and packing of two floats into a bf16 pair,
// by value (no pointer into a register array is ever formed, so the
// compiler keeps such arrays in registers).
__device__ __forceinline__ uint32_t u4w(const uint4 &v, int i) {
  return i == 0 ? v.x : (i == 1 ? v.y : (i == 2 ? v.z : v.w));
}
// One cvt.rn.bf16x2.f32: the first source goes to the upper half.
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ int warp_sum_i(int v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Exact fp32 neighbour predicate shared by the cell-list kernels: each
// operation rounded to nearest, no fused multiply-add.
struct Geom {
  float box[3];
  float half[3];
  int periodic[3];
  float rc;
  float rc2;
};

__device__ __forceinline__ float min_image_1d(float d, float b, float h, int per) {
  if (per) {
    if (d > h) d = __fsub_rn(d, b);
    else if (d < -h) d = __fadd_rn(d, b);
  }
  return d;
}

__device__ __forceinline__ void pair_disp(const Geom &g, float3 pi, float3 pj, float &dx, float &dy,
                                          float &dz) {
  dx = min_image_1d(__fsub_rn(pj.x, pi.x), g.box[0], g.half[0], g.periodic[0]);
  dy = min_image_1d(__fsub_rn(pj.y, pi.y), g.box[1], g.half[1], g.periodic[1]);
  dz = min_image_1d(__fsub_rn(pj.z, pi.z), g.box[2], g.half[2], g.periodic[2]);
}

__device__ __forceinline__ float pair_r2(float dx, float dy, float dz) {
  return __fadd_rn(__fadd_rn(__fmul_rn(dx, dx), __fmul_rn(dy, dy)), __fmul_rn(dz, dz));
}

// SO(2)-stacked order of one edge's rotated features: the entries of degree
// +-m for l = |m|..L, l-major then channel; m = 0 first, then (+m, -m) for
// m = 1..L.  Offset of the block of +-m:
__host__ __device__ __forceinline__ int stack_off(int L, int C, int m) {
  const int am = m < 0 ? -m : m;
  if (am == 0) return 0;
  int off = (L + 1) * C;
  for (int t = 1; t < am; ++t) off += 2 * (L - t + 1) * C;
  return m > 0 ? off : off + (L - am + 1) * C;
}

// Index of the radial output g_{m,l}: (m, l) pairs in the order m = 0..L,
// then l = m..L.
__host__ __device__ __forceinline__ int pair_index(int L, int m, int l) {
  return m * (L + 1) - m * (m - 1) / 2 + (l - m);
}

__device__ __forceinline__ float3 load_pos(const float *pos, int i) {
  return make_float3(pos[3 * i], pos[3 * i + 1], pos[3 * i + 2]);
}

}  // namespace e2f
