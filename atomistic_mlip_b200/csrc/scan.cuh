// Device-wide exclusive prefix sum of int32 counts (three launches:
// per-tile scan, scan of tile totals, add tile offsets).  out has n + 1
// entries, out[n] = total; `total64` (device, may be null) receives the
// total as int64 so the host can detect int32 overflow.
#pragma once

#include "common.cuh"

namespace e2f {

constexpr int SCAN_THREADS = 1024;
constexpr int SCAN_PER_THREAD = 4;
constexpr int SCAN_TILE = SCAN_THREADS * SCAN_PER_THREAD;

__device__ __forceinline__ long long block_exclusive_scan(long long v, long long *warp_tot,
                                                          long long *block_total) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  long long incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    long long t = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += t;
  }
  if (lane == 31) warp_tot[wid] = incl;
  __syncthreads();
  if (wid == 0) {
    const int nw = blockDim.x >> 5;
    long long w = lane < nw ? warp_tot[lane] : 0;
    long long wi = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      long long t = __shfl_up_sync(0xffffffffu, wi, o);
      if (lane >= o) wi += t;
    }
    if (lane < nw) warp_tot[lane] = wi - w;
    if (lane == nw - 1) *block_total = wi;
  }
  __syncthreads();
  long long r = incl - v + warp_tot[wid];
  __syncthreads();
  return r;
}

// Tile-local exclusive scan; tile totals to `sums`.
__global__ void scan_tiles_kernel(const int32_t *__restrict__ in, int64_t n, int32_t *__restrict__ out,
                                  long long *__restrict__ sums) {
  __shared__ long long wt[32];
  __shared__ long long tot;
  const int64_t base = (int64_t)blockIdx.x * SCAN_TILE + (int64_t)threadIdx.x * SCAN_PER_THREAD;
  long long vals[SCAN_PER_THREAD];
  long long s = 0;
#pragma unroll
  for (int k = 0; k < SCAN_PER_THREAD; ++k) {
    vals[k] = (base + k < n) ? (long long)in[base + k] : 0;
    s += vals[k];
  }
  long long ex = block_exclusive_scan(s, wt, &tot);
#pragma unroll
  for (int k = 0; k < SCAN_PER_THREAD; ++k) {
    if (base + k < n) out[base + k] = (int32_t)ex;   // tile-local, fixed up later
    ex += vals[k];
  }
  if (threadIdx.x == 0) sums[blockIdx.x] = tot;
}

// Exclusive scan of the tile totals (single block, loops over chunks).
__global__ void scan_sums_kernel(long long *__restrict__ sums, int64_t ntiles,
                                 long long *__restrict__ total) {
  __shared__ long long wt[32];
  __shared__ long long tot;
  long long carry = 0;
  for (int64_t b = 0; b < ntiles; b += blockDim.x) {
    int64_t i = b + threadIdx.x;
    long long v = i < ntiles ? sums[i] : 0;
    long long ex = block_exclusive_scan(v, wt, &tot);
    if (i < ntiles) sums[i] = ex + carry;
    carry += tot;
    __syncthreads();
  }
  if (threadIdx.x == 0) *total = carry;
}

__global__ void scan_add_kernel(int32_t *__restrict__ out, int64_t n, const long long *__restrict__ sums,
                                const long long *__restrict__ total) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) out[i] = (int32_t)((long long)out[i] + sums[i / SCAN_TILE]);
  if (i == n) out[n] = (int32_t)(*total);
}

// Scratch needed by exclusive_scan: (ntiles + 1) long longs.
inline size_t scan_scratch_bytes(int64_t n) {
  int64_t ntiles = (n + SCAN_TILE - 1) / SCAN_TILE;
  return (size_t)(ntiles + 1) * sizeof(long long);
}

// `scratch` must hold scan_scratch_bytes(n); the int64 total lands in
// ((long long*)scratch)[ntiles].
inline e2f_status exclusive_scan(const int32_t *in, int64_t n, int32_t *out, void *scratch,
                                 cudaStream_t s, long long **total_out) {
  int64_t ntiles = (n + SCAN_TILE - 1) / SCAN_TILE;
  long long *sums = static_cast<long long *>(scratch);
  long long *total = sums + ntiles;
  if (ntiles > 0) {
    E2F_LAUNCH(scan_tiles_kernel, (unsigned)ntiles, SCAN_THREADS, 0, s, in, n, out, sums);
  }
  E2F_LAUNCH(scan_sums_kernel, 1, SCAN_THREADS, 0, s, sums, ntiles, total);
  E2F_LAUNCH(scan_add_kernel, (unsigned)((n + 1 + 255) / 256), 256, 0, s, out, n, sums, total);
  if (total_out) *total_out = total;
  return E2F_OK;
}

}  // namespace e2f
