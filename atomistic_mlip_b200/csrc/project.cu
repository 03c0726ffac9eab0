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
// Tensor-core path (bf16, C = 128): persistent CTAs (one per SM, 256
// threads).  A tile is 128 rows (node, m) of one degree l, gathered from x
// into a K-major core-matrix tile in shared memory.  q, k and v of the tile
// come from three tcgen05.mma chains (M = 128, N = 128, K = 128) into three
// 128-column TMEM accumulators, against Wq[l], Wk[l], Wv[l] (out x in, the
// B operands), which stay in shared memory while the CTA's tiles are of
// degree l.  x is read once for all three outputs, and the next tile's rows
// are loaded into registers while the current tile's MMAs and epilogue run.
// The epilogue rounds to bf16 and scatters the rows back to [N][Q][C].
// ---------------------------------------------------------------------------
namespace ptc {
constexpr int CH = 128, TR = 128, NT = 256;
constexpr size_t TILE_BYTES = (size_t)TR * CH * 2;   // one 128 x 128 bf16 tile
constexpr size_t SMEM = 4 * TILE_BYTES + 64;         // Wq, Wk, Wv, rows of x; barrier

__global__ void __launch_bounds__(NT, 1) project_tc_kernel(const __nv_bfloat16 *__restrict__ x, int N, int L,
                                                             ProjArgs a, long long ntiles, int *err) {
  using namespace tc;
  extern __shared__ __align__(1024) uint8_t smem[];
  uint8_t *sW = smem, *sA = smem + 3 * TILE_BYTES;
  uint64_t *bar = reinterpret_cast<uint64_t *>(smem + 4 * TILE_BYTES);
  __shared__ uint32_t tslot;
  const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
  const int Q = (L + 1) * (L + 1);
  const int row = t & (TR - 1), half = t >> 7;   // staging: tile row, 64-channel half
  if (t == 0) { mbar_init(bar, 1); mbar_fence_init(); }
  __syncthreads();
  if (warp == 0) { tmem_alloc(&tslot, 512); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tb = tslot;

  // flat tile index -> degree l and first row r0 of the tile
  auto decode = [&](long long g, int &l, long long &r0) {
    l = 0;
    for (;; ++l) {
      const long long nt = ((long long)N * (2 * l + 1) + TR - 1) / TR;
      if (g < nt || l == L) break;
      g -= nt;
    }
    r0 = g * TR;
  };
  // element offset of row r (node, m) of degree l in x / q / k / v, or -1
  auto row_off = [&](int l, long long r) -> long long {
    const int w = 2 * l + 1;
    if (r >= (long long)N * w) return -1;
    const long long node = r / w;
    return (node * Q + l * l + (r - node * w)) * CH;
  };
  uint4 pre[8];   // this thread's 64 channels of the next tile's row
  auto fetch = [&](long long g) {
    int l;
    long long r0;
    decode(g, l, r0);
    const long long off = row_off(l, r0 + row);
#pragma unroll
    for (int c = 0; c < 8; ++c)
      pre[c] = off >= 0 ? *reinterpret_cast<const uint4 *>(x + off + 64 * half + 8 * c) : make_uint4(0u, 0u, 0u, 0u);
  };

  int cur_l = -1;
  uint32_t phase = 0;
  bool dead = false;
  if ((long long)blockIdx.x < ntiles) fetch(blockIdx.x);
  for (long long g = blockIdx.x; g < ntiles && !dead; g += gridDim.x) {
    int l;
    long long r0;
    decode(g, l, r0);
    // the previous tile's MMAs have completed and its accumulators been read
#pragma unroll
    for (int c = 0; c < 8; ++c) *reinterpret_cast<uint4 *>(sA + kmajor_off(row, 64 * half + 8 * c, CH)) = pre[c];
    if (l != cur_l) {   // this degree's weights
      for (int which = 0; which < 3; ++which) {
        const __nv_bfloat16 *W = static_cast<const __nv_bfloat16 *>(a.W[which][l]);
#pragma unroll
        for (int c = 0; c < 8; ++c)
          *reinterpret_cast<uint4 *>(sW + which * TILE_BYTES + kmajor_off(row, 64 * half + 8 * c, CH)) =
              *reinterpret_cast<const uint4 *>(W + (size_t)row * CH + 64 * half + 8 * c);
      }
      cur_l = l;
    }
    fence_async_smem();
    __syncthreads();
    tc_fence_after();
    if (t == 0) {
      constexpr uint32_t id = idesc_bf16(128, 128, 0, 0);
      const uint32_t a0 = smem_addr(sA), w0 = smem_addr(sW);
#pragma unroll
      for (int which = 0; which < 3; ++which)
#pragma unroll
        for (int kk = 0; kk < CH / 16; ++kk)
          mma_bf16_ss(tb + 128 * which, smem_desc(a0 + kmajor_off(0, 16 * kk, CH), 128, CH * 16),
                      smem_desc(w0 + which * TILE_BYTES + kmajor_off(0, 16 * kk, CH), 128, CH * 16), id, kk > 0);
      mma_commit(bar);
    }
    // the next tile's rows, loaded while the MMAs and the epilogue run
    if (g + gridDim.x < ntiles) fetch(g + gridDim.x);
    const bool ok = mbar_wait(bar, phase, 1u << 26);
    phase ^= 1u;
    dead = __syncthreads_or(!ok) != 0;
    if (dead) {
      if (t == 0) atomicExch(err, E2F_ERR_TIMEOUT);
      break;
    }
    tc_fence_after();
    // epilogue: warp w reads TMEM lanes 32 (w % 4) + [0, 32) (tile rows),
    // channels [64 (w / 4), +64) of each output
    {
      const int erow = 32 * (warp & 3) + lane, ecol = 64 * (warp >> 2);
      const long long off = row_off(l, r0 + erow);
#pragma unroll 1
      for (int which = 0; which < 3; ++which) {
        __nv_bfloat16 *out = static_cast<__nv_bfloat16 *>(a.out[which]);
#pragma unroll 1
        for (int c0 = 0; c0 < 64; c0 += 16) {
          float v[16];
          tmem_ld_32x32b_x16(tb + ((uint32_t)(32 * (warp & 3)) << 16) + 128 * which + ecol + c0, v);
          if (off >= 0) {
            *reinterpret_cast<uint4 *>(out + off + ecol + c0) =
                make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]), pack_bf16x2(v[4], v[5]),
                           pack_bf16x2(v[6], v[7]));
            *reinterpret_cast<uint4 *>(out + off + ecol + c0 + 8) =
                make_uint4(pack_bf16x2(v[8], v[9]), pack_bf16x2(v[10], v[11]), pack_bf16x2(v[12], v[13]),
                           pack_bf16x2(v[14], v[15]));
          }
        }
      }
    }
    tc_fence_before();
    __syncthreads();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tb, 512);
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
    int dev = 0, nsm = 148;
    E2F_CUDA_TRY(cudaGetDevice(&dev));
    E2F_CUDA_TRY(cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev));
    const int grid = (int)std::min<long long>(tiles, nsm);
    E2F_CUDA_TRY(cudaFuncSetAttribute(ptc::project_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      (int)ptc::SMEM));
    E2F_LAUNCH(ptc::project_tc_kernel, grid, ptc::NT, ptc::SMEM, s, (const __nv_bfloat16 *)x, (int)N, L, a,
               tiles, err);
  } else {
    E2F_CUDA_TRY(cudaFuncSetAttribute(project_simt_kernel<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
    E2F_LAUNCH(project_simt_kernel<__nv_bfloat16>, grid, PROJ_THREADS, smem, s, (const __nv_bfloat16 *)x, (int)N, L, C, a);
  }
  return E2F_OK;
}

}  // namespace e2f
