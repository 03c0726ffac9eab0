// The E2Former-V2 block around the attention: merged equivariant RMS layer
// norm ("EquiformerV3 ...", technical summary §2B.1: one RMS statistic shared
// by all degrees), a node FFN with hidden width Hd and a scalar SwiGLU gate
// (§2B.2, §2C: the non-linear gate acts on the l = 0 features only), and the
// pre-norm residual connections:
//
//   x1 = x + Attn(Norm1(x)),   x2 = x1 + FFN(Norm2(x1)),
//   Norm(x)[n,(l,m),c] = gamma[l][c] x[n,(l,m),c] / sqrt(mean_{l,m,c} x^2 + 1e-6),
//   FFN(y)[n,(l,m)]    = Wd[l] (SiLU(Wa y[n,(0,0)]) * (Wb[l] y[n,(l,m)])).
//
// Kernels:
//   rms_norm_kernel      one warp per node: optional residual sum x + a
//                        (written out), the node's mean square, the scaled
//                        features in the storage type.  HBM-bound.
//   dgemm_tc_kernel      per-degree GEMM on the tensor cores (bf16, fp32
//                        accumulation): rows (node, m) of one degree l times
//                        W[l]^T, with one of three epilogues -- SiLU (the
//                        gate), multiply by the node's gate (the hidden
//                        features), add into the fp32 residual stream.  The
//                        degree's weight matrix stays in shared memory while
//                        the CTA's tiles are of that degree; rows stream in
//                        K-chunks of 128 through two buffers.
//   dgemm_simt_kernel    the same GEMM and epilogues on CUDA cores (fp32
//                        storage, or widths the tensor-core path does not
//                        take).
#include <algorithm>

#include "common.cuh"
#include "tc_common.cuh"

namespace e2f {

e2f_status attention_forward_impl(const void *x, const float *pos, const e2f_csr *csr, const e2f_weights *w,
                                  float *out, cudaStream_t s, int F = 1, const float *focus_a = nullptr);

namespace blk {

constexpr float RMS_EPS = 1e-6f;
constexpr int EPI_SILU = 0;    // out (fp32) = SiLU(acc)
constexpr int EPI_GATE = 1;    // out (storage type) = acc * gate[node][col]
constexpr int EPI_RESID = 2;   // out (fp32) += acc

__device__ __forceinline__ int degree_of(int q) {
  int l = (int)sqrtf((float)q);
  while (l * l > q) --l;
  while ((l + 1) * (l + 1) <= q) ++l;
  return l;
}

__device__ __forceinline__ void store4(float *p, float a, float b, float c, float d) {
  *reinterpret_cast<float4 *>(p) = make_float4(a, b, c, d);
}
__device__ __forceinline__ void store4(__nv_bfloat16 *p, float a, float b, float c, float d) {
  *reinterpret_cast<uint2 *>(p) = make_uint2(pack_bf16x2(a, b), pack_bf16x2(c, d));
}

// ---------------------------------------------------------------------------
// merged RMS norm: one warp per node
// ---------------------------------------------------------------------------
template <typename TOUT>
__global__ void __launch_bounds__(256) rms_norm_kernel(const float *__restrict__ x, const float *__restrict__ add,
                                                       float *__restrict__ x1, const float *__restrict__ gamma,
                                                       int N, int L, int C, TOUT *__restrict__ out, bool vec) {
  const int lane = threadIdx.x & 31;
  const int Q = (L + 1) * (L + 1), QC = Q * C;
  if (vec) {
    // C a multiple of 4, every pointer 16-byte aligned: rows (l, m) of four
    // channels per lane, the degree found once per row
    const int C4 = C >> 2;
    for (int n = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); n < N; n += gridDim.x * (blockDim.x >> 5)) {
      const size_t nb = (size_t)n * QC;
      float ss = 0.f;
      for (int q = 0; q < Q; ++q)
        for (int c4 = lane; c4 < C4; c4 += 32) {
          const size_t o = nb + (size_t)q * C + 4 * c4;
          float4 v = *reinterpret_cast<const float4 *>(x + o);
          if (add) {
            const float4 t = *reinterpret_cast<const float4 *>(add + o);
            v.x += t.x; v.y += t.y; v.z += t.z; v.w += t.w;
            *reinterpret_cast<float4 *>(x1 + o) = v;
          }
          ss = fmaf(v.x, v.x, fmaf(v.y, v.y, fmaf(v.z, v.z, fmaf(v.w, v.w, ss))));
        }
      ss = warp_sum(ss);
      const float inv = 1.f / sqrtf(ss / (float)QC + RMS_EPS);
      const float *vr = add ? x1 : x;   // this lane wrote the x1 entries it reads back
      int l = 0;
      for (int q = 0; q < Q; ++q) {
        if ((l + 1) * (l + 1) <= q) ++l;
        for (int c4 = lane; c4 < C4; c4 += 32) {
          const size_t o = nb + (size_t)q * C + 4 * c4;
          const float4 v = *reinterpret_cast<const float4 *>(vr + o);
          const float *gr = gamma + l * C + 4 * c4;
          store4(out + o, gr[0] * v.x * inv, gr[1] * v.y * inv, gr[2] * v.z * inv, gr[3] * v.w * inv);
        }
      }
    }
    return;
  }
  for (int n = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); n < N; n += gridDim.x * (blockDim.x >> 5)) {
    const float *xr = x + (size_t)n * QC;
    const float *ar = add ? add + (size_t)n * QC : nullptr;
    float ss = 0.f;
    for (int i = lane; i < QC; i += 32) {
      float v = xr[i];
      if (ar) {
        v += ar[i];
        x1[(size_t)n * QC + i] = v;
      }
      ss = fmaf(v, v, ss);
    }
    ss = warp_sum(ss);
    const float inv = 1.f / sqrtf(ss / (float)QC + RMS_EPS);
    const float *vr = ar ? x1 + (size_t)n * QC : xr;
    for (int i = lane; i < QC; i += 32) {
      const int q = i / C, c = i - q * C;
      out[(size_t)n * QC + i] = from_f<TOUT>(gamma[degree_of(q) * C + c] * vr[i] * inv);
    }
  }
}

// ---------------------------------------------------------------------------
// per-degree GEMM: for the rows r = (node, m) of degree l in [l_lo, l_hi],
// acc[r][o] = sum_k A[node][l^2 + m][k] W[l][o][k]; A has a_q rows per node
// and K columns, out has out_q rows per node and Nout columns.
// ---------------------------------------------------------------------------
struct DG {
  const void *A;
  int a_q, K;
  const void *W[E2F_MAX_L + 1];
  void *out;
  int out_q, Nout;
  const float *gate;   // [N][Nout] fp32 (EPI_GATE)
  int N, l_lo, l_hi;
};

__device__ __forceinline__ float silu(float z) { return z / (1.f + expf(-z)); }

template <typename T, int EPI>
__device__ __forceinline__ void epi_store(const DG &a, long long node, int l, int m, int o, float acc) {
  const size_t oi = ((size_t)node * a.out_q + l * l + m) * a.Nout + o;
  if (EPI == EPI_SILU) {
    static_cast<float *>(a.out)[oi] = silu(acc);
  } else if (EPI == EPI_GATE) {
    static_cast<T *>(a.out)[oi] = from_f<T>(acc * a.gate[(size_t)node * a.Nout + o]);
  } else {
    static_cast<float *>(a.out)[oi] += acc;
  }
}

constexpr int SG_THREADS = 256;
constexpr int SG_ROWS = 16;

// CUDA-core form: a block takes SG_ROWS rows of one degree (blockIdx.y) and
// all output columns; the rows are staged in shared memory in fp32.
template <typename T, int EPI>
__global__ void __launch_bounds__(SG_THREADS) dgemm_simt_kernel(DG a) {
  extern __shared__ float sx[];   // [SG_ROWS][K]
  const int l = a.l_lo + blockIdx.y, w = 2 * l + 1;
  const long long rows = (long long)a.N * w;
  const T *W = static_cast<const T *>(a.W[l]);
  const T *A = static_cast<const T *>(a.A);
  for (long long r0 = (long long)blockIdx.x * SG_ROWS; r0 < rows; r0 += (long long)gridDim.x * SG_ROWS) {
    const int nr = (int)(rows - r0 < SG_ROWS ? rows - r0 : SG_ROWS);
    __syncthreads();
    for (int idx = threadIdx.x; idx < nr * a.K; idx += blockDim.x) {
      const long long r = r0 + idx / a.K;
      const int k = idx % a.K;
      const long long node = r / w;
      sx[idx] = to_f(A[((size_t)node * a.a_q + l * l + (int)(r - node * w)) * a.K + k]);
    }
    __syncthreads();
    for (int idx = threadIdx.x; idx < nr * a.Nout; idx += blockDim.x) {
      const int rr = idx / a.Nout, o = idx % a.Nout;
      const float *xr = sx + (size_t)rr * a.K;
      const T *wr = W + (size_t)o * a.K;
      float acc = 0.f;
      for (int k = 0; k < a.K; ++k) acc = fmaf(to_f(wr[k]), xr[k], acc);
      const long long r = r0 + rr, node = r / w;
      epi_store<T, EPI>(a, node, l, (int)(r - node * w), o, acc);
    }
  }
}

// ---------------------------------------------------------------------------
// tensor-core form (bf16, K and Nout multiples of 128, Nout K <= 65536)
// ---------------------------------------------------------------------------
constexpr int TR = 128, NT = 256, KC = 128;
constexpr size_t A_BYTES = (size_t)TR * KC * 2;    // one 128 x 128 bf16 chunk of rows
constexpr size_t W_BYTES = 65536 * 2;              // resident weights of one degree
constexpr size_t TC_SMEM = W_BYTES + 2 * A_BYTES + 64;

template <int EPI>
__global__ void __launch_bounds__(NT, 1) dgemm_tc_kernel(DG a, long long ntiles, int *err) {
  using namespace tc;
  extern __shared__ __align__(1024) uint8_t smem[];
  uint8_t *sW = smem, *sA = smem + W_BYTES;
  uint64_t *bar = reinterpret_cast<uint64_t *>(smem + W_BYTES + 2 * A_BYTES);
  __shared__ uint32_t tslot;
  const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
  const int row = t & (TR - 1), half = t >> 7;   // staging: chunk row, 64-column half of the K chunk
  const int K = a.K, Nout = a.Nout, nkc = K / KC;
  if (t == 0) { mbar_init(bar, 1); mbar_fence_init(); }
  __syncthreads();
  if (warp == 0) { tmem_alloc(&tslot, 512); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tb = tslot;
  const __nv_bfloat16 *A = static_cast<const __nv_bfloat16 *>(a.A);

  auto decode = [&](long long g, int &l, long long &r0) {
    l = a.l_lo;
    for (;; ++l) {
      const long long nt = ((long long)a.N * (2 * l + 1) + TR - 1) / TR;
      if (g < nt || l == a.l_hi) break;
      g -= nt;
    }
    r0 = g * TR;
  };
  auto a_off = [&](int l, long long r) -> long long {   // element offset of row r of degree l, or -1
    const int w = 2 * l + 1;
    if (r >= (long long)a.N * w) return -1;
    const long long node = r / w;
    return ((size_t)node * a.a_q + l * l + (r - node * w)) * (size_t)K;
  };
  uint4 pre[8];   // this thread's 64 columns of the next K chunk
  auto fetch = [&](long long g, int kc) {
    int l;
    long long r0;
    decode(g, l, r0);
    const long long off = a_off(l, r0 + row);
#pragma unroll
    for (int c = 0; c < 8; ++c)
      pre[c] = off >= 0 ? *reinterpret_cast<const uint4 *>(A + off + kc * KC + 64 * half + 8 * c)
                        : make_uint4(0u, 0u, 0u, 0u);
  };

  int cur_l = -1;
  uint32_t phase = 0;
  bool dead = false;
  if ((long long)blockIdx.x < ntiles) fetch(blockIdx.x, 0);
  for (long long g = blockIdx.x; g < ntiles && !dead; g += gridDim.x) {
    int l;
    long long r0;
    decode(g, l, r0);
    for (int kc = 0; kc < nkc && !dead; ++kc) {
      uint8_t *buf = sA + (kc & 1) * A_BYTES;
#pragma unroll
      for (int c = 0; c < 8; ++c) *reinterpret_cast<uint4 *>(buf + kmajor_off(row, 64 * half + 8 * c, KC)) = pre[c];
      if (l != cur_l) {   // this degree's weights: [Nout][K], K-major core matrices, Kc = K
        const __nv_bfloat16 *W = static_cast<const __nv_bfloat16 *>(a.W[l]);
        for (int idx = t; idx < Nout * (K / 8); idx += NT) {
          const int o = idx / (K / 8), k8 = (idx % (K / 8)) * 8;
          *reinterpret_cast<uint4 *>(sW + kmajor_off(o, k8, K)) = *reinterpret_cast<const uint4 *>(W + (size_t)o * K + k8);
        }
        cur_l = l;
      }
      fence_async_smem();
      __syncthreads();
      tc_fence_after();
      if (t == 0) {
        constexpr uint32_t id = idesc_bf16(128, 128, 0, 0);
        const uint32_t a0 = smem_addr(buf), w0 = smem_addr(sW);
        for (int nc = 0; nc < Nout / 128; ++nc)
#pragma unroll
          for (int kk = 0; kk < KC / 16; ++kk)
            mma_bf16_ss(tb + 128 * nc, smem_desc(a0 + kmajor_off(0, 16 * kk, KC), 128, KC * 16),
                        smem_desc(w0 + kmajor_off(128 * nc, kc * KC + 16 * kk, K), 128, (uint32_t)K * 16), id,
                        (kc > 0 || kk > 0) ? 1u : 0u);
        mma_commit(bar);
      }
      // the next chunk's rows (this tile's, or the next tile's first), loaded
      // while the MMAs run
      if (kc + 1 < nkc) fetch(g, kc + 1);
      else if (g + gridDim.x < ntiles) fetch(g + gridDim.x, 0);
      const bool ok = mbar_wait(bar, phase, 1u << 26);
      phase ^= 1u;
      dead = __syncthreads_or(!ok) != 0;
      if (dead && t == 0) atomicExch(err, E2F_ERR_TIMEOUT);
    }
    if (dead) break;
    tc_fence_after();
    // epilogue: warp w reads TMEM lanes 32 (w % 4) + [0, 32) (tile rows),
    // columns [Nout/2 (w / 4), +Nout/2)
    {
      const int erow = 32 * (warp & 3) + lane;
      const int w2 = 2 * l + 1;
      const long long r = r0 + erow;
      const bool live = r < (long long)a.N * w2;
      const long long node = r / w2;
      const int m = (int)(r - node * w2);
      const int cb = (Nout / 2) * (warp >> 2);
#pragma unroll 1
      for (int c0 = 0; c0 < Nout / 2; c0 += 16) {
        float v[16];
        tmem_ld_32x32b_x16(tb + ((uint32_t)(32 * (warp & 3)) << 16) + cb + c0, v);
        if (live) {
          const size_t oi = ((size_t)node * a.out_q + l * l + m) * Nout + cb + c0;
          if (EPI == EPI_SILU) {
            float4 *o4 = reinterpret_cast<float4 *>(static_cast<float *>(a.out) + oi);
#pragma unroll
            for (int i = 0; i < 4; ++i)
              o4[i] = make_float4(silu(v[4 * i]), silu(v[4 * i + 1]), silu(v[4 * i + 2]), silu(v[4 * i + 3]));
          } else if (EPI == EPI_GATE) {
            const float4 *g4 = reinterpret_cast<const float4 *>(a.gate + (size_t)node * Nout + cb + c0);
            uint32_t w[8];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const float4 gg = g4[i];
              w[2 * i] = pack_bf16x2(v[4 * i] * gg.x, v[4 * i + 1] * gg.y);
              w[2 * i + 1] = pack_bf16x2(v[4 * i + 2] * gg.z, v[4 * i + 3] * gg.w);
            }
            __nv_bfloat16 *op = static_cast<__nv_bfloat16 *>(a.out) + oi;
            *reinterpret_cast<uint4 *>(op) = make_uint4(w[0], w[1], w[2], w[3]);
            *reinterpret_cast<uint4 *>(op + 8) = make_uint4(w[4], w[5], w[6], w[7]);
          } else {
            float4 *o4 = reinterpret_cast<float4 *>(static_cast<float *>(a.out) + oi);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              float4 cur = o4[i];
              cur.x += v[4 * i]; cur.y += v[4 * i + 1]; cur.z += v[4 * i + 2]; cur.w += v[4 * i + 3];
              o4[i] = cur;
            }
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

static bool tc_shape(const DG &a, int dtype) {
  return dtype == E2F_BF16 && a.K % KC == 0 && a.Nout % 128 == 0 && (long long)a.K * a.Nout <= 65536 &&
         a.Nout <= 512;
}

template <int EPI>
static e2f_status run_gemm(const DG &a, int dtype, cudaStream_t s) {
  if (a.N == 0) return E2F_OK;
  if (tc_shape(a, dtype)) {
    long long tiles = 0;
    for (int l = a.l_lo; l <= a.l_hi; ++l) tiles += ((long long)a.N * (2 * l + 1) + TR - 1) / TR;
    int *err = device_error_flag();
    if (!err) return E2F_ERR_CUDA;
    int dev = 0, nsm = 148;
    E2F_CUDA_TRY(cudaGetDevice(&dev));
    E2F_CUDA_TRY(cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev));
    const int grid = (int)std::min<long long>(tiles, nsm);
    E2F_CUDA_TRY(cudaFuncSetAttribute(dgemm_tc_kernel<EPI>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)TC_SMEM));
    E2F_LAUNCH(dgemm_tc_kernel<EPI>, grid, NT, TC_SMEM, s, a, tiles, err);
    return E2F_OK;
  }
  const size_t smem = sizeof(float) * (size_t)SG_ROWS * a.K;
  if (smem > 200 * 1024) return E2F_ERR_UNSUPPORTED;
  const long long rows_max = (long long)a.N * (2 * a.l_hi + 1);
  dim3 grid((unsigned)std::min<long long>(std::max<long long>(1, (rows_max + SG_ROWS - 1) / SG_ROWS), 4096),
            a.l_hi - a.l_lo + 1);
  if (dtype == E2F_F32) {
    E2F_CUDA_TRY(cudaFuncSetAttribute(dgemm_simt_kernel<float, EPI>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
    E2F_LAUNCH((dgemm_simt_kernel<float, EPI>), grid, SG_THREADS, smem, s, a);
  } else {
    E2F_CUDA_TRY(cudaFuncSetAttribute(dgemm_simt_kernel<__nv_bfloat16, EPI>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      (int)smem));
    E2F_LAUNCH((dgemm_simt_kernel<__nv_bfloat16, EPI>), grid, SG_THREADS, smem, s, a);
  }
  return E2F_OK;
}

template <typename TOUT>
static e2f_status run_norm(const float *x, const float *add, float *x1, const float *gamma, int N, int L, int C,
                           TOUT *out, cudaStream_t s) {
  if (N == 0) return E2F_OK;
  const int grid = (int)std::min<long long>((N + 7) / 8, 148LL * 16);
  auto al16 = [](const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; };
  const bool vec = (C & 3) == 0 && al16(x) && al16(add) && al16(x1) && al16(out);
  E2F_LAUNCH(rms_norm_kernel<TOUT>, grid, 256, 0, s, x, add, x1, gamma, N, L, C, out, vec);
  return E2F_OK;
}

}  // namespace blk

// ---------------------------------------------------------------------------
// one block: x (fp32) -> out (fp32)
// ---------------------------------------------------------------------------
e2f_status block_forward_impl(const float *x, const float *pos, const e2f_csr *csr, const e2f_block_weights *w,
                              float *out, cudaStream_t s) {
  using namespace blk;
  const e2f_weights &aw = w->attn;
  const int L = aw.L_max, C = aw.C, Hd = w->hidden;
  const int64_t N = csr->n_nodes;
  const size_t Q = (size_t)(L + 1) * (L + 1);
  const size_t esz = aw.dtype == E2F_F32 ? 4 : 2;
  const size_t feat = (size_t)N * Q * C;
  auto up = [](size_t b) { return (b + 255) & ~(size_t)255; };
  const size_t o_xn = 0, o_att = up(feat * esz), o_gate = o_att + up(feat * 4),
               o_h = o_gate + up((size_t)N * Hd * 4);
  Scratch ws;
  E2F_CUDA_TRY(ws.alloc(o_h + (size_t)N * Q * Hd * esz, s));
  char *wb = ws.as<char>();
  void *xn = wb + o_xn;                                      // normalised features (storage type)
  float *att = reinterpret_cast<float *>(wb + o_att);        // attention output
  float *gate = reinterpret_cast<float *>(wb + o_gate);      // SiLU(Wa y_0), fp32 [N][Hd]
  void *h = wb + o_h;                                        // gated hidden features [N][Q][Hd]
  const bool f32 = aw.dtype == E2F_F32;
  e2f_status st;
  // x1 = x + Attn(Norm1(x))
  st = f32 ? run_norm<float>(x, nullptr, nullptr, w->gamma1, (int)N, L, C, (float *)xn, s)
           : run_norm<__nv_bfloat16>(x, nullptr, nullptr, w->gamma1, (int)N, L, C, (__nv_bfloat16 *)xn, s);
  if (st != E2F_OK) return st;
  st = attention_forward_impl(xn, pos, csr, &aw, att, s);
  if (st != E2F_OK) return st;
  // out = x1 = x + att;  xn = Norm2(x1)
  st = f32 ? run_norm<float>(x, att, out, w->gamma2, (int)N, L, C, (float *)xn, s)
           : run_norm<__nv_bfloat16>(x, att, out, w->gamma2, (int)N, L, C, (__nv_bfloat16 *)xn, s);
  if (st != E2F_OK) return st;
  // gate = SiLU(Wa y_0);  h = gate * (Wb[l] y);  out += Wd[l] h
  DG g{};
  g.A = xn; g.a_q = (int)Q; g.K = C; g.W[0] = w->Wa; g.out = gate; g.out_q = 1; g.Nout = Hd; g.gate = nullptr;
  g.N = (int)N; g.l_lo = 0; g.l_hi = 0;
  st = run_gemm<EPI_SILU>(g, aw.dtype, s);
  if (st != E2F_OK) return st;
  DG u{};
  u.A = xn; u.a_q = (int)Q; u.K = C; u.out = h; u.out_q = (int)Q; u.Nout = Hd; u.gate = gate;
  u.N = (int)N; u.l_lo = 0; u.l_hi = L;
  for (int l = 0; l <= L; ++l) u.W[l] = w->Wb[l];
  st = run_gemm<EPI_GATE>(u, aw.dtype, s);
  if (st != E2F_OK) return st;
  DG d{};
  d.A = h; d.a_q = (int)Q; d.K = Hd; d.out = out; d.out_q = (int)Q; d.Nout = C; d.gate = nullptr;
  d.N = (int)N; d.l_lo = 0; d.l_hi = L;
  for (int l = 0; l <= L; ++l) d.W[l] = w->Wd[l];
  return run_gemm<EPI_RESID>(d, aw.dtype, s);
}

}  // namespace e2f
