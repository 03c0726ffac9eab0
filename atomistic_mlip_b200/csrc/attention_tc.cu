// Fused on-the-fly equivariant attention on the tensor cores (tcgen05/TMEM).
//
// What it computes is the operator of e2f_attention_forward ("E2Former-V2
// ...", §2.1 EAAS change of basis, §2.2 node-centric streaming with no edge
// materialisation; "EquiformerV3 ...", §2B.3 envelope in the softmax).
//
// Structure (one persistent CTA per SM, 512 threads; CTA b owns the nodes
// whose rows start in its share of the edges, so no node is split between
// CTAs; tiles of <= 64 edges (32 for L = 5, 6) covering <= 4 destination
// nodes):
//
//   producers (warps 8-15)  per tile: edge geometry, Wigner blocks of the
//                           y-rotation in the two-angle frame (parity blocks),
//                           envelope, radial MLP, logits, and the online-
//                           softmax statistics of the tile (per node and head:
//                           the node's reference maximum, alpha, the factor
//                           for its earlier sums, the running denominator);
//                           then, block by block, the rotated neighbour
//                           features v~ = D v_j written as bf16 MMA operands
//                           (one 64 x 128 "unit" per (degree, +-m)).
//   loaders (warps 1-2)     stream pre-packed weight tiles (Wr|Wi, or W0)
//                           from L2 with 1-D bulk copies.
//   MMA (warp 0)            SO(2) block products as tcgen05.mma (M = 64
//                           edges, N = 128 channels of one output degree,
//                           K streamed over the block's units), complex form:
//                           y+ += v+ Wr^T - v- Wi^T,  y- += v- Wr^T + v+ Wi^T,
//                           y+ / y- accumulate in the two lane halves of a TMEM
//                           buffer.
//   back-rotation (warp 3)  the back-rotation + per-node sum as a second GEMM
//                           per (l, +-m) group, issued as soon as the epilogue
//                           hands it over:
//                           Out_l[c, (slot, m')] += sum_e A[c, e] R[(slot,m'), e]
//                           with A = alpha g y (bf16) and R = D^l[+-m][m'].
//   epilogue (warps 4-7)    TMEM y -> A (scaled bf16, shared memory), builds R;
//                           at tile end, finished nodes' Out columns / the
//                           denominator -> o_i, and the continuing node's
//                           columns rescaled when its reference maximum moved.
//
// All waits are bounded; a timeout raises a CTA-wide abort flag and the
// device error word (E2F_ERR_TIMEOUT) and every role exits its loops.
#include <algorithm>
#include <mutex>
#include <type_traits>
#include <utility>

#include "common.cuh"
#include "tc_common.cuh"
#include "wigner.cuh"

namespace e2f {
namespace tca {

using namespace tc;

constexpr int CH = 128;            // channels on this path
constexpr int TE64 = 64;           // edges per tile for L <= 4 (MMA M)
constexpr int S = 4;               // destination-node slots per tile
constexpr int NSTAGE = 2;          // weight ring stages
constexpr int STAGE_BYTES = 32768; // one weight stage: W0 128 x 128, or Wr|Wi 128 x 64 each
constexpr int NTHREADS = 512;
constexpr int HMAX = 16;
constexpr int ALS = HMAX + 1;     // alpha row stride (odd: conflict-free per-edge rows)
constexpr uint32_t WAIT_LIMIT = 1u << 25;
// online softmax: how far (in logit units) a node's later tiles may exceed
// its reference maximum before the reference moves; alpha = e^(s - M) then
// stays below e^8 (< 3000, exact range of the fp16 alpha store)
constexpr float SOFTMAX_MARGIN = 8.f;
// TMEM columns: [0, 256) two y buffers (y+ in lanes 0-15, y- in lanes 16-31 of
// each 32-lane subpartition), [256, 256 + OUT_COLS) the per-node output sums,
// [384, 512) one rotated-feature unit pair used as the MMA A operand.
constexpr uint32_t TM_OUT = 256;
constexpr uint32_t TM_UNIT = 384;

template <int L> struct Cfg {
  // Tile edges: 64 up to L = 4; 32 for L = 5, 6, where the SO(2) units of
  // one degree m would not fit otherwise.  With 32 edges the M = 64 MMA reads
  // its rows 32..63 from the next unit (units are contiguous), whose rows of
  // D are never used.
  static constexpr int TE = L >= 5 ? 32 : TE64;
  static constexpr int UNIT_BYTES = TE * CH * 2;
  static constexpr int A2_BYTES = CH * TE * 2;
  static constexpr int Q = (L + 1) * (L + 1);
  static constexpr int P = (L + 1) * (L + 2) / 2;
  static constexpr int NUNIT = (L + 1 > 2 * L) ? L + 1 : 2 * L;
  // From L = 3 on, the unit pair of (m = 1, l' = L) lives in TMEM: those two
  // units are used by the m = 1 passes only, and shared memory is tight.
  static constexpr bool TMU = (L == 3 || L == 4);
  static constexpr int TMU_SP = 2 * L - 2;                 // first TMEM unit index
  static constexpr int NSU = TMU ? NUNIT - 2 : NUNIT;      // units in shared memory
  // Unit slot of (m, l'): for m >= 1 the first of the (+m, -m) pair (the
  // pair is (slot, slot + 1)); slots from NSU on are the TMEM pair.  For
  // L = 4 the last degree's pair sits in slots 4-5, which m = 3 does not
  // use, so the producers build it while m = 3 runs, and the next tile's
  // m = 0 units 0-3 while m = 4 runs (instead of waiting for the MMA to
  // release slots 0-1).
  static __host__ __device__ constexpr int unit_slot(int m, int lp) {
    return (L == 4 && m == 4) ? 4 : (m == 0 ? lp : 2 * (lp - m));
  }
  // The producers' fill order within degree m: the t-th unit filled is
  // l' = fill_lp(m, t) (for L = 4 and m = 1 the TMEM pair first, since it
  // is free while m = 0 runs).
  static __host__ __device__ constexpr int fill_lp(int m, int t) { return (L == 4 && m == 1) ? (t == 0 ? L : t) : m + t; }
  static constexpr int NDYE = (L + 1) * (L + 2) * (2 * L + 3) / 6;   // sum (l+1)^2
  static constexpr int NDYO = L * (L + 1) * (2 * L + 1) / 6;         // sum l^2
  static constexpr int NDYP = ((NDYE + NDYO) + 1) & ~1;
  static constexpr int WIG = L * (4 * L * L - 1) / 3 + (2 * L + 1) * (2 * L + 1);
  // Output-sum columns: the R-GEMM of degree l writes NL(l) columns from
  // OB(l); its S (2l+1) real columns start RO(l) into that block, the rest of
  // the block only ever receives exact zeros (zero rows of R), so real
  // columns of another degree may sit there.
  static __host__ __device__ constexpr int NL(int l) { return ((S * (2 * l + 1) + 15) / 16) * 16; }
  static __host__ __device__ constexpr int OCB(int l) {   // plain consecutive blocks
    int s = 0;
    for (int k = 0; k < l; ++k) s += NL(k);
    return s;
  }
  static __host__ __device__ constexpr int OB(int l) {
    return L >= 5 ? OCB(l) : (l <= 1 ? 0 : (l == 2 ? (L >= 3 ? 32 : 16) : (l == 3 ? 16 : 64)));
  }
  static __host__ __device__ constexpr int RO(int l) { return L >= 5 ? 0 : (l == 0 ? 12 : (l == 2 && L >= 3 ? 12 : 0)); }
  static constexpr int OUT_COLS = L >= 5 ? OCB(L + 1) : (L == 1 ? 16 : (L == 2 ? 48 : (L == 3 ? 64 : 112)));
  static constexpr int NLMAX = NL(L);
  // shared-memory carve-up (bytes)
  static constexpr size_t OFF_UNIT = 0;
  static constexpr size_t OFF_W = OFF_UNIT + (size_t)(NSU + (TE < 64 ? 1 : 0)) * UNIT_BYTES;
  static constexpr size_t OFF_A2 = OFF_W + (size_t)NSTAGE * STAGE_BYTES;
  static constexpr size_t OFF_R = OFF_A2 + (size_t)A2_BYTES;   // one A2 buffer: the signs take turns
  // per-tile geometry, two copies (tile parity): the producers build the
  // next tile's while the epilogue still reads the current one's
  static __host__ __device__ constexpr size_t r16(size_t x) { return (x + 15) & ~(size_t)15; }
  static constexpr size_t G_AL = 0;                                             // half [TE][ALS]
  static constexpr size_t G_DY = r16(G_AL + (size_t)TE * ALS * 2);              // half [TE][NDYP]
  static constexpr size_t G_CS = r16(G_DY + (size_t)TE * NDYP * 2);             // float cos [L][TE], sin [L][TE]
  static constexpr size_t G_GS = r16(G_CS + 2 * (size_t)TE * (L > 0 ? L : 1) * 4);  // half [TE][P]
  static constexpr size_t G_J = r16(G_GS + (size_t)TE * P * 2);                 // int j [TE], node [TE]
  // online softmax per (node slot, head): the factor that rescales the
  // node's earlier sums when its running max grows in this tile, and the
  // running denominator after this tile
  static constexpr size_t G_F = r16(G_J + 2 * (size_t)TE * 4);                  // float [S][HMAX]
  static constexpr size_t G_LS = G_F + (size_t)S * HMAX * 4;                     // float [S][HMAX]
  static constexpr size_t GEO_BYTES = r16(G_LS + (size_t)S * HMAX * 4);
  static constexpr size_t OFF_G2 = OFF_R + 2 * (size_t)NLMAX * TE * 2;
  static constexpr size_t OFF_GEO = OFF_G2 + 2 * GEO_BYTES;          // float [TE][4]: ct, st, u, pad
  // producers' running softmax state per (slot, head): max, denominator,
  // tile max (order-preserving int), tile sum, current max
  static constexpr size_t OFF_SMX = OFF_GEO + (size_t)TE * 4 * 4;
  static constexpr size_t OFF_TILE = OFF_SMX + 5 * (size_t)S * HMAX * 4;   // 8 ints
  static constexpr size_t OFF_BAR = (OFF_TILE + 32 + 7) & ~(size_t)7;
  static constexpr int NBAR = 2 * NUNIT + 2 * NSTAGE + 2 + 2 + 2 + 2 + 8;
  static constexpr size_t SMEM = OFF_BAR + NBAR * 8 + 16;
  static_assert(SMEM <= 232448, "shared memory budget");
  static_assert(TM_OUT + OUT_COLS <= (TMU ? TM_UNIT : 512u), "TMEM budget");
  // weight stages per tile
  static __host__ __device__ constexpr int stages_of_m(int m) { return (L - m + 1) * (L - m + 1) * (m == 0 ? 1 : 2); }
  static __host__ __device__ constexpr int stages_per_tile() {
    int s = 0;
    for (int m = 0; m <= L; ++m) s += stages_of_m(m);
    return s;
  }
};

struct TcArgs {
  const __nv_bfloat16 *q, *k, *v;
  const float *pos;
  Geom g;
  const int32_t *row_ptr, *col_idx;
  int N;
  int64_t E;
  int H;
  float inv_sqrt_d;
  const uint8_t *wpack;
  const float *W1, *W2;
  float *out;
  int *err;
  // multi-focus variant: F streams of CH / F channels (1: plain operator),
  // focus vector a [CH] (fp32), log2 of the stream width
  int F, fshift;
  const float *focus_a;
};

// ---------------------------------------------------------------------------
// helpers
// ---------------------------------------------------------------------------
__device__ __forceinline__ void named_bar(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}
// Named barrier that also ORs a predicate over the participating threads, so
// that every thread of a role takes the same branch (no thread may leave a
// loop that others still synchronise in).
__device__ __forceinline__ bool bar_or(int id, int nthreads, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, %2, %3, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)pred), "r"(id), "r"(nthreads)
      : "memory");
  return r != 0;
}

struct Waiter {
  volatile int *abort_flag;
  int *err;
  // sleep_ns > 0: back off between polls, so that a waiting warp leaves the
  // issue slots of its scheduler to the warps that share it (the MMA issuer
  // polls without sleeping).
  __device__ bool wait(uint64_t *bar, uint32_t parity, uint32_t sleep_ns = 0) {
    for (uint32_t it = 0; it < WAIT_LIMIT; ++it) {
      if (mbar_try_wait(bar, parity)) return true;
      if ((it & 255) == 255 && *abort_flag) return false;
      if (sleep_ns) __nanosleep(sleep_ns);
    }
    *abort_flag = 1;
    atomicExch(err, E2F_ERR_TIMEOUT);
    return false;
  }
  __device__ bool aborted() const { return *abort_flag != 0; }
};

// f(std::integral_constant<int, l>) for l = 0..L, each degree a compile-time
// constant.
template <int... ls, class F>
__device__ __forceinline__ void for_degrees_impl(std::integer_sequence<int, ls...>, F &&f) {
  (f(std::integral_constant<int, ls>{}), ...);
}
template <int L, class F> __device__ __forceinline__ void for_degrees(F &&f) {
  for_degrees_impl(std::make_integer_sequence<int, L + 1>{}, f);
}

// Edge range of one CTA, aligned to node boundaries: CTA b of G owns the
// nodes [n_b, n_{b+1}) with n_0 = 0, n_G = N and, in between, n_b the first
// node whose row starts at or after edge E b / G; its edges are
// [row_ptr[n_b], row_ptr[n_{b+1}]).  No node is split between CTAs, so every
// output row is written by exactly one CTA and the softmax of a node runs
// inside one CTA.
__device__ __forceinline__ int first_node_at(const int32_t *rp, int N, int64_t e) {
  int lo = 0, hi = N;   // smallest n in [0, N] with rp[n] >= e
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if ((int64_t)rp[mid] >= e) hi = mid;
    else lo = mid + 1;
  }
  return lo;
}

struct TileIter {
  const int32_t *rp;
  int N;
  int te;   // edges per tile
  int64_t ebeg, eend;
  int64_t e0, e1;
  int n0;
  // node range of CTA b of G (computed once per CTA, then shared)
  static __device__ int2 node_range(const int32_t *rp, int N, int b, int G, int64_t E) {
    return make_int2(b == 0 ? 0 : first_node_at(rp, N, E * (int64_t)b / G),
                     b + 1 == G ? N : first_node_at(rp, N, E * (int64_t)(b + 1) / G));
  }
  __device__ void bounds() {
    const int nlim = min(n0 + S, N);
    int64_t e = e0 + te;
    if (eend < e) e = eend;
    if ((int64_t)rp[nlim] < e) e = rp[nlim];
    e1 = e;
  }
  __device__ bool start() {
    e0 = ebeg;
    if (e0 >= eend) return false;
    int lo = 0, hi = N - 1;   // largest n with rp[n] <= e0
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if ((int64_t)rp[mid] <= e0) lo = mid;
      else hi = mid - 1;
    }
    n0 = lo;
    while ((int64_t)rp[n0 + 1] <= e0) ++n0;
    bounds();
    return true;
  }
  __device__ bool next() {
    e0 = e1;
    if (e0 >= eend) return false;
    while ((int64_t)rp[n0 + 1] <= e0) ++n0;
    bounds();
    return true;
  }
};

// D^l of the y-rotation in parity blocks: even rows/cols m >= 0, odd m < 0.
template <int L> __device__ __forceinline__ int dye_off(int l) { return l * (l + 1) * (2 * l + 1) / 6; }
template <int L> __device__ __forceinline__ int dyo_off(int l) {
  return Cfg<L>::NDYE + (l - 1) * l * (2 * l - 1) / 6;
}

// ---------------------------------------------------------------------------
// weight packing: one 32 KB stage per (m, l, l', half), in the order the MMA
// warp consumes them.  m = 0: W0 rows of degree l, columns of degree l'
// (128 x 128, K-major core matrices, Kc = 128).  m >= 1: Wr then Wi rows of
// degree l, columns of degree l', K half `kh` (128 x 64 each, Kc = 64).
// ---------------------------------------------------------------------------
struct PackArgs {
  const __nv_bfloat16 *W0;
  const __nv_bfloat16 *Wr[E2F_MAX_L + 1];
  const __nv_bfloat16 *Wi[E2F_MAX_L + 1];
  uint8_t *dst;
  int L;
  int F;   // focus streams: entries between channels of different streams are packed as zero
};

__global__ void __launch_bounds__(256) pack_w_kernel(PackArgs a) {
  // blockIdx.x = stage index; consecutive threads take consecutive source
  // columns, so the reads of a source row are coalesced
  const int L = a.L;
  int s = blockIdx.x;
  int m = 0;
  for (;; ++m) {
    const int n = (L - m + 1) * (L - m + 1) * (m == 0 ? 1 : 2);
    if (s < n) break;
    s -= n;
  }
  const int nk = (m == 0) ? 1 : 2;
  const int kh = s % nk;
  const int l = m + (s / nk) / (L - m + 1), lp = m + (s / nk) % (L - m + 1);
  uint8_t *stage = a.dst + (size_t)blockIdx.x * STAGE_BYTES;
  const int n = (L - m + 1) * CH;
  if (m == 0) {
    const int scol = lp * CH;
    const int cf = CH / a.F;
    for (int x = threadIdx.x; x < 128 * 128; x += blockDim.x) {
      const int row = x >> 7, k = x & 127;
      const size_t srow = (size_t)(l - m) * CH + row;
      const __nv_bfloat16 w = (row / cf == k / cf) ? a.W0[srow * n + scol + k] : __float2bfloat16_rn(0.f);
      *reinterpret_cast<__nv_bfloat16 *>(stage + kmajor_off(row, k, 128)) = w;
    }
  } else {
    const int scol = (lp - m) * CH + kh * 64;
    const int cf = CH / a.F;
    for (int x = threadIdx.x; x < 2 * 128 * 64; x += blockDim.x) {
      const int t = x >> 13, row = (x >> 6) & 127, k = x & 63;
      const size_t srow = (size_t)(l - m) * CH + row;
      const __nv_bfloat16 *src = (t == 0) ? a.Wr[m] : a.Wi[m];
      const __nv_bfloat16 w = (row / cf == (kh * 64 + k) / cf) ? src[srow * n + scol + k] : __float2bfloat16_rn(0.f);
      *reinterpret_cast<__nv_bfloat16 *>(stage + t * 16384 + kmajor_off(row, k, 64)) = w;
    }
  }
}

// ---------------------------------------------------------------------------
// Wigner blocks of the y-rotation Ry(-theta) as polynomials.  In the real
// basis, D^l(Ry(-theta))[m][m'] is zero unless m and m' have the same sign
// (m = 0 counting as cos-type), and otherwise equals
//   sin(theta)^eps * sum_j c_j cos(theta)^j,   eps = (|m| + |m'|) mod 2,
// a polynomial of degree l - eps (the half-angle powers of the Wigner
// small-d sum pair up into cos and sin of the full angle).  The coefficients
// are fitted once on the host, in double, to the Ivanic-Ruedenberg recursion
// of the same rotation (exact up to rounding: the fit is interpolation of a
// polynomial of known degree) and kept in constant memory; a residual above
// 1e-9 at any sample aborts the fit.
// Table entry of (l, m, m'): DYP_STRIDE floats at
// DYP_STRIDE * (wig_offset(l) + (m + l)(2l + 1) + (m' + l)): [eps, c_0, .., c_l].
// ---------------------------------------------------------------------------
__constant__ float c_dypoly[DYP_ENTRIES * DYP_STRIDE];

static bool fit_dy_poly(float *tab) {
  constexpr int L = E2F_MAX_L, K = 4 * (L + 1);
  static double D[K][DYP_ENTRIES];
  double ct[K], st[K];
  for (int k = 0; k < K; ++k) {
    const double th = 3.14159265358979323846 * (k + 0.5) / K;
    ct[k] = cos(th); st[k] = sin(th);
    const double R[9] = {ct[k], 0.0, -st[k], 0.0, 1.0, 0.0, st[k], 0.0, ct[k]};
    wig_all_serial<double>(R, L, D[k]);
  }
  for (int l = 0; l <= L; ++l) {
    const int w = 2 * l + 1;
    for (int m = -l; m <= l; ++m)
      for (int mp = -l; mp <= l; ++mp) {
        const int idx = wig_offset(l) + (m + l) * w + (mp + l);
        float *out = tab + (size_t)DYP_STRIDE * idx;
        for (int j = 0; j < DYP_STRIDE; ++j) out[j] = 0.f;
        if ((m < 0) != (mp < 0)) continue;
        const int eps = ((m < 0 ? -m : m) + (mp < 0 ? -mp : mp)) & 1;
        const int nc = l - eps + 1;
        // normal equations of the least-squares fit (nc <= 7), solved by
        // Gaussian elimination with partial pivoting
        double A[8][9] = {};
        for (int k = 0; k < K; ++k) {
          double basis[8];
          double pw = eps ? st[k] : 1.0;
          for (int j = 0; j < nc; ++j) { basis[j] = pw; pw *= ct[k]; }
          for (int i = 0; i < nc; ++i) {
            for (int j = 0; j < nc; ++j) A[i][j] += basis[i] * basis[j];
            A[i][nc] += basis[i] * D[k][idx];
          }
        }
        for (int c = 0; c < nc; ++c) {
          int piv = c;
          for (int r = c + 1; r < nc; ++r)
            if (fabs(A[r][c]) > fabs(A[piv][c])) piv = r;
          for (int j = 0; j <= nc; ++j) { const double t = A[c][j]; A[c][j] = A[piv][j]; A[piv][j] = t; }
          for (int r = 0; r < nc; ++r) {
            if (r == c) continue;
            const double f = A[r][c] / A[c][c];
            for (int j = c; j <= nc; ++j) A[r][j] -= f * A[c][j];
          }
        }
        double coef[8];
        for (int j = 0; j < nc; ++j) coef[j] = A[j][nc] / A[j][j];
        for (int k = 0; k < K; ++k) {
          double pw = eps ? st[k] : 1.0, v = 0.0;
          for (int j = 0; j < nc; ++j) { v += coef[j] * pw; pw *= ct[k]; }
          if (fabs(v - D[k][idx]) > 1e-9) return false;
        }
        out[0] = (float)eps;
        for (int j = 0; j < nc; ++j) out[1 + j] = (float)coef[j];
      }
  }
  return true;
}

}  // namespace tca

// Host copy of the table, fitted once per process (thread-safe); null if the
// fit failed.  The CG convolution uploads it into its own constant bank.
const float *dy_poly_host_table() {
  static float tab[DYP_ENTRIES * DYP_STRIDE];
  static std::once_flag fit_once;
  static bool fitted_ok = false;
  std::call_once(fit_once, [] { fitted_ok = tca::fit_dy_poly(tab); });
  return fitted_ok ? tab : nullptr;
}

namespace tca {

// Uploads the table to each device once; safe to call from several host
// threads.
static e2f_status ensure_dy_poly() {
  static std::mutex up_mu;
  static bool uploaded[64] = {};
  const float *tab = dy_poly_host_table();
  if (!tab) return E2F_ERR_CUDA;
  int dev = 0;
  E2F_CUDA_TRY(cudaGetDevice(&dev));
  if (dev < 0 || dev >= 64) return E2F_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lk(up_mu);
  if (!uploaded[dev]) {
    E2F_CUDA_TRY(cudaMemcpyToSymbol(c_dypoly, tab, sizeof(float) * DYP_ENTRIES * DYP_STRIDE));
    uploaded[dev] = true;
  }
  return E2F_OK;
}

// ---------------------------------------------------------------------------
// the fused kernel
// ---------------------------------------------------------------------------
template <int L, bool MF>
__global__ void __launch_bounds__(NTHREADS, 1) attn_tc_kernel(TcArgs a) {
  using Cf = Cfg<L>;
  constexpr int Q = Cf::Q, P = Cf::P, NUNIT = Cf::NUNIT;
  constexpr int TE = Cf::TE, UNIT_BYTES = Cf::UNIT_BYTES;
  extern __shared__ __align__(1024) uint8_t smem[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + Cf::OFF_BAR);
  uint64_t *unit_full = bars;
  uint64_t *unit_empty = unit_full + NUNIT;
  uint64_t *w_full = unit_empty + NUNIT;
  uint64_t *w_empty = w_full + NSTAGE;
  uint64_t *y_full = w_empty + NSTAGE;
  uint64_t *y_empty = y_full + 2;
  uint64_t *a2r_full = y_empty + 2;
  uint64_t *rg_done = a2r_full + 2;
  uint64_t *tile_done = rg_done + 2;
  uint64_t *slots_clean = tile_done + 1;
  uint64_t *geo_full = slots_clean + 1;    // [2], per geometry copy
  uint64_t *geo_empty = geo_full + 2;     // [2]
  uint64_t *mma_drain = geo_empty + 2;
  uint64_t *rg_drain = mma_drain + 1;
  uint32_t *tslot = reinterpret_cast<uint32_t *>(bars + Cf::NBAR);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tslot + 1);

  uint8_t *units = smem + Cf::OFF_UNIT;
  uint8_t *wst = smem + Cf::OFF_W;
  uint8_t *A2 = smem + Cf::OFF_A2;
  uint8_t *Rb = smem + Cf::OFF_R;
  float *geo = reinterpret_cast<float *>(smem + Cf::OFF_GEO);        // [TE][4]
  // geometry copy c
  auto g_al = [&](int c) { return reinterpret_cast<__half *>(smem + Cf::OFF_G2 + c * Cf::GEO_BYTES + Cf::G_AL); };
  auto g_dy = [&](int c) { return reinterpret_cast<__half *>(smem + Cf::OFF_G2 + c * Cf::GEO_BYTES + Cf::G_DY); };
  auto g_cs = [&](int c) { return reinterpret_cast<float *>(smem + Cf::OFF_G2 + c * Cf::GEO_BYTES + Cf::G_CS); };
  auto g_gs = [&](int c) { return reinterpret_cast<__half *>(smem + Cf::OFF_G2 + c * Cf::GEO_BYTES + Cf::G_GS); };
  auto g_jj = [&](int c) { return reinterpret_cast<int *>(smem + Cf::OFF_G2 + c * Cf::GEO_BYTES + Cf::G_J); };
  auto g_f = [&](int c) { return reinterpret_cast<float *>(smem + Cf::OFF_G2 + c * Cf::GEO_BYTES + Cf::G_F); };
  auto g_ls = [&](int c) { return reinterpret_cast<float *>(smem + Cf::OFF_G2 + c * Cf::GEO_BYTES + Cf::G_LS); };

  if (tid == 0) {
    // unit_full: one arrival per producer warp (the warps fill units independently)
    for (int s = 0; s < NUNIT; ++s) { mbar_init(&unit_full[s], 8); mbar_init(&unit_empty[s], 1); }
    for (int s = 0; s < NSTAGE; ++s) { mbar_init(&w_full[s], 1); mbar_init(&w_empty[s], 1); }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&y_full[b], 1); mbar_init(&y_empty[b], 4);
      mbar_init(&a2r_full[b], 1); mbar_init(&rg_done[b], 1);
    }
    mbar_init(tile_done, 1); mbar_init(slots_clean, 4);
    for (int c = 0; c < 2; ++c) { mbar_init(&geo_full[c], 1); mbar_init(&geo_empty[c], 4); }
    mbar_init(mma_drain, 1); mbar_init(rg_drain, 1);
    *abort_flag = 0;
    *reinterpret_cast<int2 *>(tslot + 2) = TileIter::node_range(a.row_ptr, a.N, blockIdx.x, gridDim.x, a.E);
    mbar_fence_init();
  }
  __syncthreads();
  if (warp == 0) { tmem_alloc(tslot, 512); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tslot;
  Waiter W{abort_flag, a.err};

  TileIter ti;
  ti.rp = a.row_ptr; ti.N = a.N; ti.te = Cf::TE;
  {
    const int2 nr = *reinterpret_cast<const int2 *>(tslot + 2);
    ti.ebeg = a.row_ptr[nr.x];
    ti.eend = a.row_ptr[nr.y];
  }
  const int H = a.H, Ch = CH / H;
  const int hshift = 31 - __clz(Ch);   // Ch is a power of two

  if (warp == 0) {
    // ======================= MMA issuer =======================
    if (lane == 0) {
      constexpr uint32_t ID_MAIN = idesc_bf16(64, 128, 0, 0);
      constexpr uint32_t ID_NEGB = ID_MAIN | (1u << 14);
      uint32_t st = 0, pc = 0;
      uint32_t fillpar = 0;        // bit sp: parity of unit sp's fill count
      const uint32_t s_units = smem_addr(units), s_w = smem_addr(wst);
      const uint64_t ud0 = smem_desc(s_units, 128, 128 * 16);   // unit 0, K-major, Kc = 128
      const uint64_t wd128 = smem_desc(s_w, 128, 128 * 16);     // stage 0 as 128 x 128 (m = 0)
      const uint64_t wd64 = smem_desc(s_w, 128, 64 * 16);       // stage 0 as 2 x 128 x 64 (m >= 1)
      bool ok = ti.start();
      auto mw = [&](uint64_t *bar, uint32_t parity) -> bool {
        for (uint32_t it = 0; it < WAIT_LIMIT; ++it) {
          if (mbar_test_wait(bar, parity)) return true;
          if ((it & 255) == 255 && W.aborted()) return false;
        }
        *abort_flag = 1;
        atomicExch(a.err, E2F_ERR_TIMEOUT);
        return false;
      };
      while (ok && !W.aborted()) {
        bool bad = false;
        #pragma unroll 1
        for (int m = 0; m <= L && !bad; ++m) {
          #pragma unroll 1
          for (int l = m; l <= L && !bad; ++l) {
            const uint32_t b = pc & 1;
            if (!mw(&y_empty[b], ((pc >> 1) & 1) ^ 1)) { bad = true; break; }
            tc_fence_after();
            const bool first_pass = (l == m), last_pass = (l == L);
            const uint32_t dp = tbase + 128 * b, dmn = tbase + (16u << 16) + 128 * b;
            #pragma unroll 1
            for (int lp = m; lp <= L && !bad; ++lp) {
              const int sp = Cf::unit_slot(m, lp);
              if (first_pass) {
                if (!mw(&unit_full[sp], (fillpar >> sp) & 1)) { bad = true; break; }
                if (m > 0 && !mw(&unit_full[sp + 1], (fillpar >> (sp + 1)) & 1)) { bad = true; break; }
                tc_fence_after();
              }
              const bool in_tmem = Cf::TMU && sp >= Cf::NSU;
              // descriptors advance by (byte offset >> 4): 16 per 16-wide K step
              const uint64_t adp = ud0 + (uint64_t)sp * (UNIT_BYTES >> 4), adm = adp + (UNIT_BYTES >> 4);
              const int nk = (m == 0) ? 1 : 2;
              #pragma unroll 1
              for (int kh = 0; kh < nk; ++kh) {
                const uint32_t s = st % NSTAGE;
                if (!mw(&w_full[s], (st / NSTAGE) & 1)) { bad = true; break; }
                const uint32_t acc0 = (lp > m || kh > 0) ? 1u : 0u;
                if (m == 0) {
                  // the whole 128 x 128 block: 8 steps of 16
                  const uint64_t bd = wd128 + (uint64_t)s * (STAGE_BYTES >> 4);
                  mma_bf16_ss(dp, adp, bd, ID_MAIN, acc0);
#pragma unroll
                  for (int sub = 1; sub < 8; ++sub) mma_bf16_ss(dp, adp + 16 * sub, bd + 16 * sub, ID_MAIN, 1u);
                } else {
                  // K half of 64: 4 steps of 16
                  const uint64_t br = wd64 + (uint64_t)s * (STAGE_BYTES >> 4), bi = br + (16384 >> 4);
                  if (in_tmem) {
                    // lane half 0 holds [v+ | v-], lane half 1 holds [v- | v+]
                    const uint32_t a0 = tbase + TM_UNIT + 32 * kh, a1 = a0 + (16u << 16);
#pragma unroll
                    for (int sub = 0; sub < 4; ++sub) {
                      const uint32_t acc = sub > 0 ? 1u : acc0;
                      mma_bf16_ts(dp, a0 + 8 * sub, br + 16 * sub, ID_MAIN, acc);
                      mma_bf16_ts(dp, a0 + 64 + 8 * sub, bi + 16 * sub, ID_NEGB, 1u);
                      mma_bf16_ts(dmn, a1 + 8 * sub, br + 16 * sub, ID_MAIN, acc);
                      mma_bf16_ts(dmn, a1 + 64 + 8 * sub, bi + 16 * sub, ID_MAIN, 1u);
                    }
                  } else {
                    const uint64_t ap = adp + 64 * kh, am = adm + 64 * kh;
#pragma unroll
                    for (int sub = 0; sub < 4; ++sub) {
                      const uint32_t acc = sub > 0 ? 1u : acc0;
                      mma_bf16_ss(dp, ap + 16 * sub, br + 16 * sub, ID_MAIN, acc);
                      mma_bf16_ss(dp, am + 16 * sub, bi + 16 * sub, ID_NEGB, 1u);
                      mma_bf16_ss(dmn, am + 16 * sub, br + 16 * sub, ID_MAIN, acc);
                      mma_bf16_ss(dmn, ap + 16 * sub, bi + 16 * sub, ID_MAIN, 1u);
                    }
                  }
                }
                mma_commit(&w_empty[s]);
                ++st;
              }
              if (bad) break;
              if (last_pass) {
                mma_commit(&unit_empty[sp]);
                fillpar ^= 1u << sp;
                if (m > 0) { mma_commit(&unit_empty[sp + 1]); fillpar ^= 1u << (sp + 1); }
              }
            }
            if (bad) break;
            mma_commit(&y_full[b]);
            ++pc;
          }
        }
        if (bad || W.aborted()) break;
        ok = ti.next();
      }
      // every MMA this thread issued has completed before TMEM is released
      mma_commit(mma_drain);
      for (uint32_t it = 0; it < WAIT_LIMIT; ++it)
        if (mbar_try_wait(mma_drain, 0)) break;
    }
  } else if (warp == 1 || warp == 2) {
    // ======================= weight loaders =======================
    if (lane == 0) {
      const int me = warp - 1;
      constexpr int SPT = Cf::stages_per_tile();
      uint32_t st = 0;
      bool ok = ti.start();
      while (ok && !W.aborted()) {
        for (int i = 0; i < SPT; ++i, ++st) {
          if ((int)(st % 2) != me) continue;
          const uint32_t s = st % NSTAGE;
          if (!W.wait(&w_empty[s], ((st / NSTAGE) & 1) ^ 1)) break;
          mbar_arrive_expect_tx(&w_full[s], STAGE_BYTES);
          bulk_g2s(wst + s * STAGE_BYTES, a.wpack + (size_t)i * STAGE_BYTES, STAGE_BYTES, &w_full[s]);
        }
        if (W.aborted()) break;
        ok = ti.next();
      }
      // drain: wait for this loader's last copy so no bulk write lands after exit
      if (st > 0) {
        for (uint32_t back = 1; back <= (uint32_t)NSTAGE && back <= st; ++back) {
          const uint32_t s_last = st - back;
          if ((int)(s_last % 2) != me) continue;
          const uint32_t s = s_last % NSTAGE;
          for (uint32_t it = 0; it < WAIT_LIMIT; ++it)
            if (mbar_try_wait(&w_full[s], (s_last / NSTAGE) & 1)) break;
        }
      }
    }
  } else if (warp == 3) {
    // ======================= back-rotation GEMM issuer =======================
    // Out[c][slot m'] += sum_e A2[c][e] R[slot m'][e] for each pass and sign,
    // issued as soon as the epilogue hands A2 / R over (a2r_full), so that
    // the SO(2) MMA thread never stops to poll for them.
    if (lane == 0) {
      const uint64_t a2d = smem_desc(smem_addr(A2), 128, TE * 16);   // A2, MN-major, K = TE edges
      const uint64_t rd = smem_desc(smem_addr(Rb), 128, TE * 16);    // R, K-major, K = TE edges
      uint32_t rgpar = 0;   // bit sg: parity of the GEMMs issued for sign sg
      int t = 0;
      bool ok = ti.start();
      while (ok && !W.aborted()) {
        bool bad = false;
        #pragma unroll 1
        for (int m = 0; m <= L && !bad; ++m) {
          #pragma unroll 1
          for (int l = m; l <= L && !bad; ++l) {
            const int ng = (m == 0) ? 1 : 2;
            for (int hs = 0; hs < ng; ++hs) {
              if (!W.wait(&a2r_full[hs], (rgpar >> hs) & 1)) { bad = true; break; }
              if (m == 0 && l == 0 && hs == 0 && t > 0)   // first GEMM of a tile: Out columns cleared
                if (!W.wait(slots_clean, (t - 1) & 1)) { bad = true; break; }
              tc_fence_after();
              const uint32_t id = idesc_bf16(128, Cf::NL(l), 1, 0);
              const uint32_t d = tbase + TM_OUT + Cf::OB(l);
              const uint64_t bd = rd + (uint64_t)hs * ((Cf::NLMAX * TE * 2) >> 4);
#pragma unroll
              for (int kk = 0; kk < TE / 16; ++kk) mma_bf16_ss(d, a2d + 16 * kk, bd + 16 * kk, id, 1u);
              mma_commit(&rg_done[hs]);
              rgpar ^= 1u << hs;
            }
          }
        }
        if (bad || W.aborted()) break;
        mma_commit(tile_done);   // the tile's Out sums are complete once these GEMMs are
        ++t;
        ok = ti.next();
      }
      // every GEMM this thread issued has completed before TMEM is released
      mma_commit(rg_drain);
      for (uint32_t it = 0; it < WAIT_LIMIT; ++it)
        if (mbar_try_wait(rg_drain, 0)) break;
    }
  } else if (warp >= 4 && warp < 8) {
    // ======================= epilogue =======================
    const int ew = warp - 4;
    const int et = tid - 128;   // 0..127
    const uint32_t lane_base = (uint32_t)(32 * ew) << 16;
    // zero the Out accumulators
    {
      float z[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) z[i] = 0.f;
      for (int c = 0; c < Cf::OUT_COLS; c += 16) tmem_st_32x32b_x16(tbase + lane_base + TM_OUT + c, z);
      tmem_st_wait();
      tc_fence_before();
    }
    // rows of this CTA's nodes with no neighbour are never visited by a
    // tile: o_i = 0 for them
    const int2 nrange = *reinterpret_cast<const int2 *>(tslot + 2);
    for (int base = nrange.x + 32 * ew; base < nrange.y; base += 128) {
      const int n = base + lane;
      const bool empty = n < nrange.y && a.row_ptr[n] == a.row_ptr[n + 1];
      uint32_t msk = __ballot_sync(0xffffffffu, empty);
      while (msk) {
        const int nn = base + __ffs(msk) - 1;
        msk &= msk - 1;
        float4 *row = reinterpret_cast<float4 *>(a.out + (size_t)nn * Q * CH);
        for (int x = lane; x < Q * CH / 4; x += 32) __stcs(row + x, make_float4(0.f, 0.f, 0.f, 0.f));
      }
    }
    named_bar(1, 128);
    uint32_t pc = 0, nA0 = 0, nA1 = 0;   // R hand-overs per sign
    float beta[MF ? 8 : 1];              // multi-focus: this edge's stream weights (set at pass (0, 0))
    beta[0] = 1.f;
    int t = 0;
    bool dead = false;
    bool ok = ti.start();
    while (ok && !dead) {
      // this tile's geometry copy (tile parity), filled by the producers
      const int gc = t & 1;
      dead = bar_or(1, 128, et == 0 && !W.wait(&geo_full[gc], (t >> 1) & 1, 100));
      if (dead) break;
      const __half *al = g_al(gc), *gs = g_gs(gc), *dy = g_dy(gc);
      const float *csb = g_cs(gc), *snb = csb + TE * (L > 0 ? L : 1);
      const int *nodeof = g_jj(gc) + TE;
      const int ne = (int)(ti.e1 - ti.e0);
      #pragma unroll 1
      for (int m = 0; m <= L && !dead; ++m) {
        #pragma unroll 1
        for (int l = m; l <= L && !dead; ++l) {
          const uint32_t b = pc & 1;
          bool f = false;
          // y ready, and the A2 / R buffers free: the latest R-GEMM of each
          // sign has completed (one thread polls, the barrier hands it over)
          if (et == 0) {
            f = !W.wait(&y_full[b], (pc >> 1) & 1, 40);
            if (!f && nA0 > 0) f = !W.wait(&rg_done[0], (nA0 - 1) & 1, 40);
            if (!f && nA1 > 0) f = !W.wait(&rg_done[1], (nA1 - 1) & 1, 40);
          }
          dead = bar_or(1, 128, f);
          if (dead) break;
          tc_fence_after();
          // ---- y -> A2 (scaled by alpha g, bf16, MN-major [c][e]), one sign
          // at a time through the single A2 buffer
          const int sg = lane >> 4;                // 0: y+ rows, 1: y- rows
          const int e = 16 * ew + (lane & 15);
          const int p_ml = m * (L + 1) - m * (m - 1) / 2 + (l - m);
          const float ge = (e < ne) ? __half2float(gs[e * P + p_ml]) : 0.f;
          if constexpr (MF) {
            if (m == 0 && l == 0) {
              // stream weights of this edge ("DPA4 ...", §2.1 A2): z_f = sum
              // over the stream's channels of a_c (g y)[(0,0), c] / sqrt(C/F),
              // beta = softmax_f z.  The y+ lanes hold the edge rows of the
              // m = 0 pass; lanes 16-31 take their partner's weights.
              float z[8];
#pragma unroll
              for (int ff = 0; ff < 8; ++ff) z[ff] = 0.f;
#pragma unroll 1
              for (int i = 0; i < 8; i += 2) {
                float v[2][16];
                tmem_ld_32x32b_x16x2(tbase + lane_base + 128 * b + 16 * i, tbase + lane_base + 128 * b + 16 * i + 16,
                                     v[0], v[1]);
#pragma unroll
                for (int h2 = 0; h2 < 2; ++h2) {
                  const int c0 = 16 * (i + h2);
                  const float4 *ap = reinterpret_cast<const float4 *>(a.focus_a + c0);
                  float part = 0.f;
#pragma unroll
                  for (int k4 = 0; k4 < 4; ++k4) {
                    const float4 av = __ldg(ap + k4);
                    part = fmaf(av.x, v[h2][4 * k4], fmaf(av.y, v[h2][4 * k4 + 1],
                           fmaf(av.z, v[h2][4 * k4 + 2], fmaf(av.w, v[h2][4 * k4 + 3], part))));
                  }
                  const int f = c0 >> a.fshift;
#pragma unroll
                  for (int ff = 0; ff < 8; ++ff)
                    if (ff == f) z[ff] += part;
                }
              }
              const float zs = ge * rsqrtf((float)(CH / a.F));
              float zmax = -INFINITY;
#pragma unroll
              for (int ff = 0; ff < 8; ++ff)
                if (ff < a.F) zmax = fmaxf(zmax, z[ff] * zs);
              float zsum = 0.f;
#pragma unroll
              for (int ff = 0; ff < 8; ++ff) {
                beta[ff] = (ff < a.F) ? expf(z[ff] * zs - zmax) : 0.f;
                zsum += beta[ff];
              }
#pragma unroll
              for (int ff = 0; ff < 8; ++ff) beta[ff] = __shfl_sync(0xffffffffu, beta[ff] / zsum, lane & 15);
            }
          }
          auto to_a2 = [&](int which) {
#pragma unroll 1
            for (int i = 0; i < 8; i += 2) {
              float v[2][16];
              tmem_ld_32x32b_x16x2(tbase + lane_base + 128 * b + 16 * i, tbase + lane_base + 128 * b + 16 * i + 16,
                                   v[0], v[1]);
              if (sg == which) {
#pragma unroll
                for (int h2 = 0; h2 < 2; ++h2) {
                  const int c0 = 16 * (i + h2);
                  // channels [c0, c0 + 8) and [c0 + 8, c0 + 16) lie in one head each
                  float s_lo = (e < ne) ? __half2float(al[e * ALS + (c0 >> hshift)]) * ge : 0.f;
                  float s_hi = (e < ne) ? __half2float(al[e * ALS + ((c0 + 8) >> hshift)]) * ge : 0.f;
                  if constexpr (MF) {   // the 16 channels lie in one stream (C / F >= 16)
                    const int f = c0 >> a.fshift;
                    float bf = beta[0];
#pragma unroll
                    for (int ff = 1; ff < 8; ++ff)
                      if (ff == f) bf = beta[ff];
                    s_lo *= bf;
                    s_hi *= bf;
                  }
                  const float *vv = v[h2];
                  const uint4 lo = make_uint4(pack_bf16x2(vv[0] * s_lo, vv[1] * s_lo), pack_bf16x2(vv[2] * s_lo, vv[3] * s_lo),
                                              pack_bf16x2(vv[4] * s_lo, vv[5] * s_lo), pack_bf16x2(vv[6] * s_lo, vv[7] * s_lo));
                  const uint4 hi = make_uint4(pack_bf16x2(vv[8] * s_hi, vv[9] * s_hi), pack_bf16x2(vv[10] * s_hi, vv[11] * s_hi),
                                              pack_bf16x2(vv[12] * s_hi, vv[13] * s_hi), pack_bf16x2(vv[14] * s_hi, vv[15] * s_hi));
                  if (e < TE) {   // TMEM rows of edges >= TE (32-edge tiles) are not real
                    *reinterpret_cast<uint4 *>(A2 + mnmajor_off(c0, e, TE)) = lo;
                    *reinterpret_cast<uint4 *>(A2 + mnmajor_off(c0 + 8, e, TE)) = hi;
                  }
                }
              }
            }
          };
          to_a2(0);
          // ---- R for each sign.  R_s has rows (slot, m') (from row RO(l)),
          // columns edges; the only nonzero entry of an edge's column is
          // D^l[+-m][m'] in its own slot's rows.  Zero both R buffers, then one
          // thread per (edge, sign) writes its 2l + 1 entries.
          const int ng = (m == 0) ? 1 : 2;
          const int w2 = 2 * l + 1;
          const int nrow = Cf::NL(l);
          constexpr int RCH = TE / 8;   // 16-byte chunks per R row
          for (int idx = et; idx < ng * nrow * RCH; idx += 128) {
            const int s2 = idx / (nrow * RCH), rem = idx - s2 * nrow * RCH;
            *reinterpret_cast<uint4 *>(Rb + (size_t)s2 * Cf::NLMAX * TE * 2 + kmajor_off(rem / RCH, (rem % RCH) * 8, TE)) =
                make_uint4(0u, 0u, 0u, 0u);
          }
          named_bar(1, 128);
          {
            const int e = et % TE, s2 = et / TE;
            if (s2 < ng && e < ne) {
              uint8_t *Rs = Rb + (size_t)s2 * Cf::NLMAX * TE * 2;
              const __half *d = dy + e * Cf::NDYP;
              const int row0 = Cf::RO(l) + (nodeof[e] % S) * w2;
#pragma unroll 1
              for (int tq = 0; tq < w2; ++tq) {
                const int mp = tq - l, amp = mp < 0 ? -mp : mp;
                float val = 0.f;
                if (s2 == 0) {
                  const float de = __half2float(d[dye_off<L>(l) + m * (l + 1) + amp]);
                  val = (mp == 0) ? de : (mp > 0 ? de * csb[(amp - 1) * TE + e] : de * snb[(amp - 1) * TE + e]);
                } else if (mp != 0) {
                  const float dd = __half2float(d[dyo_off<L>(l) + (m - 1) * l + (amp - 1)]);
                  val = (mp > 0) ? -dd * snb[(amp - 1) * TE + e] : dd * csb[(amp - 1) * TE + e];
                }
                *reinterpret_cast<__nv_bfloat16 *>(Rs + kmajor_off(row0 + tq, e, TE)) = __float2bfloat16_rn(val);
              }
            }
          }
          fence_async_smem();
          named_bar(1, 128);
          if (et == 0) mbar_arrive(&a2r_full[0]);
          ++nA0;
          if (ng > 1) {
            // the second sign waits for the first sign's GEMM to release A2
            bool f2 = false;
            if (et == 0) f2 = !W.wait(&rg_done[0], (nA0 - 1) & 1, 20);
            dead = bar_or(1, 128, f2);
            if (dead) break;
            to_a2(1);
            fence_async_smem();
            named_bar(1, 128);
            if (et == 0) mbar_arrive(&a2r_full[1]);
            ++nA1;
          }
          tc_fence_before();
          named_bar(1, 128);
          if (lane == 0) mbar_arrive(&y_empty[b]);   // y of this pass fully read
          ++pc;
        }
      }
      if (dead) break;
      // ---- tile end: read out the nodes that finished here; the node that
      // continues into the next tile has its sums rescaled to the next
      // tile's running max (online softmax), before the next tile's first
      // back-rotation GEMM (which waits for slots_clean)
      dead = bar_or(1, 128, et == 0 && !W.wait(tile_done, t & 1, 40));
      if (dead) break;
      const int n1 = nodeof[ne - 1];
      const bool cont = (int64_t)a.row_ptr[n1 + 1] > ti.e1;   // node n1 continues (next tile exists)
      if (cont) {
        dead = bar_or(1, 128, et == 0 && !W.wait(&geo_full[gc ^ 1], ((t + 1) >> 1) & 1, 100));
        if (dead) break;
      }
      tc_fence_after();
      {
        const int c = 32 * ew + lane;       // this thread's channel (TMEM lane)
        const int h = c >> hshift;
        const float *ls = g_ls(gc), *fnext = g_f(gc ^ 1);
        for (int i = ti.n0; i <= n1; ++i) {
          if (a.row_ptr[i + 1] == a.row_ptr[i]) continue;   // empty row: zeroed at the start
          const int slot = i % S;
          const bool fin = !(cont && i == n1);
          // a continuing node whose reference maximum did not move (factor 1
          // for every head of this warp's channels) needs no rescale
          if (!fin && __all_sync(0xffffffffu, fnext[slot * HMAX + h] == 1.f)) continue;
          const float lsum = ls[slot * HMAX + h];
          const float scale = fin ? (lsum > 0.f ? 1.f / lsum : 0.f) : fnext[slot * HMAX + h];
          float *orow = a.out + (size_t)i * Q * CH + c;
          // degree by degree: the node's 2l + 1 columns are consecutive and
          // are read as one load of the next power-of-two width (the extra
          // columns lie inside the allocation and are ignored)
          for_degrees<L>([&](auto lc) {
            constexpr int l = decltype(lc)::value;
            constexpr int NW = l == 0 ? 1 : (l == 1 ? 4 : (l <= 3 ? 8 : 16));
            const uint32_t col0 = TM_OUT + Cf::OB(l) + Cf::RO(l) + slot * (2 * l + 1);
            uint32_t r[NW];
            tmem_ld_cols<NW>(tbase + lane_base + col0, r);
#pragma unroll
            for (int mp = 0; mp < 2 * l + 1; ++mp) {
              const float val = __uint_as_float(r[mp]) * scale;
              if (fin) __stcs(orow + (size_t)(l * l + mp) * CH, val);   // written once: evict-first
              asm volatile("tcgen05.st.sync.aligned.32x32b.x1.b32 [%0], {%1};" ::"r"(tbase + lane_base + col0 + mp),
                           "r"(fin ? 0u : __float_as_uint(val))
                           : "memory");
            }
          });
        }
        tmem_st_wait();
        tc_fence_before();
      }
      named_bar(1, 128);
      if (lane == 0) {
        mbar_arrive(&geo_empty[gc]);   // this geometry copy is free again
        mbar_arrive(slots_clean);
      }
      ++t;
      ok = ti.next();
    }
  } else if (warp >= 8) {
    // ======================= producers =======================
    // Per tile t (geometry copy t & 1): the rotated units, degree m by degree
    // m.  While the MMA warp works through the passes of degree m, the
    // producers (which wait for units to be released) build the geometry of
    // tile t + 1 into the other copy, a step at a time: basics, Wigner blocks,
    // logits in two halves.
    const int pt = tid - 256;        // 0..255
    const int pw = pt >> 5;          // 0..7
    uint32_t pfillpar = 0;   // bit sp: parity of unit sp's fill count
    // ---- per-edge basics: four threads per edge (consecutive lanes); the
    // first computes the frame, all four share the radial MLP (hidden units
    // 4q..4q+3 each, outputs reduced with shuffles)
    auto basics = [&](const TileIter &g, int c) {
      const int ne = (int)(g.e1 - g.e0);
      int *jj = g_jj(c), *nodeof = jj + TE;
      float *csb = g_cs(c), *snb = csb + TE * (L > 0 ? L : 1);
      __half *gs = g_gs(c);
      const int e = pt >> 2, q4 = pt & 3;   // (TE < 64: threads past 4 TE only help the shuffles)
      const bool live = e < ne;
      float r = 0.f;
      if (live) {
        const int64_t E = g.e0 + e;
        int i = g.n0;
        while ((int64_t)a.row_ptr[i + 1] <= E) ++i;
        const int j = a.col_idx[E];
        float dx, dyv, dz;
        pair_disp(a.g, load_pos(a.pos, i), load_pos(a.pos, j), dx, dyv, dz);
        r = sqrtf(dx * dx + dyv * dyv + dz * dz);
        if (q4 == 0) {
          jj[e] = j;
          nodeof[e] = i;
          float ux = 0.f, uy = 0.f, uz = 1.f;
          if (r > 0.f) { ux = dx / r; uy = dyv / r; uz = dz / r; }
          const float rho = sqrtf(ux * ux + uy * uy);
          float cp = 1.f, sp = 0.f;
          if (rho > 0.f) { cp = ux / rho; sp = uy / rho; }
          float cm = 1.f, sm = 0.f;
          for (int mm = 1; mm <= L; ++mm) {
            const float c2 = cm * cp - sm * sp, s2 = sm * cp + cm * sp;
            cm = c2; sm = s2;
            csb[(mm - 1) * TE + e] = cm;
            snb[(mm - 1) * TE + e] = sm;
          }
          geo[e * 4 + 0] = uz;
          geo[e * 4 + 1] = rho;
          geo[e * 4 + 2] = 0.5f * (cospif(r / a.g.rc) + 1.f);
        }
      } else if (q4 == 0 && e < TE) {
        jj[e] = -1;
        nodeof[e] = -1;
        for (int mm = 0; mm < L; ++mm) { csb[mm * TE + e] = 1.f; snb[mm * TE + e] = 0.f; }
        geo[e * 4 + 0] = 1.f; geo[e * 4 + 1] = 0.f; geo[e * 4 + 2] = 0.f;
      }
      // radial MLP: 8 Gaussians (centres k r_c / 7, sigma 0.5), 16 SiLU, P outputs
      float phi[8];
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        const float dd = r - (float)kk * (a.g.rc / 7.f);
        phi[kk] = expf(-dd * dd * 2.f);
      }
      float hid[4];
#pragma unroll
      for (int h = 0; h < 4; ++h) {
        float z = 0.f;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) z = fmaf(__ldg(a.W1 + (4 * q4 + h) * 8 + kk), phi[kk], z);
        hid[h] = z / (1.f + expf(-z));
      }
#pragma unroll
      for (int p = 0; p < P; ++p) {
        float gv = 0.f;
#pragma unroll
        for (int h = 0; h < 4; ++h) gv = fmaf(__ldg(a.W2 + p * 16 + 4 * q4 + h), hid[h], gv);
        gv += __shfl_xor_sync(0xffffffffu, gv, 1);
        gv += __shfl_xor_sync(0xffffffffu, gv, 2);
        if ((p & 3) == q4 && e < TE) gs[e * P + p] = __float2half_rn(live ? gv : 0.f);
      }
    };
    // ---- Wigner blocks of Ry(-theta), parity blocks straight to fp16:
    // warp = entry (coefficients broadcast from constant memory), lane = edge
    auto wigner = [&](int c) {
      __half *dy = g_dy(c);
      for (int x = pw; x < Cf::NDYE + Cf::NDYO; x += 8) {
        int l = 0, off = 0, m, mp;
        if (x < Cf::NDYE) {
          while (off + (l + 1) * (l + 1) <= x) { off += (l + 1) * (l + 1); ++l; }
          m = (x - off) / (l + 1);
          mp = (x - off) % (l + 1);
        } else {
          const int y = x - Cf::NDYE;
          l = 1;
          while (off + l * l <= y) { off += l * l; ++l; }
          m = -((y - off) / l + 1);
          mp = -((y - off) % l + 1);
        }
        const float *cf = c_dypoly + DYP_STRIDE * (wig_offset(l) + (m + l) * (2 * l + 1) + (mp + l));
        float cc[L + 1];
#pragma unroll
        for (int jd = 0; jd <= L; ++jd) cc[jd] = cf[1 + jd];   // zero above the entry's degree
        const bool eps = cf[0] != 0.f;
#pragma unroll
        for (int h2 = 0; h2 < TE / 32; ++h2) {
          const int e = lane + 32 * h2;
          const float ct = geo[e * 4 + 0], stt = geo[e * 4 + 1];
          float p = cc[L];
#pragma unroll
          for (int jd = L - 1; jd >= 0; --jd) p = fmaf(p, ct, cc[jd]);
          dy[e * Cf::NDYP + x] = __float2half_rn(eps ? p * stt : p);
        }
      }
    };
    // ---- logits -> alpha, items (edge, 8-channel block) of one half of the
    // tile: q and k rows loaded a degree at a time; the blocks of one head
    // are summed with shuffles (16 consecutive lanes = one edge's 16 blocks)
    constexpr int IPH = TE * 8 / 256;   // items per thread and half
    float sk0[IPH], sk1[IPH];           // logits of this thread's items, by half
    auto logits = [&](const TileIter &g, int c, int half, float (&sk)[IPH]) {
      const int ne = (int)(g.e1 - g.e0);
      const int *jj = g_jj(c), *nodeof = jj + TE;
      const float *csb = g_cs(c), *snb = csb + TE * (L > 0 ? L : 1);
      const __half *dy = g_dy(c);
#pragma unroll 1
      for (int it = 0; it < IPH; ++it) {
        const int item = pt + half * (TE * 8) + it * 256;
        const int e = item >> 4, c0 = (item & 15) * 8;
        float acc = 0.f;
        if (e < ne) {
          const int i = nodeof[e], j = jj[e];
          const __half *d = dy + e * Cf::NDYP;
          const __nv_bfloat16 *qr = a.q + (size_t)i * Q * CH + c0;
          const __nv_bfloat16 *kr = a.k + (size_t)j * Q * CH + c0;
          float2 accv[4];
#pragma unroll
          for (int x = 0; x < 4; ++x) accv[x] = make_float2(0.f, 0.f);
          auto pair = [](uint32_t w) { return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u)); };
#pragma unroll
          for (int l = 0; l <= L; ++l) {
            uint4 qv[2 * L + 1], kv[2 * L + 1];
#pragma unroll
            for (int tt = 0; tt < 2 * l + 1; ++tt) {
              qv[tt] = *reinterpret_cast<const uint4 *>(qr + (size_t)(l * l + tt) * CH);
              kv[tt] = *reinterpret_cast<const uint4 *>(kr + (size_t)(l * l + tt) * CH);
            }
            float2 qh[4], kh[4];
#pragma unroll
            for (int x = 0; x < 4; ++x) { qh[x] = make_float2(0.f, 0.f); kh[x] = make_float2(0.f, 0.f); }
#pragma unroll
            for (int tt = 0; tt < 2 * l + 1; ++tt) {
              const int mp = tt - l, amp = mp < 0 ? -mp : mp;
              const float de = __half2float(d[dye_off<L>(l) + amp]);   // row 0 of the even block
              const float coef = (mp == 0) ? de : (mp > 0 ? de * csb[(amp - 1) * TE + e] : de * snb[(amp - 1) * TE + e]);
              const float2 c2 = make_float2(coef, coef);
#pragma unroll
              for (int x = 0; x < 4; ++x) {
                qh[x] = __ffma2_rn(c2, pair(u4w(qv[tt], x)), qh[x]);
                kh[x] = __ffma2_rn(c2, pair(u4w(kv[tt], x)), kh[x]);
              }
            }
#pragma unroll
            for (int x = 0; x < 4; ++x) accv[x] = __ffma2_rn(qh[x], kh[x], accv[x]);
          }
#pragma unroll
          for (int x = 0; x < 4; ++x) acc += accv[x].x + accv[x].y;
        }
        const int nb = Ch >> 3;   // 8-channel blocks per head: 1, 2 or 4
        for (int o = 1; o < nb; o <<= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
        // the softmax logit with the envelope folded in: u e^s = e^(s + log u)
        // (the lane owning the head's first block keeps it for the
        // statistics step)
        sk[it] = (e < ne) ? acc * a.inv_sqrt_d + logf(geo[e * 4 + 2]) : -INFINITY;
      }
    };
    // ---- online softmax statistics of tile g (copy c), after both logit
    // halves ("E2Former-V2 ...", §2.2 online softmax; "EquiformerV3 ...",
    // §2B.3 envelope in numerator and denominator).  Per (node slot, head):
    // tile max of the logits, the node's reference maximum M (its first
    // tile's maximum, moved up only when a later tile exceeds it by more than
    // SOFTMAX_MARGIN), alpha = e^(s + log u - M) for the tile's edges (fp16,
    // at most e^margin), the factor e^(M_old - M) for the node's earlier sums
    // (1 unless M moved), and the running denominator l = l_old f + sum alpha.
    int *smx = reinterpret_cast<int *>(smem + Cf::OFF_SMX);      // tile max, order-preserving int
    float *ssum = reinterpret_cast<float *>(smx + S * HMAX);    // tile sum of alpha
    float *mcur = ssum + S * HMAX;                               // running max after the tile
    float *rs_m = mcur + S * HMAX;                               // running max (persists)
    float *rs_l = rs_m + S * HMAX;                               // running denominator (persists)
    auto ord = [](float x) { const int i = __float_as_int(x); return i >= 0 ? i : i ^ 0x7fffffff; };
    auto unord = [](int i) { return __int_as_float(i >= 0 ? i : i ^ 0x7fffffff); };
    auto stats_reset = [&]() {
      if (pt < S * HMAX) { smx[pt] = ord(-INFINITY); ssum[pt] = 0.f; }
    };
    auto softmax_stats = [&](const TileIter &g, int c) {
      const int ne = (int)(g.e1 - g.e0);
      const int *nodeof = g_jj(c) + TE;
      __half *al = g_al(c);
      const int nb = Ch >> 3;
      // phase A: tile max per (slot, head)
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
#pragma unroll
        for (int it = 0; it < IPH; ++it) {
          const int item = pt + hf * (TE * 8) + it * 256;
          const int e = item >> 4, blk = item & 15;
          if (e < ne && (blk & (nb - 1)) == 0)
            atomicMax(&smx[(nodeof[e] % S) * HMAX + blk / nb], ord(hf ? sk1[it] : sk0[it]));
        }
      }
      named_bar(2, 256);
      // phase B: running max of the node in each slot
      bool live = false, starts = false;
      if (pt < S * HMAX) {
        const int sl = pt / HMAX, h = pt % HMAX;
        int node = -1;
        for (int n = g.n0; n < min(g.n0 + S, a.N); ++n)
          if (n % S == sl) node = n;
        float Mn = -INFINITY, f = 1.f;
        live = node >= 0 && h < H;
        if (live) {
          starts = (int64_t)a.row_ptr[node] >= g.e0;
          const float Mo = starts ? -INFINITY : rs_m[pt], tmax = unord(smx[pt]);
          // the node keeps its reference maximum while the tile's stays
          // within SOFTMAX_MARGIN of it (alpha <= e^margin, no rescale);
          // otherwise the reference moves up and the earlier sums are
          // rescaled by e^(M_old - M)
          if (Mo == -INFINITY || tmax > Mo + SOFTMAX_MARGIN) {
            Mn = tmax;
            f = (Mo == -INFINITY) ? 1.f : expf(Mo - Mn);
          } else {
            Mn = Mo;
          }
        }
        mcur[pt] = Mn;
        g_f(c)[pt] = f;
      }
      named_bar(2, 256);
      // phase C: alpha of the tile's edges and its per-(slot, head) sum
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
#pragma unroll
        for (int it = 0; it < IPH; ++it) {
          const int item = pt + hf * (TE * 8) + it * 256;
          const int e = item >> 4, blk = item & 15;
          if (e < TE && (blk & (nb - 1)) == 0) {
            const int h = blk / nb;
            float av = 0.f;
            int sl = 0;
            if (e < ne) {
              sl = nodeof[e] % S;
              const float M = mcur[sl * HMAX + h];
              av = (M == -INFINITY) ? 0.f : expf((hf ? sk1[it] : sk0[it]) - M);
            }
            const __half hv = __float2half_rn(av);
            al[e * ALS + h] = hv;
            if (e < ne) atomicAdd(&ssum[sl * HMAX + h], __half2float(hv));   // the rounded values used
          }
        }
      }
      named_bar(2, 256);
      // phase D: running denominator after this tile
      if (pt < S * HMAX) {
        float lnew = 0.f;
        if (live) {
          lnew = (starts ? 0.f : rs_l[pt] * g_f(c)[pt]) + ssum[pt];
          rs_l[pt] = lnew;
          rs_m[pt] = mcur[pt];
        }
        g_ls(c)[pt] = lnew;
      }
    };
    // geometry step k (0 basics, 1 Wigner, 2 / 3 logits halves) of tile g
    // into copy c; step 0 first waits until the epilogue has released the copy
    auto geo_step = [&](int k, const TileIter &g, int c, int tg) -> bool {
      if (k == 0) {
        bool f = false;
        if (pt == 0) f = !W.wait(&geo_empty[c], ((tg >> 1) & 1) ^ 1, 100);
        if (bar_or(2, 256, f || W.aborted())) return false;
        basics(g, c);
      } else if (k == 1) {
        wigner(c);
      } else if (k == 2) {
        stats_reset();
        logits(g, c, 0, sk0);
      } else {
        logits(g, c, 1, sk1);
        softmax_stats(g, c);
      }
      named_bar(2, 256);
      if (k == 3 && pt == 0) mbar_arrive(&geo_full[c]);
      return true;
    };
    int t = 0;
    bool dead = false;
    bool ok = ti.start();
    if (ok) {
      for (int k = 0; k < 4 && !dead; ++k) dead = !geo_step(k, ti, 0, 0);
    }
    while (ok && !dead) {
      const int gc = t & 1;
      TileIter tn = ti;
      const bool has_next = tn.next();
      const int ne = (int)(ti.e1 - ti.e0);
      const int *jj = g_jj(gc);
      const float *csb = g_cs(gc), *snb = csb + TE * (L > 0 ? L : 1);
      const __half *dy = g_dy(gc);
      // ---- rotate in, block by block
      #pragma unroll 1
      for (int m = 0; m <= L && !dead; ++m) {
        #pragma unroll 1
        for (int tf = 0; tf <= L - m; ++tf) {
          const int lp = Cf::fill_lp(m, tf);
          const int sp = Cf::unit_slot(m, lp);
          {
            // each producer warp waits for the unit on its own: the warps run
            // through the units independently (a warp that finished its part
            // of one unit starts loading for the next)
            bool f = false;
            if (lane == 0) {
              f = !W.wait(&unit_empty[sp], ((pfillpar >> sp) & 1) ^ 1, 40);
              if (!f && m > 0) f = !W.wait(&unit_empty[sp + 1], ((pfillpar >> (sp + 1)) & 1) ^ 1, 40);
            }
            dead = __shfl_sync(0xffffffffu, (int)(f || W.aborted()), 0) != 0;
            if (dead) break;
          }
          // v~(+m), v~(-m) of degree l' (compile-time constant: register use
          // follows the degree) for NB (edge, 8-channel block) items of this
          // thread: block b belongs to edge ea (first half of the blocks, or
          // all of them when NEc = 1) or eb (second half), and covers
          // channels [cbs[b], +8).  Pairs of channels go through packed fp32
          // FMAs.  emit(b, wp, wm) receives block b as packed bf16 pairs (wp:
          // +m, wm: -m); edges past the tile's end come out zero.
          auto rot4 = [&](auto LPc, auto NEc, const int ea, const int eb, const auto &cbs, auto &&emit) {
            constexpr int LP = decltype(LPc)::value;
            constexpr int NR = 2 * LP + 1;
            constexpr int NB = (int)(sizeof(cbs) / sizeof(int));   // blocks of this thread
            constexpr int NE = decltype(NEc)::value;               // distinct edges: 1 or 2
            constexpr int BPE = NB / NE;                           // blocks per edge
            if constexpr (NE == 1) {
              if (ea >= ne) {
                const uint4 z = make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
                for (int bb = 0; bb < NB; ++bb) emit(bb, z, z);
                return;
              }
            }
            // rows of edges past the tile's end: node 0's, scaled by zero
            const __nv_bfloat16 *vra = a.v + (size_t)(ea < ne ? jj[ea] : 0) * Q * CH + (size_t)(LP * LP) * CH;
            const __nv_bfloat16 *vrb = NE == 1 ? vra : a.v + (size_t)(eb < ne ? jj[eb] : 0) * Q * CH + (size_t)(LP * LP) * CH;
            // per-edge coefficients: u+ = c v+ + s v-, u- = -s v+ + c v-, scaled
            // by the y-rotation entries of row +m (even block) / -m (odd block)
            float c0 = 0.f, app[LP > 0 ? LP : 1], apm[LP > 0 ? LP : 1], amp[LP > 0 ? LP : 1], amm[LP > 0 ? LP : 1];
            {
              const int e = ea;
              const bool live = e < ne;
              const __half *d = dy + (live ? e : 0) * Cf::NDYP;
              c0 = live ? __half2float(d[dye_off<L>(LP) + m * (LP + 1)]) : 0.f;
#pragma unroll
              for (int kq = 1; kq <= LP; ++kq) {
                const float ck = csb[(kq - 1) * TE + e], sk = snb[(kq - 1) * TE + e];
                const float de = live ? __half2float(d[dye_off<L>(LP) + m * (LP + 1) + kq]) : 0.f;
                const float dd = (live && m > 0) ? __half2float(d[dyo_off<L>(LP) + (m - 1) * LP + (kq - 1)]) : 0.f;
                app[kq - 1] = de * ck; apm[kq - 1] = de * sk;
                amp[kq - 1] = -dd * sk; amm[kq - 1] = dd * ck;
              }
            }
            // two blocks of gathered rows in flight: block b + 1 is loaded
            // while block b is computed
            constexpr int DEPTH = 2;
            uint4 buf[DEPTH][NR];
#pragma unroll
            for (int bb = 0; bb < DEPTH - 1; ++bb)
#pragma unroll
              for (int t = 0; t < NR; ++t) buf[bb][t] = *reinterpret_cast<const uint4 *>((bb < BPE ? vra : vrb) + (size_t)t * CH + cbs[bb]);
#pragma unroll
            for (int bb = 0; bb < NB; ++bb) {
              if (bb > 0 && bb % BPE == 0)   // next edge
              {
                const int e = eb;
                const bool live = e < ne;
                const __half *d = dy + (live ? e : 0) * Cf::NDYP;
                c0 = live ? __half2float(d[dye_off<L>(LP) + m * (LP + 1)]) : 0.f;
#pragma unroll
                for (int kq = 1; kq <= LP; ++kq) {
                  const float ck = csb[(kq - 1) * TE + e], sk = snb[(kq - 1) * TE + e];
                  const float de = live ? __half2float(d[dye_off<L>(LP) + m * (LP + 1) + kq]) : 0.f;
                  const float dd = (live && m > 0) ? __half2float(d[dyo_off<L>(LP) + (m - 1) * LP + (kq - 1)]) : 0.f;
                  app[kq - 1] = de * ck; apm[kq - 1] = de * sk;
                  amp[kq - 1] = -dd * sk; amm[kq - 1] = dd * ck;
                }
              }
              if (bb + DEPTH - 1 < NB) {
                const int nb = bb + DEPTH - 1 < NB ? bb + DEPTH - 1 : 0;
#pragma unroll
                for (int t = 0; t < NR; ++t)
                  buf[(bb + DEPTH - 1) % DEPTH][t] = *reinterpret_cast<const uint4 *>((nb < BPE ? vra : vrb) + (size_t)t * CH + cbs[nb]);
              }
              auto pair = [](uint32_t w) { return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u)); };
              float2 ap[4], am[4];
              {
#pragma unroll
                for (int x = 0; x < 4; ++x) {
                  const float2 v0 = pair(u4w(buf[bb % DEPTH][LP], x));
                  ap[x] = make_float2(c0 * v0.x, c0 * v0.y);
                  am[x] = make_float2(0.f, 0.f);
                }
              }
#pragma unroll
              for (int kq = 1; kq <= LP; ++kq) {

                const float2 cpp = make_float2(app[kq - 1], app[kq - 1]), cpm = make_float2(apm[kq - 1], apm[kq - 1]);
                const float2 cmp = make_float2(amp[kq - 1], amp[kq - 1]), cmm = make_float2(amm[kq - 1], amm[kq - 1]);
#pragma unroll
                for (int x = 0; x < 4; ++x) {
                  const float2 vp2 = pair(u4w(buf[bb % DEPTH][LP + kq], x)), vn2 = pair(u4w(buf[bb % DEPTH][LP - kq], x));
                  ap[x] = __ffma2_rn(cpp, vp2, __ffma2_rn(cpm, vn2, ap[x]));
                  am[x] = __ffma2_rn(cmp, vp2, __ffma2_rn(cmm, vn2, am[x]));
                }
              }
              const uint4 wp = make_uint4(pack_bf16x2(ap[0].x, ap[0].y), pack_bf16x2(ap[1].x, ap[1].y),
                                          pack_bf16x2(ap[2].x, ap[2].y), pack_bf16x2(ap[3].x, ap[3].y));
              const uint4 wm = make_uint4(pack_bf16x2(am[0].x, am[0].y), pack_bf16x2(am[1].x, am[1].y),
                                          pack_bf16x2(am[2].x, am[2].y), pack_bf16x2(am[3].x, am[3].y));
              emit(bb, wp, wm);
            }
          };
          if (Cf::TMU && sp >= Cf::NSU) {
            if constexpr (Cf::TMU) {
            // unit pair in TMEM as the M = 64 A operand: row e at lane
            // 32 (e / 16) + e % 16 (+16 in the upper half); lane half 0 holds
            // [v+ | v-], half 1 holds [v- | v+] (64 columns each, channel
            // pairs packed low / high).  Warp 8 + pw writes subpartition pw % 4,
            // channels [64 (pw / 4), +64).
            const int q = pw & 3, chb = (pw >> 2) * 64;
            const int e = 16 * q + (lane & 15), half = lane >> 4;
            // lane half h computes channels [chb + 32h, +32) of both signs;
            // the two halves swap what the other one stores
            uint32_t wpl[16], wmi[16];
            {
              const int cb0 = chb + 32 * half;
              const int cbs[4] = {cb0, cb0 + 8, cb0 + 16, cb0 + 24};
              rot4(std::integral_constant<int, L>{}, std::integral_constant<int, 1>{}, e, e, cbs, [&](int bb, const uint4 &wp, const uint4 &wm) {
#pragma unroll
                for (int i = 0; i < 4; ++i) { wpl[4 * bb + i] = u4w(wp, i); wmi[4 * bb + i] = u4w(wm, i); }
              });
            }
            uint32_t opl[16], omi[16];   // the partner half's block
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              opl[i] = __shfl_xor_sync(0xffffffffu, wpl[i], 16);
              omi[i] = __shfl_xor_sync(0xffffffffu, wmi[i], 16);
            }
            const uint32_t ta = tbase + ((uint32_t)(32 * q) << 16) + TM_UNIT + (uint32_t)chb / 2;
            uint32_t st0[16], st1[16], st2[16], st3[16];   // warp-collective stores: select per lane
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              st0[i] = half ? omi[i] : wpl[i];   // cols [ta, +16):      v+ (half 0) / v- (half 1), block A
              st1[i] = half ? opl[i] : wmi[i];   // cols [ta + 64, +16): v- / v+, block A
              st2[i] = half ? wmi[i] : opl[i];   // cols [ta + 16, +16): v+ / v-, block B
              st3[i] = half ? wpl[i] : omi[i];   // cols [ta + 80, +16): v- / v+, block B
            }
            tmem_st_32x32b_x16u(ta, st0);
            tmem_st_32x32b_x16u(ta + 64, st1);
            tmem_st_32x32b_x16u(ta + 16, st2);
            tmem_st_32x32b_x16u(ta + 80, st3);
            tmem_st_wait();
            tc_fence_before();
            }
          } else {
            uint8_t *up = units + (size_t)sp * UNIT_BYTES;
            uint8_t *um = up + UNIT_BYTES;
            // a warp covers EPW = TE / 8 edges, in groups of four: a gathered
            // row is read as four edges x 128 contiguous bytes, and the stores
            // fill whole 128-byte rows of the K-major unit.  Thread: edge
            // 4 g + (lane & 3) of group g, channels [8 (lane >> 2), +8) and
            // the same + 64.
            constexpr int NG = TE / 32;
            const int cb0 = (lane >> 2) * 8;
            const int ea = pw * (TE / 8) + (lane & 3), eb = ea + 4;
            auto fill = [&](auto LPc) {
              int cbs[2 * NG];
#pragma unroll
              for (int k = 0; k < 2 * NG; ++k) cbs[k] = cb0 + 64 * (k & 1);
              rot4(LPc, std::integral_constant<int, NG>{}, ea, eb, cbs, [&](int bb, const uint4 &wp, const uint4 &wm) {
                const int e = bb < 2 ? ea : eb;
                *reinterpret_cast<uint4 *>(up + kmajor_off(e, cbs[bb], 128)) = wp;
                if (m > 0) *reinterpret_cast<uint4 *>(um + kmajor_off(e, cbs[bb], 128)) = wm;
              });
            };
            switch (lp) {
              case 0: fill(std::integral_constant<int, 0>{}); break;
              case 1: if constexpr (L >= 1) fill(std::integral_constant<int, (L >= 1 ? 1 : 0)>{}); break;
              case 2: if constexpr (L >= 2) fill(std::integral_constant<int, (L >= 2 ? 2 : 0)>{}); break;
              case 3: if constexpr (L >= 3) fill(std::integral_constant<int, (L >= 3 ? 3 : 0)>{}); break;
              case 4: if constexpr (L >= 4) fill(std::integral_constant<int, (L >= 4 ? 4 : 0)>{}); break;
              case 5: if constexpr (L >= 5) fill(std::integral_constant<int, (L >= 5 ? 5 : 0)>{}); break;
              default: if constexpr (L >= 6) fill(std::integral_constant<int, (L >= 6 ? 6 : 0)>{}); break;
            }
          }
          fence_async_smem();
          __syncwarp();
          if (lane == 0) {
            mbar_arrive(&unit_full[sp]);
            if (m > 0) mbar_arrive(&unit_full[sp + 1]);
          }
          pfillpar ^= 1u << sp;
          if (m > 0) pfillpar ^= 1u << (sp + 1);
        }
        // every producer warp reaches this point (done, or broken out on an
        // abort), so the geometry barriers never wait for a missing warp
        dead = bar_or(2, 256, dead || W.aborted());
        if (dead) break;
        // while the passes of degree m run: geometry steps of the next tile
        if (has_next) {
          for (int k = 0; k < 4 && !dead; ++k)
            if ((k < L ? k : L) == m) dead = !geo_step(k, tn, gc ^ 1, t + 1);
        }
      }
      if (dead) break;
      ++t;
      ti = tn;
      ok = has_next;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tbase, 512);
}

template <int L, bool MF = false>
static e2f_status launch_tc(const TcArgs &args, int grid, cudaStream_t s) {
  using Cf = Cfg<L>;
  E2F_CUDA_TRY(cudaFuncSetAttribute(attn_tc_kernel<L, MF>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)Cf::SMEM));
  E2F_LAUNCH((attn_tc_kernel<L, MF>), grid, NTHREADS, Cf::SMEM, s, args);
  return E2F_OK;
}

}  // namespace tca

e2f_status attention_tc_available(const e2f_weights *w) {
  if (w->dtype != E2F_BF16 || w->C != tca::CH) return E2F_ERR_UNSUPPORTED;
  if (w->L_max < 1 || w->L_max > 6) return E2F_ERR_UNSUPPORTED;
  // L = 3 is not instantiated: its build of this kernel stopped on the GPU
  // with a misaligned-address fault whose cause has not been found (every
  // address the source forms is 16-byte aligned by construction); L = 3
  // inputs run on the CUDA-core kernel instead
  if (w->L_max == 3) return E2F_ERR_UNSUPPORTED;
  // heads of 8..32 channels (the head reductions run inside one warp)
  if (w->H < 4 || w->H > tca::HMAX || tca::CH % w->H != 0) return E2F_ERR_UNSUPPORTED;
  return E2F_OK;
}

e2f_status attention_tc_impl(const void *q, const void *k, const void *v, const float *pos, const e2f_csr *csr,
                             const e2f_weights *w, float *out, cudaStream_t s, cudaEvent_t ev0, cudaEvent_t ev1,
                             int F, const float *focus_a) {
  using namespace tca;
  if (F != 1 && w->L_max != 2 && w->L_max != 4) return E2F_ERR_UNSUPPORTED;
  const int L = w->L_max;
  const int64_t N = csr->n_nodes, E = csr->n_edges;
  const size_t Q = (size_t)(L + 1) * (L + 1);
  if (E == 0) {   // every row is empty: o = 0
    E2F_CUDA_TRY(cudaMemsetAsync(out, 0, (size_t)N * Q * CH * sizeof(float), s));
    return E2F_OK;
  }
  {
    const e2f_status ps = ensure_dy_poly();
    if (ps != E2F_OK) return ps;
  }
  // pack weights
  int nst = 0;
  for (int m = 0; m <= L; ++m) nst += (L - m + 1) * (L - m + 1) * (m == 0 ? 1 : 2);
  const size_t wbytes = (size_t)nst * STAGE_BYTES;
  Scratch wp;
  E2F_CUDA_TRY(wp.alloc(wbytes, s));
  PackArgs pa;
  pa.W0 = static_cast<const __nv_bfloat16 *>(w->W0);
  for (int m = 0; m <= E2F_MAX_L; ++m) {
    pa.Wr[m] = (m >= 1 && m <= L) ? static_cast<const __nv_bfloat16 *>(w->Wr[m]) : nullptr;
    pa.Wi[m] = (m >= 1 && m <= L) ? static_cast<const __nv_bfloat16 *>(w->Wi[m]) : nullptr;
  }
  pa.dst = wp.as<uint8_t>();
  pa.L = L;
  pa.F = F;
  E2F_LAUNCH(pack_w_kernel, nst, 256, 0, s, pa);

  TcArgs a;
  a.q = static_cast<const __nv_bfloat16 *>(q);
  a.k = static_cast<const __nv_bfloat16 *>(k);
  a.v = static_cast<const __nv_bfloat16 *>(v);
  a.pos = pos;
  for (int kk = 0; kk < 3; ++kk) {
    a.g.box[kk] = csr->box[kk] > 0.f ? csr->box[kk] : 0.f;
    a.g.half[kk] = 0.5f * a.g.box[kk];
    a.g.periodic[kk] = csr->box[kk] > 0.f;
  }
  a.g.rc = csr->r_c;
  a.g.rc2 = csr->r_c * csr->r_c;
  a.row_ptr = csr->row_ptr;
  a.col_idx = csr->col_idx;
  a.N = (int)N;
  a.E = E;
  a.H = w->H;
  a.inv_sqrt_d = 1.f / sqrtf((float)((L + 1) * (CH / w->H)));
  a.wpack = wp.as<uint8_t>();
  a.W1 = w->rad_W1;
  a.W2 = w->rad_W2;
  a.out = out;
  a.err = device_error_flag();
  a.F = F;
  a.fshift = 31 - __builtin_clz((unsigned)(CH / F));
  a.focus_a = focus_a;
  if (!a.err) return E2F_ERR_CUDA;
  e2f_status r = E2F_OK;
  int dev = 0, nsm = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
  const int te = L >= 5 ? Cfg<6>::TE : TE64;
  const int grid = (int)std::max<int64_t>(1, std::min<int64_t>(nsm, (E + te - 1) / te));
  if (ev0) E2F_CUDA_TRY(cudaEventRecord(ev0, s));
  switch (L) {
    case 1: r = launch_tc<1>(a, grid, s); break;
    case 2: r = F > 1 ? launch_tc<2, true>(a, grid, s) : launch_tc<2>(a, grid, s); break;
    case 4: r = F > 1 ? launch_tc<4, true>(a, grid, s) : launch_tc<4>(a, grid, s); break;
    case 5: r = launch_tc<5>(a, grid, s); break;
    case 6: r = launch_tc<6>(a, grid, s); break;
    default: return E2F_ERR_UNSUPPORTED;
  }
  if (ev1) E2F_CUDA_TRY(cudaEventRecord(ev1, s));
  return r;
}

}  // namespace e2f
