// Backward of the on-the-fly equivariant attention: dL/dx and dL/dpos of a
// scalar L = sum(G * o) -- the conservative forces are -dL/dpos ("E2Former-V2
// ...", technical summary §4: the conservative variant, forces as the
// gradient of the energy; "DPA4 ...", §2.2 energy-to-force path).
//
// Recompute, per chunk of whole destination nodes (at most CHUNK_E edges):
//   K0 edge_dst     the destination node of every edge of the chunk
//   K1 edge_fwd     geometry, D^l blocks of the two-angle frame, envelope,
//                   radial MLP, logits s; the rotated features
//                   v~ = D v_j in SO(2)-stacked order
//   K2 node_stats   per (node, head) max and denominator of e^(s + log u)
//   GEMM            Y_m = V~_m Wc_m^T for every m: Wc_0 = W0, Wc_m =
//                   [[Wr, -Wi], [Wi, Wr]] acting on (v~+, v~-)  (cuBLAS)
//   K3 edge_dalpha  y = g Y; GD = D G_i (the output gradient in the edge
//                   frame); dalpha_h = <y, GD>_h; alpha_h
//   K4 node_delta   Delta_h = sum_e alpha_h dalpha_h  (= <G_i, o_i>_h)
//   K5 edge_dy      ds_h = alpha_h (dalpha_h - Delta_h); dL/du; dy = alpha GD;
//                   dL/dg; dw = g dy (stacked)
//   GEMM            dV~_m = dW_m Wc_m  (transposed SO(2) products)
//   K6 edge_bwd     dL/dD^l from the rotate-in, the back-rotation and the
//                   m = 0 rows of the logits; the rotation generators turn
//                   it into a torque tau_k = -<D^T dL/dD, J_k>, so that
//                   dL/dr_ij = (dL/dr) rhat + tau x rhat / r; atomics into
//                   dL/dpos of both atoms and into dL/dq_i, dL/dk_j, dL/dv_j
// then
//   GEMM            dL/dx = per degree dq Wq + dk Wk + dv Wv (cuBLAS, fp32).
//
// Per-edge tensors live only inside a chunk (bounded scratch); the SO(2)
// products are dense GEMMs over the chunk's edges.
#include <cublas_v2.h>
#include <math.h>

#include <algorithm>
#include <mutex>
#include <type_traits>
#include <vector>

#include "common.cuh"
#include "wigner.cuh"

namespace e2f {

e2f_status project_impl(const void *, int64_t, const e2f_weights *, void *, void *, void *, cudaStream_t);

namespace bwd {

constexpr int BT = 128;            // threads per edge block
constexpr int CHUNK_E = 1 << 16;   // edges per chunk (at least one whole node)
constexpr int JMAX = (E2F_MAX_L + 1) * (2 * E2F_MAX_L + 1) * (2 * E2F_MAX_L + 3) / 3;   // sum (2l+1)^2

// J_k^l = d/dt D^l(exp(t K_k)) at t = 0, k = x, y, z (K_k v = e_k x v),
// blocks laid out like the Wigner blocks; fitted on the host by a central
// difference of the Ivanic-Ruedenberg construction.  Global memory, not
// __constant__: the torque reads it at a different entry in every lane.
__device__ float g_gen[3 * JMAX];

struct Args {
  int L, C, H, N;
  float inv_sqrt_d;
  Geom g;
  const int32_t *row_ptr, *col_idx;
  const float *pos;
  const void *q, *k, *v;          // [N][Q][C], storage type
  const float *G;                 // dL/do [N][Q][C]
  const float *W1, *W2;
  // chunk
  int na, nb;                     // nodes [na, nb)
  int64_t ea, ne;                 // edges [ea, ea + ne)
  int32_t *dst;                   // [ne] destination node of each edge
  void *A, *dY;                   // [ne][QC] storage type (stacked)
  float *Y, *dA;                  // [ne][QC] fp32 (stacked)
  float *Dm, *gv, *zv, *sv, *uv, *rv, *al, *dal, *dsv, *duv, *dgv;
  float *Mv, *denv, *dlt;         // per node of the chunk [nb - na][H]
  // accumulators
  float *dq, *dk, *dv;            // [N][Q][C] fp32
  float *dpos;                    // [N][3]
};

template <typename T> __device__ __forceinline__ float ldf(const void *p, size_t i) {
  return to_f(static_cast<const T *>(p)[i]);
}

// K0: dst[e - ea] = n for every edge e of row n (warp per node, lanes over
// the row), so that the per-edge kernels get their node with one load
__global__ void edge_dst_kernel(Args a) {
  const int lane = threadIdx.x & 31;
  for (int n = a.na + blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); n < a.nb;
       n += gridDim.x * (blockDim.x >> 5)) {
    const int64_t e0 = a.row_ptr[n] - a.ea, e1 = a.row_ptr[n + 1] - a.ea;
    for (int64_t e = e0 + lane; e < e1; e += 32) a.dst[e] = n;
  }
}

// The next edge's destination node (and source node, D blocks), loaded one
// iteration of the CTA's serial edge loop ahead into registers, so that the
// dependent loads of an edge do not start with an index round trip.  The
// CTA has BT threads.
template <int S, bool J, bool DD>
struct EdgePrefetch {
  static constexpr int DPT = DD ? (S + BT - 1) / BT : 1;
  int i = 0, j = 0;
  float d[DPT];
  __device__ __forceinline__ void load(const Args &a, int64_t el) {
    if (el >= a.ne) return;
    i = a.dst[el];
    if (J) j = a.col_idx[a.ea + el];
    if (DD) {
#pragma unroll
      for (int k = 0; k < DPT; ++k) {
        const int x = threadIdx.x + k * BT;
        if (x < S) d[k] = a.Dm[el * S + x];
      }
    }
  }
  __device__ __forceinline__ void store_d(float *D) const {
#pragma unroll
    for (int k = 0; k < DPT; ++k) {
      const int x = threadIdx.x + k * BT;
      if (x < S) D[x] = d[k];
    }
  }
};

// ---------------------------------------------------------------------------
// K1: geometry, D, envelope, radial MLP, logits; v~ = D v_j (stacked).  One
// warp per edge (FWD_WARPS edges per CTA in flight, warp-level
// synchronisation only): most steps of an edge use a few lanes, so one edge
// per CTA would leave the CTA's other warps waiting at its barriers.
// ---------------------------------------------------------------------------
constexpr int FWD_WARPS = BT / 32;
constexpr int FWD_CPL = 2;   // channels per lane in the logits and the rotate-in

template <typename T, int L>
__global__ void __launch_bounds__(BT, 6) edge_fwd_kernel(Args a) {
  constexpr int Q = (L + 1) * (L + 1), S = L * (4 * L * L - 1) / 3 + (2 * L + 1) * (2 * L + 1);
  constexpr int P = (L + 1) * (L + 2) / 2;
  __shared__ float Dw[FWD_WARPS][S];
  __shared__ float hidw[FWD_WARPS][16];
  extern __shared__ float partw[];   // [FWD_WARPS][C]: per-channel logit partials
  const int C = a.C, QC = Q * C, H = a.H, Ch = C / H;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  float *D = Dw[warp], *hid = hidw[warp], *part = partw + warp * C;
  for (int64_t el = (int64_t)blockIdx.x * FWD_WARPS + warp; el < a.ne; el += (int64_t)gridDim.x * FWD_WARPS) {
    const int i = a.dst[el], j = a.col_idx[a.ea + el];
    __syncwarp();   // the previous edge's readers of D, hid and part are done
    // geometry (every lane; the two position loads are broadcasts)
    float dx, dy, dz;
    pair_disp(a.g, load_pos(a.pos, i), load_pos(a.pos, j), dx, dy, dz);
    const float r = sqrtf(dx * dx + dy * dy + dz * dz);
    if (lane == 0) {
      a.rv[el * 4 + 0] = dx; a.rv[el * 4 + 1] = dy; a.rv[el * 4 + 2] = dz; a.rv[el * 4 + 3] = r;
      a.uv[el] = 0.5f * (cospif(r / a.g.rc) + 1.f);
      // D^0, D^1 of the two-angle frame
      float ux = 0.f, uy = 0.f, uz = 1.f;
      if (r > 0.f) { ux = dx / r; uy = dy / r; uz = dz / r; }
      D[0] = 1.f;
      if (L >= 1) {
        float R[9];
        edge_frame_two_angle(ux, uy, uz, R);
        wig_l1_from_rotation(R, D + 1);
      }
    }
    // radial MLP: 8 Gaussians (centres k r_c / 7, sigma 0.5) -> 16 SiLU -> P
    if (lane >= 16) {
      const int h = lane - 16;
      float z = 0.f;
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        const float dd = r - (float)kk * (a.g.rc / 7.f);
        z = fmaf(a.W1[h * 8 + kk], expf(-dd * dd * 2.f), z);
      }
      a.zv[el * 16 + h] = z;
      hid[h] = z / (1.f + expf(-z));
    }
    __syncwarp();
    // D^l, l >= 2, by the Ivanic-Ruedenberg recursion, a level at a time
    for (int l = 2; l <= L; ++l) {
      const int w = 2 * l + 1;
      for (int x = lane; x < w * w; x += 32)
        D[wig_offset(l) + x] = wig_entry(l, x / w - l, x % w - l, D + 1, D + wig_offset(l - 1));
      __syncwarp();
    }
    for (int x = lane; x < S; x += 32) a.Dm[el * S + x] = D[x];
    for (int p = lane; p < P; p += 32) {
      float gg = 0.f;
#pragma unroll
      for (int hh = 0; hh < 16; ++hh) gg = fmaf(a.W2[p * 16 + hh], hid[hh], gg);
      a.gv[el * P + p] = gg;
    }
    // logits: the m = 0 rows of D q_i and D k_j, per head.  A lane takes
    // FWD_CPL channels (32 apart) at once, so each D entry is read once for
    // all of them.
    for (int c0 = lane; c0 < C; c0 += 32 * FWD_CPL) {
      float s[FWD_CPL];
#pragma unroll
      for (int r = 0; r < FWD_CPL; ++r) s[r] = 0.f;
#pragma unroll
      for (int l = 0; l <= L; ++l) {
        asm volatile("" ::: "memory");   // one degree's loads in flight at a time
        const int w = 2 * l + 1;
        const float *row0 = D + wig_offset(l) + l * w;
        float qh[FWD_CPL], kh[FWD_CPL];
#pragma unroll
        for (int r = 0; r < FWD_CPL; ++r) qh[r] = kh[r] = 0.f;
#pragma unroll
        for (int mp = 0; mp < w; ++mp) {
          const float d = row0[mp];
#pragma unroll
          for (int r = 0; r < FWD_CPL; ++r) {
            const int c = c0 + 32 * r;
            if (c < C) {
              qh[r] = fmaf(d, ldf<T>(a.q, ((size_t)i * Q + l * l + mp) * C + c), qh[r]);
              kh[r] = fmaf(d, ldf<T>(a.k, ((size_t)j * Q + l * l + mp) * C + c), kh[r]);
            }
          }
        }
#pragma unroll
        for (int r = 0; r < FWD_CPL; ++r) s[r] = fmaf(qh[r], kh[r], s[r]);
      }
#pragma unroll
      for (int r = 0; r < FWD_CPL; ++r)
        if (c0 + 32 * r < C) part[c0 + 32 * r] = s[r];
    }
    __syncwarp();
    if (lane < H) {
      float hsum = 0.f;
      for (int c = lane * Ch; c < (lane + 1) * Ch; ++c) hsum += part[c];
      a.sv[el * H + lane] = hsum * a.inv_sqrt_d;
    }
    // rotate in: v~[(l,m),c] = sum_m' D^l[m][m'] v_j[(l,m'),c], stacked; a
    // lane takes FWD_CPL channels at once (each D entry read once for all)
    T *Arow = static_cast<T *>(a.A) + (size_t)el * QC;
    for (int c0 = lane; c0 < C; c0 += 32 * FWD_CPL) {
#pragma unroll
      for (int l = 0; l <= L; ++l) {
        asm volatile("" ::: "memory");   // one degree's loads in flight at a time
        const int w = 2 * l + 1;
        float vv[FWD_CPL][2 * L + 1];
#pragma unroll
        for (int r = 0; r < FWD_CPL; ++r) {
          const int c = c0 + 32 * r;
#pragma unroll
          for (int mp = 0; mp < w; ++mp) vv[r][mp] = c < C ? ldf<T>(a.v, ((size_t)j * Q + l * l + mp) * C + c) : 0.f;
        }
        const float *Dl = D + wig_offset(l);
#pragma unroll
        for (int m = -l; m <= l; ++m) {
          float acc[FWD_CPL];
#pragma unroll
          for (int r = 0; r < FWD_CPL; ++r) acc[r] = 0.f;
#pragma unroll
          for (int mp = 0; mp < w; ++mp) {
            const float d = Dl[(m + l) * w + mp];
#pragma unroll
            for (int r = 0; r < FWD_CPL; ++r) acc[r] = fmaf(d, vv[r][mp], acc[r]);
          }
          const int so = stack_off(L, C, m) + (l - (m < 0 ? -m : m)) * C;
#pragma unroll
          for (int r = 0; r < FWD_CPL; ++r)
            if (c0 + 32 * r < C) Arow[so + c0 + 32 * r] = from_f<T>(acc[r]);
        }
      }
    }
  }
}

// ---------------------------------------------------------------------------
// K2 / K4: per (node, head) reductions over the node's edges (warp per node)
// ---------------------------------------------------------------------------
__global__ void node_stats_kernel(Args a) {
  const int lane = threadIdx.x & 31;
  for (int n = a.na + blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); n < a.nb;
       n += gridDim.x * (blockDim.x >> 5)) {
    const int64_t e0 = a.row_ptr[n] - a.ea, e1 = a.row_ptr[n + 1] - a.ea;
    if (lane < a.H) {
      float M = -INFINITY;
      for (int64_t e = e0; e < e1; ++e) M = fmaxf(M, a.sv[e * a.H + lane] + logf(a.uv[e]));
      float den = 0.f;
      if (M > -INFINITY)
        for (int64_t e = e0; e < e1; ++e) den += expf(a.sv[e * a.H + lane] + logf(a.uv[e]) - M);
      a.Mv[(size_t)(n - a.na) * a.H + lane] = M;
      a.denv[(size_t)(n - a.na) * a.H + lane] = den;
    }
  }
}

__global__ void node_delta_kernel(Args a) {
  const int lane = threadIdx.x & 31;
  for (int n = a.na + blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); n < a.nb;
       n += gridDim.x * (blockDim.x >> 5)) {
    const int64_t e0 = a.row_ptr[n] - a.ea, e1 = a.row_ptr[n + 1] - a.ea;
    if (lane < a.H) {
      float d = 0.f;
      for (int64_t e = e0; e < e1; ++e) d = fmaf(a.al[e * a.H + lane], a.dal[e * a.H + lane], d);
      a.dlt[(size_t)(n - a.na) * a.H + lane] = d;
    }
  }
}

// GD[(l,m),c] = sum_m' D^l[m][m'] G_i[(l,m'),c] for one (l, c)
template <int L>
__device__ __forceinline__ void rotate_col(const float *D, const float *src, int l, int c, int C, float *out) {
  const int w = 2 * l + 1;
  float gg[2 * L + 1];
#pragma unroll
  for (int mp = 0; mp < 2 * L + 1; ++mp) gg[mp] = mp < w ? src[(size_t)(l * l + mp) * C + c] : 0.f;
  const float *Dl = D + wig_offset(l);
#pragma unroll
  for (int m = 0; m < 2 * L + 1; ++m) {
    if (m >= w) break;
    float acc = 0.f;
#pragma unroll
    for (int mp = 0; mp < 2 * L + 1; ++mp)
      if (mp < w) acc = fmaf(Dl[m * w + mp], gg[mp], acc);
    out[m] = acc;
  }
}

// ---------------------------------------------------------------------------
// K3: alpha and dalpha per (edge, head)
// ---------------------------------------------------------------------------
template <int L>
__global__ void __launch_bounds__(BT, 4) edge_dalpha_kernel(Args a) {
  constexpr int Q = (L + 1) * (L + 1), S = L * (4 * L * L - 1) / 3 + (2 * L + 1) * (2 * L + 1);
  constexpr int P = (L + 1) * (L + 2) / 2;
  __shared__ float D[S];
  extern __shared__ float part[];   // [C]: per-channel partials of dL/dalpha
  const int C = a.C, QC = Q * C, H = a.H, Ch = C / H;
  EdgePrefetch<S, false, true> pf;
  pf.load(a, blockIdx.x);
  for (int64_t el = blockIdx.x; el < a.ne; el += gridDim.x) {
    const int i = pf.i;
    __syncthreads();
    pf.store_d(D);
    pf.load(a, el + gridDim.x);
    __syncthreads();
    const float *Gi = a.G + (size_t)i * QC;
    const float *Yr = a.Y + (size_t)el * QC;
    const float *gvp = a.gv + el * P;
    for (int c = threadIdx.x; c < C; c += blockDim.x) {
      float sacc = 0.f;
#pragma unroll
      for (int l = 0; l <= L; ++l) {
        float gd[2 * L + 1];
        asm volatile("" ::: "memory");   // one degree's loads in flight at a time (no spills)
        rotate_col<L>(D, Gi, l, c, C, gd);
#pragma unroll
        for (int m = -l; m <= l; ++m) {
          const int am = m < 0 ? -m : m;
          const float y = gvp[pair_index(L, am, l)] * Yr[stack_off(L, C, m) + (l - am) * C + c];
          sacc = fmaf(y, gd[m + l], sacc);
        }
      }
      part[c] = sacc;
    }
    __syncthreads();
    if (threadIdx.x < H) {
      const int h = threadIdx.x;
      float hsum = 0.f;
      for (int c = h * Ch; c < (h + 1) * Ch; ++c) hsum += part[c];
      const float M = a.Mv[(size_t)(i - a.na) * H + h], den = a.denv[(size_t)(i - a.na) * H + h];
      const float sp = a.sv[el * H + h] + logf(a.uv[el]);
      a.al[el * H + h] = (den > 0.f && M > -INFINITY) ? expf(sp - M) / den : 0.f;
      a.dal[el * H + h] = hsum;
    }
  }
}

// ---------------------------------------------------------------------------
// K5: ds, dL/du, dy = alpha GD, dL/dg, dw = g dy (stacked).  Channel-major:
// a thread takes channel c through every (l, m) (compile-time), and the
// per-(m, l) sums dL/dg are warp reductions over a padded [Q][C + 1] table
// of products (no shared-memory atomics).
// ---------------------------------------------------------------------------
template <typename T, int L>
__global__ void __launch_bounds__(BT, 6) edge_dy_kernel(Args a) {
  constexpr int Q = (L + 1) * (L + 1), S = L * (4 * L * L - 1) / 3 + (2 * L + 1) * (2 * L + 1);
  constexpr int P = (L + 1) * (L + 2) / 2;
  extern __shared__ float prod[];   // [Q][C + 1]: dy * Y per (l, m), channel
  __shared__ float D[S];
  __shared__ float alh[16];
  const int C = a.C, CP = C + 1, QC = Q * C, H = a.H, Ch = C / H;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  EdgePrefetch<S, false, true> pf;
  pf.load(a, blockIdx.x);
  for (int64_t el = blockIdx.x; el < a.ne; el += gridDim.x) {
    const int i = pf.i;
    __syncthreads();
    pf.store_d(D);
    pf.load(a, el + gridDim.x);
    if (warp == 0) {
      // ds_h = alpha_h (dalpha_h - Delta_h); dL/du = sum_h e^(s - M) / den
      // (dalpha_h - Delta_h)  (no division by u), summed over the lanes
      float du = 0.f;
      if (lane < H) {
        const int h = lane;
        const size_t nh = (size_t)(i - a.na) * H + h;
        const float al = a.al[el * H + h], diff = a.dal[el * H + h] - a.dlt[nh];
        alh[h] = al;
        a.dsv[el * H + h] = al * diff;
        const float M = a.Mv[nh], den = a.denv[nh];
        if (den > 0.f && M > -INFINITY) du = expf(a.sv[el * H + h] - M) / den * diff;
      }
      du = warp_sum(du);
      if (lane == 0) a.duv[el] = du;
    }
    __syncthreads();
    const float *Gi = a.G + (size_t)i * QC;
    const float *Yr = a.Y + (size_t)el * QC;
    const float *gvp = a.gv + el * P;
    T *dYr = static_cast<T *>(a.dY) + (size_t)el * QC;
    for (int c = threadIdx.x; c < C; c += blockDim.x) {
      const float alc = alh[c / Ch];
#pragma unroll
      for (int l = 0; l <= L; ++l) {
        float gd[2 * L + 1];
        asm volatile("" ::: "memory");   // one degree's loads in flight at a time (no spills)
        rotate_col<L>(D, Gi, l, c, C, gd);
#pragma unroll
        for (int m = -l; m <= l; ++m) {
          const int am = m < 0 ? -m : m;
          const int so = stack_off(L, C, m) + (l - am) * C + c;
          const float dy = alc * gd[m + l];
          prod[(l * l + l + m) * CP + c] = dy * Yr[so];
          dYr[so] = from_f<T>(dy * gvp[pair_index(L, am, l)]);
        }
      }
    }
    __syncthreads();
    for (int p = warp; p < P; p += nw) {
      int m = 0, rem = p;   // (m, l) of pair p
      while (rem > L - m) { rem -= L - m + 1; ++m; }
      const int l = m + rem;
      float sacc = 0.f;
      for (int c = lane; c < C; c += 32) {
        sacc += prod[(l * l + l + m) * CP + c];
        if (m > 0) sacc += prod[(l * l + l - m) * CP + c];
      }
      sacc = warp_sum(sacc);
      if (lane == 0) a.dgv[el * P + p] = sacc;
    }
  }
}

// four consecutive values as floats (16-byte / 8-byte aligned)
__device__ __forceinline__ float4 ld4f(const float *p) { return *reinterpret_cast<const float4 *>(p); }
__device__ __forceinline__ float4 ld4f(const __nv_bfloat16 *p) {
  const uint2 u = *reinterpret_cast<const uint2 *>(p);
  const float2 lo = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&u.x));
  const float2 hi = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&u.y));
  return make_float4(lo.x, lo.y, hi.x, hi.y);
}

// One row (l, m) = q of dL/dD^l from the staged rows: this lane's partial over
// the 4-channel chunks 4 qq, 4 qq + 16, ... (C a multiple of 16), summed over
// the four lanes of the row (mask quad) and stored by the first of them.
template <int LL, typename T>
__device__ __forceinline__ void dd_row_l(int rr, int qq, unsigned quad, int C, int CP, int CPV, const float *dvt,
                                         const T *vj, const float *yv, const float *dz, float *dD) {
  constexpr int W = 2 * LL + 1;
  const int q = LL * LL + rr;
  const float *pa = dvt + q * CP, *ya = yv + q * CP;
  const T *vb = vj + LL * LL * CPV;
  const float *zb = dz + LL * LL * CP;
  float acc[W];
#pragma unroll
  for (int cc = 0; cc < W; ++cc) acc[cc] = 0.f;
  for (int c = 4 * qq; c < C; c += 16) {
    const float4 xa = ld4f(pa + c), za = ld4f(ya + c);
#pragma unroll
    for (int cc = 0; cc < W; ++cc) {
      const float4 xb = ld4f(vb + cc * CPV + c), zz = ld4f(zb + cc * CP + c);
      acc[cc] = fmaf(xa.x, xb.x, fmaf(xa.y, xb.y, fmaf(xa.z, xb.z, fmaf(xa.w, xb.w, acc[cc]))));
      acc[cc] = fmaf(za.x, zz.x, fmaf(za.y, zz.y, fmaf(za.z, zz.z, fmaf(za.w, zz.w, acc[cc]))));
    }
  }
#pragma unroll
  for (int cc = 0; cc < W; ++cc) {
    acc[cc] += __shfl_xor_sync(quad, acc[cc], 1);
    acc[cc] += __shfl_xor_sync(quad, acc[cc], 2);
  }
  if (qq == 0) {
#pragma unroll
    for (int cc = 0; cc < W; ++cc) dD[wig_offset(LL) + rr * W + cc] = acc[cc];
  }
}

template <typename T, int L>
__device__ __forceinline__ void dd_row(int q, int qq, unsigned quad, int C, int CP, int CPV, const float *dvt,
                                       const T *vj, const float *yv, const float *dz, float *dD) {
  int l = 0;
  while ((l + 1) * (l + 1) <= q) ++l;
  const int rr = q - l * l;
  switch (l) {
#define E2F_DD_ROW(LL) \
  case LL: if (LL <= L) dd_row_l<(LL <= L ? LL : 0), T>(rr, qq, quad, C, CP, CPV, dvt, vj, yv, dz, dD); break;
    E2F_DD_ROW(0) E2F_DD_ROW(1) E2F_DD_ROW(2) E2F_DD_ROW(3) E2F_DD_ROW(4) E2F_DD_ROW(5) E2F_DD_ROW(6)
#undef E2F_DD_ROW
    default: break;
  }
}

// ---------------------------------------------------------------------------
// K6: dL/dD, torque, radius; atomics into dpos, dq, dk, dv.  Channel-major
// staging into padded [Q][C + 1] rows (a thread per channel, (l, m) at
// compile time), then one dL/dD entry per thread as a C-long dot product
// over the padded rows (conflict-free), the m = 0 row terms as warp
// reductions, and the scatter of dv, dq, dk with consecutive threads on
// consecutive channels.
// ---------------------------------------------------------------------------
template <typename T, int L>
__global__ void __launch_bounds__(BT, 4) edge_bwd_kernel(Args a) {
  constexpr int Q = (L + 1) * (L + 1), S = L * (4 * L * L - 1) / 3 + (2 * L + 1) * (2 * L + 1);
  constexpr int P = (L + 1) * (L + 2) / 2;
  extern __shared__ float sm[];
  // rows padded to C + 4 floats: 16-byte aligned for the vector dot products,
  // and rows of different (l, m) start 4 banks apart (conflict-free for the
  // eight threads of one 128-byte phase)
  // v_j is staged in its storage type (exact), rows padded to 16 bytes more
  const int C = a.C, CP = C + 4, CPV = C + 16 / (int)sizeof(T), QC = Q * C, H = a.H, Ch = C / H;
  float *dvt = sm;                                         // [Q][CP]  dL/dv~ (unstacked)
  T *vj = reinterpret_cast<T *>(dvt + Q * CP);             // [Q][CPV]
  float *yv = dvt + Q * CP + (Q * CPV * (int)sizeof(T) + 15) / 16 * 4;   // [Q][CP]  y = g Y (unstacked)
  float *dz = yv + Q * CP;                                 // [Q][CP]  alpha G_i
  float *qk = dz + Q * CP;                                 // [2][L+1][C]  ds q~0, ds k~0 (/ sqrt d)
  __shared__ float D[S], dD[S], dD0[Q];
  __shared__ float dsh[16], misc[32], tau[3];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  EdgePrefetch<S, true, true> pf;
  pf.load(a, blockIdx.x);
  for (int64_t el = blockIdx.x; el < a.ne; el += gridDim.x) {
    const int i = pf.i, j = pf.j;
    __syncthreads();
    pf.store_d(D);
    pf.load(a, el + gridDim.x);
    if (threadIdx.x < H) dsh[threadIdx.x] = a.dsv[el * H + threadIdx.x] * a.inv_sqrt_d;
    if (threadIdx.x < 3) tau[threadIdx.x] = 0.f;
    __syncthreads();
    const float *Gi = a.G + (size_t)i * QC;
    const float *Yr = a.Y + (size_t)el * QC, *dAr = a.dA + (size_t)el * QC;
    const float *gvp = a.gv + el * P;
    const T *qi = static_cast<const T *>(a.q) + (size_t)i * QC;
    const T *kj = static_cast<const T *>(a.k) + (size_t)j * QC;
    const T *vjr = static_cast<const T *>(a.v) + (size_t)j * QC;
    for (int c = threadIdx.x; c < C; c += blockDim.x) {
      const float alc = a.al[el * H + c / Ch], dsc = dsh[c / Ch];
#pragma unroll
      for (int l = 0; l <= L; ++l) {
        asm volatile("" ::: "memory");   // one degree's loads in flight at a time
        const float *row0 = D + wig_offset(l) + l * (2 * l + 1);
        float qh = 0.f, kh = 0.f;
#pragma unroll
        for (int m = -l; m <= l; ++m) {
          const int am = m < 0 ? -m : m, q = l * l + l + m;
          const int so = stack_off(L, C, m) + (l - am) * C + c;
          dvt[q * CP + c] = dAr[so];
          vj[q * CPV + c] = vjr[(size_t)q * C + c];
          yv[q * CP + c] = gvp[pair_index(L, am, l)] * Yr[so];
          dz[q * CP + c] = alc * Gi[(size_t)q * C + c];
          qh = fmaf(row0[m + l], to_f(qi[(size_t)q * C + c]), qh);
          kh = fmaf(row0[m + l], to_f(kj[(size_t)q * C + c]), kh);
        }
        qk[l * C + c] = dsc * qh;               // dk~0 = ds q~0 / sqrt d
        qk[(L + 1) * C + l * C + c] = dsc * kh; // dq~0 = ds k~0 / sqrt d
      }
    }
    __syncthreads();
    // dL/dD^l[m][m'] = sum_c dv~[m] v_j[m'] + y[m] dz[m'] ...
    if ((C & 15) == 0) {
      // four lanes per row (l, m) of dD^l, each over every fourth 4-channel
      // chunk and all 2l + 1 entries of the row, so that the row's dv~ and y
      // chunks are read once; the four partials are then summed by shuffles
      const int qq = threadIdx.x & 3;
      const unsigned quad = 0xFu << (lane & ~3);
      for (int q = threadIdx.x >> 2; q < Q; q += blockDim.x >> 2)
        dd_row<T, L>(q, qq, quad, C, CP, CPV, dvt, vj, yv, dz, dD);
    } else {
      for (int ent = threadIdx.x; ent < S; ent += blockDim.x) {
        int l = 0;
        while (wig_offset(l + 1) <= ent) ++l;
        const int w = 2 * l + 1, rr = (ent - wig_offset(l)) / w, cc = (ent - wig_offset(l)) % w;
        const float *pa = dvt + (l * l + rr) * CP;
        const T *pb = vj + (l * l + cc) * CPV;
        const float *ya = yv + (l * l + rr) * CP, *zb = dz + (l * l + cc) * CP;
        float s0 = 0.f;
        for (int c = 0; c < C; ++c) s0 = fmaf(pa[c], to_f(pb[c]), fmaf(ya[c], zb[c], s0));
        dD[ent] = s0;
      }
    }
    // ... + the m = 0 row: dq~0 q_i[m'] + dk~0 k_j[m'] (one warp per (l, m'),
    // lanes over channels)
    for (int idx = warp; idx < Q; idx += nw) {
      int l = 0;
      while ((l + 1) * (l + 1) <= idx) ++l;
      float sacc = 0.f;
#pragma unroll 4
      for (int c = lane; c < C; c += 32)
        sacc += qk[(L + 1) * C + l * C + c] * to_f(qi[(size_t)idx * C + c]) +
                qk[l * C + c] * to_f(kj[(size_t)idx * C + c]);
      sacc = warp_sum(sacc);
      if (lane == 0) dD0[idx] = sacc;
    }
    __syncthreads();
    for (int idx = threadIdx.x; idx < Q; idx += blockDim.x) {
      int l = 0;
      while ((l + 1) * (l + 1) <= idx) ++l;
      dD[wig_offset(l) + l * (2 * l + 1) + (idx - l * l)] += dD0[idx];
    }
    __syncthreads();
    // torque tau_k = -<D^T dD, J_k>, one (l, a, b) entry per thread
    {
      float t0 = 0.f, t1 = 0.f, t2 = 0.f;
      for (int ent = threadIdx.x; ent < S; ent += blockDim.x) {
        int l = 0;
        while (wig_offset(l + 1) <= ent) ++l;
        const int w = 2 * l + 1, ra = (ent - wig_offset(l)) / w, cb = (ent - wig_offset(l)) % w;
        const float *Dl = D + wig_offset(l), *dDl = dD + wig_offset(l);
        float mab = 0.f;   // (D^T dD)[ra][cb]
        for (int m = 0; m < w; ++m) mab = fmaf(Dl[m * w + ra], dDl[m * w + cb], mab);
        t0 = fmaf(mab, __ldg(&g_gen[ent]), t0);
        t1 = fmaf(mab, __ldg(&g_gen[JMAX + ent]), t1);
        t2 = fmaf(mab, __ldg(&g_gen[2 * JMAX + ent]), t2);
      }
      t0 = warp_sum(t0); t1 = warp_sum(t1); t2 = warp_sum(t2);
      if (lane == 0) { atomicAdd(&tau[0], -t0); atomicAdd(&tau[1], -t1); atomicAdd(&tau[2], -t2); }
    }
    // radial: dL/dg -> hidden -> RBF -> r, plus the envelope
    if (warp == 0) {
      float dr = 0.f;
      const float r = a.rv[el * 4 + 3];
      if (lane < 16) {
        float dh = 0.f;
        for (int p = 0; p < P; ++p) dh = fmaf(a.dgv[el * P + p], a.W2[p * 16 + lane], dh);
        const float z = a.zv[el * 16 + lane], sg = 1.f / (1.f + expf(-z));
        misc[lane] = dh * sg * (1.f + z * (1.f - sg));   // dL/dz (SiLU')
      }
      __syncwarp();
      if (lane < 8) {
        float dphi = 0.f;
        for (int hh = 0; hh < 16; ++hh) dphi = fmaf(misc[hh], a.W1[hh * 8 + lane], dphi);
        const float mu = (float)lane * (a.g.rc / 7.f), dd = r - mu;
        dr = dphi * expf(-dd * dd * 2.f) * (-dd * 4.f);   // d phi / dr = -phi (r - mu) / sigma^2
      }
      dr = warp_sum(dr);
      if (lane == 0) misc[16] = dr + a.duv[el] * (-0.5f * 3.14159265358979f / a.g.rc) * sinpif(r / a.g.rc);
    }
    __syncthreads();
    if (threadIdx.x == 0) {
      const float dx = a.rv[el * 4 + 0], dy = a.rv[el * 4 + 1], dzz = a.rv[el * 4 + 2], r = a.rv[el * 4 + 3];
      float gx = 0.f, gy = 0.f, gz = 0.f;
      if (r > 0.f) {
        const float ux = dx / r, uy = dy / r, uz = dzz / r, dr = misc[16];
        // (tau x rhat) / r
        gx = dr * ux + (tau[1] * uz - tau[2] * uy) / r;
        gy = dr * uy + (tau[2] * ux - tau[0] * uz) / r;
        gz = dr * uz + (tau[0] * uy - tau[1] * ux) / r;
      }
      atomicAdd(&a.dpos[3 * j + 0], gx); atomicAdd(&a.dpos[3 * j + 1], gy); atomicAdd(&a.dpos[3 * j + 2], gz);
      atomicAdd(&a.dpos[3 * i + 0], -gx); atomicAdd(&a.dpos[3 * i + 1], -gy); atomicAdd(&a.dpos[3 * i + 2], -gz);
    }
    // dv_j += D^T dv~; dq_i, dk_j += row0^T dq~0 / dk~0 (consecutive threads
    // on consecutive channels)
    for (int c = threadIdx.x; c < C; c += blockDim.x) {
#pragma unroll
      for (int l = 0; l <= L; ++l) {
        const int w = 2 * l + 1;
        const float *Dl = D + wig_offset(l);
        const float gq = qk[(L + 1) * C + l * C + c], gk = qk[l * C + c];
#pragma unroll
        for (int mp = 0; mp < w; ++mp) {
          float acc = 0.f;
#pragma unroll
          for (int m = 0; m < w; ++m) acc = fmaf(Dl[m * w + mp], dvt[(l * l + m) * CP + c], acc);
          const size_t o = (size_t)(l * l + mp) * C + c;
          atomicAdd(&a.dv[(size_t)j * QC + o], acc);
          const float r0 = Dl[l * w + mp];
          atomicAdd(&a.dq[(size_t)i * QC + o], r0 * gq);
          atomicAdd(&a.dk[(size_t)j * QC + o], r0 * gk);
        }
      }
    }
  }
}

// fp32 copy of a weight matrix (the dL/dx GEMMs run in fp32)
template <typename T>
__global__ void to_f32_kernel(const T *src, int64_t n, float *dst) {
  for (int64_t x = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; x < n; x += (int64_t)gridDim.x * blockDim.x)
    dst[x] = to_f(src[x]);
}

// Wc_m = [[Wr, -Wi], [Wi, Wr]] (2n x 2n, row-major), m >= 1
template <typename T>
__global__ void complex_block_kernel(const T *Wr, const T *Wi, int n, T *out) {
  const int64_t tot = 4LL * n * n;
  for (int64_t x = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; x < tot; x += (int64_t)gridDim.x * blockDim.x) {
    const int r = (int)(x / (2 * n)), c = (int)(x % (2 * n));
    const int rb = r / n, cb = c / n, ri = r % n, ci = c % n;
    const float vr = to_f(Wr[(size_t)ri * n + ci]), vi = to_f(Wi[(size_t)ri * n + ci]);
    float v;
    if (rb == 0) v = (cb == 0) ? vr : -vi;
    else v = (cb == 0) ? vi : vr;
    out[x] = from_f<T>(v);
  }
}

// ---------------------------------------------------------------------------
// host
// ---------------------------------------------------------------------------
static std::once_flag g_gen_once;
static float g_gen_tab[3 * JMAX];
static std::mutex g_gen_mu;
static bool g_gen_up[64] = {};

static void fit_generators() {
  // J_k^l = (D(R_k(+eps)) - D(R_k(-eps))) / (2 eps), R_k(t) = exp(t K_k)
  const double eps = 1e-5;
  std::vector<double> Dp(JMAX), Dm(JMAX);
  for (int k = 0; k < 3; ++k) {
    for (int sgn = 0; sgn < 2; ++sgn) {
      const double t = sgn ? -eps : eps, c = cos(t), s = sin(t);
      double R[9];
      if (k == 0) { double RR[9] = {1, 0, 0, 0, c, -s, 0, s, c}; for (int x = 0; x < 9; ++x) R[x] = RR[x]; }
      else if (k == 1) { double RR[9] = {c, 0, s, 0, 1, 0, -s, 0, c}; for (int x = 0; x < 9; ++x) R[x] = RR[x]; }
      else { double RR[9] = {c, -s, 0, s, c, 0, 0, 0, 1}; for (int x = 0; x < 9; ++x) R[x] = RR[x]; }
      wig_all_serial<double>(R, E2F_MAX_L, sgn ? Dm.data() : Dp.data());
    }
    for (int x = 0; x < JMAX; ++x) g_gen_tab[k * JMAX + x] = (float)((Dp[x] - Dm[x]) / (2 * eps));
  }
}

static e2f_status ensure_generators() {
  std::call_once(g_gen_once, fit_generators);
  int dev = 0;
  E2F_CUDA_TRY(cudaGetDevice(&dev));
  if (dev < 0 || dev >= 64) return E2F_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lk(g_gen_mu);
  if (!g_gen_up[dev]) {
    E2F_CUDA_TRY(cudaMemcpyToSymbol(g_gen, g_gen_tab, sizeof(g_gen_tab)));
    g_gen_up[dev] = true;
  }
  return E2F_OK;
}

// One cuBLAS handle per (host thread, device): a handle carries the stream
// it was last given, so calls from different threads on different streams
// must not share one.
static thread_local cublasHandle_t tl_blas[64] = {};

static e2f_status blas_handle(cublasHandle_t *h, cudaStream_t s) {
  int dev = 0;
  E2F_CUDA_TRY(cudaGetDevice(&dev));
  if (dev < 0 || dev >= 64) return E2F_ERR_UNSUPPORTED;
  if (!tl_blas[dev] && cublasCreate(&tl_blas[dev]) != CUBLAS_STATUS_SUCCESS) return E2F_ERR_CUDA;
  if (cublasSetStream(tl_blas[dev], s) != CUBLAS_STATUS_SUCCESS) return E2F_ERR_CUDA;
  *h = tl_blas[dev];
  return E2F_OK;
}

// C[E][w] (ld QC) = A[E][w] (ld QC) op(Wc): trans = true -> A Wc^T, false -> A Wc
template <typename T>
static e2f_status stacked_gemm(cublasHandle_t h, const T *Wc, int w, const void *A, float *Cout, int64_t E, int QC,
                               bool trans) {
  const float one = 1.f, zero = 0.f;
  const cudaDataType_t dt = std::is_same<T, float>::value ? CUDA_R_32F : CUDA_R_16BF;
  // column-major view: C^T [w x E] = op(Wc') [w x w] * A^T [w x E], with the
  // row-major Wc seen as Wc^T
  const cublasStatus_t st = cublasGemmEx(h, trans ? CUBLAS_OP_T : CUBLAS_OP_N, CUBLAS_OP_N, w, (int)E, w, &one, Wc, dt,
                                         w, A, dt, QC, &zero, Cout, CUDA_R_32F, QC, CUBLAS_COMPUTE_32F,
                                         CUBLAS_GEMM_DEFAULT);
  return st == CUBLAS_STATUS_SUCCESS ? E2F_OK : E2F_ERR_CUDA;
}

template <typename T, int L>
static e2f_status run(const void *x, const float *pos, const e2f_csr *csr, const e2f_weights *w, const float *G,
                      float *dx, float *dpos, cudaStream_t s) {
  constexpr int Q = (L + 1) * (L + 1), S = L * (4 * L * L - 1) / 3 + (2 * L + 1) * (2 * L + 1);
  constexpr int P = (L + 1) * (L + 2) / 2;
  const int C = w->C, H = w->H, QC = Q * C;
  const int64_t N = csr->n_nodes;
  e2f_status st = ensure_generators();
  if (st != E2F_OK) return st;
  cublasHandle_t bh;
  st = blas_handle(&bh, s);
  if (st != E2F_OK) return st;
  auto up = [](size_t b) { return (b + 255) & ~(size_t)255; };
  const size_t feat = (size_t)N * QC;
  // q, k, v and the fp32 accumulators dq, dk, dv
  Scratch node;
  const size_t o_qkv = 0, o_acc = up(3 * feat * sizeof(T));
  E2F_CUDA_TRY(node.alloc(o_acc + 3 * feat * sizeof(float), s));
  char *nb = node.as<char>();
  T *q = reinterpret_cast<T *>(nb + o_qkv), *k = q + feat, *v = k + feat;
  float *dq = reinterpret_cast<float *>(nb + o_acc), *dk = dq + feat, *dv = dk + feat;
  st = project_impl(x, N, w, q, k, v, s);
  if (st != E2F_OK) return st;
  E2F_CUDA_TRY(cudaMemsetAsync(dq, 0, 3 * feat * sizeof(float), s));
  E2F_CUDA_TRY(cudaMemsetAsync(dpos, 0, (size_t)N * 3 * sizeof(float), s));
  // complex SO(2) blocks
  std::vector<size_t> woff(L + 1);
  size_t wtot = 0;
  for (int m = 0; m <= L; ++m) {
    const size_t wm = m == 0 ? (size_t)(L + 1) * C : 2 * (size_t)(L - m + 1) * C;
    woff[m] = wtot;
    wtot += up(wm * wm * sizeof(T)) / sizeof(T);
  }
  Scratch wcs;
  E2F_CUDA_TRY(wcs.alloc(wtot * sizeof(T), s));
  T *wc = wcs.as<T>();
  E2F_CUDA_TRY(cudaMemcpyAsync(wc, w->W0, sizeof(T) * (size_t)(L + 1) * C * (L + 1) * C, cudaMemcpyDeviceToDevice, s));
  for (int m = 1; m <= L; ++m) {
    const int n = (L - m + 1) * C;
    E2F_LAUNCH(complex_block_kernel<T>, 256, 256, 0, s, static_cast<const T *>(w->Wr[m]),
               static_cast<const T *>(w->Wi[m]), n, wc + woff[m]);
  }
  // chunks of whole nodes (host copy of row_ptr: one synchronisation)
  std::vector<int32_t> rp(N + 1);
  E2F_CUDA_TRY(cudaMemcpyAsync(rp.data(), csr->row_ptr, sizeof(int32_t) * (N + 1), cudaMemcpyDeviceToHost, s));
  E2F_CUDA_TRY(cudaStreamSynchronize(s));
  int64_t maxce = 0;
  std::vector<std::pair<int, int>> chunks;
  for (int n0 = 0; n0 < N;) {
    int n1 = n0 + 1;
    while (n1 < N && (int64_t)rp[n1 + 1] - rp[n0] <= CHUNK_E) ++n1;
    chunks.emplace_back(n0, n1);
    maxce = std::max<int64_t>(maxce, (int64_t)rp[n1] - rp[n0]);
    n0 = n1;
  }
  int64_t maxcn = 0;
  for (auto &c : chunks) maxcn = std::max<int64_t>(maxcn, c.second - c.first);
  const size_t ce = (size_t)std::max<int64_t>(maxce, 1), cn = (size_t)std::max<int64_t>(maxcn, 1);
  size_t off = 0;
  auto carve = [&](size_t bytes) { const size_t o = off; off += up(bytes); return o; };
  const size_t oA = carve(ce * QC * sizeof(T)), odY = carve(ce * QC * sizeof(T));
  const size_t oY = carve(ce * QC * 4), odA = carve(ce * QC * 4), oD = carve(ce * S * 4), og = carve(ce * P * 4);
  const size_t oz = carve(ce * 16 * 4), os = carve(ce * H * 4), ou = carve(ce * 4), orr = carve(ce * 16);
  const size_t oal = carve(ce * H * 4), odal = carve(ce * H * 4), ods = carve(ce * H * 4), odu = carve(ce * 4);
  const size_t odg = carve(ce * P * 4), oM = carve(cn * H * 4), oden = carve(cn * H * 4), odl = carve(cn * H * 4);
  const size_t odst = carve(ce * 4);
  Scratch cs;
  E2F_CUDA_TRY(cs.alloc(off, s));
  char *cb = cs.as<char>();
  Args a;
  a.L = L; a.C = C; a.H = H; a.N = (int)N;
  a.inv_sqrt_d = 1.f / sqrtf((float)((L + 1) * (C / H)));
  for (int kk = 0; kk < 3; ++kk) {
    a.g.box[kk] = csr->box[kk] > 0.f ? csr->box[kk] : 0.f;
    a.g.half[kk] = 0.5f * a.g.box[kk];
    a.g.periodic[kk] = csr->box[kk] > 0.f;
  }
  a.g.rc = csr->r_c; a.g.rc2 = csr->r_c * csr->r_c;
  a.row_ptr = csr->row_ptr; a.col_idx = csr->col_idx; a.pos = pos;
  a.q = q; a.k = k; a.v = v; a.G = G; a.W1 = w->rad_W1; a.W2 = w->rad_W2;
  a.A = cb + oA; a.dY = cb + odY;
  a.Y = reinterpret_cast<float *>(cb + oY); a.dA = reinterpret_cast<float *>(cb + odA);
  a.Dm = reinterpret_cast<float *>(cb + oD); a.gv = reinterpret_cast<float *>(cb + og);
  a.zv = reinterpret_cast<float *>(cb + oz); a.sv = reinterpret_cast<float *>(cb + os);
  a.uv = reinterpret_cast<float *>(cb + ou); a.rv = reinterpret_cast<float *>(cb + orr);
  a.al = reinterpret_cast<float *>(cb + oal); a.dal = reinterpret_cast<float *>(cb + odal);
  a.dsv = reinterpret_cast<float *>(cb + ods); a.duv = reinterpret_cast<float *>(cb + odu);
  a.dgv = reinterpret_cast<float *>(cb + odg);
  a.Mv = reinterpret_cast<float *>(cb + oM); a.denv = reinterpret_cast<float *>(cb + oden);
  a.dlt = reinterpret_cast<float *>(cb + odl);
  a.dst = reinterpret_cast<int32_t *>(cb + odst);
  a.dq = dq; a.dk = dk; a.dv = dv; a.dpos = dpos;
  const size_t smem6 = sizeof(float) * ((size_t)3 * Q * (C + 4) + 2 * (size_t)(L + 1) * C) +
                       ((size_t)Q * (C + 16 / sizeof(T)) * sizeof(T) + 15) / 16 * 16;
  const size_t smem5 = sizeof(float) * (size_t)Q * (C + 1);
  if (smem6 > 200 * 1024) return E2F_ERR_UNSUPPORTED;
  E2F_CUDA_TRY(cudaFuncSetAttribute(edge_bwd_kernel<T, L>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem6));
  E2F_CUDA_TRY(cudaFuncSetAttribute(edge_dy_kernel<T, L>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem5));
  for (auto &ch : chunks) {
    a.na = ch.first; a.nb = ch.second;
    a.ea = rp[ch.first];
    a.ne = (int64_t)rp[ch.second] - rp[ch.first];
    if (a.ne == 0) continue;
    const int eg = (int)std::min<int64_t>(a.ne, 148LL * 16);
    const int ng = (int)std::min<int64_t>((a.nb - a.na + 7) / 8, 148LL * 8);
    E2F_LAUNCH(edge_dst_kernel, ng, 256, 0, s, a);
    const int fg = (int)std::min<int64_t>((a.ne + FWD_WARPS - 1) / FWD_WARPS, 148LL * 16);
    E2F_LAUNCH((edge_fwd_kernel<T, L>), fg, BT, sizeof(float) * FWD_WARPS * C, s, a);
    E2F_LAUNCH(node_stats_kernel, ng, 256, 0, s, a);
    for (int m = 0; m <= L; ++m) {
      const int wm = m == 0 ? (L + 1) * C : 2 * (L - m + 1) * C;
      const int so = stack_off(L, C, m);
      st = stacked_gemm<T>(bh, wc + woff[m], wm, static_cast<T *>(a.A) + so, a.Y + so, a.ne, QC, true);
      if (st != E2F_OK) return st;
    }
    E2F_LAUNCH((edge_dalpha_kernel<L>), eg, BT, sizeof(float) * C, s, a);
    E2F_LAUNCH(node_delta_kernel, ng, 256, 0, s, a);
    E2F_LAUNCH((edge_dy_kernel<T, L>), eg, BT, smem5, s, a);
    for (int m = 0; m <= L; ++m) {
      const int wm = m == 0 ? (L + 1) * C : 2 * (L - m + 1) * C;
      const int so = stack_off(L, C, m);
      st = stacked_gemm<T>(bh, wc + woff[m], wm, static_cast<T *>(a.dY) + so, a.dA + so, a.ne, QC, false);
      if (st != E2F_OK) return st;
    }
    E2F_LAUNCH((edge_bwd_kernel<T, L>), eg, BT, smem6, s, a);
  }
  // dL/dx[n, (l, m), :] = dq[n, (l, m), :] Wq[l] + dk Wk[l] + dv Wv[l]: per
  // degree one strided-batched GEMM per projection over the 2l + 1 rows m
  // (rows of one m are Q C apart), fp32 (weights converted once per call)
  Scratch wf;
  const float *Wf[3][L + 1];
  if (std::is_same<T, float>::value) {
    for (int l = 0; l <= L; ++l) {
      Wf[0][l] = static_cast<const float *>(w->Wq[l]);
      Wf[1][l] = static_cast<const float *>(w->Wk[l]);
      Wf[2][l] = static_cast<const float *>(w->Wv[l]);
    }
  } else {
    const int64_t cc = (int64_t)C * C;
    E2F_CUDA_TRY(wf.alloc(sizeof(float) * 3 * (L + 1) * cc, s));
    float *wb = wf.as<float>();
    for (int t = 0; t < 3; ++t)
      for (int l = 0; l <= L; ++l) {
        const void *src = t == 0 ? w->Wq[l] : (t == 1 ? w->Wk[l] : w->Wv[l]);
        float *d = wb + (t * (L + 1) + l) * cc;
        E2F_LAUNCH(to_f32_kernel<T>, (int)std::min<int64_t>((cc + 255) / 256, 1024), 256, 0, s,
                   static_cast<const T *>(src), cc, d);
        Wf[t][l] = d;
      }
  }
  const float *grads[3] = {dq, dk, dv};
  for (int l = 0; l <= L; ++l)
    for (int t = 0; t < 3; ++t) {
      // column-major: dx^T[C x N] (ld QC) (+)= W^T[C x C] (the row-major W, ld C) * g^T[C x N] (ld QC)
      const float one = 1.f, beta = t == 0 ? 0.f : 1.f;
      const size_t o = (size_t)l * l * C;
      if (cublasSgemmStridedBatched(bh, CUBLAS_OP_N, CUBLAS_OP_N, C, (int)N, C, &one, Wf[t][l], C, 0,
                                    grads[t] + o, QC, C, &beta, dx + o, QC, C, 2 * l + 1) != CUBLAS_STATUS_SUCCESS)
        return E2F_ERR_CUDA;
    }
  return E2F_OK;
}

}  // namespace bwd

e2f_status attention_backward_impl(const void *x, const float *pos, const e2f_csr *csr, const e2f_weights *w,
                                   const float *G, float *dx, float *dpos, cudaStream_t s) {
  const bool f32 = w->dtype == E2F_F32;
  switch (w->L_max) {
#define E2F_BWD_CASE(LL)                                                                                   \
  case LL:                                                                                                 \
    return f32 ? bwd::run<float, LL>(x, pos, csr, w, G, dx, dpos, s)                                       \
               : bwd::run<__nv_bfloat16, LL>(x, pos, csr, w, G, dx, dpos, s);
    E2F_BWD_CASE(0)
    E2F_BWD_CASE(1)
    E2F_BWD_CASE(2)
    E2F_BWD_CASE(3)
    E2F_BWD_CASE(4)
    E2F_BWD_CASE(5)
    E2F_BWD_CASE(6)
#undef E2F_BWD_CASE
    default: return E2F_ERR_INVALID_ARG;
  }
}

}  // namespace e2f
