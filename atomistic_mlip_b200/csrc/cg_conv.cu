// Re-indexed Clebsch-Gordan convolution (EAAS) on the CUDA cores.
//
// What it computes ("E2Former-V2 ...", §2.1 "Axis-aligned equivariant
// sparsification (EAAS)", "Re-indexing operator"), per destination i and
// channel c:
//
//   o_i[(l3,m3), c] = sum_{j in N(i)} u(r_ij) sum_{paths p = (l1,l2,l3)} W[p][c]
//                     (x_j^{l1}[., c] (x) Y^{l2}(rhat_ij))^{l3}_{m3}
//
// with (a (x) b)^{l3}_{m3} = sum_{m1,m2} C_p[m1][m2][m3] a_{m1} b_{m2} the real
// coupling tensor (Racah's complex Clebsch-Gordan coefficients taken to the
// real harmonics: the real part for even l1 + l2 + l3, the imaginary part
// for odd), Y the orthonormal real harmonics, u(r) = (cos(pi r / r_c) + 1) / 2,
// paths every (l1, l2, l3) <= L with |l1 - l2| <= l3 <= l1 + l2 in
// lexicographic order.
//
// How: the coupling is equivariant, so with R the edge frame (R rhat = +z),
//   (x (x) Y(rhat))^{l3} = D^{l3}(R)^T ((D(R) x) (x) Y(+z))^{l3},
// and Y^{l2}(+z) has only its m = 0 entry, sqrt((2 l2 + 1) / (4 pi))
// (Lemma 4.1).  Only the m2 = 0 slice of each coupling tensor survives, and
// it is block sparse: (l1, m1) feeds (l3, m3) only for |m1| = |m3|; even
// paths keep the sign of m, odd paths exchange it, and every (m >= 1, l3,
// l1) pair becomes [y+; y-] = [[A, B], [-B, A]] [x+; x-] with A the even and B
// the odd paths' sum.  Summed over l2 with the path weights once per call
// (one (A, B) pair per channel; A alone for m = 0), the dense contraction
// becomes this per-channel SO(2) map between a rotate-in and a rotate-out:
// the parity re-indexing.
//
// Frame: R = Ry(-theta) Rz(-phi) (theta, phi the polar angles of rhat); the
// z part rotates the (+m, -m) pairs by m phi, the y part applies the
// parity-split polynomial blocks fitted for the fused attention.
//
// Layout and threads: one CTA per destination node (grid-stride over nodes),
// C / CPT threads, CPT consecutive channels per thread (2 up to L = 4, 1
// above, where the per-thread feature vectors would not fit in registers);
// the node's edges are taken EB at a time: the geometry, the z phases and
// the y blocks of EB edges go to shared memory, then every thread runs the
// whole chain for its channels and the EB edges, accumulating o_i in
// shared memory (each thread owns its columns).  o_i is written once; no
// atomics, no per-edge tensor in device memory.
#include <complex>
#include <mutex>
#include <vector>

#include "common.cuh"
#include "wigner.cuh"

namespace e2f {

const float *dy_poly_host_table();   // attention_tc.cu

namespace cgc {

constexpr int EB = 8;         // edges staged per round
constexpr int ESTRIDE = 256;  // floats per SO(2) weight slot (C <= 256): compile-time weight offsets

__constant__ float c_cgdy[DYP_ENTRIES * DYP_STRIDE];

template <int L> struct Cfg {
  static constexpr int Q = (L + 1) * (L + 1);
  static constexpr int NDYE = (L + 1) * (L + 2) * (2 * L + 3) / 6;   // sum (l+1)^2: blocks m, m' >= 0
  static constexpr int NDYO = L * (L + 1) * (2 * L + 1) / 6;         // sum l^2:     blocks m, m' < 0
  static constexpr int NDY = NDYE + NDYO;
  static constexpr int NS = (L + 1) * (L + 1) + 2 * (L * (L + 1) * (2 * L + 1) / 6);   // SO(2) weight slots
  static constexpr int CPT = L <= 4 ? 2 : 1;
};

__host__ __device__ __forceinline__ constexpr int dye_off(int l) { return l * (l + 1) * (2 * l + 1) / 6; }
template <int L> __host__ __device__ __forceinline__ constexpr int dyo_off(int l) {
  return Cfg<L>::NDYE + (l - 1) * l * (2 * l - 1) / 6;
}
// slot of (m = 0, l3, l1): one weight; slot of (m >= 1, l3, l1): the pair (A, B)
__host__ __device__ __forceinline__ constexpr int slot0(int L, int l3, int l1) { return l3 * (L + 1) + l1; }
__host__ __device__ __forceinline__ constexpr int slotm(int L, int m, int l3, int l1) {
  // sum_{k=1}^{m-1} (L-k+1)^2 pairs before degree m
  return (L + 1) * (L + 1) +
         2 * (L * (L + 1) * (2 * L + 1) / 6 - (L - m + 1) * (L - m + 2) * (2 * (L - m + 1) + 1) / 6) +
         2 * ((l3 - m) * (L - m + 1) + (l1 - m));
}

// ---- per-thread channel vectors ---------------------------------------------------
__device__ __forceinline__ float vmad(float s, float x, float a) { return fmaf(s, x, a); }
__device__ __forceinline__ float2 vmad(float s, float2 x, float2 a) { return __ffma2_rn(make_float2(s, s), x, a); }
__device__ __forceinline__ float2 vmad(float2 s, float2 x, float2 a) { return __ffma2_rn(s, x, a); }
__device__ __forceinline__ float vneg(float x) { return -x; }
__device__ __forceinline__ float2 vneg(float2 x) { return make_float2(-x.x, -x.y); }
template <typename V> __device__ __forceinline__ V vzero();
template <> __device__ __forceinline__ float vzero<float>() { return 0.f; }
template <> __device__ __forceinline__ float2 vzero<float2>() { return make_float2(0.f, 0.f); }

__device__ __forceinline__ void ldv(const float *p, float &v) { v = *p; }
__device__ __forceinline__ void ldv(const __nv_bfloat16 *p, float &v) { v = __bfloat162float(*p); }
__device__ __forceinline__ void ldv(const float *p, float2 &v) { v = *reinterpret_cast<const float2 *>(p); }
__device__ __forceinline__ void ldv(const __nv_bfloat16 *p, float2 &v) {
  v = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(p));
}
__device__ __forceinline__ void stv(float *p, float v) { *p = v; }
__device__ __forceinline__ void stv(float *p, float2 v) { *reinterpret_cast<float2 *>(p) = v; }

// Stage fence: a warp synchronisation over the warp's threads (all of them
// run the same edge chain, so it waits for nobody); loads are not moved
// across it, so the weights and y blocks of one stage are not all loaded
// (and kept live) at once.
__device__ __forceinline__ void stage_fence(unsigned wmask) { __syncwarp(wmask); }

struct Args {
  const void *x;
  const float *pos;
  Geom g;
  const int32_t *row_ptr, *col_idx;
  int N, C;
  const float *E;   // [NS][ESTRIDE] per-channel SO(2) weights (channels 0..C-1 used)
  float *out;
};

// E[s][c] = sum over the (path, coefficient) entries of slot s of coef W[path][c]
__global__ void so2_weights_kernel(const float *__restrict__ W, int C, int NS, const int32_t *__restrict__ sstart,
                                   const int32_t *__restrict__ epath, const float *__restrict__ ecoef,
                                   float *__restrict__ E) {
  for (int idx = blockIdx.x * blockDim.x + threadIdx.x; idx < NS * C; idx += gridDim.x * blockDim.x) {
    const int s = idx / C, c = idx - s * C;
    float acc = 0.f;
    for (int k = sstart[s]; k < sstart[s + 1]; ++k) acc = fmaf(ecoef[k], W[(size_t)epath[k] * C + c], acc);
    E[(size_t)s * ESTRIDE + c] = acc;
  }
}

template <typename T, int L>
__global__ void __launch_bounds__(256, 2) cg_conv_kernel(Args a) {
  using Cf = Cfg<L>;
  using V = typename std::conditional<Cf::CPT == 2, float2, float>::type;
  constexpr int Q = Cf::Q, NDY = Cf::NDY, CPT = Cf::CPT;
  constexpr int LZ = L > 0 ? L : 1;
  __shared__ float s_dy[EB][NDY > 0 ? NDY : 1];
  __shared__ float s_cs[EB][LZ], s_sn[EB][LZ];
  __shared__ float s_geo[EB][4];   // u, cos(theta), sin(theta), unused
  __shared__ int s_j[EB];
  const int C = a.C;
  const int c0 = CPT * threadIdx.x;
  const T *xg = static_cast<const T *>(a.x);
  const float *Ec = a.E + c0;
  extern __shared__ float s_o[];   // [Q][C]
  const int wfirst = threadIdx.x & ~31, wn = min(32, (int)blockDim.x - wfirst);
  const unsigned wmask = wn == 32 ? 0xffffffffu : ((1u << wn) - 1u);
  float *ob = s_o + c0;
  for (int i = blockIdx.x; i < a.N; i += gridDim.x) {
    const int e0 = a.row_ptr[i], e1 = a.row_ptr[i + 1];
    // the node's accumulator lives in shared memory (each thread owns its
    // columns), so that registers hold only the edge's vector
#pragma unroll
    for (int q = 0; q < Q; ++q) stv(ob + (size_t)q * C, vzero<V>());
    const float3 pi = load_pos(a.pos, i);
#pragma unroll 1
    for (int eb = e0; eb < e1; eb += EB) {
      const int nb = min(EB, e1 - eb);
      __syncthreads();   // the previous round's tables are no longer read
      // ---- geometry of the round's edges: frame angles, z phases, envelope
      for (int b = threadIdx.x; b < nb; b += blockDim.x) {
        const int j = a.col_idx[eb + b];
        float dx, dy, dz;
        pair_disp(a.g, pi, load_pos(a.pos, j), dx, dy, dz);
        const float r = sqrtf(dx * dx + dy * dy + dz * dz);
        float ux = 0.f, uy = 0.f, uz = 1.f;
        if (r > 0.f) { ux = dx / r; uy = dy / r; uz = dz / r; }
        const float rho = sqrtf(ux * ux + uy * uy);
        float cp = 1.f, sp = 0.f;
        if (rho > 0.f) { cp = ux / rho; sp = uy / rho; }
        float cm = 1.f, sm = 0.f;
        for (int m = 1; m <= L; ++m) {
          const float c2 = cm * cp - sm * sp, s2 = sm * cp + cm * sp;
          cm = c2; sm = s2;
          s_cs[b][m - 1] = cm;
          s_sn[b][m - 1] = sm;
        }
        s_j[b] = j;
        s_geo[b][0] = 0.5f * (cospif(r / a.g.rc) + 1.f);
        s_geo[b][1] = uz;
        s_geo[b][2] = rho;
      }
      __syncthreads();
      // ---- y-rotation blocks D^l(Ry(-theta)) of the round's edges
      for (int idx = threadIdx.x; idx < nb * NDY; idx += blockDim.x) {
        const int b = idx / NDY, x = idx - b * NDY;
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
        const float *cf = c_cgdy + DYP_STRIDE * (wig_offset(l) + (m + l) * (2 * l + 1) + (mp + l));
        const float ct = s_geo[b][1], st = s_geo[b][2];
        float p = cf[1 + L];
        for (int jd = L - 1; jd >= 0; --jd) p = fmaf(p, ct, cf[1 + jd]);   // zero above the entry's degree
        s_dy[b][x] = cf[0] != 0.f ? p * st : p;
      }
      __syncthreads();
      // ---- per edge: rotate in, re-indexed coupling, rotate out, accumulate
#pragma unroll 1
      for (int b = 0; b < nb; ++b) {
        // (an opaque copy of C: the Q row offsets are formed per edge, not
        // hoisted into Q live registers)
        int Cq = C;
        asm volatile("" : "+r"(Cq));
        const T *xr = xg + (size_t)s_j[b] * Q * Cq + c0;
        V x[Q];
#pragma unroll
        for (int q = 0; q < Q; ++q) ldv(xr + q * Cq, x[q]);
        const float *dyb = s_dy[b];
        // the weights do not depend on the edge: an opaque copy of their base
        // keeps the compiler from hoisting all of them into registers
        const float *Eb = Ec;
        asm volatile("" : "+l"(Eb));
        // z: (+m, -m) <- (c v+ + s v-, -s v+ + c v-)
#pragma unroll
        for (int l = 1; l <= L; ++l)
#pragma unroll
          for (int m = 1; m <= l; ++m) {
            const float c = s_cs[b][m - 1], s = s_sn[b][m - 1];
            const V p = x[l * l + l + m], n = x[l * l + l - m];
            x[l * l + l + m] = vmad(c, p, vmad(s, n, vzero<V>()));
            x[l * l + l - m] = vmad(c, n, vmad(-s, p, vzero<V>()));
          }
        // y: even block (m, m' >= 0), odd block (m, m' < 0)
#pragma unroll
        for (int l = 1; l <= L; ++l) {
          stage_fence(wmask);
          V t[L + 1];
#pragma unroll
          for (int m = 0; m <= l; ++m) {
            V acc = vzero<V>();
#pragma unroll
            for (int mp = 0; mp <= l; ++mp) acc = vmad(dyb[dye_off(l) + m * (l + 1) + mp], x[l * l + l + mp], acc);
            t[m] = acc;
          }
#pragma unroll
          for (int m = 0; m <= l; ++m) x[l * l + l + m] = t[m];
#pragma unroll
          for (int m = 1; m <= l; ++m) {
            V acc = vzero<V>();
#pragma unroll
            for (int mp = 1; mp <= l; ++mp) acc = vmad(dyb[dyo_off<L>(l) + (m - 1) * l + (mp - 1)], x[l * l + l - mp], acc);
            t[m] = acc;
          }
#pragma unroll
          for (int m = 1; m <= l; ++m) x[l * l + l - m] = t[m];
        }
        // re-indexed coupling, order by order
        {
          stage_fence(wmask);
          V t[L + 1];
#pragma unroll
          for (int l3 = 0; l3 <= L; ++l3) {
            V acc = vzero<V>();
#pragma unroll
            for (int l1 = 0; l1 <= L; ++l1) {
              V w;
              ldv(Eb + slot0(L, l3, l1) * ESTRIDE, w);
              acc = vmad(w, x[l1 * l1 + l1], acc);
            }
            t[l3] = acc;
          }
#pragma unroll
          for (int l3 = 0; l3 <= L; ++l3) x[l3 * l3 + l3] = t[l3];
        }
#pragma unroll
        for (int m = 1; m <= L; ++m) {
          stage_fence(wmask);
          V tp[L + 1], tm[L + 1];
#pragma unroll
          for (int l3 = m; l3 <= L; ++l3) {
            if (l3 > m) stage_fence(wmask);
            V ap = vzero<V>(), am = vzero<V>();
#pragma unroll
            for (int l1 = m; l1 <= L; ++l1) {
              V A, B;
              ldv(Eb + slotm(L, m, l3, l1) * ESTRIDE, A);
              ldv(Eb + (slotm(L, m, l3, l1) + 1) * ESTRIDE, B);
              const V xp = x[l1 * l1 + l1 + m], xm = x[l1 * l1 + l1 - m];
              ap = vmad(A, xp, vmad(B, xm, ap));
              am = vmad(A, xm, vmad(vneg(B), xp, am));
            }
            tp[l3] = ap;
            tm[l3] = am;
          }
#pragma unroll
          for (int l3 = m; l3 <= L; ++l3) { x[l3 * l3 + l3 + m] = tp[l3]; x[l3 * l3 + l3 - m] = tm[l3]; }
        }
        // y back: D^T per block
#pragma unroll
        for (int l = 1; l <= L; ++l) {
          stage_fence(wmask);
          V t[L + 1];
#pragma unroll
          for (int mp = 0; mp <= l; ++mp) {
            V acc = vzero<V>();
#pragma unroll
            for (int m = 0; m <= l; ++m) acc = vmad(dyb[dye_off(l) + m * (l + 1) + mp], x[l * l + l + m], acc);
            t[mp] = acc;
          }
#pragma unroll
          for (int mp = 0; mp <= l; ++mp) x[l * l + l + mp] = t[mp];
#pragma unroll
          for (int mp = 1; mp <= l; ++mp) {
            V acc = vzero<V>();
#pragma unroll
            for (int m = 1; m <= l; ++m) acc = vmad(dyb[dyo_off<L>(l) + (m - 1) * l + (mp - 1)], x[l * l + l - m], acc);
            t[mp] = acc;
          }
#pragma unroll
          for (int mp = 1; mp <= l; ++mp) x[l * l + l - mp] = t[mp];
        }
        // z back (+m, -m) <- (c y+ - s y-, s y+ + c y-), scaled by the envelope
        stage_fence(wmask);
        const float u = s_geo[b][0];
        int Co = C;
        asm volatile("" : "+r"(Co));
        {
          V t;
          ldv(ob, t);
          stv(ob, vmad(u, x[0], t));
        }
#pragma unroll
        for (int l = 1; l <= L; ++l) {
          {
            V t;
            ldv(ob + (l * l + l) * Co, t);
            stv(ob + (l * l + l) * Co, vmad(u, x[l * l + l], t));
          }
#pragma unroll
          for (int m = 1; m <= l; ++m) {
            const float c = u * s_cs[b][m - 1], s = u * s_sn[b][m - 1];
            const V p = x[l * l + l + m], n = x[l * l + l - m];
            V tp, tn;
            ldv(ob + (l * l + l + m) * Co, tp);
            ldv(ob + (l * l + l - m) * Co, tn);
            stv(ob + (l * l + l + m) * Co, vmad(c, p, vmad(-s, n, tp)));
            stv(ob + (l * l + l - m) * Co, vmad(s, p, vmad(c, n, tn)));
          }
        }
      }
    }
    float *orow = a.out + (size_t)i * Q * C + c0;
#pragma unroll
    for (int q = 0; q < Q; ++q) {
      V t;
      ldv(ob + (size_t)q * C, t);
      stv(orow + (size_t)q * C, t);
    }
  }
}

// ---------------------------------------------------------------------------
// host: coupling coefficients of the edge frame
// ---------------------------------------------------------------------------
// <l1 m1; l2 m2 | l3 m3> by the Racah formula (double).
static double cg_racah(int l1, int m1, int l2, int m2, int l3, int m3) {
  if (m1 + m2 != m3 || l3 < abs(l1 - l2) || l3 > l1 + l2) return 0.0;
  if (abs(m1) > l1 || abs(m2) > l2 || abs(m3) > l3) return 0.0;
  auto f = [](int n) { double r = 1.0; for (int k = 2; k <= n; ++k) r *= k; return r; };
  const double pre = (2 * l3 + 1) * f(l1 + l2 - l3) * f(l1 - l2 + l3) * f(-l1 + l2 + l3) / f(l1 + l2 + l3 + 1) *
                     f(l1 + m1) * f(l1 - m1) * f(l2 + m2) * f(l2 - m2) * f(l3 + m3) * f(l3 - m3);
  double s = 0.0;
  const int kmin = std::max(0, std::max(l2 - l3 - m1, l1 - l3 + m2));
  const int kmax = std::min(l1 + l2 - l3, std::min(l1 - m1, l2 + m2));
  for (int k = kmin; k <= kmax; ++k)
    s += ((k & 1) ? -1.0 : 1.0) /
         (f(k) * f(l1 + l2 - l3 - k) * f(l1 - m1 - k) * f(l2 + m2 - k) * f(l3 - l2 + m1 + k) * f(l3 - l1 - m2 + k));
  return sqrt(pre) * s;
}

// Complex -> real unitary of the library's real harmonics (Y_real = U
// Y_complex, complex harmonics with the Condon-Shortley phase): row m + l is
// the real index, column M + l the complex one.
static std::complex<double> u_c2r(int l, int m, int M) {
  const double r2 = 1.0 / sqrt(2.0);
  if (m == 0) return M == 0 ? 1.0 : 0.0;
  const int am = abs(m);
  const double sg = (am & 1) ? -1.0 : 1.0;
  if (m > 0) {
    if (M == am) return sg * r2;
    if (M == -am) return r2;
    return 0.0;
  }
  if (M == -am) return std::complex<double>(0.0, r2);
  if (M == am) return std::complex<double>(0.0, -sg * r2);
  return 0.0;
}

// The m2 = 0 slice of the real coupling tensor of path (l1, l2, l3), times
// Y^{l2}(+z) = sqrt((2 l2 + 1) / (4 pi)): entry (m1 -> m3).
static double edge_coupling(int l1, int l2, int l3, int m1, int m3) {
  std::complex<double> k = 0.0;
  for (int M = -std::min(l1, l3); M <= std::min(l1, l3); ++M)
    k += u_c2r(l3, m3, M) * cg_racah(l1, M, l2, 0, l3, M) * std::conj(u_c2r(l1, m1, M));
  const double v = ((l1 + l2 + l3) & 1) ? k.imag() : k.real();
  return v * sqrt((2.0 * l2 + 1.0) / (4.0 * 3.14159265358979323846));
}

struct Table {
  int32_t *sstart = nullptr, *epath = nullptr;
  float *ecoef = nullptr;
};

// (path, coefficient) lists per SO(2) weight slot, built once per (device,
// L) and kept on the device for the process.  Returns false if the edge-frame
// slice is not of the block form above (cannot happen for a valid table).
static bool build_table(int L, std::vector<int32_t> &sstart, std::vector<int32_t> &epath, std::vector<float> &ecoef) {
  const int NS = (L + 1) * (L + 1) + 2 * (L * (L + 1) * (2 * L + 1) / 6);
  std::vector<std::vector<std::pair<int, double>>> lists(NS);
  int p = 0;
  for (int l1 = 0; l1 <= L; ++l1)
    for (int l2 = 0; l2 <= L; ++l2)
      for (int l3 = 0; l3 <= L; ++l3) {
        if (l3 < abs(l1 - l2) || l3 > l1 + l2) continue;
        const bool odd = (l1 + l2 + l3) & 1;
        // structure check over the whole slice
        for (int m1 = -l1; m1 <= l1; ++m1)
          for (int m3 = -l3; m3 <= l3; ++m3) {
            const double v = edge_coupling(l1, l2, l3, m1, m3);
            if (fabs(v) < 1e-13) continue;
            if (abs(m1) != abs(m3)) return false;
            if (m1 != 0 && ((m1 == m3) == odd)) return false;
          }
        for (int m = 0; m <= std::min(l1, l3); ++m) {
          if (m == 0) {
            const double a0 = edge_coupling(l1, l2, l3, 0, 0);
            if (fabs(a0) > 1e-13) lists[slot0(L, l3, l1)].emplace_back(p, a0);
            continue;
          }
          const double pp = edge_coupling(l1, l2, l3, m, m), mm = edge_coupling(l1, l2, l3, -m, -m);
          const double pm = edge_coupling(l1, l2, l3, -m, m), mp = edge_coupling(l1, l2, l3, m, -m);
          if (fabs(pp - mm) > 1e-12 || fabs(pm + mp) > 1e-12) return false;
          // y+ = A x+ + B x-, y- = -B x+ + A x-
          if (fabs(pp) > 1e-13) lists[slotm(L, m, l3, l1)].emplace_back(p, pp);
          if (fabs(pm) > 1e-13) lists[slotm(L, m, l3, l1) + 1].emplace_back(p, pm);
        }
        ++p;
      }
  sstart.assign(1, 0);
  for (auto &li : lists) {
    for (auto &pc : li) { epath.push_back(pc.first); ecoef.push_back((float)pc.second); }
    sstart.push_back((int32_t)epath.size());
  }
  return true;
}

static e2f_status ensure_tables(int L, Table *out) {
  static std::mutex mu;
  static Table tabs[64][E2F_MAX_L + 1];
  static bool dy_up[64] = {};
  int dev = 0;
  E2F_CUDA_TRY(cudaGetDevice(&dev));
  if (dev < 0 || dev >= 64) return E2F_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lk(mu);
  if (!dy_up[dev]) {
    const float *tab = dy_poly_host_table();
    if (!tab) return E2F_ERR_CUDA;
    E2F_CUDA_TRY(cudaMemcpyToSymbol(c_cgdy, tab, sizeof(float) * DYP_ENTRIES * DYP_STRIDE));
    dy_up[dev] = true;
  }
  Table &t = tabs[dev][L];
  if (!t.sstart) {
    std::vector<int32_t> ss, ep;
    std::vector<float> ec;
    if (!build_table(L, ss, ep, ec)) return E2F_ERR_CUDA;
    const size_t b_ss = ss.size() * 4, b_ep = std::max<size_t>(ep.size(), 1) * 4, b_ec = std::max<size_t>(ec.size(), 1) * 4;
    char *d = nullptr;
    E2F_CUDA_TRY(cudaMalloc(&d, b_ss + b_ep + b_ec));
    E2F_CUDA_TRY(cudaMemcpy(d, ss.data(), b_ss, cudaMemcpyHostToDevice));
    if (!ep.empty()) {
      E2F_CUDA_TRY(cudaMemcpy(d + b_ss, ep.data(), ep.size() * 4, cudaMemcpyHostToDevice));
      E2F_CUDA_TRY(cudaMemcpy(d + b_ss + b_ep, ec.data(), ec.size() * 4, cudaMemcpyHostToDevice));
    }
    t.sstart = reinterpret_cast<int32_t *>(d);
    t.epath = reinterpret_cast<int32_t *>(d + b_ss);
    t.ecoef = reinterpret_cast<float *>(d + b_ss + b_ep);
  }
  *out = t;
  return E2F_OK;
}

template <typename T, int L>
static e2f_status launch(const Args &a, cudaStream_t s) {
  const int nt = a.C / Cfg<L>::CPT;
  int dev = 0, nsm = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
  const int grid = (int)std::max<int64_t>(1, std::min<int64_t>(a.N, (int64_t)nsm * 16));
  const size_t smem = sizeof(float) * (size_t)Cfg<L>::Q * a.C;
  E2F_CUDA_TRY(cudaFuncSetAttribute(cg_conv_kernel<T, L>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
  E2F_LAUNCH((cg_conv_kernel<T, L>), grid, nt, smem, s, a);
  return E2F_OK;
}

}  // namespace cgc

int64_t cg_num_paths(int L) {
  int64_t n = 0;
  for (int l1 = 0; l1 <= L; ++l1)
    for (int l2 = 0; l2 <= L; ++l2)
      for (int l3 = 0; l3 <= L; ++l3)
        if (l3 >= abs(l1 - l2) && l3 <= l1 + l2) ++n;
  return n;
}

e2f_status cg_conv_impl(const void *x, int dtype, const float *pos, const e2f_csr *csr, int L, int C,
                        const float *W, float *out, cudaStream_t s) {
  using namespace cgc;
  const int64_t N = csr->n_nodes;
  if (N == 0) return E2F_OK;
  Table tab;
  e2f_status st = ensure_tables(L, &tab);
  if (st != E2F_OK) return st;
  static const int NSL[E2F_MAX_L + 1] = {Cfg<0>::NS, Cfg<1>::NS, Cfg<2>::NS, Cfg<3>::NS, Cfg<4>::NS, Cfg<5>::NS, Cfg<6>::NS};
  const int NS = NSL[L];
  Scratch es;
  E2F_CUDA_TRY(es.alloc(sizeof(float) * (size_t)NS * ESTRIDE, s));
  float *E = es.as<float>();
  const int pg = (int)std::min<int64_t>(((int64_t)NS * C + 255) / 256, 1024);
  E2F_LAUNCH(so2_weights_kernel, pg, 256, 0, s, W, C, NS, tab.sstart, tab.epath, tab.ecoef, E);
  Args a;
  a.x = x;
  a.pos = pos;
  for (int k = 0; k < 3; ++k) {
    a.g.box[k] = csr->box[k] > 0.f ? csr->box[k] : 0.f;
    a.g.half[k] = 0.5f * a.g.box[k];
    a.g.periodic[k] = csr->box[k] > 0.f;
  }
  a.g.rc = csr->r_c;
  a.g.rc2 = csr->r_c * csr->r_c;
  a.row_ptr = csr->row_ptr;
  a.col_idx = csr->col_idx;
  a.N = (int)N;
  a.C = C;
  a.E = E;
  a.out = out;
  const bool f32 = dtype == E2F_F32;
  switch (L) {
#define E2F_CG_CASE(LL) \
  case LL: return f32 ? launch<float, LL>(a, s) : launch<__nv_bfloat16, LL>(a, s);
    E2F_CG_CASE(0)
    E2F_CG_CASE(1)
    E2F_CG_CASE(2)
    E2F_CG_CASE(3)
    E2F_CG_CASE(4)
    E2F_CG_CASE(5)
    E2F_CG_CASE(6)
#undef E2F_CG_CASE
    default: return E2F_ERR_UNSUPPORTED;
  }
}

}  // namespace e2f
