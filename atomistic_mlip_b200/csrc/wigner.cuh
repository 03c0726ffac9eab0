// Real Wigner-D blocks from a 3x3 rotation, and the per-edge frame.
//
// The SO(3) -> SO(2) change of basis of E2Former-V2 ("E2Former-V2 ...",
// §2.1 EAAS) and DPA4's EMFA (§2.1 A1) rotates every edge onto +z; the
// features then move with the real Wigner-D matrices of that rotation.
//
// Construction: the recursion of Ivanic & Ruedenberg (J. Phys. Chem. 100,
// 6342 (1996); erratum J. Phys. Chem. A 102, 9099 (1998)), which builds
// D^l from D^1 and D^(l-1) for real harmonics, written here from the
// published formulas.  D^1 is the rotation matrix itself in (y, z, x)
// order.  Result: Y_l(R u) = D^l(R) Y_l(u) for the real harmonics without
// Condon-Shortley phase (l = 1 ordered (y, z, x)).
//
// Layout: block l occupies (2l+1)^2 floats starting at l(4l^2-1)/3,
// row-major with row index m + l and column index m' + l.
#pragma once

#include <math.h>

#include "../../include/e2f.h"

#ifdef __CUDACC__
#define E2F_HD __host__ __device__ __forceinline__
#else
#define E2F_HD inline
#endif

namespace e2f {

E2F_HD int wig_offset(int l) { return l * (4 * l * l - 1) / 3; }

// Polynomial table of the y-rotation blocks (fitted in attention_tc.cu):
// entry (l, m, m') holds DYP_STRIDE floats [eps, c_0, .., c_l] at
// DYP_STRIDE * (wig_offset(l) + (m + l)(2l + 1) + (m' + l)).
constexpr int DYP_STRIDE = E2F_MAX_L + 2;
constexpr int DYP_ENTRIES = (E2F_MAX_L + 1) * (2 * E2F_MAX_L + 1) * (2 * E2F_MAX_L + 3) / 3;   // sum (2l+1)^2
E2F_HD int wig_size(int L) { return wig_offset(L + 1); }

E2F_HD float wig_sqrt(float x) { return sqrtf(x); }
E2F_HD double wig_sqrt(double x) { return sqrt(x); }

// D^1 from a row-major rotation R (index order (y, z, x) = (1, 2, 0)).
template <typename T> E2F_HD void wig_l1_from_rotation(const T R[9], T D1[9]) {
  const int p[3] = {1, 2, 0};
  for (int a = 0; a < 3; ++a)
    for (int b = 0; b < 3; ++b) D1[a * 3 + b] = R[p[a] * 3 + p[b]];
}

// Helper P^i_{a,b} of the recursion: i in {-1,0,1}, a in -(l-1)..(l-1),
// b in -l..l.  D1 is 3x3 (index +1), Dp is the (2l-1)^2 block of l-1.
template <typename T> E2F_HD T wig_P(int i, int a, int b, int l, const T *D1, const T *Dp) {
  const int w = 2 * l - 1;            // width of the l-1 block
  const int ra = a + (l - 1);         // row in the l-1 block
  const T ri1 = D1[(i + 1) * 3 + 2];   // R1(i, +1)
  const T rim = D1[(i + 1) * 3 + 0];   // R1(i, -1)
  const T ri0 = D1[(i + 1) * 3 + 1];   // R1(i,  0)
  if (b == l) return ri1 * Dp[ra * w + (2 * l - 2)] - rim * Dp[ra * w + 0];
  if (b == -l) return ri1 * Dp[ra * w + 0] + rim * Dp[ra * w + (2 * l - 2)];
  return ri0 * Dp[ra * w + (b + l - 1)];
}

// One entry D^l[m][m'] (l >= 2) from D^1 and D^(l-1).
template <typename T> E2F_HD T wig_entry(int l, int m, int mp, const T *D1, const T *Dp) {
  const int am = m < 0 ? -m : m;
  const T den = (mp == l || mp == -l) ? (T)(2 * l * (2 * l - 1)) : (T)((l + mp) * (l - mp));
  const T sqrt2 = (T)1.41421356237309504880;
  T acc = 0;
  // u term
  const T uu = (T)((l + m) * (l - m));
  if (uu > 0) acc += wig_sqrt(uu / den) * wig_P<T>(0, m, mp, l, D1, Dp);
  // v term
  {
    const T kd = (m == 0) ? (T)2 : (T)1;
    T v = (T)0.5 * wig_sqrt(kd * (T)((l + am - 1) * (l + am)) / den);
    if (m == 0) v = -v;
    T V;
    if (m == 0) {
      V = wig_P<T>(1, 1, mp, l, D1, Dp) + wig_P<T>(-1, -1, mp, l, D1, Dp);
    } else if (m > 0) {
      V = wig_P<T>(1, m - 1, mp, l, D1, Dp) * (m == 1 ? sqrt2 : (T)1);
      if (m != 1) V -= wig_P<T>(-1, -m + 1, mp, l, D1, Dp);
    } else {
      V = wig_P<T>(-1, -m - 1, mp, l, D1, Dp) * (m == -1 ? sqrt2 : (T)1);
      if (m != -1) V += wig_P<T>(1, m + 1, mp, l, D1, Dp);
    }
    acc += v * V;
  }
  // w term (zero for m = 0 and for |m| >= l - 1)
  if (m != 0 && am + 1 <= l - 1) {
    const T w = (T)-0.5 * wig_sqrt((T)((l - am - 1) * (l - am)) / den);
    T Wt;
    if (m > 0) Wt = wig_P<T>(1, m + 1, mp, l, D1, Dp) + wig_P<T>(-1, -m - 1, mp, l, D1, Dp);
    else       Wt = wig_P<T>(1, m - 1, mp, l, D1, Dp) - wig_P<T>(-1, -m + 1, mp, l, D1, Dp);
    acc += w * Wt;
  }
  return acc;
}

// All blocks l = 0..L of one rotation, sequentially (one thread).
template <typename T> E2F_HD void wig_all_serial(const T R[9], int L, T *D) {
  D[0] = 1;
  if (L < 1) return;
  wig_l1_from_rotation<T>(R, D + 1);
  for (int l = 2; l <= L; ++l) {
    const T *Dp = D + wig_offset(l - 1);
    T *Dl = D + wig_offset(l);
    const int w = 2 * l + 1;
    for (int m = -l; m <= l; ++m)
      for (int mp = -l; mp <= l; ++mp) Dl[(m + l) * w + (mp + l)] = wig_entry<T>(l, m, mp, D + 1, Dp);
  }
}

// Edge frame in the two-angle gauge R = Ry(-theta) Rz(-phi), which takes
// rhat = (sin t cos p, sin t sin p, cos t) to +z.  Any extra rotation about
// z leaves the attention output unchanged (SO(2) blocks commute with it and
// the logits use m = 0 entries only), so this cheaper gauge is used instead
// of the minimal rotation.  rhat must be a unit vector; at rho = 0 the
// azimuth is taken as 0.
E2F_HD void edge_frame_two_angle(float x, float y, float z, float R[9]) {
  const float rho = sqrtf(x * x + y * y);
  float cp = 1.f, sp = 0.f;
  if (rho > 0.f) { cp = x / rho; sp = y / rho; }
  const float ct = z, st = rho;
  R[0] = ct * cp; R[1] = ct * sp; R[2] = -st;
  R[3] = -sp;     R[4] = cp;      R[5] = 0.f;
  R[6] = st * cp; R[7] = st * sp; R[8] = ct;
}

}  // namespace e2f
