// Fused on-the-fly equivariant attention, CUDA-core (SIMT) kernel.
//
// This is the fp32 parity path (and the bf16-storage path before the
// tensor-core kernel takes over).  It follows the same node-centric
// streaming structure as the tensor-core kernel ("E2Former-V2 ...", §2.2):
// one block owns a destination atom i, streams its CSR row in batches of
// TB edges, and keeps the running max, the envelope-weighted denominator
// and the [Q][C] accumulator on chip; nothing per edge reaches global
// memory ("no edge materialisation", online softmax).
//
// Per edge batch:
//   A  geometry: r_ij (minimum image, fp32), two-angle frame, Wigner-D
//      blocks (wigner.cuh), envelope u(r), radial MLP g(r)
//   B  logits s^h from the m = 0 rows of D q_i and D k_j
//   C  online-softmax update: M, l, rescale of the accumulator
//   D  rotate in: vt = D v_j, written in SO(2)-stacked order
//   E  per m: SO(2) block product (y+, y-), radial scale g_{m,l},
//      rotate out with D^T and add alpha-weighted into the accumulator
#include <algorithm>

#include "common.cuh"
#include "wigner.cuh"

namespace e2f {

constexpr int ATT_THREADS = 256;

template <int L> struct SimtShape {
  static constexpr int Q = (L + 1) * (L + 1);
  static constexpr int S = L * (4 * L * L - 1) / 3 + (2 * L + 1) * (2 * L + 1);  // sum_{l<=L}(2l+1)^2
  static constexpr int P = (L + 1) * (L + 2) / 2;
  static constexpr int TB = L <= 4 ? 8 : 4;
};

template <typename T> struct AttnArgs {
  const T *q, *k, *v;
  const float *pos;
  Geom g;
  const int32_t *row_ptr, *col_idx;
  int N, C, H;
  float inv_sqrt_d;
  const T *W0T;
  const T *WrT[E2F_MAX_L + 1];
  const T *WiT[E2F_MAX_L + 1];
  const float *W1, *W2;
  float *out;
};

template <typename T, int L>
__global__ void __launch_bounds__(ATT_THREADS)
attention_simt_kernel(AttnArgs<T> a) {
  using Sh = SimtShape<L>;
  constexpr int Q = Sh::Q, S = Sh::S, P = Sh::P, TB = Sh::TB;
  const int C = a.C, H = a.H, Ch = C / H;
  const int QC = Q * C;
  extern __shared__ float sm[];
  float *qi = sm;                  // [Q][C]
  float *acc = qi + QC;            // [Q][C]
  float *vt = acc + QC;            // [TB][QC] stacked
  float *Dm = vt + TB * QC;        // [TB][S]
  float *gs = Dm + TB * S;         // [TB][P]
  float *us = gs + TB * P;         // [TB]
  float *hid = us + TB;            // [TB][16]
  float *part = hid + TB * 16;     // [TB][C]
  float *sc = part + TB * C;       // [TB][H]
  float *wg = sc + TB * H;         // [TB][H]
  float *Ms = wg + TB * H;         // [H]
  float *ell = Ms + H;             // [H]
  float *scl = ell + H;            // [H]
  int *js = reinterpret_cast<int *>(scl + H);   // [TB]

  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;

  for (int i = blockIdx.x; i < a.N; i += gridDim.x) {
    const int rp0 = a.row_ptr[i], rp1 = a.row_ptr[i + 1];
    __syncthreads();
    for (int idx = t; idx < QC; idx += ATT_THREADS) {
      qi[idx] = to_f(a.q[(size_t)i * QC + idx]);
      acc[idx] = 0.f;
    }
    for (int h = t; h < H; h += ATT_THREADS) { Ms[h] = -INFINITY; ell[h] = 0.f; }
    const float3 pi = load_pos(a.pos, i);

    for (int e0 = rp0; e0 < rp1; e0 += TB) {
      const int nb = min(TB, rp1 - e0);
      __syncthreads();
      // ---- A: geometry, Wigner-D, envelope, radial MLP (warp per edge)
      for (int e = warp; e < TB; e += ATT_THREADS / 32) {
        float *D = Dm + e * S;
        if (e >= nb) {
          for (int x = lane; x < S; x += 32) D[x] = 0.f;
          if (lane < P) gs[e * P + lane] = 0.f;
          if (lane == 0) { us[e] = 0.f; js[e] = -1; }
          continue;
        }
        const int j = a.col_idx[e0 + e];
        float dx, dy, dz;
        pair_disp(a.g, pi, load_pos(a.pos, j), dx, dy, dz);
        const float r = sqrtf(dx * dx + dy * dy + dz * dz);
        float ux = 0.f, uy = 0.f, uz = 1.f;
        if (r > 0.f) { ux = dx / r; uy = dy / r; uz = dz / r; }
        if (lane == 0) {
          js[e] = j;
          us[e] = 0.5f * (cospif(r / a.g.rc) + 1.f);
          D[0] = 1.f;
          if (L >= 1) {
            float R[9];
            edge_frame_two_angle(ux, uy, uz, R);
            wig_l1_from_rotation(R, D + 1);
          }
        }
        // radial MLP: 8 Gaussians (centres k r_c / 7, sigma 0.5), 16 hidden SiLU
        if (lane < 16) {
          float z = 0.f;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const float mu = (float)kk * (a.g.rc / 7.f);
            const float dd = r - mu;
            z = fmaf(a.W1[lane * 8 + kk], expf(-dd * dd * 2.f), z);
          }
          hid[e * 16 + lane] = z / (1.f + expf(-z));
        }
        __syncwarp();
        for (int l = 2; l <= L; ++l) {
          const int w = 2 * l + 1;
          for (int x = lane; x < w * w; x += 32)
            D[wig_offset(l) + x] = wig_entry(l, x / w - l, x % w - l, D + 1, D + wig_offset(l - 1));
          __syncwarp();
        }
        if (lane < P) {
          float gv = 0.f;
#pragma unroll
          for (int hh = 0; hh < 16; ++hh) gv = fmaf(a.W2[lane * 16 + hh], hid[e * 16 + hh], gv);
          gs[e * P + lane] = gv;
        }
      }
      __syncthreads();
      // ---- B: logits from the m = 0 rows (Lemma 4.1 of the summary)
      for (int item = t; item < nb * C; item += ATT_THREADS) {
        const int e = item / C, c = item % C;
        const T *kj = a.k + (size_t)js[e] * QC;
        const float *D = Dm + e * S;
        float s = 0.f;
#pragma unroll
        for (int l = 0; l <= L; ++l) {
          const float *row0 = D + wig_offset(l) + l * (2 * l + 1);
          float qh = 0.f, kh = 0.f;
          for (int mp = 0; mp < 2 * l + 1; ++mp) {
            const int qidx = (l * l + mp) * C + c;
            qh = fmaf(row0[mp], qi[qidx], qh);
            kh = fmaf(row0[mp], to_f(kj[qidx]), kh);
          }
          s = fmaf(qh, kh, s);
        }
        part[e * C + c] = s;
      }
      __syncthreads();
      for (int item = t; item < nb * H; item += ATT_THREADS) {
        const int e = item / H, h = item % H;
        float s = 0.f;
        for (int c = h * Ch; c < (h + 1) * Ch; ++c) s += part[e * C + c];
        sc[e * H + h] = s * a.inv_sqrt_d;
      }
      __syncthreads();
      // ---- C: online softmax (envelope in numerator and denominator)
      for (int h = t; h < H; h += ATT_THREADS) {
        float mn = Ms[h];
        for (int e = 0; e < nb; ++e) mn = fmaxf(mn, sc[e * H + h]);
        const float scale = (Ms[h] == -INFINITY) ? 0.f : expf(Ms[h] - mn);
        float sum = 0.f;
        for (int e = 0; e < TB; ++e) {
          const float wv = e < nb ? us[e] * expf(sc[e * H + h] - mn) : 0.f;
          wg[e * H + h] = wv;
          sum += wv;
        }
        ell[h] = ell[h] * scale + sum;
        Ms[h] = mn;
        scl[h] = scale;
      }
      __syncthreads();
      for (int idx = t; idx < QC; idx += ATT_THREADS) acc[idx] *= scl[(idx % C) / Ch];
      // ---- D: rotate in, vt = D v_j in SO(2)-stacked order
      for (int item = t; item < TB * (L + 1) * C; item += ATT_THREADS) {
        const int e = item / ((L + 1) * C);
        const int rem = item % ((L + 1) * C);
        const int l = rem / C, c = rem % C;
        float *vrow = vt + e * QC;
        const int w = 2 * l + 1;
        if (e >= nb) {
          for (int m = -l; m <= l; ++m) vrow[stack_off(L, C, m) + (l - (m < 0 ? -m : m)) * C + c] = 0.f;
          continue;
        }
        const T *vj = a.v + (size_t)js[e] * QC + (size_t)(l * l) * C + c;
        float vv[2 * L + 1];
#pragma unroll
        for (int mp = 0; mp < 2 * L + 1; ++mp) vv[mp] = mp < w ? to_f(vj[mp * C]) : 0.f;
        const float *Dl = Dm + e * S + wig_offset(l);
        for (int m = -l; m <= l; ++m) {
          float sacc = 0.f;
#pragma unroll
          for (int mp = 0; mp < 2 * L + 1; ++mp)
            if (mp < w) sacc = fmaf(Dl[(m + l) * w + mp], vv[mp], sacc);
          vrow[stack_off(L, C, m) + (l - (m < 0 ? -m : m)) * C + c] = sacc;
        }
      }
      __syncthreads();
      // ---- E: SO(2) blocks per m, radial scale, rotate out, accumulate
#pragma unroll 1
      for (int m = 0; m <= L; ++m) {
        const int nm = (L - m + 1) * C;
        const int offp = stack_off(L, C, m), offm = stack_off(L, C, -m);
        for (int aa = t; aa < nm; aa += ATT_THREADS) {
          const int l = m + aa / C, c = aa % C, h = c / Ch;
          float yp[TB], ym[TB];
#pragma unroll
          for (int e = 0; e < TB; ++e) { yp[e] = 0.f; ym[e] = 0.f; }
          if (m == 0) {
            const T *W = a.W0T + aa;
            for (int kk = 0; kk < nm; ++kk) {
              const float w0 = to_f(W[(size_t)kk * nm]);
#pragma unroll
              for (int e = 0; e < TB; ++e) yp[e] = fmaf(w0, vt[e * QC + kk], yp[e]);
            }
          } else {
            const T *Wr = a.WrT[m] + aa;
            const T *Wi = a.WiT[m] + aa;
            for (int kk = 0; kk < nm; ++kk) {
              const float wr = to_f(Wr[(size_t)kk * nm]);
              const float wi = to_f(Wi[(size_t)kk * nm]);
#pragma unroll
              for (int e = 0; e < TB; ++e) {
                const float vp = vt[e * QC + offp + kk], vm = vt[e * QC + offm + kk];
                yp[e] = fmaf(wr, vp, fmaf(-wi, vm, yp[e]));
                ym[e] = fmaf(wi, vp, fmaf(wr, vm, ym[e]));
              }
            }
          }
          const int p = pair_index(L, m, l);
          const int w = 2 * l + 1;
          for (int mp = -l; mp <= l; ++mp) {
            float add = 0.f;
#pragma unroll
            for (int e = 0; e < TB; ++e) {
              if (e < nb) {
                const float *Dl = Dm + e * S + wig_offset(l);
                const float coef = wg[e * H + h] * gs[e * P + p];
                float contrib = Dl[(m + l) * w + (mp + l)] * yp[e];
                if (m > 0) contrib = fmaf(Dl[(-m + l) * w + (mp + l)], ym[e], contrib);
                add = fmaf(coef, contrib, add);
              }
            }
            acc[(l * l + l + mp) * C + c] += add;
          }
        }
        __syncthreads();
      }
    }
    // ---- finalise: o_i = acc / l (zero for an empty row)
    __syncthreads();
    for (int idx = t; idx < QC; idx += ATT_THREADS) {
      const float den = ell[(idx % C) / Ch];
      a.out[(size_t)i * QC + idx] = den > 0.f ? acc[idx] / den : 0.f;
    }
  }
}

// ---------------------------------------------------------------------------
// weight packing for the SIMT kernel: transposed blocks W^T[k][a]
template <typename T>
__global__ void transpose_kernel(const T *__restrict__ in, T *__restrict__ out, int n) {
  __shared__ T tile[32][33];
  const int bx = blockIdx.x * 32, by = blockIdx.y * 32;
  for (int yy = threadIdx.y; yy < 32; yy += 8) {
    const int r = by + yy, c = bx + threadIdx.x;
    if (r < n && c < n) tile[yy][threadIdx.x] = in[(size_t)r * n + c];
  }
  __syncthreads();
  for (int yy = threadIdx.y; yy < 32; yy += 8) {
    const int r = bx + yy, c = by + threadIdx.x;
    if (r < n && c < n) out[(size_t)r * n + c] = tile[threadIdx.x][yy];
  }
}

template <typename T, int L>
static e2f_status launch_simt(const T *q, const T *k, const T *v, const float *pos, const e2f_csr *csr,
                              const e2f_weights *w, const T *packed, const size_t *offs, float *out,
                              cudaStream_t s, cudaEvent_t ev0, cudaEvent_t ev1) {
  using Sh = SimtShape<L>;
  AttnArgs<T> a;
  a.q = q; a.k = k; a.v = v; a.pos = pos;
  for (int kk = 0; kk < 3; ++kk) {
    a.g.box[kk] = csr->box[kk] > 0.f ? csr->box[kk] : 0.f;
    a.g.half[kk] = 0.5f * a.g.box[kk];
    a.g.periodic[kk] = csr->box[kk] > 0.f;
  }
  a.g.rc = csr->r_c;
  a.g.rc2 = csr->r_c * csr->r_c;
  a.row_ptr = csr->row_ptr; a.col_idx = csr->col_idx;
  a.N = (int)csr->n_nodes; a.C = w->C; a.H = w->H;
  a.inv_sqrt_d = 1.f / sqrtf((float)((L + 1) * (w->C / w->H)));
  a.W0T = packed + offs[0];
  for (int m = 0; m <= E2F_MAX_L; ++m) {
    a.WrT[m] = (m >= 1 && m <= L) ? packed + offs[2 * m - 1] : nullptr;
    a.WiT[m] = (m >= 1 && m <= L) ? packed + offs[2 * m] : nullptr;
  }
  a.W1 = w->rad_W1; a.W2 = w->rad_W2; a.out = out;
  const int C = w->C, H = w->H, QC = Sh::Q * C, TB = Sh::TB;
  const size_t smem = sizeof(float) * ((size_t)2 * QC + (size_t)TB * QC + TB * Sh::S + TB * Sh::P + TB +
                                       TB * 16 + TB * C + 2 * TB * H + 3 * H) + sizeof(int) * TB;
  if (smem > 227 * 1024) return E2F_ERR_UNSUPPORTED;
  E2F_CUDA_TRY(cudaFuncSetAttribute(attention_simt_kernel<T, L>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
  int dev = 0, nsm = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
  int per_sm = 1;
  cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, attention_simt_kernel<T, L>, ATT_THREADS, smem);
  const int grid = (int)std::min<int64_t>(csr->n_nodes, (int64_t)nsm * std::max(per_sm, 1) * 8);
  if (ev0) E2F_CUDA_TRY(cudaEventRecord(ev0, s));
  E2F_LAUNCH((attention_simt_kernel<T, L>), grid, ATT_THREADS, smem, s, a);
  if (ev1) E2F_CUDA_TRY(cudaEventRecord(ev1, s));
  return E2F_OK;
}

template <typename T>
e2f_status attention_simt_impl(const T *q, const T *k, const T *v, const float *pos, const e2f_csr *csr,
                               const e2f_weights *w, float *out, cudaStream_t s, cudaEvent_t ev0,
                               cudaEvent_t ev1) {
  const int L = w->L_max, C = w->C;
  // pack transposed SO(2) blocks: W0^T, then (Wr_m^T, Wi_m^T) for m = 1..L
  size_t offs[2 * E2F_MAX_L + 1];
  size_t total = 0;
  const size_t n0 = (size_t)(L + 1) * C;
  offs[0] = 0; total = n0 * n0;
  for (int m = 1; m <= L; ++m) {
    const size_t nm = (size_t)(L - m + 1) * C;
    offs[2 * m - 1] = total; total += nm * nm;
    offs[2 * m] = total; total += nm * nm;
  }
  Scratch pk;
  E2F_CUDA_TRY(pk.alloc(total * sizeof(T), s));
  T *packed = pk.as<T>();
  {
    const int n = (int)n0;
    dim3 g((n + 31) / 32, (n + 31) / 32), b(32, 8);
    E2F_LAUNCH(transpose_kernel<T>, g, b, 0, s, static_cast<const T *>(w->W0), packed + offs[0], n);
    for (int m = 1; m <= L; ++m) {
      const int nm = (L - m + 1) * C;
      dim3 gm((nm + 31) / 32, (nm + 31) / 32);
      E2F_LAUNCH(transpose_kernel<T>, gm, b, 0, s, static_cast<const T *>(w->Wr[m]), packed + offs[2 * m - 1], nm);
      E2F_LAUNCH(transpose_kernel<T>, gm, b, 0, s, static_cast<const T *>(w->Wi[m]), packed + offs[2 * m], nm);
    }
  }
  switch (L) {
    case 0: return launch_simt<T, 0>(q, k, v, pos, csr, w, packed, offs, out, s, ev0, ev1);
    case 1: return launch_simt<T, 1>(q, k, v, pos, csr, w, packed, offs, out, s, ev0, ev1);
    case 2: return launch_simt<T, 2>(q, k, v, pos, csr, w, packed, offs, out, s, ev0, ev1);
    case 3: return launch_simt<T, 3>(q, k, v, pos, csr, w, packed, offs, out, s, ev0, ev1);
    case 4: return launch_simt<T, 4>(q, k, v, pos, csr, w, packed, offs, out, s, ev0, ev1);
    case 5: return launch_simt<T, 5>(q, k, v, pos, csr, w, packed, offs, out, s, ev0, ev1);
    case 6: return launch_simt<T, 6>(q, k, v, pos, csr, w, packed, offs, out, s, ev0, ev1);
    default: return E2F_ERR_INVALID_ARG;
  }
}

template e2f_status attention_simt_impl<float>(const float *, const float *, const float *, const float *,
                                               const e2f_csr *, const e2f_weights *, float *, cudaStream_t,
                                               cudaEvent_t, cudaEvent_t);
template e2f_status attention_simt_impl<__nv_bfloat16>(const __nv_bfloat16 *, const __nv_bfloat16 *,
                                                       const __nv_bfloat16 *, const float *, const e2f_csr *,
                                                       const e2f_weights *, float *, cudaStream_t, cudaEvent_t,
                                                       cudaEvent_t);

}  // namespace e2f
