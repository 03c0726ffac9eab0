/*
 * e2f.h -- C ABI of libe2f, the B200 (sm_100a) implementation of
 * E2Former-V2's node-centric on-the-fly equivariant attention forward.
 *
 * Sources (web pages):
 *   [E2F]  "E2Former-V2: On-the-Fly Equivariant Attention with Linear
 *          Activation Memory" (technical summary), §2.1 "Axis-aligned
 *          equivariant sparsification (EAAS)", §2.2 "On-the-fly equivariant
 *          attention" (node-centric factorisation, streaming reduction over
 *          j in N(i), no edge materialisation, online softmax).
 *   [EqV3] "EquiformerV3 ..." (technical summary), §2B.3 "Smooth radius
 *          cutoff attention" (envelope in numerator and denominator).
 *   [DPA4] "DPA4 ... EMFA SO(2) Convolution", §2.1 A1 (features moved to a
 *          local SO(2) frame per edge) and A3 (envelope-gated attention).
 *
 * Conventions shared by every call:
 *   - All pointers marked "device" are CUDA device pointers on the current
 *     device; "host" pointers are ordinary host memory.  The caller owns
 *     every buffer it passes; the library never frees or retains them.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  All device work is enqueued on it.
 *   - Node features are stored [N][Q][C], Q = (L+1)^2, channel fastest;
 *     coefficient (l, m), m = -l..l, sits at index l*l + l + m of the Q
 *     axis (real spherical harmonics without the Condon-Shortley phase,
 *     l = 1 ordered (y, z, x)).
 *   - Feature arrays (x, q, k, v, out) and the weight matrices Wq/Wk/Wv,
 *     W0, Wr, Wi are accessed as 16-byte vectors: their device pointers
 *     must be 16-byte aligned (E2F_ERR_INVALID_ARG otherwise).
 *   - Errors are returned as e2f_status; nothing is written to outputs when
 *     argument validation fails.  Device-side problems (a bounded wait that
 *     gave up) are latched in a per-device flag that e2f_stream_status()
 *     reads and clears.  Kernels never trap.
 *   - Temporary device memory is taken stream-ordered from a library-owned
 *     memory pool (cudaMallocFromPoolAsync / cudaFreeAsync on `stream`)
 *     and released before the call returns, in stream order.
 */
#ifndef E2F_H_
#define E2F_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define E2F_API __attribute__((visibility("default")))
#else
#define E2F_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef int32_t e2f_status;
#define E2F_OK                   0  /* success */
#define E2F_ERR_INVALID_ARG      1  /* NULL pointer, N < 0, r_c <= 0, L > 6, ... */
#define E2F_ERR_CUTOFF_TOO_LARGE 2  /* r_c >= box[k]/2 in a periodic dimension */
#define E2F_ERR_CAPACITY         3  /* col_idx too small; *n_edges = edges needed */
#define E2F_ERR_UNSUPPORTED      4  /* shape/dtype combination not implemented */
#define E2F_ERR_CUDA             5  /* a CUDA runtime call failed (e2f_last_cuda_error) */
#define E2F_ERR_TIMEOUT          6  /* a bounded device-side wait gave up */
#define E2F_ERR_DOMAIN           7  /* a coordinate outside [0, box[k]) in a periodic dim */
#define E2F_ERR_SCRATCH_LIMIT    8  /* input larger than a fixed-scratch entry point allows */

#define E2F_F32  0
#define E2F_BF16 1

#define E2F_MAX_L 6

/* Text of a status code (static storage). */
E2F_API const char *e2f_status_string(e2f_status s);

/* Text of the last CUDA error seen by this thread inside the library. */
E2F_API const char *e2f_last_cuda_error(void);

/* ---------------------------------------------------------------------------
 * Radius graph (the neighbour set j in N(i) that [E2F] §2.2 streams over).
 * --------------------------------------------------------------------------*/
typedef struct e2f_csr {
  const int32_t *row_ptr;  /* device, [n_nodes + 1] */
  const int32_t *col_idx;  /* device, [n_edges]     */
  int64_t n_nodes;
  int64_t n_edges;
  float box[3];            /* > 0: periodic edge length; 0: open */
  float r_c;
} e2f_csr;

/*
 * e2f_build_neighbors -- sorted CSR radius graph with a cell list.
 *
 *   pos      device, [N][3] fp32, AoS.  In periodic dimensions every
 *            coordinate must lie in [0, box[k]) (else E2F_ERR_DOMAIN).
 *   N        number of atoms, >= 0.
 *   box      host, 3 floats or NULL.  box[k] > 0 makes dimension k periodic
 *            (orthorhombic box, minimum image); box[k] == 0 or box == NULL
 *            leaves it open.  r_c must be < box[k]/2 for periodic k.
 *   r_c      cutoff radius, > 0.
 *   row_ptr  device, caller-allocated [N + 1] int32.
 *   col_idx  device, caller-allocated [capacity] int32.
 *   capacity length of col_idx.
 *   n_edges  host out: E = row_ptr[N].
 *   out_csr  host out (may be NULL): descriptor for e2f_attention_forward.
 *
 * Row i lists every j != i with r2 < r_c*r_c, in ascending j, where, in
 * fp32 with round-to-nearest and no fused multiply-add,
 *   d_k = p_j,k - p_i,k;  periodic k: d_k > b_k/2 -> d_k -= b_k,
 *   d_k < -b_k/2 -> d_k += b_k;  r2 = (d_x*d_x + d_y*d_y) + d_z*d_z.
 * If E > capacity the call returns E2F_ERR_CAPACITY with *n_edges = E and
 * writes nothing past col_idx[capacity - 1] (row_ptr is written).
 * Host synchronisations: one to read the bounding box when any dimension
 * is open, one to read E.
 */
E2F_API e2f_status e2f_build_neighbors(const float *pos, int64_t N, const float *box, float r_c,
                               int32_t *row_ptr, int32_t *col_idx, int64_t capacity,
                               int64_t *n_edges, e2f_csr *out_csr, void *stream);

/*
 * e2f_build_neighbors_noalloc -- the same CSR as e2f_build_neighbors,
 * computed without allocating any device memory.  The pages describe no
 * such call; it is an interface addition for callers that cannot allocate:
 * MD engines and plugin hosts that reserve the device memory budget once
 * at start-up and own every later allocation, and step loops that must not
 * meet an allocation (its failure mode, its implicit synchronisation) in
 * the middle of a step.
 *
 * All temporary arrays live in one fixed array of about 4.7 MB that is part
 * of the library's device image, so every GPU that loads the library holds
 * it until the process exits.  The caller still passes pos, row_ptr and
 * col_idx; arguments, result and status codes are those of
 * e2f_build_neighbors, plus E2F_ERR_SCRATCH_LIMIT when N > 131072.  The
 * cell grid is coarsened to at most 131072 cells when needed (same result,
 * more candidate pairs tested).
 *
 * The first call on a device looks up the array's device address
 * (cudaGetSymbolAddress); make that first call before any stream capture.
 * The address is kept for the life of the process: a cudaDeviceReset (or
 * any teardown of the device's primary context) invalidates this entry
 * point for the rest of the process.
 * Every call on a device uses the same array and finds the previous call's
 * contents in it (the call clears what must start at zero); calls whose GPU
 * work can overlap, e.g. on two streams with no ordering between them,
 * race on the array and must be serialised by the caller.
 */
E2F_API e2f_status e2f_build_neighbors_noalloc(const float *pos, int64_t N, const float *box, float r_c,
                                               int32_t *row_ptr, int32_t *col_idx, int64_t capacity,
                                               int64_t *n_edges, e2f_csr *out_csr, void *stream);

/* ---------------------------------------------------------------------------
 * Attention weights.
 * --------------------------------------------------------------------------*/
typedef struct e2f_weights {
  int32_t L_max;     /* 0..6 */
  int32_t C;         /* channels; C % H == 0 */
  int32_t H;         /* heads; head h owns channels [h*C/H, (h+1)*C/H) */
  int32_t dtype;     /* E2F_F32 or E2F_BF16: type of x, Wq/Wk/Wv, W0, Wr, Wi */
  /* device, [C][C] row-major (out x in), one per degree l = 0..L_max:
   * q(l,m) = Wq[l] x(l,m), likewise k, v ([E2F] §2.2, Eq. 6 projections). */
  const void *Wq[E2F_MAX_L + 1];
  const void *Wk[E2F_MAX_L + 1];
  const void *Wv[E2F_MAX_L + 1];
  /* device, [n0][n0] with n_m = (L_max - m + 1) * C: the m = 0 SO(2) block. */
  const void *W0;
  /* device, [n_m][n_m] for m = 1..L_max (index 0 unused): the SO(2) block
   * [y+; y-] = [[Wr, -Wi], [Wi, Wr]] [v+; v-], where v+-m stacks the
   * entries (l, +-m) for l = m..L_max, l-major, then channel ([E2F] §2.1,
   * [DPA4] A1). */
  const void *Wr[E2F_MAX_L + 1];
  const void *Wi[E2F_MAX_L + 1];
  /* device fp32 radial MLP: phi_k(r) = exp(-(r - k r_c/7)^2 / 0.5), k=0..7;
   * g = rad_W2 SiLU(rad_W1 phi); rad_W1 [16][8], rad_W2 [P][16] with
   * P = (L+1)(L+2)/2 rows ordered (m, l): m = 0..L, l = m..L. */
  const float *rad_W1;
  const float *rad_W2;
} e2f_weights;

/*
 * e2f_attention_forward -- o = on-the-fly equivariant attention of x.
 *
 *   x      device, [N][Q][C] in w->dtype.
 *   pos    device, [N][3] fp32 (the positions the CSR was built from).
 *   csr    host descriptor from e2f_build_neighbors (device arrays).
 *   w      host struct of device weight pointers.
 *   out    device, [N][Q][C] fp32, caller-allocated; fully overwritten.
 *
 * For each i and each j in N(i) ([E2F] §2.1-§2.2): r_ij = p_j - p_i
 * (minimum image), the edge frame R_ij puts r_ij on +z; q, k, v are the
 * per-degree projections of x; s^h = (1/sqrt((L+1) C/H)) sum over l and the
 * head's channels of (D q_i)(l,0) (D k_j)(l,0); y = SO(2) mix of D v_j,
 * scaled per (m, l) by g(r); alpha = u e^s / sum u e^s with
 * u = (cos(pi r / r_c) + 1)/2 ([EqV3] §2B.3); o_i = sum_j alpha D^T y.
 * o_i = 0 for an empty row.  No per-edge tensor is written to device memory.
 * Fully asynchronous (no host synchronisation).
 */
E2F_API e2f_status e2f_attention_forward(const void *x, const float *pos, const e2f_csr *csr,
                                 const e2f_weights *w, float *out, void *stream);

/*
 * e2f_attention_backward -- gradients of L = sum(grad_out * o), o the
 * output of e2f_attention_forward for the same x, pos, csr and w, with
 * respect to the node features and the positions.  The conservative forces
 * of an energy are -grad_pos ("E2Former-V2 ..." §4, the conservative
 * variant; "DPA4 ..." §2.2, the energy-to-force path).  Weight gradients
 * (training) are not computed.
 *
 *   x         device, [N][Q][C] in w->dtype (as for the forward).
 *   grad_out  device fp32 [N][Q][C]: dL/do.
 *   grad_x    device fp32 [N][Q][C], fully overwritten: dL/dx.
 *   grad_pos  device fp32 [N][3], fully overwritten: dL/dpos.
 * Requires H <= 16.  Per-edge quantities are recomputed in chunks of whole
 * destination nodes (at most 65,536 edges each) in library scratch; the
 * SO(2) block products of the forward recompute and their transposes run
 * as dense GEMMs over a chunk's edges (cuBLAS, fp32 accumulation).  One
 * host synchronisation (the chunk plan reads row_ptr).  Gradients reach
 * grad_pos through fp32 atomics, so their summation order (and last bits)
 * can vary from run to run.
 */
E2F_API e2f_status e2f_attention_backward(const void *x, const float *pos, const e2f_csr *csr,
                                          const e2f_weights *w, const float *grad_out, float *grad_x,
                                          float *grad_pos, void *stream);

/* ---------------------------------------------------------------------------
 * The E2Former-V2 block around the attention.
 * --------------------------------------------------------------------------*/
typedef struct e2f_block_weights {
  e2f_weights attn;          /* the block's attention weights (L_max, C, H, dtype) */
  int32_t hidden;            /* Hd, FFN hidden width */
  const float *gamma1;       /* device fp32 [L+1][C]: gains of the first merged norm */
  const float *gamma2;       /* device fp32 [L+1][C]: gains of the second merged norm */
  const void *Wa;            /* device [Hd][C] (attn.dtype): the scalar gate's map */
  const void *Wb[E2F_MAX_L + 1];   /* device [Hd][C] per degree l = 0..L_max */
  const void *Wd[E2F_MAX_L + 1];   /* device [C][Hd] per degree l = 0..L_max */
} e2f_block_weights;

/*
 * e2f_block_forward -- one pre-norm residual block:
 *   x1 = x + Attn(Norm1(x)),  out = x1 + FFN(Norm2(x1)).
 * Norm is the merged equivariant RMS layer norm ("EquiformerV3 ..." §2B.1:
 * one RMS statistic shared by all degrees): Norm(x)[n,(l,m),c] =
 * gamma[l][c] x[n,(l,m),c] / sqrt(mean_{l,m,c} x[n]^2 + 1e-6).  FFN is the
 * node feed-forward network with a scalar gate (§2B.2 hidden width, §2C
 * gate on the l = 0 features): FFN(y)[n,(l,m)] =
 * Wd[l] (SiLU(Wa y[n,(0,0)]) * (Wb[l] y[n,(l,m)])).  Attn is
 * e2f_attention_forward with w->attn, on the normalised features stored in
 * w->attn.dtype.
 *
 *   x    device fp32 [N][Q][C], the residual stream in.
 *   out  device fp32 [N][Q][C], fully overwritten; must not be x.
 * Library scratch (stream-ordered pool): the normalised features, the
 * attention output, the gate [N][Hd] fp32 and the hidden features
 * [N][Q][Hd] in w->attn.dtype.  Fully asynchronous.
 */
E2F_API e2f_status e2f_block_forward(const float *x, const float *pos, const e2f_csr *csr,
                                     const e2f_block_weights *w, float *out, void *stream);

/*
 * e2f_attention_forward_multifocus -- the attention of e2f_attention_forward
 * with F focus streams ([DPA4] §2.1 A2, multi-focus EMFA message).
 *
 *   x, pos, csr, w, out   as for e2f_attention_forward.
 *   F        1, 2, 4 or 8 streams; stream f owns channels [f C/F, (f+1) C/F).
 *   focus_a  device fp32 [C], 16-byte aligned: the focus vector (unused
 *            for F = 1).
 *
 * Each stream has its own SO(2) stack: of W0, Wr[m], Wi[m] only the entries
 * between input and output channels of the same stream are used (the others
 * are read as zero).  Per edge, after the SO(2) mix and the radial scale,
 * z_f = sqrt(F/C) sum_{c in f} focus_a[c] y[(0,0), c] (the l = 0 section of
 * the message), beta = softmax_f z, and every channel of stream f is scaled
 * by beta_f before the rotate-out and the envelope-gated attention sum.  F =
 * 1 is exactly e2f_attention_forward.  F > 1 runs on the tensor-core kernel
 * only: bf16, C = 128, L_max 2 or 4, 4 <= H <= 16 (else
 * E2F_ERR_UNSUPPORTED).  Fully asynchronous.
 */
E2F_API e2f_status e2f_attention_forward_multifocus(const void *x, const float *pos, const e2f_csr *csr,
                                                   const e2f_weights *w, int32_t F, const float *focus_a,
                                                   float *out, void *stream);

/*
 * e2f_cg_num_paths -- number of coupling paths (l1, l2, l3) of the CG
 * convolution of degree L: 0 <= l1, l2, l3 <= L with |l1 - l2| <= l3 <=
 * l1 + l2.  -1 for L outside 0..E2F_MAX_L.
 */
E2F_API int64_t e2f_cg_num_paths(int32_t L);

/*
 * e2f_cg_conv_forward -- Clebsch-Gordan convolution of node features with the
 * harmonics of the edge directions, evaluated by re-indexing in the edge
 * frame ([E2F] §2.1 EAAS, "Re-indexing operator").
 *
 *   x      device, [N][Q][C], Q = (L+1)^2, type `dtype` (E2F_F32 or
 *          E2F_BF16); 16-byte aligned.
 *   pos    device, [N][3] fp32 (the positions the CSR was built from).
 *   csr    host descriptor from e2f_build_neighbors (device arrays).
 *   L      0..E2F_MAX_L.   C  channels, even, 2..256.
 *   W      device fp32 [e2f_cg_num_paths(L)][C]: the weight of path p and
 *          channel c, paths in lexicographic (l1, l2, l3) order.
 *   out    device, [N][Q][C] fp32, 16-byte aligned; fully overwritten.
 *
 * o_i[(l3,m3),c] = sum_{j in N(i)} u(r_ij) sum_p W[p][c]
 *                  (x_j^{l1}[.,c] (x) Y^{l2}(rhat_ij))^{l3}_{m3},
 * with (x) the real Clebsch-Gordan coupling (Racah's coefficients taken to
 * the real harmonics of e2f_wigner_d: the real part for even l1 + l2 + l3,
 * the imaginary part for odd), Y the orthonormal real harmonics, r_ij =
 * p_j - p_i (minimum image), u = (cos(pi r / r_c) + 1)/2.  In the edge frame
 * the harmonics of the edge keep only m = 0, so each path reduces to a
 * block-sparse map between equal |m|; the dense contraction is never formed.
 * o_i = 0 for an empty row.  The first call per device and L builds a small
 * coefficient table (synchronous host-to-device copy); later calls are
 * asynchronous.  Errors: E2F_ERR_INVALID_ARG (null or misaligned pointers, C
 * out of range), E2F_ERR_UNSUPPORTED (L or dtype out of range).
 */
E2F_API e2f_status e2f_cg_conv_forward(const void *x, int32_t dtype, const float *pos, const e2f_csr *csr,
                                       int32_t L, int32_t C, const float *W, float *out, void *stream);

/*
 * e2f_stream_status -- synchronise `stream`, then return (and clear) any
 * error latched by a kernel of this library on the current device
 * (E2F_ERR_TIMEOUT for a bounded wait that gave up), or E2F_ERR_CUDA.
 *
 * Scope: the latched word is per DEVICE, not per stream.  Kernels on every
 * stream of the device write the same word, so a call for stream s1 also
 * reports (and clears) an error raised by work on stream s2 that has
 * finished by then.  Callers that run independent work on several streams
 * and need to tell whose work failed synchronise those streams and call
 * this once per device.  Argument validation itself keeps no state: the
 * entry points may be called from several host threads at once.
 */
E2F_API e2f_status e2f_stream_status(void *stream);

/* ---------------------------------------------------------------------------
 * Unit-level entry points (used by the tests; same conventions).
 * --------------------------------------------------------------------------*/

/*
 * e2f_wigner_d -- real Wigner-D blocks of rotation matrices ([E2F] §2.1:
 * the SO(3) -> SO(2) change of basis).
 *   R  device, [n][3][3] fp32 row-major proper rotations.
 *   D  device, [n][S] fp32 with S = sum_{l<=L} (2l+1)^2; block l starts at
 *      l(4l^2 - 1)/3 and is (2l+1) x (2l+1) row-major (row m+l, col m'+l),
 *      defined by Y_l(R u) = D^l(R) Y_l(u).
 */
E2F_API e2f_status e2f_wigner_d(const float *R, int64_t n, int32_t L, float *D, void *stream);

/*
 * e2f_project_qkv -- q, k, v = per-degree C x C maps of x (the node-level
 * projections of [E2F] §2.2).  x, q, k, v device [N][Q][C] in w->dtype
 * (bf16 outputs are rounded to nearest even from an fp32 accumulation).
 */
E2F_API e2f_status e2f_project_qkv(const void *x, int64_t N, const e2f_weights *w,
                           void *q, void *k, void *v, void *stream);

/* ---------------------------------------------------------------------------
 * Diagnostics.
 * --------------------------------------------------------------------------*/

/* Number of kernels this library has launched in this process so far. */
E2F_API int64_t e2f_kernel_launches(void);

/*
 * Timing of the dominant kernel (the fused attention kernel).  While
 * enabled, every e2f_attention_forward records a CUDA event pair around
 * that kernel on its stream.  e2f_profile_read() synchronises those
 * events, returns the number of launches and their summed duration in
 * milliseconds, and clears the record.  Process-wide: launches from every
 * host thread and stream are recorded together.
 */
E2F_API e2f_status e2f_profile_enable(int32_t on);
E2F_API e2f_status e2f_profile_read(int64_t *launches, double *total_ms);

/* Peak bytes held at once in the library's temporary-memory pool on the
 * current device since the last reset; reset when reset != 0. */
E2F_API e2f_status e2f_scratch_high_water(int64_t *bytes, int32_t reset);

#ifdef __cplusplus
}
#endif

#endif /* E2F_H_ */
