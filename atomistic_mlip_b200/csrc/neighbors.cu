// Cell-list radius graph -> sorted CSR (the neighbour set j in N(i) that
// E2Former-V2's node-centric attention streams over, "E2Former-V2 ...",
// §2.2 "Streaming reduction").
//
// Steps (all on `stream`):
//   bbox (open dims only; one host read)  -> grid of cells of edge >= r_c
//   cell_assign: cell of each atom + per-cell counts (+ domain check)
//   scan -> cell_start;  cell_scatter -> positions grouped by cell
//   count: warp per atom (in cell order) over the 27-cell stencil, exact
//          fp32 predicate
//   scan -> row_ptr, E read back (one host read), capacity check
//   fill: warp per atom, same stencil; the row is collected in shared
//         memory and written in ascending j (rank placement), or, for rows
//         longer than the shared buffer, written then sorted in place.
#include <math.h>

#include <algorithm>
#include <mutex>

#include "common.cuh"
#include "scan.cuh"

namespace e2f {

struct CellGrid {
  int nc[3];
  float lo[3];    // grid origin (0 in periodic dims)
  float inv[3];   // cells per Angstrom
  int stencil[3]; // 1: offsets -1..1, 0: offset 0 only
};

constexpr int ROW_CAP = 256;   // shared-memory row buffer per warp (longer rows: sorted in global memory)

__global__ void bbox_partial_kernel(const float *__restrict__ pos, int n, float *__restrict__ part) {
  float mn[3] = {INFINITY, INFINITY, INFINITY}, mx[3] = {-INFINITY, -INFINITY, -INFINITY};
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) {
#pragma unroll
    for (int k = 0; k < 3; ++k) {
      float v = pos[3 * i + k];
      mn[k] = fminf(mn[k], v);
      mx[k] = fmaxf(mx[k], v);
    }
  }
  __shared__ float sm[6][32];
#pragma unroll
  for (int k = 0; k < 3; ++k) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      mn[k] = fminf(mn[k], __shfl_xor_sync(0xffffffffu, mn[k], o));
      mx[k] = fmaxf(mx[k], __shfl_xor_sync(0xffffffffu, mx[k], o));
    }
  }
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, nw = blockDim.x >> 5;
  if (lane == 0) {
    for (int k = 0; k < 3; ++k) { sm[k][wid] = mn[k]; sm[3 + k][wid] = mx[k]; }
  }
  __syncthreads();
  if (threadIdx.x < 6) {
    float v = sm[threadIdx.x][0];
    for (int w = 1; w < nw; ++w) v = threadIdx.x < 3 ? fminf(v, sm[threadIdx.x][w]) : fmaxf(v, sm[threadIdx.x][w]);
    part[blockIdx.x * 6 + threadIdx.x] = v;
  }
}

__global__ void bbox_final_kernel(const float *__restrict__ part, int nparts, float *__restrict__ out) {
  if (threadIdx.x < 6) {
    float v = part[threadIdx.x];
    for (int b = 1; b < nparts; ++b)
      v = threadIdx.x < 3 ? fminf(v, part[b * 6 + threadIdx.x]) : fmaxf(v, part[b * 6 + threadIdx.x]);
    out[threadIdx.x] = v;
  }
}

__device__ __forceinline__ int cell_coord(float p, const CellGrid &cg, int k) {
  int c = (int)floorf(__fmul_rn(__fsub_rn(p, cg.lo[k]), cg.inv[k]));
  return min(max(c, 0), cg.nc[k] - 1);
}

__global__ void cell_assign_kernel(const float *__restrict__ pos, int n, CellGrid cg, Geom g,
                                   int32_t *__restrict__ cell_of, int32_t *__restrict__ cell_count,
                                   int32_t *__restrict__ domain_err) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n) return;
  int c[3];
#pragma unroll
  for (int k = 0; k < 3; ++k) {
    float p = pos[3 * i + k];
    bool ok = g.periodic[k] ? (p >= 0.f && p < g.box[k]) : (p == p && fabsf(p) < INFINITY);
    if (!ok) atomicExch(domain_err, 1);
    c[k] = cell_coord(p, cg, k);
  }
  const int cid = c[0] + cg.nc[0] * (c[1] + cg.nc[1] * c[2]);
  cell_of[i] = cid;
  atomicAdd(&cell_count[cid], 1);
}

// Atoms grouped by cell: spos[k] = (x_i, y_i, z_i, bits of i) for the k-th
// atom in cell order, so that a candidate is one 16-byte load.
__global__ void cell_scatter_kernel(const float *__restrict__ pos, const int32_t *__restrict__ cell_of, int n,
                                    const int32_t *__restrict__ cell_start, int32_t *__restrict__ cursor,
                                    float4 *__restrict__ spos) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n) return;
  const int c = cell_of[i];
  const int k = cell_start[c] + atomicAdd(&cursor[c], 1);
  const float3 p = load_pos(pos, i);
  spos[k] = make_float4(p.x, p.y, p.z, __int_as_float(i));
}

// ---------------------------------------------------------------------------
// Pair tests, one CTA per home cell (grid-stride over cells).  The atoms of
// the home cell's stencil cells (27, fewer at open faces or for dimensions
// of fewer than 3 cells) are staged once in shared memory as candidates,
// CAND_CAP at a time, and every home atom is tested against them by one warp
// (lanes over candidates), so a candidate is loaded from global memory once
// per home cell instead of once per home atom.
//
// The minimum image is the exact predicate: d = p_j - p_i rounded, then
// -b if d > b/2, +b if d < -b/2, each rounded.  When every periodic
// dimension has at least 5 cells, the branch taken is the same for all
// candidates of one stencil cell (|d| <= 2 cell edges < b/2 for a cell that
// does not wrap, |d| >= b - 2 cell edges > b/2 for one that does), so the
// staged candidate carries that cell's shift s in {-b, 0, +b} and
// d = fl(fl(p_j - p_i) + s) -- the same rounded operations (adding 0 is
// exact).  Otherwise every pair takes the branch test.
// ---------------------------------------------------------------------------
constexpr int CAND_CAP = 1024;      // candidates staged at a time
constexpr int COUNT_HPW = 3;        // home atoms per warp and sweep in the count pass
constexpr int CELL_THREADS = 256;

struct Stencil {
  int n;                // stencil cells
  int start[27], cnt[27], off[28];
  float sh[27][3];      // per-cell shift (fast path)
};

// Stencil of home cell cid into shared memory, by warp 0: lane q < 27 takes
// stencil offset q (dx fastest), the cells that exist are compacted in lane
// order with a ballot, and the candidate offsets are a warp prefix sum.
__device__ void make_stencil(int cid, const CellGrid &cg, const Geom &g, const int32_t *__restrict__ cell_start,
                             Stencil &st, int lane) {
  const int c0[3] = {cid % cg.nc[0], (cid / cg.nc[0]) % cg.nc[1], cid / (cg.nc[0] * cg.nc[1])};
  bool ok = lane < 27;
  int cc[3] = {0, 0, 0};
  float shv[3] = {0.f, 0.f, 0.f};
  if (ok) {
    const int d[3] = {lane % 3 - 1, (lane / 3) % 3 - 1, lane / 9 - 1};
#pragma unroll
    for (int k = 0; k < 3; ++k) {
      if (d[k] != 0 && cg.stencil[k] == 0) ok = false;
      int v = c0[k] + d[k];
      if (g.periodic[k]) {
        if (v < 0) { v += cg.nc[k]; shv[k] = -g.box[k]; }            // p_j near b, p_i near 0: d > b/2
        else if (v >= cg.nc[k]) { v -= cg.nc[k]; shv[k] = g.box[k]; }  // d < -b/2
      } else if (v < 0 || v >= cg.nc[k]) {
        ok = false;
      }
      cc[k] = v;
    }
  }
  int start = 0, cnt = 0;
  if (ok) {
    const int c = cc[0] + cg.nc[0] * (cc[1] + cg.nc[1] * cc[2]);
    start = cell_start[c];
    cnt = cell_start[c + 1] - start;
  }
  const unsigned m = __ballot_sync(0xffffffffu, ok);
  const int slot = __popc(m & ((1u << lane) - 1u));
  int incl = cnt;   // inclusive prefix of cnt over lanes (zero for lanes that are not cells)
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (ok) {
    st.start[slot] = start;
    st.cnt[slot] = cnt;
    st.off[slot] = incl - cnt;
    st.sh[slot][0] = shv[0]; st.sh[slot][1] = shv[1]; st.sh[slot][2] = shv[2];
  }
  if (lane == 31) {
    st.n = __popc(m);
    st.off[__popc(m)] = incl;
  }
}

// Candidates [c0, c0 + nc) of the stencil into shared memory.
__device__ __forceinline__ void stage_candidates(const Stencil &st, int c0, int nc, const float4 *__restrict__ spos,
                                                 float4 *cp, float4 *cs) {
  for (int k = threadIdx.x; k < nc; k += blockDim.x) {
    const int q = c0 + k;
    int s = 0, hi = st.n - 1;   // last stencil cell with off <= q
    while (s < hi) {
      const int mid = (s + hi + 1) >> 1;
      if (st.off[mid] <= q) s = mid;
      else hi = mid - 1;
    }
    cp[k] = spos[st.start[s] + (q - st.off[s])];
    cs[k] = make_float4(st.sh[s][0], st.sh[s][1], st.sh[s][2], 0.f);
  }
}

// The exact predicate for candidate (pj, shift) against pi.
template <bool FAST>
__device__ __forceinline__ bool is_edge(const Geom &g, float3 pi, float4 pj, float4 sj) {
  float dx, dy, dz;
  if (FAST) {
    dx = __fadd_rn(__fsub_rn(pj.x, pi.x), sj.x);
    dy = __fadd_rn(__fsub_rn(pj.y, pi.y), sj.y);
    dz = __fadd_rn(__fsub_rn(pj.z, pi.z), sj.z);
  } else {
    pair_disp(g, pi, make_float3(pj.x, pj.y, pj.z), dx, dy, dz);
  }
  return pair_r2(dx, dy, dz) < g.rc2;
}

template <bool FAST>
__global__ void __launch_bounds__(CELL_THREADS) cell_count_kernel(int ncell, CellGrid cg, Geom g,
                                                                  const int32_t *__restrict__ cell_start,
                                                                  const float4 *__restrict__ spos,
                                                                  int32_t *__restrict__ deg) {
  __shared__ float4 cp[CAND_CAP], cs[CAND_CAP];
  __shared__ Stencil st;
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, nw = blockDim.x >> 5;
  for (int cid = blockIdx.x; cid < ncell; cid += gridDim.x) {
    const int h0 = cell_start[cid], hn = cell_start[cid + 1] - h0;
    if (hn == 0) continue;   // uniform across the block
    __syncthreads();
    if (wid == 0) make_stencil(cid, cg, g, cell_start, st, lane);
    __syncthreads();
    const int ntot = st.off[st.n];
    // home atoms handled by this warp: counts kept per lane slot
    for (int c0 = 0; c0 < ntot; c0 += CAND_CAP) {
      const int nc = min(CAND_CAP, ntot - c0);
      __syncthreads();
      stage_candidates(st, c0, nc, spos, cp, cs);
      __syncthreads();
      // COUNT_HPW home atoms per warp in one sweep: each staged candidate is
      // read from shared memory once for all of them
      for (int a0 = wid; a0 < hn; a0 += nw * COUNT_HPW) {
        float3 pi[COUNT_HPW];
        int ii[COUNT_HPW], cnt[COUNT_HPW];
#pragma unroll
        for (int q = 0; q < COUNT_HPW; ++q) {
          const int a = a0 + q * nw;
          const float4 me = a < hn ? spos[h0 + a] : make_float4(0.f, 0.f, 0.f, __int_as_float(-1));
          ii[q] = __float_as_int(me.w);
          pi[q] = make_float3(me.x, me.y, me.z);
          cnt[q] = 0;
        }
        for (int k = lane; k < nc; k += 32) {
          const float4 pj = cp[k], sj = cs[k];
          const int j = __float_as_int(pj.w);
#pragma unroll
          for (int q = 0; q < COUNT_HPW; ++q)
            if (j != ii[q] && is_edge<FAST>(g, pi[q], pj, sj)) ++cnt[q];
        }
#pragma unroll
        for (int q = 0; q < COUNT_HPW; ++q) {
          const int c = warp_sum_i(cnt[q]);
          if (lane == 0 && ii[q] >= 0) {
            if (c0 == 0) deg[ii[q]] = c;
            else deg[ii[q]] += c;
          }
        }
      }
    }
  }
}

template <bool FAST>
__global__ void __launch_bounds__(CELL_THREADS) cell_fill_kernel(int ncell, CellGrid cg, Geom g,
                                                                 const int32_t *__restrict__ cell_start,
                                                                 const float4 *__restrict__ spos,
                                                                 const int32_t *__restrict__ row_ptr,
                                                                 int32_t *__restrict__ col_idx) {
  __shared__ float4 cp[CAND_CAP], cs[CAND_CAP];
  __shared__ Stencil st;
  __shared__ int32_t rows[CELL_THREADS / 32][ROW_CAP];
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, nw = blockDim.x >> 5;
  for (int cid = blockIdx.x; cid < ncell; cid += gridDim.x) {
    const int h0 = cell_start[cid], hn = cell_start[cid + 1] - h0;
    if (hn == 0) continue;
    __syncthreads();
    if (wid == 0) make_stencil(cid, cg, g, cell_start, st, lane);
    __syncthreads();
    const int ntot = st.off[st.n];
    if (ntot <= CAND_CAP) {
      // one chunk: each warp builds its home atoms' rows in shared memory
      __syncthreads();
      stage_candidates(st, 0, ntot, spos, cp, cs);
      __syncthreads();
      for (int a = wid; a < hn; a += nw) {
        const float4 me = spos[h0 + a];
        const int i = __float_as_int(me.w);
        const float3 pi = make_float3(me.x, me.y, me.z);
        const int r0 = row_ptr[i], dg = row_ptr[i + 1] - r0;
        int32_t *out = col_idx + r0;
        int32_t *b = rows[wid];
        const bool in_smem = dg <= ROW_CAP;
        int w = 0;
        for (int k0 = 0; k0 < ntot; k0 += 32) {
          const int k = k0 + lane;
          bool pass = false;
          int j = -1;
          if (k < ntot) {
            const float4 pj = cp[k];
            j = __float_as_int(pj.w);
            pass = j != i && is_edge<FAST>(g, pi, pj, cs[k]);
          }
          const unsigned m = __ballot_sync(0xffffffffu, pass);
          const int p = w + __popc(m & ((1u << lane) - 1u));
          if (pass && p < dg) {
            if (in_smem) b[p] = j;
            else out[p] = j;
          }
          w += __popc(m);
        }
        __syncwarp();
        if (in_smem) {
          // rank placement: keys are distinct atom indices
          for (int e = lane; e < dg; e += 32) {
            const int key = b[e];
            int rank = 0;
            for (int t = 0; t < dg; ++t) rank += (b[t] < key);
            out[rank] = key;
          }
        } else {
          for (int round = 0; round < dg; ++round) {   // odd-even transposition sort in place (rare)
            for (int k = 2 * lane + (round & 1); k + 1 < dg; k += 64) {
              const int x = out[k], y = out[k + 1];
              if (x > y) { out[k] = y; out[k + 1] = x; }
            }
            __syncwarp();
          }
        }
        __syncwarp();
      }
    } else {
      // dense stencil (more candidates than one chunk): rows written to
      // global memory chunk by chunk, then sorted in place per row
      int wpos[8];   // per home atom slot of this warp: fill position (up to 8 atoms per warp per pass)
      for (int a0 = 0; a0 < hn; a0 += 8 * nw) {
        for (int q = 0; q < 8; ++q) wpos[q] = 0;
        for (int c0 = 0; c0 < ntot; c0 += CAND_CAP) {
          const int nc = min(CAND_CAP, ntot - c0);
          __syncthreads();
          stage_candidates(st, c0, nc, spos, cp, cs);
          __syncthreads();
#pragma unroll 1
          for (int q = 0; q < 8; ++q) {
            const int a = a0 + q * nw + wid;
            if (a >= hn) break;
            const float4 me = spos[h0 + a];
            const int i = __float_as_int(me.w);
            const float3 pi = make_float3(me.x, me.y, me.z);
            const int r0 = row_ptr[i], dg = row_ptr[i + 1] - r0;
            for (int k0 = 0; k0 < nc; k0 += 32) {
              const int k = k0 + lane;
              bool pass = false;
              int j = -1;
              if (k < nc) {
                const float4 pj = cp[k];
                j = __float_as_int(pj.w);
                pass = j != i && is_edge<FAST>(g, pi, pj, cs[k]);
              }
              const unsigned m = __ballot_sync(0xffffffffu, pass);
              const int p = wpos[q] + __popc(m & ((1u << lane) - 1u));
              if (pass && p < dg) col_idx[r0 + p] = j;
              wpos[q] += __popc(m);
            }
          }
        }
        __syncwarp();
#pragma unroll 1
        for (int q = 0; q < 8; ++q) {
          const int a = a0 + q * nw + wid;
          if (a >= hn) break;
          const int i = __float_as_int(spos[h0 + a].w);
          const int r0 = row_ptr[i], dg = row_ptr[i + 1] - r0;
          int32_t *out = col_idx + r0;
          for (int round = 0; round < dg; ++round) {
            for (int k = 2 * lane + (round & 1); k + 1 < dg; k += 64) {
              const int x = out[k], y = out[k + 1];
              if (x > y) { out[k] = y; out[k + 1] = x; }
            }
            __syncwarp();
          }
        }
      }
    }
  }
}

// Both stencil passes for one grid: the fast shift form when every periodic
// dimension has at least 5 cells.
static bool fast_shift_ok(const CellGrid &cg, const Geom &g) {
  for (int k = 0; k < 3; ++k)
    if (g.periodic[k] && cg.nc[k] < 5) return false;
  return true;
}

static int cell_grid_blocks(long long ncell) {
  int dev = 0, nsm = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
  // one CTA per cell (up to 16 waves of resident CTAs, grid-stride beyond):
  // cells differ in cost, so the hardware's block scheduler balances them
  return (int)std::max<long long>(1, std::min<long long>(ncell, (long long)nsm * 96));
}

static e2f_status launch_count(long long ncell, const CellGrid &cg, const Geom &g, const int32_t *cstart,
                               const float4 *spos, int32_t *deg, cudaStream_t s) {
  const int grid = cell_grid_blocks(ncell);
  if (fast_shift_ok(cg, g))
    E2F_LAUNCH(cell_count_kernel<true>, grid, CELL_THREADS, 0, s, (int)ncell, cg, g, cstart, spos, deg);
  else
    E2F_LAUNCH(cell_count_kernel<false>, grid, CELL_THREADS, 0, s, (int)ncell, cg, g, cstart, spos, deg);
  return E2F_OK;
}

static e2f_status launch_fill(long long ncell, const CellGrid &cg, const Geom &g, const int32_t *cstart,
                              const float4 *spos, const int32_t *row_ptr, int32_t *col_idx, cudaStream_t s) {
  const int grid = cell_grid_blocks(ncell);
  if (fast_shift_ok(cg, g))
    E2F_LAUNCH(cell_fill_kernel<true>, grid, CELL_THREADS, 0, s, (int)ncell, cg, g, cstart, spos, row_ptr, col_idx);
  else
    E2F_LAUNCH(cell_fill_kernel<false>, grid, CELL_THREADS, 0, s, (int)ncell, cg, g, cstart, spos, row_ptr,
               col_idx);
  return E2F_OK;
}

// --------------------------------------------------------------------------
e2f_status build_neighbors_impl(const float *pos, int64_t N, const float *box, float r_c,
                                int32_t *row_ptr, int32_t *col_idx, int64_t capacity, int64_t *n_edges,
                                cudaStream_t s) {
  Geom g;
  bool any_open = false;
  for (int k = 0; k < 3; ++k) {
    const float b = box ? box[k] : 0.f;
    g.periodic[k] = b > 0.f;
    g.box[k] = g.periodic[k] ? b : 0.f;
    g.half[k] = 0.5f * g.box[k];
    any_open |= !g.periodic[k];
  }
  g.rc = r_c;
  g.rc2 = r_c * r_c;
  const int n = (int)N;
  if (n == 0) {
    E2F_CUDA_TRY(cudaMemsetAsync(row_ptr, 0, sizeof(int32_t), s));
    *n_edges = 0;
    return E2F_OK;
  }

  // bounding box of open dimensions (host sync 1)
  float bb[6] = {0, 0, 0, 0, 0, 0};
  if (any_open) {
    const int nparts = std::min(256, (n + 255) / 256);
    Scratch part;
    E2F_CUDA_TRY(part.alloc(sizeof(float) * (6 * nparts + 6), s));
    float *pp = part.as<float>();
    E2F_LAUNCH(bbox_partial_kernel, nparts, 256, 0, s, pos, n, pp);
    E2F_LAUNCH(bbox_final_kernel, 1, 32, 0, s, pp, nparts, pp + 6 * nparts);
    E2F_CUDA_TRY(cudaMemcpyAsync(bb, pp + 6 * nparts, sizeof(bb), cudaMemcpyDeviceToHost, s));
    E2F_CUDA_TRY(cudaStreamSynchronize(s));
    for (int k = 0; k < 6; ++k)
      if (!(fabsf(bb[k]) < INFINITY)) return E2F_ERR_DOMAIN;
  }

  // cell grid: cells of edge >= r_c with a relative margin far above the
  // rounding of the cell-index computation
  CellGrid cg;
  double cs[3];
  long long ncell = 1;
  for (int k = 0; k < 3; ++k) {
    if (g.periodic[k]) {
      const double b = g.box[k];
      const double cmin = (double)r_c * 1.001 + b * 1e-6;
      int nc = (int)floor(b / cmin);
      if (nc < 3) nc = 1;
      cg.nc[k] = nc;
      cg.lo[k] = 0.f;
      cs[k] = b / nc;
      cg.inv[k] = (float)(nc / b);
      cg.stencil[k] = nc >= 3 ? 1 : 0;
    } else {
      const double ext = (double)bb[3 + k] - (double)bb[k];
      cs[k] = (double)r_c * 1.001 + fabs(ext) * 1e-6 + 1e-6 * fabs((double)bb[k]);
      cg.lo[k] = bb[k];
    }
  }
  // bound the number of cells (sparse open systems): grow open cells
  for (int it = 0; it < 64; ++it) {
    ncell = 1;
    for (int k = 0; k < 3; ++k) {
      if (!g.periodic[k]) {
        const double ext = (double)bb[3 + k] - (double)bb[k];
        cg.nc[k] = (int)std::min<double>(floor(ext / cs[k]) + 1.0, 1 << 20);
        cg.inv[k] = (float)(1.0 / cs[k]);
        cg.stencil[k] = 1;
      }
      ncell *= cg.nc[k];
    }
    if (ncell <= std::max<long long>(4096, 8LL * n)) break;
    for (int k = 0; k < 3; ++k)
      if (!g.periodic[k]) cs[k] *= 1.25;
  }

  // one pool allocation, carved into 256-byte aligned pieces; the counters
  // that must start at zero are adjacent and cleared by one memset
  auto up = [](size_t b) { return (b + 255) & ~(size_t)255; };
  const size_t o_cnt = 0, o_cursor = up(sizeof(int32_t) * ncell), o_flag = o_cursor + up(sizeof(int32_t) * ncell);
  const size_t zero_bytes = o_flag + 16;
  const size_t o_cstart = up(zero_bytes), o_cell_of = o_cstart + up(sizeof(int32_t) * (ncell + 1));
  const size_t o_deg = o_cell_of + up(sizeof(int32_t) * n), o_scan = o_deg + up(sizeof(int32_t) * n);
  const size_t o_spos = o_scan + up(std::max(scan_scratch_bytes(ncell), scan_scratch_bytes(n)));
  const size_t total_bytes = o_spos + sizeof(float4) * n;
  Scratch ws;
  E2F_CUDA_TRY(ws.alloc(total_bytes, s));
  char *wb = ws.as<char>();
  int32_t *cnt = reinterpret_cast<int32_t *>(wb + o_cnt), *cursor = reinterpret_cast<int32_t *>(wb + o_cursor);
  int32_t *flag = reinterpret_cast<int32_t *>(wb + o_flag), *cstart = reinterpret_cast<int32_t *>(wb + o_cstart);
  int32_t *cell_of = reinterpret_cast<int32_t *>(wb + o_cell_of), *deg = reinterpret_cast<int32_t *>(wb + o_deg);
  void *scan_tmp = wb + o_scan;
  float4 *spos = reinterpret_cast<float4 *>(wb + o_spos);
  E2F_CUDA_TRY(cudaMemsetAsync(wb, 0, zero_bytes, s));

  const int tb = 256;
  E2F_LAUNCH(cell_assign_kernel, (n + tb - 1) / tb, tb, 0, s, pos, n, cg, g, cell_of,
             cnt, flag);
  e2f_status st = exclusive_scan(cnt, ncell, cstart, scan_tmp, s, nullptr);
  if (st != E2F_OK) return st;
  E2F_LAUNCH(cell_scatter_kernel, (n + tb - 1) / tb, tb, 0, s, pos, cell_of, n,
             cstart, cursor, spos);
  st = launch_count(ncell, cg, g, cstart, spos, deg, s);
  if (st != E2F_OK) return st;
  long long *total = nullptr;
  st = exclusive_scan(deg, n, row_ptr, scan_tmp, s, &total);
  if (st != E2F_OK) return st;

  // E and the domain flag (host sync 2)
  long long E = 0;
  int32_t dom = 0;
  E2F_CUDA_TRY(cudaMemcpyAsync(&E, total, sizeof(long long), cudaMemcpyDeviceToHost, s));
  E2F_CUDA_TRY(cudaMemcpyAsync(&dom, flag, sizeof(int32_t), cudaMemcpyDeviceToHost, s));
  E2F_CUDA_TRY(cudaStreamSynchronize(s));
  *n_edges = E;
  if (dom) return E2F_ERR_DOMAIN;
  if (E > INT32_MAX) return E2F_ERR_UNSUPPORTED;
  if (E > capacity) return E2F_ERR_CAPACITY;
  if (E > 0) {
    st = launch_fill(ncell, cg, g, cstart, spos, row_ptr, col_idx, s);
    if (st != E2F_OK) return st;
  }
  return E2F_OK;
}

}  // namespace e2f

// ===========================================================================
// Allocation-free variant: e2f_build_neighbors_noalloc.
//
// Same kernels and the same result as e2f_build_neighbors, but every
// temporary array lives in one fixed, file-scope device array instead of
// memory taken from a pool, so the call never allocates device memory.
// Limits: at most NOALLOC_MAX_ATOMS atoms; the cell grid is coarsened (cells
// only grow, which never drops a pair) until it has at most
// NOALLOC_MAX_CELLS cells.  Every call on a device shares the array and it
// keeps the previous call's contents, so the counters that must start at
// zero are cleared on the stream first, and two calls whose GPU work
// overlaps (different streams, no ordering between them) race on it.
// ===========================================================================
namespace e2f {

constexpr int64_t NOALLOC_MAX_ATOMS = 1 << 17;   // 131,072 atoms
constexpr int64_t NOALLOC_MAX_CELLS = 1 << 17;   // 131,072 cells

// layout of the array, in 4-byte words (offsets kept 64-word aligned)
constexpr size_t NA_CELL_OF = 0;
constexpr size_t NA_DEG = NA_CELL_OF + NOALLOC_MAX_ATOMS;
constexpr size_t NA_CNT = NA_DEG + NOALLOC_MAX_ATOMS;
constexpr size_t NA_CSTART = NA_CNT + NOALLOC_MAX_CELLS;
constexpr size_t NA_CURSOR = NA_CSTART + NOALLOC_MAX_CELLS + 64;
constexpr size_t NA_FLAG = NA_CURSOR + NOALLOC_MAX_CELLS;
constexpr size_t NA_BBOX = NA_FLAG + 64;
constexpr size_t NA_SCAN = NA_BBOX + 2048;        // 6 * 256 + 6 floats fit
constexpr size_t NA_SPOS = NA_SCAN + 256;         // scan sums: long longs; then float4 per atom
constexpr size_t NA_WORDS = NA_SPOS + 4 * NOALLOC_MAX_ATOMS;
static_assert(NA_SPOS % 4 == 0, "cell-sorted positions need 16-byte alignment");
static_assert(NA_SCAN % 2 == 0, "scan sums need 8-byte alignment");

static __device__ __align__(256) int32_t g_noalloc_scratch[NA_WORDS];

// Device address of the array on the current device (looked up once per
// device; host code cannot use the symbol itself as a device address).
static std::mutex g_na_mu;
static void *g_na_ptr[64] = {nullptr};

static e2f_status noalloc_scratch(int32_t **p) {
  int dev = 0;
  E2F_CUDA_TRY(cudaGetDevice(&dev));
  if (dev < 0 || dev >= 64) return E2F_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lk(g_na_mu);
  if (!g_na_ptr[dev]) {
    void *ptr = nullptr;
    E2F_CUDA_TRY(cudaGetSymbolAddress(&ptr, g_noalloc_scratch));
    g_na_ptr[dev] = ptr;
  }
  *p = static_cast<int32_t *>(g_na_ptr[dev]);
  return E2F_OK;
}

static e2f_status build_neighbors_noalloc_impl(const float *pos, int64_t N, const float *box, float r_c,
                                               int32_t *row_ptr, int32_t *col_idx, int64_t capacity,
                                               int64_t *n_edges, cudaStream_t s) {
  int32_t *ws = nullptr;
  e2f_status st = noalloc_scratch(&ws);
  if (st != E2F_OK) return st;
  Geom g;
  bool any_open = false;
  for (int k = 0; k < 3; ++k) {
    const float b = box ? box[k] : 0.f;
    g.periodic[k] = b > 0.f;
    g.box[k] = g.periodic[k] ? b : 0.f;
    g.half[k] = 0.5f * g.box[k];
    any_open |= !g.periodic[k];
  }
  g.rc = r_c;
  g.rc2 = r_c * r_c;
  const int n = (int)N;
  if (n == 0) {
    E2F_CUDA_TRY(cudaMemsetAsync(row_ptr, 0, sizeof(int32_t), s));
    *n_edges = 0;
    return E2F_OK;
  }
  float bb[6] = {0, 0, 0, 0, 0, 0};
  if (any_open) {
    const int nparts = std::min(256, (n + 255) / 256);
    float *pp = reinterpret_cast<float *>(ws + NA_BBOX);
    E2F_LAUNCH(bbox_partial_kernel, nparts, 256, 0, s, pos, n, pp);
    E2F_LAUNCH(bbox_final_kernel, 1, 32, 0, s, pp, nparts, pp + 6 * nparts);
    E2F_CUDA_TRY(cudaMemcpyAsync(bb, pp + 6 * nparts, sizeof(bb), cudaMemcpyDeviceToHost, s));
    E2F_CUDA_TRY(cudaStreamSynchronize(s));
    for (int k = 0; k < 6; ++k)
      if (!(fabsf(bb[k]) < INFINITY)) return E2F_ERR_DOMAIN;
  }
  CellGrid cg;
  double cs[3];
  for (int k = 0; k < 3; ++k) {
    if (g.periodic[k]) {
      const double b = g.box[k];
      const double cmin = (double)r_c * 1.001 + b * 1e-6;
      int nc = (int)floor(b / cmin);
      if (nc < 3) nc = 1;
      cg.nc[k] = nc;
      cg.lo[k] = 0.f;
    } else {
      const double ext = (double)bb[3 + k] - (double)bb[k];
      cs[k] = (double)r_c * 1.001 + fabs(ext) * 1e-6 + 1e-6 * fabs((double)bb[k]);
      cg.lo[k] = bb[k];
    }
  }
  const long long cap = std::min<long long>(std::max<long long>(4096, 8LL * n), NOALLOC_MAX_CELLS);
  long long ncell = 1;
  for (int it = 0; it < 256; ++it) {
    ncell = 1;
    for (int k = 0; k < 3; ++k) {
      if (!g.periodic[k]) {
        const double ext = (double)bb[3 + k] - (double)bb[k];
        cg.nc[k] = (int)std::min<double>(floor(ext / cs[k]) + 1.0, 1 << 20);
        cg.inv[k] = (float)(1.0 / cs[k]);
        cg.stencil[k] = 1;
      }
      ncell *= cg.nc[k];
    }
    if (ncell <= cap) break;
    // coarsen every dimension at once by the factor that brings the count to
    // the cap: cells only grow, which never drops a pair.  A periodic count
    // falls by at least one per pass and becomes 1 below 3; open cells grow
    // by at least 25 % per pass, so the loop ends after a few passes.
    const double f = cbrt((double)cap / (double)ncell);
    for (int k = 0; k < 3; ++k) {
      if (g.periodic[k]) {
        int nc = std::min((int)floor(cg.nc[k] * f), cg.nc[k] - 1);
        cg.nc[k] = nc < 3 ? 1 : nc;
      } else {
        cs[k] *= std::max(1.25, 1.0 / f);
      }
    }
  }
  if (ncell > NOALLOC_MAX_CELLS) return E2F_ERR_SCRATCH_LIMIT;
  for (int k = 0; k < 3; ++k) {
    if (g.periodic[k]) {
      cg.inv[k] = (float)(cg.nc[k] / (double)g.box[k]);
      cg.stencil[k] = cg.nc[k] >= 3 ? 1 : 0;
    }
  }
  int32_t *cell_of = ws + NA_CELL_OF, *deg = ws + NA_DEG;
  int32_t *cnt = ws + NA_CNT, *cstart = ws + NA_CSTART, *cursor = ws + NA_CURSOR, *flag = ws + NA_FLAG;
  float4 *spos = reinterpret_cast<float4 *>(ws + NA_SPOS);
  void *scan_tmp = ws + NA_SCAN;
  E2F_CUDA_TRY(cudaMemsetAsync(cnt, 0, sizeof(int32_t) * ncell, s));
  E2F_CUDA_TRY(cudaMemsetAsync(cursor, 0, sizeof(int32_t) * ncell, s));
  E2F_CUDA_TRY(cudaMemsetAsync(flag, 0, sizeof(int32_t) * 4, s));
  const int tb = 256;
  E2F_LAUNCH(cell_assign_kernel, (n + tb - 1) / tb, tb, 0, s, pos, n, cg, g, cell_of, cnt, flag);
  st = exclusive_scan(cnt, ncell, cstart, scan_tmp, s, nullptr);
  if (st != E2F_OK) return st;
  E2F_LAUNCH(cell_scatter_kernel, (n + tb - 1) / tb, tb, 0, s, pos, cell_of, n, cstart, cursor, spos);
  st = launch_count(ncell, cg, g, cstart, spos, deg, s);
  if (st != E2F_OK) return st;
  long long *total = nullptr;
  st = exclusive_scan(deg, n, row_ptr, scan_tmp, s, &total);
  if (st != E2F_OK) return st;
  long long E = 0;
  int32_t dom = 0;
  E2F_CUDA_TRY(cudaMemcpyAsync(&E, total, sizeof(long long), cudaMemcpyDeviceToHost, s));
  E2F_CUDA_TRY(cudaMemcpyAsync(&dom, flag, sizeof(int32_t), cudaMemcpyDeviceToHost, s));
  E2F_CUDA_TRY(cudaStreamSynchronize(s));
  *n_edges = E;
  if (dom) return E2F_ERR_DOMAIN;
  if (E > INT32_MAX) return E2F_ERR_UNSUPPORTED;
  if (E > capacity) return E2F_ERR_CAPACITY;
  if (E > 0) {
    st = launch_fill(ncell, cg, g, cstart, spos, row_ptr, col_idx, s);
    if (st != E2F_OK) return st;
  }
  return E2F_OK;
}

}  // namespace e2f

extern "C" e2f_status e2f_build_neighbors_noalloc(const float *pos, int64_t N, const float *box, float r_c,
                                                  int32_t *row_ptr, int32_t *col_idx, int64_t capacity,
                                                  int64_t *n_edges, e2f_csr *out_csr, void *stream) {
  using namespace e2f;
  if (N < 0 || !n_edges || !row_ptr || capacity < 0) return E2F_ERR_INVALID_ARG;
  if (N > NOALLOC_MAX_ATOMS) return E2F_ERR_SCRATCH_LIMIT;
  if (N > 0 && !pos) return E2F_ERR_INVALID_ARG;
  if (capacity > 0 && !col_idx) return E2F_ERR_INVALID_ARG;
  if (!(r_c > 0.f) || !(r_c < INFINITY)) return E2F_ERR_INVALID_ARG;
  if (box) {
    for (int k = 0; k < 3; ++k) {
      if (!(box[k] >= 0.f) || !(box[k] < INFINITY)) return E2F_ERR_INVALID_ARG;
      if (box[k] > 0.f && !(r_c < 0.5f * box[k])) return E2F_ERR_CUTOFF_TOO_LARGE;
    }
  }
  e2f_status st = build_neighbors_noalloc_impl(pos, N, box, r_c, row_ptr, col_idx, capacity, n_edges,
                                               static_cast<cudaStream_t>(stream));
  if (st != E2F_OK && st != E2F_ERR_CAPACITY) return st;
  if (out_csr) {
    out_csr->row_ptr = row_ptr;
    out_csr->col_idx = col_idx;
    out_csr->n_nodes = N;
    out_csr->n_edges = *n_edges;
    for (int k = 0; k < 3; ++k) out_csr->box[k] = box ? box[k] : 0.f;
    out_csr->r_c = r_c;
  }
  return st;
}
