/*
 * Brute-force all-pairs radius graph with the exact fp32 predicate.
 * TEST INFRASTRUCTURE ONLY (oracle); never linked into the product library.
 *
 * The neighbour set j in N(i) is the one the on-the-fly attention streams
 * over ("E2Former-V2: On-the-Fly Equivariant Attention with Linear
 * Activation Memory", §2.2 "Streaming reduction").  The pages give no
 * rounding rule; the predicate below is the reading this project fixes:
 *   d_k = p_j,k - p_i,k                       (fp32, round to nearest)
 *   periodic k:  d_k > b_k/2 -> d_k -= b_k;  d_k < -b_k/2 -> d_k += b_k
 *   r2 = (d_x*d_x + d_y*d_y) + d_z*d_z        (fp32, no fused multiply-add)
 *   edge iff i != j and r2 < r_c*r_c          (product rounded in fp32)
 * Compile with -ffp-contract=off so that no multiply-add is fused.
 *
 * Rows are listed by i, columns in ascending j.  Two passes over all pairs:
 * count, then fill.  Parallel over rows with OpenMP (each row is written
 * by one thread only, so the result is deterministic).
 */
#include <stdint.h>

static int is_edge(const float *pos, int64_t i, int64_t j, const float *box,
                   const int *periodic, float half0, float half1, float half2,
                   float rc2) {
  float d0 = pos[3 * j + 0] - pos[3 * i + 0];
  float d1 = pos[3 * j + 1] - pos[3 * i + 1];
  float d2 = pos[3 * j + 2] - pos[3 * i + 2];
  if (periodic[0]) { if (d0 > half0) d0 -= box[0]; else if (d0 < -half0) d0 += box[0]; }
  if (periodic[1]) { if (d1 > half1) d1 -= box[1]; else if (d1 < -half1) d1 += box[1]; }
  if (periodic[2]) { if (d2 > half2) d2 -= box[2]; else if (d2 < -half2) d2 += box[2]; }
  float a = d0 * d0;
  float b = d1 * d1;
  float s = a + b;
  float c = d2 * d2;
  float r2 = s + c;
  return r2 < rc2;
}

/* Count pass: deg[i] = |N(i)|. */
void oracle_bf_count(const float *pos, int64_t n, const float *box, const int *periodic,
                     float rc, int64_t *deg) {
  float rc2 = rc * rc;
  float h0 = 0.5f * box[0], h1 = 0.5f * box[1], h2 = 0.5f * box[2];
#pragma omp parallel for schedule(dynamic, 64)
  for (int64_t i = 0; i < n; ++i) {
    int64_t c = 0;
    for (int64_t j = 0; j < n; ++j)
      if (j != i && is_edge(pos, i, j, box, periodic, h0, h1, h2, rc2)) ++c;
    deg[i] = c;
  }
}

/* Fill pass: col[row_ptr[i] ..] = ascending j. */
void oracle_bf_fill(const float *pos, int64_t n, const float *box, const int *periodic,
                    float rc, const int64_t *row_ptr, int32_t *col) {
  float rc2 = rc * rc;
  float h0 = 0.5f * box[0], h1 = 0.5f * box[1], h2 = 0.5f * box[2];
#pragma omp parallel for schedule(dynamic, 64)
  for (int64_t i = 0; i < n; ++i) {
    int64_t w = row_ptr[i];
    for (int64_t j = 0; j < n; ++j)
      if (j != i && is_edge(pos, i, j, box, periodic, h0, h1, h2, rc2)) col[w++] = (int32_t)j;
  }
}
