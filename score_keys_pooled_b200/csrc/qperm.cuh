// Q_perm with two query sub-segments (gist.science technical summary,
// section 1, "Classement par Segment": the queries of a segment are reordered
// by a coarse importance score against a shared guide vector).
//
// Guide vector: the segment's pooled query qbar (from k_pool).  Importance of
// row i: the mean over the group's query heads of q_{h,i} . qbar (fp64).
// Rows ordered by importance descending, ties to the lower row; the first
// Lq/2 rows form sub-segment 0, the rest sub-segment 1.  Each sub-segment gets
// its own pooled query (the exact fp64 mean of its rows over the group's
// heads, as k_pool computes the segment's) and is then planned like a
// segment; a row attends over its own sub-segment's kept set.
//
//   k_qperm  one CTA per (segment, b*Hkv), one thread per row (importance and
//            rank) and per dimension (the two pooled queries)
#pragma once
#include "s2o_common.cuh"

namespace s2o {

constexpr int kSubRows = kLq / 2;

__global__ void __launch_bounds__(kLq) k_qperm(const uint16_t* __restrict__ Q, const double* __restrict__ qbar,
                                              double* __restrict__ qsub0, double* __restrict__ qsub1,
                                              uint8_t* __restrict__ rowsub, int Hq, int Hkv, int N, int S) {
  __shared__ double qb[kD];
  __shared__ double imp[kLq];
  __shared__ uint8_t sub[kLq];
  const int s = blockIdx.x;
  const int bk = blockIdx.y;
  const int b = bk / Hkv, kvh = bk % Hkv;
  const int G = Hq / Hkv;
  const int r0 = kLq * s;
  const int rows = min(kLq, N - r0);
  const int t = threadIdx.x;
  const size_t seg = (size_t)bk * S + s;
  qb[t] = qbar[seg * kD + t];
  __syncthreads();

  // importance of row t
  double g = 0.0;
  if (t < rows) {
    for (int h = 0; h < G; ++h) {
      const uint16_t* q = Q + ((size_t)(b * Hq + kvh * G + h) * N + r0 + t) * kD;
      double dot = 0.0;
#pragma unroll 4
      for (int c = 0; c < kD / 8; ++c) {
        const uint4 w = *reinterpret_cast<const uint4*>(q + 8 * c);
        dot += bf16_lo(w.x) * qb[8 * c] + bf16_hi(w.x) * qb[8 * c + 1];
        dot += bf16_lo(w.y) * qb[8 * c + 2] + bf16_hi(w.y) * qb[8 * c + 3];
        dot += bf16_lo(w.z) * qb[8 * c + 4] + bf16_hi(w.z) * qb[8 * c + 5];
        dot += bf16_lo(w.w) * qb[8 * c + 6] + bf16_hi(w.w) * qb[8 * c + 7];
      }
      g += dot;
    }
    g /= (double)G;
  }
  imp[t] = g;
  __syncthreads();
  // rank among the segment's rows: importance descending, ties to the lower row
  const int n0 = min(kSubRows, rows);
  uint8_t my = 1;
  if (t < rows) {
    int rank = 0;
    for (int j = 0; j < rows; ++j) rank += (imp[j] > g) || (imp[j] == g && j < t);
    my = rank < n0 ? 0 : 1;
  }
  sub[t] = my;
  rowsub[seg * kLq + t] = my;
  __syncthreads();

  // pooled queries of the two sub-segments: thread t owns dimension t
  double a0 = 0.0, a1 = 0.0;
  for (int h = 0; h < G; ++h) {
    const uint16_t* q = Q + ((size_t)(b * Hq + kvh * G + h) * N + r0) * kD + t;
    for (int i = 0; i < rows; ++i) {
      const uint32_t bits = (uint32_t)q[(size_t)i * kD] << 16;
      const double v = (double)__uint_as_float(bits);
      if (sub[i] == 0) a0 += v; else a1 += v;
    }
  }
  const int n1 = rows - n0;
  qsub0[seg * kD + t] = a0 / ((double)G * (double)n0);
  qsub1[seg * kD + t] = n1 > 0 ? a1 / ((double)G * (double)n1) : qb[t];
}

}  // namespace s2o
