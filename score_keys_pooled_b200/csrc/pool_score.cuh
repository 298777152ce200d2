// Kernel (1), first half: the pooled segment query.
//
// S2O scores the historical keys of a query segment against a representative
// query of the segment, under a causal mask (gist.science technical summary,
// section 1, "Classement par Segment").  This library takes the unweighted
// mean of the segment's rows over the GQA group's query heads as that query:
//   qbar(b,kvh,s) = mean_{g < G, i in segment s} Q[b, kvh*G+g, i, :]
// The scores s_j = qbar . k_j / sqrt(d) and the per-(segment, 128-key window)
// pairs (max, sum exp(s - max)) that the plan turns into M and Z come from
// the integer tensor-core scorer in score_i8.cuh.
#pragma once
#include "s2o_common.cuh"

namespace s2o {

// ---------------------------------------------------------------------------
// pool: one CTA per (s, b*Hkv); 256 threads; thread = (16-byte chunk, row group)
// Q is read once with 16-byte loads; sums and the mean are fp64 (exact for
// bf16 inputs whose magnitudes span less than ~2^36).
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) k_pool(const uint16_t* __restrict__ Q, double* __restrict__ qbar,
                                             int Hq, int Hkv, int N, int S) {
  const int s = blockIdx.x;
  const int bk = blockIdx.y;  // b * Hkv + kvh
  const int b = bk / Hkv, kvh = bk % Hkv;
  const int G = Hq / Hkv;
  const int r0 = s * kLq;
  const int r1 = min(N, r0 + kLq);
  const int c = threadIdx.x & 15;   // 16-byte chunk: dims 8c .. 8c+7
  const int rg = threadIdx.x >> 4;  // row group 0..15

  double acc[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) acc[k] = 0.0;
  bool bad = false;
  for (int g = 0; g < G; ++g) {
    const uint16_t* base = Q + ((size_t)(b * Hq + kvh * G + g) * N) * kD;
    for (int i = r0 + rg; i < r1; i += 16) {
      uint4 w = *reinterpret_cast<const uint4*>(base + (size_t)i * kD + 8 * c);
      bad |= bf16x2_nonfinite(w.x) | bf16x2_nonfinite(w.y) | bf16x2_nonfinite(w.z) | bf16x2_nonfinite(w.w);
      acc[0] += bf16_lo(w.x); acc[1] += bf16_hi(w.x);
      acc[2] += bf16_lo(w.y); acc[3] += bf16_hi(w.y);
      acc[4] += bf16_lo(w.z); acc[5] += bf16_hi(w.z);
      acc[6] += bf16_lo(w.w); acc[7] += bf16_hi(w.w);
    }
  }
  if (bad) set_error(kErrNonFinite);
  __shared__ double red[16][kD];
#pragma unroll
  for (int k = 0; k < 8; ++k) red[rg][8 * c + k] = acc[k];
  __syncthreads();
  if (threadIdx.x < kD) {
    double t = 0.0;
#pragma unroll
    for (int r = 0; r < 16; ++r) t += red[r][threadIdx.x];
    const double cnt = (double)G * (double)(r1 - r0);
    qbar[((size_t)bk * S + s) * kD + threadIdx.x] = t / cnt;
  }
}

}  // namespace s2o
