// Kernel (1): pooled segment query and key scores.
//
// S2O scores the historical keys of a query segment against a representative
// query of the segment, under a causal mask (gist.science technical summary,
// section 1, "Classement par Segment").  This library takes the unweighted
// mean of the segment's rows over the GQA group's query heads as that query:
//   qbar(b,kvh,s) = mean_{g < G, i in segment s} Q[b, kvh*G+g, i, :]
//   s_j           = qbar . k_j / sqrt(d),   j in [0, e(s))
// The score kernel also reduces, per (segment, 128-key tile), the running
// pair (max, sum exp(s - max)) that the plan turns into M and Z.
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

// ---------------------------------------------------------------------------
// score: CTA = (key tile t of 128 keys, chunk of 64 segments, b*Hkv).
// Only segments s >= t see tile t (e(s) = 128 s + 128 > 128 t), so CTAs whose
// chunk ends before t exit at once.  Dot products are accumulated in fp64:
// qbar is the exact fp64 mean of bf16 values and k_j is bf16, so every
// product is exact and the sum carries ~1e-15 relative error; each score is
// rounded once to fp32.  (fp32 accumulation of these 128-term dots errs by
// ~1e-6 relative when the terms share a sign, the width of the near-tie band
// the importance order is checked against.)
// The d = 128 reduction runs in two halves of 64 so that the transposed key
// tile (fp64) and pooled queries (fp64) fit twice per SM.  Thread (tk, ts)
// accumulates keys 2 tk + 32 a + {0, 1} (a < 4) x segments ts + 16 b (b < 4).
// Outputs:
//   scores[bk][off(s) + j - 64] for candidate keys j of segment s
//   part[bk][s][t] = (max over the tile's admissible keys,
//                     sum exp(s_j - that max))
// ---------------------------------------------------------------------------
constexpr int kScoreKeys = 128;
constexpr int kScoreSegs = 64;
constexpr int kScoreHalf = 64;  // d per pass
constexpr int kQtStride = kScoreSegs + 2;  // padded rows: the transposed fill is conflict-free
constexpr size_t kScoreSmem = sizeof(double) * (kScoreHalf * kScoreKeys + kScoreHalf * kQtStride);

__global__ void __launch_bounds__(256, 2) k_score(const uint16_t* __restrict__ K, const double* __restrict__ qbar,
                                                 float* __restrict__ scores, float2* __restrict__ part,
                                                 int Hkv, int N, int S, int64_t T) {
  const int t = blockIdx.x;           // key tile
  const int chunk = blockIdx.y;       // segment chunk
  const int bk = blockIdx.z;          // b * Hkv + kvh
  const int s_lo = chunk * kScoreSegs;
  const int s_hi = min(S, s_lo + kScoreSegs);
  if (s_hi - 1 < t) return;

  extern __shared__ double smd[];
  double* Kt = smd;                               // [64 d][128 keys]
  double* Qt = smd + kScoreHalf * kScoreKeys;     // [64 d][64 segs], rows padded to kQtStride
  const int tid = threadIdx.x;
  const int tk = tid & 15;
  const int ts = tid >> 4;
  const uint16_t* Kb = K + (size_t)bk * N * kD;
  const double* qb = qbar + (size_t)bk * S * kD;

  double acc[8][4];
#pragma unroll
  for (int a = 0; a < 8; ++a)
#pragma unroll
    for (int q = 0; q < 4; ++q) acc[a][q] = 0.0;

  for (int half = 0; half < 2; ++half) {
    if (half) __syncthreads();
    // key tile half -> fp64, transposed; keys >= N are zero (never admissible)
    for (int q = tid; q < kScoreKeys * 8; q += 256) {
      const int key = q & (kScoreKeys - 1), c = q >> 7;  // c: 16-byte chunk 0..7 of this half
      const int j = t * kScoreKeys + key;
      uint4 w = make_uint4(0, 0, 0, 0);
      if (j < N) w = *reinterpret_cast<const uint4*>(Kb + (size_t)j * kD + half * kScoreHalf + 8 * c);
      if (bf16x2_nonfinite(w.x) | bf16x2_nonfinite(w.y) | bf16x2_nonfinite(w.z) | bf16x2_nonfinite(w.w))
        set_error(kErrNonFinite);
      double* col = Kt + (8 * c) * kScoreKeys + key;
      col[0 * kScoreKeys] = bf16_lo(w.x); col[1 * kScoreKeys] = bf16_hi(w.x);
      col[2 * kScoreKeys] = bf16_lo(w.y); col[3 * kScoreKeys] = bf16_hi(w.y);
      col[4 * kScoreKeys] = bf16_lo(w.z); col[5 * kScoreKeys] = bf16_hi(w.z);
      col[6 * kScoreKeys] = bf16_lo(w.w); col[7 * kScoreKeys] = bf16_hi(w.w);
    }
    for (int q = tid; q < kScoreSegs * kScoreHalf; q += 256) {
      const int seg = q / kScoreHalf, dd = q % kScoreHalf;
      const int s = s_lo + seg;
      Qt[dd * kQtStride + seg] = (s < S) ? qb[(size_t)s * kD + half * kScoreHalf + dd] : 0.0;
    }
    __syncthreads();
#pragma unroll 2
    for (int dd = 0; dd < kScoreHalf; ++dd) {
      double kk[8], qq[4];
#pragma unroll
      for (int a = 0; a < 4; ++a) {  // keys 2 tk + 32 a and 2 tk + 32 a + 1, one 16-byte load
        const double2 k2 = *reinterpret_cast<const double2*>(Kt + dd * kScoreKeys + 2 * tk + 32 * a);
        kk[2 * a] = k2.x;
        kk[2 * a + 1] = k2.y;
      }
#pragma unroll
      for (int q = 0; q < 4; ++q) qq[q] = Qt[dd * kQtStride + ts + 16 * q];
#pragma unroll
      for (int a = 0; a < 8; ++a)
#pragma unroll
        for (int q = 0; q < 4; ++q) acc[a][q] = fma(kk[a], qq[q], acc[a][q]);
    }
  }

  float* sc_bk = scores + (size_t)bk * T;
  float2* part_bk = part + (size_t)bk * S * S;
  const double inv_sqrt_d = 0.08838834764831845;  // 1/sqrt(128), rounded to fp64
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const int s = s_lo + ts + 16 * q;
    const bool seg_ok = (s < s_hi) && (s >= t);
    const int cand_hi = s * kLq - kWin;  // candidates are [64, cand_hi)
    float v[8];
    float mloc = -INFINITY;
#pragma unroll
    for (int a = 0; a < 8; ++a) {
      const int j = t * kScoreKeys + 2 * tk + 32 * (a >> 1) + (a & 1);
      v[a] = (float)(acc[a][q] * inv_sqrt_d);
      const bool adm = seg_ok && (j < N);
      if (adm) {
        if (!isfinite(v[a])) set_error(kErrNonFinite);
        mloc = fmaxf(mloc, v[a]);
        if (j >= kSink && j < cand_hi) sc_bk[cand_offset(s) + (j - kSink)] = v[a];
      } else {
        v[a] = -INFINITY;
      }
    }
    // half-warp (16 lanes share ts) reductions: max, then sum exp(v - max)
#pragma unroll
    for (int o = 8; o >= 1; o >>= 1) mloc = fmaxf(mloc, __shfl_xor_sync(0xffffffffu, mloc, o));
    float z = 0.f;
    if (mloc > -INFINITY) {
#pragma unroll
      for (int a = 0; a < 8; ++a) z += (v[a] > -INFINITY) ? exp_shifted(v[a], mloc) : 0.f;
    }
#pragma unroll
    for (int o = 8; o >= 1; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
    if (tk == 0 && seg_ok) part_bk[(size_t)s * S + t] = make_float2(mloc, z);
  }
}

}  // namespace s2o
