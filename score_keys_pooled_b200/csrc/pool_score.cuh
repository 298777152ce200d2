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
// Only segments s >= t see tile t (e(s) = 128 s + 128 > 128 t), so the grid
// holds only the pairs whose chunk reaches t.  Dot products are accumulated in fp64:
// qbar is the exact fp64 mean of bf16 values and k_j is bf16, so every
// product is exact and the sum carries ~1e-15 relative error; each score is
// rounded once to fp32.  (fp32 accumulation of these 128-term dots errs by
// ~1e-6 relative when the terms share a sign, the width of the near-tie band
// the importance order is checked against.)
// The products run on the fp64 tensor path (mma.sync m8n8k4): each warp owns
// 16 segments x 64 keys (2 x 8 accumulator tiles), and its operand fragments
// are reused across 256 multiply-adds per instruction, where scalar fp64 FMAs
// were bound by shared-memory reads.  The d = 128 reduction runs in two
// halves of 64 so that the key tile and the pooled queries (fp64, rows padded
// to 68 doubles: the fragment pattern is then conflict-free) fit twice per
// SM.  The sums are then staged in shared memory for the epilogue, where
// thread (tk, ts) takes keys 2 tk + 32 a + {0, 1} (a < 4) x segments
// ts + 16 b (b < 4).
// Outputs:
//   scores[bk][off(s) + j - 64] for candidate keys j of segment s
//   part[bk][s][t] = (max over the tile's admissible keys,
//                     sum exp(s_j - that max))
// ---------------------------------------------------------------------------
constexpr int kScoreKeys = 128;
constexpr int kScoreSegs = 64;
constexpr int kScoreHalf = 64;       // d per pass
constexpr int kScoreStride = 68;     // padded rows of the fp64 operand tiles
constexpr int kStageStride = kScoreKeys + 2;  // epilogue staging [64 segs][128 keys], padded
constexpr size_t kScoreSmem = sizeof(double) * (kScoreKeys * kScoreStride + kScoreSegs * kScoreStride);
static_assert(kScoreSegs * kStageStride <= kScoreKeys * kScoreStride + kScoreSegs * kScoreStride,
              "staging must fit in the operand tiles");

__device__ __forceinline__ void dmma_8x8x4(double& c0, double& c1, double a, double b) {
  asm volatile("mma.sync.aligned.m8n8k4.row.col.f64.f64.f64.f64 {%0, %1}, {%2}, {%3}, {%0, %1};\n"
               : "+d"(c0), "+d"(c1)
               : "d"(a), "d"(b));
}

__global__ void __launch_bounds__(256, 2) k_score(const uint16_t* __restrict__ K, const double* __restrict__ qbar,
                                                 float* __restrict__ scores, float2* __restrict__ part,
                                                 int Hkv, int N, int S, int64_t T) {
  // blockIdx.x enumerates the (chunk, tile) pairs on or below the causal
  // diagonal, chunk-major: chunk c holds the tiles t < min(S, 64 (c + 1))
  const int nchunks = (S + kScoreSegs - 1) / kScoreSegs;
  int t = blockIdx.x;                 // key tile, once the chunks before are skipped
  int chunk = 0;                      // segment chunk
  while (chunk < nchunks && t >= min(S, kScoreSegs * (chunk + 1))) {
    t -= min(S, kScoreSegs * (chunk + 1));
    ++chunk;
  }
  if (chunk >= nchunks) return;
  const int bk = blockIdx.y;          // b * Hkv + kvh
  const int s_lo = chunk * kScoreSegs;
  const int s_hi = min(S, s_lo + kScoreSegs);
  if (s_hi - 1 < t) return;

  extern __shared__ double smd[];
  double* Ks = smd;                                // [128 keys][64 d], rows of kScoreStride
  double* Qs = smd + kScoreKeys * kScoreStride;    // [64 segs][64 d], rows of kScoreStride
  const int tid = threadIdx.x;
  const int lane = tid & 31, warp = tid >> 5;
  const uint16_t* Kb = K + (size_t)bk * N * kD;
  const double* qb = qbar + (size_t)bk * S * kD;
  // this warp's block: segments m0 .. m0+15, keys n0 .. n0+63
  const int m0 = 16 * (warp & 3), n0 = 64 * (warp >> 2);
  const int fr = lane >> 2, fc = lane & 3;  // fragment row / column of this lane

  double c[2][8][2];
#pragma unroll
  for (int mt = 0; mt < 2; ++mt)
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) c[mt][nt][0] = c[mt][nt][1] = 0.0;

  for (int half = 0; half < 2; ++half) {
    if (half) __syncthreads();
    // key tile half -> fp64, row-major; keys >= N are zero (never admissible)
    for (int q = tid; q < kScoreKeys * 8; q += 256) {
      const int key = q >> 3, cch = q & 7;  // cch: 16-byte chunk 0..7 of this half
      const int j = t * kScoreKeys + key;
      uint4 w = make_uint4(0, 0, 0, 0);
      if (j < N) w = *reinterpret_cast<const uint4*>(Kb + (size_t)j * kD + half * kScoreHalf + 8 * cch);
      if (bf16x2_nonfinite(w.x) | bf16x2_nonfinite(w.y) | bf16x2_nonfinite(w.z) | bf16x2_nonfinite(w.w))
        set_error(kErrNonFinite);
      double* row = Ks + key * kScoreStride + 8 * cch;
      row[0] = bf16_lo(w.x); row[1] = bf16_hi(w.x);
      row[2] = bf16_lo(w.y); row[3] = bf16_hi(w.y);
      row[4] = bf16_lo(w.z); row[5] = bf16_hi(w.z);
      row[6] = bf16_lo(w.w); row[7] = bf16_hi(w.w);
    }
    for (int q = tid; q < kScoreSegs * kScoreHalf; q += 256) {
      const int seg = q / kScoreHalf, dd = q % kScoreHalf;
      const int s = s_lo + seg;
      Qs[seg * kScoreStride + dd] = (s < S) ? qb[(size_t)s * kD + half * kScoreHalf + dd] : 0.0;
    }
    __syncthreads();
#pragma unroll 2
    for (int k0 = 0; k0 < kScoreHalf; k0 += 4) {
      double a[2], bb[8];
#pragma unroll
      for (int mt = 0; mt < 2; ++mt) a[mt] = Qs[(m0 + 8 * mt + fr) * kScoreStride + k0 + fc];
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) bb[nt] = Ks[(n0 + 8 * nt + fr) * kScoreStride + k0 + fc];
#pragma unroll
      for (int mt = 0; mt < 2; ++mt)
#pragma unroll
        for (int nt = 0; nt < 8; ++nt) dmma_8x8x4(c[mt][nt][0], c[mt][nt][1], a[mt], bb[nt]);
    }
  }
  // stage the sums: stg[seg][key] (accumulator element i of tile (mt, nt) is
  // segment m0 + 8 mt + fr, key n0 + 8 nt + 2 fc + i)
  __syncthreads();
  double* stg = smd;
#pragma unroll
  for (int mt = 0; mt < 2; ++mt)
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
      double* dst = stg + (m0 + 8 * mt + fr) * kStageStride + n0 + 8 * nt + 2 * fc;
      dst[0] = c[mt][nt][0];
      dst[1] = c[mt][nt][1];
    }
  __syncthreads();
  const int tk = tid & 15;
  const int ts = tid >> 4;
  double acc[8][4];
#pragma unroll
  for (int aa = 0; aa < 8; ++aa)
#pragma unroll
    for (int q = 0; q < 4; ++q) acc[aa][q] = stg[(ts + 16 * q) * kStageStride + 2 * tk + 32 * (aa >> 1) + (aa & 1)];

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
