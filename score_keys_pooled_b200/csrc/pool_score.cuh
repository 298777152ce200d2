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
// are reused across 256 multiply-adds per instruction.  The key tile (bf16,
// rows padded to 272 bytes) and the chunk's pooled queries (fp64, rows
// padded to 132 doubles) arrive by cp.async; both fragment patterns are then
// free of bank conflicts, and a key is widened to fp64 (exactly) as its
// fragment is loaded.  The epilogue works on the accumulators in registers:
// lane (fr, fc) of a warp holds segments m0 + 8 mt + fr and keys
// n0 + 8 nt + 2 fc + {0, 1}; scores go out as pairs, and the per-(segment,
// tile) (max, sum exp) is reduced over the lanes and the two warps that
// share a segment.
// Outputs:
//   scores[bk][off(s) + j - 64] for candidate keys j of segment s
//   part[bk][s][t] = (max over the tile's admissible keys,
//                     sum exp(s_j - that max))
// ---------------------------------------------------------------------------
constexpr int kScoreKeys = 128;
constexpr int kScoreSegs = 64;
constexpr int kScoreKRow = 272;            // bytes per key row of the tile (256 + 16 padding)
constexpr int kScoreQRow = 132;            // doubles per pooled-query row (128 + 4 padding)
constexpr size_t kScoreKBytes = (size_t)kScoreKeys * kScoreKRow;
constexpr size_t kScoreSmem = kScoreKBytes + sizeof(double) * kScoreSegs * kScoreQRow;

__device__ __forceinline__ void dmma_8x8x4(double& c0, double& c1, double a, double b) {
  asm volatile("mma.sync.aligned.m8n8k4.row.col.f64.f64.f64.f64 {%0, %1}, {%2}, {%3}, {%0, %1};\n"
               : "+d"(c0), "+d"(c1)
               : "d"(a), "d"(b));
}

// (max, sum exp(v - max)) of two partial pairs
__device__ __forceinline__ void merge_max_sum(float& m, float& z, float m2, float z2) {
  const float mm = fmaxf(m, m2);
  if (mm == -INFINITY) return;
  z = (m == -INFINITY ? 0.f : z * exp_shifted(m, mm)) + (m2 == -INFINITY ? 0.f : z2 * exp_shifted(m2, mm));
  m = mm;
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

  extern __shared__ __align__(16) uint8_t sms[];
  uint8_t* Ks = sms;                                            // [128 keys][272 B]
  double* Qs = reinterpret_cast<double*>(sms + kScoreKBytes);   // [64 segs][132]
  __shared__ float2 xw[2][kScoreSegs];                          // per-warp-half partials
  const int tid = threadIdx.x;
  const int lane = tid & 31, warp = tid >> 5;
  const uint16_t* Kb = K + (size_t)bk * N * kD;
  const double* qb = qbar + (size_t)bk * S * kD;

  // the tile's keys (rows past N are zero: never admissible) and the chunk's
  // pooled queries (segments past S are zero: never stored)
  const uint32_t ks = smem_u32(Ks), qs = smem_u32(Qs);
#pragma unroll
  for (int q = 0; q < (kScoreKeys * 16) / 256; ++q) {
    const int c = tid + 256 * q;               // 16-byte chunk c & 15 of key row c >> 4
    const int key = c >> 4, j = t * kScoreKeys + key;
    cp_async16(ks + key * kScoreKRow + (c & 15) * 16, Kb + (size_t)(j < N ? j : 0) * kD + (c & 15) * 8,
               j < N ? 16u : 0u);
  }
#pragma unroll
  for (int q = 0; q < (kScoreSegs * 64) / 256; ++q) {
    const int c = tid + 256 * q;               // 16-byte chunk c & 63 of segment row c >> 6
    const int seg = c >> 6, sg = s_lo + seg;
    cp_async16(qs + seg * (kScoreQRow * 8) + (c & 63) * 16, qb + (size_t)(sg < S ? sg : 0) * kD + (c & 63) * 2,
               sg < S ? 16u : 0u);
  }
  cp_async_wait_all();
  __syncthreads();

  // this warp's block: segments m0 .. m0+15, keys n0 .. n0+63
  const int m0 = 16 * (warp & 3), n0 = 64 * (warp >> 2);
  const int fr = lane >> 2, fc = lane & 3;  // fragment row / column of this lane
  double c[2][8][2];
#pragma unroll
  for (int mt = 0; mt < 2; ++mt)
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) c[mt][nt][0] = c[mt][nt][1] = 0.0;
  const double* qa = Qs + (m0 + fr) * kScoreQRow + fc;
  const uint16_t* kbf = reinterpret_cast<const uint16_t*>(Ks + (n0 + fr) * kScoreKRow) + fc;
#pragma unroll 2
  for (int k0 = 0; k0 < kD; k0 += 4) {
    double a[2], bb[8];
#pragma unroll
    for (int mt = 0; mt < 2; ++mt) a[mt] = qa[8 * mt * kScoreQRow + k0];
#pragma unroll
    for (int nt = 0; nt < 8; ++nt)
      bb[nt] = (double)__uint_as_float((uint32_t)kbf[8 * nt * (kScoreKRow / 2) + k0] << 16);
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) dmma_8x8x4(c[mt][nt][0], c[mt][nt][1], a[mt], bb[nt]);
  }

  // epilogue from the accumulators
  float* sc_bk = scores + (size_t)bk * T;
  float2* part_bk = part + (size_t)bk * S * S;
  const double inv_sqrt_d = 0.08838834764831845;  // 1/sqrt(128), rounded to fp64
#pragma unroll
  for (int mt = 0; mt < 2; ++mt) {
    const int seg = m0 + 8 * mt + fr;
    const int s = s_lo + seg;
    const bool seg_ok = (s < s_hi) && (s >= t);
    const int cand_hi = s * kLq - kWin;  // candidates are [64, cand_hi)
    float v[16];
    float mloc = -INFINITY;
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
      const int j = t * kScoreKeys + n0 + 8 * nt + 2 * fc;  // even; j + 1 shares j's class
      const float v0 = (float)(c[mt][nt][0] * inv_sqrt_d), v1 = (float)(c[mt][nt][1] * inv_sqrt_d);
      const bool adm0 = seg_ok && j < N, adm1 = seg_ok && j + 1 < N;
      v[2 * nt] = adm0 ? v0 : -INFINITY;
      v[2 * nt + 1] = adm1 ? v1 : -INFINITY;
      if ((adm0 && !isfinite(v0)) || (adm1 && !isfinite(v1))) set_error(kErrNonFinite);
      mloc = fmax3(mloc, v[2 * nt], v[2 * nt + 1]);
      if (seg_ok && j >= kSink && j < cand_hi) {
        float* dst = sc_bk + cand_offset(s) + (j - kSink);
        if (adm1) *reinterpret_cast<float2*>(dst) = make_float2(v0, v1);
        else if (adm0) dst[0] = v0;
      }
    }
    // the four lanes of this fragment row hold the rest of the warp's 64 keys
    mloc = fmaxf(mloc, __shfl_xor_sync(0xffffffffu, mloc, 1));
    mloc = fmaxf(mloc, __shfl_xor_sync(0xffffffffu, mloc, 2));
    float z = 0.f;
    if (mloc > -INFINITY) {
#pragma unroll
      for (int k = 0; k < 16; ++k) z += (v[k] > -INFINITY) ? exp_shifted(v[k], mloc) : 0.f;
    }
    z += __shfl_xor_sync(0xffffffffu, z, 1);
    z += __shfl_xor_sync(0xffffffffu, z, 2);
    if (fc == 0) xw[warp >> 2][seg] = make_float2(mloc, z);
  }
  __syncthreads();
  // the two warps of a segment (keys 0-63 and 64-127 of the tile) merge
  if (tid < kScoreSegs) {
    const int s = s_lo + tid;
    if (s < s_hi && s >= t) {
      float m = xw[0][tid].x, z = xw[0][tid].y;
      merge_max_sum(m, z, xw[1][tid].x, xw[1][tid].y);
      part_bk[(size_t)s * S + t] = make_float2(m, z);
    }
  }
}

}  // namespace s2o
