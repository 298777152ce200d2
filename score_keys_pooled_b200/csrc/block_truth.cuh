// Ranking accuracy: the pooled order checked against exact attention.
//
// The referee report on the pith.science page notes that the pages never
// measure how well the pooled, prefix-predicted order ranks blocks by their
// true attention mass.  For sampled segments this computes, from the exact
// causal softmax of every row over all of [0, i]:
//   col[j]    = mean over the segment's rows and the group's query heads of
//               the probability of candidate key j,
//   mass[b]   = sum of col over block b of the plan's order,
// and per segment (kept blocks C, blocks with mass >= tau, blocks in both,
// true mass of the kept blocks, true mass of all candidate blocks).
//
//   k_truth_cols   one CTA per (sampled segment, query head), one thread per
//                  row: pass 1 takes the row max and exp-sum over every
//                  admissible key, pass 2 the probabilities of the candidate
//                  keys; a warp butterfly sums each key over the warp's rows
//                  and one atomic per warp and key adds it to col
//   k_truth_stats  one CTA per (sampled segment, b, kvh): block masses along
//                  the order and the counts
// fp32 dot products and sums (a measurement, compared with the fp64 oracle
// at a relative tolerance).
#pragma once
#include "s2o_common.cuh"

namespace s2o {

constexpr int kTruthKeys = 32;         // keys per tile
constexpr int kTruthThreads = 128;     // one per row of a segment
constexpr int kTruthMaxSamples = 256;  // sampled segments per call
constexpr size_t kTruthSmem = sizeof(float) * (kD * kLq + kD * kTruthKeys);

struct TruthSegs {
  int32_t s[kTruthMaxSamples];
};

__device__ __forceinline__ void truth_load_k(const uint16_t* Kb, int j0, int e, float* kt) {
  // kt[d][key] for keys j0 .. j0+31 (keys >= e read as zero)
  for (int q = threadIdx.x; q < kTruthKeys * 16; q += kTruthThreads) {
    const int key = q & (kTruthKeys - 1), c = q >> 5;  // c: 16-byte chunk of the row
    const int j = j0 + key;
    uint4 w = make_uint4(0, 0, 0, 0);
    if (j < e) w = *reinterpret_cast<const uint4*>(Kb + (size_t)j * kD + 8 * c);
    float* dst = kt + (8 * c) * kTruthKeys + key;
    dst[0 * kTruthKeys] = __uint_as_float(w.x << 16); dst[1 * kTruthKeys] = __uint_as_float(w.x & 0xffff0000u);
    dst[2 * kTruthKeys] = __uint_as_float(w.y << 16); dst[3 * kTruthKeys] = __uint_as_float(w.y & 0xffff0000u);
    dst[4 * kTruthKeys] = __uint_as_float(w.z << 16); dst[5 * kTruthKeys] = __uint_as_float(w.z & 0xffff0000u);
    dst[6 * kTruthKeys] = __uint_as_float(w.w << 16); dst[7 * kTruthKeys] = __uint_as_float(w.w & 0xffff0000u);
  }
}

// the 32 scores of this thread's row against the tile
__device__ __forceinline__ void truth_dots(const float* qt, const float* kt, int r, float* acc) {
#pragma unroll
  for (int k = 0; k < kTruthKeys; ++k) acc[k] = 0.f;
#pragma unroll 4
  for (int dd = 0; dd < kD; ++dd) {
    const float qv = qt[dd * kLq + r];
    const float4* k4 = reinterpret_cast<const float4*>(kt + dd * kTruthKeys);
#pragma unroll
    for (int k = 0; k < kTruthKeys / 4; ++k) {
      const float4 kk = k4[k];
      acc[4 * k] = fmaf(qv, kk.x, acc[4 * k]);
      acc[4 * k + 1] = fmaf(qv, kk.y, acc[4 * k + 1]);
      acc[4 * k + 2] = fmaf(qv, kk.z, acc[4 * k + 2]);
      acc[4 * k + 3] = fmaf(qv, kk.w, acc[4 * k + 3]);
    }
  }
}

__global__ void __launch_bounds__(kTruthThreads) k_truth_cols(const uint16_t* __restrict__ Q,
                                                             const uint16_t* __restrict__ K, TruthSegs segs,
                                                             float* __restrict__ col, int Hq, int Hkv, int N,
                                                             int64_t cmaxlen) {
  const int BHkv = gridDim.y / Hq * Hkv;
  extern __shared__ float tsm[];
  float* qt = tsm;               // [128 d][128 rows]
  float* kt = tsm + kD * kLq;    // [128 d][32 keys]
  const int k = blockIdx.x;      // sampled segment
  const int bh = blockIdx.y;     // b * Hq + query head
  const int b = bh / Hq, hq = bh % Hq;
  const int G = Hq / Hkv, kvh = hq / G;
  const int bk = b * Hkv + kvh;
  const int s = segs.s[k];
  const int r0 = kLq * s;
  const int rows = min(kLq, N - r0);
  const int e = r0 + rows;
  const int r = threadIdx.x, lane = r & 31;
  const int row = r0 + r;
  const bool valid = r < rows;
  const uint16_t* Qb = Q + ((size_t)bh * N + r0) * kD;
  const uint16_t* Kb = K + (size_t)bk * N * kD;

  // the segment's rows, transposed to qt[d][row] (rows past N are zero)
  for (int q = threadIdx.x; q < kLq * 16; q += kTruthThreads) {
    const int rr = q & (kLq - 1), c = q >> 7;
    uint4 w = make_uint4(0, 0, 0, 0);
    if (rr < rows) w = *reinterpret_cast<const uint4*>(Qb + (size_t)rr * kD + 8 * c);
    float* dst = qt + (8 * c) * kLq + rr;
    dst[0 * kLq] = __uint_as_float(w.x << 16); dst[1 * kLq] = __uint_as_float(w.x & 0xffff0000u);
    dst[2 * kLq] = __uint_as_float(w.y << 16); dst[3 * kLq] = __uint_as_float(w.y & 0xffff0000u);
    dst[4 * kLq] = __uint_as_float(w.z << 16); dst[5 * kLq] = __uint_as_float(w.z & 0xffff0000u);
    dst[6 * kLq] = __uint_as_float(w.w << 16); dst[7 * kLq] = __uint_as_float(w.w & 0xffff0000u);
  }
  const float scale = 0.08838834764831845f;  // 1 / sqrt(128)
  float acc[kTruthKeys];

  // pass 1: row max and exp-sum over [0, row]
  float m = -INFINITY, l = 0.f;
  for (int j0 = 0; j0 < e; j0 += kTruthKeys) {
    __syncthreads();
    truth_load_k(Kb, j0, e, kt);
    __syncthreads();
    truth_dots(qt, kt, r, acc);
    float mt = -INFINITY;
#pragma unroll
    for (int q = 0; q < kTruthKeys; ++q)
      if (j0 + q <= row) mt = fmaxf(mt, acc[q] * scale);
    if (mt > m) {
      l = (m == -INFINITY) ? 0.f : l * expf(m - mt);
      m = mt;
    }
#pragma unroll
    for (int q = 0; q < kTruthKeys; ++q)
      if (j0 + q <= row) l += expf(acc[q] * scale - m);
  }

  // pass 2: candidate probabilities, summed over rows (and, by the atomics,
  // over the group's heads), divided by G * rows
  const int cand_hi = kLq * s - kWin;
  const float inv = valid && l > 0.f ? 1.f / (l * (float)(G * rows)) : 0.f;
  float* colk = col + ((size_t)k * BHkv + bk) * cmaxlen;
  for (int j0 = kSink; j0 < cand_hi; j0 += kTruthKeys) {
    __syncthreads();
    truth_load_k(Kb, j0, cand_hi, kt);
    __syncthreads();
    truth_dots(qt, kt, r, acc);
#pragma unroll
    for (int q = 0; q < kTruthKeys; ++q) acc[q] = (j0 + q < cand_hi) ? expf(acc[q] * scale - m) * inv : 0.f;
    // butterfly: after it lane l holds the warp's sum for key l
#pragma unroll
    for (int w = 16; w >= 1; w >>= 1) {
      const bool upper = (lane & w) != 0;
#pragma unroll
      for (int i = 0; i < w; ++i) {
        const float send = upper ? acc[i] : acc[i + w];
        const float keep = upper ? acc[i + w] : acc[i];
        acc[i] = keep + __shfl_xor_sync(0xffffffffu, send, w);
      }
    }
    if (j0 + lane < cand_hi) atomicAdd(colk + (j0 + lane - kSink), acc[0]);
  }
}

// per (sampled segment, b, kvh): block masses along the order and the counts
__global__ void __launch_bounds__(256) k_truth_stats(const int32_t* __restrict__ perm,
                                                    const int32_t* __restrict__ nblocks, TruthSegs segs,
                                                    const float* __restrict__ col, float* __restrict__ stats,
                                                    float* __restrict__ mass, int BHkv, int S, int64_t T,
                                                    int64_t cmaxlen, int nbmax, float tau) {
  __shared__ int n_true, n_both;
  __shared__ float captured, total;
  const int k = blockIdx.x, bk = blockIdx.y;
  const int s = segs.s[k];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) { n_true = 0; n_both = 0; captured = 0.f; total = 0.f; }
  __syncthreads();
  const int nb = (int)(num_cand(s) / kBk);
  int C = nblocks[(size_t)bk * S + s];
  C = C < 0 ? 0 : (C > nb ? nb : C);
  const int32_t* pseg = perm + (size_t)bk * T + cand_offset(s);
  const float* colk = col + ((size_t)k * BHkv + bk) * cmaxlen;
  const int cand_hi = kLq * s - kWin;
  for (int blk = warp; blk < nb; blk += 8) {
    float v = 0.f;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      int j = pseg[kBk * blk + 32 * h + lane];
      if (j < kSink || j >= cand_hi) {  // caller-supplied order out of Cand(s)
        set_error(kErrBadPlan);
        j = kSink;
      }
      v += colk[j - kSink];
    }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if (lane == 0) {
      if (mass) mass[((size_t)k * BHkv + bk) * nbmax + blk] = v;
      const bool t = v >= tau;
      if (t) atomicAdd(&n_true, 1);
      if (t && blk < C) atomicAdd(&n_both, 1);
      if (blk < C) atomicAdd(&captured, v);
      atomicAdd(&total, v);
    }
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    float* st = stats + ((size_t)k * BHkv + bk) * 5;
    st[0] = (float)C;
    st[1] = (float)n_true;
    st[2] = (float)n_both;
    st[3] = captured;
    st[4] = total;
  }
}

}  // namespace s2o
