// Kernel (2): per-segment (M, Z), importance sort, block masses and stop.
//
// S2O ranks each segment's historical keys by importance into an index list
// (the online permutation; gist.science technical summary, section 1) and
// walks the list in blocks from high to low importance, stopping once a
// block's attention mass falls below tau (section 2, "Regle d'Arret
// Anticipe"; pith.science abstract).  The pages report the ranking as the
// dominant cost of the preprocessing ("Resultats Experimentaux").
//
// Here, per segment s:
//   M = max_{A(s)} s_j, Z = sum_{A(s)} exp(s_j - M)       (k_seg_stats)
//   perm = candidates by s_j descending, ties to the lower index: a stable
//          LSD radix sort (4 x 8-bit digits) of an order-reversing 32-bit
//          key over index-ascending input, in global memory (k_sort, the
//          fallback of the bucketed sorter in seg_sort2.cuh)
#pragma once
#include "s2o_common.cuh"

namespace s2o {

// score -> 32-bit key whose ascending order is descending score; -0 == +0
__device__ __forceinline__ uint32_t desc_key(float f) {
  uint32_t u = __float_as_uint(f == 0.f ? 0.f : f);
  uint32_t asc = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
  return ~asc;
}
__device__ __forceinline__ float key_score(uint32_t k) {
  uint32_t asc = ~k;
  uint32_t u = (asc & 0x80000000u) ? (asc & 0x7FFFFFFFu) : ~asc;
  return __uint_as_float(u);
}

// ---------------------------------------------------------------------------
// (M, Z) per segment from the per-tile partials (max, sum exp) of the scorer:
// tiles of kTile keys, row stride `ntiles`, the first ceil(e(s) / kTile)
// entries of a row filled; one warp per segment.
// ---------------------------------------------------------------------------
template <int kTile>
__global__ void k_seg_stats(const float2* __restrict__ part, float* __restrict__ segM, double* __restrict__ segZ,
                            float* __restrict__ seg_stats, int BHkv, int S, int N, int ntiles) {
  const int warp = (int)(((unsigned long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5);
  const int lane = threadIdx.x & 31;
  if (warp >= BHkv * S) return;
  const int bk = warp / S, s = warp % S;
  const float2* p = part + ((size_t)bk * S + s) * ntiles;
  const int nt = (min(N, kLq * (s + 1)) + kTile - 1) / kTile;
  float m = -INFINITY;
  for (int t = lane; t < nt; t += 32) m = fmaxf(m, p[t].x);
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  double z = 0.0;
  for (int t = lane; t < nt; t += 32) z += (double)p[t].y * exp((double)p[t].x - (double)m);
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
  if (lane == 0) {
    segM[warp] = m;
    segZ[warp] = z;
    if (seg_stats) {
      seg_stats[2 * (size_t)warp] = m;
      seg_stats[2 * (size_t)warp + 1] = (float)z;
    }
  }
}

// ---------------------------------------------------------------------------
// Global-memory sort: one 1024-thread CTA per (b, kvh, s), largest first.
// Used for the segments the bucketed sorter hands over (mode[seg] == only):
// writes perm and the sorted scores; the stop is taken by k_mass_stop.
// ---------------------------------------------------------------------------
constexpr int kSortThreads = 1024;
constexpr int kSortWarps = kSortThreads / 32;

struct SortSmem {
  uint32_t cnt[kSortWarps][256];  // per-warp digit counts, then offsets
  uint32_t base[256];             // running bucket starts
  uint32_t total[256];
  int trivial;
};

__global__ void __launch_bounds__(kSortThreads, 2)
    k_sort(const float* __restrict__ scores, const float* __restrict__ segM, const double* __restrict__ segZ,
           uint32_t* __restrict__ keyA, uint32_t* __restrict__ keyB, uint32_t* __restrict__ valA,
           uint32_t* __restrict__ valB, int32_t* __restrict__ perm, float* __restrict__ sorted,
           const int* __restrict__ mode, int only, int BHkv, int S, int64_t T) {
  __shared__ SortSmem sm;
  const int q = blockIdx.x;
  const int s = S - 1 - q / BHkv;
  const int bk = q % BHkv;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int n = (int)num_cand(s);
  if (n == 0 || mode[(size_t)bk * S + s] != only) return;
  const size_t base = (size_t)bk * T + cand_offset(s);
  const float* sc = scores + base;
  uint32_t* kb[2] = {keyA + base, keyB + base};
  uint32_t* vb[2] = {valA + base, valB + base};
  int cur = -1;  // -1: keys implicit from scores, values = positions
  const uint32_t lt_mask = (1u << lane) - 1u;

  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 8 * pass;
    for (int k = tid; k < kSortWarps * 256; k += kSortThreads) (&sm.cnt[0][0])[k] = 0;
    __syncthreads();
    for (int i = tid; i < n; i += kSortThreads) {
      const uint32_t key = cur < 0 ? desc_key(sc[i]) : kb[cur][i];
      atomicAdd(&sm.cnt[warp][(key >> shift) & 255u], 1u);
    }
    __syncthreads();
    if (tid < 256) {
      uint32_t t = 0;
      for (int w = 0; w < kSortWarps; ++w) t += sm.cnt[w][tid];
      sm.total[tid] = t;
    }
    __syncthreads();
    if (warp == 0) {
      // exclusive scan of 256 totals: 8 per lane
      uint32_t v[8], run = 0;
#pragma unroll
      for (int k = 0; k < 8; ++k) { v[k] = run; run += sm.total[lane * 8 + k]; }
      uint32_t incl = run;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      const uint32_t excl = incl - run;
#pragma unroll
      for (int k = 0; k < 8; ++k) sm.base[lane * 8 + k] = excl + v[k];
      if (lane == 0) {
        const uint32_t key0 = cur < 0 ? desc_key(sc[0]) : kb[cur][0];
        sm.trivial = (sm.total[(key0 >> shift) & 255u] == (uint32_t)n);
      }
    }
    __syncthreads();
    if (sm.trivial) continue;  // every key has the same digit: order unchanged
    const int out = (cur == 0) ? 1 : 0;
    for (int t0 = 0; t0 < n; t0 += kSortThreads) {
      const int i = t0 + tid;
      const bool valid = i < n;
      uint32_t key = 0, val = 0;
      if (valid) {
        key = cur < 0 ? desc_key(sc[i]) : kb[cur][i];
        val = cur < 0 ? (uint32_t)i : vb[cur][i];
      }
      const uint32_t dg = (key >> shift) & 255u;
#pragma unroll
      for (int k = 0; k < 8; ++k) sm.cnt[warp][lane * 8 + k] = 0;
      __syncwarp();
      const uint32_t peers = __match_any_sync(0xffffffffu, valid ? dg : 0xFFFFFFFFu);
      const uint32_t rank = __popc(peers & lt_mask);
      if (valid && (__ffs(peers) - 1) == lane) sm.cnt[warp][dg] = __popc(peers);
      __syncthreads();
      if (tid < 256) {
        uint32_t run = sm.base[tid];
        for (int w = 0; w < kSortWarps; ++w) {
          const uint32_t c = sm.cnt[w][tid];
          sm.cnt[w][tid] = run;
          run += c;
        }
        sm.base[tid] = run;
      }
      __syncthreads();
      if (valid) {
        const uint32_t pos = sm.cnt[warp][dg] + rank;
        kb[out][pos] = key;
        vb[out][pos] = val;
      }
      __syncthreads();
    }
    cur = out;
  }

  // importance order as absolute key indices, and the scores in that order
  for (int i = tid; i < n; i += kSortThreads) {
    perm[base + i] = kSink + (int32_t)(cur < 0 ? (uint32_t)i : vb[cur][i]);
    sorted[base + i] = cur < 0 ? sc[i] : key_score(kb[cur][i]);
  }
}

// ---------------------------------------------------------------------------
// Contiguous top-k comparator: rank original-order candidate blocks by pooled
// mass (ties to the lower block), emit them as an index list.
// One 1024-thread CTA per (b, kvh, s).
// ---------------------------------------------------------------------------
constexpr int kContigMaxBlocks = 8192;  // N <= 524416

__global__ void __launch_bounds__(1024) k_contig_plan(const float* __restrict__ scores,
                                                     const float* __restrict__ seg_stats,
                                                     int32_t* __restrict__ perm_out, int BHkv, int S, int64_t T) {
  extern __shared__ unsigned long long arr[];  // [pow2 >= nb]
  const int q = blockIdx.x;
  const int s = S - 1 - q / BHkv;
  const int bk = q % BHkv;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int n = (int)num_cand(s);
  const int nb = n / kBk;
  if (nb == 0) return;
  int P = 1;
  while (P < nb) P <<= 1;
  const size_t base = (size_t)bk * T + cand_offset(s);
  const float* sc = scores + base;
  const float M = seg_stats[2 * ((size_t)bk * S + s)];
  const double Z = (double)seg_stats[2 * ((size_t)bk * S + s) + 1];
  for (int blk = warp; blk < P; blk += 32) {
    float e = 0.f;
    if (blk < nb) e = exp_shifted(sc[blk * kBk + lane], M) + exp_shifted(sc[blk * kBk + 32 + lane], M);
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) e += __shfl_xor_sync(0xffffffffu, e, o);
    if (lane == 0) {
      const float mass = (float)((double)e / Z);
      // ascending composite: larger mass first, then the lower block index
      arr[blk] = (blk < nb) ? (((unsigned long long)(~__float_as_uint(mass)) << 32) | (unsigned)blk)
                            : ~0ull;
    }
  }
  __syncthreads();
  // bitonic sort of P entries, ascending
  for (int k = 2; k <= P; k <<= 1) {
    for (int j = k >> 1; j > 0; j >>= 1) {
      for (int i = tid; i < P; i += 1024) {
        const int l = i ^ j;
        if (l > i) {
          const unsigned long long a = arr[i], b = arr[l];
          const bool up = ((i & k) == 0);
          if ((a > b) == up) { arr[i] = b; arr[l] = a; }
        }
      }
      __syncthreads();
    }
  }
  for (int i = tid; i < n; i += 1024) {
    const int r = i / kBk, k = i % kBk;
    const int c = (int)(arr[r] & 0xFFFFFFFFu);
    perm_out[base + i] = kSink + c * kBk + k;
  }
}

}  // namespace s2o
