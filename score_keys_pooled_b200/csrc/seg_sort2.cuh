// Kernel (2), bucketed form: the importance order of each segment's
// candidates (gist.science technical summary, section 1: KV_perm; the ranking
// step that dominates the preprocessing, "Resultats Experimentaux"), sorted
// mostly on chip.
//
//   k_bucket_plan  one CTA per segment: the min and max candidate score, a
//                  2048-bin histogram that is linear in the score between them
//                  (bins are monotone in the score, so bin b holds only scores
//                  >= those of bin b+1, and equal scores share a bin), and
//                  buckets = runs of consecutive bins whose starting rank falls
//                  in the same window of kBucketHalf ranks (a bucket holds at
//                  most kBucketHalf + one bin <= kBucketCap elements); then a
//                  multisplit of the segment into its buckets: (key, index)
//                  pairs land at the bucket's rank range, in no set order
//                  (each warp reserves room with shared atomics, no block
//                  barrier);
//   k_bucket_sort  one CTA per group of kSortGroup consecutive bucket slots
//                  (the empty ones, buckets a segment did not need, are
//                  skipped); per bucket: loads its range into shared memory and
//                  sorts it there: a counting sort into 4096 fine bins linear
//                  in the score, then each fine bin (a few elements) by
//                  (key, index); a bucket with a crowded fine bin, or with a
//                  single key, is sorted by a stable LSD radix sort over the
//                  bucket-relative index and then key instead; writes perm and
//                  the sorted scores at the bucket's global rank;
//   k_mass_stop    block masses of the sorted scores and the stop point C(s).
// Filtered form (the planner's `filtered` flag): a candidate of pooled mass
// exp(s - M)/Z below tau/Bk cannot lift a block to tau, so a block made only
// of such candidates fails the stop test.  With n_hi candidates at or above
// that level (counted with a small safety margin), the first block starting
// at or after n_hi fails, hence C(s) <= ceil(n_hi/Bk), and only the first
// L = Bk ceil(n_hi/Bk) entries of the order are needed.  The planner then
// buckets and moves only the score bins that start below rank L; the rest of
// the segment is never sorted.  perm[0, Bk C) and C are those of the full
// sort (the pith.science abstract calls the preprocessing very light; this
// keeps its cost proportional to what the stop rule can keep).
// A segment whose scores are all equal is already in index order.  A segment
// with a bin larger than kBucketCap - kBucketHalf (a heavy cluster of nearly
// equal scores) is sorted by the global-memory LSD kernel k_sort instead.
#pragma once
#include "s2o_common.cuh"
#include "seg_sort.cuh"

namespace s2o {

constexpr int kNumBins = 2048;
constexpr int kBucketCap = 5632;              // elements a bucket CTA sorts in shared memory
constexpr int kBucketHalf = kBucketCap / 2;   // rank window of a bucket
constexpr int kBucketThreads = 1024;          // planner CTA
constexpr int kSorterThreads = 512;           // bucket-sorter CTA (three per SM)
constexpr int kSorterWarps = kSorterThreads / 32;
constexpr int kMaxBuckets = 256;              // bucket ids per segment (N <= 2^19)

enum SegMode : int { kModeDone = 0, kModeBuckets = 1, kModeFallback = 2 };

struct BucketSlot {
  int bk, s, bin_lo, bin_hi, base, count;
};

// slots reserved for a segment of n candidates
__host__ __device__ __forceinline__ int bucket_slots(int64_t n) {
  return n == 0 ? 0 : (int)(n / kBucketHalf) + 2;
}

__device__ __forceinline__ int score_bin(float x, float hi, float scale) {
  const int b = (int)((hi - x) * scale);
  return min(max(b, 0), kNumBins - 1);
}

// block-wide exclusive scan of one value per thread (NWARPS full warps)
template <int NWARPS = 32>
__device__ __forceinline__ int block_excl_scan(int v, int* warp_tot, int& total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) warp_tot[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int w = lane < NWARPS ? warp_tot[lane] : 0;
    int wi = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, wi, o);
      if (lane >= o) wi += y;
    }
    if (lane < NWARPS) warp_tot[lane] = wi - w;  // exclusive prefix of the warp totals
    if (lane == 31) warp_tot[32] = wi;
  }
  __syncthreads();
  const int r = warp_tot[warp] + incl - v;
  total = warp_tot[32];
  __syncthreads();
  return r;
}

// ---------------------------------------------------------------------------
// planner: one 1024-thread CTA per (b, kvh, s), largest segments first
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kBucketThreads, 2) k_bucket_plan(const float* __restrict__ scores,
                                                              float* __restrict__ sorted, int32_t* __restrict__ perm,
                                                              BucketSlot* __restrict__ slots, int* __restrict__ mode,
                                                              float2* __restrict__ range,
                                                              uint32_t* __restrict__ stage_key,
                                                              uint32_t* __restrict__ stage_val,
                                                              const float* __restrict__ segM,
                                                              const double* __restrict__ segZ,
                                                              int* __restrict__ plen, double tau, int filtered,
                                                              int BHkv, int S, int64_t T) {
  __shared__ int hist[kNumBins];
  __shared__ int wtot[33];
  __shared__ float red[64];
  __shared__ int flag;
  __shared__ uint8_t bin2bkt[kNumBins];  // bucket id of each bin (< kMaxBuckets = 256)
  __shared__ int cursor[kMaxBuckets];
  __shared__ int bin_cut;  // first bin left out of the order (filtered form)
  const int q = blockIdx.x;
  const int s = S - 1 - q / BHkv;
  const int bk = q % BHkv;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int n = (int)num_cand(s);
  const size_t base = (size_t)bk * T + cand_offset(s);
  const float* sc = scores + base;

  // slot range of this segment: segments with larger s come first, heads interleaved
  int before = 0;
  for (int t = s + 1 + tid; t < S; t += kBucketThreads) before += bucket_slots(num_cand(t));
  int tot_before;
  block_excl_scan(before, wtot, tot_before);
  const int my_slots = bucket_slots(n);
  BucketSlot* myslot = slots + (size_t)tot_before * BHkv + (size_t)bk * my_slots;
  for (int k = tid; k < my_slots; k += kBucketThreads) myslot[k].count = 0;
  if (tid == 0) plen[(size_t)bk * S + s] = n;
  if (n == 0) {
    if (tid == 0) mode[(size_t)bk * S + s] = kModeDone;
    return;
  }

  // min and max candidate score; the number of candidates whose pooled mass
  // may reach tau/Bk: s >= M + ln(tau Z / Bk), less a margin of 1e-3 that
  // covers the rounding of the masses computed in k_mass_stop
  double cut = -INFINITY;
  if (filtered && tau > 0.0)
    cut = (double)segM[(size_t)bk * S + s] + log(tau * segZ[(size_t)bk * S + s] / (double)kBk) - 1e-3;
  // candidate ranges start 256-byte aligned and hold a multiple of 64
  // scores (n = 128 s - 192): every pass reads them as float4
  const float4* sc4 = reinterpret_cast<const float4*>(sc);
  const int n4 = n / 4;
  float lo = INFINITY, hi = -INFINITY;
  int nhi = 0;
  for (int i = tid; i < n4; i += kBucketThreads) {
    const float4 x = sc4[i];
    lo = fminf(lo, fminf(fminf(x.x, x.y), fminf(x.z, x.w)));
    hi = fmaxf(hi, fmaxf(fmaxf(x.x, x.y), fmaxf(x.z, x.w)));
    nhi += ((double)x.x >= cut) + ((double)x.y >= cut) + ((double)x.z >= cut) + ((double)x.w >= cut);
  }
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) {
    lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, o));
    hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, o));
  }
  if (lane == 0) { red[warp] = lo; red[32 + warp] = hi; }
  for (int k = tid; k < kNumBins; k += kBucketThreads) hist[k] = 0;
  int nhi_tot;
  block_excl_scan(nhi, wtot, nhi_tot);  // (synchronises the block)
  // entries of the order the stop rule can reach: whole blocks up to n_hi
  const int L = (int)min((int64_t)n, (int64_t)kBk * (((int64_t)nhi_tot + kBk - 1) / kBk));
  __syncthreads();
  if (warp == 0) {
    lo = red[lane];
    hi = red[32 + lane];
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) {
      lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, o));
      hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, o));
    }
    if (lane == 0) { red[0] = lo; red[32] = hi; }
  }
  __syncthreads();
  lo = red[0];
  hi = red[32];
  if (tid == 0) range[(size_t)bk * S + s] = make_float2(lo, hi);
  if (!(hi > lo)) {
    // one value (or non-finite, already flagged by the score kernel): the
    // importance order is the index order
    for (int i = tid; i < n; i += kBucketThreads) {
      sorted[base + i] = sc[i];
      perm[base + i] = kSink + i;
    }
    if (tid == 0) mode[(size_t)bk * S + s] = kModeDone;
    return;
  }
  const float scale = (float)kNumBins / (hi - lo);
  for (int i = tid; i < n4; i += kBucketThreads) {
    const float4 x = sc4[i];
    atomicAdd(&hist[score_bin(x.x, hi, scale)], 1);
    atomicAdd(&hist[score_bin(x.y, hi, scale)], 1);
    atomicAdd(&hist[score_bin(x.z, hi, scale)], 1);
    atomicAdd(&hist[score_bin(x.w, hi, scale)], 1);
  }
  __syncthreads();
  // exclusive scan over the bins: 2 per thread
  const int c0 = hist[2 * tid], c1 = hist[2 * tid + 1];
  int total;
  const int st0 = block_excl_scan(c0 + c1, wtot, total);
  const int st1 = st0 + c0;
  if (tid == 0) flag = 0;
  __syncthreads();
  if (c0 > kBucketCap - kBucketHalf || c1 > kBucketCap - kBucketHalf) atomicOr(&flag, 1);
  __syncthreads();
  if (flag) {
    if (tid == 0) mode[(size_t)bk * S + s] = kModeFallback;
    return;
  }
  // bins that start at rank >= L are left out (none when L = n); start ranks
  // grow with the bin, so they form a suffix
  if (tid == 0) bin_cut = kNumBins;
  __syncthreads();
  if (st0 >= L && (tid == 0 || st0 - hist[2 * tid - 1] < L)) atomicMin(&bin_cut, 2 * tid);
  else if (st1 >= L && st0 < L) atomicMin(&bin_cut, 2 * tid + 1);
  __syncthreads();
  const int bcut = bin_cut;
  if (tid == 0) plen[(size_t)bk * S + s] = L;
  // a bucket = the bins below bin_cut whose start rank lies in
  // [k*H, (k+1)*H); the thread of its first bin records the first bin and
  // base rank, the thread of its last bin the end bin, then (after a
  // barrier) the size
  hist[2 * tid] = st0;
  hist[2 * tid + 1] = st1;
  __syncthreads();
  // both bins of a thread may end a bucket (a bin that is a bucket by itself,
  // or the last bin before bin_cut), so each keeps its own record
  int end_id[2] = {-1, -1}, end_rank[2] = {0, 0};
#pragma unroll
  for (int e = 0; e < 2; ++e) {
    const int b = 2 * tid + e;
    if (b >= bcut) break;
    const int stb = e ? st1 : st0;
    const int id = stb / kBucketHalf;
    const bool first = (b == 0) || (hist[b - 1] / kBucketHalf != id);
    const bool last = (b == kNumBins - 1) || (b + 1 == bcut) || (hist[b + 1] / kBucketHalf != id);
    if (first) {
      myslot[id].bk = bk;
      myslot[id].s = s;
      myslot[id].bin_lo = b;
      myslot[id].base = stb;
    }
    if (last) {
      myslot[id].bin_hi = b + 1;
      end_id[e] = id;
      end_rank[e] = stb + (e ? c1 : c0);
    }
  }
  __syncthreads();
#pragma unroll
  for (int e = 0; e < 2; ++e)
    if (end_id[e] >= 0) myslot[end_id[e]].count = end_rank[e] - myslot[end_id[e]].base;
  // multisplit into the buckets: each warp reserves room for its elements
  // with one shared atomic per bucket id it holds, with no block barrier;
  // the order inside a bucket is whatever the atomics give (the bucket
  // sorter orders every bucket by (key, index))
  bin2bkt[2 * tid] = (uint8_t)(st0 / kBucketHalf);
  bin2bkt[2 * tid + 1] = (uint8_t)(st1 / kBucketHalf);
  __syncthreads();
  // cursor[k] = base rank of bucket k = start rank of its first bin
#pragma unroll
  for (int e = 0; e < 2; ++e) {
    const int b = 2 * tid + e;
    const int id = bin2bkt[b];
    if (b < bcut && (b == 0 || bin2bkt[b - 1] != id)) cursor[id] = e ? st1 : st0;
  }
  __syncthreads();
  const uint32_t lt_mask = (1u << lane) - 1u;
  uint32_t* skey = stage_key + base;
  uint32_t* sval = stage_val + base;
  if (bcut == 0) {
    if (tid == 0) mode[(size_t)bk * S + s] = kModeBuckets;
    return;
  }
  for (int t0 = 0; t0 < n4; t0 += kBucketThreads) {
    const int i4 = t0 + tid;
    const float4 x4 = i4 < n4 ? sc4[i4] : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int i = 4 * i4 + k;
      const float x = k == 0 ? x4.x : k == 1 ? x4.y : k == 2 ? x4.z : x4.w;
      const int bin = score_bin(x, hi, scale);
      const bool valid = i4 < n4 && bin < bcut;
      if (!__any_sync(0xffffffffu, valid)) continue;
      // lanes holding the same bucket id (the lanes left out share one value:
      // a match costs more the more distinct values a warp holds)
      const uint32_t dg = valid ? (uint32_t)bin2bkt[bin] : 0xFFFFFFFFu;
      const uint32_t peers = __match_any_sync(0xffffffffu, dg);
      const int leader = __ffs(peers) - 1;
      uint32_t at = 0;
      if (valid && lane == leader) at = (uint32_t)atomicAdd(&cursor[dg], __popc(peers));
      at = __shfl_sync(0xffffffffu, at, leader);
      if (valid) {
        const uint32_t pos = at + __popc(peers & lt_mask);
        skey[pos] = desc_key(x);
        sval[pos] = (uint32_t)i;
      }
    }
  }
  if (tid == 0) mode[(size_t)bk * S + s] = kModeBuckets;
}

// ---------------------------------------------------------------------------
// bucket sorter: one 512-thread CTA per group of slots, three CTAs per SM.
// A bucket's pairs live in registers while they are counted and scattered
// (pair k of thread tid is element tid + 512 k of the bucket's range, the
// order the radix passes keep stable); shared memory holds one key/value
// array, the scatter target.
// ---------------------------------------------------------------------------
constexpr int kFine = 4096;     // fine bins of a bucket (= kSorterWarps * 256 counters)
constexpr int kFineMax = 64;    // larger fine bins send the bucket to the radix path
constexpr int kSortPer = kBucketCap / kSorterThreads;  // pairs per thread
static_assert(kSortPer * kSorterThreads == kBucketCap, "a bucket fills the sorter's registers exactly");
static_assert(kFine == kSorterWarps * 256, "fine counters reuse the radix count rows");


struct BucketSmem {
  uint32_t key[kBucketCap];
  uint32_t val[kBucketCap];
  uint32_t cnt[kSorterWarps][256];  // radix digit counts, or the kFine fine-bin counters
  uint32_t dbase[256];
  int wtot[33];
  uint32_t kmin, kmax, vmin, vmax;
  int big;
};
constexpr size_t kBucketSmem = sizeof(BucketSmem);

// one bucket: sorted by (key, index) and written back at its global ranks
__device__ __forceinline__ void sort_bucket(const BucketSlot& slot, BucketSmem& sm,
                                            const uint32_t* __restrict__ stage_key,
                                            const uint32_t* __restrict__ stage_val, const float2* __restrict__ range,
                                            float* __restrict__ sorted, int32_t* __restrict__ perm, int S, int64_t T) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const size_t base = (size_t)slot.bk * T + cand_offset(slot.s) + slot.base;
  const int m = slot.count;

  // the bucket's pairs at its rank range, in no particular order
  uint32_t rk[kSortPer], rv[kSortPer];
#pragma unroll
  for (int k = 0; k < kSortPer; ++k) {
    const int i = tid + kSorterThreads * k;
    rk[k] = 0u;
    rv[k] = 0u;
    if (i < m) {
      rk[k] = stage_key[base + i];
      rv[k] = stage_val[base + i];
    }
  }
  const uint32_t lt_mask = (1u << lane) - 1u;

  // Fine counting sort: kFine bins linear in the score over the bucket's
  // share of the segment's bins (the planner's binning, so no pass over the
  // bucket is needed to find its extremes; monotone, ties share a bin), a
  // scatter in any order, then each bin sorted by (key, index) -- a total
  // order, so the result is unique.
  {
    const float2 rg = range[(size_t)slot.bk * S + slot.s];
    const float hi = rg.y, scale = (float)kNumBins / (rg.y - rg.x);  // the planner's bins
    const float b0 = (float)slot.bin_lo;
    const float ffac = (float)kFine / (float)(slot.bin_hi - slot.bin_lo);
    auto fbin = [&](uint32_t key) {
      const float u = ((hi - key_score(key)) * scale - b0) * ffac;
      return min(max((int)u, 0), kFine - 1);
    };
    uint32_t* fcnt = &sm.cnt[0][0];  // kFine counters, then cursors
    constexpr int kPerT = kFine / kSorterThreads;  // counters per thread
    for (int k = tid; k < kFine; k += kSorterThreads) fcnt[k] = 0;
    if (tid == 0) sm.big = 0;
    __syncthreads();
#pragma unroll
    for (int k = 0; k < kSortPer; ++k)
      if (tid + kSorterThreads * k < m) atomicAdd(&fcnt[fbin(rk[k])], 1u);
    __syncthreads();
    int mine = 0, big = 0;
#pragma unroll
    for (int e = 0; e < kPerT; ++e) {
      const uint32_t c = fcnt[tid * kPerT + e];
      mine += (int)c;
      big |= c > kFineMax;
    }
    if (big) atomicOr(&sm.big, 1);
    int total;
    int run = block_excl_scan<kSorterWarps>(mine, sm.wtot, total);
    if (!sm.big) {
      // counters become cursors (start ranks) and the pairs are scattered
#pragma unroll
      for (int e = 0; e < kPerT; ++e) {
        const uint32_t c = fcnt[tid * kPerT + e];
        fcnt[tid * kPerT + e] = (uint32_t)run;
        run += (int)c;
      }
      __syncthreads();
#pragma unroll
      for (int k = 0; k < kSortPer; ++k) {
        if (tid + kSorterThreads * k < m) {
          const uint32_t pos = atomicAdd(&fcnt[fbin(rk[k])], 1u);
          sm.key[pos] = rk[k];
          sm.val[pos] = rv[k];
        }
      }
      __syncthreads();
      // insertion sort of every fine bin (typically 1-3 elements); the
      // cursors now hold each bin's end, so a bin starts where the last ended
#pragma unroll
      for (int e = 0; e < kPerT; ++e) {
        const int b = tid * kPerT + e;
        const int end = (int)fcnt[b];
        const int beg = b ? (int)fcnt[b - 1] : 0;
        for (int a2 = beg + 1; a2 < end; ++a2) {
          const uint32_t kk = sm.key[a2], vv = sm.val[a2];
          int b2 = a2 - 1;
          while (b2 >= beg && (sm.key[b2] > kk || (sm.key[b2] == kk && sm.val[b2] > vv))) {
            sm.key[b2 + 1] = sm.key[b2];
            sm.val[b2 + 1] = sm.val[b2];
            --b2;
          }
          sm.key[b2 + 1] = kk;
          sm.val[b2 + 1] = vv;
        }
      }
      __syncthreads();
      for (int i = tid; i < m; i += kSorterThreads) {
        sorted[base + i] = key_score(sm.key[i]);
        perm[base + i] = kSink + (int32_t)sm.val[i];
      }
      return;
    }
  }

  // a crowded fine bin (a cluster of near-equal or equal keys): stable LSD
  // radix sort by (key, index), passes over the bucket-relative index first
  // and then over the bucket-relative key, each pass scattering from the
  // registers into the shared array
  if (tid == 0) { sm.kmin = 0xFFFFFFFFu; sm.kmax = 0u; sm.vmin = 0xFFFFFFFFu; sm.vmax = 0u; }
  __syncthreads();
  {
    uint32_t kmin = 0xFFFFFFFFu, kmax = 0u, vmin = 0xFFFFFFFFu, vmax = 0u;
#pragma unroll
    for (int k = 0; k < kSortPer; ++k) {
      if (tid + kSorterThreads * k < m) {
        kmin = min(kmin, rk[k]);
        kmax = max(kmax, rk[k]);
        vmin = min(vmin, rv[k]);
        vmax = max(vmax, rv[k]);
      }
    }
    kmin = __reduce_min_sync(0xffffffffu, kmin);
    kmax = __reduce_max_sync(0xffffffffu, kmax);
    vmin = __reduce_min_sync(0xffffffffu, vmin);
    vmax = __reduce_max_sync(0xffffffffu, vmax);
    if (lane == 0) {
      atomicMin(&sm.kmin, kmin);
      atomicMax(&sm.kmax, kmax);
      atomicMin(&sm.vmin, vmin);
      atomicMax(&sm.vmax, vmax);
    }
  }
  __syncthreads();
  const uint32_t k0 = sm.kmin;
  const uint32_t span = sm.kmax - k0;
  const uint32_t v0 = sm.vmin;
  const uint32_t vspan = sm.vmax - v0;
  const int vpasses = (32 - __clz(vspan) + 7) / 8;
  const int kpasses = span ? (32 - __clz(span) + 7) / 8 : 0;
  const int passes = vpasses + kpasses;
  if (passes == 0) {
    // a single element
    if (tid < m) {
      sorted[base + tid] = key_score(rk[0]);
      perm[base + tid] = kSink + (int32_t)rv[0];
    }
    return;
  }
  for (int pass = 0; pass < passes; ++pass) {
    const bool on_val = pass < vpasses;
    const int shift = 8 * (on_val ? pass : pass - vpasses);
    const uint32_t org = on_val ? v0 : k0;
    if (pass) {
      // the previous pass's order, back into the registers
#pragma unroll
      for (int k = 0; k < kSortPer; ++k) {
        const int i = tid + kSorterThreads * k;
        if (i < m) {
          rk[k] = sm.key[i];
          rv[k] = sm.val[i];
        }
      }
    }
    // digit totals
    for (int k = tid; k < kSorterWarps * 256; k += kSorterThreads) (&sm.cnt[0][0])[k] = 0;
    __syncthreads();
#pragma unroll
    for (int k = 0; k < kSortPer; ++k)
      if (tid + kSorterThreads * k < m) atomicAdd(&sm.cnt[warp][(((on_val ? rv[k] : rk[k]) - org) >> shift) & 255u], 1u);
    __syncthreads();
    if (tid < 256) {
      uint32_t t = 0;
      for (int w = 0; w < kSorterWarps; ++w) t += sm.cnt[w][tid];
      sm.dbase[tid] = t;
    }
    __syncthreads();
    if (warp == 0) {
      uint32_t v[8], run = 0;
#pragma unroll
      for (int k = 0; k < 8; ++k) { v[k] = run; run += sm.dbase[lane * 8 + k]; }
      uint32_t incl = run;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      const uint32_t excl = incl - run;
      __syncwarp();
#pragma unroll
      for (int k = 0; k < 8; ++k) sm.dbase[lane * 8 + k] = excl + v[k];
    }
    __syncthreads();
    // stable scatter, 512 pairs (one per thread) per step, in register order
#pragma unroll
    for (int k = 0; k < kSortPer; ++k) {
      const bool valid = tid + kSorterThreads * k < m;
      const uint32_t dg = (((on_val ? rv[k] : rk[k]) - org) >> shift) & 255u;
#pragma unroll
      for (int q = 0; q < 8; ++q) sm.cnt[warp][lane * 8 + q] = 0;
      __syncwarp();
      const uint32_t peers = __match_any_sync(0xffffffffu, valid ? dg : 0xFFFFFFFFu);
      const uint32_t rank = __popc(peers & lt_mask);
      if (valid && (__ffs(peers) - 1) == lane) sm.cnt[warp][dg] = __popc(peers);
      __syncthreads();
      if (tid < 256) {
        uint32_t run = sm.dbase[tid];
        for (int w = 0; w < kSorterWarps; ++w) {
          const uint32_t c = sm.cnt[w][tid];
          sm.cnt[w][tid] = run;
          run += c;
        }
        sm.dbase[tid] = run;
      }
      __syncthreads();
      if (valid) {
        const uint32_t pos = sm.cnt[warp][dg] + rank;
        sm.key[pos] = rk[k];
        sm.val[pos] = rv[k];
      }
      __syncthreads();
    }
  }
  for (int i = tid; i < m; i += kSorterThreads) {
    sorted[base + i] = key_score(sm.key[i]);
    perm[base + i] = kSink + (int32_t)sm.val[i];
  }
}

// CTA = a group of kSortGroup consecutive slots; empty slots (the buckets a
// segment did not need) cost one read of the group's records
constexpr int kSortGroup = 8;
__global__ void __launch_bounds__(kSorterThreads, 3) k_bucket_sort(const uint32_t* __restrict__ stage_key,
                                                                  const uint32_t* __restrict__ stage_val,
                                                                  const BucketSlot* __restrict__ slots,
                                                                  const float2* __restrict__ range,
                                                                  float* __restrict__ sorted,
                                                                  int32_t* __restrict__ perm, int64_t nslots,
                                                                  int S, int64_t T) {
  extern __shared__ uint8_t bsm_raw[];
  BucketSmem& sm = *reinterpret_cast<BucketSmem*>(bsm_raw);
  __shared__ BucketSlot group[kSortGroup];
  const int64_t g0 = (int64_t)blockIdx.x * kSortGroup;
  if (threadIdx.x < kSortGroup) {
    const int64_t k = g0 + threadIdx.x;
    BucketSlot sl{};
    if (k < nslots) sl = slots[k];
    group[threadIdx.x] = sl;
  }
  __syncthreads();
  for (int gi = 0; gi < kSortGroup; ++gi) {
    const BucketSlot slot = group[gi];
    if (slot.count == 0) continue;
    sort_bucket(slot, sm, stage_key, stage_val, range, sorted, perm, S, T);
    __syncthreads();  // the next bucket reuses the shared arrays
  }
}

// ---------------------------------------------------------------------------
// block masses of the sorted scores and the stop point: one CTA per segment
// ---------------------------------------------------------------------------
// Blocks past plen[(b,kvh,s)] / Bk are not evaluated: the planner proved the
// block starting there fails the test (it is the stop point if no earlier
// block fails).
__global__ void __launch_bounds__(256) k_mass_stop(const float* __restrict__ sorted, const float* __restrict__ segM,
                                                  const double* __restrict__ segZ, const int* __restrict__ plen,
                                                  int32_t* __restrict__ nblocks, int BHkv, int S, int64_t T,
                                                  double tau) {
  __shared__ int cmin;
  const int q = blockIdx.x;
  const int s = S - 1 - q / BHkv;
  const int bk = q % BHkv;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int nb = min((int)(num_cand(s) / kBk), plen[(size_t)bk * S + s] / kBk);
  if (threadIdx.x == 0) cmin = nb;
  __syncthreads();
  const float* ss = sorted + (size_t)bk * T + cand_offset(s);
  const float M = segM[(size_t)bk * S + s];
  const double Z = segZ[(size_t)bk * S + s];
  for (int blk = warp; blk < nb; blk += 8) {
    float e = exp_shifted(ss[blk * kBk + lane], M) + exp_shifted(ss[blk * kBk + 32 + lane], M);
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) e += __shfl_xor_sync(0xffffffffu, e, o);
    if (lane == 0 && (double)e / Z < tau) atomicMin(&cmin, blk);
  }
  __syncthreads();
  if (threadIdx.x == 0) nblocks[(size_t)bk * S + s] = cmin;
}

}  // namespace s2o
