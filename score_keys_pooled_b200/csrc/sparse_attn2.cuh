// Kernel (3), GQA form: two query heads of a KV group per CTA, warp-specialised.
//
// Same method as k_sparse_attn (gist.science technical summary, section 3:
// pass 1 = the segment's dense causal window, pass 2 = keys in permuted order
// up to the stop; section 1, "Chargement Planifie par Coordonnees": K/V rows
// gathered by index), laid out for the B200 tensor core:
//
//   * one CTA = (b, kvh, s, pair): query heads h0 = kvh*G + 2*pair and h0+1
//     share every gathered K/V tile (each tile is fetched once for 256 rows);
//   * 128-key tiles: 64-key blocks of the key walk taken two at a time
//     (diagonal, previous window, sinks, then the kept candidate blocks; an
//     odd last block leaves an empty, zero-filled and masked half); the
//     tensor core and the softmax step through them one 64-key chunk (one
//     block, half a tile) at a time;
//   * warp roles (384 threads): warps 0-3 and 4-7 run the online softmax of
//     head 0 and head 1 (thread = row = TMEM lane), one thread of warp 8 and
//     one of warp 11 issue the tcgen05.mma of head 0 and head 1 (a single
//     issuer stalls the tensor pipe whenever it waits on one head's softmax,
//     and one thread cannot issue fast enough to keep it busy anyway), warps
//     9 and 10 gather K and V rows with cp.async (16 bytes a lane, written in
//     the tensor core's 128B-swizzled layout) into a 3-stage K ring and a
//     2-stage V ring; a loader arrives on a stage's mbarrier once its copies
//     have landed (K is released as soon as both heads' S are computed, so
//     its loads run up to three tiles ahead); the key indices of the next
//     tile are fetched while the copies of this one fly; Q arrives as 2D
//     TMA tiles;
//   * tensor memory (512 columns): O_i in [128 i, 128 i + 128); S_i of one
//     chunk in [256 + 64 i, +64); two P buffers per head (bf16, two per
//     column) in [384 + 64 i + 32 b, +32).  P is the A operand of
//     O_i += P_i V straight from tensor memory, so it never touches shared
//     memory.  S_i is released as soon as the softmax has read it into
//     registers, so Q K^T of the next chunk runs while the softmax of this
//     one computes; the exp2 work (bound by the special-function unit) and
//     the tensor core then overlap instead of waiting on each other;
//   * registers are rebalanced per warpgroup (setmaxnreg): the launch gives
//     168 per thread; warps 8-11 drop to 80 and the two softmax warpgroups
//     rise to 208 (per SM sub-partition 2 x 208 + 80 <= 3 x 168), enough to
//     hold a thread's 128 scores of a tile at once.
// Online softmax: exp2 domain, lazy rescale (the row's reference max moves
// only when it grows by more than 2^8, which leaves the result exact).
// Every mbarrier wait is bounded; a wait that runs out sets the device error
// word and the CTA winds down without hanging.
#pragma once
#include <cuda.h>  // CUtensorMap (the encoder is fetched from the driver at run time)

#include "s2o_common.cuh"

namespace s2o {

constexpr int kKT2 = 128;                 // keys per tile
constexpr int kAttn2Threads = 384;
constexpr int kMmaWarp = 8;                          // issuer of head 0 (and TMEM owner)
constexpr int kMmaWarp1 = 11;                        // issuer of head 1
constexpr int kLoadWarp0 = 9;
constexpr int kStagesK = 3;                          // K ring (freed once Q K^T of both heads is done)
constexpr int kStagesV = 2;                          // V ring (freed once P V of both heads is done)
constexpr uint32_t kTile2Bytes = 2 * 128 * 128;      // one 128-row operand tile: 2 atoms x 128 rows x 128 B
constexpr uint32_t kOff2Q = 0;                       // Q0, Q1
constexpr uint32_t kOff2K = 2 * kTile2Bytes;         // K stages
constexpr uint32_t kOff2V = kOff2K + kStagesK * kTile2Bytes;
constexpr uint32_t kOff2Bar = kOff2V + kStagesV * kTile2Bytes;
constexpr uint32_t kOff2Keys = kOff2Bar + 256;         // per loader warp: keys of its tile rows, by row parity
constexpr uint32_t kOff2Rows = kOff2Keys + 2 * 512;     // regrouped Q_perm: the segment rows of one sub-segment
constexpr uint32_t kAttn2SmemData = kOff2Rows + 4 * (kLq / 2 + 4);
constexpr size_t kAttn2Smem = kAttn2SmemData + 1024;  // + alignment slack
constexpr uint32_t kTmem2Cols = 512;

// barrier slots (8 bytes each) from kOff2Bar
constexpr int kBarKFull = 0;    // [3]  K loader (after its copies landed) -> MMA
constexpr int kBarKEmpty = 3;   // [3]  MMA commits of both issuers (count 2) -> K loader
constexpr int kBarVFull = 6;    // [2]  V loader (after its copies landed) -> MMA
constexpr int kBarVEmpty = 8;   // [2]  MMA commits of both issuers (count 2) -> V loader
constexpr int kBarQFull = 10;   //      K loader -> MMA (TMA bytes)
// per head i (and P buffer b)
constexpr int kBarSFull = 11;   // [2]     MMA commit (S_i written) -> softmax i
constexpr int kBarSEmpty = 13;  // [2]     softmax i, one arrive per warp (S_i read) -> MMA
constexpr int kBarPFull = 15;   // [2][2]  softmax i, one arrive per warp (P_i,b written) -> MMA; slot + 2 i + b
constexpr int kBarODone = 19;   // [2][2]  MMA commit (P_i,b consumed, O_i updated) -> softmax i
constexpr int kBarGain = 23;    //      online stop: the 8 softmax warps (count 8) added their rows' gains
constexpr int kSlotTmem = 24;
constexpr int kSlotGain = 25;   //      online stop: 3 fp32 gain accumulators (slots 25, 26)
constexpr int kSlotStop = 27;   //      online stop: index of the chunk after which the tile stops
constexpr int kBarDrain = 28;   // [2]  issuer i's final commit: every tensor-core op it issued is done
constexpr int kNoStop = 0x7fffffff;
// tensor-memory columns
__device__ __forceinline__ uint32_t col_o(int i) { return 128u * i; }
__device__ __forceinline__ uint32_t col_s(int i) { return 256u + 64u * i; }
__device__ __forceinline__ uint32_t col_p(int i, int b) { return 384u + 64u * i + 32u * b; }

__device__ __forceinline__ void tc_mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n"
      " setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n}\n" ::"r"(d_tmem),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
template <uint32_t R>
__device__ __forceinline__ void regs_increase() {
  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;\n" ::"n"(R));
}
template <uint32_t R>
__device__ __forceinline__ void regs_decrease() {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;\n" ::"n"(R));
}
constexpr uint32_t kRegsSoftmax = 208, kRegsOther = 80;
static_assert(2 * kRegsSoftmax + kRegsOther <= 3 * 168, "register split exceeds the launch's budget");

// packed pairs of fp32 (sm_100 f32x2 arithmetic): one instruction, two lanes
__device__ __forceinline__ uint64_t f2_pack(float lo, float hi) {
  return ((uint64_t)__float_as_uint(hi) << 32) | (uint64_t)__float_as_uint(lo);
}
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ float f2_lo(uint64_t v) { return __uint_as_float((uint32_t)v); }
__device__ __forceinline__ float f2_hi(uint64_t v) { return __uint_as_float((uint32_t)(v >> 32)); }

// 2D tiled TMA load (box of the tensor map) into shared memory
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int x, int y, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];\n" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
      : "memory");
}
// warp-uniform bounded wait: every lane polls, all agree on the outcome
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, uint32_t limit) {
  const bool ok = mbar_wait_bounded(bar, parity, limit);
  return __all_sync(0xffffffffu, ok);
}

// 64-key block b of a work item: kind 0 = diagonal (causal, keys j0..j0+63),
// 1 = contiguous, 2 = gathered candidate block j0 of perm, 3 = empty.
struct Walk2 {
  int n_diag, n_prev, n_sink, nb;
};
__device__ __forceinline__ Walk2 make_walk2(int s, int N, int C) {
  Walk2 w;
  const int rows = min(N, kLq * s + kLq) - kLq * s;
  w.n_diag = (rows + kBk - 1) / kBk;
  w.n_prev = (s >= 1) ? 2 : 0;
  w.n_sink = (s >= 2) ? 1 : 0;
  w.nb = w.n_diag + w.n_prev + w.n_sink + C;
  return w;
}
__device__ __forceinline__ int walk2_block(const Walk2& w, int s, int b, int& j0) {
  if (b >= w.nb) { j0 = 0; return 3; }
  if (b < w.n_diag) { j0 = kLq * s + kBk * b; return 0; }
  b -= w.n_diag;
  if (b < w.n_prev) { j0 = kLq * s - kLq + kBk * b; return 1; }
  b -= w.n_prev;
  if (b < w.n_sink) { j0 = 0; return 1; }
  j0 = b - w.n_sink;
  return 2;
}

struct Attn2Args {
  const uint16_t* Q;
  const uint16_t* K;
  const uint16_t* V;
  const int32_t* perm;
  const int32_t* nblocks;
  void* O;
  int B, Hq, Hkv, N, S;
  int64_t T;
  int out_f32;
  // run-time stop (k_sparse_attn2<true>; gist.science technical summary,
  // section 2): walk every candidate block of the full order and stop after
  // the first one whose mean relative gain over the tile's rows is below tau;
  // blocks processed per query head go to cout [B, Hq, S]
  float tau;
  int32_t* cout;
  // Q_perm (k_sparse_attn2<false, true>): the segment's rows form two
  // sub-segments (rowsub [B, Hkv, S, 128]) with their own orders and stops;
  // the key walk covers sub-segment 0's kept blocks (perm, nblocks) then
  // sub-segment 1's (perm1, nblocks1), each masked for the other's rows
  const int32_t* perm1;
  const int32_t* nblocks1;
  const uint8_t* rowsub;
  // polls of every pipeline wait before it gives up (kSpinLimit; smaller only
  // to exercise the timeout path).  The final drains always use kSpinLimit.
  uint32_t spin;
};

// The loader warps of the attention kernels (warp kLoadWarp0 = K ring and
// Q, warp kLoadWarp0 + 1 = V ring): for tile t of the key walk, gather its
// 128 K (or V) rows by index into ring stage t % stages once the stage is
// free, and arrive on the stage's full barrier after the copies landed.
template <bool ONLINE, bool QPERM, bool QTMA = true>
__device__ __forceinline__ void attn_load_ring(const Attn2Args& a, const CUtensorMap* tmQ, uint32_t sbase,
                                               uint8_t* sgen, int warp, int lane, int b, int bk, int s, int h0,
                                               int row0, const Walk2& wk, int ntiles, int C0,
                                               volatile int* stop_word) {
  auto bar = [&](int k) { return sbase + kOff2Bar + 8u * (uint32_t)k; };
  const bool is_k = warp == kLoadWarp0;
  const int nst = is_k ? kStagesK : kStagesV;
  const int bar_full = is_k ? kBarKFull : kBarVFull;
  const int bar_empty = is_k ? kBarKEmpty : kBarVEmpty;
  const uint32_t ring = sbase + (is_k ? kOff2K : kOff2V);
  const uint16_t* kv = (is_k ? a.K : a.V) + (size_t)bk * a.N * kD;
  if (QTMA && is_k && lane == 0) {
    mbar_expect_tx(bar(kBarQFull), 2 * kTile2Bytes);
#pragma unroll
    for (int qi = 0; qi < 2; ++qi)
#pragma unroll
      for (int half = 0; half < 2; ++half)
        tma_load_2d(sbase + kOff2Q + qi * kTile2Bytes + half * (128 * 128), tmQ, 64 * half,
                    (b * a.Hq + h0 + qi) * a.N + row0, bar(kBarQFull));
  }
  const int32_t* pseg = a.perm + (size_t)bk * a.T + cand_offset(s);
  const int cand_hi = kLq * s - kWin;
  // raw key indices of tile rows 4 lane .. 4 lane + 3 (loaded, not yet used)
  auto fetch_keys = [&](int t, int* y) {
    int j0;
    const int kind = walk2_block(wk, s, 2 * t + (lane >> 4), j0);
    const int rr = (4 * lane) & 63;
    if (kind == 2) {
      const int32_t* ps = pseg;
      if (QPERM && j0 >= C0) {
        ps = a.perm1 + (size_t)bk * a.T + cand_offset(s);
        j0 -= C0;
      }
      const int4 v = *reinterpret_cast<const int4*>(ps + kBk * j0 + rr);
      y[0] = v.x; y[1] = v.y; y[2] = v.z; y[3] = v.w;
    } else {
#pragma unroll
      for (int k = 0; k < 4; ++k) y[k] = kind == 3 ? -1 : j0 + rr + k;
    }
  };
  // checked keys (-1: a zero row: an empty half or a key past N) into the
  // warp's table: row r = 2 jj + p at keys[p][jj]; true if any is -1
  int32_t* keys = reinterpret_cast<int32_t*>(sgen + kOff2Keys + (is_k ? 0 : 512));
  const uint32_t keys_s = sbase + kOff2Keys + (is_k ? 0u : 512u);
  auto stage_keys = [&](int t, const int* y) {
    int j0;
    const int kind = walk2_block(wk, s, 2 * t + (lane >> 4), j0);
    int k4[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      int j = y[k];
      if (kind == 2) {
        if (j < kSink || j >= cand_hi) {  // caller-supplied plan out of Cand(s)
          set_error(kErrBadPlan);
          j = kSink;
        }
      } else if (j >= a.N) {
        j = -1;
      }
      k4[k] = j;
    }
    // rows 4 lane + k: parity k & 1, slot 2 lane + (k >> 1)
    *reinterpret_cast<int2*>(keys + 2 * lane) = make_int2(k4[0], k4[2]);
    *reinterpret_cast<int2*>(keys + 64 + 2 * lane) = make_int2(k4[1], k4[3]);
    __syncwarp();
    return __any_sync(0xffffffffu, k4[0] < 0 || k4[1] < 0 || k4[2] < 0 || k4[3] < 0);
  };
  // this lane copies 16-byte chunk q of rows 2 jj + sel (swizzle atom q / 8,
  // chunk q % 8 xor row % 8); its destination offsets repeat with jj % 4
  const int q = lane & 15, sel = lane >> 4;
  uint32_t dsw[4];
#pragma unroll
  for (int m = 0; m < 4; ++m)
    dsw[m] = (uint32_t)(q >> 3) * (128 * 128) + (uint32_t)sel * 128 +
             ((uint32_t)((q & 7) ^ ((2 * m + sel) & 7)) << 4);
  const char* src0 = reinterpret_cast<const char*>(kv) + 16 * q;
  const uint32_t ktab = keys_s + 256u * (uint32_t)sel;
  int y[4];
  if (ntiles > 0) fetch_keys(0, y);
  // with the run-time stop a tile past the stop point is not needed: the
  // last products issued after a stop at chunk c read K of chunk c + 1
  auto not_needed = [&](int t) {
    const int sc = *stop_word;
    return sc != kNoStop && t > sc / 2 + 1;
  };
  for (int t = 0; t < ntiles; ++t) {
    const int st = t % nst;
    const int round = t / nst;
    if (ONLINE && not_needed(t)) break;
    const bool ragged = stage_keys(t, y);
    if (t + 1 < ntiles) fetch_keys(t + 1, y);  // in flight while this stage fills
    bool okw;
    if (!ONLINE) {
      okw = warp_wait(bar(bar_empty + st), (uint32_t)((round & 1) ^ 1), a.spin);
    } else {
      // lane 0 waits for the stage or for a stop that makes it unneeded;
      // after a free stage every lane acquires the barrier itself
      int r = 0;
      if (lane == 0) {
        for (uint32_t it = 0; it < a.spin && r == 0; ++it) {
          if (mbar_try_wait(bar(bar_empty + st), (uint32_t)((round & 1) ^ 1))) r = 1;
          else if (not_needed(t)) r = 2;
        }
      }
      r = __shfl_sync(0xffffffffu, r, 0);
      if (r == 2) break;
      okw = r == 1 && warp_wait(bar(bar_empty + st), (uint32_t)((round & 1) ^ 1), a.spin);
    }
    if (!okw) {
      if (lane == 0) set_error(kErrTimeout);
      break;
    }
    const uint32_t dst0 = ring + st * kTile2Bytes;
    // 64 copies per lane; the key table is read four keys at a time.  A tile
    // with a zero row (rare: an empty half or keys past N) takes the loop
    // with per-row source sizes; the branch stays outside the unrolled loop
    // so that each copy issues once.
    if (!ragged) {
#pragma unroll
      for (int j4 = 0; j4 < 16; ++j4) {
        int4 kk;
        asm volatile("ld.shared.v4.s32 {%0, %1, %2, %3}, [%4];\n"
                     : "=r"(kk.x), "=r"(kk.y), "=r"(kk.z), "=r"(kk.w)
                     : "r"(ktab + 16u * (uint32_t)j4)
                     : "memory");
        const int key4[4] = {kk.x, kk.y, kk.z, kk.w};
#pragma unroll
        for (int m = 0; m < 4; ++m)
          cp_async16(dst0 + dsw[m] + 256u * (uint32_t)(4 * j4 + m), src0 + (size_t)key4[m] * (kD * 2), 16u);
      }
    } else {
#pragma unroll 4
      for (int jj = 0; jj < 64; ++jj) {
        const int key = keys[64 * sel + jj];
        cp_async16(dst0 + dsw[jj & 3] + 256u * (uint32_t)jj, src0 + (size_t)(key < 0 ? 0 : key) * (kD * 2),
                   key < 0 ? 0u : 16u);
      }
    }
    cp_async_wait_all();
    fence_proxy_async_smem();  // generic-proxy writes -> tensor-core reads
    __syncwarp();
    if (lane == 0) mbar_arrive(bar(bar_full + st));
  }
  // Q's TMA tiles may still be landing if the issuers gave up waiting for
  // them: shared memory must not change after the CTA ends
  if (is_k && lane == 0 && !mbar_wait_bounded(bar(kBarQFull), 0)) set_error(kErrTimeout);
}

// ONLINE selects the run-time stop, QPERM the two query sub-segments (walked
// together by every row, each masked for the other's rows); QGROUP (with
// QPERM, group sizes divisible by 4) regroups the rows instead: a CTA takes
// one sub-segment of a segment for four query heads, its two 128-row tiles
// holding two heads' 64 rows of that sub-segment each, so every row of the
// CTA walks the same kept set and nothing is masked.  The planned-stop
// kernel is compiled without any of their code.
template <bool ONLINE, bool QPERM = false, bool QGROUP = false>
__global__ void __launch_bounds__(kAttn2Threads, 1)
    k_sparse_attn2(Attn2Args a, const __grid_constant__ CUtensorMap tmQ) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t sbase = (smem_u32(smem_raw) + 1023u) & ~1023u;
  uint8_t* sgen = smem_raw + (sbase - smem_u32(smem_raw));
  auto bar = [&](int k) { return sbase + kOff2Bar + 8u * (uint32_t)k; };
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(sgen + kOff2Bar + 8 * kSlotTmem);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = a.Hq / a.Hkv;
  const int pairs = G / 2;
  // work order: KV head by KV head (the CTAs running together then share one
  // head's K/V, which stays in L2), segments longest first, the pairs of a
  // segment adjacent (they gather the same rows)
  const int w = blockIdx.x;
  // units of a segment: head pairs, or (QGROUP) head quads x sub-segments
  const int units = QGROUP ? (G / 4) * 2 : pairs;
  const int per_bk = a.S * units;
  const int bk = w / per_bk;
  const int rest = w % per_bk;
  const int s = a.S - 1 - rest / units;
  const int unit = rest % units;
  const int qsub = QGROUP ? (unit & 1) : 0;  // the sub-segment of a QGROUP CTA
  const int b = bk / a.Hkv, kvh = bk % a.Hkv;
  // first query head of the CTA: tile i holds heads h0 + i (or, QGROUP,
  // h0 + 2 i and h0 + 2 i + 1)
  const int h0 = QGROUP ? kvh * G + 4 * (unit >> 1) : kvh * G + 2 * unit;

  const int cmax = (int)(num_cand(s) / kBk);
  int C = ONLINE ? cmax : ((QGROUP && qsub) ? a.nblocks1 : a.nblocks)[(size_t)bk * a.S + s];
  if (C < 0 || C > cmax) {
    if (tid == 0) set_error(kErrBadPlan);
    C = C < 0 ? 0 : cmax;
  }
  const int C0 = C;  // blocks of the first list (Q_perm: sub-segment 0)
  if (QPERM && !QGROUP) {
    int C1 = a.nblocks1[(size_t)bk * a.S + s];
    if (C1 < 0 || C1 > cmax) {
      if (tid == 0) set_error(kErrBadPlan);
      C1 = C1 < 0 ? 0 : cmax;
    }
    C = C0 + C1;
  }
  const Walk2 wk = make_walk2(s, a.N, C);
  const int ntiles = (wk.nb + 1) / 2;
  const int row0 = kLq * s;

  if (tid == 0) {
    for (int k = 0; k < kSlotTmem; ++k) {
      uint32_t count = 1;
      if ((k >= kBarSEmpty && k < kBarSEmpty + 2) || (k >= kBarPFull && k < kBarPFull + 4)) count = 4;
      if ((k >= kBarKEmpty && k < kBarKEmpty + kStagesK) || (k >= kBarVEmpty && k < kBarVEmpty + kStagesV)) count = 2;
      if (k == kBarGain) count = 8;
      mbar_init(bar(k), count);
    }
    mbar_init(bar(kBarDrain), 1);
    mbar_init(bar(kBarDrain + 1), 1);
    float* gacc = reinterpret_cast<float*>(sgen + kOff2Bar + 8 * kSlotGain);
    gacc[0] = gacc[1] = gacc[2] = 0.f;
    *reinterpret_cast<volatile int*>(sgen + kOff2Bar + 8 * kSlotStop) = kNoStop;
    fence_mbar_init();
  }
  // QGROUP: the segment rows of sub-segment qsub, ascending (entries 0 ..
  // n - 1), and their number n (entry kLq / 2); read by every role after the
  // block barrier below
  int32_t* rows_tab = reinterpret_cast<int32_t*>(sgen + kOff2Rows);
  if (QGROUP && warp == 0) {
    const uint32_t sub4 =
        *reinterpret_cast<const uint32_t*>(a.rowsub + ((size_t)bk * a.S + s) * kLq + 4 * lane);
    int f[4], cnt = 0;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      f[k] = (int)((sub4 >> (8 * k)) & 0xFFu) == qsub && row0 + 4 * lane + k < a.N;
      cnt += f[k];
    }
    int incl = cnt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    int pos = incl - cnt;
#pragma unroll
    for (int k = 0; k < 4; ++k)
      if (f[k]) {
        if (pos < kLq / 2) rows_tab[pos] = row0 + 4 * lane + k;
        ++pos;
      }
    if (lane == 31) {
      // a sub-segment holds at most half the rows (caller-supplied rowsub
      // otherwise: flagged, extra rows dropped)
      if (incl > kLq / 2) set_error(kErrBadPlan);
      rows_tab[kLq / 2] = min(incl, kLq / 2);
    }
  }
  volatile int* stop_word = reinterpret_cast<volatile int*>(sgen + kOff2Bar + 8 * kSlotStop);
  if (warp == kMmaWarp) {
    tmem_alloc(smem_u32((const void*)tmem_slot), kTmem2Cols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  if (warp >= kLoadWarp0 && warp < kMmaWarp1) {
    // ------------------------------------------------------------------ loaders
    // warp 9 loads Q (2D TMA) and the K ring, warp 10 the V ring.  The
    // gathered rows go through cp.async, 16 bytes per lane: lanes 0-15 copy
    // one 256-byte row, lanes 16-31 the next, written in the 128B-swizzled
    // layout the tensor core reads (one TMA gather4 per four rows issues far
    // slower than the load/store unit takes these copies).
    regs_decrease<kRegsOther>();
    if (QGROUP) {
      if (warp == kLoadWarp0) {
        // Q rows by index (lanes take 16-byte chunks of tile rows in turn),
        // into the 128B-swizzled layout the 2D TMA writes otherwise; rows
        // past the sub-segment's are zero
        const int nq = rows_tab[kLq / 2];
        for (int idx = lane; idx < 2 * kLq * 16; idx += 32) {
          const int rr = idx >> 4, q16 = idx & 15;
          const int ti = rr >> 7, r = rr & 127, k = r & 63;
          const int head = h0 + 2 * ti + (r >> 6);
          const int row = k < nq ? rows_tab[k] : -1;
          const uint16_t* src = a.Q + ((size_t)(b * a.Hq + head) * a.N + (size_t)(row < 0 ? 0 : row)) * kD + 8 * q16;
          const uint32_t dst = sbase + kOff2Q + ti * kTile2Bytes + (q16 >> 3) * (128 * 128) + r * 128 +
                               (((q16 & 7) ^ (r & 7)) << 4);
          cp_async16(dst, src, row < 0 ? 0u : 16u);
        }
        cp_async_wait_all();
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(kBarQFull));
      }
      Attn2Args aq = a;
      aq.perm = qsub ? a.perm1 : a.perm;
      attn_load_ring<ONLINE, false, false>(aq, &tmQ, sbase, sgen, warp, lane, b, bk, s, h0, row0, wk, ntiles, C,
                                           stop_word);
    } else {
      attn_load_ring<ONLINE, QPERM>(a, &tmQ, sbase, sgen, warp, lane, b, bk, s, h0, row0, wk, ntiles, C0,
                                    stop_word);
    }
  } else if (warp == kMmaWarp || warp == kMmaWarp1) {
    // ------------------------------------------------------------------ MMA issuers
    // head i's products, in order: its P V of tile t-1 and half h precedes its
    // Q K^T of tile t and half h, which overwrites that P.  The two issuers
    // share only the K/V stages (both commit before a stage is refilled).
    regs_decrease<kRegsOther>();
    const int i = warp == kMmaWarp ? 0 : 1;
    if (lane == 0) {
      const uint32_t idesc_qk = idesc_bf16_f32(128, kBk, false);   // one 64-key half
      const uint32_t idesc_pv = idesc_bf16_f32(128, 128, true);
      bool ok = mbar_wait_bounded(bar(kBarQFull), 0, a.spin);
      // chunk c = half c & 1 of tile c >> 1: S of chunk c as soon as the
      // softmax has read S of chunk c - 1, then P V of chunk c - 1
      const int nch = 2 * ntiles;
      for (int c = 0; ok && c <= nch; ++c) {
        if (c < nch) {
          const int t = c >> 1, h = c & 1;
          if (h == 0) {
            ok = mbar_wait_bounded(bar(kBarKFull + t % kStagesK), (uint32_t)((t / kStagesK) & 1), a.spin);
            if (!ok) break;
          }
          if (c > 0) {
            if (ONLINE) {
              // S of chunk c - 1 read, or the tile stopped before it
              int r = 0;
              for (uint32_t it = 0; it < a.spin && r == 0; ++it) {
                if (mbar_try_wait(bar(kBarSEmpty + i), (uint32_t)((c - 1) & 1))) r = 1;
                else if (*stop_word != kNoStop && c - 1 > *stop_word) r = 2;
              }
              if (r == 2) break;
              ok = r == 1;
            } else {
              ok = mbar_wait_bounded(bar(kBarSEmpty + i), (uint32_t)((c - 1) & 1), a.spin);
            }
            if (!ok) break;
            tc_fence_after();
          }
          const uint32_t sQ = sbase + kOff2Q + i * kTile2Bytes;
          const uint32_t sK = sbase + kOff2K + (t % kStagesK) * kTile2Bytes + kBk * h * 128;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint64_t ad = sdesc_sw128(sQ + (kk >> 2) * (128 * 128) + (kk & 3) * 32, 16, 1024);
            const uint64_t bd = sdesc_sw128(sK + (kk >> 2) * (128 * 128) + (kk & 3) * 32, 16, 1024);
            tc_mma_ss(tmem + col_s(i), ad, bd, idesc_qk, kk > 0 ? 1u : 0u);
          }
          tc_commit(bar(kBarSFull + i));
          if (h == 1) tc_commit(bar(kBarKEmpty + t % kStagesK));
        }
        if (c > 0) {
          const int cp = c - 1, tp = cp >> 1, hp = cp & 1;
          if (hp == 0) {
            ok = mbar_wait_bounded(bar(kBarVFull + tp % kStagesV), (uint32_t)((tp / kStagesV) & 1), a.spin);
            if (!ok) break;
          }
          if (ONLINE) {
            // P of chunk cp written, or the tile stopped before it
            int r = 0;
            for (uint32_t it = 0; it < a.spin && r == 0; ++it) {
              if (mbar_try_wait(bar(kBarPFull + 2 * i + hp), (uint32_t)((cp >> 1) & 1))) r = 1;
              else if (*stop_word != kNoStop && cp > *stop_word) r = 2;
            }
            if (r == 2) break;
            ok = r == 1;
          } else {
            ok = mbar_wait_bounded(bar(kBarPFull + 2 * i + hp), (uint32_t)((cp >> 1) & 1), a.spin);
          }
          if (!ok) break;
          tc_fence_after();
          const uint32_t sV = sbase + kOff2V + (tp % kStagesV) * kTile2Bytes;
#pragma unroll
          for (int kk = 0; kk < kBk / 16; ++kk) {
            const uint64_t bd = sdesc_sw128(sV + (kBk * hp + 16 * kk) * 128, 128 * 128, 1024);
            tc_mma_ts(tmem + col_o(i), tmem + col_p(i, hp) + 8 * kk, bd, idesc_pv, (cp > 0 || kk > 0) ? 1u : 0u);
          }
          tc_commit(bar(kBarODone + 2 * i + hp));
          if (hp == 1) tc_commit(bar(kBarVEmpty + tp % kStagesV));
          // the tile stopped after chunk cp: nothing more to multiply (products
          // still in flight are drained below)
          if (ONLINE && cp == *stop_word) break;
        }
      }
      if (!ok) set_error(kErrTimeout);
      // every product this thread issued must be done before the tensor
      // memory is freed (a given-up wait may leave some in flight)
      tc_commit(bar(kBarDrain + i));
      if (!mbar_wait_bounded(bar(kBarDrain + i), 0)) set_error(kErrTimeout);
    }
  } else {
    // ------------------------------------------------------------------ softmax
    regs_increase<kRegsSoftmax>();
    const int qi = warp >> 2;               // head of the pair
    const int r = tid & 127;                // row of the tile
    int row = row0 + r;                     // its row in the sequence
    int head = h0 + qi;                     // and its query head
    bool row_ok = row < a.N;
    if (QGROUP) {
      const int nq = rows_tab[kLq / 2];
      head = h0 + 2 * qi + (r >> 6);
      row_ok = (r & 63) < nq;
      row = row_ok ? rows_tab[r & 63] : row0;
    }
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    const int my_sub = (QPERM && !QGROUP) ? (int)a.rowsub[((size_t)bk * a.S + s) * kLq + r] : 0;
    const uint32_t tS = tmem + col_s(qi) + lane_base;
    const uint32_t tO = tmem + col_o(qi) + lane_base;
    const float sl2 = 1.4426950408889634f * 0.08838834764831845f;  // log2(e) / sqrt(d)
    float m_run = -INFINITY, ell = 0.f;
    bool ok = true;
    const int nch = 2 * ntiles;
    // online stop: rows of the tile that exist (both heads)
    const float nrows_valid = 2.f * (float)min(kLq, a.N - row0);
    volatile float* gacc = reinterpret_cast<volatile float*>(sgen + kOff2Bar + 8 * kSlotGain);
    int c_online = cmax;
    int nch_done = nch;
    for (int c = 0; ok && c < nch; ++c) {
      // key k of the chunk is visible iff k <= lim
      int j0;
      const int kind = walk2_block(wk, s, c, j0);
      int lim = kind == 3 ? -1 : (kind == 0 ? row - j0 : kBk);
      if (QPERM && !QGROUP && kind == 2 && (j0 >= C0 ? 1 : 0) != my_sub) lim = -1;  // the other sub-segment's block
      if (!warp_wait(bar(kBarSFull + qi), (uint32_t)(c & 1), a.spin)) { ok = false; break; }
      tc_fence_after();
      float x[kBk];
      tmem_ld32(tS, x);
      tmem_ld32(tS + 32, x + 32);
      tc_wait_ld();
      // S_i is free for the next chunk's Q K^T
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(kBarSEmpty + qi));
      const bool full = lim >= kBk;  // no key masked
      float mt = -INFINITY;
      if (full) {
        float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
        for (int k = 0; k < kBk; k += 2) m4[(k >> 1) & 3] = fmax3(m4[(k >> 1) & 3], x[k], x[k + 1]);
        mt = fmaxf(fmax3(m4[0], m4[1], m4[2]), m4[3]);
      } else {
#pragma unroll
        for (int k = 0; k < kBk; ++k)
          if (k <= lim) mt = fmaxf(mt, x[k]);
      }
      mt *= sl2;
      const bool move = mt > m_run + 8.f;
      float alpha = 1.f;
      if (move) {
        alpha = (m_run == -INFINITY) ? 0.f : ex2_approx(m_run - mt);
        m_run = mt;
        ell *= alpha;
      }
      // a moved reference rescales O once every P V issued so far (the last
      // one is chunk c - 1's) is done
      if (c > 0 && __any_sync(0xffffffffu, move)) {
        if (!warp_wait(bar(kBarODone + 2 * qi + ((c - 1) & 1)), (uint32_t)(((c - 1) >> 1) & 1), a.spin)) {
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll
        for (int cc = 0; cc < 128; cc += 32) {
          float o[32];
          tmem_ld32(tO + cc, o);
          tc_wait_ld();
#pragma unroll
          for (int k = 0; k < 32; ++k) o[k] *= alpha;
          tmem_st32(tO + cc, o);
        }
      }
      // P = exp2(S - m) as bf16 pairs, packed in place into x[0 .. 31]
      float rs;
      if (full) {
        const uint64_t s2 = f2_pack(sl2, sl2), nm2 = f2_pack(-m_run, -m_run);
        uint64_t rs2 = 0;
#pragma unroll
        for (int k = 0; k < kBk; k += 2) {
          const uint64_t v = f2_fma(f2_pack(x[k], x[k + 1]), s2, nm2);
          const float p0 = ex2_approx(f2_lo(v)), p1 = ex2_approx(f2_hi(v));
          rs2 = f2_add(rs2, f2_pack(p0, p1));
          x[k / 2] = __uint_as_float(pack_bf16x2(p0, p1));
        }
        rs = f2_lo(rs2) + f2_hi(rs2);
      } else {
        rs = 0.f;
#pragma unroll
        for (int k = 0; k < kBk; k += 2) {
          const float p0 = (k <= lim) ? ex2_approx(fmaf(x[k], sl2, -m_run)) : 0.f;
          const float p1 = (k + 1 <= lim) ? ex2_approx(fmaf(x[k + 1], sl2, -m_run)) : 0.f;
          rs += p0 + p1;
          x[k / 2] = __uint_as_float(pack_bf16x2(p0, p1));
        }
      }
      if (ONLINE && kind == 2 && j0 > 0) {
        // the tile's decision on the previous candidate block, whose gains
        // every warp posted one chunk ago (deciding here, not right after
        // posting, keeps the warps from waiting on each other every chunk):
        // below tau, the tile stopped after that block and this chunk does
        // not count
        const int qp = j0 - 1;
        if (!warp_wait(bar(kBarGain), (uint32_t)(qp & 1), a.spin)) { ok = false; break; }
        const float tot = gacc[qp % 3];
        // the slot used for qp - 1: every warp read it before posting qp
        if (warp == 0 && lane == 0) gacc[(qp + 2) % 3] = 0.f;
        if (tot < a.tau * nrows_valid) {
          c_online = qp + 1;
          if ((warp & 3) == 0 && lane == 0) *stop_word = c - 1;  // the last chunk that counts
          nch_done = c;
          break;
        }
      }
      ell += rs;
      if (ONLINE && kind == 2) {
        // the block's gain for this row, relative to everything the row has
        // processed (the block included; both sums share the reference
        // m_run), summed over the tile's rows; decided at the next
        // candidate block
        float gsum = row < a.N ? rs / ell : 0.f;
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) gsum += __shfl_xor_sync(0xffffffffu, gsum, o);
        if (lane == 0) {
          atomicAdd(const_cast<float*>(gacc + j0 % 3), gsum);
          mbar_arrive(bar(kBarGain));
        }
      }
      // P buffer c & 1 was last read by chunk c - 2's P V, which this head's
      // issuer committed before chunk c's Q K^T: the S-full barrier of chunk c
      // (waited above) already covers it
      tmem_st32(tmem + col_p(qi, c & 1) + lane_base, x);
      tc_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(kBarPFull + 2 * qi + (c & 1)));
    }
    if (ONLINE && tid == 0) {
      for (int k = 0; k < 2; ++k) a.cout[((size_t)b * a.Hq + h0 + k) * a.S + s] = c_online;
    }
    if (ok && nch_done > 0)
      ok = warp_wait(bar(kBarODone + 2 * qi + ((nch_done - 1) & 1)), (uint32_t)(((nch_done - 1) >> 1) & 1), a.spin);
    if (!ok) {
      if (lane == 0) set_error(kErrTimeout);
    } else {
      tc_fence_after();
      const float inv = ell > 0.f ? 1.f / ell : 0.f;
      const bool store = row_ok;
      const size_t orow = ((size_t)(b * a.Hq + head) * a.N + (size_t)(store ? row : 0)) * kD;
#pragma unroll
      for (int cc = 0; cc < 128; cc += 32) {
        float o[32];
        tmem_ld32(tO + cc, o);
        tc_wait_ld();
        if (store) {
          if (a.out_f32) {
            float4* dst = reinterpret_cast<float4*>(static_cast<float*>(a.O) + orow + cc);
#pragma unroll
            for (int k = 0; k < 8; ++k)
              dst[k] = make_float4(o[4 * k] * inv, o[4 * k + 1] * inv, o[4 * k + 2] * inv, o[4 * k + 3] * inv);
          } else {
            uint4* dst = reinterpret_cast<uint4*>(static_cast<uint16_t*>(a.O) + orow + cc);
#pragma unroll
            for (int k = 0; k < 4; ++k)
              dst[k] = make_uint4(pack_bf16x2(o[8 * k] * inv, o[8 * k + 1] * inv),
                                  pack_bf16x2(o[8 * k + 2] * inv, o[8 * k + 3] * inv),
                                  pack_bf16x2(o[8 * k + 4] * inv, o[8 * k + 5] * inv),
                                  pack_bf16x2(o[8 * k + 6] * inv, o[8 * k + 7] * inv));
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmem2Cols);
  }
}

}  // namespace s2o
