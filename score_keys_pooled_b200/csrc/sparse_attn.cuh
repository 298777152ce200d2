// Kernel (3): sparse prefill attention over the kept keys, on tcgen05.
//
// S2O's kernel is two-pass (gist.science technical summary, section 3,
// "Implementation du Noyau"): pass 1 computes the segment's dense causal
// window and initialises the online-softmax state (m, l, acc); pass 2 resumes
// that state and visits the historical keys in permuted order, up to the
// early stop.  Keys are gathered by index into on-chip memory ("Chargement
// Planifie par Coordonnees", section 1) while K/V keep their HBM layout.
//
// One CTA = one (b, head h, segment s): 128 query rows, 128 threads, thread r
// owns row r (= TMEM lane r).  The key list of the segment is walked in
// 64-key tiles:
//   pass 1: [128s, 128s+64), [128s+64, 128s+128) with the causal mask,
//           then the previous window [128s-128, 128s) and the sinks [0, 64)
//           (for s <= 1 the window already holds the sinks);
//   pass 2: perm[off(s) + 64c .. +64) for c < C(s).
// Per tile: S = Q K^T (tcgen05.mma, M=128, N=64, K=128, fp32 in TMEM) ->
// registers (tcgen05.ld) -> online softmax in the exp2 domain with a lazy
// rescale (the running max is only moved when a row's max grows by more than
// 2^8, which keeps the result exact: every term and the normaliser share the
// same reference) -> P (bf16, 128-byte-swizzled shared memory) ->
// O += P V (tcgen05.mma, M=128, N=128, K=64, fp32 in TMEM).
// Loads are 16-byte cp.async row gathers into 128-byte-swizzled shared
// memory; K is single-buffered (refilled once S of the tile is done), V is
// double-buffered (refilled once the previous P V is done).
// Two CTAs fit on an SM (97 KB shared memory, 256 TMEM columns each), so one
// CTA's softmax overlaps the other's MMAs.
#pragma once
#include "s2o_common.cuh"

namespace s2o {

constexpr int kKT = 64;                // keys per tile
constexpr int kAttnThreads = 128;
constexpr uint32_t kQBytes = 2 * 128 * 128;   // 2 atoms x 128 rows x 128 B
constexpr uint32_t kKVBytes = 2 * kKT * 128;  // 2 atoms x 64 rows x 128 B
constexpr uint32_t kPBytes = 128 * 128;       // 1 atom x 128 rows x 128 B
constexpr uint32_t kOffQ = 0;
constexpr uint32_t kOffK = kOffQ + kQBytes;
constexpr uint32_t kOffV0 = kOffK + kKVBytes;
constexpr uint32_t kOffV1 = kOffV0 + kKVBytes;
constexpr uint32_t kOffP = kOffV1 + kKVBytes;
constexpr uint32_t kOffBar = kOffP + kPBytes;  // 2 mbarriers + TMEM slot
constexpr uint32_t kAttnSmemData = kOffBar + 64;
constexpr size_t kAttnSmem = kAttnSmemData + 1024;  // + alignment slack
constexpr uint32_t kTmemCols = 256;                 // S: cols [0,64), O: cols [128,256)
constexpr uint32_t kColS = 0, kColO = 128;

struct AttnArgs {
  const uint16_t* Q;
  const uint16_t* K;
  const uint16_t* V;
  const int32_t* perm;
  const int32_t* nblocks;
  void* O;
  int B, Hq, Hkv, N, S;
  int64_t T;
  int out_f32;
};

// Tile geometry of one work item.
struct TileList {
  int n_diag, n_prev, n_sink, n_cand, total;
};

__device__ __forceinline__ TileList make_tiles(int s, int N, int C) {
  TileList tl;
  const int rows = min(N, kLq * s + kLq) - kLq * s;
  tl.n_diag = (rows + kKT - 1) / kKT;
  tl.n_prev = (s >= 1) ? 2 : 0;
  tl.n_sink = (s >= 2) ? 1 : 0;
  tl.n_cand = C;
  tl.total = tl.n_diag + tl.n_prev + tl.n_sink + tl.n_cand;
  return tl;
}

// Key index of row r (0..63) of tile t; `causal` set for the diagonal tiles.
__device__ __forceinline__ int tile_key(const TileList& tl, int t, int r, int s, const int32_t* pseg, int lo,
                                        int hi) {
  if (t < tl.n_diag) return kLq * s + kKT * t + r;
  t -= tl.n_diag;
  if (t < tl.n_prev) return kLq * s - kLq + kKT * t + r;
  t -= tl.n_prev;
  if (t < tl.n_sink) return r;
  t -= tl.n_sink;
  int j = pseg[kKT * t + r];
  if (j < lo || j >= hi) {  // caller-supplied plan out of Cand(s)
    set_error(kErrBadPlan);
    j = lo;
  }
  return j;
}

// Issue the 16-byte cp.async copies of 64 rows (K or V) of tile t.
// Thread tid copies chunk column c16 = tid % 16 of rows tid/16 + 8k.
__device__ __forceinline__ void load_kv_tile(uint32_t dst, const uint16_t* src_head, const TileList& tl, int t,
                                             int s, int N, const int32_t* pseg, int lo, int hi) {
  const int tid = threadIdx.x;
  const int c16 = tid & 15;
  const uint32_t atom = (uint32_t)(c16 >> 3) * (kKT * 128);
  const uint32_t chunk = (uint32_t)(c16 & 7);
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const int r = (tid >> 4) + 8 * k;
    const int j = tile_key(tl, t, r, s, pseg, lo, hi);
    const bool ok = j < N;
    const uint16_t* src = src_head + (size_t)(ok ? j : 0) * kD + 8 * c16;
    cp_async16(dst + atom + swz128((uint32_t)r, chunk), src, ok ? 16u : 0u);
  }
}

__global__ void __launch_bounds__(kAttnThreads, 2) k_sparse_attn(AttnArgs a) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t sbase = (smem_u32(smem_raw) + 1023u) & ~1023u;
  uint8_t* sgen = smem_raw + (sbase - smem_u32(smem_raw));
  const uint32_t sQ = sbase + kOffQ, sK = sbase + kOffK, sP = sbase + kOffP;
  const uint32_t sV[2] = {sbase + kOffV0, sbase + kOffV1};
  const uint32_t bar_s = sbase + kOffBar, bar_o = sbase + kOffBar + 8;
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(sgen + kOffBar + 16);

  const int tid = threadIdx.x, warp = tid >> 5;
  const int G = a.Hq / a.Hkv;
  const int w = blockIdx.x;
  const int s = a.S - 1 - w / (a.B * a.Hq);
  const int bh = w % (a.B * a.Hq);
  const int b = bh / a.Hq, h = bh % a.Hq, kvh = h / G;
  const int bk = b * a.Hkv + kvh;

  int C = a.nblocks[(size_t)bk * a.S + s];
  const int cmax = (int)(num_cand(s) / kBk);
  if (C < 0 || C > cmax) {
    set_error(kErrBadPlan);
    C = C < 0 ? 0 : cmax;
  }
  const TileList tl = make_tiles(s, a.N, C);
  const int32_t* pseg = a.perm + (size_t)bk * a.T + cand_offset(s);
  const int cand_lo = kSink, cand_hi = kLq * s - kWin;
  const uint16_t* Kh = a.K + (size_t)bk * a.N * kD;
  const uint16_t* Vh = a.V + (size_t)bk * a.N * kD;
  const uint16_t* Qh = a.Q + ((size_t)(b * a.Hq + h) * a.N) * kD;
  const int row0 = kLq * s;

  // --- setup: barriers, TMEM ---------------------------------------------------
  if (tid == 0) {
    mbar_init(bar_s, 1);
    mbar_init(bar_o, 1);
    fence_mbar_init();
  }
  __syncwarp();
  if (warp == 0) {
    tmem_alloc(smem_u32((const void*)tmem_slot), kTmemCols);
    tmem_relinquish();
  }

  // --- prologue loads: Q + K(0) as group 0, V(0) as group 1 --------------------
  {
    const int c16 = tid & 15;
    const uint32_t atom = (uint32_t)(c16 >> 3) * (128 * 128);
    const uint32_t chunk = (uint32_t)(c16 & 7);
#pragma unroll
    for (int k = 0; k < 16; ++k) {
      const int r = (tid >> 4) + 8 * k;
      const bool ok = row0 + r < a.N;
      const uint16_t* src = Qh + (size_t)(ok ? row0 + r : 0) * kD + 8 * c16;
      cp_async16(sQ + atom + swz128((uint32_t)r, chunk), src, ok ? 16u : 0u);
    }
  }
  load_kv_tile(sK, Kh, tl, 0, s, a.N, pseg, cand_lo, cand_hi);
  cp_async_commit();
  load_kv_tile(sV[0], Vh, tl, 0, s, a.N, pseg, cand_lo, cand_hi);
  cp_async_commit();

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
  const uint32_t tS = tmem + kColS + lane_base;
  const uint32_t tO = tmem + kColO + lane_base;

  const uint32_t idesc_qk = idesc_bf16_f32(128, kKT, false);
  const uint32_t idesc_pv = idesc_bf16_f32(128, 128, true);
  const float sl2 = 1.4426950408889634f * 0.08838834764831845f;  // log2(e) / sqrt(d)

  float m_run = -INFINITY;  // running reference max (log2 domain)
  float ell = 0.f;          // running normaliser
  const int row = row0 + tid;
  bool failed = false;

  for (int t = 0; t < tl.total; ++t) {
    // K(t) (and Q) landed; V(t) may still be in flight
    cp_async_wait_group<1>();
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    if (tid == 0) {
      tc_fence_after();
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        const uint64_t ad = sdesc_sw128(sQ + (kk >> 2) * (128 * 128) + (kk & 3) * 32, 16, 1024);
        const uint64_t bd = sdesc_sw128(sK + (kk >> 2) * (kKT * 128) + (kk & 3) * 32, 16, 1024);
        tc_mma_ss(tmem + kColS, ad, bd, idesc_qk, kk > 0 ? 1u : 0u);
      }
      tc_commit(bar_s);
    }
    // wait for S(t)
    bool ok = mbar_wait_bounded(bar_s, (uint32_t)(t & 1));
    if (__syncthreads_or(!ok)) { failed = true; break; }
    tc_fence_after();

    // K buffer is free again: fetch K(t+1)
    if (t + 1 < tl.total) load_kv_tile(sK, Kh, tl, t + 1, s, a.N, pseg, cand_lo, cand_hi);
    cp_async_commit();

    // S(t) -> registers, scaled to the log2 domain, masked
    float x[kKT];
    tmem_ld32(tS, x);
    tmem_ld32(tS + 32, x + 32);
    tc_wait_ld();
    const bool diag = t < tl.n_diag;
    const int j0 = kLq * s + kKT * t;  // meaningful for diagonal tiles only
    float mt = -INFINITY;
#pragma unroll
    for (int c = 0; c < kKT; ++c) {
      float v = x[c] * sl2;
      if (diag && (j0 + c > row)) v = -INFINITY;
      x[c] = v;
      mt = fmaxf(mt, v);
    }
    const bool move = (mt > m_run + 8.f);  // also true on the first visible tile
    float alpha = 1.f;
    if (move) {
      alpha = (m_run == -INFINITY) ? 0.f : ex2_approx(m_run - mt);
      m_run = mt;
      ell *= alpha;
    }
    float rs = 0.f;
    uint32_t pk[kKT / 2];
#pragma unroll
    for (int c = 0; c < kKT; c += 2) {
      const float p0 = (x[c] == -INFINITY) ? 0.f : ex2_approx(x[c] - m_run);
      const float p1 = (x[c + 1] == -INFINITY) ? 0.f : ex2_approx(x[c + 1] - m_run);
      rs += p0 + p1;
      pk[c / 2] = pack_bf16x2(p0, p1);
    }
    ell += rs;

    // previous P V must be done before P, O and V[(t+1)%2] are touched
    if (t > 0) {
      ok = mbar_wait_bounded(bar_o, (uint32_t)((t - 1) & 1));
      if (__syncthreads_or(!ok)) { failed = true; break; }
      tc_fence_after();
    }
    if (t + 1 < tl.total) load_kv_tile(sV[(t + 1) & 1], Vh, tl, t + 1, s, a.N, pseg, cand_lo, cand_hi);
    cp_async_commit();

    // lazy rescale of O (warp-collective TMEM access)
    if (t > 0 && __any_sync(0xffffffffu, move)) {
#pragma unroll
      for (int cc = 0; cc < 128; cc += 32) {
        float o[32];
        tmem_ld32(tO + cc, o);
        tc_wait_ld();
#pragma unroll
        for (int k = 0; k < 32; ++k) o[k] *= alpha;
        tmem_st32(tO + cc, o);
      }
      tc_wait_st();
    }

    // P (row tid, 64 keys) into the swizzled A-operand tile
    {
      uint8_t* prow = sgen + kOffP;
#pragma unroll
      for (int ch = 0; ch < 8; ++ch) {
        uint4 v = make_uint4(pk[4 * ch], pk[4 * ch + 1], pk[4 * ch + 2], pk[4 * ch + 3]);
        *reinterpret_cast<uint4*>(prow + swz128((uint32_t)tid, (uint32_t)ch)) = v;
      }
    }
    // V(t) landed (groups after it: K(t+1), V(t+1))
    cp_async_wait_group<2>();
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    if (tid == 0) {
      tc_fence_after();
      const uint32_t vb = sV[t & 1];
#pragma unroll
      for (int kk = 0; kk < kKT / 16; ++kk) {
        const uint64_t ad = sdesc_sw128(sP + kk * 32, 16, 1024);
        const uint64_t bd = sdesc_sw128(vb + kk * (16 * 128), kKT * 128, 1024);
        tc_mma_ss(tmem + kColO, ad, bd, idesc_pv, (t > 0 || kk > 0) ? 1u : 0u);
      }
      tc_commit(bar_o);
    }
  }

  if (!failed) {
    const bool ok = mbar_wait_bounded(bar_o, (uint32_t)((tl.total - 1) & 1));
    failed = __syncthreads_or(!ok);
  }
  if (failed) {
    if (tid == 0) set_error(kErrTimeout);
    cp_async_wait_all();
  } else {
    tc_fence_after();
    const float inv = ell > 0.f ? 1.f / ell : 0.f;
    const bool store = row < a.N;
    const size_t orow = ((size_t)(b * a.Hq + h) * a.N + (size_t)(store ? row : 0)) * kD;
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
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace s2o
