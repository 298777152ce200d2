// Kernel (1) on the integer tensor core: the pooled-query scores
//   s_j = qbar . k_j / sqrt(d),   j in [0, e(s))
// (gist.science technical summary, section 1, "Classement par Segment": each
// query segment ranks its historical keys against a representative query)
// as integer dot products of fixed-point digits.
//
// Representation.  A key row k_j (bf16) is written in fixed point against its
// own largest binary exponent E_j: F = round(k * 2^(148 - E_j)), |F| < 2^22,
// which is exact for every element within 2^-14 of the row's largest
// magnitude (bf16 carries 8 significant bits).  A pooled-query row (fp64)
// is written against its own exponent f: G = round(qbar * 2^(28 - f)),
// |G| <= 2^29.  F is split into three signed 8-bit digits and G into four:
//   F = d0 2^16 + d1 2^8 + d2,   G = c0 2^24 + c1 2^16 + c2 2^8 + c3.
// Every digit product P_ab = sum_d c_a[d] d_b[d] is exact on the int8 tensor
// core (int32 accumulation, |P| < 2^21), and
//   sum_d G F = 2^8 (2^32 S0 + 2^24 S1 + 2^16 S2 + 2^8 S3 + S4) + 2^0 P_32,
//   S_t = sum_{a+b=t} P_ab.
// The last product (weight 2^0 against a sum of order 2^58) is left out, so
// each score is Y sqrt(2) 2^(f + E_j - 172) with Y the exact 51-bit integer
// above, rounded once in fp64 and once to fp32.  The difference from the
// exact score is at most
//   2^(f-29) ||k_j||_1 / sqrt(d)        (rounding of qbar to 29 bits)
// + 2^(E_j-149) ||qbar||_1 / sqrt(d)    (elements of k_j below 2^-14 of its max)
// + 2^(f+E_j-156) / sqrt(d)             (the omitted product)
// + half an fp32 ulp,
// about 1e-9 of |qbar| ||k_j|| -- three orders below the 1e-6 band inside
// which the importance order treats two scores as tied.
//
// Kernels:
//   k_kdig   K -> key digits, per 32-key tile already in the tensor core's
//            128B-swizzled K-major layout (3 digit planes x 32 rows x 128 B),
//            and E_j per key;
//   k_qdig   qbar -> query digits (4 planes x 128 B per segment) and f;
//   k_score8 one persistent CTA per SM.  A work unit is (b*Hkv, block of 128
//            segments, run of 128-key windows).  The unit's query digits sit
//            in tensor memory as the A operand (M = 128 segments); each
//            32-key tile of key digits arrives by bulk copy into a 10-stage
//            ring and is the B operand (N = 32).  The 11 digit products of a
//            tile go to five int32 accumulators (one per S_t) in one of two
//            tensor-memory buffers, so the epilogue of a tile overlaps the
//            products of the next.  Warp roles (320 threads): warp 0 copies,
//            one thread of warp 1 issues the MMAs (and warp 1 owns tensor
//            memory), warps 2-9 are the epilogue: thread = segment row = TMEM
//            lane, warps w and w+4 taking the tile's first and last 16 keys.
//            The epilogue rebuilds Y exactly in int64, scales it, stores the
//            candidate scores and keeps the running (max, sum exp) of each
//            (segment, 128-key window), which the two warps of a row merge
//            into part[bk][s][window].
// Every mbarrier wait is bounded; a wait that runs out sets the device error
// word, every role stops taking new work but keeps its barrier schedule, and
// the CTA waits for its started copies and products before freeing tensor
// memory.
#pragma once
#include "s2o_common.cuh"

namespace s2o {

constexpr int kI8TileKeys = 32;                                 // keys per tile (the MMA's N)
constexpr uint32_t kI8Plane = kI8TileKeys * 128;                // one digit plane of a tile: 4 KB
constexpr uint32_t kI8TileBytes = 3 * kI8Plane;                 // three key-digit planes: 12 KB
constexpr uint32_t kI8QRowBytes = 4 * 128;                      // four query-digit planes of one segment
constexpr int kI8Stages = 10;                                   // key-digit ring (also keeps one CTA per SM)
constexpr int kI8Threads = 320;
constexpr uint32_t kI8OffBar = kI8Stages * kI8TileBytes;
constexpr uint32_t kI8OffQexp = kI8OffBar + 256;                // [2][128] int32, by unit parity
constexpr uint32_t kI8OffXw = kI8OffQexp + 2 * 128 * 4;         // [2][128] float2, by window parity
constexpr uint32_t kI8SmemData = kI8OffXw + 2 * 128 * 8;
constexpr size_t kI8Smem = kI8SmemData + 1024;                  // + alignment slack
// barrier slots (8 bytes each)
constexpr int kI8Full = 0;                    // [10] copy landed -> MMA
constexpr int kI8Empty = kI8Stages;           // [10] MMA commit -> copier
constexpr int kI8AccFull = 2 * kI8Stages;     // [2]  MMA commit -> epilogue
constexpr int kI8AccEmpty = kI8AccFull + 2;   // [2]  8 epilogue warps read it -> MMA
constexpr int kI8AFull = kI8AccEmpty + 2;     //      4 epilogue warps stored the unit's query digits -> MMA
constexpr int kI8Drain = kI8AFull + 1;        //      final commit of the MMA issuer
constexpr int kI8SlotTmem = kI8Drain + 1;     //      tensor-memory base address
constexpr int kI8SlotAbort = kI8SlotTmem + 1; //      set once any wait ran out
constexpr int kI8SlotCount = kI8SlotAbort + 1; //     tiles copied / tiles the MMA issuer took
static_assert((kI8SlotCount + 1) * 8 <= 256, "barrier slots overflow their area");
// tensor-memory columns: query digits [0, 128), accumulator buffer b at
// 128 + 160 b, S_t at + 32 t
constexpr uint32_t kI8ColAcc = 128, kI8AccCols = 160;

// kind::i8 instruction descriptor: signed 8-bit A and B, int32 D, both K-major
//   bits 4-5 D format (2 = s32), 7-9 A format (1 = s8), 10-12 B format,
//   bits 17-22 N >> 3, bits 24-28 M >> 4.
__host__ __device__ constexpr uint32_t idesc_s8_s32(int M, int N) {
  return (2u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}
// D[tmem] (+)= A[tmem] * B[smem], kind::i8
__device__ __forceinline__ void tc_mma_ts_i8(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc,
                                             uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n"
      " setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::i8 [%0], [%1], %2, %3, p;\n}\n" ::"r"(d_tmem),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// sign-extended low byte
__device__ __forceinline__ int sbyte(int x) { return (int)(int8_t)(x & 0xFF); }

// fixed point of one bf16 element against the row exponent E (>= 1):
// round(k * 2^(148 - E)), ties away from zero in magnitude
__device__ __forceinline__ int kfixed(uint32_t b, int E) {
  const int ex = (int)((b >> 7) & 0xFFu);
  int m = (int)(b & 0x7Fu);
  int sh;
  if (ex == 0) {
    sh = 15 - E;  // subnormal: no implicit bit, exponent 1
  } else {
    m |= 0x80;
    sh = ex - E + 14;
  }
  int F;
  if (sh >= 0) {
    F = m << sh;  // sh <= 14: F < 2^22
  } else {
    const int r = min(-sh, 9);  // m < 2^8 rounds to 0 from 9 bits down
    F = (m + (1 << (r - 1))) >> r;
  }
  return (b & 0x8000u) ? -F : F;
}

// ---------------------------------------------------------------------------
// key digits: CTA = (32-key tile, b*Hkv), 256 threads; a half-warp owns one
// key row (16 lanes x 8 elements), two rows per pass, two passes.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) k_kdig(const uint16_t* __restrict__ K, uint8_t* __restrict__ kd,
                                             int32_t* __restrict__ kexp, int N) {
  const int tile = blockIdx.x, bk = blockIdx.y, ntiles = gridDim.x;
  const uint16_t* Kb = K + (size_t)bk * N * kD;
  uint8_t* dst = kd + ((size_t)bk * ntiles + tile) * kI8TileBytes;
  bool bad = false;
#pragma unroll
  for (int pass = 0; pass < 2; ++pass) {
    const int r = (threadIdx.x >> 4) + 16 * pass, c = threadIdx.x & 15;
    const int j = tile * kI8TileKeys + r;
    uint4 w = make_uint4(0u, 0u, 0u, 0u);
    if (j < N) w = *reinterpret_cast<const uint4*>(Kb + (size_t)j * kD + 8 * c);
    bad |= bf16x2_nonfinite(w.x) | bf16x2_nonfinite(w.y) | bf16x2_nonfinite(w.z) | bf16x2_nonfinite(w.w);
    const uint32_t u[4] = {w.x, w.y, w.z, w.w};
    uint32_t mb = 0;
#pragma unroll
    for (int k = 0; k < 4; ++k) mb = max(mb, max(u[k] & 0x7FFFu, (u[k] >> 16) & 0x7FFFu));
#pragma unroll
    for (int o = 8; o >= 1; o >>= 1) mb = max(mb, __shfl_xor_sync(0xffffffffu, mb, o));
    const int E = max(1, (int)(mb >> 7));
    uint32_t p[3][2] = {{0u, 0u}, {0u, 0u}, {0u, 0u}};
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const uint32_t bits = (e & 1) ? (u[e >> 1] >> 16) : (u[e >> 1] & 0xFFFFu);
      const int F = kfixed(bits, E);
      const int d2 = sbyte(F);
      const int F1 = (F - d2) >> 8;
      const int d1 = sbyte(F1);
      const int d0 = (F1 - d1) >> 8;
      const int sh = 8 * (e & 3);
      p[0][e >> 2] |= (uint32_t)(d0 & 0xFF) << sh;
      p[1][e >> 2] |= (uint32_t)(d1 & 0xFF) << sh;
      p[2][e >> 2] |= (uint32_t)(d2 & 0xFF) << sh;
    }
    // dims 8c .. 8c+7 are bytes 8c .. 8c+7 of the row: half (c & 1) of
    // 16-byte chunk c >> 1, whose place in the row is chunk XOR (row mod 8)
    const uint32_t off = (uint32_t)r * 128u + ((((uint32_t)c >> 1) ^ ((uint32_t)r & 7u)) << 4) + (((uint32_t)c & 1u) << 3);
#pragma unroll
    for (int b = 0; b < 3; ++b) *reinterpret_cast<uint2*>(dst + b * kI8Plane + off) = make_uint2(p[b][0], p[b][1]);
    if (c == 0) kexp[(size_t)bk * ntiles * kI8TileKeys + j] = E;
  }
  if (bad) set_error(kErrNonFinite);
}

// ---------------------------------------------------------------------------
// query digits: one warp per (b*Hkv, s); lane l owns dims 4l .. 4l+3.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) k_qdig(const double* __restrict__ qbar, uint8_t* __restrict__ qd,
                                             int32_t* __restrict__ qexp, int rows) {
  const int row = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  const double4 q = *reinterpret_cast<const double4*>(qbar + (size_t)row * kD + 4 * lane);
  double mx = fmax(fmax(fabs(q.x), fabs(q.y)), fmax(fabs(q.z), fabs(q.w)));
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) mx = fmax(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  int f = 0;
  if (mx > 0.0) {
    int e;
    frexp(mx, &e);  // mx in [2^(e-1), 2^e)
    f = e - 1;
  }
  const double scale = ldexp(1.0, 28 - f);  // exact: |qbar| < 2^(f+1) maps below 2^29
  const double v[4] = {q.x, q.y, q.z, q.w};
  uint32_t p[4] = {0u, 0u, 0u, 0u};
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const int G = (int)__double2ll_rn(v[e] * scale);
    const int c3 = sbyte(G);
    const int G1 = (G - c3) >> 8;
    const int c2 = sbyte(G1);
    const int G2 = (G1 - c2) >> 8;
    const int c1 = sbyte(G2);
    const int c0 = (G2 - c1) >> 8;
    p[0] |= (uint32_t)(c0 & 0xFF) << (8 * e);
    p[1] |= (uint32_t)(c1 & 0xFF) << (8 * e);
    p[2] |= (uint32_t)(c2 & 0xFF) << (8 * e);
    p[3] |= (uint32_t)(c3 & 0xFF) << (8 * e);
  }
  uint32_t* out = reinterpret_cast<uint32_t*>(qd + (size_t)row * kI8QRowBytes);
#pragma unroll
  for (int a = 0; a < 4; ++a) out[a * 32 + lane] = p[a];
  if (lane == 0) qexp[row] = f;
}

// ---------------------------------------------------------------------------
// work units of k_score8
// ---------------------------------------------------------------------------
struct I8Geom {
  int S, N, nsb, wu, units_per_bk, ntiles;  // ntiles: 32-key tiles per b*Hkv
};
struct I8Unit {
  int bk, sb, t0, t1, w_last;  // tiles [t0, t1); windows up to w_last
};
// segment block sb admits the windows w <= its last segment, i.e. min(S, 128 (sb + 1))
__host__ __device__ __forceinline__ int i8_windows(const I8Geom& g, int sb) { return min(g.S, 128 * (sb + 1)); }
__device__ __forceinline__ I8Unit i8_unit(const I8Geom& g, int u) {
  I8Unit r;
  r.bk = u / g.units_per_bk;
  int rem = u - r.bk * g.units_per_bk;
  int sb = 0;
  for (; sb < g.nsb; ++sb) {
    const int nu = (i8_windows(g, sb) + g.wu - 1) / g.wu;
    if (rem < nu) break;
    rem -= nu;
  }
  r.sb = sb;
  const int w0 = rem * g.wu, w1 = min(i8_windows(g, sb), w0 + g.wu);
  r.t0 = 4 * w0;
  r.t1 = min(4 * w1, g.ntiles);
  r.w_last = w1 - 1;
  return r;
}

__device__ __forceinline__ bool i8_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag) {
  for (uint32_t i = 0; i < kSpinLimit; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((i & 1023u) == 1023u && *abort_flag) return false;
  }
  return false;
}
__device__ __forceinline__ void i8_fail(volatile int* abort_flag) {
  if (!*abort_flag) set_error(kErrTimeout);
  *abort_flag = 1;
}

// ---------------------------------------------------------------------------
// the scorer
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kI8Threads, 1) k_score8(const uint8_t* __restrict__ kd,
                                                         const int32_t* __restrict__ kexp,
                                                         const uint8_t* __restrict__ qd,
                                                         const int32_t* __restrict__ qexp, float* __restrict__ scores,
                                                         float2* __restrict__ part, I8Geom g, int64_t T,
                                                         int total_units) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(sm);
  auto bar = [&](int i) { return sbase + kI8OffBar + 8u * (uint32_t)i; };
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + kI8OffBar + 8 * kI8SlotAbort);
  volatile uint32_t* counts = reinterpret_cast<volatile uint32_t*>(sm + kI8OffBar + 8 * kI8SlotCount);
  int* qexp_s = reinterpret_cast<int*>(sm + kI8OffQexp);
  float2* xw = reinterpret_cast<float2*>(sm + kI8OffXw);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  if (tid == 0) {
    for (int i = 0; i < kI8Stages; ++i) {
      mbar_init(bar(kI8Full + i), 1);
      mbar_init(bar(kI8Empty + i), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar(kI8AccFull + i), 1);
      mbar_init(bar(kI8AccEmpty + i), 8);
    }
    mbar_init(bar(kI8AFull), 4);
    mbar_init(bar(kI8Drain), 1);
    *abort_flag = 0;
    counts[0] = counts[1] = 0u;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(bar(kI8SlotTmem), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(sm + kI8OffBar + 8 * kI8SlotTmem);

  if (warp == 0) {
    // ---- copier ------------------------------------------------------------
    if (lane == 0) {
      uint32_t gi = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < total_units && ok; u += gridDim.x) {
        const I8Unit w = i8_unit(g, u);
        const uint8_t* src = kd + (size_t)w.bk * g.ntiles * kI8TileBytes;
        for (int t = w.t0; t < w.t1; ++t, ++gi) {
          const int st = (int)(gi % kI8Stages);
          if (!i8_wait(bar(kI8Empty + st), ((gi / kI8Stages) & 1u) ^ 1u, abort_flag)) {
            i8_fail(abort_flag);
            ok = false;
            break;
          }
          mbar_expect_tx(bar(kI8Full + st), kI8TileBytes);
          bulk_load(sbase + (uint32_t)st * kI8TileBytes, src + (size_t)t * kI8TileBytes, kI8TileBytes,
                    bar(kI8Full + st));
        }
      }
      counts[0] = gi;
    }
  } else if (warp == 1) {
    // ---- MMA issuer -------------------------------------------------------
    if (lane == 0) {
      const uint32_t idesc = idesc_s8_s32(128, kI8TileKeys);
      uint32_t gc = 0, uc = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < total_units && ok; u += gridDim.x, ++uc) {
        const I8Unit w = i8_unit(g, u);
        if (!i8_wait(bar(kI8AFull), uc & 1u, abort_flag)) {
          i8_fail(abort_flag);
          break;
        }
        tc_fence_after();
        for (int t = w.t0; t < w.t1; ++t, ++gc) {
          const int st = (int)(gc % kI8Stages), buf = (int)(gc & 1u);
          if (!i8_wait(bar(kI8Full + st), (gc / kI8Stages) & 1u, abort_flag) ||
              !i8_wait(bar(kI8AccEmpty + buf), ((gc >> 1) & 1u) ^ 1u, abort_flag)) {
            i8_fail(abort_flag);
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t bstage = sbase + (uint32_t)st * kI8TileBytes;
          const uint32_t dacc = tmem + kI8ColAcc + kI8AccCols * (uint32_t)buf;
          // digit pairs (a, b) by group t = a + b; the first of a group overwrites
#pragma unroll
          for (int t8 = 0; t8 < 5; ++t8) {
#pragma unroll
            for (int a = 0; a < 4; ++a) {
              const int b = t8 - a;
              if (b < 0 || b > 2) continue;
              const bool first = (a == (t8 > 2 ? t8 - 2 : 0));
#pragma unroll
              for (int k = 0; k < 4; ++k) {
                const uint64_t bd = sdesc_sw128(bstage + (uint32_t)b * kI8Plane + 32u * (uint32_t)k, 16, 1024);
                tc_mma_ts_i8(dacc + 32u * (uint32_t)t8, tmem + 32u * (uint32_t)a + 8u * (uint32_t)k, bd, idesc,
                             (first && k == 0) ? 0u : 1u);
              }
            }
          }
          tc_commit(bar(kI8Empty + st));
          tc_commit(bar(kI8AccFull + buf));
        }
      }
      counts[1] = gc;
      tc_commit(bar(kI8Drain));
    }
  } else {
    // ---- epilogue -----------------------------------------------------------
    const int q = warp & 3, h = (warp - 2) >> 2;
    const int row = 32 * q + lane;
    const uint32_t lane_base = (uint32_t)(32 * q) << 16;
    const double kSqrt2 = 1.4142135623730951;  // sqrt(2) rounded to fp64
    uint32_t gc = 0, uc = 0;
    bool ok = true;
    for (int u = blockIdx.x; u < total_units; u += gridDim.x, ++uc) {
      const I8Unit w = i8_unit(g, u);
      const int s = 128 * w.sb + row;
      const bool seg_ok = s < g.S;
      if (h == 0) {
        // the previous unit's products are complete (its last accumulator
        // was waited for), so the query digits can be replaced
        const uint4* src = reinterpret_cast<const uint4*>(qd + ((size_t)w.bk * g.S + (seg_ok ? s : 0)) * kI8QRowBytes);
#pragma unroll
        for (int a = 0; a < 4; ++a) {
          uint32_t r[32];
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            uint4 v = seg_ok ? src[8 * a + c] : make_uint4(0u, 0u, 0u, 0u);
            r[4 * c] = v.x; r[4 * c + 1] = v.y; r[4 * c + 2] = v.z; r[4 * c + 3] = v.w;
          }
          if (ok) tmem_st32(tmem + lane_base + 32u * (uint32_t)a, reinterpret_cast<const float*>(r));
        }
        tc_wait_st();
        qexp_s[(uc & 1u) * 128 + row] = seg_ok ? qexp[(size_t)w.bk * g.S + s] : 0;
        tc_fence_before();
      }
      named_sync(1, 256);
      if (h == 0) {
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(kI8AFull));
      }
      const int f = qexp_s[(uc & 1u) * 128 + row];
      const long long pq_bits = __double_as_longlong(ldexp(kSqrt2, f - 172));
      float* sc_row = scores + (size_t)w.bk * T + (seg_ok ? cand_offset(s) : 0) - kSink;
      float2* part_row = part + ((size_t)w.bk * g.S + (seg_ok ? s : 0)) * g.S;
      const int cand_hi = s * kLq - kWin;
      float m_run = -INFINITY, z_run = 0.f;
      for (int t = w.t0; t < w.t1; ++t, ++gc) {
        const int buf = (int)(gc & 1u);
        uint32_t acc[5][16];
        if (ok) {
          bool got = true;
          if (lane == 0) got = i8_wait(bar(kI8AccFull + buf), (gc >> 1) & 1u, abort_flag);
          got = __shfl_sync(0xffffffffu, got, 0);
          if (!got) {
            if (lane == 0) i8_fail(abort_flag);
            ok = false;
          }
        }
        if (ok) {
          tc_fence_after();
          const uint32_t a0 = tmem + lane_base + kI8ColAcc + kI8AccCols * (uint32_t)buf + 16u * (uint32_t)h;
#pragma unroll
          for (int t8 = 0; t8 < 5; ++t8) tmem_ld16(a0 + 32u * (uint32_t)t8, acc[t8]);
          tc_wait_ld();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(bar(kI8AccEmpty + buf));
          const int jg = kI8TileKeys * t + 16 * h;  // this thread's 16 keys: jg .. jg+15
          const int4* ep = reinterpret_cast<const int4*>(kexp + (size_t)w.bk * g.ntiles * kI8TileKeys + jg);
          int E[16];
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            const int4 e4 = __ldg(ep + c);
            E[4 * c] = e4.x; E[4 * c + 1] = e4.y; E[4 * c + 2] = e4.z; E[4 * c + 3] = e4.w;
          }
          float v[16];
          float mloc = -INFINITY;
          bool bad = false;
#pragma unroll
          for (int c = 0; c < 16; ++c) {
            const int j = jg + c;
            const bool adm = seg_ok && j < g.N && (j >> 7) <= s;
            const int hi = (int)acc[0][c] * 256 + (int)acc[1][c];
            const int mid = (int)acc[2][c] * 256 + (int)acc[3][c];
            const long long Y = (long long)hi * 16777216LL + (long long)mid * 256LL + (long long)(int)acc[4][c];
            // |Y| < 2^51: exact through the 1.5 * 2^52 offset
            const double y = __longlong_as_double(Y + 0x4338000000000000LL) - 6755399441055744.0;
            const double sc = __longlong_as_double(pq_bits + ((long long)E[c] << 52));
            const float x = __double2float_rn(y * sc);
            bad |= adm && !isfinite(x);
            v[c] = adm ? x : -INFINITY;
            mloc = fmaxf(mloc, v[c]);
          }
          if (bad) set_error(kErrNonFinite);
          if (seg_ok && jg >= kSink && jg + 16 <= cand_hi) {
            float4* dst = reinterpret_cast<float4*>(sc_row + jg);
#pragma unroll
            for (int c = 0; c < 4; ++c) dst[c] = make_float4(v[4 * c], v[4 * c + 1], v[4 * c + 2], v[4 * c + 3]);
          }
          if (mloc > -INFINITY) {
            const float mt = fmaxf(m_run, mloc);
            float z = (m_run == -INFINITY) ? 0.f : z_run * exp_shifted(m_run, mt);
#pragma unroll
            for (int c = 0; c < 16; ++c) z += (v[c] > -INFINITY) ? exp_shifted(v[c], mt) : 0.f;
            m_run = mt;
            z_run = z;
          }
        }
        // window end: the two warps of this row merge their halves
        if ((t & 3) == 3 || t == w.t1 - 1) {
          const int win = t >> 2;
          if (h == 1) xw[(win & 1) * 128 + row] = make_float2(m_run, z_run);
          named_sync(2 + q, 64);
          if (h == 0 && ok && seg_ok && win <= s) {
            const float2 o = xw[(win & 1) * 128 + row];
            float m = m_run, z = z_run;
            if (m == -INFINITY) {
              m = o.x;
              z = o.y;
            } else if (o.x > -INFINITY) {
              const float mm = fmaxf(m, o.x);
              z = z * exp_shifted(m, mm) + o.y * exp_shifted(o.x, mm);
              m = mm;
            }
            part_row[win] = make_float2(m, z);
          }
          m_run = -INFINITY;
          z_run = 0.f;
        }
      }
    }
  }

  // ---- wind-down ---------------------------------------------------------
  __syncthreads();
  if (warp == 0 && lane == 0) {
    // copies started but never taken by the MMA issuer (only after a wait
    // ran out): each lands before the CTA ends
    const uint32_t gi = counts[0], gc = counts[1];
    for (uint32_t x = gc; x < gi; ++x)
      if (!mbar_wait_bounded(bar(kI8Full + (int)(x % kI8Stages)), (x / kI8Stages) & 1u)) set_error(kErrTimeout);
  }
  if (warp == 1) {
    if (lane == 0 && !mbar_wait_bounded(bar(kI8Drain), 0)) set_error(kErrTimeout);
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace s2o
