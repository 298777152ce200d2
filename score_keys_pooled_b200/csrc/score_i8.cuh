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
//   k_kdig   K -> key digits, per 96-key tile already in the tensor core's
//            128B-swizzled K-major layout (3 digit planes x 96 rows x 128 B),
//            and E_j per key followed by the tile's largest E_j;
//   k_qdig   qbar -> query digits, per block of 128 segments in the same
//            layout (4 planes x 128 rows x 128 B), and f per segment;
//   k_score8 one persistent CTA per SM.  A work unit is (b*Hkv, block of 128
//            segments, run of 96-key tiles).  The unit's query digits are the
//            A operand (M = 128 segments, shared memory); each tile of key
//            digits is the B operand (N = 96; a 128 x 32-byte int8 product
//            costs the tensor core max(48, N/2) cycles, so N = 96 is the
//            narrowest tile at full rate).  The 11 digit products of a tile go
//            to five int32 accumulators S_t (5 x 96 of the 512 tensor-memory
//            columns); each accumulator has its own full/empty barrier pair,
//            so the products of the next tile overwrite S_t as soon as the
//            epilogue has read it.  Warp roles (576 threads): warp 0 copies
//            (bulk copies of the unit's query digits, of each key-digit tile
//            into a 3-stage ring and of its exponents into a 4-slot ring),
//            one thread of warp 1 issues the MMAs (warp 1 owns tensor
//            memory), warps 2-17 are the epilogue: thread = segment row =
//            TMEM lane, the four warps of a lane quarter taking 24 keys of the
//            tile each.  The epilogue rebuilds Y exactly in int64, scales it,
//            stores the candidate scores and forms (max, sum exp) of each
//            (segment, tile), which the four warps of a row merge into
//            part[bk][s][tile].
// Every mbarrier wait is bounded; a wait that runs out sets the device error
// word, every role stops taking new work but keeps its barrier schedule, and
// the CTA waits for its started copies and products before freeing tensor
// memory.
#pragma once
#include "s2o_common.cuh"

namespace s2o {

constexpr int kI8TileKeys = 96;                                 // keys per tile (the MMA's N)
constexpr uint32_t kI8Plane = kI8TileKeys * 128;                // one key-digit plane of a tile: 12 KB
constexpr uint32_t kI8TileBytes = 3 * kI8Plane;                 // three key-digit planes: 36 KB
constexpr uint32_t kI8QPlane = 128 * 128;                       // one query-digit plane of a segment block
constexpr uint32_t kI8QBytes = 4 * kI8QPlane;                   // four planes: 64 KB
constexpr int kI8ExpRec = kI8TileKeys + 4;                     // a tile's exponents, then their max, 3 zeros
constexpr uint32_t kI8ExpBytes = kI8ExpRec * 4;
constexpr int kI8Stages = 3;                                    // key-digit ring
constexpr int kI8ESlots = 4;                                    // exponent ring
constexpr int kI8EpiWarps = 16;                                 // 4 lane quarters x 4 column groups
constexpr int kI8ColsPer = kI8TileKeys / 4;                     // keys of a tile per epilogue warp: 24
constexpr int kI8Threads = 32 * (2 + kI8EpiWarps);
constexpr uint32_t kI8OffA = 0;
constexpr uint32_t kI8OffB = kI8QBytes;
constexpr uint32_t kI8OffE = kI8OffB + kI8Stages * kI8TileBytes;
constexpr uint32_t kI8OffBar = kI8OffE + kI8ESlots * kI8ExpBytes;
constexpr uint32_t kI8OffXw = kI8OffBar + 256;                  // [2][3][128] float2, by tile parity
constexpr uint32_t kI8SmemData = kI8OffXw + 2 * 3 * 128 * 8;
constexpr size_t kI8Smem = kI8SmemData + 1024;                  // + alignment slack
// barrier slots (8 bytes each)
constexpr int kI8BFull = 0;                       // [3] key-digit copy landed -> MMA
constexpr int kI8BEmpty = kI8BFull + kI8Stages;   // [3] MMA commit -> copier
constexpr int kI8EFull = kI8BEmpty + kI8Stages;   // [4] exponent copy landed -> epilogue
constexpr int kI8EEmpty = kI8EFull + kI8ESlots;   // [4] 16 epilogue warps read it -> copier
constexpr int kI8AFull = kI8EEmpty + kI8ESlots;   //     query-digit copy landed -> MMA
constexpr int kI8AEmpty = kI8AFull + 1;           //     MMA commit after a unit's last product -> copier
constexpr int kI8AccFull = kI8AEmpty + 1;         // [5] MMA commit (S_t written) -> epilogue
constexpr int kI8AccEmpty = kI8AccFull + 5;       // [5] 16 epilogue warps read S_t -> MMA
constexpr int kI8Drain = kI8AccEmpty + 5;         //     final commit of the MMA issuer
constexpr int kI8SlotTmem = kI8Drain + 1;         //     tensor-memory base address
constexpr int kI8SlotAbort = kI8SlotTmem + 1;     //     set once any wait ran out
static_assert((kI8SlotAbort + 1) * 8 <= 256, "barrier slots overflow their area");
static_assert(kI8SmemData + 1024 <= 227 * 1024, "shared memory over the per-CTA limit");

// kind::i8 instruction descriptor: signed 8-bit A and B, int32 D, both K-major
//   bits 4-5 D format (2 = s32), 7-9 A format (1 = s8), 10-12 B format,
//   bits 17-22 N >> 3, bits 24-28 M >> 4.
__host__ __device__ constexpr uint32_t idesc_s8_s32(int M, int N) {
  return (2u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}
// D[tmem] (+)= A[smem] * B[smem], kind::i8
__device__ __forceinline__ void tc_mma_ss_i8(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                             uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n"
      " setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n}\n" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

constexpr float kLog2e = 1.4426950408889634f;

// a * b + c with a 64-bit product and addend
__device__ __forceinline__ long long mad_wide(int a, int b, long long c) {
  long long d;
  asm("mad.wide.s32 %0, %1, %2, %3;" : "=l"(d) : "r"(a), "r"(b), "l"(c));
  return d;
}

// 12 consecutive accumulator columns of this warp's lanes
__device__ __forceinline__ void tmem_ld12(uint32_t taddr, uint32_t* r) {
  tmem_ld8(taddr, r);
  tmem_ld4(taddr + 8, r + 8);
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
// key digits: CTA = (96-key tile, b*Hkv), 256 threads; a half-warp owns one
// key row (16 lanes x 8 elements), sixteen rows per pass, six passes.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) k_kdig(const uint16_t* __restrict__ K, uint8_t* __restrict__ kd,
                                             int32_t* __restrict__ kexp, int N) {
  const int tile = blockIdx.x, bk = blockIdx.y, ntiles = gridDim.x;
  const uint16_t* Kb = K + (size_t)bk * N * kD;
  uint8_t* dst = kd + ((size_t)bk * ntiles + tile) * kI8TileBytes;
  int32_t* erec = kexp + ((size_t)bk * ntiles + tile) * kI8ExpRec;
  __shared__ int emax_s;
  if (threadIdx.x == 0) emax_s = 1;
  __syncthreads();
  bool bad = false;
#pragma unroll 2
  for (int pass = 0; pass < kI8TileKeys / 16; ++pass) {
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
    if (c == 0) {
      erec[r] = E;
      atomicMax(&emax_s, E);
    }
  }
  __syncthreads();
  if (threadIdx.x < 4) erec[kI8TileKeys + threadIdx.x] = threadIdx.x == 0 ? emax_s : 0;
  if (bad) set_error(kErrNonFinite);
}

// ---------------------------------------------------------------------------
// query digits: one warp per (b*Hkv, segment row of a 128-segment block);
// lane l owns dims 4l .. 4l+3.  Rows past S get zero digits.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) k_qdig(const double* __restrict__ qbar, uint8_t* __restrict__ qd,
                                             int32_t* __restrict__ qexp, int BH, int S, int nsb) {
  const int gw = (int)(((unsigned long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5);
  const int lane = threadIdx.x & 31;
  if (gw >= BH * nsb * 128) return;
  const int bk = gw / (nsb * 128), rem = gw - bk * nsb * 128;
  const int sb = rem >> 7, r = rem & 127, s = rem;
  double4 q = make_double4(0.0, 0.0, 0.0, 0.0);
  if (s < S) q = *reinterpret_cast<const double4*>(qbar + ((size_t)bk * S + s) * kD + 4 * lane);
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
  // dims 4l .. 4l+3: bytes 4 (l & 3) of 16-byte chunk l >> 2, swizzled by row
  uint8_t* blk = qd + ((size_t)bk * nsb + sb) * kI8QBytes;
  const uint32_t off = (uint32_t)r * 128u + ((((uint32_t)lane >> 2) ^ ((uint32_t)r & 7u)) << 4) + (((uint32_t)lane & 3u) << 2);
#pragma unroll
  for (int a = 0; a < 4; ++a) *reinterpret_cast<uint32_t*>(blk + a * kI8QPlane + off) = p[a];
  if (lane == 0 && s < S) qexp[(size_t)bk * S + s] = f;
}

// ---------------------------------------------------------------------------
// work units of k_score8
// ---------------------------------------------------------------------------
struct I8Geom {
  int S, N, nsb, wu, units_per_bk, ntiles;  // ntiles: 96-key tiles per b*Hkv (also the row stride of part)
};
struct I8Unit {
  int bk, sb, t0, t1;  // tiles [t0, t1) of segment block sb
};
// segment block sb admits the keys below min(N, 128 * 128 (sb + 1))
__host__ __device__ __forceinline__ int i8_tiles(const I8Geom& g, int sb) {
  return (min(g.N, kLq * 128 * (sb + 1)) + kI8TileKeys - 1) / kI8TileKeys;
}
__device__ __forceinline__ I8Unit i8_unit(const I8Geom& g, int u) {
  I8Unit r;
  r.bk = u / g.units_per_bk;
  int rem = u - r.bk * g.units_per_bk;
  int sb = 0;
  for (; sb < g.nsb; ++sb) {
    const int nu = (i8_tiles(g, sb) + g.wu - 1) / g.wu;
    if (rem < nu) break;
    rem -= nu;
  }
  r.sb = sb;
  r.t0 = rem * g.wu;
  r.t1 = min(i8_tiles(g, sb), r.t0 + g.wu);
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
// warp-uniform wait: lane 0 polls, the others take its answer
__device__ __forceinline__ bool i8_warp_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag, int lane) {
  bool got = true;
  if (lane == 0) {
    got = i8_wait(bar, parity, abort_flag);
    if (!got) i8_fail(abort_flag);
  }
  return __shfl_sync(0xffffffffu, got, 0);
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
  float2* xw = reinterpret_cast<float2*>(sm + kI8OffXw);
  const int32_t* es = reinterpret_cast<const int32_t*>(sm + kI8OffE);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  if (tid == 0) {
    for (int i = 0; i < kI8Stages; ++i) {
      mbar_init(bar(kI8BFull + i), 1);
      mbar_init(bar(kI8BEmpty + i), 1);
    }
    for (int i = 0; i < kI8ESlots; ++i) {
      mbar_init(bar(kI8EFull + i), 1);
      mbar_init(bar(kI8EEmpty + i), kI8EpiWarps);
    }
    mbar_init(bar(kI8AFull), 1);
    mbar_init(bar(kI8AEmpty), 1);
    for (int i = 0; i < 5; ++i) {
      mbar_init(bar(kI8AccFull + i), 1);
      mbar_init(bar(kI8AccEmpty + i), kI8EpiWarps);
    }
    mbar_init(bar(kI8Drain), 1);
    *abort_flag = 0;
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
      uint32_t gb = 0, ge = 0, na = 0;  // copies started: key tiles, exponent tiles, query digits
      bool ok = true;
      for (int u = blockIdx.x; u < total_units && ok; u += gridDim.x) {
        const I8Unit w = i8_unit(g, u);
        const uint8_t* src = kd + (size_t)w.bk * g.ntiles * kI8TileBytes;
        const int32_t* esrc = kexp + (size_t)w.bk * g.ntiles * kI8ExpRec;
        const int t_a = min(w.t0 + kI8Stages - 1, w.t1 - 1);  // the query digits follow this tile's copy
        for (int t = w.t0; t < w.t1; ++t, ++gb, ++ge) {
          const int st = (int)(gb % kI8Stages), es_slot = (int)(ge % kI8ESlots);
          if (!i8_wait(bar(kI8BEmpty + st), ((gb / kI8Stages) & 1u) ^ 1u, abort_flag) ||
              !i8_wait(bar(kI8EEmpty + es_slot), ((ge / kI8ESlots) & 1u) ^ 1u, abort_flag)) {
            i8_fail(abort_flag);
            ok = false;
            break;
          }
          mbar_expect_tx(bar(kI8BFull + st), kI8TileBytes);
          bulk_load(sbase + kI8OffB + (uint32_t)st * kI8TileBytes, src + (size_t)t * kI8TileBytes, kI8TileBytes,
                    bar(kI8BFull + st));
          mbar_expect_tx(bar(kI8EFull + es_slot), kI8ExpBytes);
          bulk_load(sbase + kI8OffE + (uint32_t)es_slot * kI8ExpBytes, esrc + (size_t)t * kI8ExpRec, kI8ExpBytes,
                    bar(kI8EFull + es_slot));
          if (t == t_a) {
            // the previous unit's products are done with the query digits;
            // the first key tiles of this unit are already on their way
            if (!i8_wait(bar(kI8AEmpty), (na & 1u) ^ 1u, abort_flag)) {
              i8_fail(abort_flag);
              ok = false;
              ++gb, ++ge;
              break;
            }
            mbar_expect_tx(bar(kI8AFull), kI8QBytes);
            bulk_load(sbase + kI8OffA, qd + ((size_t)w.bk * g.nsb + w.sb) * kI8QBytes, kI8QBytes, bar(kI8AFull));
            ++na;
          }
        }
        if (!ok) break;
      }
      // every copy started lands before the CTA ends: the last one into each
      // slot is waited for (earlier ones landed before it was started)
      for (uint32_t x = (gb > kI8Stages ? gb - kI8Stages : 0); x < gb; ++x)
        if (!mbar_wait_bounded(bar(kI8BFull + (int)(x % kI8Stages)), (x / kI8Stages) & 1u)) set_error(kErrTimeout);
      for (uint32_t x = (ge > kI8ESlots ? ge - kI8ESlots : 0); x < ge; ++x)
        if (!mbar_wait_bounded(bar(kI8EFull + (int)(x % kI8ESlots)), (x / kI8ESlots) & 1u)) set_error(kErrTimeout);
      if (na > 0 && !mbar_wait_bounded(bar(kI8AFull), (na - 1) & 1u)) set_error(kErrTimeout);
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
        for (int t = w.t0; t < w.t1 && ok; ++t, ++gc) {
          const int st = (int)(gc % kI8Stages);
          if (!i8_wait(bar(kI8BFull + st), (gc / kI8Stages) & 1u, abort_flag)) {
            i8_fail(abort_flag);
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t bstage = sbase + kI8OffB + (uint32_t)st * kI8TileBytes;
#pragma unroll
          for (int t8 = 0; t8 < 5; ++t8) {
            // S_t of the previous tile has been read
            if (!i8_wait(bar(kI8AccEmpty + t8), (gc & 1u) ^ 1u, abort_flag)) {
              i8_fail(abort_flag);
              ok = false;
              break;
            }
            tc_fence_after();
            // digit pairs (a, b) with a + b = t8; the first one overwrites
#pragma unroll
            for (int a = 0; a < 4; ++a) {
              const int b = t8 - a;
              if (b < 0 || b > 2) continue;
              const bool first = (a == (t8 > 2 ? t8 - 2 : 0));
#pragma unroll
              for (int k = 0; k < 4; ++k) {
                const uint64_t ad = sdesc_sw128(sbase + kI8OffA + (uint32_t)a * kI8QPlane + 32u * (uint32_t)k, 16, 1024);
                const uint64_t bd = sdesc_sw128(bstage + (uint32_t)b * kI8Plane + 32u * (uint32_t)k, 16, 1024);
                tc_mma_ss_i8(tmem + (uint32_t)(kI8TileKeys * t8), ad, bd, idesc, (first && k == 0) ? 0u : 1u);
              }
            }
            tc_commit(bar(kI8AccFull + t8));
          }
          if (!ok) break;
          tc_commit(bar(kI8BEmpty + st));
        }
        tc_commit(bar(kI8AEmpty));
      }
      tc_commit(bar(kI8Drain));
    }
  } else {
    // ---- epilogue -----------------------------------------------------------
    const int q = warp & 3, h = (warp - 2) >> 2;  // lane quarter; column group (24 keys of a tile)
    const int row = 32 * q + lane;
    const uint32_t lane_base = (uint32_t)(32 * q) << 16;
    const double kSqrt2 = 1.4142135623730951;  // sqrt(2) rounded to fp64
    uint32_t gc = 0;
    bool ok = true;
    for (int u = blockIdx.x; u < total_units; u += gridDim.x) {
      const I8Unit w = i8_unit(g, u);
      const int s = 128 * w.sb + row;
      const bool seg_ok = s < g.S;
      const int f = seg_ok ? __ldg(qexp + (size_t)w.bk * g.S + s) : 0;
      const double pq = ldexp(kSqrt2, f - 172);
      const int pq_hi = __double2hiint(pq), pq_lo = __double2loint(pq);
      const size_t cand_base = (size_t)w.bk * T + (seg_ok ? cand_offset(s) : 0);  // + j - 64 for candidate j
      float2* part_row = part + ((size_t)w.bk * g.S + (seg_ok ? s : 0)) * g.ntiles;
      const int cand_hi = s * kLq - kWin;
      const int e_end = seg_ok ? min(g.N, kLq * (s + 1)) : 0;  // admissible keys: j < e_end
      for (int t = w.t0; t < w.t1; ++t, ++gc) {
        const int jg = kI8TileKeys * t + kI8ColsPer * h;  // this thread's keys: jg .. jg+23
        float m = -INFINITY, z = 0.f;
        if (ok) {
          const uint32_t a0 = tmem + lane_base + kI8ColsPer * (uint32_t)h;
          // accumulators are read in halves of 12 columns, which keeps at most
          // hi, mid and half of S4 (60 values) live
          int hi[kI8ColsPer], mid[kI8ColsPer];
          uint32_t x0[12], x1[12];
          // S0, S1 -> hi = 256 S0 + S1
          ok = i8_warp_wait(bar(kI8AccFull + 0), gc & 1u, abort_flag, lane) &&
               i8_warp_wait(bar(kI8AccFull + 1), gc & 1u, abort_flag, lane);
          if (ok) {
            tc_fence_after();
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
              tmem_ld12(a0 + 12 * hf, x0);
              tmem_ld12(a0 + kI8TileKeys + 12 * hf, x1);
              tc_wait_ld();
#pragma unroll
              for (int c = 0; c < 12; ++c) hi[12 * hf + c] = (int)x0[c] * 256 + (int)x1[c];
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
              mbar_arrive(bar(kI8AccEmpty + 0));
              mbar_arrive(bar(kI8AccEmpty + 1));
            }
            // S2, S3 -> mid = 256 S2 + S3
            ok = i8_warp_wait(bar(kI8AccFull + 2), gc & 1u, abort_flag, lane) &&
                 i8_warp_wait(bar(kI8AccFull + 3), gc & 1u, abort_flag, lane);
          }
          if (ok) {
            tc_fence_after();
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
              tmem_ld12(a0 + 2 * kI8TileKeys + 12 * hf, x0);
              tmem_ld12(a0 + 3 * kI8TileKeys + 12 * hf, x1);
              tc_wait_ld();
#pragma unroll
              for (int c = 0; c < 12; ++c) mid[12 * hf + c] = (int)x0[c] * 256 + (int)x1[c];
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
              mbar_arrive(bar(kI8AccEmpty + 2));
              mbar_arrive(bar(kI8AccEmpty + 3));
            }
            ok = i8_warp_wait(bar(kI8AccFull + 4), gc & 1u, abort_flag, lane);
          }
          const int eslot = (int)(gc % kI8ESlots);
          if (ok) ok = i8_warp_wait(bar(kI8EFull + eslot), (gc / kI8ESlots) & 1u, abort_flag, lane);
          if (ok) {
            tc_fence_after();
            const int32_t* erec = es + eslot * kI8ExpRec;
            const int4* e4 = reinterpret_cast<const int4*>(erec + kI8ColsPer * h);
            const int lim = e_end - jg;  // keys jg + c with c < lim are admissible
            // |s| < 2^(51.5 + f + E - 172): only f + E >= 249 can leave the fp32 range
            const bool check = f + erec[kI8TileKeys] >= 249;
            // tiles whose 24 keys are admissible candidates for all 32 rows of
            // the warp take the path without per-key selects and tests
            const bool full = __all_sync(0xffffffffu, lim >= kI8ColsPer && jg >= kSink && jg + kI8ColsPer <= cand_hi);
            float mc[6], zc[6];  // per 4-key chunk (max, sum exp): independent chains
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
              tmem_ld12(a0 + 4 * kI8TileKeys + 12 * hf, x0);  // S4
              tc_wait_ld();
              if (hf == 1) {
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(kI8AccEmpty + 4));
              }
#pragma unroll
              for (int cq = 0; cq < 3; ++cq) {
                const int ch = 3 * hf + cq;
                const int4 ev = e4[ch];
                const int E[4] = {ev.x, ev.y, ev.z, ev.w};
                float v[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                  const int c = 4 * ch + i;
                  const long long Y = mad_wide(hi[c], 1 << 24, mad_wide(mid[c], 256, (long long)(int)x0[4 * cq + i]));
                  // |Y| < 2^51: exact through the 1.5 * 2^52 offset (added to the high word)
                  const double y =
                      __hiloint2double((int)(Y >> 32) + 0x43380000, (int)(uint32_t)Y) - 6755399441055744.0;
                  const double sc = __hiloint2double(pq_hi + (E[i] << 20), pq_lo);  // sqrt(2) 2^(f + E_j - 172)
                  const float x = __double2float_rn(y * sc);
                  v[i] = (full || c < lim) ? x : -INFINITY;
                }
                const int jc = jg + 4 * ch;
                if (full || (seg_ok && jc >= kSink && jc + 4 <= cand_hi))
                  *reinterpret_cast<float4*>(scores + cand_base + (jc - kSink)) = make_float4(v[0], v[1], v[2], v[3]);
                if (check) {
                  bool bad = false;
#pragma unroll
                  for (int i = 0; i < 4; ++i) bad |= (4 * ch + i < lim) && !isfinite(v[i]);
                  if (bad) set_error(kErrNonFinite);
                }
                // exp(x) = 2^(x log2 e) on the special-function unit, x = v - max
                // formed first so a term's error stays near ex2's own where the
                // term matters (|x| small); -inf terms give 0
                mc[ch] = fmaxf(fmax3(v[0], v[1], v[2]), v[3]);
                const float ml = (mc[ch] > -INFINITY) ? mc[ch] : 0.f;
                zc[ch] = (ex2_approx((v[0] - ml) * kLog2e) + ex2_approx((v[1] - ml) * kLog2e)) +
                         (ex2_approx((v[2] - ml) * kLog2e) + ex2_approx((v[3] - ml) * kLog2e));
              }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(kI8EEmpty + eslot));
            m = fmax3(fmax3(mc[0], mc[1], mc[2]), fmax3(mc[3], mc[4], mc[5]), -INFINITY);
            if (m > -INFINITY) {
              z = 0.f;
#pragma unroll
              for (int ch = 0; ch < 6; ++ch) z += zc[ch] * ex2_approx((mc[ch] - m) * kLog2e);  // empty chunk: 0 * 0
            }
          }
        }
        // the four warps of this lane quarter merge their (max, sum exp)
        float2* xs = xw + (t & 1) * (3 * 128);
        if (h > 0) xs[(h - 1) * 128 + row] = make_float2(m, z);
        named_sync(1 + q, 4 * 32);
        if (h == 0 && ok && kI8TileKeys * t < e_end) {
          const float2 o1 = xs[row], o2 = xs[128 + row], o3 = xs[256 + row];
          const float mm = fmaxf(fmax3(m, o1.x, o2.x), o3.x);
          // a partial of max -inf has sum 0; its factor 2^(-inf) = 0
          const float zz = (z * ex2_approx((m - mm) * kLog2e) + o1.y * ex2_approx((o1.x - mm) * kLog2e)) +
                           (o2.y * ex2_approx((o2.x - mm) * kLog2e) + o3.y * ex2_approx((o3.x - mm) * kLog2e));
          part_row[t] = make_float2(mm, zz);
        }
      }
    }
  }

  // ---- wind-down ---------------------------------------------------------
  __syncthreads();
  if (warp == 1) {
    if (lane == 0 && !mbar_wait_bounded(bar(kI8Drain), 0)) set_error(kErrTimeout);
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace s2o
