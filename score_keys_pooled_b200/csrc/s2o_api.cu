// C ABI of the S2O library: argument checks, workspace layout and launches.
// Everything that computes runs in the kernels of pool_score.cuh,
// seg_sort.cuh and sparse_attn.cuh.
#include <cmath>
#include <cstring>
#include <mutex>

#include "s2o.h"
#include "s2o_common.cuh"
#include "pool_score.cuh"
#include "score_i8.cuh"
#include "seg_sort.cuh"
#include "seg_sort2.cuh"
#include "sparse_attn.cuh"
#include "sparse_attn2.cuh"
#include "block_truth.cuh"
#include "qperm.cuh"

using namespace s2o;

// Scratch of s2o_plan_noalloc: the plan's whole workspace lives here, so that
// entry point never allocates.  Every GPU that loads the library holds these
// 32 MiB until the process exits.
constexpr size_t kNoAllocScratchBytes = size_t(32) << 20;
static __device__ __align__(256) unsigned char g_s2o_plan_scratch[kNoAllocScratchBytes];

namespace {

thread_local int32_t t_launches = 0;

constexpr int kMaxN = 1 << 19;  // bounds the S x S partial-statistics table

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline size_t round256(size_t x) { return (x + 255) & ~size_t(255); }

s2o_status check_cfg(const s2o_config* c) {
  if (!c) return S2O_ERR_INVALID_ARG;
  if (c->B <= 0 || c->Hq <= 0 || c->Hkv <= 0 || c->N <= 0 || c->d <= 0) return S2O_ERR_INVALID_ARG;
  if (c->Hq % c->Hkv) return S2O_ERR_INVALID_ARG;
  if (!std::isfinite(c->tau) || c->tau < 0) return S2O_ERR_INVALID_ARG;
  if (c->d != kD || c->Lq != kLq || c->Bk != kBk || c->n_sink != kSink || c->window_prev != kWin)
    return S2O_ERR_UNSUPPORTED_SHAPE;
  if (c->N > kMaxN) return S2O_ERR_UNSUPPORTED_SHAPE;
  if ((int64_t)c->B * c->Hkv > 65535 || (int64_t)c->B * c->Hq > 65535) return S2O_ERR_UNSUPPORTED_SHAPE;
  return S2O_OK;
}

int32_t nseg(const s2o_config* c) { return (c->N + kLq - 1) / kLq; }
int64_t ncand_total(const s2o_config* c) { return cand_offset(nseg(c)); }

struct PlanWs {
  double* qbar;
  float2* part;
  float* segM;
  double* segZ;
  uint32_t *keyA, *keyB, *valA, *valB;
  float* sorted;
  BucketSlot* slots;
  int* mode;
  int* plen;
  float2* range;
  uint8_t* kd;      // key digits, per 32-key tile
  int32_t* kexp;    // row exponent per key (tiles padded to 32 keys)
  uint8_t* qd;      // pooled-query digits, per segment
  int32_t* qexp;    // row exponent per segment
  int64_t nslots;
  size_t bytes;
};

PlanWs plan_layout(const s2o_config* c, void* base) {
  const size_t BH = (size_t)c->B * c->Hkv, S = (size_t)nseg(c), T = (size_t)ncand_total(c);
  PlanWs w{};
  size_t off = 0;
  auto take = [&](size_t bytes) {
    uint8_t* p = static_cast<uint8_t*>(base) + off;
    off += round256(bytes);
    return static_cast<void*>(p);
  };
  w.qbar = static_cast<double*>(take(BH * S * kD * sizeof(double)));
  const size_t ntiles = ((size_t)c->N + kI8TileKeys - 1) / kI8TileKeys;
  const size_t nsb = (S + 127) / 128;
  w.part = static_cast<float2*>(take(BH * S * ntiles * sizeof(float2)));
  w.segM = static_cast<float*>(take(BH * S * sizeof(float)));
  w.segZ = static_cast<double*>(take(BH * S * sizeof(double)));
  w.keyA = static_cast<uint32_t*>(take(BH * T * 4 + 16));
  w.keyB = static_cast<uint32_t*>(take(BH * T * 4 + 16));
  w.valA = static_cast<uint32_t*>(take(BH * T * 4 + 16));
  w.valB = static_cast<uint32_t*>(take(BH * T * 4 + 16));
  w.sorted = static_cast<float*>(take(BH * T * 4 + 16));
  int64_t per_bk = 0;
  for (int s = 0; s < (int)S; ++s) per_bk += bucket_slots(num_cand(s));
  w.nslots = per_bk * (int64_t)BH;
  w.slots = static_cast<BucketSlot*>(take((size_t)w.nslots * sizeof(BucketSlot) + 16));
  w.mode = static_cast<int*>(take(BH * S * sizeof(int)));
  w.plen = static_cast<int*>(take(BH * S * sizeof(int)));
  w.range = static_cast<float2*>(take(BH * S * sizeof(float2)));
  w.kd = static_cast<uint8_t*>(take(BH * ntiles * kI8TileBytes));
  w.kexp = static_cast<int32_t*>(take(BH * ntiles * kI8ExpRec * sizeof(int32_t)));
  w.qd = static_cast<uint8_t*>(take(BH * nsb * kI8QBytes));
  w.qexp = static_cast<int32_t*>(take(BH * S * sizeof(int32_t)));
  w.bytes = off;
  return w;
}

std::once_flag g_attr_once;
cudaError_t g_attr_err = cudaSuccess;

cudaError_t set_kernel_attributes() {
  std::call_once(g_attr_once, [] {
    cudaError_t e = cudaFuncSetAttribute(k_score8, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kI8Smem);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(k_sparse_attn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kAttnSmem);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(k_sparse_attn2<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kAttn2Smem);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(k_sparse_attn2<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kAttn2Smem);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(k_sparse_attn2<false, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)kAttn2Smem);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(k_sparse_attn2<false, true, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)kAttn2Smem);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(k_bucket_sort, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kBucketSmem);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(k_truth_cols, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kTruthSmem);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(k_contig_plan, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)(kContigMaxBlocks * sizeof(unsigned long long)));
    g_attr_err = e;
  });
  return g_attr_err;
}

// Tensor-map encoder of the driver, fetched through the runtime once.
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
std::once_flag g_encode_once;
EncodeTiledFn g_encode = nullptr;

EncodeTiledFn tensor_map_encoder() {
  std::call_once(g_encode_once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<EncodeTiledFn>(fn);
  });
  return g_encode;
}

// [rows, 128] bf16 rows of 256 bytes, boxes of 64 columns x box_rows rows,
// 128-byte swizzle (the layout the tensor-core descriptors expect).
bool encode_rows_map(CUtensorMap* map, const void* base, uint64_t rows, uint32_t box_rows) {
  EncodeTiledFn enc = tensor_map_encoder();
  if (!enc) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)kD, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)kD * 2};
  const cuuint32_t box[2] = {64, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The context current on the calling thread (driver entry point fetched
// through the runtime once).  Per-device state below is tied to the context
// it was made in: after cudaDeviceReset, or with another context current on
// the same device, the module is loaded again at new addresses and old
// streams are gone, so each cache entry remembers its context and is made
// again when the context changes.
using CtxGetCurrentFn = CUresult (*)(CUcontext*);
std::once_flag g_ctx_once;
CtxGetCurrentFn g_ctx_get = nullptr;

CUcontext current_context() {
  std::call_once(g_ctx_once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_ctx_get = reinterpret_cast<CtxGetCurrentFn>(fn);
  });
  CUcontext c = nullptr;
  if (!g_ctx_get || g_ctx_get(&c) != CUDA_SUCCESS) return nullptr;
  return c;
}

// Device address of g_s2o_plan_scratch, looked up once per device and context.
std::mutex g_scratch_mu;
constexpr int kMaxDevices = 64;
void* g_scratch_addr[kMaxDevices] = {};
CUcontext g_scratch_ctx[kMaxDevices] = {};

// Copy streams of s2o_prefill_host (host->device, device->host), created on
// the first call on each device (and context) and kept for the life of that
// context.
std::mutex g_copy_mu;
cudaStream_t g_copy_in[kMaxDevices] = {}, g_copy_out[kMaxDevices] = {};
CUcontext g_copy_ctx[kMaxDevices] = {};
bool copy_streams(cudaStream_t& in, cudaStream_t& out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return false;
  std::lock_guard<std::mutex> lock(g_copy_mu);
  const CUcontext ctx = current_context();
  if (!g_copy_in[dev] || !ctx || ctx != g_copy_ctx[dev]) {
    // streams of an earlier context died with it: make new ones, drop the old handles
    cudaStream_t a = nullptr, b = nullptr;
    if (cudaStreamCreateWithFlags(&a, cudaStreamNonBlocking) != cudaSuccess) return false;
    if (cudaStreamCreateWithFlags(&b, cudaStreamNonBlocking) != cudaSuccess) {
      cudaStreamDestroy(a);
      return false;
    }
    g_copy_in[dev] = a;
    g_copy_out[dev] = b;
    g_copy_ctx[dev] = current_context();
  }
  in = g_copy_in[dev];
  out = g_copy_out[dev];
  return true;
}

s2o_status launch_status() {
  return cudaGetLastError() == cudaSuccess ? S2O_OK : S2O_ERR_CUDA;
}

// Optional per-stage timing (s2o_stage_timing): an event on the caller's
// stream before the first kernel of a call and after each kernel, per host
// thread; s2o_last_stage_times reads the gaps.
constexpr int kMaxStages = 16;
struct StageClock {
  bool on = false;
  cudaEvent_t ev[kMaxStages + 1] = {};
  const char* name[kMaxStages] = {};
  int n = 0;
};
thread_local StageClock t_clock;

void stage_begin(cudaStream_t s) {
  if (!t_clock.on) return;
  t_clock.n = 0;
  cudaEventRecord(t_clock.ev[0], s);
}

void stage_mark(cudaStream_t s, const char* name) {
  if (!t_clock.on || t_clock.n >= kMaxStages) return;
  t_clock.name[t_clock.n] = name;
  cudaEventRecord(t_clock.ev[++t_clock.n], s);
}

}  // namespace

extern "C" {

int32_t s2o_num_segments(const s2o_config* cfg) {
  if (check_cfg(cfg) != S2O_OK) return -1;
  return nseg(cfg);
}

int64_t s2o_num_candidates(const s2o_config* cfg) {
  if (check_cfg(cfg) != S2O_OK) return -1;
  return ncand_total(cfg);
}

int64_t s2o_candidate_offset(const s2o_config* cfg, int32_t s) {
  if (check_cfg(cfg) != S2O_OK || s < 0 || s > nseg(cfg)) return -1;
  return cand_offset(s);
}

s2o_status s2o_plan_workspace_size(const s2o_config* cfg, size_t* bytes) {
  s2o_status st = check_cfg(cfg);
  if (st != S2O_OK) return st;
  if (!bytes) return S2O_ERR_INVALID_ARG;
  *bytes = plan_layout(cfg, nullptr).bytes;
  return S2O_OK;
}

static void launch_plan_core(const s2o_config* cfg, const double* qbar, const uint16_t* K, float* scores,
                             int32_t* perm, int32_t* nblocks, float* seg_stats, const PlanWs& w, cudaStream_t s,
                             int filtered, bool key_digits);

// the plan's launches; `filtered` sorts only the prefix of each segment's
// order that the stop rule can reach
static s2o_status run_plan(const s2o_config* cfg, const uint16_t* Q, const uint16_t* K, float* scores, int32_t* perm,
                    int32_t* nblocks, float* seg_stats, void* workspace, size_t workspace_bytes,
                    s2o_stream_t stream, int filtered) {
  t_launches = 0;
  s2o_status st = check_cfg(cfg);
  if (st != S2O_OK) return st;
  if (!Q || !K || !scores || !perm || !nblocks || !workspace) return S2O_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(scores) || !aligned16(perm) || !aligned16(nblocks) ||
      (seg_stats && !aligned16(seg_stats)) || (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return S2O_ERR_INVALID_ARG;
  const PlanWs w = plan_layout(cfg, workspace);
  if (workspace_bytes < w.bytes) return S2O_ERR_WORKSPACE_TOO_SMALL;
  if (set_kernel_attributes() != cudaSuccess) return S2O_ERR_CUDA;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int S = nseg(cfg);
  const int BH = cfg->B * cfg->Hkv;

  stage_begin(s);
  k_pool<<<dim3(S, BH), 256, 0, s>>>(Q, w.qbar, cfg->Hq, cfg->Hkv, cfg->N, S);
  ++t_launches;
  stage_mark(s, "k_pool");
  launch_plan_core(cfg, w.qbar, K, scores, perm, nblocks, seg_stats, w, s, filtered, true);
  return launch_status();
}

// the plan's stages after the pooled query: scores and (max, sumexp)
// partials, (M, Z), the order (bucketed sort, global fallback), the stop
static void launch_plan_core(const s2o_config* cfg, const double* qbar, const uint16_t* K, float* scores,
                             int32_t* perm, int32_t* nblocks, float* seg_stats, const PlanWs& w, cudaStream_t s,
                             int filtered, bool key_digits) {
  const int S = nseg(cfg);
  const int BH = cfg->B * cfg->Hkv;
  const int64_t T = ncand_total(cfg);
  I8Geom g;
  g.S = S;
  g.N = cfg->N;
  g.nsb = (S + 127) / 128;
  g.ntiles = (cfg->N + kI8TileKeys - 1) / kI8TileKeys;
  if (key_digits) {
    k_kdig<<<dim3(g.ntiles, BH), 256, 0, s>>>(K, w.kd, w.kexp, cfg->N);
    ++t_launches;
    stage_mark(s, "k_kdig");
  }
  k_qdig<<<BH * g.nsb * 16, 256, 0, s>>>(qbar, w.qd, w.qexp, BH, S, g.nsb);  // a warp per segment row
  ++t_launches;
  stage_mark(s, "k_qdig");
  // work units: (b*Hkv, 128-segment block, run of wu 96-key tiles); wu is
  // the largest power of two up to 32 that still gives two units per SM
  int dev = 0, nsm = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
  auto units_for = [&](int wu) {
    int n = 0;
    for (int sb = 0; sb < g.nsb; ++sb) n += (i8_tiles(g, sb) + wu - 1) / wu;
    return n;
  };
  g.wu = 32;
  while (g.wu > 1 && (int64_t)BH * units_for(g.wu) < 2 * nsm) g.wu >>= 1;
  g.units_per_bk = units_for(g.wu);
  const int total_units = BH * g.units_per_bk;
  k_score8<<<min(total_units, nsm), kI8Threads, kI8Smem, s>>>(w.kd, w.kexp, w.qd, w.qexp, scores, w.part, g, T,
                                                              total_units);
  ++t_launches;
  stage_mark(s, "k_score8");
  const int nwarps = BH * S;
  k_seg_stats<kI8TileKeys><<<(nwarps + 7) / 8, 256, 0, s>>>(w.part, w.segM, w.segZ, seg_stats, BH, S,
                                                                      cfg->N, g.ntiles);
  ++t_launches;
  stage_mark(s, "k_seg_stats");
  k_bucket_plan<<<BH * S, kBucketThreads, 0, s>>>(scores, w.sorted, perm, w.slots, w.mode, w.range, w.keyB, w.valB,
                                                   w.segM, w.segZ, w.plen, cfg->tau, filtered, BH, S, T);
  ++t_launches;
  stage_mark(s, "k_bucket_plan");
  if (w.nslots > 0) {
    k_bucket_sort<<<(unsigned)((w.nslots + kSortGroup - 1) / kSortGroup), kSorterThreads, kBucketSmem, s>>>(
        w.keyB, w.valB, w.slots, w.range, w.sorted, perm, w.nslots, S, T);
    ++t_launches;
    stage_mark(s, "k_bucket_sort");
  }
  k_sort<<<BH * S, kSortThreads, 0, s>>>(scores, w.segM, w.segZ, w.keyA, w.keyB, w.valA, w.valB, perm, w.sorted,
                                         w.mode, kModeFallback, BH, S, T);
  ++t_launches;
  stage_mark(s, "k_sort");
  k_mass_stop<<<BH * S, 256, 0, s>>>(w.sorted, w.segM, w.segZ, w.plen, nblocks, BH, S, T, cfg->tau);
  ++t_launches;
  stage_mark(s, "k_mass_stop");
}

s2o_status s2o_plan(const s2o_config* cfg, const uint16_t* Q, const uint16_t* K, float* scores, int32_t* perm,
                    int32_t* nblocks, float* seg_stats, void* workspace, size_t workspace_bytes,
                    s2o_stream_t stream) {
  return run_plan(cfg, Q, K, scores, perm, nblocks, seg_stats, workspace, workspace_bytes, stream, 0);
}

s2o_status s2o_plan_filtered(const s2o_config* cfg, const uint16_t* Q, const uint16_t* K, float* scores,
                             int32_t* perm, int32_t* nblocks, float* seg_stats, void* workspace,
                             size_t workspace_bytes, s2o_stream_t stream) {
  return run_plan(cfg, Q, K, scores, perm, nblocks, seg_stats, workspace, workspace_bytes, stream, 1);
}

s2o_status s2o_plan_qperm_workspace_size(const s2o_config* cfg, size_t* bytes) {
  s2o_status st = check_cfg(cfg);
  if (st != S2O_OK) return st;
  if (!bytes) return S2O_ERR_INVALID_ARG;
  *bytes = plan_layout(cfg, nullptr).bytes + round256((size_t)2 * cfg->B * cfg->Hkv * nseg(cfg) * kD * sizeof(double));
  return S2O_OK;
}

s2o_status s2o_plan_qperm(const s2o_config* cfg, const uint16_t* Q, const uint16_t* K, float* scores, int32_t* perm,
                          int32_t* nblocks, uint8_t* rowsub, void* workspace, size_t workspace_bytes,
                          s2o_stream_t stream) {
  t_launches = 0;
  s2o_status st = check_cfg(cfg);
  if (st != S2O_OK) return st;
  if (!Q || !K || !scores || !perm || !nblocks || !rowsub || !workspace) return S2O_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(scores) || !aligned16(perm) || !aligned16(nblocks) ||
      (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return S2O_ERR_INVALID_ARG;
  size_t need = 0;
  s2o_plan_qperm_workspace_size(cfg, &need);
  if (workspace_bytes < need) return S2O_ERR_WORKSPACE_TOO_SMALL;
  if (set_kernel_attributes() != cudaSuccess) return S2O_ERR_CUDA;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const PlanWs w = plan_layout(cfg, workspace);
  const int S = nseg(cfg);
  const int BH = cfg->B * cfg->Hkv;
  const int64_t T = ncand_total(cfg);
  double* qsub0 = reinterpret_cast<double*>(static_cast<uint8_t*>(workspace) + w.bytes);
  double* qsub1 = qsub0 + (size_t)BH * S * kD;
  k_pool<<<dim3(S, BH), 256, 0, s>>>(Q, w.qbar, cfg->Hq, cfg->Hkv, cfg->N, S);
  ++t_launches;
  k_qperm<<<dim3(S, BH), kLq, 0, s>>>(Q, w.qbar, qsub0, qsub1, rowsub, cfg->Hq, cfg->Hkv, cfg->N, S);
  ++t_launches;
  launch_plan_core(cfg, qsub0, K, scores, perm, nblocks, nullptr, w, s, 1, true);
  launch_plan_core(cfg, qsub1, K, scores + (size_t)BH * T, perm + (size_t)BH * T, nblocks + (size_t)BH * S, nullptr,
                   w, s, 1, false);  // same keys: their digits are already in the workspace
  return launch_status();
}

s2o_status s2o_plan_contiguous(const s2o_config* cfg, const float* scores, const float* seg_stats,
                               const int32_t* nblocks_match, int32_t* perm_out, s2o_stream_t stream) {
  t_launches = 0;
  s2o_status st = check_cfg(cfg);
  if (st != S2O_OK) return st;
  if (!scores || !seg_stats || !nblocks_match || !perm_out) return S2O_ERR_INVALID_ARG;
  if (!aligned16(scores) || !aligned16(seg_stats) || !aligned16(perm_out)) return S2O_ERR_INVALID_ARG;
  if (set_kernel_attributes() != cudaSuccess) return S2O_ERR_CUDA;
  const int S = nseg(cfg);
  const int BH = cfg->B * cfg->Hkv;
  int P = 1;
  while (P < (int)(num_cand(S - 1) / kBk)) P <<= 1;
  if (P > kContigMaxBlocks) return S2O_ERR_UNSUPPORTED_SHAPE;
  (void)nblocks_match;  // the ranking covers every block; attention reads the first nblocks_match
  k_contig_plan<<<BH * S, 1024, P * sizeof(unsigned long long), reinterpret_cast<cudaStream_t>(stream)>>>(
      scores, seg_stats, perm_out, BH, S, ncand_total(cfg));
  ++t_launches;
  return launch_status();
}

static s2o_status run_attention(const s2o_config* cfg, const uint16_t* Q, const uint16_t* K, const uint16_t* V,
                                const int32_t* perm, const int32_t* nblocks, void* O, int32_t out_dtype,
                                s2o_stream_t stream, uint32_t spin);

s2o_status s2o_attention(const s2o_config* cfg, const uint16_t* Q, const uint16_t* K, const uint16_t* V,
                         const int32_t* perm, const int32_t* nblocks, void* O, int32_t out_dtype,
                         s2o_stream_t stream) {
  return run_attention(cfg, Q, K, V, perm, nblocks, O, out_dtype, stream, kSpinLimit);
}

s2o_status s2o_attention_bounded(const s2o_config* cfg, const uint16_t* Q, const uint16_t* K, const uint16_t* V,
                                 const int32_t* perm, const int32_t* nblocks, void* O, int32_t out_dtype,
                                 uint32_t max_polls, s2o_stream_t stream) {
  if (max_polls > kSpinLimit) return S2O_ERR_INVALID_ARG;
  return run_attention(cfg, Q, K, V, perm, nblocks, O, out_dtype, stream, max_polls);
}

static s2o_status run_attention(const s2o_config* cfg, const uint16_t* Q, const uint16_t* K, const uint16_t* V,
                                const int32_t* perm, const int32_t* nblocks, void* O, int32_t out_dtype,
                                s2o_stream_t stream, uint32_t spin) {
  t_launches = 0;
  s2o_status st = check_cfg(cfg);
  if (st != S2O_OK) return st;
  if (!Q || !K || !V || !perm || !nblocks || !O) return S2O_ERR_INVALID_ARG;
  if (out_dtype != S2O_OUT_BF16 && out_dtype != S2O_OUT_F32) return S2O_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O) || !aligned16(perm))
    return S2O_ERR_INVALID_ARG;
  if (set_kernel_attributes() != cudaSuccess) return S2O_ERR_CUDA;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int G = cfg->Hq / cfg->Hkv;
  // row coordinates of the tensor maps are 32-bit
  const bool rows_fit = (int64_t)cfg->B * cfg->Hq * cfg->N < (int64_t)INT32_MAX;
  if (G % 2 == 0 && rows_fit) {
    // two query heads of a KV group per CTA share every gathered K/V tile
    Attn2Args a;
    a.Q = Q; a.K = K; a.V = V; a.perm = perm; a.nblocks = nblocks; a.O = O;
    a.B = cfg->B; a.Hq = cfg->Hq; a.Hkv = cfg->Hkv; a.N = cfg->N; a.S = nseg(cfg);
    a.T = ncand_total(cfg);
    a.out_f32 = out_dtype == S2O_OUT_F32;
    a.tau = 0.f; a.cout = nullptr; a.perm1 = nullptr; a.nblocks1 = nullptr; a.rowsub = nullptr;
    a.spin = spin;
    CUtensorMap tmQ;
    if (!encode_rows_map(&tmQ, Q, (uint64_t)cfg->B * cfg->Hq * cfg->N, 128))
      return S2O_ERR_CUDA;
    const int64_t ncta = (int64_t)cfg->B * cfg->Hkv * a.S * (G / 2);
    k_sparse_attn2<false><<<(unsigned)ncta, kAttn2Threads, kAttn2Smem, s>>>(a, tmQ);
  } else {
    // this kernel's waits always take the default limit
    if (spin != kSpinLimit) return S2O_ERR_UNSUPPORTED_SHAPE;
    AttnArgs a;
    a.Q = Q; a.K = K; a.V = V; a.perm = perm; a.nblocks = nblocks; a.O = O;
    a.B = cfg->B; a.Hq = cfg->Hq; a.Hkv = cfg->Hkv; a.N = cfg->N; a.S = nseg(cfg);
    a.T = ncand_total(cfg);
    a.out_f32 = out_dtype == S2O_OUT_F32;
    const int64_t ncta = (int64_t)cfg->B * cfg->Hq * a.S;
    k_sparse_attn<<<(unsigned)ncta, kAttnThreads, kAttnSmem, s>>>(a);
  }
  ++t_launches;
  return launch_status();
}

s2o_status s2o_attention_online(const s2o_config* cfg, const uint16_t* Q, const uint16_t* K, const uint16_t* V,
                                const int32_t* perm, void* O, int32_t out_dtype, int32_t* nblocks_out,
                                s2o_stream_t stream) {
  t_launches = 0;
  s2o_status st = check_cfg(cfg);
  if (st != S2O_OK) return st;
  if (!Q || !K || !V || !perm || !O || !nblocks_out) return S2O_ERR_INVALID_ARG;
  if (out_dtype != S2O_OUT_BF16 && out_dtype != S2O_OUT_F32) return S2O_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O) || !aligned16(perm) ||
      !aligned16(nblocks_out))
    return S2O_ERR_INVALID_ARG;
  const int G = cfg->Hq / cfg->Hkv;
  // the tile of the rule is the pair of query heads one CTA computes
  if (G % 2 != 0 || (int64_t)cfg->B * cfg->Hq * cfg->N >= (int64_t)INT32_MAX) return S2O_ERR_UNSUPPORTED_SHAPE;
  if (set_kernel_attributes() != cudaSuccess) return S2O_ERR_CUDA;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  Attn2Args a;
  a.Q = Q; a.K = K; a.V = V; a.perm = perm; a.nblocks = nullptr; a.O = O;
  a.B = cfg->B; a.Hq = cfg->Hq; a.Hkv = cfg->Hkv; a.N = cfg->N; a.S = nseg(cfg);
  a.T = ncand_total(cfg);
  a.out_f32 = out_dtype == S2O_OUT_F32;
  a.tau = (float)cfg->tau; a.cout = nblocks_out; a.perm1 = nullptr; a.nblocks1 = nullptr; a.rowsub = nullptr;
  a.spin = kSpinLimit;
  CUtensorMap tmQ;
  if (!encode_rows_map(&tmQ, Q, (uint64_t)cfg->B * cfg->Hq * cfg->N, 128)) return S2O_ERR_CUDA;
  const int64_t ncta = (int64_t)cfg->B * cfg->Hkv * a.S * (G / 2);
  k_sparse_attn2<true><<<(unsigned)ncta, kAttn2Threads, kAttn2Smem, s>>>(a, tmQ);
  ++t_launches;
  return launch_status();
}

s2o_status s2o_block_truth_workspace_size(const s2o_config* cfg, int32_t nsamp, size_t* bytes) {
  s2o_status st = check_cfg(cfg);
  if (st != S2O_OK) return st;
  if (!bytes || nsamp < 1 || nsamp > kTruthMaxSamples) return S2O_ERR_INVALID_ARG;
  *bytes = round256((size_t)nsamp * cfg->B * cfg->Hkv * (size_t)num_cand(nseg(cfg) - 1) * sizeof(float) + 16);
  return S2O_OK;
}

s2o_status s2o_block_truth(const s2o_config* cfg, const uint16_t* Q, const uint16_t* K, const int32_t* perm,
                           const int32_t* nblocks, const int32_t* segments, int32_t nsamp, float* stats, float* mass,
                           void* workspace, size_t workspace_bytes, s2o_stream_t stream) {
  t_launches = 0;
  s2o_status st = check_cfg(cfg);
  if (st != S2O_OK) return st;
  if (!Q || !K || !perm || !nblocks || !segments || !stats || !workspace) return S2O_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(perm) || (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return S2O_ERR_INVALID_ARG;
  size_t need = 0;
  st = s2o_block_truth_workspace_size(cfg, nsamp, &need);
  if (st != S2O_OK) return st;
  if (workspace_bytes < need) return S2O_ERR_WORKSPACE_TOO_SMALL;
  const int S = nseg(cfg);
  TruthSegs segs;
  for (int k = 0; k < nsamp; ++k) {
    if (segments[k] < 0 || segments[k] >= S) return S2O_ERR_INVALID_ARG;
    segs.s[k] = segments[k];
  }
  if (set_kernel_attributes() != cudaSuccess) return S2O_ERR_CUDA;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int64_t cmaxlen = num_cand(S - 1);
  if (cudaMemsetAsync(workspace, 0, need, s) != cudaSuccess) return S2O_ERR_CUDA;
  k_truth_cols<<<dim3(nsamp, cfg->B * cfg->Hq), kTruthThreads, kTruthSmem, s>>>(Q, K, segs,
                                                                              static_cast<float*>(workspace),
                                                                              cfg->Hq, cfg->Hkv, cfg->N, cmaxlen);
  ++t_launches;
  k_truth_stats<<<dim3(nsamp, cfg->B * cfg->Hkv), 256, 0, s>>>(perm, nblocks, segs, static_cast<float*>(workspace),
                                                                stats, mass, cfg->B * cfg->Hkv, S, ncand_total(cfg),
                                                                cmaxlen, (int)(cmaxlen / kBk), (float)cfg->tau);
  ++t_launches;
  return launch_status();
}

s2o_status s2o_attention_qperm(const s2o_config* cfg, const uint16_t* Q, const uint16_t* K, const uint16_t* V,
                               const int32_t* perm, const int32_t* nblocks, const uint8_t* rowsub, void* O,
                               int32_t out_dtype, s2o_stream_t stream) {
  t_launches = 0;
  s2o_status st = check_cfg(cfg);
  if (st != S2O_OK) return st;
  if (!Q || !K || !V || !perm || !nblocks || !rowsub || !O) return S2O_ERR_INVALID_ARG;
  if (out_dtype != S2O_OUT_BF16 && out_dtype != S2O_OUT_F32) return S2O_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O) || !aligned16(perm) || !aligned16(rowsub))
    return S2O_ERR_INVALID_ARG;
  const int G = cfg->Hq / cfg->Hkv;
  if (G % 2 != 0 || (int64_t)cfg->B * cfg->Hq * cfg->N >= (int64_t)INT32_MAX) return S2O_ERR_UNSUPPORTED_SHAPE;
  if (set_kernel_attributes() != cudaSuccess) return S2O_ERR_CUDA;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int64_t T = ncand_total(cfg);
  const size_t BH = (size_t)cfg->B * cfg->Hkv;
  Attn2Args a;
  a.Q = Q; a.K = K; a.V = V; a.perm = perm; a.nblocks = nblocks; a.O = O;
  a.B = cfg->B; a.Hq = cfg->Hq; a.Hkv = cfg->Hkv; a.N = cfg->N; a.S = nseg(cfg);
  a.T = T;
  a.out_f32 = out_dtype == S2O_OUT_F32;
  a.tau = 0.f; a.cout = nullptr;
  a.perm1 = perm + BH * T;
  a.nblocks1 = nblocks + BH * a.S;
  a.rowsub = rowsub;
  a.spin = kSpinLimit;
  CUtensorMap tmQ;
  if (!encode_rows_map(&tmQ, Q, (uint64_t)cfg->B * cfg->Hq * cfg->N, 128)) return S2O_ERR_CUDA;
  if (G % 4 == 0) {
    // every CTA: one sub-segment of a segment, four query heads
    const int64_t ncta = (int64_t)cfg->B * cfg->Hkv * a.S * (G / 4) * 2;
    k_sparse_attn2<false, true, true><<<(unsigned)ncta, kAttn2Threads, kAttn2Smem, s>>>(a, tmQ);
  } else {
    const int64_t ncta = (int64_t)cfg->B * cfg->Hkv * a.S * (G / 2);
    k_sparse_attn2<false, true><<<(unsigned)ncta, kAttn2Threads, kAttn2Smem, s>>>(a, tmQ);
  }
  ++t_launches;
  return launch_status();
}

s2o_status s2o_prefill_arena_size(const s2o_config* cfg, int32_t out_dtype, size_t* bytes) {
  s2o_status st = check_cfg(cfg);
  if (st != S2O_OK) return st;
  if (!bytes || (out_dtype != S2O_OUT_BF16 && out_dtype != S2O_OUT_F32)) return S2O_ERR_INVALID_ARG;
  const size_t q = (size_t)cfg->B * cfg->Hq * cfg->N * kD, kv = (size_t)cfg->B * cfg->Hkv * cfg->N * kD;
  const size_t T = (size_t)cfg->B * cfg->Hkv * ncand_total(cfg), S = (size_t)cfg->B * cfg->Hkv * nseg(cfg);
  size_t ws = 0;
  s2o_plan_workspace_size(cfg, &ws);
  // nblocks: one 16-byte aligned slot of ceil(S/4)*4 entries per (b, kvh)
  const size_t snb = (size_t)cfg->B * cfg->Hkv * (((size_t)nseg(cfg) + 3) & ~(size_t)3);
  *bytes = round256(q * 2) + 2 * round256(kv * 2) + round256(q * (out_dtype == S2O_OUT_F32 ? 4 : 2)) +
           round256(T * 4 + 16) * 2 + round256(snb * 4) + ws;
  (void)S;
  return S2O_OK;
}

s2o_status s2o_prefill_host(const s2o_config* cfg, const uint16_t* Q_host, const uint16_t* K_host,
                            const uint16_t* V_host, void* O_host, int32_t out_dtype, int32_t* nblocks_host,
                            void* arena, size_t arena_bytes, s2o_stream_t stream) {
  s2o_status st = check_cfg(cfg);
  if (st != S2O_OK) return st;
  if (!Q_host || !K_host || !V_host || !O_host || !arena) return S2O_ERR_INVALID_ARG;
  size_t need = 0;
  st = s2o_prefill_arena_size(cfg, out_dtype, &need);
  if (st != S2O_OK) return st;
  if (arena_bytes < need) return S2O_ERR_WORKSPACE_TOO_SMALL;
  if (reinterpret_cast<uintptr_t>(arena) & 255u) return S2O_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const size_t q = (size_t)cfg->B * cfg->Hq * cfg->N * kD, kv = (size_t)cfg->B * cfg->Hkv * cfg->N * kD;
  const size_t T = (size_t)cfg->B * cfg->Hkv * ncand_total(cfg), S = (size_t)cfg->B * cfg->Hkv * nseg(cfg);
  const size_t obytes = q * (out_dtype == S2O_OUT_F32 ? 4 : 2);
  uint8_t* p = static_cast<uint8_t*>(arena);
  uint16_t* dQ = reinterpret_cast<uint16_t*>(p); p += round256(q * 2);
  uint16_t* dK = reinterpret_cast<uint16_t*>(p); p += round256(kv * 2);
  uint16_t* dV = reinterpret_cast<uint16_t*>(p); p += round256(kv * 2);
  void* dO = p; p += round256(obytes);
  float* dscores = reinterpret_cast<float*>(p); p += round256(T * 4 + 16);
  int32_t* dperm = reinterpret_cast<int32_t*>(p); p += round256(T * 4 + 16);
  const size_t Sp = ((size_t)nseg(cfg) + 3) & ~(size_t)3;  // nblocks slot per (b, kvh), 16-byte aligned
  int32_t* dnb = reinterpret_cast<int32_t*>(p); p += round256((size_t)cfg->B * cfg->Hkv * Sp * 4);
  (void)S;
  void* ws = p;
  size_t wsb = 0;
  s2o_plan_workspace_size(cfg, &wsb);

  // One unit = one (b, kvh): its query heads, K and V rows are contiguous in
  // every buffer and its plan and attention depend on nothing else.  Units
  // are copied in on one stream (K and Q first: the plan needs only those),
  // planned and attended on the caller's stream and copied out on a third,
  // so the copies of one unit overlap the kernels of the others.  With an
  // even group size a unit's attention runs one query-head pair at a time
  // (a CTA computes one pair anyway), so the output of one pair goes out
  // while the next is computed.  The kernels see exactly the inputs of a
  // whole-problem call, so the results are the same.
  cudaStream_t s_in = nullptr, s_out = nullptr;
  if (!copy_streams(s_in, s_out)) return S2O_ERR_CUDA;
  const int G = cfg->Hq / cfg->Hkv;
  const int U = cfg->B * cfg->Hkv;
  const int P = G % 2 == 0 ? G / 2 : 1;  // attention launches per unit
  s2o_config sub = *cfg;
  sub.B = 1;
  sub.Hq = G;
  sub.Hkv = 1;
  s2o_config part = sub;
  part.Hq = G / P;
  const size_t qu = (size_t)G * cfg->N * kD, kvu = (size_t)cfg->N * kD, qp = qu / P;
  const size_t Tu = (size_t)ncand_total(cfg), Su = (size_t)nseg(cfg);
  const size_t oelt = out_dtype == S2O_OUT_F32 ? 4 : 2;
  size_t wsu = 0;
  s2o_plan_workspace_size(&sub, &wsu);
  cudaEvent_t ev0 = nullptr;
  const size_t nev = 2 * (size_t)U + (size_t)U * P;  // K+Q in, V in, per-pair out
  cudaEvent_t* ev = new cudaEvent_t[nev]();
  bool cuda_ok = cudaEventCreateWithFlags(&ev0, cudaEventDisableTiming) == cudaSuccess;
  for (size_t e = 0; cuda_ok && e < nev; ++e)
    cuda_ok = cudaEventCreateWithFlags(&ev[e], cudaEventDisableTiming) == cudaSuccess;
  cudaEvent_t* ev_kq = ev;
  cudaEvent_t* ev_v = ev + U;
  cudaEvent_t* ev_o = ev + 2 * U;
  // the copies start after the caller's earlier work on its stream (the
  // arena may still be in use there)
  cuda_ok = cuda_ok && cudaEventRecord(ev0, s) == cudaSuccess && cudaStreamWaitEvent(s_in, ev0, 0) == cudaSuccess &&
            cudaStreamWaitEvent(s_out, ev0, 0) == cudaSuccess;
  for (int u = 0; cuda_ok && u < U; ++u) {
    cuda_ok = cudaMemcpyAsync(dK + u * kvu, K_host + u * kvu, kvu * 2, cudaMemcpyHostToDevice, s_in) == cudaSuccess &&
              cudaMemcpyAsync(dQ + u * qu, Q_host + u * qu, qu * 2, cudaMemcpyHostToDevice, s_in) == cudaSuccess &&
              cudaEventRecord(ev_kq[u], s_in) == cudaSuccess &&
              cudaMemcpyAsync(dV + u * kvu, V_host + u * kvu, kvu * 2, cudaMemcpyHostToDevice, s_in) == cudaSuccess &&
              cudaEventRecord(ev_v[u], s_in) == cudaSuccess;
  }
  int32_t launches = 0;
  for (int u = 0; cuda_ok && st == S2O_OK && u < U; ++u) {
    cuda_ok = cudaStreamWaitEvent(s, ev_kq[u], 0) == cudaSuccess;
    if (!cuda_ok) break;
    st = run_plan(&sub, dQ + u * qu, dK + u * kvu, dscores + u * Tu, dperm + u * Tu, dnb + u * Sp, nullptr, ws, wsu,
                  stream, 1);
    if (st != S2O_OK) break;
    launches += t_launches;
    cuda_ok = cudaStreamWaitEvent(s, ev_v[u], 0) == cudaSuccess;
    for (int p = 0; cuda_ok && st == S2O_OK && p < P; ++p) {
      uint8_t* dOp = static_cast<uint8_t*>(dO) + (u * qu + p * qp) * oelt;
      st = s2o_attention(&part, dQ + u * qu + p * qp, dK + u * kvu, dV + u * kvu, dperm + u * Tu, dnb + u * Sp, dOp,
                         out_dtype, stream);
      if (st != S2O_OK) break;
      launches += t_launches;
      cudaEvent_t e = ev_o[(size_t)u * P + p];
      cuda_ok = cudaEventRecord(e, s) == cudaSuccess && cudaStreamWaitEvent(s_out, e, 0) == cudaSuccess &&
                cudaMemcpyAsync(static_cast<uint8_t*>(O_host) + (u * qu + p * qp) * oelt, dOp, qp * oelt,
                                cudaMemcpyDeviceToHost, s_out) == cudaSuccess;
    }
    if (st != S2O_OK || !cuda_ok) break;
    cuda_ok = !nblocks_host || cudaMemcpyAsync(nblocks_host + u * Su, dnb + u * Sp, Su * 4, cudaMemcpyDeviceToHost,
                                               s_out) == cudaSuccess;
  }
  // every stream drains before the events go and the call returns
  const bool sync_ok = cudaStreamSynchronize(s_in) == cudaSuccess && cudaStreamSynchronize(s_out) == cudaSuccess &&
                       cudaStreamSynchronize(s) == cudaSuccess;
  if (ev0) cudaEventDestroy(ev0);
  for (size_t e = 0; e < nev; ++e)
    if (ev[e]) cudaEventDestroy(ev[e]);
  delete[] ev;
  t_launches = launches;
  if (st != S2O_OK) return st;
  if (!cuda_ok || !sync_ok) return S2O_ERR_CUDA;
  return s2o_last_device_error(stream);
}

s2o_status s2o_plan_noalloc(const s2o_config* cfg, const uint16_t* Q, const uint16_t* K, float* scores,
                            int32_t* perm, int32_t* nblocks, float* seg_stats, s2o_stream_t stream) {
  t_launches = 0;
  s2o_status st = check_cfg(cfg);
  if (st != S2O_OK) return st;
  if (plan_layout(cfg, nullptr).bytes > kNoAllocScratchBytes) return S2O_ERR_WORKSPACE_TOO_SMALL;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return S2O_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return S2O_ERR_UNSUPPORTED_SHAPE;
  void* scratch = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    const CUcontext ctx = current_context();
    if (!g_scratch_addr[dev] || !ctx || ctx != g_scratch_ctx[dev]) {
      // In host code the array's name is only a host-side handle; the device
      // address comes from the runtime, with this device current.  The
      // lookup loads the module into the context if it is not loaded yet.
      void* p = nullptr;
      if (cudaGetSymbolAddress(&p, g_s2o_plan_scratch) != cudaSuccess || !p) return S2O_ERR_CUDA;
      g_scratch_addr[dev] = p;
      g_scratch_ctx[dev] = current_context();
    }
    scratch = g_scratch_addr[dev];
  }
  return s2o_plan(cfg, Q, K, scores, perm, nblocks, seg_stats, scratch, kNoAllocScratchBytes, stream);
}

const char* s2o_status_string(s2o_status st) {
  switch (st) {
    case S2O_OK: return "ok";
    case S2O_ERR_INVALID_ARG: return "invalid argument";
    case S2O_ERR_UNSUPPORTED_SHAPE: return "unsupported shape or constants";
    case S2O_ERR_WORKSPACE_TOO_SMALL: return "workspace too small";
    case S2O_ERR_CUDA: return "CUDA runtime error";
    case S2O_ERR_DEVICE_TIMEOUT: return "bounded device wait ran out";
    case S2O_ERR_NONFINITE: return "non-finite input or score";
    case S2O_ERR_BAD_PLAN: return "plan index out of range";
  }
  return "unknown status";
}

s2o_status s2o_last_device_error(s2o_stream_t stream) {
  if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) return S2O_ERR_CUDA;
  unsigned word = 0;
  if (cudaMemcpyFromSymbol(&word, g_s2o_error, sizeof(word)) != cudaSuccess) return S2O_ERR_CUDA;
  const unsigned zero = 0;
  if (word && cudaMemcpyToSymbol(g_s2o_error, &zero, sizeof(zero)) != cudaSuccess) return S2O_ERR_CUDA;
  if (word & kErrTimeout) return S2O_ERR_DEVICE_TIMEOUT;
  if (word & kErrNonFinite) return S2O_ERR_NONFINITE;
  if (word & kErrBadPlan) return S2O_ERR_BAD_PLAN;
  return S2O_OK;
}

int32_t s2o_last_launch_count(void) { return t_launches; }

s2o_status s2o_stage_timing(int32_t enable) {
  if (enable && !t_clock.on) {
    for (int i = 0; i <= kMaxStages; ++i) {
      if (cudaEventCreate(&t_clock.ev[i]) != cudaSuccess) {
        for (int j = 0; j < i; ++j) cudaEventDestroy(t_clock.ev[j]);
        return S2O_ERR_CUDA;
      }
    }
    t_clock.on = true;
    t_clock.n = 0;
  } else if (!enable && t_clock.on) {
    for (int i = 0; i <= kMaxStages; ++i) cudaEventDestroy(t_clock.ev[i]);
    t_clock.on = false;
    t_clock.n = 0;
  }
  return S2O_OK;
}

int32_t s2o_last_stage_times(float* ms, const char** names, int32_t cap) {
  if (!t_clock.on || cap < 0 || (cap > 0 && !ms)) return -1;
  const int n = t_clock.n;
  if (n > 0 && cudaEventSynchronize(t_clock.ev[n]) != cudaSuccess) return -1;
  for (int i = 0; i < n && i < cap; ++i) {
    if (cudaEventElapsedTime(&ms[i], t_clock.ev[i], t_clock.ev[i + 1]) != cudaSuccess) return -1;
    if (names) names[i] = t_clock.name[i];
  }
  return n;
}

}  // extern "C"
