/*
 * s2o.h -- C ABI of the S2O sparse-prefill library for NVIDIA B200 (sm_100a).
 *
 * S2O ("S2O: Early Stopping for Sparse Attention via Online Permutation",
 * arXiv 2602.22575) splits causal prefill attention into
 *
 *   plan       for every (batch b, KV head kvh, query segment s of Lq rows):
 *              pool the segment's queries into one vector, score every
 *              causally admissible key against it, sort the non-local keys
 *              by score into an index list (the "online permutation": no
 *              K/V data moves), cut the list into blocks of Bk keys and stop
 *              at the first block whose estimated softmax mass is below tau;
 *   attention  exact online-softmax attention of every row of the segment
 *              over the kept keys: sinks, the local window and the kept
 *              blocks, gathered by index.
 *
 * Sources on the pages (no formulas are given there):
 *   - pith.science page, "read the original abstract": index-guided loading
 *     of non-contiguous tokens, blocks from high to low importance, stop once
 *     the current block score falls below a threshold;
 *   - gist.science technical summary, section 1 "Permutation en ligne via
 *     Chargement Guide par Index" (segment ranking, representative query,
 *     causal mask, index arrays over an unchanged HBM layout), section 2
 *     "Regle d'Arret Anticipe" (stop on marginal mass below tau) and section 3
 *     "Implementation du Noyau" (pass 1: dense causal window; pass 2: keys in
 *     permuted order with the early stop).
 *
 * The rule this library fixes where the pages are silent:
 *   qbar(b,kvh,s) = mean of Q[b, kvh*G + g, i, :] over the G = Hq/Hkv heads of
 *                   the group and the rows i of segment s;
 *   s_j           = qbar . k_j / sqrt(d) for j in A(s) = [0, e(s)),
 *                   e(s) = min(N, Lq*(s+1));
 *   always kept   sinks [0, n_sink) and window [max(0, Lq*s - W), e(s));
 *   candidates    Cand(s) = [n_sink, Lq*s - W) (empty when Lq*s - W <= n_sink);
 *   order         candidates by s_j descending, ties to the lower index;
 *   block mass    m_b = sum_{j in block b} exp(s_j - M) / Z, M = max_{A(s)} s_j,
 *                 Z = sum_{A(s)} exp(s_j - M);
 *   stop          C(s) = first b with m_b < tau, else the number of blocks;
 *   attention     O[b,h,i,:] = softmax_j(q_i . k_j / sqrt(d)) V over
 *                 j in Keep(s) intersected with [0, i],
 *                 Keep(s) = sinks U window U perm[0 : Bk*C(s)].
 *
 * Compiled specialisation: Lq = 128, Bk = 64, n_sink = 64, W = 128, d = 128.
 * Other values return S2O_ERR_UNSUPPORTED_SHAPE.  N may be any positive size
 * (the last segment may be partial); with these constants every candidate
 * block is full, |Cand(s)| = max(0, 128 s - 192).
 *
 * Layouts (all row-major, contiguous, device memory unless stated):
 *   Q  [B, Hq,  N, d]  bf16 (raw 16-bit patterns)
 *   K  [B, Hkv, N, d]  bf16
 *   V  [B, Hkv, N, d]  bf16
 *   O  [B, Hq,  N, d]  bf16 or fp32 (out_dtype)
 *   scores [B, Hkv, T] fp32  candidate scores in candidate order: segment s
 *                            occupies [off(s), off(s+1)), entry k is key
 *                            n_sink + k; T = s2o_num_candidates(), off(s) =
 *                            s2o_candidate_offset()
 *   perm   [B, Hkv, T] int32 absolute key indices, same packing; within a
 *                            segment the importance order (full list)
 *   nblocks   [B, Hkv, S] int32  C(s)
 *   seg_stats [B, Hkv, S, 2] fp32  (M, Z), may be NULL
 * Pointers must be 16-byte aligned.  Query head h reads KV head h / (Hq/Hkv).
 *
 * Ownership: the caller allocates every buffer, including the plan workspace
 * (size from s2o_plan_workspace_size).  The library never allocates device
 * memory.  Its only global state per device is a 32-bit device error word
 * (see s2o_last_device_error), the fixed scratch of s2o_plan_noalloc and the
 * two copy streams of s2o_prefill_host (created on its first call).
 *
 * Execution: every call except s2o_prefill_host and s2o_last_device_error is
 * asynchronous on the given stream (NULL = the legacy default stream) and
 * returns after argument checks and kernel launches.  Argument errors are
 * reported before anything is launched; launch failures map to S2O_ERR_CUDA.
 * Errors found on the device (non-finite input, an out-of-range index in a
 * caller-supplied plan, a bounded wait that ran out) set the device error
 * word; outputs of that call are then unspecified.
 */
#ifndef S2O_H
#define S2O_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* s2o_stream_t; /* a cudaStream_t */

typedef struct s2o_config {
  int32_t B, Hq, Hkv, N, d;
  int32_t Lq;          /* query segment length (128) */
  int32_t Bk;          /* keys per block, the stopping granularity (64) */
  int32_t n_sink;      /* always-kept sink tokens [0, n_sink) (64) */
  int32_t window_prev; /* always-kept keys before the segment (128) */
  double tau;          /* stop threshold on block mass, >= 0 */
} s2o_config;

typedef enum s2o_status {
  S2O_OK = 0,
  S2O_ERR_INVALID_ARG = 1,         /* null pointer, bad size, misalignment */
  S2O_ERR_UNSUPPORTED_SHAPE = 2,   /* constants other than the compiled ones */
  S2O_ERR_WORKSPACE_TOO_SMALL = 3,
  S2O_ERR_CUDA = 4,                /* a CUDA runtime call or launch failed */
  S2O_ERR_DEVICE_TIMEOUT = 5,      /* a bounded device wait ran out */
  S2O_ERR_NONFINITE = 6,           /* Inf/NaN in Q or K, or a non-finite score */
  S2O_ERR_BAD_PLAN = 7             /* perm/nblocks out of range in s2o_attention */
} s2o_status;

enum { S2O_OUT_BF16 = 0, S2O_OUT_F32 = 1 };

/* Number of query segments S = ceil(N / Lq).  Returns -1 on a bad config. */
int32_t s2o_num_segments(const s2o_config* cfg);

/* T = sum over segments of |Cand(s)| (per (b, kvh)).  -1 on a bad config. */
int64_t s2o_num_candidates(const s2o_config* cfg);

/* off(s) = sum_{t < s} |Cand(t)|, 0 <= s <= S.  -1 on a bad config or s. */
int64_t s2o_candidate_offset(const s2o_config* cfg, int32_t s);

/* Bytes of device workspace s2o_plan needs for this config. */
s2o_status s2o_plan_workspace_size(const s2o_config* cfg, size_t* bytes);

/*
 * s2o_plan -- pooled scores, importance order and stop point of every
 * segment (the pages' preprocessing / index generation: pith.science
 * abstract; gist.science technical summary, sections 1 and 2).
 *   Q, K       device bf16 inputs (layouts above)
 *   scores     out, device fp32 [B,Hkv,T]
 *   perm       out, device int32 [B,Hkv,T]
 *   nblocks    out, device int32 [B,Hkv,S]
 *   seg_stats  out, device fp32 [B,Hkv,S,2] or NULL
 *   workspace  device scratch of at least s2o_plan_workspace_size() bytes,
 *              256-byte aligned; its contents need no initialisation
 * Accuracy: a score is the exact qbar . k_j / sqrt(d) (qbar the exact mean of
 * the bf16 rows) to within half an fp32 ulp plus
 *   [2^(f-29) |k_j|_1 + 2^(E-149) sum_{d: |k_jd| < 2^(E-141)} |qbar_d|
 *    + 2^(f+E-156)] / sqrt(d),
 * f = floor(log2 max|qbar|), E = the biased bf16 exponent of max|k_j| (at
 * least 1): qbar and k_j are taken in fixed point against their own largest
 * exponents (29 and 22 bits) and multiplied exactly on the integer tensor
 * core; about 1e-9 of |qbar| |k_j|.  The order sorts these fp32 values,
 * ties to the lower key index; M and Z (seg_stats) are formed from them.
 */
s2o_status s2o_plan(const s2o_config* cfg, const uint16_t* Q, const uint16_t* K,
                    float* scores, int32_t* perm, int32_t* nblocks, float* seg_stats,
                    void* workspace, size_t workspace_bytes, s2o_stream_t stream);

/*
 * s2o_plan_filtered -- s2o_plan that sorts only the part of each segment's
 * order the stop rule can reach (the pages describe the preprocessing as very
 * light: pith.science abstract; gist.science technical summary, "Resultats
 * Experimentaux").  A candidate of pooled mass exp(s - M)/Z below tau/Bk
 * cannot lift a block to tau, so with n_hi candidates at or above that level
 * the block starting at Bk*ceil(n_hi/Bk) fails the test and C(s) can be no
 * larger; the rest of the segment is never ordered.
 *   Arguments, layouts, workspace size and errors: as s2o_plan.
 *   Results: scores, seg_stats and nblocks equal s2o_plan's; perm equals
 *   s2o_plan's on the first Bk * nblocks[b,kvh,s] entries of every segment
 *   (all that s2o_attention reads); later entries of a segment are
 *   unspecified (they may hold anything, including stale data).
 *   With tau = 0 every candidate counts and the result is s2o_plan's.
 */
s2o_status s2o_plan_filtered(const s2o_config* cfg, const uint16_t* Q, const uint16_t* K,
                             float* scores, int32_t* perm, int32_t* nblocks, float* seg_stats,
                             void* workspace, size_t workspace_bytes, s2o_stream_t stream);

/*
 * s2o_plan_noalloc -- s2o_plan without a caller-supplied workspace, for
 * callers that may not allocate device memory: plugins inside an engine or
 * framework that owns all device memory through its own pool (a cudaMalloc of
 * theirs would fail or break the pool's accounting), and code on a latency-
 * critical path where cudaMalloc/cudaFree would synchronise the device.  The
 * pages have no counterpart to this entry point; it is a deployment aid.
 *   Outputs, layouts and results are those of s2o_plan (the caller still
 *   passes Q, K and the output buffers).
 *   Scratch: a 32 MiB array in the library's device memory (a file-scope
 *   __device__ buffer that every GPU loading the library holds until the
 *   process exits).  Configs whose plan workspace (s2o_plan_workspace_size)
 *   exceeds 32 MiB -- e.g. B=1, 8 KV heads, N above ~5K -- are rejected with
 *   S2O_ERR_WORKSPACE_TOO_SMALL before anything is launched.
 *   The 32 MiB are committed by the driver when the library's device code is
 *   loaded into a context: with lazy loading (the default since CUDA 12.2)
 *   that happens on the first call into the library on a device, which may be
 *   this one, and that load can synchronise the device.  The first call on a
 *   device (and again after cudaDeviceReset or in another context) also looks
 *   up the buffer's device address with that device current.  So make one
 *   warm-up call -- e.g. s2o_plan_noalloc on a small config -- at engine
 *   start-up, before any stream capture; later calls do neither.  Nothing in
 *   the buffer has to start at zero: every word the kernels read is written
 *   earlier in the same call.  All calls share the one buffer, so calls whose
 *   work overlaps on the GPU (other streams, other host threads) race and
 *   corrupt each other's results; serialise them.
 *   Allocates nothing: no cudaMalloc, cudaFree or allocating library call.
 */
s2o_status s2o_plan_noalloc(const s2o_config* cfg, const uint16_t* Q, const uint16_t* K,
                            float* scores, int32_t* perm, int32_t* nblocks, float* seg_stats,
                            s2o_stream_t stream);

/*
 * s2o_plan_contiguous -- block-granular comparator at a matched block count:
 * the candidates of each segment are cut into Bk-key blocks in their
 * original order, ranked by pooled mass sum exp(s_j - M) / Z (ties to the
 * lower block) and the first nblocks_match[b,kvh,s] blocks of that ranking
 * are the kept set.  This is the block-sparse baseline whose intra-block
 * redundancy the pages describe (gist.science technical summary, "Enonce du
 * Probleme"); it feeds s2o_attention unchanged, with nblocks_match as its
 * nblocks.
 *   scores, seg_stats  device inputs from s2o_plan (seg_stats required)
 *   nblocks_match      device int32 [B,Hkv,S]
 *   perm_out           out, device int32 [B,Hkv,T]: ranked blocks, each
 *                      block's keys ascending
 */
s2o_status s2o_plan_contiguous(const s2o_config* cfg, const float* scores, const float* seg_stats,
                               const int32_t* nblocks_match, int32_t* perm_out, s2o_stream_t stream);

/*
 * s2o_attention -- sparse prefill output over Keep(s) (gist.science technical
 * summary, section 3 "Implementation du Noyau": pass 1 = the segment's dense
 * causal window, pass 2 = keys in permuted order up to the stop point).
 *   Q, K, V    device bf16 inputs
 *   perm       device int32 [B,Hkv,T] (s2o_plan or s2o_plan_contiguous)
 *   nblocks    device int32 [B,Hkv,S], 0 <= nblocks <= |Cand(s)| / Bk
 *   O          out, device [B,Hq,N,d], bf16 (S2O_OUT_BF16) or fp32 (S2O_OUT_F32)
 * Every perm entry read must lie in Cand(s); violations are clamped, set the
 * device error word (S2O_ERR_BAD_PLAN) and leave O unspecified.
 */
s2o_status s2o_attention(const s2o_config* cfg, const uint16_t* Q, const uint16_t* K,
                         const uint16_t* V, const int32_t* perm, const int32_t* nblocks,
                         void* O, int32_t out_dtype, s2o_stream_t stream);

/* Device bytes s2o_prefill_host needs in its arena. */
s2o_status s2o_prefill_arena_size(const s2o_config* cfg, int32_t out_dtype, size_t* bytes);

/*
 * s2o_attention_bounded -- s2o_attention with every wait of its pipeline
 * (mbarrier polls between the loader, tensor-core and softmax roles of a
 * CTA) limited to max_polls polls instead of the default 2^24, for testing
 * the timeout path (the pages have no counterpart; the library's failure
 * handling is its own).  A wait that runs out sets the device error word
 * (s2o_last_device_error then returns S2O_ERR_DEVICE_TIMEOUT) and the CTA
 * winds down: it waits, with the default limit, for the tensor-core products
 * and Q tiles it already started, frees its tensor memory and ends.  Outputs
 * are unspecified after a timeout.  max_polls = 0 makes every wait give up
 * at once.  Only the even-group-size kernel (Hq/Hkv even) takes the limit;
 * other shapes return S2O_ERR_UNSUPPORTED_SHAPE, max_polls above 2^24
 * S2O_ERR_INVALID_ARG.  Arguments otherwise as s2o_attention.
 */
s2o_status s2o_attention_bounded(const s2o_config* cfg, const uint16_t* Q, const uint16_t* K,
                                 const uint16_t* V, const int32_t* perm, const int32_t* nblocks, void* O,
                                 int32_t out_dtype, uint32_t max_polls, s2o_stream_t stream);

/*
 * s2o_attention_online -- the pages' run-time stop in place of the planned one
 * (gist.science technical summary, section 2 "Regle d'Arret Anticipe"; the
 * arxivlens "Methodology" facet: stop on the marginal softmax gain).  A tile
 * is the segment's rows of a pair of query heads of a group.  It processes
 * the always-kept keys, then the segment's candidate blocks in the order of
 * perm; after each block, each row's gain is the block's share of the
 * exp-sum the row has processed so far (the block included), and the tile
 * stops after the first block whose mean gain over its rows is below
 * cfg->tau.  That block stays in the output.
 *   Q, K, V, O, out_dtype  as s2o_attention
 *   perm         device int32 [B,Hkv,T] from s2o_plan (every segment fully
 *                ordered; the filtered plan's order is not enough)
 *   nblocks_out  out, device int32 [B,Hq,S]: candidate blocks processed by
 *                the tile of each query head (equal within a pair)
 *   Requires an even group size Hq/Hkv (S2O_ERR_UNSUPPORTED_SHAPE otherwise).
 *   A perm entry outside Cand(s) is clamped and reported as S2O_ERR_BAD_PLAN
 *   by s2o_last_device_error.
 */
s2o_status s2o_attention_online(const s2o_config* cfg, const uint16_t* Q, const uint16_t* K,
                                const uint16_t* V, const int32_t* perm, void* O, int32_t out_dtype,
                                int32_t* nblocks_out, s2o_stream_t stream);

/*
 * Q_perm with two query sub-segments (gist.science technical summary,
 * section 1, "Classement par Segment": the queries of a segment are reordered
 * by a coarse importance score against a shared guide vector).  The guide is
 * the segment's pooled query qbar; a row's importance is the mean over the
 * group's query heads of q_i . qbar; rows are ordered by importance
 * descending (ties to the lower row), the first 64 form sub-segment 0, the
 * rest sub-segment 1.  Each sub-segment is planned like a segment (same
 * admissible keys, candidates and stop rule) with its own pooled query, and a
 * row attends over its own sub-segment's kept set.
 *
 * s2o_plan_qperm -- both sub-segment plans (filtered form: each order is
 * exact on its first Bk * nblocks entries, the rest is unspecified).
 *   scores   out, device fp32 [2, B, Hkv, T]   (sub-segment major)
 *   perm     out, device int32 [2, B, Hkv, T]
 *   nblocks  out, device int32 [2, B, Hkv, S]
 *   rowsub   out, device uint8 [B, Hkv, S, 128]: sub-segment of each row of
 *            each segment (rows past N: 1)
 *   workspace  device scratch of s2o_plan_qperm_workspace_size() bytes,
 *            256-byte aligned
 * s2o_attention_qperm -- the sparse output with each row over its own
 * sub-segment's kept set; perm, nblocks, rowsub (16-byte aligned) as
 * produced above; other arguments as s2o_attention.  Requires an even group
 * size Hq/Hkv (S2O_ERR_UNSUPPORTED_SHAPE otherwise).  With Hq/Hkv divisible
 * by 4 each CTA takes one sub-segment of a segment for four query heads, so
 * a row walks only its own sub-segment's kept blocks; otherwise every row
 * walks both sub-segments' kept blocks, masked for the other's rows.  A
 * rowsub that puts more than 64 of a segment's rows in one sub-segment (not
 * one s2o_plan_qperm writes) sets S2O_ERR_BAD_PLAN; the extra rows are then
 * not computed.
 */
s2o_status s2o_plan_qperm_workspace_size(const s2o_config* cfg, size_t* bytes);
s2o_status s2o_plan_qperm(const s2o_config* cfg, const uint16_t* Q, const uint16_t* K, float* scores,
                          int32_t* perm, int32_t* nblocks, uint8_t* rowsub, void* workspace,
                          size_t workspace_bytes, s2o_stream_t stream);
s2o_status s2o_attention_qperm(const s2o_config* cfg, const uint16_t* Q, const uint16_t* K,
                               const uint16_t* V, const int32_t* perm, const int32_t* nblocks,
                               const uint8_t* rowsub, void* O, int32_t out_dtype, s2o_stream_t stream);

/*
 * s2o_block_truth -- ranking accuracy of the pooled order on sampled segments:
 * each candidate block's true mass against the plan's choice (the referee
 * report on the pith.science page: the ranking is never checked against
 * exact attention).  For sampled segment k and (b, kvh), a block's true mass
 * is the mean, over the segment's rows and the group's query heads, of the
 * exact causal softmax probability (over all of [0, i]) of its keys.
 *   Q, K          device bf16 inputs
 *   perm, nblocks device, from s2o_plan (every block of the order is read,
 *                 so a filtered plan's perm is not enough)
 *   segments      HOST int32 [nsamp], each in [0, S); 1 <= nsamp <= 256
 *   stats         out, device fp32 [nsamp, B, Hkv, 5]: C(s), blocks with true
 *                 mass >= tau, blocks in both sets, true mass of the kept
 *                 blocks, true mass of all candidate blocks
 *   mass          out, device fp32 [nsamp, B, Hkv, nbmax] or NULL: the true
 *                 mass of block b of the order; nbmax = |Cand(S-1)| / Bk
 *   workspace     device scratch of s2o_block_truth_workspace_size() bytes,
 *                 256-byte aligned (zeroed by the call itself)
 *   fp32 arithmetic (a measurement).
 */
s2o_status s2o_block_truth_workspace_size(const s2o_config* cfg, int32_t nsamp, size_t* bytes);
s2o_status s2o_block_truth(const s2o_config* cfg, const uint16_t* Q, const uint16_t* K, const int32_t* perm,
                           const int32_t* nblocks, const int32_t* segments, int32_t nsamp, float* stats,
                           float* mass, void* workspace, size_t workspace_bytes, s2o_stream_t stream);

/*
 * s2o_prefill_host -- the whole path from HOST buffers: copies Q, K, V to
 * the device arena, plans (s2o_plan_filtered: it returns no perm, and O and
 * C(s) equal those of s2o_plan), runs the attention and copies O back to
 * host O.  The work is split by (b, kvh), whose rows are contiguous in every
 * buffer: the copies in run on one library stream (K and Q of a group before
 * its V, so its plan can start first), plan and attention on `stream`, the
 * copies out on another library stream, so one group's copies overlap the
 * kernels of the others; with an even group size the attention of a group
 * runs one query-head pair at a time and each pair's O goes out while the
 * next is computed (results equal a single whole call).
 * Host buffers should be page-locked for full copy speed.  The arena is
 * caller-allocated device memory of s2o_prefill_arena_size() bytes, 256-byte
 * aligned.  Synchronises the stream before returning and reports device
 * errors of this call (like s2o_last_device_error).
 *   nblocks_host  optional host int32 [B,Hkv,S] copy of C(s), or NULL
 */
s2o_status s2o_prefill_host(const s2o_config* cfg, const uint16_t* Q_host, const uint16_t* K_host,
                            const uint16_t* V_host, void* O_host, int32_t out_dtype,
                            int32_t* nblocks_host, void* arena, size_t arena_bytes,
                            s2o_stream_t stream);

/* Static description of a status code. */
const char* s2o_status_string(s2o_status st);

/*
 * Synchronises `stream`, reads and clears the current device's error word and
 * maps it to a status (S2O_OK when no device error was recorded).  The word
 * is shared by every stream of the device.
 */
s2o_status s2o_last_device_error(s2o_stream_t stream);

/* Number of kernels the last s2o_plan / s2o_attention / s2o_plan_contiguous
 * call on this thread launched (the library's own kernels only). */
int32_t s2o_last_launch_count(void);

/*
 * Per-kernel timing of the plan calls, for measurement (the pages report no
 * per-stage times; they name the ranking step as the main preprocessing
 * cost: gist.science technical summary, "Resultats Experimentaux").
 * s2o_stage_timing(1) creates this host thread's timing events on the
 * current device; from then on every plan call on this thread (s2o_plan,
 * s2o_plan_filtered, s2o_plan_noalloc, s2o_plan_qperm) records one event on
 * its stream before its first kernel and one after each kernel.
 * s2o_stage_timing(0) destroys the events and stops the recording.  Returns
 * S2O_ERR_CUDA if the events cannot be created.  Recording costs a few
 * microseconds per kernel; leave it off outside measurements.
 */
s2o_status s2o_stage_timing(int32_t enable);

/*
 * Elapsed device time of each kernel of the last plan call on this thread
 * (between consecutive events on its stream).  Waits for that call's last
 * event.  ms[i] (and names[i], a static kernel name, when names is not NULL)
 * are written for i < min(count, cap).  Returns the number of kernels
 * recorded (at most 16), or -1 when timing is off, ms is NULL with cap > 0,
 * or a CUDA event call fails.
 */
int32_t s2o_last_stage_times(float* ms, const char** names, int32_t cap);

#ifdef __cplusplus
}
#endif

#endif /* S2O_H */
