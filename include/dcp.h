/*
 * dcp.h -- C ABI of libdcp: decode attention over a paged KV cache that is
 * sharded along the sequence (Decode Context Parallelism), for NVIDIA B200
 * (sm_100a).
 *
 * The method (web pages on Decode Context Parallelism):
 *  - "Efficient Decode Context Parallelism with vLLM for Long Context
 *    Workloads", section 4: every GPU of the group keeps the KV cache of a
 *    subset of the token positions of each request, so per-GPU KV is 1/N;
 *  - same page, section 4.1: each GPU attends the (gathered) query against its
 *    local KV slice, producing a partial output and a per-head log-sum-exp;
 *    the partials are reweighted by their LSE and summed (all-gather +
 *    reduce-scatter across GPUs);
 *  - same page, sections 5.3 / 5.4: MLA keeps one latent row per token shared
 *    by all query heads; GQA broadcasts each KV head to its query heads;
 *  - "Decode Context Parallel Guide" (vLLM Ascend), Constraints:
 *    cp_kv_cache_interleave_size sets how many consecutive positions go to
 *    one shard before moving to the next.
 *
 * The library runs all N shards on ONE GPU: shard n's pages live in the same
 * page pool as the other shards' pages (disjoint page ids), decode_partial
 * computes every shard's partial in one launch, and dcp_merge performs the
 * LSE-weighted sum that the all-gather + reduce-scatter would perform across
 * GPUs (dcp_decode_merged does both in one launch sequence).  The *_rank calls
 * serve one rank of an N-GPU group instead, whose cache holds only its shard.
 *
 * Conventions for every call:
 *  - Every pointer argument is DEVICE memory owned by the caller, unless the
 *    argument's comment says "host".  The library allocates nothing and keeps
 *    no pointer after a call returns.
 *  - `stream` is a cudaStream_t (NULL = legacy default stream).  Work is
 *    enqueued asynchronously; the return value reports host-side validation
 *    and launch errors only.  Errors found by a kernel (an unallocated page,
 *    a negative length) are recorded in a sticky per-device status word read
 *    by dcp_get_device_status(); kernels never trap and never spin without a
 *    time limit.
 *  - Device pointers must be 16-byte aligned (DCP_ERR_MISALIGNED otherwise).
 *  - Sizes are element counts unless they say bytes.
 */
#ifndef DCP_H
#define DCP_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    DCP_OK = 0,
    DCP_ERR_INVALID_ARG = 1,        /* a size, count or pointer is out of range / NULL */
    DCP_ERR_UNSUPPORTED = 2,        /* a valid shape this build has no kernel for */
    DCP_ERR_UNALLOCATED_PAGE = 3,   /* a block-table entry needed by the call is not a pool page */
    DCP_ERR_WORKSPACE_TOO_SMALL = 4,
    DCP_ERR_CUDA = 5,               /* a CUDA runtime call failed (launch, attribute, ...) */
    DCP_ERR_MISALIGNED = 6,         /* a device pointer is not 16-byte aligned */
    DCP_ERR_TIMEOUT = 7             /* a kernel gave up waiting on a copy (never expected) */
} dcp_status;

typedef enum { DCP_GQA = 0, DCP_MLA = 1 } dcp_kind;
/* what a decode call produces (workspace sizing of dcp_decode_workspace_size_ex) */
typedef enum {
    DCP_DECODE_PARTIAL = 0,  /* every shard's partial: dcp_decode_partial(_multi) */
    DCP_DECODE_MERGED = 1,   /* the merged output: dcp_decode_merged */
    DCP_DECODE_RANK = 2      /* one rank's shard of a multi-GPU group: dcp_decode_rank */
} dcp_decode_mode;
typedef enum { DCP_BF16 = 0, DCP_FP8_E4M3 = 1 } dcp_dtype;

/*
 * The sharded paged KV cache.
 *
 *  kind/dtype   DCP_GQA with DCP_BF16; or DCP_MLA with DCP_BF16 or DCP_FP8_E4M3.
 *  n_shards     N >= 1: shards of the sequence dimension.
 *  interleave   I >= 1: position p belongs to shard (p / I) mod N; within a
 *               shard the owned positions are packed in increasing order, so
 *               p has local index (p / (I*N))*I + p mod I.
 *  page_size    P tokens per page: 16 or 64.
 *  num_pages    pages in the pool (all shards together).
 *  hq, hkv      query heads and KV heads (MLA: hkv = 1); hq % hkv == 0; query
 *               head h reads KV head h / (hq/hkv).
 *  dk, dv       key and value widths.  GQA: dk = dv in {64, 128}.  MLA: dk =
 *               576 (512 + 64 rope), dv = 512; the value is the first dv
 *               entries of the latent row (absorbed MLA).
 *  scale        softmax scale applied to q.k.
 *  k_pages      GQA: keys   [num_pages][hkv][P][dk] bf16.
 *               MLA: latent [num_pages][P][576] bf16, or e4m3 bytes for fp8.
 *  v_pages      GQA: values [num_pages][hkv][P][dv] bf16.  MLA: NULL.
 *  kv_scales    MLA fp8: per-token fp32 scale [num_pages][P]; value of latent
 *               element = e4m3(code) * scale.  Otherwise NULL.
 *  block_tables int32 [n_shards][batch][max_local_pages]: shard n's local page
 *               j of request b is pool page block_tables[n][b][j]; -1 = none.
 *  batch        B: requests (rows of each shard's block table).
 */
typedef struct {
    int32_t kind;
    int32_t dtype;
    int32_t n_shards;
    int32_t interleave;
    int32_t page_size;
    int32_t num_pages;
    int32_t hq;
    int32_t hkv;
    int32_t dk;
    int32_t dv;
    float scale;
    int32_t batch;
    int32_t max_local_pages;
    int32_t reserved0;
    void* k_pages;
    void* v_pages;
    float* kv_scales;
    const int32_t* block_tables;
} dcp_cache_desc;

/* Human-readable name of a status code (static string, host). */
const char* dcp_status_string(dcp_status s);

/*
 * dcp_shard_counts -- positions each shard owns.
 * Passage: blog section 4 (positions split across GPUs) and the guide's
 * cp_kv_cache_interleave_size.
 *  seq_lens   int32 [B]: logical lengths L_b >= 0.
 *  counts_out int32 [N][B]: number of p in [0, L_b) with (p / I) mod N == n,
 *             i.e. (L/(I N))*I + clamp(L mod (I N) - n I, 0, I).
 * Errors: DCP_ERR_INVALID_ARG for B < 1, N < 1, I < 1 or NULL pointers.
 */
dcp_status dcp_shard_counts(int32_t B, const int32_t* seq_lens, int32_t N, int32_t I, int32_t* counts_out,
                            void* stream);

/*
 * dcp_shard_map -- owner and storage slot of positions.
 * Passage: blog section 4; the guide's cp_kv_cache_interleave_size.
 *  n_pos      number of positions.
 *  pos        int32 [n_pos]: positions p >= 0.
 *  req        int32 [n_pos]: request of each position, or NULL (position i
 *             belongs to request i).
 *  rank_out   int32 [n_pos]: owner shard (p / I) mod N.
 *  local_out  int32 [n_pos]: local index (p / (I N))*I + p mod I.
 *  slot_out   int64 [n_pos]: physical slot block_tables[rank][req][local / P] * P
 *             + local mod P, or -1 when that block-table entry is -1 or not a
 *             pool page (the device status word then records
 *             DCP_ERR_UNALLOCATED_PAGE).
 * Uses n_shards, interleave, page_size, num_pages, batch, max_local_pages and
 * block_tables of `cache` (page pools may be NULL).
 */
dcp_status dcp_shard_map(const dcp_cache_desc* cache, int64_t n_pos, const int32_t* pos, const int32_t* req,
                         int32_t* rank_out, int32_t* local_out, int64_t* slot_out, void* stream);

/*
 * dcp_kv_append -- write tokens into the pages of the shard that owns them.
 * Passage: blog section 4 (a position's KV lives only on its owner) and
 * sections 5.3 / 5.4 (latent row vs. per-KV-head rows).
 *  n_tok      rows to write (one decode step: n_tok = B, pos = L_b).
 *  req        int32 [n_tok] request of each row, or NULL (row i -> request i).
 *  pos        int32 [n_tok] position of each row.
 *  k_new      GQA: bf16 [n_tok][hkv][dk].  MLA: latent bf16 [n_tok][576]; for an
 *             fp8 cache the row is quantised on the way in: scale = amax/448
 *             (fp32), code = round-to-nearest-even(x / scale) saturated to
 *             +-448; amax = 0 stores scale 1 and zero codes.
 *  v_new      GQA: bf16 [n_tok][hkv][dv].  MLA: NULL.
 * Rows whose slot is unallocated are skipped and the device status word
 * records DCP_ERR_UNALLOCATED_PAGE.  Two rows with the same (req, pos) race.
 */
dcp_status dcp_kv_append(const dcp_cache_desc* cache, int64_t n_tok, const int32_t* req, const int32_t* pos,
                         const void* k_new, const void* v_new, void* stream);

/*
 * dcp_decode_workspace_size -- bytes of device workspace dcp_decode_partial
 * needs for this cache and batch on the CURRENT device (host function; no
 * GPU work).  Returns 0 for an invalid descriptor.
 */
size_t dcp_decode_workspace_size(const dcp_cache_desc* cache, int32_t B);

/*
 * dcp_decode_partial -- every shard's partial decode attention, one launch
 * sequence for all N shards.
 * Passage: blog section 4.1 ("Compute": attention between the gathered query
 * and the local KV slice, giving a partial output and its LSE).
 *  B          requests; must equal cache->batch.
 *  q          bf16 [B][hq][dk]: one query token per request (already
 *             gathered; on one GPU every shard reads the same q).
 *  seq_lens   int32 [B]: L_b, positions [0, L_b) are attended.
 *  o_partial  fp32 [N][B][hq][dv]: shard n's normalised partial output
 *             sum_p exp(s_p - m) v_p / sum_p exp(s_p - m) over its own
 *             positions, s_p = scale * q . k_p; 0 when shard n owns none.
 *  lse        fp32 [N][B][hq]: natural-log LSE of shard n's scores,
 *             -inf when it owns none.
 *  ws, ws_bytes  device workspace of at least dcp_decode_workspace_size()
 *             bytes; its contents need no initialisation and are clobbered.
 * Concurrent calls must use distinct workspaces.  The work is queued on
 * `stream`; the call does not wait for it.
 * Errors, returned before anything is launched:
 *  DCP_ERR_INVALID_ARG     a bad descriptor, B != cache->batch, or a NULL pointer;
 *  DCP_ERR_MISALIGNED      q, o_partial, lse, ws or a pool not 16-byte aligned;
 *  DCP_ERR_UNSUPPORTED     a shape no kernel of this build covers (page size,
 *                          head size, group size);
 *  DCP_ERR_WORKSPACE_TOO_SMALL  ws_bytes below dcp_decode_workspace_size();
 *  DCP_ERR_CUDA            a launch or an attribute call failed.
 * Device-side errors, read with dcp_get_device_status:
 *  DCP_ERR_UNALLOCATED_PAGE  an attended position's page is not a pool page; its
 *                          tokens are skipped;
 *  DCP_ERR_TIMEOUT         a kernel gave up waiting on a copy; the outputs of that
 *                          call are then unspecified.
 */
dcp_status dcp_decode_partial(const dcp_cache_desc* cache, int32_t B, const void* q, const int32_t* seq_lens,
                              float* o_partial, float* lse, void* ws, size_t ws_bytes, void* stream);

/*
 * dcp_decode_workspace_size_ex -- bytes of device workspace that the decode
 * call of `mode` (dcp_decode_mode: dcp_decode_partial(_multi),
 * dcp_decode_merged or dcp_decode_rank) needs for this cache, batch and query
 * length on the CURRENT device (host function; no GPU work).  Returns 0 for an
 * invalid descriptor or mode, or a shape no kernel of this build covers.
 */
size_t dcp_decode_workspace_size_ex(const dcp_cache_desc* cache, int32_t B, int32_t q_len, int32_t mode);

/*
 * dcp_decode_partial_multi -- dcp_decode_partial with q_len query tokens per
 * request: speculative decoding / multi-token prediction under DCP.
 * Passage: blog section 6 (future work: support for MTP and speculative
 * decoding with DCP) on top of section 4.1.  The pages do not state the mask;
 * this library takes the causal one: request b's last q_len positions are its
 * new tokens, and query token j attends the positions p <= L_b - q_len + j.
 *  q_len      1 <= q_len <= 64.  q_len > 1 is served by the tensor-core
 *             kernels only: MLA with 64-token pages and q_len * hq in
 *             {16, 32, 64}; GQA with q_len * hq / hkv == 16.  Other shapes
 *             return DCP_ERR_UNSUPPORTED.
 *  q          bf16 [B][q_len][hq][dk].
 *  seq_lens   int32 [B]: L_b, which must be 0 or >= q_len (0 < L_b < q_len
 *             records DCP_ERR_INVALID_ARG in the device status word; such a
 *             request's token j attends max(0, L_b - q_len + j + 1) positions).
 *  o_partial  fp32 [N][B][q_len][hq][dv]: shard n's normalised partial of each
 *             query token over the positions it owns and that token attends;
 *             0 where there are none.
 *  lse        fp32 [N][B][q_len][hq]: natural-log LSE, -inf where none.
 *  ws, ws_bytes  workspace of at least dcp_decode_workspace_size_ex(cache, B,
 *             q_len, DCP_DECODE_PARTIAL) bytes; clobbered.
 * Errors as dcp_decode_partial.
 */
dcp_status dcp_decode_partial_multi(const dcp_cache_desc* cache, int32_t B, int32_t q_len, const void* q,
                                    const int32_t* seq_lens, float* o_partial, float* lse, void* ws, size_t ws_bytes,
                                    void* stream);

/*
 * dcp_decode_merged -- every shard's partial attention and the LSE merge in
 * one call: the output of dcp_decode_partial(_multi) followed by dcp_merge,
 * with the per-shard partials kept in the workspace (and dropped from L2 by
 * the merge once read) instead of the caller's memory.
 * Passage: blog section 4.1 (each GPU's partial output and LSE, reweighted by
 * the LSE values and summed by the all-gather + reduce-scatter).  Here all
 * shards are on one GPU; the merge runs as a second kernel after the decode
 * (the kernel boundary orders the partials' stores before the merge reads
 * them, which costs less than ordering them inside the decode kernel).
 *  q_len, q, seq_lens   as dcp_decode_partial_multi (q_len = 1: one query
 *             token per request, q bf16 [B][hq][dk]).
 *  out        fp32 [B][q_len][hq][dv]: sum over shards of exp(lse_n - LSE) o_n,
 *             i.e. the unsharded decode attention; 0 where a query token
 *             attends no position.
 *  lse_out    fp32 [B][q_len][hq]: LSE = M + ln sum_n exp(lse_n - M),
 *             M = max_n lse_n; -inf where a query token attends no position.
 *  finish_ns  int64 [B] or NULL: nanoseconds (device global timer) from the
 *             start of the call's first kernel until the last shard of request
 *             b was decoded (its merged output follows in the merge kernel).
 *             For per-request latency within one batch; the values order the
 *             requests' completions, they are not a kernel timer.
 *  ws, ws_bytes  workspace of at least dcp_decode_workspace_size_ex(cache, B,
 *             q_len, DCP_DECODE_MERGED) bytes, which includes the partials (4 * N * B * q_len *
 *             hq * (dv + 1) bytes); clobbered.  Concurrent calls need distinct
 *             workspaces.
 * Errors as dcp_decode_partial (finish_ns must be 16-byte aligned too).
 */
dcp_status dcp_decode_merged(const dcp_cache_desc* cache, int32_t B, int32_t q_len, const void* q,
                             const int32_t* seq_lens, float* out, float* lse_out, int64_t* finish_ns, void* ws,
                             size_t ws_bytes, void* stream);

/*
 * Several GPUs: the cache of ONE rank of an N-GPU group.
 * Passage: blog section 4 (each GPU keeps the KV of the positions it owns) and
 * section 4.1 (each GPU attends its local slice; the partial outputs and LSEs
 * are then combined by an all-gather and a reduce-scatter across the group).
 * For these calls the descriptor is that rank's: n_shards = N (the group size),
 * the pools hold only this rank's pages, and block_tables is int32
 * [1][batch][max_local_pages]: this rank's local pages of each request.
 */

/*
 * dcp_kv_append_rank -- dcp_kv_append on rank `rank`'s cache: every rank may
 * be given every new token; it stores the ones it owns ((p / I) mod N == rank)
 * and skips the others without an error.
 */
dcp_status dcp_kv_append_rank(const dcp_cache_desc* cache, int32_t rank, int64_t n_tok, const int32_t* req,
                              const int32_t* pos, const void* k_new, const void* v_new, void* stream);

/*
 * dcp_decode_rank -- this rank's partial attention: every query token of every
 * request against the positions rank `rank` owns (0 <= rank < n_shards).
 *  q_len, q, seq_lens   as dcp_decode_partial_multi (q_len = 1: one token).
 *  o          fp32 [B][q_len][hq][dv]: the normalised partial output, 0 where
 *             the rank owns no attended position.
 *  lse        fp32 [B][q_len][hq]: its natural-log LSE, -inf where none.
 *  ws, ws_bytes  at least dcp_decode_workspace_size_ex(cache, B, q_len, DCP_DECODE_RANK).
 * Next: all-gather lse across the group, dcp_lse_rescale, reduce-scatter.
 * Errors as dcp_decode_partial.
 */
dcp_status dcp_decode_rank(const dcp_cache_desc* cache, int32_t rank, int32_t B, int32_t q_len, const void* q,
                           const int32_t* seq_lens, float* o, float* lse, void* ws, size_t ws_bytes, void* stream);

/*
 * dcp_lse_rescale -- the local step between the all-gather of the LSEs and the
 * reduce-scatter of the outputs (blog section 4.1: the LSE values reweight the
 * partials, the reduce-scatter sums them).
 *  lse_all    fp32 [N][B][H]: every rank's lse (the all-gathered tensor).
 *  o          fp32 [B][H][Dv]: this rank's partial (dcp_decode_rank's o, with
 *             H = q_len * hq rows).
 *  o_rs       fp32 [N][B][H/N][Dv], output: exp(lse_rank - LSE) * o, laid out
 *             so that block n holds the rows rank n keeps after the
 *             reduce-scatter (a sum over ranks).  H must be a multiple of N.
 *  lse_out    fp32 [B][H] or NULL: LSE = M + ln sum_n exp(lse_n - M),
 *             M = max_n lse_n (-inf when every rank has -inf).
 * Errors: DCP_ERR_INVALID_ARG for sizes out of range, rank outside [0, N),
 * H % N != 0 or NULL pointers; DCP_ERR_MISALIGNED for o / o_rs.
 */
dcp_status dcp_lse_rescale(int32_t N, int32_t rank, int32_t B, int32_t H, int32_t Dv, const float* lse_all,
                           const float* o, float* o_rs, float* lse_out, void* stream);

/*
 * DCP_STATIC_SCRATCH_BYTES -- size of the decode scratch built into the
 * library: 64 MiB of device memory per device, reserved when the library's
 * device code is loaded on that device.
 */
#define DCP_STATIC_SCRATCH_BYTES ((size_t)64 << 20)

/*
 * dcp_decode_partial_noalloc -- dcp_decode_partial with no caller workspace
 * and no allocation: the plan, the split-chunk partials and the counters live
 * in the library's built-in scratch (DCP_STATIC_SCRATCH_BYTES).
 * The method's pages have no counterpart of this call.  It serves callers that
 * cannot allocate device memory where they decode: a serving process whose
 * caching allocator has already reserved the free HBM for its paged KV pool
 * (a fresh cudaMalloc fails there, and the library has no handle on that
 * allocator), and decode loops that cannot take the implicit device
 * synchronisation of cudaMalloc / cudaFree.
 *  Arguments as dcp_decode_partial, without ws / ws_bytes.
 *  The plan is dcp_decode_partial's when dcp_decode_workspace_size() fits in
 *  the scratch; otherwise the planner's split-slot bound is shrunk (fewer
 *  units per CTA, so fewer, longer chunks) until it fits.  Returns
 *  DCP_ERR_WORKSPACE_TOO_SMALL, launching nothing, when even the smallest
 *  bound does not fit.  With T = u * C units targeted (u = units per CTA,
 *  halved from 16 -- 4 for the CUDA-core paths -- down to 1; C = the persistent
 *  grid: one CTA per SM for the tensor-core MLA path, SMs x resident CTAs per
 *  SM for the others), the scratch holds, each term rounded up to 256 bytes:
 *    32 * (N*B + T + 1)          work units
 *    4 * N*B*hq + 8 * N*B        per-shard counters
 *    4 * (2T + 2) * hq * (dv+1)  split-chunk partials and their LSE
 *    B * (128*576 + 256)         fp8 MLA on tensor cores only: the query
 *                                split into two e4m3 terms.
 *  So the fp8 MLA path with B = 512 and hq = 64 (the high-concurrency
 *  workload) does not fit at any N on a 148-SM part: its query split alone
 *  takes 37.9 MB and the smallest split area 39 MB; such callers use
 *  dcp_decode_partial with a workspace.
 *  The plan kernel, first on `stream`, clears the scratch's work ticket and
 *  done counters; nothing else in it needs initialising.
 *  Calls that can overlap in time (different streams, or threads without an
 *  order between them) race on the one scratch array and give wrong results:
 *  serialise them, e.g. on one stream.
 */
dcp_status dcp_decode_partial_noalloc(const dcp_cache_desc* cache, int32_t B, const void* q,
                                      const int32_t* seq_lens, float* o_partial, float* lse, void* stream);

/*
 * dcp_merge -- LSE-weighted merge of N partials (the arithmetic of the
 * all-gather + reduce-scatter step).
 * Passage: blog section 4.1 ("the LSE values reweight and merge the partials").
 *  o_partial  fp32 [N][B][H][Dv], lse fp32 [N][B][H] (as written by
 *             dcp_decode_partial).
 *  out        fp32 [B][H][Dv]: sum_n exp(lse_n - LSE) o_n.
 *  lse_out    fp32 [B][H]: LSE = M + ln sum_n exp(lse_n - M), M = max_n lse_n;
 *             all -inf gives out = 0, LSE = -inf.  May be NULL.
 */
dcp_status dcp_merge(int32_t N, int32_t B, int32_t H, int32_t Dv, const float* o_partial, const float* lse,
                     float* out, float* lse_out, void* stream);

/*
 * dcp_get_device_status -- read and clear the sticky device status word of
 * the current device.  Synchronises `stream` first.
 *  status_out  HOST int32: DCP_OK, or the first error a kernel recorded since
 *              the last read.
 */
dcp_status dcp_get_device_status(int32_t* status_out, void* stream);

/*
 * dcp_selftest_bounded_wait -- runs the failure path of the decode kernels'
 * bounded waits, without a fault.  The persistent kernels wait on mbarriers
 * (page copies landed, scores ready, buffers free) with a 4 s limit on the
 * GPU's nanosecond timer; a wait that runs out records DCP_ERR_TIMEOUT in the
 * sticky status word and raises its CTA's abort flag, and the kernel returns.
 * In a correct run that never happens.  Here one thread waits, through the
 * same code, on a barrier that nothing arrives on.  Not part of the method
 * ("Efficient Decode Context Parallelism with vLLM for Long Context
 * Workloads" has no counterpart); it exists so that the timeout path is
 * exercised on a GPU.
 *  result  DEVICE int64 [3], 16-byte aligned, caller-owned, written by the
 *          kernel: [0] 1 if the wait reported completion (never expected),
 *          [1] the abort flag after the wait (1 expected), [2] the
 *          nanoseconds the wait took (at least the 4 s limit).
 * Asynchronous on `stream` (about 4 s of one thread on one SM); afterwards
 * dcp_get_device_status returns DCP_ERR_TIMEOUT (and clears it), and the
 * context stays usable.  Returns DCP_ERR_INVALID_ARG for a NULL result,
 * DCP_ERR_MISALIGNED for a misaligned one, DCP_ERR_CUDA if the launch fails.
 */
dcp_status dcp_selftest_bounded_wait(int64_t* result, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* DCP_H */
