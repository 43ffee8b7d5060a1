/*
 * sparse_mla.h -- C ABI of the B200 (sm_100a) sparse-MLA decode library.
 *
 * The operation (one decode step of DeepSeek-style sparse Multi-head Latent
 * Attention): for every sequence b and head h, one query q[b,h,:] of d_qk =
 * 576 dims attends over the cache rows named by the sequence's top-k index
 * list.  Each gathered 576-dim row k_j is the key; its first d_v = 512 dims
 * are the value.  With s_j = scale * <q[b,h,:], k_j> over the valid entries
 * (index -1 is padding and takes no part),
 *
 *     out[b,h,:] = sum_j softmax(s)_j * k_j[0:512]        (bf16)
 *     lse[b,h]   = ln sum_j exp(s_j)                        (fp32, natural log)
 *
 * A sequence whose list holds no valid entry gets out = 0 and lse = -inf.
 *
 * Source pages (by title):
 *   [Design]  "The MMA Sparse-MLA Decode Kernel: A Deep Dive into AI Inference
 *              Optimization on Blackwell GPUs" -- "The Agent Reasoning":
 *              "Kernel Structure Analysis" (query vs. gathered rows, output
 *              accumulation), "Design Decisions" 1 (head-batched grid: one
 *              gather shared by the head group), 3 (split-K over top-k),
 *              6 (bf16 operands, fp32 accumulation), "Edge Case Handling"
 *              (masked entries), "Validation Strategy" (compare out and LSE).
 *   [Truth]   "The Moment of Truth: Analyzing a Custom MMA Kernel's
 *              Performance on Blackwell GPUs" -- "The Split-K Solution:
 *              Reasoning About the Fix" (partials + combine; grid fixed per
 *              batch bucket for CUDA-graph capture; scratch deterministic
 *              per bucket).
 *   [Pivot]   "The Pivot Point: When a 6.3x Kernel Speedup Reveals the Next
 *              Bottleneck" -- "The Reasoning: Weighing Two Paths" (split-K
 *              for the B=1 under-occupancy; combine handles variable NSPLIT).
 *
 * Conventions for every entry point:
 *  - All tensor pointers are DEVICE pointers owned by the caller, contiguous
 *    (row-major in the order of the dims given), 16-byte aligned.  The
 *    library never allocates, frees or retains them.
 *  - Calls are asynchronous on `stream` (a cudaStream_t passed as void*;
 *    NULL = the legacy default stream).  Nothing synchronises the host,
 *    nothing allocates device memory, so a call can be captured in a CUDA
 *    graph; the grid depends only on the shape (and nsplit).
 *  - Arguments are validated on the host before any launch.  On a
 *    validation error nothing is launched and no CUDA call is made.
 *  - Index values outside [-1, num_kv_rows) (flat) or
 *    [-1, pages_per_seq * page_size) (paged), and page-table entries that
 *    point outside the pool, are caller errors.  The kernels check every
 *    entry as they resolve it: such an entry is read as padding (it takes no
 *    part and nothing is read for it) and sets bit 2 of the device error
 *    word (sparse_mla_get_device_error).
 *  - Entry points are thread-safe; they keep no per-call state.
 */
#ifndef SPARSE_MLA_H_
#define SPARSE_MLA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define SMLA_ABI_VERSION 2

typedef enum {
  SMLA_OK = 0,
  SMLA_ERR_INVALID_ARG = 1,    /* null / misaligned pointer, bad size        */
  SMLA_ERR_UNSUPPORTED = 2,    /* shape this build does not implement        */
  SMLA_ERR_WORKSPACE = 3,      /* workspace missing or smaller than required */
  SMLA_ERR_CUDA = 4,           /* a CUDA runtime call or launch failed       */
  SMLA_ERR_DEVICE_TIMEOUT = 5, /* a kernel gave up a bounded wait (see
                                  sparse_mla_get_device_error)              */
  SMLA_ERR_DEVICE_INDEX = 6,   /* a kernel met an index, page-table entry or
                                  context length outside its range and read
                                  it as absent (error word bit 2 alone)     */
  SMLA_ERR_DEVICE_LAYOUT = 7   /* a kernel found its shared-memory window
                                  misaligned and computed nothing (bit 1)   */
} smla_status;

typedef enum {
  SMLA_KV_BF16 = 0,             /* cache rows: bf16 [num_kv_rows, 576]      */
  SMLA_KV_FP8_E4M3_ROWSCALE = 1, /* cache rows: OCP fp8 e4m3fn codes
                                   [num_kv_rows, 576] (uint8), and one fp32
                                   scale per row: value = decode(code)*scale */
  SMLA_KV_DSV4_PAGED = 2        /* DeepSeek-V4 paged cache ([Design] "The
                                   Agent Reasoning" -> "Cache Layout
                                   Understanding"): pages of 64 token slots,
                                   37,376 bytes each.  Slot i: bytes
                                   [576 i, 576 i + 448) = 448 e4m3fn "nope"
                                   codes, then 64 bf16 "rope" values; bytes
                                   [36864 + 8 i, +7) = UE8M0 scales (2^(e-127))
                                   of the nope dims 64 g .. 64 g + 63, g < 7.
                                   The 512-dim row (448 nope x scale, 64 rope)
                                   is both key and value: d_qk = d_v = 512,
                                   q is [B, 64, 512].  Paged only (page_size
                                   64); num_kv_rows = 64 * pages; no
                                   kv_row_scale. */
} smla_kv_dtype;

/* Problem description.  num_heads must be 64, d_v 512, d_qk 576 (512 for
 * SMLA_KV_DSV4_PAGED).
 *
 * Multi-token decode (tokens_per_seq = T > 1: speculative / multi-token
 * prediction steps, where several new tokens of a sequence are scored at
 * once): every tensor indexed by sequence gains a token dim after it --
 * q [B, T, 64, d_qk], indices [B, T, topk], out [B, T, 64, 512],
 * lse [B, T, 64] -- while page_table stays [B, pages_per_seq], shared by the
 * sequence's tokens.  Token t of sequence b attends over its own list
 * indices[b, t] exactly as a single decode token does, so each (b, t) row
 * is one decode problem (B * T rows in all, at most 65535). */
typedef struct {
  int32_t batch;          /* B >= 1: sequences                                 */
  int32_t num_heads;      /* H = 64                                            */
  int32_t d_qk;           /* 576 = 512 latent + 64 rope (512 for DSV4 pages)   */
  int32_t d_v;            /* 512: the value is the first 512 dims of the row   */
  int32_t topk;           /* k >= 1 entries in each index list                 */
  int32_t kv_dtype;       /* smla_kv_dtype                                     */
  int64_t num_kv_rows;    /* physical rows in the pool (>= 1)                  */
  int32_t page_size;      /* 0: flat pool, indices are physical rows.
                             64: paged pool, indices are logical positions
                             mapped through page_table                         */
  int32_t pages_per_seq;  /* width of page_table when page_size > 0           */
  int32_t nsplit;         /* 0: the planner picks the top-k split; >= 1
                             forces that many splits (clamped to the number
                             of 64-entry tiles of the list);
                             SMLA_NSPLIT_STREAMK asks for the stream-K plan
                             (see sparse_mla_plan_nsplit)                      */
  int32_t tokens_per_seq; /* T: query tokens per sequence, 0 or 1 = one token,
                             at most 16                                        */
} smla_shape;

/* smla_shape.nsplit value that asks for the stream-K plan. */
#define SMLA_NSPLIT_STREAMK (-1)

/* ABI version of the loaded library (SMLA_ABI_VERSION). */
int32_t sparse_mla_abi_version(void);

/* Human-readable name of a status code (static string, never NULL). */
const char* sparse_mla_status_string(smla_status status);

/* Number of top-k splits the decode will use for `shape` on the current
 * device: a pure function of (batch, topk, shape->nsplit, SM count, cluster
 * limit), so the grid is fixed per batch bucket.  Returns 0 if `shape` is
 * invalid.
 *
 * With more than one split, sparse_mla_decode merges the splits in one of
 * two ways (sparse_mla_plan_merge tells which).  When nsplit is a power of
 * two no larger than 16 that the device can launch as a thread-block
 * cluster, the CTAs of a sequence form a cluster: each writes its result,
 * normalised by its own softmax sum, to the workspace as fp16 -- each
 * 128-dim part of a head's row scaled by the power of two that brings its
 * largest magnitude into [2^14, 2^15), so any finite value fits, with 11
 * significant bits of that part's largest value -- the cluster
 * synchronises, and each CTA reduces one block of output columns -- one
 * kernel.  Otherwise each split writes an fp32
 * partial result and a second (combine) kernel merges them.  An automatic
 * plan (shape->nsplit == 0) takes the largest such power of two for which
 * all clusters are resident at once.
 *
 * Stream-K (shape->nsplit == SMLA_NSPLIT_STREAMK; this call then returns
 * 1): for fp8 rows (SMLA_KV_FP8_E4M3_ROWSCALE) with lists of at least 16
 * tiles of 64 entries, when there are more decode rows than half the SMs
 * but not a whole multiple of them, one split per row leaves SMs idle or
 * runs a short second wave.  Instead the grid has one CTA per SM, the rows'
 * tiles are laid end to end (row-major) and each CTA takes an equal run of
 * them.  A row then falls to one CTA, written out directly, or to two or
 * three (consecutive) CTAs: each writes its part, normalised by its own
 * softmax sum, with its log-sum-exp, to the workspace and counts itself in
 * at the row's counter; the last to arrive merges the parts with the
 * log-sum-exp combine ([Truth] "The Split-K Solution"), summing them in
 * CTA order so that the bits do not depend on which CTA merges.  No CTA
 * waits for another.  One kernel launch.  Other shapes that ask for it get
 * the automatic plan.  (On B200 each CTA's switch to its second row costs
 * more than the balance gains on the lists measured, so the automatic
 * plan does not choose it.) */
int32_t sparse_mla_plan_nsplit(const smla_shape* shape);

/* How sparse_mla_decode merges the splits of `shape` on the current device:
 * 0 = one split (nothing to merge), 1 = inside the split kernel (thread-block
 * cluster, one launch), 2 = partials and the combine kernel (two launches),
 * 3 = stream-K (one CTA per SM over the rows' tiles, a shared row merged
 * by its last CTA; one launch).  Returns -1 if `shape` is invalid. */
int32_t sparse_mla_plan_merge(const smla_shape* shape);

/* Bytes of device workspace sparse_mla_decode needs for `shape` (0 when the
 * plan uses one split).  Deterministic in the shape and the device's SM
 * count, so a workspace sized once per batch bucket can be reused by every
 * call and every graph replay.  A stream-K plan over G SMs needs
 * 2 G x 64 x 512 fp32 part results, 2 G x 64 fp32 log-sum-exps and one
 * 8-byte counter per (decode row, lane quarter of 16 heads), each region
 * rounded up to 256 bytes (about 38 MB on 148 SMs).  The counters are
 * tagged per launch and left at zero by the CTA that merges the row, so
 * they need no initialisation either; after a call that set the device
 * error word (a bounded wait gave up), replaying a graph captured before
 * it on the same workspace is not supported.
 * Returns 0 for an invalid shape. */
size_t sparse_mla_workspace_size(const smla_shape* shape);

/* One decode step: the split kernel, plus the combine kernel when the plan
 * merges its splits through a second kernel (sparse_mla_plan_merge == 2).
 * (Layouts for one token per sequence; with tokens_per_seq = T > 1 the q,
 * indices, out and lse tensors carry the extra token dim described at
 * smla_shape, and B below reads as the B * T decode rows, page_table
 * excepted.)
 *   q            [B, 64, 576] bf16 ([B, 64, 512] for SMLA_KV_DSV4_PAGED)
 *   kv_cache     [num_kv_rows, 576] bf16, or uint8 e4m3fn codes, or
 *                [num_kv_rows / 64, 37376] uint8 DeepSeek-V4 pages
 *   kv_row_scale [num_kv_rows] fp32 for SMLA_KV_FP8_E4M3_ROWSCALE, else NULL
 *   page_table   [B, pages_per_seq] int32 when page_size > 0, else NULL
 *   indices      [B, topk] int32, -1 = padding (anywhere in the list).  An
 *                entry at or past pages_per_seq * page_size (paged), or
 *                that resolves to a row outside [0, num_kv_rows), is read
 *                as padding and sets bit 2 of the device error word.
 *   scale        softmax scale (e.g. 1/sqrt(576))
 *   out          [B, 64, 512] bf16   (written)
 *   lse          [B, 64] fp32        (written; natural log, scale included)
 *   workspace    device scratch of >= sparse_mla_workspace_size() bytes,
 *                256-byte aligned; may be NULL when that size is 0.  Its
 *                contents need no initialisation and are garbage afterwards.
 * Two calls that share a workspace must be ordered on the GPU (same stream
 * or event-ordered).  Returns SMLA_OK after launching. */
smla_status sparse_mla_decode(const smla_shape* shape, const void* q, const void* kv_cache,
                              const float* kv_row_scale, const int32_t* page_table,
                              const int32_t* indices, float scale, void* out, float* lse,
                              void* workspace, size_t workspace_bytes, void* stream);

/* The split kernel alone, always in its partials form (never the on-chip
 * merge, never stream-K), with the split count sparse_mla_plan_nsplit gives.
 * With nsplit == 1 it writes out/lse directly (workspace unused).  With
 * nsplit > 1 it writes per-split partial results into the workspace, which
 * must hold B*nsplit*64*(512+1)*4 bytes rounded up to a multiple of 256:
 *   partial_o   = workspace                      [B, nsplit, 64, 512] fp32,
 *                 each split's output normalised by its own softmax sum
 *                 (0 when the split holds no valid entry)
 *   partial_lse = workspace + B*nsplit*64*512*4  [B, nsplit, 64] fp32
 *                 (that split's log-sum-exp, -inf when empty)
 * and out/lse are not touched (sparse_mla_combine finishes them).  *nsplit_out
 * (may be NULL) receives the split count used. */
smla_status sparse_mla_decode_split(const smla_shape* shape, const void* q, const void* kv_cache,
                                    const float* kv_row_scale, const int32_t* page_table,
                                    const int32_t* indices, float scale, void* out, float* lse,
                                    void* workspace, size_t workspace_bytes, int32_t* nsplit_out,
                                    void* stream);

/* Log-sum-exp combine of per-split partials ([Truth] "The Split-K Solution").
 *   partial_o   [B, nsplit, H, d_v] fp32 (normalised per split)
 *   partial_lse [B, nsplit, H] fp32 (-inf for an empty split)
 *   out         [B, H, d_v] bf16, lse [B, H] fp32
 * With L = ln sum_s exp(lse_s): out = sum_s exp(lse_s - L) * o_s, lse = L;
 * every split empty gives out = 0, lse = -inf.  Requires H == 64,
 * d_v == 512, 1 <= nsplit <= 4096. */
smla_status sparse_mla_combine(int32_t batch, int32_t num_heads, int32_t d_v, int32_t nsplit,
                               const float* partial_o, const float* partial_lse, void* out,
                               float* lse, void* stream);

/* Reads and clears the library's device error word on the current device
 * (a synchronous device-to-host copy: call it outside timed or captured
 * regions).  *code receives the raw word, 0 = no error:
 *   bit 0  a kernel gave up a bounded wait on a pipeline barrier
 *   bit 1  the shared-memory window was not 1024-byte aligned (the kernel
 *          returned without computing)
 *   bit 2  an input named something outside its range and was read as
 *          absent: a decode index entry or page-table entry outside the
 *          pool, an indexer context length outside [0, max_ctx] (clamped)
 *          or an indexer page-table entry outside the key cache.
 * Returns, for the most serious bit set: SMLA_ERR_DEVICE_TIMEOUT (bit 0),
 * SMLA_ERR_DEVICE_LAYOUT (bit 1), SMLA_ERR_DEVICE_INDEX (bit 2); SMLA_OK if
 * the word was zero; SMLA_ERR_CUDA on a copy failure. */
smla_status sparse_mla_get_device_error(uint32_t* code);

/* Test hook for the bounded waits; the source pages have no counterpart.
 * Launches the decode kernel for `shape` (SMLA_KV_BF16, flat cache: page
 * size 0; one CTA per decode row, no workspace) with every pipeline wait
 * limited to wait_limit_cycles SM clock cycles and the score-MMA warp
 * waiting on a barrier that nothing arrives on, in place of the staged
 * query.  So no MMA is issued, every warp's wait runs out, the kernel sets
 * bit 0 of the device error word, releases its tensor memory and returns;
 * out and lse are left unwritten.  The context stays usable: the next
 * sparse_mla_get_device_error returns SMLA_ERR_DEVICE_TIMEOUT, and later
 * decodes compute as usual.  Arguments as for sparse_mla_decode (q, kv_cache,
 * indices, out, lse device pointers owned by the caller).  Returns
 * SMLA_ERR_UNSUPPORTED for other cache kinds or a paged cache,
 * SMLA_ERR_INVALID_ARG for wait_limit_cycles outside [1000, 4e9]. */
smla_status sparse_mla_decode_stalled(const smla_shape* shape, const void* q, const void* kv_cache,
                                      const int32_t* indices, float scale, void* out, float* lse,
                                      int64_t wait_limit_cycles, void* stream);

/* Size of the scratch buffer that sparse_mla_decode_static_scratch uses:
 * 24 MiB, enough for rows * nsplit <= 191 split results (rows = batch x
 * tokens_per_seq; at most 131,328 bytes each).  Every split count the
 * planner picks on a 148-SM B200 fits (it keeps rows * nsplit <= 148). */
#define SMLA_STATIC_SCRATCH_BYTES ((size_t)24 << 20)

/* The whole decode step, for callers that cannot allocate device memory.
 * The source pages have no counterpart to this entry point.
 *
 * It computes exactly what sparse_mla_decode computes, with the same
 * arguments except the workspace.  When the plan has more than one split,
 * the split results go to a scratch buffer of SMLA_STATIC_SCRATCH_BYTES
 * that the library holds in device memory as a static array: one per
 * device, created when the library's device code is loaded.  Neither this
 * call nor the library allocates or frees anything.
 *
 * - Size limit.  A shape whose split results would not fit is rejected
 *   with SMLA_ERR_WORKSPACE before any launch.  When shape->nsplit fixes
 *   the split count and its results cannot fit whichever way they are
 *   merged (in-cluster merge, possible for a power of two <= 16: 67,584
 *   bytes per decode row and split; otherwise 131,328), it is rejected
 *   before any CUDA call.  Use sparse_mla_decode with your own workspace
 *   for such shapes.
 * - Zeroing.  Every split writes its whole partial (an empty split writes
 *   o = 0, lse = -inf), so nothing in the scratch has to start at zero and
 *   nothing is cleared.
 * - First call.  The first call on a device looks up the scratch address
 *   with cudaGetSymbolAddress, with that device current, and keeps it.  A
 *   failed lookup returns SMLA_ERR_CUDA.  If you capture streams, make one
 *   call on each device before capturing, so that this set-up is done.
 * - Races.  All calls on one device share the one scratch buffer.  Calls
 *   that can overlap in time (different streams, different host threads
 *   without ordering) race on it and corrupt each other's results.  Issue
 *   them on one stream, or otherwise order them.
 *
 * Errors and validation are as for sparse_mla_decode. */
smla_status sparse_mla_decode_static_scratch(const smla_shape* shape, const void* q, const void* kv_cache,
                                             const float* kv_row_scale, const int32_t* page_table,
                                             const int32_t* indices, float scale, void* out, float* lse,
                                             void* stream);

/* Bytes of device staging that sparse_mla_decode_host needs for `shape`:
 * q, indices, page table, out, lse and the decode workspace
 * (sparse_mla_workspace_size), each region rounded up to 256 bytes, in that
 * order.  Returns 0 for an invalid shape. */
size_t sparse_mla_host_staging_size(const smla_shape* shape);

/* The decode step with the per-step tensors in host memory; the cache
 * (kv_cache, kv_row_scale) stays in device memory, where a serving engine
 * keeps it.  The source pages have no counterpart to this entry point.
 *
 *   q_host, indices_host, page_table_host (when page_size > 0, else NULL):
 *       host memory, laid out as for sparse_mla_decode
 *   out_host [B, 64, 512] bf16, lse_host [B, 64] fp32: host memory, written
 *   staging: device memory of >= sparse_mla_host_staging_size() bytes,
 *       256-byte aligned, owned by the caller; contents need no
 *       initialisation and are garbage afterwards
 *
 * On `stream`, in order: one cudaMemcpyAsync per input (host to device)
 * into the staging, sparse_mla_decode on the staged copies, one
 * cudaMemcpyAsync per result (device to host).  The call returns after
 * enqueueing; the results are in out_host / lse_host once the stream has
 * reached this point (synchronise the stream or an event).  Host buffers
 * must be page-locked (cudaHostAlloc / cudaHostRegister) for the copies to
 * be asynchronous; they must stay valid until then.  Calls that can
 * overlap (different streams) need separate staging: two streams with one
 * staging each overlap one step's copies with another step's decode.
 *
 * Errors: every argument is checked before the first copy is enqueued
 * (SMLA_ERR_INVALID_ARG / SMLA_ERR_UNSUPPORTED as for sparse_mla_decode;
 * SMLA_ERR_WORKSPACE for missing, misaligned or short staging);
 * SMLA_ERR_CUDA if a copy or launch is refused. */
smla_status sparse_mla_decode_host(const smla_shape* shape, const void* q_host, const void* kv_cache,
                                   const float* kv_row_scale, const int32_t* page_table_host,
                                   const int32_t* indices_host, float scale, void* out_host, float* lse_host,
                                   void* staging, size_t staging_bytes, void* stream);

/* ------------------------------------------------------------------ indexer
 * The step upstream of the decode: it scores every position of each
 * sequence's context and picks the top-k positions the decode attends to
 * ("The Pivot Point: When a 6.3x Kernel Speedup Reveals the Next
 * Bottleneck", "Input Knowledge Required": the indexer selects the top ~512
 * cache positions per decode step; "The Context: A Campaign in Full Swing":
 * its batched matrix product runs on bf16 tensor cores; "The Moment of
 * Truth: Benchmarking a Custom MMA Kernel for DeepSeek-V4-Flash on
 * Blackwell", "Broader Context": only the real context is scored).
 *
 * Scores, in the published form of DeepSeek's sparse-attention indexer (the
 * pages name only the batched product and the top-k):
 *   I[b, s] = sum_h w[b, h] * max(0, q[b, h, :] . k[row(b, s), :]),  s < ctx_len[b]
 * accumulated in fp32 (each head's dot product on the tensor cores, the
 * weighted sum over heads in order h = 0 .. 63), with
 * row(b, s) = page_table[b, s / 64] * 64 + s % 64.
 * Selection: the min(topk, ctx_len[b]) positions with the largest I[b, s],
 * ties to the lower position, written in ascending order, then -1. */
typedef struct {
  int32_t batch;          /* B, 1 .. 65535                                     */
  int32_t heads;          /* 64                                                */
  int32_t dim;            /* 128 (bf16 per head)                               */
  int32_t topk;           /* 1 .. 65536                                        */
  int32_t max_ctx;        /* width of a score row: 1 .. 2^20, >= every ctx_len */
  int32_t page_size;      /* 64                                                */
  int32_t pages_per_seq;  /* page-table width; 64 * pages_per_seq >= max_ctx   */
  int32_t reserved;       /* must be 0                                         */
  int64_t num_key_rows;   /* rows in the key cache, a multiple of 64           */
} smla_indexer_shape;

/* Scores of every position (the indexer's batched product).
 *   q         [B, 64, 128] bf16, 16-byte aligned
 *   w         [B, 64] fp32 head weights
 *   k_cache   [num_key_rows, 128] bf16 keys, 16-byte aligned (64-row pages)
 *   page_table[B, pages_per_seq] int32, ctx_len [B] int32
 *   scores    [B, max_ctx] fp32, written: I[b, s] for s < ctx_len[b], -inf
 *             after (-0 is written as +0)
 * All device memory, caller-owned.  A ctx_len outside [0, max_ctx] is
 * clamped and a page-table entry outside the cache reads as absent keys;
 * both set bit 2 of the device error word.  Returns after launching. */
smla_status sparse_mla_indexer_scores(const smla_indexer_shape* shape, const void* q, const float* w,
                                      const void* k_cache, const int32_t* page_table, const int32_t* ctx_len,
                                      float* scores, void* stream);

/* Top-k positions from a score matrix laid out as above:
 *   indices [B, topk] int32, written (ascending positions, -1 padding).
 * Reads scores[b, 0 .. ctx_len[b]) only; ctx_len as above. */
smla_status sparse_mla_indexer_topk(const smla_indexer_shape* shape, const float* scores, const int32_t* ctx_len,
                                    int32_t* indices, void* stream);

/* Both steps: scores into the caller's `scores` buffer ([B, max_ctx] fp32,
 * kept for inspection), then the top-k into `indices`.  Two launches on
 * `stream`; the second may start its prologue early (programmatic
 * dependent launch) and waits for the first. */
smla_status sparse_mla_indexer(const smla_indexer_shape* shape, const void* q, const float* w, const void* k_cache,
                               const int32_t* page_table, const int32_t* ctx_len, float* scores,
                               int32_t* indices, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* SPARSE_MLA_H_ */
