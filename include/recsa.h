/*
 * recsa.h -- C ABI of the RecSA (Recursive Sparse Attention) build -> select ->
 * attend hot path, hand-written CUDA for sm_100a (B200).  Library: librecsa.so.
 *
 * Method: "Recursive Sparse Attention: Million-Token Length Extrapolation at
 * Logarithmic Cost" (arXiv:2611.07232).  Tree construction is Eq.1 ("Tree
 * Construction"), top-down selection Eq.3 ("Hierarchical Selection") with
 * candidate-local RoPE ("Key Theoretical Insight"), and the unified softmax over
 * level-0 tokens and unselected summaries Eq.4 ("Unified Softmax").
 *
 * Conventions for every call:
 *   - Device buffers are allocated and owned by the caller.  The library owns only
 *     the small host handle returned by recsa_tree_init.  It never calls cudaMalloc.
 *   - Calls that take a stream are asynchronous on that stream (a cudaStream_t,
 *     passed as void*; NULL is the legacy default stream) and issue only kernel
 *     launches, so they can be captured in a CUDA graph.  recsa_get_status is the
 *     one call that synchronises.
 *   - Argument, shape, alignment and capacity errors are detected on the host and
 *     returned before anything is launched.  Conditions only the device can see (a
 *     query position beyond the current length after graph replays, a length that
 *     would pass the capacity) set a sticky device status word and the affected
 *     work is skipped; recsa_get_status reports it.  Kernels never trap.
 *   - Layouts are row-major with the head dimension d contiguous.  Element type of
 *     K, V, q, out and the level tables is the config's dtype (fp32 or bf16).
 */
#ifndef RECSA_H
#define RECSA_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define RECSA_API __attribute__((visibility("default")))
#else
#define RECSA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    RECSA_OK = 0,
    RECSA_E_INVAL = 1,        /* NULL pointer, bad size, misaligned pointer/stride, bad config   */
    RECSA_E_UNSUPPORTED = 2,  /* valid but not built here: head_dim, group size, C, k, C*k       */
    RECSA_E_CAPACITY = 3,     /* a length would exceed capacity, or a buffer is too small        */
    RECSA_E_CUDA = 4,         /* a CUDA runtime call or kernel launch failed                      */
    RECSA_E_TIMEOUT = 5,      /* a bounded device wait gave up                                    */
    RECSA_E_DEVICE = 6        /* device status word: a query or append was out of range, a       */
                              /* staging buffer was misaligned, or (bounds-checked build only) an */
                              /* index failed its range check                                     */
} recsa_status;

typedef enum { RECSA_F32 = 0, RECSA_BF16 = 1 } recsa_dtype;

#define RECSA_MAX_C 32
#define RECSA_MAX_BATCH 64
#define RECSA_MAX_LEVELS 32

/* Method and shape parameters.
 *   head_dim   d, 64 or 128.
 *   n_q_heads  Hq; n_kv_heads Hkv; Hq/Hkv = G in {1, 2, 4, 8}.  Query head h reads
 *              KV head h / G (contiguous groups); the G heads of a group share one
 *              selection, scored by the mean of their logits (GQA stand-in, since
 *              the importance I of Eq.3 is not defined on the pages).
 *   C          branching factor of the tree, 2..32 (the pages use 16).
 *   k          per-level selection budget, 1..512 (the pages use 256); C*k <= 8192.
 *   dtype      storage of K, V, q, outputs and level tables (recsa_dtype).
 *   rope_base  RoPE base b > 1: pair (j, j+d/2) turns by pos * b^(-2j/d).
 *   scale      logit scale; 0 selects 1/sqrt(d).
 *   pooler_w   pooler logits w[0..C-1].  Stand-in pooler: a parent key is
 *              sum_c softmax(w)_c K_child_c over its present children (Eq.1 with
 *              Pool fixed to a softmax-weighted sum shared by all levels/heads). */
typedef struct {
    int32_t head_dim;
    int32_t n_q_heads;
    int32_t n_kv_heads;
    int32_t C;
    int32_t k;
    int32_t dtype;
    double rope_base;
    float scale;
    float pooler_w[RECSA_MAX_C];
} recsa_config;

typedef struct recsa_tree recsa_tree;   /* opaque host handle; does not own device memory */

/* Sizes of the caller-allocated buffers for a tree of `capacity` tokens per
 * sequence, `batch` sequences and at most `max_queries` queries per kernel wave
 * (decode uses `batch` queries; prefill chunks are processed in waves of
 * max_queries).  Pure host computation.
 *   level_bytes      bytes for the level tables (levels 1.. up to a single root).
 *   workspace_bytes  bytes for the workspace (status word, device lengths, RoPE
 *                    table, per-level selections, split-softmax partials).
 *   n_levels         number of tree levels at capacity, level 0 included.
 * Any output pointer may be NULL.  Errors: RECSA_E_INVAL, RECSA_E_UNSUPPORTED. */
RECSA_API recsa_status recsa_query_sizes(const recsa_config* cfg, int64_t capacity, int32_t batch,
                               int32_t max_queries, size_t* level_bytes,
                               size_t* workspace_bytes, int32_t* n_levels);

/* Bind a tree to caller memory and initialise its workspace on `stream` (status
 * word cleared, all lengths 0, RoPE cos/sin table for positions [0, C*k) computed
 * in fp64 and stored fp32).
 *   k0, v0      level-0 KV cache, element (b, h, t, :) at base + b*s[0] + h*s[1]
 *               + t*s[2] elements, d contiguous.  16-byte aligned; each stride a
 *               multiple of 16 bytes; s[2] >= d.  The library writes rows here
 *               only in recsa_append.
 *   kv_strides  s[3] in elements (host array, copied).
 *   levels      level tables, >= level_bytes, 256-byte aligned.  Level l >= 1 of
 *               KV head h of sequence b is a [rows_l][d] K table and a [rows_l][d]
 *               V table (recsa_level_info gives offsets).
 *   workspace   >= workspace_bytes, 256-byte aligned.
 * On success *out receives a new handle (free with recsa_tree_free). */
RECSA_API recsa_status recsa_tree_init(const recsa_config* cfg, int64_t capacity, int32_t batch,
                             int32_t max_queries, void* k0, void* v0,
                             const int64_t kv_strides[3], void* levels, size_t level_bytes,
                             void* workspace, size_t workspace_bytes, void* stream,
                             recsa_tree** out);

/* Eq.1 over the whole cache: set the length of sequence b to lengths[b] (host
 * array of `batch` values, 0 <= lengths[b] <= capacity) and compute every level
 * l >= 1 from level 0.  Node i of level l pools children C*i .. min(C*i+C-1,
 * n_{l-1}-1): K = sum_c alpha_c K_c with alpha = softmax(w) over the m present
 * children, V = (1/m) sum_c V_c, accumulated in fp64 and rounded once (to nearest
 * even) to the storage dtype; the next level pools the rounded values. */
RECSA_API recsa_status recsa_build(recsa_tree* tree, const int64_t* lengths, void* stream);

/* Append n >= 1 tokens to every sequence: k_new, v_new are device arrays
 * [batch][Hkv][n][d] (contiguous, 16-byte aligned).  Rows are written at the
 * device-side length L of each sequence, then every ancestor node of the new
 * tokens is re-pooled exactly as recsa_build would compute it (build(L) followed
 * by append(n) is bitwise equal to build(L+n)), and L grows by n.  If L + n would
 * exceed capacity the sequence is left unchanged and the status word records
 * RECSA_E_CAPACITY (the host also rejects this synchronously while its own copy
 * of the lengths is current, i.e. outside graph replays).
 * With n == 1 this call writes the new rows and the lengths only (one launch).  The
 * re-pooling of the new tokens' ancestors is carried out by the next call on the
 * handle: recsa_decode does it inside its level-0 launch (a decode at the new
 * position reads none of those ancestors: each is the current node of its level,
 * never scored and never a summary); every other call (recsa_append,
 * recsa_prefill_chunk, recsa_get_status) first runs it as a separate launch on its
 * own stream, and recsa_build makes it unnecessary.  A caller that reads the level
 * tables directly does so after one of those calls. */
RECSA_API recsa_status recsa_append(recsa_tree* tree, const void* k_new, const void* v_new, int32_t n,
                          void* stream);

/* Decode one query per sequence at its last position t = L_b - 1 (so the newest
 * token attends to itself).
 *   q        [batch][Hq][d] device, 16-byte aligned.
 *   out      [batch][Hq][d] device: Eq.4 output, rounded to the storage dtype.
 *            A sequence of length 0 gets zeros.
 *   sel_out  optional [batch][Hkv][NL][k] int32: selected node indices S^(l) of
 *            scored level l at index l-1 (ascending, current node last, -1 where
 *            unused or where the level is above the first scored level).  NL is
 *            recsa_tree_info's n_sel_levels.
 *   counts_out optional [batch][Hkv][NL+1] int32: |A^(l)| at index l for levels
 *            that are scored (index 0: the level-0 list), 0 above them. */
RECSA_API recsa_status recsa_decode(recsa_tree* tree, const void* q, void* out, int32_t* sel_out,
                          int32_t* counts_out, void* stream);

/* One decode step fused into one launch: the same as recsa_append(tree, k_new, v_new,
 * 1, stream) followed by recsa_decode(tree, q, out, sel_out, counts_out, stream) --
 * the same outputs, selections and counts, bit for bit, and the same tree afterwards
 * ("Practical Implications": one token appended and attended per decode step).
 *   k_new, v_new  device [B][Hkv][d] each, the token of every sequence (16-byte
 *                 aligned); q, out, sel_out, counts_out as for recsa_decode.
 * The walk CTAs of the launch write the token's rows at level 0 and re-pool its
 * ancestors; the attention CTAs take the token's rows from k_new / v_new; the last CTA
 * of each sequence advances its length.  Nothing is allocated; the caller keeps
 * ownership of every buffer, which must stay valid until the stream reaches the call.
 * Errors: RECSA_E_INVAL (null or misaligned pointer), RECSA_E_CAPACITY (a sequence
 * at capacity), RECSA_E_UNSUPPORTED (a tree with the gated pooler or with level 0 in
 * host memory: use the two separate calls), RECSA_E_CUDA (a launch failed). */
RECSA_API recsa_status recsa_append_decode(recsa_tree* tree, const void* k_new, const void* v_new,
                                           const void* q, void* out, int32_t* sel_out,
                                           int32_t* counts_out, void* stream);

/* Causal queries of a chunk: row i of sequence b sits at position pos0 + i and
 * must already be in the tree (pos0 + n <= L_b).
 *   Q  [batch][n][Hq][d] device;  O [batch][n][Hq][d] device.
 *   sel_out / counts_out as in recsa_decode with batch*n queries (b-major).
 * Each row is the RecSA output of a tree holding only tokens [0..pos0+i].
 * When the tree was created with max_queries >= 128 (see recsa_tree_info's
 * tc_queries), the rows of a sequence are taken in groups of up to tc_queries, and
 * at the first scored level of the group's last row ("Hierarchical Selection",
 * Eq.3: the list [0..a_t] shared by the group up to each row's cut) the logits of
 * every row and head against every node come from one tensor-core product
 * (split-precision tf32, fp32 accumulation).  Rows then match recsa_decode of the
 * truncated tree up to fp32 rounding of those logits, and their selections agree
 * except at near-ties.  Otherwise every level is scored per row, and each row is
 * bitwise equal to that decode. */
RECSA_API recsa_status recsa_prefill_chunk(recsa_tree* tree, const void* Q, int64_t pos0, int32_t n,
                                 void* O, int32_t* sel_out, int32_t* counts_out, void* stream);

/* Run any pending ancestor re-pooling on `stream`, then read and clear the device
 * status word in stream order (a copy and, if it was set, a clear on `stream`) and
 * synchronise `stream` (not the device).  Returns RECSA_OK or the first device-side
 * error recorded since the last call. */
RECSA_API recsa_status recsa_get_status(recsa_tree* tree, void* stream);

/* Self-test of the device-side timeout path.  Runs one CTA that waits, through the
 * same bounded mbarrier wait every kernel of the library uses, on a barrier that
 * nothing completes.  The wait gives up after its poll limit (about one second),
 * records the timeout in `status_dev` and the kernel returns; no GPU fault, trap or
 * hang is involved.
 *   status_dev  device pointer to one uint32, caller-owned; zeroed here, then
 *               written by the kernel (3 = timeout);
 *   stream      the stream to run on, synchronised before returning.
 * Returns RECSA_E_TIMEOUT when the wait gave up as designed, RECSA_OK if it did not
 * (the path is broken), RECSA_E_INVAL for a NULL pointer, RECSA_E_CUDA on a CUDA
 * error. */
RECSA_API recsa_status recsa_probe_bounded_wait(uint32_t* status_dev, void* stream);

typedef struct {
    int32_t n_levels;       /* levels stored at capacity, level 0 included           */
    int32_t n_sel_levels;   /* NL: highest level that any position can score         */
    int32_t splits;         /* CTAs (a thread-block cluster) per unit for levels >= 1 */
    int32_t splits0;        /* CTAs per unit for level 0                               */
    int64_t capacity;
    int32_t batch;
    int32_t max_queries;
    /* tensor-core prefill path (0 when disabled): rows per product, the length of a
     * logits row, and where the logits of the last product sit in the workspace:
     * fp32 [tc_queries][Hkv][G][tc_row_stride], scaled by the softmax scale, row
     * (q, h, g) = that group's row q, KV head h, query head h*G + g; entry j is node
     * j of the level the product scored.  For diagnostics. */
    int32_t tc_queries;
    int32_t tc_row_stride;
    int64_t tc_logits_offset;
} recsa_tree_info_t;

RECSA_API recsa_status recsa_tree_info(const recsa_tree* tree, recsa_tree_info_t* info);

/* Where level `level` (1 <= level < n_levels) lives inside the `levels` buffer:
 * byte offsets of its K and V tables and rows per (sequence, KV head).  Row i of
 * head h of sequence b is at offset + ((b*Hkv + h)*rows + i)*d*elem_size. */
RECSA_API recsa_status recsa_level_info(const recsa_tree* tree, int32_t level, int64_t* k_offset,
                              int64_t* v_offset, int64_t* rows);

/* Host lengths as the library last set them (exact unless a captured graph was
 * replayed since).  lengths: host array of batch values. */
RECSA_API recsa_status recsa_host_lengths(const recsa_tree* tree, int64_t* lengths);

/* Kernel timing hook.  From the next call on, record CUDA event `start` (a
 * cudaEvent_t, created by the caller with timing enabled) on the call's stream just
 * before the kernel selected by `which` is launched and `stop` just after it:
 *   which = 0: the select/attend pass kernel (every level of every unit), in
 *           recsa_decode and in each prefill wave;
 *   which = -1: the append kernel(s) of recsa_append;  -2: the tensor-core product
 *   of recsa_prefill_chunk (the last one of the call).
 * Records use cudaEventRecordExternal, so they also become event nodes when the
 * call is captured in a CUDA graph.  start = stop = NULL clears the hook.
 * No device memory is touched. */
RECSA_API recsa_status recsa_set_profile_events(recsa_tree* tree, int32_t which, void* start,
                                                void* stop);

/* Decode without any device allocation by the caller or the library.  The paper
 * has no counterpart to this call; it exists for callers that cannot allocate device
 * memory where they call decode (inside a stream capture in global capture mode, in
 * a loop bound to a fixed pre-planned memory budget, or in a runtime with no device
 * allocator for per-call scratch) and so cannot provide recsa_decode's workspace.
 * Same result as recsa_decode on a tree with these buffers and lengths.
 *   cfg, capacity, batch   as for recsa_tree_init (one query per sequence).
 *   k0, v0, kv_strides     level-0 cache, as for recsa_tree_init.
 *   levels, level_bytes    level tables already built by recsa_build/recsa_append
 *                          for these lengths, laid out as recsa_query_sizes states.
 *   lengths                host array [batch]; query b sits at lengths[b] - 1.
 *   q, out                 [batch][Hq][d] device, 16-byte aligned.
 *   status_out             optional device uint32 (4-byte aligned), caller-owned: set
 *                          to 0 at the start of the call, then to the first
 *                          device-side error of this call (3: a bounded wait gave up,
 *                          4: a staging buffer was misaligned).  Read it after the
 *                          stream has reached the end of the call.  NULL: such errors
 *                          are not reported.
 * Scratch: a fixed 8 MiB device array inside the library (held by every GPU that
 * loads it until exit), shared by all calls: calls that may overlap on the GPU race.
 * A shape whose workspace (recsa_query_sizes with max_queries = batch) exceeds 8 MiB
 * is rejected with RECSA_E_CAPACITY.  The first call on a device looks up the array's
 * device address (cudaGetSymbolAddress) with that device current; make that first
 * call before any stream capture.  No cudaMalloc, cudaFree or allocating library
 * routine is called. */
RECSA_API recsa_status recsa_decode_noalloc(const recsa_config* cfg, int64_t capacity,
                                            int32_t batch, const void* k0, const void* v0,
                                            const int64_t kv_strides[3], const void* levels,
                                            size_t level_bytes, const int64_t* lengths,
                                            const void* q, void* out, uint32_t* status_out,
                                            void* stream);

/* Eq.5 ("Pooler Distillation"), forward only: the gated key pooler, used in place of
 * the stand-in pooler by every later recsa_build and recsa_append on the tree (call
 * recsa_build after switching).  For a node with present children x_1..x_m:
 *   mu = mean_c x_c;  sigma = sqrt(mean over children and dims of (x - mu)^2 + 1e-6);
 *   alpha = softmax_c(tau * w . (x_c - mu) / sigma);  p = sum_c alpha_c x_c;
 *   K = mu + g (p - mu) + sigma * W2 SiLU(W1 [mu / rho ; (p - mu) / sigma] + b1).
 * The node's value stays Eq.1's mean of the children's values.  Computed in fp64 with
 * one rounding to the storage dtype; build and append give bit-identical trees.
 *   hidden  h, the MLP's hidden width, 1..64 (the fp64 weights are staged in shared
 *           memory); larger widths return RECSA_E_UNSUPPORTED.
 *   w       device fp64 [d];  W1t device fp64 [2d][h] (W1 transposed);  b1 device
 *           fp64 [h];  W2t device fp64 [h][d] (W2 transposed).  Caller-owned, 8-byte
 *           aligned, kept alive and unchanged while the tree uses them.
 * p == NULL switches back to the stand-in pooler.  The pages do not give the trained
 * parameters; the tests use seeded ones. */
typedef struct {
    int32_t hidden;
    double tau, g, rho;
    const double* w;
    const double* W1t;
    const double* b1;
    const double* W2t;
} recsa_gated_pooler;
RECSA_API recsa_status recsa_tree_set_gated_pooler(recsa_tree* tree, const recsa_gated_pooler* p);

/* Level 0 in host memory ("Efficiency Results": decode at 1M and 2M tokens with the KV
 * cache offloaded to the host; "Practical Implications": the levels above 0 are under
 * 7 % of the cache).  A tree whose k0/v0 passed to recsa_tree_init are pinned host
 * memory (cudaHostAlloc / cudaMallocHost, mapped into the device address space; they
 * must both be host or both be device memory, else RECSA_E_INVAL) keeps level 0 there
 * and its levels >= 1 in the device level tables.  Build and append read and write
 * level 0 through the host mapping.  recsa_decode then needs a device staging buffer:
 * after the levels >= 1 have selected S^(1), the rows of each query's level-0 list (the
 * children of S^(1), Eq.3) are gathered from host memory into it, and level 0 is
 * attended from there; the result is the same as with level 0 in device memory.
 * recsa_prefill_chunk returns RECSA_E_UNSUPPORTED on such a tree.
 *   recsa_offload_staging_bytes: bytes of the staging buffer for `batch` sequences,
 *     2 * batch * Hkv * C * k * d * element size.
 *   recsa_tree_set_offload_staging: the caller's device buffer (256-byte aligned, at
 *     least that many bytes), used by every later decode.  RECSA_E_UNSUPPORTED when
 *     level 0 is in device memory; a decode on a host-level-0 tree without one returns
 *     RECSA_E_UNSUPPORTED. */
RECSA_API recsa_status recsa_offload_staging_bytes(const recsa_config* cfg, int32_t batch,
                                                   size_t* bytes);
RECSA_API recsa_status recsa_tree_set_offload_staging(recsa_tree* tree, void* staging,
                                                      size_t bytes);

/* Free the host handle.  Device memory stays with the caller. */
RECSA_API recsa_status recsa_tree_free(recsa_tree* tree);

RECSA_API const char* recsa_status_str(recsa_status s);

#ifdef __cplusplus
}
#endif
#endif /* RECSA_H */
