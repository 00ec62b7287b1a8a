/*
 * csa.h -- C ABI of libcsa: the compressed-attention decode step of
 * DeepSeek-V4-style CSA / HCA layers on one NVIDIA B200 (sm_100a).
 *
 * What is computed (one decode step of one layer for a batch of requests):
 *
 *   csa_compress_append   token-level compressor + cache write
 *       Source: page "V4终于终于终于终于是来了", section "CSA——压缩稀疏注意力"
 *       (every 4 tokens' KV become one entry) and section "HCA——重度压缩注意力"
 *       (128 tokens become one entry; state cache holds the last 128 raw
 *       tokens and the unfinished tails; classic cache blocks of 128 raw
 *       tokens hold 32 CSA entries and 1 HCA entry); page "深度解读DeepSeek V4
 *       看清Benchmark以外的三个范式创新", section 01, "混合注意力的精细解剖"
 *       (CSA windows overlap).
 *   csa_index_scores      lightning indexer, FP4 query x FP4 keys
 *       Source: page "V4终于终于终于终于是来了", section "CSA——压缩稀疏注意力"
 *       (down/up-projected index queries, ReLU, scores against compressed
 *       index keys); podcast summary page, section "2.1 推理与计算效率" (FP4
 *       on the indexer path).
 *   csa_topk              top-k selector
 *       Source: page "V4终于终于终于终于是来了", section "CSA——压缩稀疏注意力"
 *       (top 512 / 1024 compressed entries).
 *   csa_hca_decode_attn   multi-query attention over the selected (CSA) or all
 *                         (HCA) compressed entries plus the 128-token raw
 *                         window, with a per-head sink logit
 *       Source: page "V4终于终于终于终于是来了", sections "CSA——压缩稀疏注意力"
 *       and "HCA——重度压缩注意力" (MQA core, sliding window, sink logit in the
 *       denominator, RoPE on the last 64 dims, FP8 + BF16 KV).
 *
 * The precise definition of every step (gating form, overlap geometry,
 * quantiser rules, RoPE pairing and positions, tie-break, visibility) is the
 * specification shipped with this library; the points the pages leave open
 * are settled there and repeated in the comments below.
 *
 * Conventions that hold for every function:
 *   - All device pointers are CUDA device memory owned by the caller; they
 *     must stay valid until the work queued on `stream` has finished.
 *   - The library never allocates device memory.  The caller hands one
 *     device buffer (the arena) to csa_cache_init; the library carves the
 *     state cache, the classic-cache page pool, page tables and lengths out
 *     of it.  Host memory owned by the library: the handle and its host-side
 *     page allocator.
 *   - Every compute call is asynchronous on `stream` (NULL = legacy default
 *     stream).  Argument errors are detected on the host and returned before
 *     anything is launched.  Errors found on the device (request id out of
 *     range, capacity exceeded, a top-k index out of range) are recorded in a
 *     device error word, the offending work item is skipped, and
 *     csa_check_device_error reports them.  No kernel traps.
 *   - No C++ exception crosses the ABI.  csa_last_error() returns a
 *     thread-local message for the last failing call.
 *   - Results are batch-invariant: a request's outputs do not depend on the
 *     batch size, its position in the batch or the other requests, and the
 *     two launch variants (csa_variant) return identical bits.
 *   - BF16 values are passed as uint16_t bit patterns.
 *   - A cache holds one storage format (csa_fmt): the pages' mixed FP8 /
 *     BF16 / MXFP4 format, or plain fp32 for the tiny fp32 configuration.
 */
#ifndef CSA_H_
#define CSA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct csa_cache csa_cache_t;          /* opaque host-side handle        */
typedef struct CUstream_st* csa_stream_t;      /* same type as cudaStream_t      */

typedef enum {
  CSA_OK = 0,
  CSA_ERR_ARG = -1,             /* invalid argument (host-side check)             */
  CSA_ERR_CAPACITY = -2,        /* page pool or request capacity exhausted        */
  CSA_ERR_CUDA = -3,            /* a CUDA runtime call failed                     */
  CSA_ERR_DEVICE_TIMEOUT = -4,  /* a bounded device-side wait gave up             */
  CSA_ERR_DEVICE_BOUNDS = -5    /* a device-side index check failed               */
} csa_status;

typedef enum {
  CSA_VARIANT_AUTO = 0,         /* library picks by batch size                    */
  CSA_VARIANT_HIGH_OCC = 1,     /* launch shape for a well-fed GPU (large batch)  */
  CSA_VARIANT_LOW_OCC = 2       /* launch shape for an under-fed GPU (small batch)*/
} csa_variant;                  /* both return identical bits                     */

/*
 * Flag OR-ed into the variant of csa_hca_decode_attn: the attention may read
 * the requests' lengths, their window rows, q and sink before the kernel
 * queued directly ahead of it on the stream has finished (it still waits for
 * that kernel before it reads a top-k list or a compressed entry, and before
 * it writes anything).  Set it only when that kernel writes none of those
 * inputs: in a decode step of a CSA layer, when the call directly follows
 * the step's csa_index_topk (the step's csa_compress_append having been
 * queued before it).  The results are the same with or without it.
 */
#define CSA_ATTN_STATE_READY 0x100

/* Storage format of a cache (csa_cfg.fmt). */
typedef enum {
  CSA_FMT_MIXED = 0,            /* the pages' formats: KV rows FP8 E4M3 (non-RoPE
                                   dims, one fp32 scale per row) + BF16 (RoPE dims),
                                   index keys MXFP4; queries and outputs BF16     */
  CSA_FMT_F32 = 1               /* every stored vector, query and output in fp32
                                   (the tiny fp32 configuration)                  */
} csa_fmt;

/* Regions addressed by csa_debug_rows. */
typedef enum {
  CSA_REGION_KV = 0,            /* compressed KV entries, by entry index          */
  CSA_REGION_INDEX = 1,         /* compressed index keys (CSA layers), by entry   */
  CSA_REGION_WINDOW = 2         /* raw-token window rows, by token position       */
} csa_region;

/*
 * Layer configuration, shared by all layers of the cache.  Layers
 * 0 .. n_csa_layers-1 are CSA layers, the next n_hca_layers are HCA layers.
 *   H        query heads (one shared KV head: multi-query attention), <= 128
 *   D        head dim, multiple of 32, 64 <= D <= 512
 *   D_rope   RoPE dims (the last D_rope dims of q and KV), even, 16 <= D_rope
 *            <= 64, D - D_rope a multiple of 16
 *   H_I      indexer heads, 1 <= H_I <= 64 (ignored when n_csa_layers == 0)
 *   d_I      index dim, one of 32, 64, 96, 128
 *   window   raw-token sliding window; must be 128
 *   max_requests            request slots
 *   max_pages_per_request   pool pages a request may hold
 *   pool_pages              pages in the shared pool
 *                           (a page = 4 classic-cache blocks = 512 raw tokens:
 *                           128 CSA entries and 4 HCA entries per layer)
 *   rope_base               RoPE frequency base (10000)
 *   fmt                     storage format (csa_fmt); 0 = CSA_FMT_MIXED
 * Entry geometry (fixed): CSA m = 4 with windows of 8 tokens overlapping by 4;
 * HCA m = 128, no overlap.
 */
typedef struct {
  int32_t n_csa_layers;
  int32_t n_hca_layers;
  int32_t H;
  int32_t D;
  int32_t D_rope;
  int32_t H_I;
  int32_t d_I;
  int32_t window;
  int32_t max_requests;
  int32_t max_pages_per_request;
  int32_t pool_pages;
  float rope_base;
  int32_t fmt;
} csa_cfg;

/* Bytes of device memory the arena must have for `cfg` (0 if cfg invalid). */
size_t csa_cache_required_bytes(const csa_cfg* cfg);

/*
 * Initialise a cache in the caller's device buffer `dev_mem` (256-byte
 * aligned, `bytes` >= csa_cache_required_bytes).  Position biases of the
 * compressor gates are copied in from host memory:
 *   b_pos_csa  float [n_csa_layers][8][D]    bias of KV gates, CSA window slot
 *   b_pos_idx  float [n_csa_layers][8][d_I]  bias of index-key gates
 *   b_pos_hca  float [n_hca_layers][128][D]  bias of KV gates, HCA window slot
 * (NULL allowed when the corresponding layer count is 0).  Synchronous.  All
 * request lengths start at 0 and no pages are allocated.
 */
csa_status csa_cache_init(const csa_cfg* cfg, void* dev_mem, size_t bytes,
                          const float* b_pos_csa, const float* b_pos_idx,
                          const float* b_pos_hca, csa_cache_t** out);

/* Release the host handle (the arena stays the caller's). */
void csa_cache_destroy(csa_cache_t* cache);

/*
 * Give request slot `req` room for `capacity_tokens` raw tokens: pages are
 * taken from the pool (in the allocator's order, so a request's pages are
 * not contiguous) and its page table is written; every layer's length is
 * reset to 0.  A slot that already holds pages is released first.
 * Synchronous (device copies on the legacy stream).  CSA_ERR_CAPACITY when
 * the pool or max_pages_per_request is too small.
 */
csa_status csa_request_alloc(csa_cache_t* cache, int32_t req, int64_t capacity_tokens);

/* Return request slot `req`'s pages to the pool; its lengths become 0. */
csa_status csa_request_free(csa_cache_t* cache, int32_t req);

/*
 * Compressor + cache write for `n_tok` new tokens of each of `n` requests of
 * layer `layer`.  Request i appends tokens at positions L_i .. L_i+n_tok-1,
 * L_i its current length (held on the device).
 *   req_ids   device int32 [n]               request slots (distinct)
 *   kv_cand   device float [n][n_tok][D]     KV candidates c_t
 *   kv_gate   device float [n][n_tok][D]     gate logits z_t
 *   idx_cand  device float [n][n_tok][d_I]   index-key candidates (CSA only)
 *   idx_gate  device float [n][n_tok][d_I]   index-key gate logits (CSA only)
 * For every completed CSA entry j (4j+3 < L_i+n_tok) the gated pool
 *   e = sum_t softmax_t(z_t + b_pos[t-4j+4]) * c_t over t in [4j-4, 4j+4), t >= 0
 * is rotated (RoPE at position 4j on the last D_rope dims) and stored as FP8
 * E4M3 (first D-D_rope dims, one fp32 scale amax/448 per row) + BF16 (RoPE
 * dims) in classic-cache block j/32 (page j/128); the index key pools (idx_cand, idx_gate)
 * the same way without RoPE and is stored as MXFP4 (E2M1 + one E8M0 scale
 * per 32 values).  HCA entry j pools t in [128j, 128j+128) and is rotated at
 * 128j.  Each token's own KV, rotated at its position, is written to the raw
 * window ring; the unfinished tails are kept in the state cache.
 * Returns before the work runs.  Capacity overflow and bad request ids are
 * device errors (the request's append is skipped).
 */
csa_status csa_compress_append(csa_cache_t* cache, int32_t layer, int32_t n,
                               const int32_t* req_ids, int32_t n_tok,
                               const float* kv_cand, const float* kv_gate,
                               const float* idx_cand, const float* idx_gate,
                               csa_stream_t stream);

/*
 * Lightning-indexer scores of each query against every completed index key
 * of its request (CSA layers only).  For query i (request req_ids[i], whose
 * length is T = L after the step's append, N = floor(T/4) entries):
 *   scores[i*ld + j] = sum_h w[i][h] * max(0, q^_h . k^_j),   j < N
 * where, in the mixed format, q^_h is q_idx[i][h] quantised to MXFP4 in the
 * kernel and k^_j the stored MXFP4 key (block-scaled FP4 tensor-core MMA,
 * fp32 accumulation); in the fp32 format q^_h = q_idx[i][h] and k^_j the
 * stored fp32 key (fp32 FMA, d ascending, heads ascending).  Entries j >= N
 * of the row are not written.  Both variants return identical bits: the
 * mixed format's persistent grid is two CTAs per SM (AUTO, HIGH_OCC) or one
 * (LOW_OCC), each owning a different range of the (query, tile) list; the
 * fp32 format gives a query one CTA (HIGH_OCC) or several (LOW_OCC; AUTO
 * when n is below the SM count).
 *   q_idx    device float [n][H_I][d_I]
 *   w        device float [n][H_I]
 *   scores   device float [n][ld]   (ld >= the largest N; checked on device)
 *   n_valid  device int32 [n]       receives N per query
 */
csa_status csa_index_scores(const csa_cache_t* cache, int32_t layer, int32_t n,
                            const int32_t* req_ids, const float* q_idx, const float* w,
                            float* scores, int64_t ld, int32_t* n_valid,
                            csa_variant variant, csa_stream_t stream);

/*
 * Top-k per query row: the k largest of scores[i*ld + 0 .. n_valid[i]-1];
 * equal scores go to the lower index; -0.0 equals +0.0; output ascending,
 * padded with -1 when n_valid[i] < k.
 *   idx_out  device int32 [n][k]
 * Scores must not be NaN (a NaN is ordered above +inf).  One thread-block
 * cluster per query: 16 blocks (LOW_OCC), 8 (HIGH_OCC), and for AUTO the
 * largest of 16, 8 and 4 whose n clusters the device holds at once (else
 * 4); rows of at most 4096 scores take a single block (AUTO, HIGH_OCC) or
 * 8 (LOW_OCC).  Every form returns identical indices.
 */
csa_status csa_topk(const float* scores, int64_t ld, const int32_t* n_valid, int32_t n,
                    int32_t k, int32_t* idx_out, csa_variant variant, csa_stream_t stream);

/*
 * csa_index_scores followed by csa_topk in one launch: the same scores,
 * n_valid and indices, bit for bit (page "V4终于终于终于终于是来了", section
 * "CSA——压缩稀疏注意力": the lightning indexer scores every compressed index
 * key and the top-k selector keeps the best; podcast summary page, section
 * "2.1 推理与计算效率": FP4 on the indexer path).
 *
 * While the indexer's thread blocks score their tiles they count each
 * query's score keys (order-preserving 32-bit keys) over their top 12 bits;
 * once every block of a query has added its counts they find the bin that
 * holds the k-th largest key, write their own keys at or above that bin
 * (the candidates, in index order) to the workspace, and the last block of
 * the query selects exactly among the candidates (when more than 8192 keys
 * fall at or above the bin, it radix-selects over the whole score row
 * instead).  The scores are still written to `scores`.  The blocks wait for
 * one another, so the kernel is launched cooperatively (all blocks resident);
 * every wait is bounded (CSA_ERR_DEVICE_TIMEOUT).
 *   q_idx, w, scores, ld, n_valid  as csa_index_scores
 *   k          top-k, >= 1
 *   idx_out    device int32 [n][k]: ascending, -1 padded, as csa_topk
 *   workspace  device scratch of csa_index_topk_workspace_bytes(cache, n, ld)
 *              bytes, 256-byte aligned, owned by the caller; the call clears
 *              the part it needs (one memset queued on `stream`); it must not
 *              be used by other work until the call's work has finished.
 * Caches in the fp32 format run the two separate kernels instead (same
 * results; the workspace is not used).
 */
size_t     csa_index_topk_workspace_bytes(const csa_cache_t* cache, int32_t n, int64_t ld);
csa_status csa_index_topk(const csa_cache_t* cache, int32_t layer, int32_t n,
                          const int32_t* req_ids, const float* q_idx, const float* w,
                          float* scores, int64_t ld, int32_t* n_valid, int32_t k,
                          int32_t* idx_out, void* workspace, size_t workspace_bytes,
                          csa_variant variant, csa_stream_t stream);

/*
 * Multi-query attention of each query over its rows: for CSA layers the
 * entries listed in topk_idx[i][0..k) in list order (-1 = an empty row), for
 * HCA layers (topk_idx == NULL) every completed entry in order, then the raw
 * window of positions max(0, t-127) .. t, t = L-1 the query's own position.
 * K = V = the stored row (mixed format: FP8 x scale, BF16; fp32 format: the
 * fp32 row).  With q rotated at t:
 *   u_hr = scale * q_h . K_r,  mu_h = max(max_r u_hr, sink_h)
 *   out_h = sum_r e^{u_hr-mu_h} V_r / (sum_r e^{u_hr-mu_h} + e^{sink_h-mu_h})
 *   q     device [n][H][D] before RoPE, 16-byte aligned: BF16 bit patterns
 *         (uint16) in the mixed format, fp32 in the fp32 format
 *   sink  device float [H]
 *   out   device [n][H][D], the type of q
 * The mixed format runs QK^T and PV on the tensor cores (BF16 operands, fp32
 * accumulation, P rounded to BF16); the fp32 format runs them as fp32 FMA
 * chains on the CUDA cores (tf32 would keep only 10 mantissa bits).
 * Source: page "V4终于终于终于终于是来了", sections "CSA——压缩稀疏注意力"
 * and "HCA——重度压缩注意力".
 *
 * Reduction order: the rows are cut into tiles of 128; each tile yields
 * (max, sum of exponentials, weighted sum of V).  The tiles are grouped
 * into chunks of consecutive tiles (one tile per chunk on CSA layers,
 * max(1, floor(tiles / 8)) on HCA layers for the query's own tile count);
 * the tiles of a chunk are folded in order into the
 * chunk's result and the chunk results are folded in order, the sink last.
 * The order depends on the query and the layer kind alone, never on the
 * batch.
 *
 * Launch variants (page "DeepSeek不惜代价保住它！V4关键特性被挖出来了",
 * section "牺牲了什么": two decode-attention kernels for a well-fed and an
 * under-fed GPU that agree bit for bit):
 *   CSA_VARIANT_HIGH_OCC  one thread block per (query, 32 heads) walks all
 *                         tiles; `workspace` is not used (may be NULL).
 *   CSA_VARIANT_LOW_OCC   one thread block per (query, 32 heads, chunk);
 *                         the chunks' results go to `workspace` and a second
 *                         kernel folds them -- or, when every (query, 32
 *                         heads) group of blocks fits on the GPU at once as
 *                         one thread-block cluster (at most 16 chunks), the
 *                         blocks of a cluster fold the results through
 *                         distributed shared memory instead, in the same
 *                         order and with the same arithmetic.  Needs
 *                         workspace_bytes >= csa_attn_workspace_bytes(cache,
 *                         layer, n, k) and a 16-byte aligned workspace, else
 *                         CSA_ERR_ARG (whichever fold runs).
 *   CSA_VARIANT_AUTO      LOW_OCC when the workspace suffices and HIGH_OCC
 *                         would leave SMs idle, else HIGH_OCC.
 * All three return identical bits.  Any of them may carry the flag
 * CSA_ATTN_STATE_READY (defined with csa_variant above).  The workspace is
 * scratch owned by the caller; its contents before and after the call are
 * irrelevant, and it must not be used by other work on the stream until the
 * call's kernels finish.
 */
size_t     csa_attn_workspace_bytes(const csa_cache_t* cache, int32_t layer, int32_t n, int32_t k);
csa_status csa_hca_decode_attn(const csa_cache_t* cache, int32_t layer, int32_t n,
                               const int32_t* req_ids, const void* q,
                               const int32_t* topk_idx, int32_t k, const float* sink,
                               float scale, void* out, void* workspace,
                               size_t workspace_bytes, csa_variant variant,
                               csa_stream_t stream);

/*
 * csa_hca_decode_attn without a caller workspace, for callers that cannot
 * allocate device memory: an engine whose memory planner hands out every
 * device buffer ahead of time and forbids allocation while serving, or a
 * plugin that only receives device pointers and has no allocator of its own.
 * (The source pages have no counterpart; this is a library convenience.)
 *
 * Same arguments and results as csa_hca_decode_attn with
 * CSA_VARIANT_LOW_OCC (identical bits), except that the tiles' partials go
 * to a 16 MiB array built into the library instead of `workspace`:
 *   - every GPU that loads libcsa holds those 16 MiB until the process exits;
 *   - a batch whose scratch (csa_attn_workspace_bytes) exceeds 16 MiB is
 *     rejected with CSA_ERR_CAPACITY before anything is launched.  The
 *     scratch holds one partial per chunk of tiles: n x chunks x H x
 *     (4 D + 8) bytes; with H = 128 and D = 512 that allows
 *     n x chunks <= 63.  On CSA layers a chunk is one tile and chunks =
 *     ceil((k + 128) / 128) (k = 1024: up to 7 queries; 4 queries need about
 *     9.5 MiB).  On HCA layers a query has at most 15 chunks (fewer when
 *     the cache's capacity holds fewer than 15 tiles), so at H = 128,
 *     D = 512 up to 4 queries fit whatever the capacity;
 *   - the first call on each device looks up the array's device address;
 *     make that first call before any stream capture;
 *   - all calls share the array: calls whose kernels may overlap on the GPU
 *     (different streams, or different threads on one device) race on it and
 *     must be ordered by the caller.  Nothing in it needs clearing between
 *     calls.
 * The call allocates no device memory.
 */
csa_status csa_hca_decode_attn_noalloc(const csa_cache_t* cache, int32_t layer, int32_t n,
                                       const int32_t* req_ids, const void* q,
                                       const int32_t* topk_idx, int32_t k, const float* sink,
                                       float scale, void* out, csa_stream_t stream);

/* ---------------------------------------------------------------------
 * One decode step with host buffers: the step's inputs are copied from host
 * memory, the step runs, and its output is copied back to host memory, all
 * on `stream`.  Source: the same four steps as above (page
 * "V4终于终于终于终于是来了", sections "CSA——压缩稀疏注意力" and
 * "HCA——重度压缩注意力"): csa_compress_append of one token, on a CSA layer
 * csa_index_scores and csa_topk (variant AUTO), then csa_hca_decode_attn
 * (variant AUTO, with CSA_ATTN_STATE_READY on a CSA layer).
 *
 *   host_in   pinned host buffer of csa_decode_step_input_bytes(cache,
 *             layer, n) bytes holding, each field on a 256-byte boundary and
 *             in this order:  c [n][D] fp32, z [n][D] fp32 (the token's KV
 *             candidate and gate logits); on a CSA layer c_I [n][d_I] fp32,
 *             z_I [n][d_I] fp32, q_I [n][H_I][d_I] fp32, w [n][H_I] fp32;
 *             last q [n][H][D] (BF16, or fp32 in the fp32 format).
 *   host_out  pinned host buffer [n][H][D], the type of q.
 *   req_ids   device int32 [n]; sink device fp32 [H]; scale as for
 *             csa_hca_decode_attn; k the top-k size (CSA layers, 1..8192).
 *   dev_buf   caller device scratch of csa_decode_step_dev_bytes(cache,
 *             layer, n, k) bytes, 256-byte aligned (the inputs' copy, the
 *             scores, counts and indices, the attention workspace, the
 *             output before its copy), owned by the caller.
 * The inputs before q travel first; q travels on a second stream owned by
 * the cache, beside the append and the selection, and the attention waits
 * for it.  When host_in is page-locked (pinned or registered) the inputs
 * are read by copy kernels straight from host memory, and when
 * host_out is, the attention writes the output straight into it: no
 * copy-engine transfer (each costs about 12 us of fixed latency) on the
 * step's critical path.  Other host memory goes through cudaMemcpyAsync.  The call is asynchronous: host_in must not change, and
 * host_out must not be read, until the stream has passed the call.  It can
 * be captured in a CUDA graph (the host pointers are then fixed).  Calls on
 * one cache must not run concurrently from several host threads (the
 * second stream is shared).  Errors: as the four calls it makes.
 * ------------------------------------------------------------------- */
size_t     csa_decode_step_input_bytes(const csa_cache_t* cache, int32_t layer, int32_t n);
size_t     csa_decode_step_dev_bytes(const csa_cache_t* cache, int32_t layer, int32_t n, int32_t k);
csa_status csa_decode_step(csa_cache_t* cache, int32_t layer, int32_t n, const int32_t* req_ids, int32_t k,
                           const float* sink, float scale, const void* host_in, void* host_out,
                           void* dev_buf, size_t dev_bytes, csa_stream_t stream);

/* ---------------------------------------------------------------------
 * A chunk of queries with causal visibility (prefill): n requests each
 * append n_tok (1 .. 128) new tokens together, and every one of those
 * tokens is also a query.  Source: the data flow of page
 * "V4终于终于终于终于是来了", section "CSA——压缩稀疏注意力" (compressor,
 * indexer, top-k, attention over the selected entries and the 128-token
 * window), applied to every token of a chunk; the pages describe the decode
 * step, and the reading taken here is that the query at position t sees
 * exactly what a decode query at t sees: the tokens 0 .. t, hence the
 * compressed entries completed by token t (floor((t + 1) / 4) on CSA
 * layers, floor((t + 1) / 128) on HCA layers), its own window
 * max(0, t - 127) .. t and RoPE at position t.  The results are
 * bit-identical to appending the chunk's tokens one at a time and running
 * the decode calls after each (batch invariance), whatever n_tok and the
 * chunk's other requests.
 *
 * Steps, all on `stream`: copy each request's window ring to the workspace
 * (the chunk's append overwrites up to n_tok of its rows, which the chunk's
 * early queries still see), csa_compress_append of the n_tok tokens, on a
 * CSA layer the index scores of the n x n_tok queries over their visible
 * keys and csa_topk, then the attention.
 *
 *   req_ids    device int32 [n], distinct requests
 *   kv_cand, kv_gate, idx_cand, idx_gate   as csa_compress_append with
 *              n_tok tokens: [n][n_tok][D] and [n][n_tok][d_I] fp32
 *   q          device [n][n_tok][H][D], BF16 (fp32 in the fp32 format),
 *              16-byte aligned, before RoPE
 *   q_idx, w   CSA layers: device fp32 [n][n_tok][H_I][d_I] and [n][n_tok][H_I]
 *   k          top-k size (CSA layers, 1 .. 8192)
 *   sink, scale  as csa_hca_decode_attn
 *   out        device [n][n_tok][H][D], the type of q
 *   topk_out   CSA layers: device int32 [n][n_tok][k] for the selected
 *              entries, as csa_topk writes them, or NULL (they then stay in
 *              the workspace)
 *   workspace  caller device scratch of csa_prefill_workspace_bytes(cache,
 *              layer, n, n_tok, k, variant) bytes, 256-byte aligned (ring
 *              copies, per-query request ids, scores [n n_tok][ld] with
 *              ld = max(128 x max_pages_per_request, 128), counts, indices,
 *              the split attention's partials when the variant takes it)
 *   variant    AUTO / HIGH_OCC / LOW_OCC, as the three calls (no flags);
 *              every variant returns identical bits
 * Limits: n * n_tok <= 65535.  Errors: CSA_ERR_ARG for a bad shape, a NULL
 * or a short or misaligned workspace (nothing launched); otherwise as the
 * calls it makes.  Asynchronous.
 * csa_prefill_workspace_bytes returns 0 for a bad shape.
 * ------------------------------------------------------------------- */
size_t     csa_prefill_workspace_bytes(const csa_cache_t* cache, int32_t layer, int32_t n, int32_t n_tok,
                                       int32_t k, csa_variant variant);
csa_status csa_prefill_chunk(csa_cache_t* cache, int32_t layer, int32_t n, const int32_t* req_ids,
                             int32_t n_tok, const float* kv_cand, const float* kv_gate,
                             const float* idx_cand, const float* idx_gate, const void* q,
                             const float* q_idx, const float* w, int32_t k, const float* sink,
                             float scale, void* out, int32_t* topk_out, void* workspace,
                             size_t workspace_bytes, csa_variant variant, csa_stream_t stream);

/* ---------------------------------------------------------------------
 * Batch-invariant projection GEMM:  Y[t][o] = sum_k X[t][k] W[o][k]
 * (BF16 operands, fp32 accumulation), for the projections around the path:
 * hidden state -> compressor candidates and gates, query down-projection to
 * d_c and up-projection to the (index) query heads, index head weights
 * (page "V4终于终于终于终于是来了", section "CSA——压缩稀疏注意力"); and the
 * grouped output projection, 16 groups of 8 heads x 512 dims projected
 * separately, then to the model width (page "深度解读DeepSeek V4 看清
 * Benchmark以外的三个范式创新", section 01, "「精度补偿」的无限套娃游戏").
 *
 * Batch invariance (page "DeepSeek不惜代价保住它！V4关键特性被挖出来了",
 * section "牺牲了什么"): a token's output never depends on the batch.  The
 * weight rows are the MMA's M (128 per tile), the tokens its N, always in
 * chunks of 32 (zero padded); the K order is fixed.  A weight with few row
 * tiles has its K range cut into a number of parts (enough to give every
 * SM two CTAs, each part at least 256 K values) that depends on the
 * weight's shape and the device's SM count alone, never on the batch, and
 * the parts are summed in part order (by whichever CTA of a row tile
 * finishes last; the order of the sum does not depend on which one).
 *
 * Groups: with `groups` (1 .. 65535) > 1 the weight is block diagonal; group g's rows
 * (n_out / groups of them, a multiple of 128) read the columns
 * [g k_in / groups, (g + 1) k_in / groups) of X, and the host weight holds
 * only those k_in / groups columns per row: W is [n_out][k_in / groups].
 *
 *   csa_gemm_weight_bytes   device bytes of a packed weight (0 for a bad shape)
 *   csa_gemm_pack_weight    host BF16 W (row-major, as above) -> packed
 *                           device tiles; synchronous
 *   csa_gemm_workspace_bytes  scratch of one call (packed activations, and
 *                           when K is split the parts' partials and one
 *                           counter per 128-row tile)
 *   csa_gemm_bf16           X device BF16 [n_tok][k_in], 1 <= n_tok <= 256.
 *                           Y is written as n_seg (1 .. 8) row segments:
 *                           rows [r_s, r_s + segs[s].rows) of Y go to the
 *                           device buffer segs[s].y as a contiguous
 *                           [n_tok][segs[s].rows] matrix, BF16 when
 *                           segs[s].bf16 != 0, else fp32 (the rows add up
 *                           to n_out; one fused weight then feeds several
 *                           outputs).  `segs` is host memory.  workspace
 *                           256-byte aligned, owned by the caller, not used
 *                           by other work until the call's kernels finish.
 *                           Asynchronous on `stream`.
 *   csa_gemm_check_device_error  read and clear the GEMM's device error word
 *                           (a bounded pipeline wait that gave up);
 *                           synchronises `stream`.
 * ------------------------------------------------------------------- */
typedef struct {
  int32_t rows;                 /* rows of Y in this segment                      */
  int32_t bf16;                 /* nonzero: BF16 output, else fp32                */
  void* y;                      /* device [n_tok][rows]                           */
} csa_gemm_out;

size_t     csa_gemm_weight_bytes(int32_t n_out, int32_t k_in, int32_t groups);
csa_status csa_gemm_pack_weight(const uint16_t* w_host, int32_t n_out, int32_t k_in, int32_t groups,
                                void* w_dev, size_t bytes);
size_t     csa_gemm_workspace_bytes(int32_t n_out, int32_t k_in, int32_t groups, int32_t n_tok);
csa_status csa_gemm_bf16(const void* w_packed, int32_t n_out, int32_t k_in, int32_t groups,
                         const uint16_t* x, int32_t n_tok, int32_t n_seg, const csa_gemm_out* segs,
                         void* workspace, size_t workspace_bytes, csa_stream_t stream);
csa_status csa_gemm_check_device_error(csa_stream_t stream);

/*
 * Read and clear the device error word (synchronises `stream`).  Returns
 * CSA_OK or the first device error recorded since the last check;
 * csa_last_error() then describes it.
 */
csa_status csa_check_device_error(csa_cache_t* cache, csa_stream_t stream);

/* Number of CUDA kernels libcsa has queued since it was loaded (all
 * threads, all caches).  A library-side count for measurement, not a
 * device-side event: the kernels may still be pending. */
uint64_t   csa_launch_count(void);

/* Thread-local description of the last failing call ("" if none). */
const char* csa_last_error(void);

/* ---------------------------------------------------------------------
 * Test helpers (synchronous).  They move rows between host memory and the
 * cache in a packed host format, so that tests can fill a cache from
 * known codes and read back what the kernels stored.
 *   CSA_REGION_KV / CSA_REGION_WINDOW rows: D-D_rope bytes E4M3 codes, then
 *     D_rope BF16 values (2 bytes each, little endian), then one fp32 scale.
 *   CSA_REGION_INDEX rows: d_I/2 bytes of packed E2M1 codes (element 2i in
 *     the low nibble of byte i), then d_I/32 E8M0 scale bytes.
 * `first`/`count` are entry indices (KV, INDEX) or token positions (WINDOW;
 * only the last 128 positions of the current length are held).
 * ------------------------------------------------------------------- */
size_t     csa_debug_row_bytes(const csa_cache_t* cache, int32_t region);
csa_status csa_debug_rows(csa_cache_t* cache, int32_t layer, int32_t req, int32_t region,
                          int64_t first, int64_t count, void* host, int32_t write);
csa_status csa_debug_set_length(csa_cache_t* cache, int32_t layer, int32_t req, int64_t len);
int64_t    csa_debug_get_length(csa_cache_t* cache, int32_t layer, int32_t req);

/*
 * Test helper for the device-side failure path: queue one thread block that
 * waits on a shared-memory barrier nothing arrives on, through the same
 * bounded-wait routine the tensor-core kernels use, with a limit of
 * `limit_us` microseconds (1 .. 1000000).  The wait gives up, the block
 * records a timeout in the cache's device error word and returns, so that
 * csa_check_device_error then reports CSA_ERR_DEVICE_TIMEOUT and the context
 * stays usable.  Asynchronous on `stream`; CSA_ERR_ARG for a NULL cache or a
 * limit out of range.
 */
csa_status csa_debug_wait_timeout(csa_cache_t* cache, int32_t limit_us, csa_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif  /* CSA_H_ */
