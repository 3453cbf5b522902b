/*
 * dca.h -- C ABI of the B200 (sm_100a) Dual Chunk Attention prefill library.
 *
 * Dual Chunk Attention (DCA) is causal grouped-query attention whose RoPE
 * positions are remapped per (query i, key j) pair so that every relative
 * distance stays below the pretraining window c.  With chunk size s, local
 * window w, n_x = x / s and r_x = x mod s (chunks start at token 0):
 *   key position   Pk(j)   = j mod s                     (periodic key index)
 *   query position Pq(i,j) = r_i        if n_i == n_j    (intra-chunk)
 *                          = s + r_i    if n_i - n_j == 1 and r_i < w
 *                                                         (successive chunk, local window)
 *                          = c - 1      otherwise         (inter-chunk: fixed large index)
 *   logit = m^2 / sqrt(d) * < R(Pq) q_i, R(Pk) k_j >, R(p) = RoPE rotation of the
 *   pairs (x_k, x_{k+d/2}) by p * base^(-2k/d); m = 1 for yarn_scale <= 1, else
 *   0.1 ln(yarn_scale) + 1 (YaRN attention temperature).
 *   out_i = sum_{j <= i} softmax_j(logit) v_j;  query head h reads KV head h / (Hq/Hkv).
 * Sources: "Qwen2.5-1M 不重训外推 1M" (mizuki-eaf.pages.dev), sections 核心思想,
 * Intra-Chunk / Successive-Chunk / Inter-Chunk Attention, "DCA + YaRN",
 * "Chunked Prefill"; news article on the Qwen2.5-1M release (7a8v.yksolo.com),
 * section 如何炼成的？ (RoPE base 10,000,000).  The window test r_i < w is one
 * reading of the Successive-Chunk section (the pages do not fix it).
 *
 * Conventions for every entry point
 *   - Tensors are contiguous row-major: q, out [L][Hq][d]; k, v [L][Hkv][d].
 *   - Device pointers must be 16-byte aligned; the workspace 256-byte aligned.
 *   - The caller owns every buffer; the library never allocates or frees
 *     device memory and never synchronises, except dca_device_status().
 *   - Work is enqueued on `cuda_stream` (a cudaStream_t; NULL = legacy default
 *     stream) of the current device and returns immediately.
 *   - Errors are return codes (dca_status); nothing is thrown across the ABI.
 *     Argument errors are detected on the host before any launch.
 *   - d must be 128.  dtype DCA_BF16 runs the tcgen05/TMA tensor-core kernel
 *     (bf16 in, fp32 accumulate, bf16 out); DCA_F32 runs an fp32 CUDA-core
 *     kernel (fp32 in/out).
 *   - Parameter domain: Hq % Hkv == 0, chunk_size >= 1,
 *     0 <= local_window <= chunk_size, pretrain_window >= 1, and
 *     chunk_size + local_window <= pretrain_window whenever the key length
 *     exceeds chunk_size (so every remapped distance stays below
 *     pretrain_window).  rope_base > 0, yarn_scale > 0.
 */
#ifndef DCA_B200_H
#define DCA_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum { DCA_BF16 = 0, DCA_F32 = 1 } dca_dtype;

/*
 * Reading of the local window of successive-chunk attention ("Qwen2.5-1M
 * 不重训外推 1M", section Successive-Chunk Attention: pairs inside the window
 * keep their true relative position, the others fall back to the inter-chunk
 * rule; the page does not say what the window is measured on).
 *   DCA_WINDOW_QUERY_OFFSET  (default) the pair (i, j) of adjacent chunks keeps
 *                            its true distance when the query's offset in its
 *                            chunk r_i < w;
 *   DCA_WINDOW_TRUE_DISTANCE it keeps its true distance when i - j < w.
 * Either way a kept distance is the true i - j and every other adjacent-chunk
 * pair uses query position c - 1 against key position j mod s.
 */
typedef enum { DCA_WINDOW_QUERY_OFFSET = 0, DCA_WINDOW_TRUE_DISTANCE = 1 } dca_window_reading;

/* Options of the _ex entry points (NULL means all defaults; reserved must be 0). */
typedef struct {
  int32_t window_reading; /* dca_window_reading */
  int32_t reserved[7];
} dca_options;

typedef enum {
  DCA_OK = 0,
  DCA_ERR_ARG = -1,         /* bad size, pointer, alignment or parameter       */
  DCA_ERR_UNSUPPORTED = -2, /* valid but not implemented (e.g. d != 128)       */
  DCA_ERR_CUDA = -3,        /* a CUDA runtime/driver call failed               */
  DCA_ERR_WORKSPACE = -4,   /* workspace missing, misaligned or too small      */
  DCA_ERR_TIMEOUT = -5      /* a kernel gave up on a bounded wait (device status) */
} dca_status;

/* Library version (major*10000 + minor*100 + patch). */
int dca_version(void);

/* Human-readable name of a dca_status value (static string, never NULL). */
const char* dca_status_string(int status);

/*
 * Workspace bytes needed for key lengths up to `kv_capacity` with these
 * parameters.  Returns 0 when the arguments are invalid.  The workspace holds
 * a status header, a RoPE cos/sin table computed in float64 and stored fp32,
 * and the keys rotated to their periodic positions (R(j mod s) k_j).  Its
 * layout depends only on (kv_capacity, Hkv, d, chunk sizes, dtype), so one
 * workspace can be reused across the calls of a chunked prefill.
 */
size_t dca_workspace_size(int64_t kv_capacity, int Hq, int Hkv, int d, int64_t chunk_size,
                          int64_t local_window, int64_t pretrain_window, int dtype);

/* Zero the workspace status header (call once after allocating it). */
int dca_workspace_init(void* workspace, size_t ws_bytes, void* cuda_stream);

/*
 * One-shot DCA prefill: q [L][Hq][d], k, v [L][Hkv][d] -> out [L][Hq][d].
 * Equivalent to dca_prefill_chunked(q, k, v, out, 0, L, L, ...).
 */
int dca_prefill(const void* q, const void* k, const void* v, void* out, int64_t L, int Hq,
                int Hkv, int d, int64_t chunk_size, int64_t local_window,
                int64_t pretrain_window, double rope_base, double yarn_scale, int dtype,
                void* workspace, size_t ws_bytes, void* cuda_stream);

/*
 * Chunked prefill ("Chunked Prefill" section: the input is processed in query
 * blocks that attend to the growing KV cache).  Query block row t has absolute
 * position q_start + t and attends cache rows j <= q_start + t.
 *   q_block, out_block [Lq][Hq][d];  k_cache, v_cache [Lk][Hkv][d] holding
 *   UNROTATED keys.  Requires q_start >= 0, Lq >= 0, q_start + Lq <= Lk.
 * The result equals rows [q_start, q_start + Lq) of the one-shot call.
 * Stateless: rotates all Lk keys into the workspace, then attends
 * (= dca_prepare(..., k_rows_valid = 0) followed by dca_attend).
 */
int dca_prefill_chunked(const void* q_block, const void* k_cache, const void* v_cache,
                        void* out_block, int64_t q_start, int64_t Lq, int64_t Lk, int Hq,
                        int Hkv, int d, int64_t chunk_size, int64_t local_window,
                        int64_t pretrain_window, double rope_base, double yarn_scale,
                        int dtype, void* workspace, size_t ws_bytes, void* cuda_stream);

/* dca_prefill_chunked with options (window reading).  DCA_ERR_ARG for invalid options. */
int dca_prefill_chunked_ex(const void* q_block, const void* k_cache, const void* v_cache,
                           void* out_block, int64_t q_start, int64_t Lq, int64_t Lk, int Hq,
                           int Hkv, int d, int64_t chunk_size, int64_t local_window,
                           int64_t pretrain_window, double rope_base, double yarn_scale,
                           int dtype, const dca_options* opts, void* workspace, size_t ws_bytes,
                           void* cuda_stream);

/*
 * Stage 1 of a prefill call: build the RoPE table and rotate keys
 * [k_rows_valid, Lk) of k_cache into the workspace.  k_rows_valid = 0 rebuilds
 * everything; k_rows_valid > 0 promises that the table and rotated rows
 * [0, k_rows_valid) already in this workspace were produced by earlier calls
 * with identical parameters and workspace size (an engine appending one block
 * of keys per call passes the previous Lk).
 */
int dca_prepare(const void* k_cache, int64_t Lk, int64_t k_rows_valid, int Hkv, int d,
                int64_t chunk_size, int64_t local_window, int64_t pretrain_window,
                double rope_base, int dtype, void* workspace, size_t ws_bytes,
                void* cuda_stream);

/*
 * Stage 2: the fused DCA attention kernel over a query block, reading the
 * rotated keys from the workspace (prepared for at least Lk rows) and v_cache.
 * Arguments as for dca_prefill_chunked (rope_base is fixed by dca_prepare).
 */
int dca_attend(const void* q_block, const void* v_cache, void* out_block, int64_t q_start,
               int64_t Lq, int64_t Lk, int Hq, int Hkv, int d, int64_t chunk_size,
               int64_t local_window, int64_t pretrain_window, double yarn_scale, int dtype,
               void* workspace, size_t ws_bytes, void* cuda_stream);

/* dca_attend with options (window reading).  DCA_ERR_ARG for invalid options. */
int dca_attend_ex(const void* q_block, const void* v_cache, void* out_block, int64_t q_start,
                  int64_t Lq, int64_t Lk, int Hq, int Hkv, int d, int64_t chunk_size,
                  int64_t local_window, int64_t pretrain_window, double yarn_scale, int dtype,
                  const dca_options* opts, void* workspace, size_t ws_bytes, void* cuda_stream);

/*
 * Decode: a few new query tokens against the whole cache.  The "Chunked
 * Prefill" section of "Qwen2.5-1M 不重训外推 1M" splits a long prompt into
 * blocks so that generation (one new token per request per step) is not
 * held up behind it; a decode step is the same attention with Lq tokens at
 * the end of the cache.  Rows t of q_block have absolute positions
 * q_start + t and attend cache rows j <= q_start + t, exactly as in
 * dca_attend_ex, and the result equals those rows of the one-shot prefill.
 * The rotated keys [0, Lk) must be in the workspace (dca_prepare; a decode
 * step that appended Lq keys passes k_rows_valid = Lk - Lq).
 *   q_block, out_block [Lq][Hq][d]; v_cache [Lk][Hkv][d];
 *   lse: NULL or [Lq][Hq] fp32, receives ln sum_j exp(logit_ij) per row;
 *   scratch: device memory of dca_decode_scratch_size(Lq, Hq, Hkv) bytes,
 *   16-byte aligned, for the partial results of the split-KV kernel (bf16;
 *   the fp32 path does not use it but the argument is checked the same way).
 * 1 <= Lq <= DCA_DECODE_MAX_TOKENS (Lq = 0: nothing to do).  bf16 runs a
 * split-KV tcgen05 kernel (the cache is cut into slices, one CTA per KV head,
 * group of 16 (token, head) rows and slice) followed by a merge kernel; fp32
 * runs the fp32 attention kernel.  Overlapping calls must not share scratch.
 */
#define DCA_DECODE_MAX_TOKENS 256
size_t dca_decode_scratch_size(int64_t Lq, int Hq, int Hkv);
int dca_decode(const void* q_block, const void* v_cache, void* out_block, float* lse,
               int64_t q_start, int64_t Lq, int64_t Lk, int Hq, int Hkv, int d,
               int64_t chunk_size, int64_t local_window, int64_t pretrain_window,
               double yarn_scale, int dtype, const dca_options* opts, void* workspace,
               size_t ws_bytes, void* scratch, size_t scratch_bytes, void* cuda_stream);

/*
 * Vertical-slash sparse DCA ("Qwen2.5-1M 不重训外推 1M", sections
 * "跟 NSA / 其他稀疏注意力的区别" and "稀疏注意力 + 核优化": per query head a few key
 * columns and diagonals carry the attention; per-head sparse patterns are
 * chosen offline and only the selected keys are attended).  For query head h
 * with vertical keys V_h and slash offsets S_h, row i attends exactly
 *     { j <= i : j in V_h } U { i - o : o in S_h, o <= i } U { i }
 * (each key once) with the DCA logits, softmax over those keys.
 *
 * dca_sparse_config fixes the sparse workspace layout: the key capacity its
 * bitmaps cover and the most vertical keys / slash offsets of any head.
 * Each head's slash offsets may form at most DCA_SPARSE_MAX_RUNS runs of
 * consecutive values.
 *
 * dca_sparse_prepare takes the patterns as HOST arrays in CSR form (v_ptr,
 * s_ptr [Hq + 1] offsets; v_idx, s_off the per-head lists, each sorted
 * ascending without repeats, inside [0, Lk)) and the DCA sizes of the
 * workspace (chunk_size, local_window, pretrain_window), copies them into the sparse
 * workspace, builds membership bitmaps and gathers the vertical keys' rotated
 * rows (from `workspace`, prepared by dca_prepare for rows [0, Lk)) and value
 * rows (from v_cache) into it.  The host arrays may be freed on return.  A
 * chunked prefill calls it again when the cache grows (vertical keys past Lk
 * are not gathered: pass the lists restricted to keys < Lk).
 * dca_sparse_attend then runs the sparse kernel for a query block (rows
 * q_start .., keys [0, Lk)).  bf16 only (DCA_ERR_UNSUPPORTED otherwise).
 * Argument and pattern errors are DCA_ERR_ARG, before any copy or launch;
 * a too-small sparse workspace is DCA_ERR_WORKSPACE.
 */
#define DCA_SPARSE_MAX_RUNS 1023
typedef struct {
  int64_t kv_capacity;  /* keys the bitmaps cover (>= every Lk used) */
  int64_t max_vertical; /* most vertical keys of a head */
  int64_t max_slash;    /* most slash offsets of a head */
} dca_sparse_config;
size_t dca_sparse_workspace_size(const dca_sparse_config* cfg, int Hq);
int dca_sparse_prepare(const dca_sparse_config* cfg, const int64_t* v_ptr, const int32_t* v_idx,
                       const int64_t* s_ptr, const int32_t* s_off, int64_t Lk, int Hq, int Hkv,
                       int d, int64_t chunk_size, int64_t local_window, int64_t pretrain_window,
                       int dtype, const void* v_cache, const void* workspace, size_t ws_bytes,
                       void* sparse_ws, size_t sparse_bytes, void* cuda_stream);
int dca_sparse_attend(const dca_sparse_config* cfg, const void* q_block, const void* v_cache,
                      void* out_block, int64_t q_start, int64_t Lq, int64_t Lk, int Hq, int Hkv,
                      int d, int64_t chunk_size, int64_t local_window, int64_t pretrain_window,
                      double yarn_scale, int dtype, const dca_options* opts, void* workspace,
                      size_t ws_bytes, const void* sparse_ws, size_t sparse_bytes,
                      void* cuda_stream);

/*
 * Online key selection ("稀疏注意力 + 核优化": the fix restores continuous
 * relative positions at the key-selection stage, because DCA's remapped
 * positions break the diagonal pattern).  From the last n_last (1..64) rows
 * i of the query block (absolute rows q_start + Lq - n_last ..), per query
 * head: p_ij = softmax over keys j <= i of the logits -- the DCA logits, or
 * with continuous_positions = 1 RoPE logits at the true positions i and j --
 * vertical score of key j = sum_rows p_ij, slash score of offset o =
 * sum_rows p_{i, i-o}; the n_vertical keys and n_slash offsets of largest
 * score (ties: the smaller index) become the head's pattern in sparse_ws,
 * with its bitmaps and gathered vertical rows, ready for dca_sparse_attend
 * (no host round trip).  Requires the rotated keys [0, Lk) in `workspace`
 * (dca_prepare), n_vertical <= cfg->max_vertical, n_slash <= min(cfg->max_slash,
 * DCA_SPARSE_MAX_RUNS), bf16.  scratch: dca_sparse_select_scratch_size bytes,
 * 256-byte aligned.
 */
size_t dca_sparse_select_scratch_size(int64_t Lk, int Hq, int64_t chunk_size);
int dca_sparse_select(const dca_sparse_config* cfg, const void* q_block, const void* v_cache,
                      int64_t q_start, int64_t Lq, int64_t Lk, int Hq, int Hkv, int d,
                      int64_t chunk_size, int64_t local_window, int64_t pretrain_window,
                      double rope_base, double yarn_scale, int dtype, const dca_options* opts,
                      int n_last, int continuous_positions, int64_t n_vertical, int64_t n_slash,
                      void* workspace, size_t ws_bytes, void* sparse_ws, size_t sparse_bytes,
                      void* scratch, size_t scratch_bytes, void* cuda_stream);

/*
 * Copies the pattern held by sparse_ws to host memory (synchronises the
 * stream): per head the count and sorted list of vertical keys
 * (v_counts [Hq], v_idx [Hq][cfg->max_vertical]) and of slash offsets
 * (s_counts [Hq], s_off [Hq][cfg->max_slash]).
 */
int dca_sparse_pattern_get(const dca_sparse_config* cfg, int Hq, const void* sparse_ws,
                           size_t sparse_bytes, int32_t* v_counts, int32_t* v_idx,
                           int32_t* s_counts, int32_t* s_off, void* cuda_stream);

/*
 * Host-side introspection of the sparse kernel's work list (no GPU needed):
 * for the query tile whose rows are [i0, i0 + 128) (i0 a multiple of 128) with
 * real rows up to i_last, and one head's sorted vertical keys / slash offsets
 * (host arrays), writes up to max_items triples (src, start, class): src 0 =
 * the 128 gathered vertical keys at list positions start .. start + 127
 * (start a multiple of 128), src 1 = the 128 cache keys start .. start + 127,
 * a window over what the slash diagonals and the diagonal j = i reach from
 * the tile's rows; class as in dca_plan_items.  Returns the number of items
 * (which may exceed max_items) or DCA_ERR_ARG; DCA_ERR_UNSUPPORTED if the
 * plan's item count disagrees with its list (an internal consistency check:
 * the kernels size their loops by that count).
 */
int dca_sparse_plan_items(const int32_t* v_idx, int64_t n_v, const int32_t* s_off, int64_t n_s,
                          int64_t i0, int64_t i_last, int64_t chunk_size, int64_t local_window,
                          int window_reading, int32_t* items, int max_items);

/*
 * Device-side status: synchronises `cuda_stream`, reads and clears the status
 * word that kernels set when a bounded wait gave up.  Returns DCA_OK,
 * DCA_ERR_TIMEOUT or DCA_ERR_CUDA.
 */
int dca_device_status(void* workspace, void* cuda_stream);

/*
 * Host-buffer entry point: whole prefill of L tokens from HOST memory.
 * q_h, out_h [L][Hq][d]; k_h, v_h [L][Hkv][d] in host memory (pinned memory
 * gives full copy bandwidth and lets the copies overlap the kernels).  The
 * input is processed in query blocks of `block` rows (block <= 0: one block):
 * per block the library copies the block's q, k and v rows host->device,
 * appends the keys to the rotated-key cache, runs the attention kernel and
 * copies the block's output rows back.  The copies run on a copy stream of
 * the library's own (one non-blocking stream per device, created on first
 * use), ordered against `cuda_stream` by events: block b + 1's inputs and
 * block b - 1's outputs move while block b is attended (two query and two
 * output block buffers in the arena).  All device memory comes from the
 * caller's `arena` (dca_host_arena_size bytes, 256-byte aligned).  Returns
 * after enqueuing; `cuda_stream` waits for every copy, so synchronising it
 * (or dca_device_status) makes out_h readable.
 */
size_t dca_host_arena_size(int64_t L, int64_t block, int Hq, int Hkv, int d,
                           int64_t chunk_size, int64_t local_window, int64_t pretrain_window,
                           int dtype);
int dca_prefill_host(const void* q_h, const void* k_h, const void* v_h, void* out_h, int64_t L,
                     int64_t block, int Hq, int Hkv, int d, int64_t chunk_size,
                     int64_t local_window, int64_t pretrain_window, double rope_base,
                     double yarn_scale, int dtype, void* arena, size_t arena_bytes,
                     void* cuda_stream);

/*
 * Host-side introspection of the tile plan the attention kernels follow
 * (no GPU needed).  For the query tile whose rows are [i0, i0 + tile_rows)
 * with real rows up to i_last, key tiles of `bn` keys, local window
 * `local_window` and window reading `window_reading`, writes up to
 * `max_items` triples (k_tile, class, full) in work-list order: class 2 =
 * inter-chunk rule (query position c - 1), 1 = successive chunk with its true
 * distance kept (under the query-offset reading: every adjacent-chunk pair,
 * the row choosing s + r_i or c - 1), 0 = intra-chunk (the three parts of the
 * score matrix in section 核心思想 of "Qwen2.5-1M 不重训外推 1M"); full = 1
 * when every pair of the tile is causal and of that class (no mask).
 * Returns the number of items (which may exceed max_items) or DCA_ERR_ARG.
 */
int dca_plan_items(int64_t i0, int64_t i_last, int64_t tile_rows, int64_t chunk_size,
                   int64_t local_window, int window_reading, int bn, int32_t* items,
                   int max_items);

/*
 * Host-side introspection of the key selection's masking (no GPU needed):
 * for key j and the block of estimate rows at positions i_first + r,
 * 0 <= r < n_rows (n_rows <= 64), writes to range[0..1] the rows [ra, rb) that
 * pair with j -- causal (j <= i), j < kv_len, and either of work-list class
 * `cls` (0, 1, 2 as in dca_plan_items; cls >= 0) or, with cls = -1, with
 * j in key chunk `chunk` (j / chunk_size == chunk; continuous positions).
 * These rows are one contiguous range because a key's class does not
 * decrease as i grows.  Returns DCA_OK, or DCA_ERR_ARG (0 <= j < 2^31,
 * i_first >= 0, 1 <= n_rows <= 64, chunk_size >= 1, 0 <= local_window <=
 * chunk_size, cls in -1..2, range not NULL).
 */
int dca_class_rows(int64_t j, int64_t i_first, int n_rows, int64_t kv_len, int64_t chunk_size,
                   int64_t local_window, int window_reading, int cls, int64_t chunk,
                   int32_t* range);

/*
 * Host-side introspection of the attention kernel's per-row masking (no GPU
 * needed): the keys [range[0], range[1]) that form pairs of work-list class
 * `cls` (0, 1, 2 as in dca_plan_items) with query row i, causal (j <= i)
 * included -- one contiguous range per row and class (empty: range[0] ==
 * range[1]).  A masked tile keeps exactly its columns inside this range.
 * Computed in 32-bit arithmetic as on the device.  Returns DCA_OK, or
 * DCA_ERR_ARG (0 <= i < 2^31 - 1, cls in 0..2, chunk_size >= 1,
 * 0 <= local_window <= chunk_size, range not NULL).
 */
int dca_row_keys(int64_t i, int cls, int64_t chunk_size, int64_t local_window, int window_reading,
                 int64_t* range);

/*
 * No-allocation one-shot prefill (an addition for integrators; the pages on
 * DCA have no counterpart).  For callers that cannot call cudaMalloc: e.g. a
 * serving process that hands all free HBM to its own pool at start-up, where a
 * later allocation fails or stalls the device, or a plugin whose host
 * framework owns every device allocation.  Same arguments and result as
 * dca_prefill, minus the workspace: the library uses a fixed scratch area of
 * DCA_NOALLOC_SCRATCH_BYTES that is part of its image, and calls no
 * cudaMalloc, cudaFree or allocating library routine.
 *   - The scratch exists on a device once the library's device code is loaded
 *     there, and stays until the process exits.  Under lazy module loading
 *     (CUDA_MODULE_LOADING=LAZY, the default of recent CUDA) that happens at
 *     the first use on the device, not when the library is opened: call
 *     dca_noalloc_prepare() once per device, with that device current, before
 *     reserving the rest of the device's memory and before any stream capture.
 *     Otherwise the first dca_prefill_noalloc call does it.
 *   - The scratch address is looked up once per device and kept; do not use
 *     these entry points across cudaDeviceReset (the kept address is stale).
 *   - Returns DCA_ERR_WORKSPACE, before any device work, when
 *     dca_workspace_size(L, ...) exceeds DCA_NOALLOC_SCRATCH_BYTES (about
 *     L <= 16384 for 4 KV heads in bf16).  Every other argument is checked
 *     as dca_prefill checks it, also before any device work.
 *   - All calls share the one scratch area: calls that overlap on the GPU
 *     (other streams, other threads) race and must be serialised by the caller.
 *   - The status word in the scratch is cleared at the start of each call;
 *     dca_noalloc_device_status reads it back after the call.
 */
#define DCA_NOALLOC_SCRATCH_BYTES (32u * 1024u * 1024u)
int dca_prefill_noalloc(const void* q, const void* k, const void* v, void* out, int64_t L,
                        int Hq, int Hkv, int d, int64_t chunk_size, int64_t local_window,
                        int64_t pretrain_window, double rope_base, double yarn_scale, int dtype,
                        void* cuda_stream);

/*
 * Loads the library's device code on the current device and looks up the
 * no-allocation scratch there (no device memory is allocated beyond the
 * library image).  Returns DCA_OK or DCA_ERR_CUDA.
 */
int dca_noalloc_prepare(void);

/*
 * dca_device_status for the no-allocation scratch of the current device:
 * synchronises `cuda_stream`, returns DCA_ERR_TIMEOUT (and clears the word)
 * when a bounded device wait of the last dca_prefill_noalloc call ran out
 * (its output is then incomplete), DCA_OK otherwise, DCA_ERR_CUDA on a CUDA
 * error.
 */
int dca_noalloc_device_status(void* cuda_stream);

/*
 * Test hooks.  dca_set_wait_timeout_ns sets the limit of every bounded device
 * wait (default 10 s).  dca_set_debug_flags(1) makes the next attention launch
 * withhold its first key-tile load, so that its waits run out and the kernel
 * returns through the timeout path (status word set, DCA_ERR_TIMEOUT from
 * dca_device_status); flags reset to 0 after that launch.  The decode and
 * sparse kernels honour the same flag.
 */
void dca_set_wait_timeout_ns(int64_t ns);
void dca_set_debug_flags(int flags);

#ifdef __cplusplus
}
#endif
#endif /* DCA_B200_H */
