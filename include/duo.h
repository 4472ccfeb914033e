/*
 * duo.h -- C ABI of libduo: attention over a head-split KV cache
 * (DuoAttention: retrieval heads with a full KV cache, streaming heads with a
 * constant-length cache of attention sinks plus recent tokens), for NVIDIA
 * B200 (sm_100a).
 *
 * Sources (pages; the method is stated in prose only):
 *  - "DuoAttention: Efficient Long-Context LLM Inference with Retrieval and
 *    Streaming Heads" (hotpaper.ai), abstract: retrieval heads need full
 *    attention over all tokens; streaming heads attend to recent tokens and
 *    attention sinks through a light-weight constant-length KV cache; this
 *    cuts both decoding and pre-filling cost.  Same page, section
 *    "기술적 접근법" (technical approach): two KV caches per layer; MHA and GQA;
 *    compatible with a 4-bit KV cache.
 *  - "What is DuoAttention" (nav.superapi.store), section "Technical
 *    principles of DuoAttention": full KV cache for retrieval heads,
 *    fixed-length KV cache for streaming heads.
 *  - "韩松团队长上下文LLM推理高效框架" (cn.bg3.co), section "研究背景": decoding
 *    cost grows linearly and pre-filling cost quadratically with the context.
 *
 * Definitions used by every call (readings where the pages are silent):
 *  - Query head h uses KV head h / G, G = n_q_heads / n_kv_heads.  One mask bit
 *    per KV head: 1 = retrieval, 0 = streaming.
 *  - A query at absolute position i sees key j iff j <= i and, for a streaming
 *    head, (j < S or i - j < R).  Softmax scale defaults to 1/sqrt(head_dim).
 *  - Streaming slot of position p: p if p < S, else S + ((p - S) mod R).
 *  - Q and K arrive post-RoPE; the library does no position arithmetic.
 *
 * Conventions:
 *  - The caller owns all device memory: the cache storage (bound once with
 *    duo_cache_bind), Q/K/V/O and workspaces.  The handle owns host metadata.
 *  - Tensors are dense, row-major, in device memory:
 *      decode  q, out   [batch, n_q_heads, head_dim]
 *      append  k, v     [batch, n_tokens, n_kv_heads, head_dim]
 *      prefill q, out   [batch, C, n_q_heads, head_dim]; k, v [batch, C, n_kv_heads, head_dim]
 *    Element type: float32 for a DUO_F32 cache; bfloat16 for DUO_BF16 and for
 *    the K/V/Q/O of a DUO_INT4 cache (K/V are quantised on append).  Decode
 *    outputs of bf16 and 4-bit caches can be float32 instead
 *    (duo_set_decode_output).
 *  - Every call with a stream is asynchronous on that stream.  Argument,
 *    capacity and layout errors are detected on the host and returned before
 *    anything is enqueued; a failed launch returns DUO_ERR_CUDA.  Nothing
 *    throws across this boundary.  Calls on one cache must be ordered by the
 *    caller (one stream, or events).
 *  - Host threads: a handle's metadata (lengths, block tables, the block
 *    pool) is updated by the calls without locking, so calls on one cache
 *    from several host threads must be serialised by the caller.  Different
 *    caches share nothing on the host (duo_decode_attn_static's device
 *    scratch is shared; see there).
 *  - Ordering: decode is append-then-attend (duo_append_kv with one token, then
 *    duo_decode_attn; the new token sees itself).  Pre-fill is
 *    attend-then-append (duo_prefill_attn reads the cache as it stood before
 *    the chunk plus the chunk's own K/V; the caller then appends the chunk).
 *  - Rows: each batch row is a sequence slot with its own length per layer.
 *    The plain calls act on every row, each at its own length; the *_rows
 *    calls act on a list of distinct rows, and their tensors hold only the
 *    listed rows, in list order (the leading "batch" dimension becomes the
 *    list length).
 */
#ifndef DUO_H
#define DUO_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define DUO_MAX_KV_HEADS 64
#define DUO_MAX_SPLITS 512
#define DUO_PAGE_TOKENS 256     /* tokens per retrieval block of the paged layout */
#define DUO_MAX_LAUNCH_ROWS 128 /* rows per kernel launch; longer row lists take several */

typedef struct CUstream_st *duo_stream; /* a cudaStream_t; NULL = legacy stream */

typedef enum duo_status {
  DUO_OK = 0,
  DUO_ERR_ARG = 1,         /* null pointer, bad size, bad layer, misaligned pointer */
  DUO_ERR_CAPACITY = 2,    /* an append would pass capacity, or the block pool is exhausted */
  DUO_ERR_LAYOUT = 3,      /* head mask / head counts inconsistent */
  DUO_ERR_WORKSPACE = 4,   /* workspace missing or smaller than required */
  DUO_ERR_CUDA = 5,        /* a CUDA runtime call or launch failed */
  DUO_ERR_TIMEOUT = 6,     /* a bounded in-kernel wait gave up (see duo_poll_device_error) */
  DUO_ERR_UNSUPPORTED = 7, /* valid request this build does not implement */
  DUO_ERR_STATE = 8        /* cache not bound, or call out of order */
} duo_status;

typedef enum duo_kv_dtype { DUO_F32 = 0, DUO_BF16 = 1, DUO_INT4 = 2 } duo_kv_dtype;

typedef enum duo_layout {
  /* Retrieval KV heads: one contiguous [capacity, d] page each for K and V.
   * Streaming KV heads: one [S + R, d] slot buffer each for K and V. */
  DUO_LAYOUT_PACKED = 0,
  /* Retrieval KV heads: blocks of DUO_PAGE_TOKENS tokens from a pool shared
   * by all rows, found through a per-row block table (duo_cache_create_paged).
   * Streaming KV heads as in the packed layout. */
  DUO_LAYOUT_PAGED = 1
} duo_layout;

typedef struct duo_cache_desc {
  int32_t layers;
  int32_t batch;
  int32_t n_q_heads;
  int32_t n_kv_heads;  /* <= DUO_MAX_KV_HEADS, divides n_q_heads */
  int32_t head_dim;    /* 64 or 128 */
  int32_t kv_dtype;    /* duo_kv_dtype */
  int64_t capacity;    /* max tokens of one row (INT4: rounded up to 128) */
} duo_cache_desc;

typedef struct duo_cache duo_cache;

/* Where one layer's buffers live inside the bound device memory.  Offsets are
 * in bytes from the bound base pointer; -1 where a buffer does not exist. */
typedef struct duo_layout_view {
  int32_t n_retrieval;   /* retrieval KV heads in this layer */
  int32_t n_streaming;   /* streaming KV heads in this layer */
  int32_t window;        /* S + R */
  int32_t window_stride; /* rows per streaming head buffer: window, rounded up to 4 for INT4 */
  int32_t row_bytes;     /* bytes of one token of one head: d*4 (f32), d*2 (bf16), d/2 (int4 codes) */
  int64_t capacity;
  int64_t seq_len;       /* the longest row's length */
  int64_t ret_k, ret_v;  /* packed [batch][n_retrieval][capacity][row];
                            paged  [pool_blocks][n_retrieval][DUO_PAGE_TOKENS][row] */
  int64_t str_k, str_v;  /* [batch][n_streaming][window_stride][row] */
  int64_t ret_k_sz, ret_v_sz, str_k_sz, str_v_sz; /* int4 only: fp16 (scale, zero) per token, same indexing */
  int32_t kind[DUO_MAX_KV_HEADS];         /* 1 retrieval, 0 streaming, per KV head */
  int32_t packed_index[DUO_MAX_KV_HEADS]; /* index among heads of the same kind */
  int32_t layout;        /* duo_layout */
  int32_t page_tokens;   /* paged: DUO_PAGE_TOKENS; packed: 0 */
  int32_t table_stride;  /* paged: block-table entries per row */
  int64_t pool_blocks;   /* paged: blocks in the pool */
  int64_t block_table;   /* paged: int32 [batch][table_stride] (shared by all layers); else -1 */
} duo_layout_view;

/* Create a cache description.  head_mask: host array [layers][n_kv_heads] of
 * 0/1 (1 = retrieval).  S >= 0 sinks, R >= 1 recent slots.  layout must be
 * DUO_LAYOUT_PACKED (use duo_cache_create_paged for the paged layout).  No
 * device memory is touched.
 * Errors: DUO_ERR_ARG (null/out-of-range), DUO_ERR_LAYOUT (heads inconsistent). */
duo_status duo_cache_create(duo_cache **out, const duo_cache_desc *desc,
                            const uint8_t *head_mask, int32_t S, int32_t R,
                            int32_t layout);

/* Create a cache with the paged layout, for serving many sequences of
 * different lengths: retrieval K/V live in a pool of pool_blocks blocks of
 * DUO_PAGE_TOKENS tokens (every layer holds its own pool of the same block
 * count), which rows take as they grow and give back on duo_release_rows or
 * duo_cache_reset; block ids are shared by all layers of a row.
 * desc.capacity bounds one row's length.  The allocator runs on the host;
 * new block-table entries are written on the stream before the kernels that
 * need them.  Requires a configuration the tensor-core decode serves (bf16 or
 * 4-bit KV, head_dim 128); pre-fill works on both (a 4-bit cache through the
 * workspace of duo_prefill_workspace_bytes).
 * Errors: as duo_cache_create; DUO_ERR_ARG for pool_blocks <= 0;
 * DUO_ERR_UNSUPPORTED for other configurations. */
duo_status duo_cache_create_paged(duo_cache **out, const duo_cache_desc *desc,
                                  const uint8_t *head_mask, int32_t S, int32_t R,
                                  int64_t pool_blocks);

void duo_cache_destroy(duo_cache *cache);

/* Bytes of device memory the cache needs (cache_bytes), and the decode
 * workspace size that covers every layer and split count (workspace_bytes). */
duo_status duo_cache_required_bytes(const duo_cache *cache, size_t *cache_bytes,
                                    size_t *workspace_bytes);

/* Bind caller-owned device memory (256-byte aligned, >= cache_bytes).  The
 * memory is zero-filled synchronously and every length reset to 0 (paged:
 * every block returned to the pool). */
duo_status duo_cache_bind(duo_cache *cache, void *device_mem, size_t bytes);

/* Reset every row of every layer to length 0 (paged: return every block to
 * the pool) without touching device memory. */
duo_status duo_cache_reset(duo_cache *cache);

/* Rows n_rows listed in rows (distinct, in range) go back to length 0 in every
 * layer; paged: their blocks return to the pool.  rows == NULL: every row.
 * Host only. */
duo_status duo_release_rows(duo_cache *cache, const int32_t *rows, int32_t n_rows);

/* Append n_tokens tokens to one layer of every row (each row at its own
 * positions len .. len+n_tokens-1).  Defined by "What is DuoAttention"
 * (nav.superapi.store), section "Technical principles of DuoAttention": a
 * full KV cache for retrieval heads, a fixed-length cache of attention sinks
 * and recent tokens for streaming heads.  Retrieval heads write page (or block)
 * rows, streaming heads write only the positions that survive the chunk
 * (sinks and the last R positions) into their slots, evicting what was
 * there.  INT4 caches quantise each (token, head) row of head_dim channels
 * (asymmetric min/max, fp16 scale and zero, 4-bit codes, low nibble = even
 * channel).  Paged: rows take the blocks they need from the pool first.
 * Advances each row's length by n_tokens.  n_tokens == 0 changes nothing
 * and reads neither k nor v (either may be NULL then).
 * Errors: DUO_ERR_CAPACITY if a row would pass capacity or the pool cannot
 * cover every row (nothing is changed then). */
duo_status duo_append_kv(duo_cache *cache, int32_t layer, const void *k,
                         const void *v, int32_t n_tokens, duo_stream stream);

/* duo_append_kv for the n_rows rows listed (k, v: [n_rows, n_tokens,
 * n_kv_heads, head_dim]).  rows == NULL: every row.  Errors also DUO_ERR_ARG
 * for a repeated or out-of-range row. */
duo_status duo_append_kv_rows(duo_cache *cache, int32_t layer, const int32_t *rows,
                              int32_t n_rows, const void *k, const void *v,
                              int32_t n_tokens, duo_stream stream);

/* Single-token decode attention for one layer: in every row, the query at
 * position len-1 (len = that row's length) of every query head attends to its
 * KV head's visible set.  Defined by "DuoAttention: Efficient Long-Context
 * LLM Inference with Retrieval and Streaming Heads" (hotpaper.ai), abstract:
 * retrieval heads attend over all tokens, streaming heads over the attention
 * sinks and recent tokens only.  Retrieval heads run split-K flash decoding
 * (per-split log-sum-exp partials in the workspace, merged by the last split
 * of each head; the tensor-core decode gives each row a split count in
 * proportion to its length); streaming heads run one pass over their slot
 * buffer.  softmax_scale <= 0 means 1/sqrt(d).  The workspace must be
 * zero-filled before its first use with any cache; each call leaves its
 * counters at zero again.  Workspace size: from duo_cache_required_bytes.
 * Errors: DUO_ERR_STATE if a row is empty; DUO_ERR_UNSUPPORTED for rows of
 * different lengths on a configuration without the tensor-core decode (fp32
 * caches, head_dim 64). */
duo_status duo_decode_attn(duo_cache *cache, int32_t layer, const void *q,
                           void *out, float softmax_scale, void *workspace,
                           size_t workspace_bytes, duo_stream stream);

/* duo_decode_attn for the n_rows rows listed (q, out: [n_rows, n_q_heads,
 * head_dim]).  Tensor-core decode configurations only (other configurations
 * accept only rows == NULL). */
duo_status duo_decode_attn_rows(duo_cache *cache, int32_t layer, const int32_t *rows,
                                int32_t n_rows, const void *q, void *out,
                                float softmax_scale, void *workspace,
                                size_t workspace_bytes, duo_stream stream);

/* One decode step for one layer in a single launch where the kernels allow
 * it (the two operations of the abstract of "DuoAttention: Efficient
 * Long-Context LLM Inference with Retrieval and Streaming Heads"
 * (hotpaper.ai) and of section "Technical principles of DuoAttention" of
 * "What is DuoAttention" (nav.superapi.store), in one pass): append each row's new token (k_new, v_new: [batch, n_kv_heads,
 * head_dim]) at position len and attend with q at that position, exactly as
 * duo_append_kv(.., 1, ..) followed by duo_decode_attn.  One warp of the
 * launch takes the new token's K/V from the inputs (4-bit caches: quantises
 * it with duo_append_kv's encoder) and writes it to the cache; the attention
 * adds that key from the inputs.  Configurations without a fused kernel (fp32
 * caches, head_dim 64) run the two calls.  Advances each row's length
 * by one.  The launch uses programmatic dependent launch, so its set-up
 * overlaps the previous kernel in the stream.  Errors as for the two calls. */
duo_status duo_decode_step(duo_cache *cache, int32_t layer, const void *q,
                           const void *k_new, const void *v_new, void *out,
                           float softmax_scale, void *workspace,
                           size_t workspace_bytes, duo_stream stream);

/* duo_decode_step for the n_rows rows listed (q, out: [n_rows, n_q_heads,
 * head_dim]; k_new, v_new: [n_rows, n_kv_heads, head_dim]). */
duo_status duo_decode_step_rows(duo_cache *cache, int32_t layer, const int32_t *rows,
                                int32_t n_rows, const void *q, const void *k_new,
                                const void *v_new, void *out, float softmax_scale,
                                void *workspace, size_t workspace_bytes,
                                duo_stream stream);

/* Decode attention like duo_decode_attn, but with no workspace argument and
 * no device memory allocation (no cudaMalloc, cudaFree or allocating library
 * routine; the host-side planning uses a few small heap buffers, like every
 * other call): the split-K scratch (partial outputs, log-sum-exp values,
 * merge tickets) lives in a fixed array inside the library,
 * DUO_DECODE_STATIC_SCRATCH_BYTES in size, that every GPU loading the library
 * holds until the process exits.  The paper has no counterpart to this call.
 * It is for callers that cannot call cudaMalloc (or any allocator) to get a
 * workspace: a serving loop that must never stall, since cudaMalloc and
 * cudaFree can synchronise the device; a host program whose device memory is
 * entirely reserved by another allocator it may not call into; a plugin given
 * only the input and output pointers.
 *  - The first call on each device looks up the array's device address
 *    (cudaGetSymbolAddress, with that device current); make that first call
 *    before any stream capture.
 *  - Every call shares the one array: calls that may overlap on the GPU (other
 *    streams, other threads, other caches) race and must be serialised by the
 *    caller.  The merge tickets are cleared on the stream before each launch.
 *  - If the scratch this layer needs (the retrieval splits of all rows x
 *    group x (head_dim + 1) x 4 bytes, plus tickets and counters) exceeds the
 *    array, the call returns DUO_ERR_WORKSPACE before enqueuing anything.
 * Results equal duo_decode_attn's for the same cache state (bit for bit with
 * duo_set_decode_reproducible, else up to rounding). */
#define DUO_DECODE_STATIC_SCRATCH_BYTES (8u << 20)
duo_status duo_decode_attn_static(duo_cache *cache, int32_t layer, const void *q,
                                  void *out, float softmax_scale, duo_stream stream);

/* Chunked pre-fill attention for one layer: in every row, C queries at
 * positions len .. len+C-1 attend to the cache as it stands (positions below
 * len) plus the chunk's own k/v.  Defined by "DuoAttention: Efficient
 * Long-Context LLM Inference with Retrieval and Streaming Heads"
 * (hotpaper.ai), abstract (the split applies to pre-filling as well as
 * decoding), and "韩松团队长上下文LLM推理高效框架" (cn.bg3.co), section "研究背景"
 * (pre-fill cost quadratic in the context): causal for retrieval heads, Lambda mask
 * (sinks plus the R most recent positions) for streaming heads, with key tiles
 * outside the Lambda band skipped.  Runs on the sm_100a tensor cores
 * (tcgen05.mma, accumulators in tensor memory, operands loaded by TMA).  Does
 * not append; call duo_append_kv with the same k/v afterwards.  Requires
 * head_dim 128 and a DUO_BF16 or DUO_INT4 cache (other cases:
 * DUO_ERR_UNSUPPORTED).  DUO_BF16: the workspace is unused (pass NULL, 0).
 * DUO_INT4: the part of the cache the chunk reads (retrieval keys below each
 * row's length, filled streaming slots) is first expanded to bf16, x = sc*u+zp
 * rounded to bf16, in the workspace (duo_prefill_workspace_bytes, 256-byte
 * aligned), which the tensor-core pass then reads; the chunk's own k/v enter
 * exactly as given.  Key tiles are 128 rows, so a tile can cover rows past a
 * row's length (probability 0); the expansion writes zeros there, so the
 * workspace needs no initialisation.
 * Errors: DUO_ERR_CAPACITY if len + C would pass capacity in a row;
 * DUO_ERR_WORKSPACE if an INT4 cache gets a missing or small workspace. */
duo_status duo_prefill_attn(duo_cache *cache, int32_t layer, const void *q,
                            const void *k, const void *v, int32_t C, void *out,
                            float softmax_scale, void *workspace,
                            size_t workspace_bytes, duo_stream stream);

/* duo_prefill_attn for the n_rows rows listed (q, out: [n_rows, C, n_q_heads,
 * head_dim]; k, v: [n_rows, C, n_kv_heads, head_dim]), each at its own length. */
duo_status duo_prefill_attn_rows(duo_cache *cache, int32_t layer, const int32_t *rows,
                                 int32_t n_rows, const void *q, const void *k,
                                 const void *v, int32_t C, void *out,
                                 float softmax_scale, void *workspace,
                                 size_t workspace_bytes, duo_stream stream);

/* Workspace bytes duo_prefill_attn needs: 0 for a DUO_BF16 cache; for a
 * DUO_INT4 cache the bf16 size of one layer's retrieval storage rows plus its
 * streaming buffers (K and V), for the largest layer. */
duo_status duo_prefill_workspace_bytes(const duo_cache *cache, size_t *bytes);

/* Sequence sharding, for a sequence too long for one GPU's retrieval caches:
 * several caches (normally one per GPU) each keep a contiguous range of the
 * retrieval heads' positions, and every one keeps the whole, tiny, streaming
 * state.  After this call the cache's retrieval heads store only positions
 * [lo, hi) of each row, at page (or block) rows position - lo; appends still
 * pass every token (positions outside [lo, hi) touch only the streaming
 * heads), and capacity counts the rows this shard stores.  Such a cache
 * decodes only through duo_decode_attn_partial, and pre-fill is not offered.
 * Call while every length is 0 (fresh, bound or reset cache).  Tensor-core
 * decode configurations only (bf16 or 4-bit KV, head_dim 128).
 * Errors: DUO_ERR_ARG (lo < 0 or hi <= lo), DUO_ERR_STATE (tokens present),
 * DUO_ERR_UNSUPPORTED (other configurations). */
duo_status duo_set_retrieval_shard(duo_cache *cache, int64_t lo, int64_t hi);

/* Decode attention of every row over this cache's share of the keys, as a
 * partial to merge with the other shards': per (row, query head) the output
 * normalised over this share, o_part [batch, n_q_heads, head_dim] float32, and
 * the natural-log log-sum-exp of the scaled scores over it, lse_part [batch,
 * n_q_heads] float32 (-inf with o_part 0 where the share holds no visible
 * key).  Streaming heads are included only when owns_streaming is 1 (exactly
 * one shard should own them; every shard holds the same streaming state).
 * Does not append.  Workspace as for duo_decode_attn.  Works on unsharded
 * caches too (the whole sequence as one share). */
duo_status duo_decode_attn_partial(duo_cache *cache, int32_t layer, const void *q,
                                   float *o_part, float *lse_part, int32_t owns_streaming,
                                   float softmax_scale, void *workspace,
                                   size_t workspace_bytes, duo_stream stream);

/* Merge n_parts partials (the shards' o_part / lse_part, gathered in device
 * memory as o_parts [n_parts, rows, head_dim] and lse_parts [n_parts, rows]
 * float32, rows = batch * n_q_heads) into out [rows, head_dim] of out_dtype
 * (DUO_BF16 or DUO_F32): out = sum_i exp(lse_i - L) o_i, L = log sum_i
 * exp(lse_i); rows no shard saw a key of are 0.  The exchange of the partials
 * between GPUs (an all-gather over NVLink) is the caller's. */
duo_status duo_merge_partials(int32_t n_parts, int64_t rows, int32_t head_dim,
                              const float *o_parts, const float *lse_parts, void *out,
                              int32_t out_dtype, duo_stream stream);

/* The longest row's length in one layer (every row's, when all rows advance
 * together). */
duo_status duo_seq_len(const duo_cache *cache, int32_t layer, int64_t *n);

/* One row's length in one layer. */
duo_status duo_row_seq_len(const duo_cache *cache, int32_t layer, int32_t row, int64_t *n);

/* Paged layout: the blocks row holds, in logical order (block i holds
 * positions [DUO_PAGE_TOKENS i, DUO_PAGE_TOKENS (i+1)) of the row in every
 * layer).  *n_blocks receives the count; blocks (may be NULL) receives the
 * ids if max_blocks is large enough (else DUO_ERR_ARG).  Packed: 0 blocks. */
duo_status duo_row_blocks(const duo_cache *cache, int32_t row, int32_t *blocks,
                          int32_t max_blocks, int32_t *n_blocks);

/* Paged layout: blocks in the pool that no row holds.  Packed: 0. */
duo_status duo_pool_free_blocks(const duo_cache *cache, int64_t *free_blocks);

/* KV bytes held now (kept) and what a full cache of every head would hold
 * (full_equivalent): kept = sum over layers, rows, KV heads of
 * (retrieval ? n : min(n, S+R)) * bytes_per_token_per_head, n = the row's
 * length in that layer. */
duo_status duo_kv_bytes(const duo_cache *cache, int64_t *kept,
                        int64_t *full_equivalent);

duo_status duo_layout_info(const duo_cache *cache, int32_t layer,
                           duo_layout_view *out);

/* Force the split count of retrieval decode (1..DUO_MAX_SPLITS), or 0 for the
 * automatic choice (enough splits to fill every SM once).  The result never
 * depends on it beyond rounding. */
duo_status duo_set_decode_splits(duo_cache *cache, int32_t splits);

/* How the tensor-core decode (bf16 and 4-bit caches, head_dim 128) shares a
 * split retrieval head's keys among its splits.  By default (on = 0) each
 * split takes a fixed share of 13/16 of the key tiles (7/8 on a 4-bit cache)
 * and the rest goes, one tile at a time, to whichever warps finish first, so
 * that splits running
 * on SMs that get less memory bandwidth do less work and all finish together.
 * Which keys each split sums then varies between calls, and outputs can differ
 * in the last bits.  on = 1 gives every split an even fixed share instead:
 * repeated calls on the same cache state return bit-identical outputs, at
 * about 1-2% more time per call at long contexts.  Applies to duo_decode_attn,
 * duo_decode_step and duo_decode_attn_static.  Errors: DUO_ERR_ARG for a null
 * cache or on outside {0, 1}. */
duo_status duo_set_decode_reproducible(duo_cache *cache, int32_t on);

/* Element type of decode outputs: DUO_BF16 (the default for DUO_BF16 and
 * DUO_INT4 caches) or DUO_F32 (float32; the only type of a DUO_F32 cache).
 * Applies to duo_decode_attn, duo_decode_step, duo_decode_attn_static and
 * their *_rows forms: out is then [rows, n_q_heads, head_dim] of that type.
 * The kernels accumulate in float32 either way; DUO_F32 skips the final
 * rounding to bf16 (whose half-ulp exceeds 2e-2 once |out| passes 8).
 * Errors: DUO_ERR_ARG (null cache, other types), DUO_ERR_UNSUPPORTED (DUO_BF16
 * for a DUO_F32 cache). */
duo_status duo_set_decode_output(duo_cache *cache, int32_t dtype);

/* Split count the next decode of this layer will use (tensor-core decode: the
 * largest any row gets at the current lengths). */
duo_status duo_decode_splits(const duo_cache *cache, int32_t layer,
                             int32_t *splits);

/* Streaming heads per streaming CTA that the next decode of this layer will
 * use (a scheduling choice; the pages have no counterpart).  The tensor-core
 * decode (bf16 and 4-bit caches) may run 2, 4 or 8 of a row's streaming heads
 * in one CTA, one group of warps each, when their windows are short next to the
 * retrieval splits: the SMs this frees take more retrieval splits.  1 for
 * every other configuration.  Outputs do not depend on it beyond rounding.
 * Errors: DUO_ERR_ARG (null cache or pointer, layer out of range). */
duo_status duo_decode_streaming_pack(const duo_cache *cache, int32_t layer,
                                     int32_t *heads_per_cta);

/* Testing hook for the failure path of the bounded in-kernel waits (the
 * pages have no counterpart).  The next duo_prefill_attn or
 * duo_prefill_attn_rows on this cache issues none of its tile loads, and its
 * waits give up after wait_ns nanoseconds (1000 .. 1e9) instead of a second:
 * every CTA records the timeout in the device error word, frees its tensor
 * memory and returns without writing its output, and duo_poll_device_error
 * then returns DUO_ERR_TIMEOUT.  Nothing faults, traps or hangs; the next call
 * runs normally.  Errors: DUO_ERR_ARG. */
duo_status duo_test_stall_next_prefill(duo_cache *cache, int64_t wait_ns);

/* Testing hook for the tensor-core decode's launch planner (a scheduling
 * choice; the pages have no counterpart), host only: no device is touched.
 * For one launch of n_rows rows (1 .. DUO_MAX_LAUNCH_ROWS) of this layer
 * whose lengths, the query included, are lens[r] >= 1, on a device of
 * num_sms SMs taking ctas_per_sm decode CTAs each, writes each row's split
 * count per retrieval head to splits[r] and the streaming heads per
 * streaming CTA to *pack: the plan duo_decode_attn_rows would launch with
 * those lengths (duo_set_decode_splits applies).  Errors: DUO_ERR_ARG;
 * DUO_ERR_UNSUPPORTED for a configuration without the tensor-core decode
 * (fp32 caches, head_dim 64). */
duo_status duo_test_plan_decode(const duo_cache *cache, int32_t layer,
                                const int32_t *lens, int32_t n_rows,
                                int32_t num_sms, int32_t ctas_per_sm,
                                int32_t *splits, int32_t *pack);

/* Read and clear the device-side error word that bounded in-kernel waits set
 * when they give up.  Synchronises the device.  Returns DUO_ERR_TIMEOUT if it
 * was set, DUO_OK otherwise; *code (may be NULL) receives the raw word.
 * The outputs of a call whose wait gave up are undefined.  A decode CTA that
 * gives up still leaves an empty partial and takes its merge ticket, so the
 * decode workspace is left with its counters at zero and stays usable. */
duo_status duo_poll_device_error(int32_t *code);

const char *duo_status_string(duo_status status);

#ifdef __cplusplus
}
#endif

#endif /* DUO_H */
