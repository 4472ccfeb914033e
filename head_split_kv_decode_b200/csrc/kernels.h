// Internal interface between the C-ABI layer (duo_api.cpp) and the CUDA
// kernels.  Not part of the public ABI.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace duo {

constexpr int kMaxKvHeads = 64;
constexpr int kMaxSplits = 512;
// u32 slots between the per-head chunk counters of the decode workspace (one
// 256-byte line each, so that concurrent claims on different heads do not
// queue on one line)
constexpr int kChunkCounterStride = 64;
constexpr int kMaxDevices = 64;
// Paged layout: retrieval tokens per block of the pool.
constexpr int kPageShift = 8;
constexpr int kPageTokens = 1 << kPageShift;
// Batch rows one launch can take (row lists live in the kernel parameters).
constexpr int kMaxLaunchRows = 128;

enum KvType : int { kF32 = 0, kBF16 = 1, kINT4 = 2 };

// Limit of the pre-fill kernel's bounded waits (ns) unless a test shortens it.
constexpr uint64_t kPrefillWaitNs = 1000000000ull;

// Error word set by bounded in-kernel waits that give up (bit flags).
enum DeviceError : int {
  kErrWaitTileLoad = 1,
  kErrWaitMma = 2,
  kErrWaitPrefillLoad = 4,
};

// Byte pointers into the bound cache for one layer.
struct LayerPtrs {
  uint8_t *ret_k, *ret_v;        // [B][n_ret][cap][row]
  uint8_t *str_k, *str_v;        // [B][n_str][W][row]
  uint8_t *ret_k_sz, *ret_v_sz;  // int4: [B][n_ret][cap] x (fp16 scale, fp16 zero)
  uint8_t *str_k_sz, *str_v_sz;  // int4: [B][n_str][W]   x (fp16 scale, fp16 zero)
};

struct HeadTables {
  int8_t kind[kMaxKvHeads];      // 1 retrieval, 0 streaming
  int8_t index[kMaxKvHeads];     // packed index among heads of that kind
  int8_t ret_heads[kMaxKvHeads]; // packed retrieval index -> KV head
  int8_t str_heads[kMaxKvHeads]; // packed streaming index -> KV head
};

// The batch rows (sequence slots) a launch works on and each one's cache
// length: before the new tokens (append), including the new token (decode),
// or before the chunk (pre-fill).  A launch's inputs and outputs are indexed by
// the position r in this list, the cache by row[r].
struct LaunchRows {
  int n;
  int32_t row[kMaxLaunchRows];
  int32_t len[kMaxLaunchRows];
};

// Where the retrieval rows of a layer live.  Packed: (b, head, key) is
// storage row (b*n_ret + head)*cap + key.  Paged: key's block is
// table[b*stride + key/kPageTokens] and the storage row is
// (block*n_ret + head)*kPageTokens + key%kPageTokens.  Row r of a buffer is
// at byte r*row_bytes; the int4 (scale, zero) arrays at byte r*4.
struct RetMap {
  const int32_t *table;  // device block table [B][stride]; null: packed layout
  int stride;            // table entries per batch row
  int n_ret;
  int64_t cap;           // packed: rows per (b, head)
  int64_t blocks;        // paged: blocks in the pool
};

struct AppendParams {
  const void *k, *v;   // [rows.n][n_tok][Hkv][D]
  LayerPtrs p;
  HeadTables h;
  RetMap ret;
  LaunchRows rows;     // len = tokens in the cache before this append
  int64_t shard_lo, shard_hi;  // retrieval heads keep positions [lo, hi) at row p - lo
  int Hkv, D, n_ret, n_str, S, R, W;
  int Ws;              // rows per streaming head buffer (W, or W rounded up to 4 for int4)
  int64_t n_tok;
};

// Most streaming heads one tensor-core decode CTA takes (DecodeParams::str_pack).
constexpr int kMaxStrPack = 8;

struct DecodeParams {
  const void *q;   // [B][Hq][D] (tensor-core decode: [rows.n][Hq][D])
  void *out;       // same shape as q
  LayerPtrs p;
  HeadTables h;
  int B, Hq, Hkv, G, D, n_ret, n_str, S, R, W;
  int Ws;              // rows per streaming head buffer
  int64_t cap;
  // CUDA-core decode (packed layout, every row at length n): splits of
  // split_len rows, nsplit per retrieval head.
  int64_t n;           // tokens in the cache, the query is at position n-1
  int nsplit;          // splits per retrieval head
  int64_t split_len;   // rows per split (multiple of the tile)
  // Tensor-core decode: per launch row r (length rows.len[r], query at
  // len-1), nsplit_r[r] splits per retrieval head; its retrieval CTAs are
  // cta0[r] .. cta0[r+1]-1, head-major, and CTA c leaves its partial in
  // slot c of ws_o / ws_lse.  Merge tickets and tile counters are indexed by
  // r*n_ret + head.
  LaunchRows rows;
  int32_t cta0[kMaxLaunchRows + 1];
  int16_t nsplit_r[kMaxLaunchRows];
  RetMap ret;
  // Sequence shard: retrieval heads hold positions [shard_lo, shard_hi) at
  // page row position - shard_lo (default [0, 2^62)).
  int64_t shard_lo, shard_hi;
  // Partial mode (part_o non-null): instead of out, every query head leaves
  // its normalised output [rows.n][Hq][D] f32 in part_o and its natural-log
  // log-sum-exp [rows.n][Hq] in part_lse (-inf and zeros where it saw no
  // key); streaming heads contribute only when own_str.
  float *part_o, *part_lse;
  int own_str;
  float scale_log2;    // softmax scale * log2(e)
  float *ws_o;         // [partial slots][G][D]
  float *ws_lse;       // [partial slots][G]
  unsigned *ws_cnt;    // [units] merge tickets
  unsigned *ws_next;   // [units][kChunkCounterStride] pool counter of each retrieval head (tensor-core decode)
  int *err;            // device error word
  // Fused append (duo_decode_step): the K/V of the token at position len-1 of
  // each launch row, [rows.n][Hkv][D]; null when it is already in the cache.
  // The warp whose key tile holds the token's row reads it from here and
  // writes it to the cache.
  const void *knew, *vnew;
  int pdl;             // launched with programmatic dependent launch
  int out_f32;         // bf16 and 4-bit caches: out is float32 instead of bf16
  int pool;            // tensor-core decode: the last 3/16 (4-bit: 1/8) of a
                       // split head's tiles is claimed at run time (0: every
                       // split gets an even, fixed share)
  int str_pack;        // tensor-core decode: streaming heads per streaming CTA
                       // (1, 2, 4 or 8 = kMaxStrPack), each on NWARPS/str_pack
                       // warps; the CTAs of launch row r are
                       // cta0[rows.n] + r*ceil(n_str/str_pack) + i
};

struct PrefillParams {
  const void *q, *k, *v;  // q [rows.n][C][Hq][D], k/v [rows.n][C][Hkv][D]
  void *out;              // [rows.n][C][Hq][D]
  LayerPtrs p;
  HeadTables h;
  RetMap ret;
  LaunchRows rows;        // len = tokens already in the cache (the chunk starts there)
  int B, Hq, Hkv, G, D, n_ret, n_str, S, R, W, C;
  int64_t retrieval_rows; // storage rows of each retrieval buffer of the layer
  float scale_log2;
  int *err;
  uint64_t wait_ns;       // limit of every bounded wait (normally kWaitNs)
  int skip_loads;         // testing hook: issue no TMA loads (every wait then gives up)
};

// 4-bit history expanded to bf16 for the pre-fill: retrieval rows keep their
// storage row; streaming rows go to [B][n_str][W][D] (slot order).
struct DequantParams {
  LayerPtrs p;         // the 4-bit cache buffers of the layer
  HeadTables h;
  RetMap ret;
  LaunchRows rows;     // len = tokens of each row to expand (its history)
  int n_ret, n_str, S, R, W, Ws, D;
  __nv_bfloat16 *ret_k, *ret_v, *str_k, *str_v;  // bf16 scratch
};

// Block-table writes of the paged layout, applied in stream order.
constexpr int kMaxTableWrites = 256;
struct TableWrites {
  int n;
  int32_t index[kMaxTableWrites];  // entry b*stride + i
  int32_t block[kMaxTableWrites];
};

// Launch configuration facts the host needs to size splits and workspaces.
struct DecodeConfig {
  int tile_rows;        // rows per pipeline tile
  int ctas_per_sm;      // occupancy of the decode kernel
  int num_sms;
};

cudaError_t decode_config(int kv_type, int D, int G, DecodeConfig *cfg);
cudaError_t launch_append(const AppendParams &a, int kv_type, cudaStream_t s);
cudaError_t launch_decode(const DecodeParams &d, int kv_type, cudaStream_t s);
// True when launch_decode can take the new token's K/V itself (fused append).
bool decode_can_fuse_append(int kv_type, int D, int G);
// True when the tensor-core decode serves this configuration: it alone reads
// DecodeParams.rows (any launch rows, each at its own length) and the paged
// layout; the CUDA-core decode takes every batch row at one length, packed.
bool decode_mma_supported(int kv_type, int D, int G);
// Keys a CTA of the tensor-core decode walks per iteration (16 warps x one
// tile each); host-only, no device needed.
int decode_mma_tile_rows(int kv_type);
cudaError_t launch_prefill(const PrefillParams &p, cudaStream_t s);
cudaError_t launch_table_writes(int32_t *table, const TableWrites &w, cudaStream_t s);
cudaError_t launch_dequant_history(const DequantParams &d, cudaStream_t s);
// out[rows][D] = sum_i exp(lse_i - L) o_i, L = log sum_i exp(lse_i), over
// n_parts partials o [n_parts][rows][D] f32, lse [n_parts][rows] (natural log);
// out_type kBF16 or kF32.
cudaError_t launch_merge_partials(int n_parts, int64_t rows, int D, const float *o,
                                  const float *lse, void *out, int out_type, cudaStream_t s);
int *device_error_word();  // device address of the error word

// Library-owned decode scratch for duo_decode_attn_static (decode_static.cu).
size_t decode_static_scratch_bytes();
cudaError_t decode_static_scratch(void **ptr);

}  // namespace duo
