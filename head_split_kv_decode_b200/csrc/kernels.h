// Internal interface between the C-ABI layer (duo_api.cpp) and the CUDA
// kernels.  Not part of the public ABI.
#pragma once

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

enum KvType : int { kF32 = 0, kBF16 = 1, kINT4 = 2 };

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

struct AppendParams {
  const void *k, *v;   // [B][n_tok][Hkv][D]
  LayerPtrs p;
  HeadTables h;
  int B, Hkv, D, n_ret, n_str, S, R, W;
  int Ws;              // rows per streaming head buffer (W, or W rounded up to 4 for int4)
  int64_t cap, n_cur, n_tok;
};

struct DecodeParams {
  const void *q;   // [B][Hq][D]
  void *out;       // [B][Hq][D]
  LayerPtrs p;
  HeadTables h;
  int B, Hq, Hkv, G, D, n_ret, n_str, S, R, W;
  int Ws;              // rows per streaming head buffer
  int64_t cap;
  int64_t n;           // tokens in the cache, the query is at position n-1
  int nsplit;          // splits per retrieval head
  int64_t split_len;   // rows per split (multiple of the tile)
  float scale_log2;    // softmax scale * log2(e)
  float *ws_o;         // [B][n_ret][nsplit][G][D]
  float *ws_lse;       // [B][n_ret][nsplit][G]
  unsigned *ws_cnt;    // [B][n_ret] merge tickets
  unsigned *ws_next;   // [B][n_ret][kChunkCounterStride] pool counter of each retrieval head (tensor-core decode)
  int *err;            // device error word
  // Fused append (duo_decode_step): the K/V of the token at position n-1,
  // [B][Hkv][D]; null when it is already in the cache.  The CTA that owns the
  // token's row reads it from here and writes it to the cache.
  const void *knew, *vnew;
  int64_t new_slot;    // streaming slot of position n-1
  int pdl;             // launched with programmatic dependent launch
  int pool;            // tensor-core decode: the last eighth of a split head's
                       // tiles is claimed at run time (0: every split gets an
                       // even, fixed share)
};

struct PrefillParams {
  const void *q, *k, *v;  // q [B][C][Hq][D], k/v [B][C][Hkv][D]
  void *out;              // [B][C][Hq][D]
  LayerPtrs p;
  HeadTables h;
  int B, Hq, Hkv, G, D, n_ret, n_str, S, R, W, C;
  int64_t cap, c0;        // c0: tokens already in the cache
  float scale_log2;
  int *err;
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
cudaError_t launch_prefill(const PrefillParams &p, cudaStream_t s);
int *device_error_word();  // device address of the error word

// Library-owned decode scratch for duo_decode_attn_static (decode_static.cu).
size_t decode_static_scratch_bytes();
cudaError_t decode_static_scratch(void **ptr);

}  // namespace duo
