// C-ABI layer of libduo: validates arguments, plans the layout of the
// head-split KV cache, tracks the length of every (layer, batch row), runs the
// block allocator of the paged layout, and launches the kernels.
//
// Per layer, each buffer 256-byte aligned:
//   retrieval K, V : packed [batch][n_retrieval][capacity][row]
//                    paged  [pool_blocks][n_retrieval][DUO_PAGE_TOKENS][row]
//   streaming K, V : [batch][n_streaming][S + R][row]
//   int4 only      : (fp16 scale, fp16 zero) per row, same indexing, for each
// row = head_dim elements (f32 / bf16) or head_dim/2 bytes of 4-bit codes.
// Paged: one block table [batch][ceil(capacity / DUO_PAGE_TOKENS)] of int32
// after the layers; block ids are shared by all layers (logical block i of
// row b holds positions [256 i, 256 i + 256) of that row in every layer).
// Retrieval heads keep every token; streaming heads keep S sinks plus an
// R-slot ring ("DuoAttention: Efficient Long-Context LLM Inference with
// Retrieval and Streaming Heads" (hotpaper.ai), section "기술적 접근법": a
// full KV cache for retrieval heads and a fixed-length one for streaming
// heads in every layer).
#include <algorithm>
#include <climits>
#include <cmath>
#include <cstring>
#include <new>
#include <vector>

#include <cuda_runtime.h>

#include "../../include/duo.h"
#include "kernels.h"

static_assert(DUO_MAX_KV_HEADS == duo::kMaxKvHeads, "head table size");
static_assert(DUO_MAX_SPLITS == duo::kMaxSplits, "split limit");
static_assert(DUO_DECODE_STATIC_SCRATCH_BYTES == (8u << 20), "static decode scratch size");
static_assert(DUO_PAGE_TOKENS == duo::kPageTokens, "page size");
static_assert(DUO_MAX_LAUNCH_ROWS == duo::kMaxLaunchRows, "rows per launch");

struct duo_cache {
  duo_cache_desc desc;
  int layout;                 // DUO_LAYOUT_PACKED or DUO_LAYOUT_PAGED
  int S, R, W;
  int Ws;                     // rows per streaming head buffer
  std::vector<uint8_t> mask;  // [layers][Hkv]
  struct Layer {
    int n_ret, n_str;
    duo::HeadTables h;
    int64_t off_ret_k, off_ret_v, off_str_k, off_str_v;
    int64_t off_ret_k_sz, off_ret_v_sz, off_str_k_sz, off_str_v_sz;
    int64_t ret_rows;         // storage rows of each retrieval buffer
  };
  std::vector<Layer> layers;
  std::vector<int64_t> seq_len;  // [layers][batch]
  // paged layout
  int64_t pool_blocks;
  int table_stride;                  // entries per batch row
  int64_t off_table;                 // device block table (int32)
  std::vector<int32_t> table;        // host copy, -1 = no block
  std::vector<int32_t> held;         // blocks held by each batch row
  std::vector<int32_t> free_blocks;  // stack of unused block ids
  size_t cache_bytes;
  size_t ws_bytes;
  int n_ret_max;
  int row_bytes;
  uint8_t *base;
  int forced_splits;
  int64_t shard_lo, shard_hi;  // retrieval heads keep positions [lo, hi) (sequence shard)
  bool reproducible;       // decode splits take fixed key shares only
  int32_t out_dtype;       // decode output element type (DUO_F32 or DUO_BF16)
  int64_t stall_ns;        // testing hook: the next pre-fill loads nothing, waits this long
  bool have_cfg;           // decode launch facts, queried once per cache
  duo::DecodeConfig cfg;
};

namespace {

constexpr int64_t kAlign = 256;

int64_t round_up(int64_t x, int64_t a) { return (x + a - 1) / a * a; }

int elem_bytes(int kv) { return kv == DUO_F32 ? 4 : 2; }

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

int64_t &len_of(duo_cache *c, int layer, int row) {
  return c->seq_len[(size_t)layer * c->desc.batch + row];
}
int64_t len_of(const duo_cache *c, int layer, int row) {
  return c->seq_len[(size_t)layer * c->desc.batch + row];
}

constexpr int64_t kNoShardEnd = 1LL << 62;

bool sharded(const duo_cache *c) { return c->shard_lo != 0 || c->shard_hi != kNoShardEnd; }

// Retrieval rows a row holds in this cache's shard when its length is n.
int64_t ret_len(const duo_cache *c, int64_t n) {
  return std::max<int64_t>(0, std::min(n, c->shard_hi) - c->shard_lo);
}

bool mma_path(const duo_cache *c) {
  const duo_cache_desc &d = c->desc;
  return duo::decode_mma_supported(d.kv_dtype, d.head_dim, d.n_q_heads / d.n_kv_heads);
}

duo::LayerPtrs layer_ptrs(const duo_cache *c, int layer) {
  const auto &L = c->layers[layer];
  auto at = [&](int64_t off) { return off < 0 ? nullptr : c->base + off; };
  return duo::LayerPtrs{at(L.off_ret_k),    at(L.off_ret_v),    at(L.off_str_k),
                        at(L.off_str_v),    at(L.off_ret_k_sz), at(L.off_ret_v_sz),
                        at(L.off_str_k_sz), at(L.off_str_v_sz)};
}

duo::RetMap ret_map(const duo_cache *c, int layer) {
  duo::RetMap m{};
  m.n_ret = c->layers[layer].n_ret;
  m.cap = c->desc.capacity;
  if (c->layout == DUO_LAYOUT_PAGED) {
    m.table = reinterpret_cast<const int32_t *>(c->base + c->off_table);
    m.stride = c->table_stride;
    m.blocks = c->pool_blocks;
  }
  return m;
}

// Workspace: [merge tickets: B*n_ret_max u32][chunk counters: B*n_ret_max
//            lines of kChunkCounterStride u32][lse: B*n_ret_max*MAXS*G f32][o: ...*D f32]
struct WsLayout {
  int64_t cnt, next, lse, o, total;
};

WsLayout ws_layout(const duo_cache_desc &d, int n_ret_max) {
  const int G = d.n_q_heads / d.n_kv_heads;
  const int64_t units = (int64_t)d.batch * (n_ret_max > 0 ? n_ret_max : 1);
  WsLayout w;
  w.cnt = 0;
  w.next = round_up(units * 4, kAlign);
  w.lse = w.next + round_up(units * duo::kChunkCounterStride * 4, kAlign);
  w.o = w.lse + round_up(units * duo::kMaxSplits * G * 4, kAlign);
  w.total = w.o + round_up(units * duo::kMaxSplits * G * (int64_t)d.head_dim * 4, kAlign);
  return w;
}

// Compact scratch of one launch in the library's static array: tickets, tile
// counters, lse, partial O.
struct StaticLayout {
  int64_t next, lse, o, total;
};

StaticLayout static_layout(int64_t units, int64_t slots, int G, int D) {
  StaticLayout s;
  s.next = round_up(units * 4, kAlign);
  s.lse = s.next + round_up(units * duo::kChunkCounterStride * 4, kAlign);
  s.o = s.lse + round_up(slots * G * 4, kAlign);
  s.total = s.o + slots * G * (int64_t)D * 4;
  return s;
}

duo_status cuda_status(cudaError_t e) { return e == cudaSuccess ? DUO_OK : DUO_ERR_CUDA; }

duo_status launch_status(cudaError_t e) {
  if (e == cudaErrorInvalidValue || e == cudaErrorNotSupported) return DUO_ERR_UNSUPPORTED;
  return cuda_status(e);
}

// Occupancy and tile facts of the decode kernel for this cache's dtype, head
// size and group size; queried from the runtime on first use only.
cudaError_t cached_decode_config(duo_cache *c, duo::DecodeConfig *out) {
  if (!c->have_cfg) {
    const duo_cache_desc &d = c->desc;
    cudaError_t e = duo::decode_config(d.kv_dtype, d.head_dim, d.n_q_heads / d.n_kv_heads, &c->cfg);
    if (e != cudaSuccess) return e;
    c->have_cfg = true;
  }
  *out = c->cfg;
  return cudaSuccess;
}

// CUDA-core decode (every batch row at length n): splits per retrieval head,
// enough CTAs to occupy every SM once (the streaming heads' CTAs included), at
// least two tiles per split.
int choose_splits(const duo_cache *c, int layer, int64_t n, const duo::DecodeConfig &cfg) {
  const auto &L = c->layers[layer];
  if (L.n_ret == 0) return 1;
  const int64_t min_rows = 2LL * cfg.tile_rows;
  const int64_t by_len = (n + min_rows - 1) / min_rows;
  int64_t want;
  if (c->forced_splits > 0) {
    want = c->forced_splits;
  } else {
    const int64_t slots = (int64_t)cfg.num_sms * (cfg.ctas_per_sm > 0 ? cfg.ctas_per_sm : 1);
    const int64_t units = (int64_t)c->desc.batch * L.n_ret;
    const int64_t free_slots = slots - (int64_t)c->desc.batch * L.n_str;
    want = free_slots / units;
    if (want < 1) want = 1;
    if (want > by_len) want = by_len;
  }
  if (want > duo::kMaxSplits) want = duo::kMaxSplits;
  if (want > n) want = n;
  if (want < 1) want = 1;
  return (int)want;
}

// Tensor-core decode: splits per retrieval head of each launch row.  The
// SMs' CTA slots left after the str_ctas streaming CTAs are handed out one
// split at a time to the row whose splits currently hold the most keys (every
// row starts with one), which minimises the longest split; a row gets at most
// one split per two CTA iterations of keys and at most DUO_MAX_SPLITS.  A
// forced count applies to every row, capped by its length.
void choose_row_splits(const duo_cache *c, int layer, const int32_t *lens, int nrows,
                       const duo::DecodeConfig &cfg, int64_t str_ctas, int16_t *out) {
  const auto &L = c->layers[layer];
  std::vector<int64_t> cap(nrows);
  for (int r = 0; r < nrows; ++r) {
    const int64_t n = std::max<int32_t>(1, lens[r]);
    int64_t m = c->forced_splits > 0 ? c->forced_splits
                                     : (n + 2LL * cfg.tile_rows - 1) / (2LL * cfg.tile_rows);
    m = std::min<int64_t>(std::min<int64_t>(m, duo::kMaxSplits), n);
    cap[r] = L.n_ret == 0 ? 1 : std::max<int64_t>(1, m);
    out[r] = (int16_t)(c->forced_splits > 0 ? cap[r] : 1);
  }
  if (L.n_ret == 0 || c->forced_splits > 0) return;
  const int64_t slots = (int64_t)cfg.num_sms * (cfg.ctas_per_sm > 0 ? cfg.ctas_per_sm : 1);
  const int64_t budget = (slots - str_ctas) / L.n_ret;  // splits over all rows
  std::vector<std::pair<double, int>> heap;  // (keys per split, row), max-heap
  for (int r = 0; r < nrows; ++r)
    if (cap[r] > 1) heap.emplace_back((double)std::max<int32_t>(1, lens[r]), r);
  std::make_heap(heap.begin(), heap.end());
  for (int64_t used = nrows; used < budget && !heap.empty(); ++used) {
    std::pop_heap(heap.begin(), heap.end());
    const int r = heap.back().second;
    heap.pop_back();
    ++out[r];
    if (out[r] < cap[r]) {
      heap.emplace_back((double)std::max<int32_t>(1, lens[r]) / out[r], r);
      std::push_heap(heap.begin(), heap.end());
    }
  }
}

// Tensor-core decode: streaming heads per streaming CTA.
// A streaming head is a window of at most S + R keys, so its CTA is short
// next to a retrieval split of a long row; packing hp heads into one CTA (one
// group of 16/hp warps each) frees SM slots for retrieval splits.  Taken:
// the hp in {1, 2, 4, 8}, at most the row's streaming heads, that gives the
// most retrieval CTAs while a streaming warp's keys (its head's window over
// its group) stay within 3/4 of a retrieval warp's in the longest split; the
// smallest such hp on a tie.  Lengths are the rows' retrieval keys (lens)
// and the longest streaming window (win).
int choose_str_pack(const duo_cache *c, int layer, const int32_t *lens, int nrows, int64_t win,
                    const duo::DecodeConfig &cfg) {
  const auto &L = c->layers[layer];
  if (L.n_ret == 0 || L.n_str <= 1 || c->forced_splits > 0) return 1;
  const int64_t win_t = (win + 15) / 16 * 16;  // rows of the window's tiles of 16 keys
  int best = 1;
  int64_t best_ctas = -1;
  int16_t ns[duo::kMaxLaunchRows];
  for (int hp = 1; hp <= duo::kMaxStrPack && hp <= 2 * L.n_str - 1; hp *= 2) {
    const int64_t str_ctas = (int64_t)nrows * ((L.n_str + hp - 1) / hp);
    choose_row_splits(c, layer, lens, nrows, cfg, str_ctas, ns);
    int64_t ret_ctas = 0;
    double longest = 0.0;  // keys of the longest split
    for (int r = 0; r < nrows; ++r) {
      ret_ctas += (int64_t)L.n_ret * ns[r];
      longest = std::max(longest, (double)std::max<int32_t>(1, lens[r]) / ns[r]);
    }
    if (hp > 1 && (double)(hp * win_t) > 0.75 * longest) break;
    if (ret_ctas > best_ctas) {
      best = hp;
      best_ctas = ret_ctas;
    }
  }
  return best;
}

// One tensor-core decode launch of nr rows, with retrieval keys rlen and
// lengths len (the query included): split counts into ns; returns the
// streaming heads per streaming CTA.
int plan_launch(const duo_cache *c, int layer, const int32_t *rlen, const int32_t *len, int nr,
                const duo::DecodeConfig &cfg, int16_t *ns) {
  const auto &L = c->layers[layer];
  int64_t win = 0;  // the longest streaming window of the launch
  for (int r = 0; r < nr; ++r) win = std::max<int64_t>(win, std::min<int64_t>(len[r], c->W));
  const int hp = choose_str_pack(c, layer, rlen, nr, win, cfg);
  choose_row_splits(c, layer, rlen, nr, cfg, (int64_t)nr * ((L.n_str + hp - 1) / hp), ns);
  return hp;
}

// Rows of one call: every batch row in order (rows == NULL), or a list of
// distinct rows in range.
duo_status make_rows(const duo_cache *c, const int32_t *rows, int32_t n_rows,
                     std::vector<int32_t> *out) {
  out->clear();
  if (!rows) {
    for (int b = 0; b < c->desc.batch; ++b) out->push_back(b);
    return DUO_OK;
  }
  if (n_rows <= 0 || n_rows > c->desc.batch) return DUO_ERR_ARG;
  std::vector<char> seen(c->desc.batch, 0);
  for (int i = 0; i < n_rows; ++i) {
    const int b = rows[i];
    if (b < 0 || b >= c->desc.batch || seen[b]) return DUO_ERR_ARG;
    seen[b] = 1;
    out->push_back(b);
  }
  return DUO_OK;
}

// Length checks before n_tokens more tokens go into `rows` of a layer.
duo_status check_room(const duo_cache *c, int layer, const std::vector<int32_t> &rows,
                      int64_t n_tokens) {
  if (c->layers[layer].n_ret == 0 && c->layout == DUO_LAYOUT_PACKED) return DUO_OK;
  for (int b : rows)
    if (ret_len(c, len_of(c, layer, b) + n_tokens) > c->desc.capacity) return DUO_ERR_CAPACITY;
  return DUO_OK;
}

// Paged layout: give every row in `rows` the blocks that positions up to
// len + n_tokens - 1 of `layer` need, and write the new table entries on the
// stream (before the kernels that use them).  All or nothing: if the pool
// cannot cover every row, nothing changes and DUO_ERR_CAPACITY is returned.
duo_status reserve_blocks(duo_cache *c, int layer, const std::vector<int32_t> &rows,
                          int64_t n_tokens, cudaStream_t s) {
  if (c->layout != DUO_LAYOUT_PAGED) return DUO_OK;
  std::vector<int32_t> need(rows.size());
  int64_t total = 0;
  for (size_t i = 0; i < rows.size(); ++i) {
    const int64_t end = ret_len(c, len_of(c, layer, rows[i]) + n_tokens);
    const int64_t blocks = (end + duo::kPageTokens - 1) / duo::kPageTokens;
    need[i] = (int32_t)std::max<int64_t>(0, blocks - c->held[rows[i]]);
    total += need[i];
  }
  if (total > (int64_t)c->free_blocks.size()) return DUO_ERR_CAPACITY;
  duo::TableWrites w{};
  int32_t *dev_table = reinterpret_cast<int32_t *>(c->base + c->off_table);
  for (size_t i = 0; i < rows.size(); ++i) {
    const int b = rows[i];
    for (int k = 0; k < need[i]; ++k) {
      const int32_t blk = c->free_blocks.back();
      c->free_blocks.pop_back();
      const int32_t idx = b * c->table_stride + c->held[b]++;
      c->table[idx] = blk;
      w.index[w.n] = idx;
      w.block[w.n] = blk;
      if (++w.n == duo::kMaxTableWrites) {
        if (duo::launch_table_writes(dev_table, w, s) != cudaSuccess) return DUO_ERR_CUDA;
        w.n = 0;
      }
    }
  }
  return cuda_status(duo::launch_table_writes(dev_table, w, s));
}

void release_blocks(duo_cache *c, int b) {
  if (c->layout != DUO_LAYOUT_PAGED) return;
  for (int i = c->held[b] - 1; i >= 0; --i) {
    c->free_blocks.push_back(c->table[(size_t)b * c->table_stride + i]);
    c->table[(size_t)b * c->table_stride + i] = -1;
  }
  c->held[b] = 0;
}

void reset_lengths(duo_cache *c) {
  for (auto &n : c->seq_len) n = 0;
  for (int b = 0; c->layout == DUO_LAYOUT_PAGED && b < c->desc.batch; ++b) release_blocks(c, b);
}

duo_status check_layer(const duo_cache *c, int32_t layer) {
  if (!c) return DUO_ERR_ARG;
  if (layer < 0 || layer >= c->desc.layers) return DUO_ERR_ARG;
  if (!c->base) return DUO_ERR_STATE;
  return DUO_OK;
}

duo_status create(duo_cache **out, const duo_cache_desc *desc, const uint8_t *head_mask, int32_t S,
                  int32_t R, int32_t layout, int64_t pool_blocks) {
  if (!out || !desc || !head_mask) return DUO_ERR_ARG;
  *out = nullptr;
  const duo_cache_desc d = *desc;
  if (d.layers <= 0 || d.batch <= 0 || d.n_q_heads <= 0 || d.n_kv_heads <= 0) return DUO_ERR_ARG;
  if (d.n_kv_heads > DUO_MAX_KV_HEADS || d.n_q_heads % d.n_kv_heads) return DUO_ERR_LAYOUT;
  if (d.head_dim != 64 && d.head_dim != 128) return DUO_ERR_ARG;
  if (d.kv_dtype != DUO_F32 && d.kv_dtype != DUO_BF16 && d.kv_dtype != DUO_INT4) return DUO_ERR_ARG;
  if (d.capacity <= 0 || d.capacity > INT32_MAX - duo::kPageTokens || S < 0 || R < 1)
    return DUO_ERR_ARG;
  for (int64_t i = 0; i < (int64_t)d.layers * d.n_kv_heads; ++i)
    if (head_mask[i] > 1) return DUO_ERR_LAYOUT;
  const bool paged = layout == DUO_LAYOUT_PAGED;
  if (paged) {
    if (pool_blocks <= 0 || pool_blocks > INT32_MAX) return DUO_ERR_ARG;
    if (!duo::decode_mma_supported(d.kv_dtype, d.head_dim, d.n_q_heads / d.n_kv_heads))
      return DUO_ERR_UNSUPPORTED;
  }

  duo_cache *c = new (std::nothrow) duo_cache();
  if (!c) return DUO_ERR_ARG;
  c->desc = d;
  c->layout = layout;
  c->S = S;
  c->R = R;
  c->W = S + R;
  // INT4 keeps scale/zero rows in 16-byte groups of four tokens, so its row
  // counts per head are rounded up to a multiple of 4.
  c->Ws = d.kv_dtype == DUO_INT4 ? (int)round_up(c->W, 4) : c->W;
  // 4-bit: whole 16-byte groups of (scale, zero) rows, and whole 128-key
  // pre-fill tiles per packed retrieval head, so that a tile of the bf16
  // expansion never reaches into the next head's rows
  if (d.kv_dtype == DUO_INT4) c->desc.capacity = round_up(d.capacity, 128);
  c->mask.assign(head_mask, head_mask + (size_t)d.layers * d.n_kv_heads);
  c->seq_len.assign((size_t)d.layers * d.batch, 0);
  c->base = nullptr;
  c->forced_splits = 0;
  c->shard_lo = 0;
  c->shard_hi = kNoShardEnd;
  c->reproducible = false;
  c->out_dtype = desc->kv_dtype == DUO_F32 ? DUO_F32 : DUO_BF16;
  c->stall_ns = 0;
  c->have_cfg = false;
  c->row_bytes = d.kv_dtype == DUO_INT4 ? d.head_dim / 2 : d.head_dim * elem_bytes(d.kv_dtype);
  c->pool_blocks = paged ? pool_blocks : 0;
  c->table_stride = paged ? (int)((c->desc.capacity + duo::kPageTokens - 1) / duo::kPageTokens) : 0;
  const bool q4 = d.kv_dtype == DUO_INT4;

  int64_t off = 0;
  auto take = [&](int64_t bytes) {
    const int64_t at = off;
    off = round_up(off + bytes, kAlign);
    return at;
  };
  c->n_ret_max = 0;
  for (int l = 0; l < d.layers; ++l) {
    duo_cache::Layer L{};
    L.n_ret = L.n_str = 0;
    for (int h = 0; h < d.n_kv_heads; ++h) {
      const bool ret = c->mask[(size_t)l * d.n_kv_heads + h] != 0;
      L.h.kind[h] = ret ? 1 : 0;
      if (ret) {
        L.h.index[h] = (int8_t)L.n_ret;
        L.h.ret_heads[L.n_ret++] = (int8_t)h;
      } else {
        L.h.index[h] = (int8_t)L.n_str;
        L.h.str_heads[L.n_str++] = (int8_t)h;
      }
    }
    L.ret_rows = paged ? pool_blocks * L.n_ret * duo::kPageTokens
                       : (int64_t)d.batch * L.n_ret * c->desc.capacity;
    const int64_t str_rows = (int64_t)d.batch * L.n_str * c->Ws;
    L.off_ret_k = L.n_ret ? take(L.ret_rows * c->row_bytes) : -1;
    L.off_ret_v = L.n_ret ? take(L.ret_rows * c->row_bytes) : -1;
    L.off_str_k = L.n_str ? take(str_rows * c->row_bytes) : -1;
    L.off_str_v = L.n_str ? take(str_rows * c->row_bytes) : -1;
    L.off_ret_k_sz = (q4 && L.n_ret) ? take(L.ret_rows * 4) : -1;
    L.off_ret_v_sz = (q4 && L.n_ret) ? take(L.ret_rows * 4) : -1;
    L.off_str_k_sz = (q4 && L.n_str) ? take(str_rows * 4) : -1;
    L.off_str_v_sz = (q4 && L.n_str) ? take(str_rows * 4) : -1;
    if (L.n_ret > c->n_ret_max) c->n_ret_max = L.n_ret;
    c->layers.push_back(L);
  }
  c->off_table = paged ? take((int64_t)d.batch * c->table_stride * 4) : -1;
  if (paged) {
    c->table.assign((size_t)d.batch * c->table_stride, -1);
    c->held.assign(d.batch, 0);
    c->free_blocks.clear();
    for (int64_t i = pool_blocks - 1; i >= 0; --i) c->free_blocks.push_back((int32_t)i);
  }
  c->cache_bytes = (size_t)off;
  c->ws_bytes = (size_t)ws_layout(c->desc, c->n_ret_max).total;
  *out = c;
  return DUO_OK;
}

// ---------------------------------------------------------------- append

duo_status append_rows(duo_cache *c, int32_t layer, const std::vector<int32_t> &rows,
                       const void *k, const void *v, int32_t n_tokens, cudaStream_t s) {
  if (n_tokens < 0) return DUO_ERR_ARG;
  if (n_tokens > 0 && (!k || !v || !aligned16(k) || !aligned16(v))) return DUO_ERR_ARG;
  duo_status st = check_room(c, layer, rows, n_tokens);
  if (st != DUO_OK) return st;
  if (n_tokens == 0) return DUO_OK;  // k and v are not read (may be NULL)
  if ((st = reserve_blocks(c, layer, rows, n_tokens, s)) != DUO_OK) return st;
  const auto &L = c->layers[layer];
  const duo_cache_desc &d = c->desc;
  duo::AppendParams a{};
  a.p = layer_ptrs(c, layer);
  a.h = L.h;
  a.ret = ret_map(c, layer);
  a.Hkv = d.n_kv_heads;
  a.D = d.head_dim;
  a.n_ret = L.n_ret;
  a.n_str = L.n_str;
  a.S = c->S;
  a.R = c->R;
  a.W = c->W;
  a.Ws = c->Ws;
  a.n_tok = n_tokens;
  a.shard_lo = c->shard_lo;
  a.shard_hi = c->shard_hi;
  // inputs [rows][n_tokens][Hkv][D] in f32 (f32 caches) or bf16
  const int64_t in_row = (int64_t)n_tokens * d.n_kv_heads * d.head_dim * elem_bytes(d.kv_dtype);
  for (size_t g0 = 0; g0 < rows.size(); g0 += duo::kMaxLaunchRows) {
    const int nr = (int)std::min<size_t>(duo::kMaxLaunchRows, rows.size() - g0);
    a.rows.n = nr;
    for (int r = 0; r < nr; ++r) {
      a.rows.row[r] = rows[g0 + r];
      a.rows.len[r] = (int32_t)len_of(c, layer, rows[g0 + r]);
    }
    a.k = static_cast<const uint8_t *>(k) + (int64_t)g0 * in_row;
    a.v = static_cast<const uint8_t *>(v) + (int64_t)g0 * in_row;
    if ((st = cuda_status(duo::launch_append(a, d.kv_dtype, s))) != DUO_OK) return st;
  }
  for (int b : rows) len_of(c, layer, b) += n_tokens;
  return DUO_OK;
}

// ---------------------------------------------------------------- decode

// Fields of a decode launch that do not depend on its rows.
void fill_decode_common(const duo_cache *c, int32_t layer, const void *q, void *out, float scale,
                        duo::DecodeParams *p) {
  const auto &L = c->layers[layer];
  const duo_cache_desc &d = c->desc;
  std::memset(p, 0, sizeof(*p));
  p->q = q;
  p->out = out;
  p->p = layer_ptrs(c, layer);
  p->h = L.h;
  p->ret = ret_map(c, layer);
  p->B = d.batch;
  p->Hq = d.n_q_heads;
  p->Hkv = d.n_kv_heads;
  p->G = d.n_q_heads / d.n_kv_heads;
  p->D = d.head_dim;
  p->n_ret = L.n_ret;
  p->n_str = L.n_str;
  p->S = c->S;
  p->R = c->R;
  p->W = c->W;
  p->Ws = c->Ws;
  p->cap = d.capacity;
  const float sc = scale > 0.f ? scale : 1.0f / std::sqrt((float)d.head_dim);
  p->scale_log2 = sc * 1.4426950408889634f;
  p->err = duo::device_error_word();
  p->pool = c->reproducible ? 0 : 1;
  p->str_pack = 1;
  p->out_f32 = (d.kv_dtype != DUO_F32 && c->out_dtype == DUO_F32) ? 1 : 0;
  p->shard_lo = c->shard_lo;
  p->shard_hi = c->shard_hi;
}

// Partial-mode outputs of a decode (sequence shards), or none.
struct Partial {
  float *o, *lse;
  int own_str;
};

// Where a decode launch keeps its split partials: the caller's workspace, or
// the library's static array (cleared on the stream before the launch).
struct Scratch {
  void *ws;
  size_t ws_bytes;
  bool is_static;
};

// Checks a launch that needs scratch for `units` tickets and `slots` partials
// can get it; nothing is enqueued.
duo_status check_scratch(const duo_cache *c, int64_t units, int64_t slots, const Scratch &sc,
                         int G) {
  if (sc.is_static) {
    const StaticLayout sl = static_layout(units, slots, G, c->desc.head_dim);
    return sl.total > (int64_t)duo::decode_static_scratch_bytes() ? DUO_ERR_WORKSPACE : DUO_OK;
  }
  const WsLayout w = ws_layout(c->desc, c->n_ret_max);
  if (!sc.ws || sc.ws_bytes < (size_t)w.total) return DUO_ERR_WORKSPACE;
  if ((reinterpret_cast<uintptr_t>(sc.ws) % kAlign) != 0) return DUO_ERR_ARG;
  return DUO_OK;
}

// Point launch p at its (already checked) scratch.
duo_status attach_scratch(const duo_cache *c, int64_t units, int64_t slots, const Scratch &sc,
                          cudaStream_t s, duo::DecodeParams *p) {
  if (!sc.is_static) {
    const WsLayout w = ws_layout(c->desc, c->n_ret_max);
    uint8_t *wsb = static_cast<uint8_t *>(sc.ws);
    p->ws_cnt = reinterpret_cast<unsigned *>(wsb + w.cnt);
    p->ws_next = reinterpret_cast<unsigned *>(wsb + w.next);
    p->ws_lse = reinterpret_cast<float *>(wsb + w.lse);
    p->ws_o = reinterpret_cast<float *>(wsb + w.o);
    return DUO_OK;
  }
  const StaticLayout sl = static_layout(units, slots, p->G, p->D);
  void *ptr = nullptr;
  if (duo::decode_static_scratch(&ptr) != cudaSuccess) return DUO_ERR_CUDA;
  uint8_t *scratch = static_cast<uint8_t *>(ptr);
  // tickets and counters start at zero for this launch (the array keeps
  // earlier calls' bytes)
  if (cudaMemsetAsync(scratch, 0, (size_t)sl.lse, s) != cudaSuccess) return DUO_ERR_CUDA;
  p->ws_cnt = reinterpret_cast<unsigned *>(scratch);
  p->ws_next = reinterpret_cast<unsigned *>(scratch + sl.next);
  p->ws_lse = reinterpret_cast<float *>(scratch + sl.lse);
  p->ws_o = reinterpret_cast<float *>(scratch + sl.o);
  return DUO_OK;
}

// Decode attention for `rows` of a layer.  With k_new/v_new ([rows][Hkv][D])
// each row's new token is appended in the same launch (fused step).
duo_status decode_rows(duo_cache *c, int32_t layer, const std::vector<int32_t> &rows,
                       const void *q, const void *k_new, const void *v_new, void *out, float scale,
                       const Scratch &scratch, cudaStream_t s, const Partial *part = nullptr) {
  if (!q || !std::isfinite(scale)) return DUO_ERR_ARG;
  if (part ? (!part->o || !part->lse) : !out) return DUO_ERR_ARG;
  const bool fused = k_new != nullptr;
  // A shard's decode is only meaningful as a partial to be merged; partials
  // come from the tensor-core decode and do not append.
  if (sharded(c) && !part) return DUO_ERR_UNSUPPORTED;
  if (part && (fused || !mma_path(c))) return DUO_ERR_UNSUPPORTED;
  const duo_cache_desc &d = c->desc;
  const auto &L = c->layers[layer];
  const int G = d.n_q_heads / d.n_kv_heads;
  for (int b : rows)
    if (len_of(c, layer, b) + (fused ? 1 : 0) <= 0) return DUO_ERR_STATE;
  duo::DecodeConfig cfg{};
  cudaError_t e = cached_decode_config(c, &cfg);
  if (e != cudaSuccess) return launch_status(e);
  duo_status st;

  if (!mma_path(c)) {
    // CUDA-core decode: every batch row, in order, at one length
    bool whole = rows.size() == (size_t)d.batch && !fused;
    for (size_t i = 0; whole && i < rows.size(); ++i)
      whole = rows[i] == (int)i && len_of(c, layer, (int)i) == len_of(c, layer, 0);
    if (!whole) return DUO_ERR_UNSUPPORTED;
    const int64_t n = len_of(c, layer, 0);
    duo::DecodeParams p;
    fill_decode_common(c, layer, q, out, scale, &p);
    const int want = choose_splits(c, layer, n, cfg);
    const int64_t split_len = round_up((n + want - 1) / want, cfg.tile_rows);
    p.n = n;
    p.nsplit = (int)((n + split_len - 1) / split_len);
    p.split_len = split_len;
    if (L.n_ret > 0 && p.nsplit > 1) {
      const int64_t units = (int64_t)d.batch * L.n_ret;
      if ((st = check_scratch(c, units, units * p.nsplit, scratch, G)) != DUO_OK) return st;
      if ((st = attach_scratch(c, units, units * p.nsplit, scratch, s, &p)) != DUO_OK) return st;
    }
    return launch_status(duo::launch_decode(p, d.kv_dtype, s));
  }

  // Tensor-core decode: plan every launch (up to DUO_MAX_LAUNCH_ROWS rows
  // each) and check its scratch before anything is enqueued.
  const int64_t q_row = (int64_t)d.n_q_heads * d.head_dim * 2;   // bf16 q per row
  const int64_t o_row = (int64_t)d.n_q_heads * d.head_dim * (c->out_dtype == DUO_F32 ? 4 : 2);
  const int64_t kv_row = (int64_t)d.n_kv_heads * d.head_dim * 2;  // bf16 k_new / v_new per row
  std::vector<duo::DecodeParams> plans((rows.size() + duo::kMaxLaunchRows - 1) / duo::kMaxLaunchRows);
  std::vector<char> needs(plans.size(), 0);
  for (size_t i = 0; i < plans.size(); ++i) {
    const size_t g0 = i * duo::kMaxLaunchRows;
    const int nr = (int)std::min<size_t>(duo::kMaxLaunchRows, rows.size() - g0);
    duo::DecodeParams &p = plans[i];
    fill_decode_common(c, layer, static_cast<const uint8_t *>(q) + (int64_t)g0 * q_row,
                       out ? static_cast<uint8_t *>(out) + (int64_t)g0 * o_row : nullptr, scale, &p);
    p.rows.n = nr;
    int32_t rlen[duo::kMaxLaunchRows];  // retrieval keys of each row in this shard
    for (int r = 0; r < nr; ++r) {
      p.rows.row[r] = rows[g0 + r];
      p.rows.len[r] = (int32_t)(len_of(c, layer, rows[g0 + r]) + (fused ? 1 : 0));
      rlen[r] = (int32_t)ret_len(c, p.rows.len[r]);
    }
    p.str_pack = plan_launch(c, layer, rlen, p.rows.len, nr, cfg, p.nsplit_r);
    if (part) {
      p.part_o = part->o + (int64_t)g0 * d.n_q_heads * d.head_dim;
      p.part_lse = part->lse + (int64_t)g0 * d.n_q_heads;
      p.own_str = part->own_str;
    }
    p.cta0[0] = 0;
    for (int r = 0; r < nr; ++r) {
      p.cta0[r + 1] = p.cta0[r] + L.n_ret * p.nsplit_r[r];
      needs[i] = needs[i] || (L.n_ret > 0 && p.nsplit_r[r] > 1);
    }
    if (fused) {
      p.knew = static_cast<const uint8_t *>(k_new) + (int64_t)g0 * kv_row;
      p.vnew = static_cast<const uint8_t *>(v_new) + (int64_t)g0 * kv_row;
    }
    p.pdl = 1;
    if (needs[i] && (st = check_scratch(c, (int64_t)nr * L.n_ret, p.cta0[nr], scratch, G)) != DUO_OK)
      return st;
  }
  if (fused) {
    if ((st = check_room(c, layer, rows, 1)) != DUO_OK) return st;
    if ((st = reserve_blocks(c, layer, rows, 1, s)) != DUO_OK) return st;
  }
  for (size_t i = 0; i < plans.size(); ++i) {
    duo::DecodeParams &p = plans[i];
    if (needs[i] &&
        (st = attach_scratch(c, (int64_t)p.rows.n * L.n_ret, p.cta0[p.rows.n], scratch, s, &p)) != DUO_OK)
      return st;
    if ((st = launch_status(duo::launch_decode(p, d.kv_dtype, s))) != DUO_OK) return st;
  }
  if (fused)
    for (int b : rows) len_of(c, layer, b) += 1;
  return DUO_OK;
}

duo_status step_rows(duo_cache *c, int32_t layer, const std::vector<int32_t> &rows, const void *q,
                     const void *k_new, const void *v_new, void *out, float scale,
                     const Scratch &scratch, cudaStream_t s) {
  if (!q || !out || !k_new || !v_new || !aligned16(k_new) || !aligned16(v_new)) return DUO_ERR_ARG;
  const duo_cache_desc &d = c->desc;
  if (!duo::decode_can_fuse_append(d.kv_dtype, d.head_dim, d.n_q_heads / d.n_kv_heads)) {
    // no fused kernel for this configuration: append, then attend
    duo_status st = append_rows(c, layer, rows, k_new, v_new, 1, s);
    if (st != DUO_OK) return st;
    return decode_rows(c, layer, rows, q, nullptr, nullptr, out, scale, scratch, s);
  }
  return decode_rows(c, layer, rows, q, k_new, v_new, out, scale, scratch, s);
}

// ---------------------------------------------------------------- pre-fill

// Pre-fill scratch of a 4-bit cache: the bf16 expansion of one layer's
// history, [retrieval K][retrieval V] at the layer's storage rows and
// [streaming K][streaming V] as [batch][n_str][S+R][d]; the largest layer.
struct PrefillScratch {
  int64_t ret_v, str_k, str_v, total;
};

PrefillScratch prefill_scratch(const duo_cache *c, int layer) {
  const int64_t row = (int64_t)c->desc.head_dim * 2;
  const auto &L = c->layers[layer];
  PrefillScratch ps;
  const int64_t ret = round_up(L.ret_rows * row, kAlign);
  const int64_t str = round_up((int64_t)c->desc.batch * L.n_str * c->W * row, kAlign);
  ps.ret_v = ret;
  ps.str_k = 2 * ret;
  ps.str_v = 2 * ret + str;
  ps.total = 2 * ret + 2 * str;
  return ps;
}

size_t prefill_ws_bytes(const duo_cache *c) {
  if (c->desc.kv_dtype != DUO_INT4) return 0;
  int64_t m = 0;
  for (int l = 0; l < c->desc.layers; ++l) m = std::max(m, prefill_scratch(c, l).total);
  return (size_t)m;
}

duo_status prefill_rows(duo_cache *c, int32_t layer, const std::vector<int32_t> &rows,
                        const void *q, const void *k, const void *v, int32_t C, void *out,
                        float scale, void *ws, size_t ws_bytes, cudaStream_t s) {
  if (!q || !k || !v || !out || C <= 0) return DUO_ERR_ARG;
  if (!std::isfinite(scale)) return DUO_ERR_ARG;
  const duo_cache_desc &d = c->desc;
  if ((d.kv_dtype != DUO_BF16 && d.kv_dtype != DUO_INT4) || d.head_dim != 128)
    return DUO_ERR_UNSUPPORTED;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)) return DUO_ERR_ARG;
  const auto &L = c->layers[layer];
  duo_status st = check_room(c, layer, rows, C);
  if (st != DUO_OK) return st;
  if (sharded(c)) return DUO_ERR_UNSUPPORTED;
  const bool q4 = d.kv_dtype == DUO_INT4;
  uint8_t *wsb = static_cast<uint8_t *>(ws);
  if (q4) {
    if (!ws || ws_bytes < prefill_ws_bytes(c)) return DUO_ERR_WORKSPACE;
    if ((reinterpret_cast<uintptr_t>(ws) % kAlign) != 0) return DUO_ERR_ARG;
  }
  duo::PrefillParams p{};
  p.p = layer_ptrs(c, layer);
  duo::DequantParams dq{};
  if (q4) {
    // the kernel reads the bf16 expansion of the history instead of the codes
    const PrefillScratch ps = prefill_scratch(c, layer);
    dq.p = p.p;
    dq.h = L.h;
    dq.ret = ret_map(c, layer);
    dq.n_ret = L.n_ret;
    dq.n_str = L.n_str;
    dq.S = c->S;
    dq.R = c->R;
    dq.W = c->W;
    dq.Ws = c->Ws;
    dq.D = d.head_dim;
    dq.ret_k = reinterpret_cast<__nv_bfloat16 *>(wsb);
    dq.ret_v = reinterpret_cast<__nv_bfloat16 *>(wsb + ps.ret_v);
    dq.str_k = reinterpret_cast<__nv_bfloat16 *>(wsb + ps.str_k);
    dq.str_v = reinterpret_cast<__nv_bfloat16 *>(wsb + ps.str_v);
    p.p = duo::LayerPtrs{};
    if (L.n_ret) {
      p.p.ret_k = wsb;
      p.p.ret_v = wsb + ps.ret_v;
    }
    if (L.n_str) {
      p.p.str_k = wsb + ps.str_k;
      p.p.str_v = wsb + ps.str_v;
    }
  }
  p.h = L.h;
  p.ret = ret_map(c, layer);
  p.B = d.batch;
  p.Hq = d.n_q_heads;
  p.Hkv = d.n_kv_heads;
  p.G = d.n_q_heads / d.n_kv_heads;
  p.D = d.head_dim;
  p.n_ret = L.n_ret;
  p.n_str = L.n_str;
  p.S = c->S;
  p.R = c->R;
  p.W = c->W;
  p.C = C;
  p.retrieval_rows = L.ret_rows;
  const float sc = scale > 0.f ? scale : 1.0f / std::sqrt((float)d.head_dim);
  p.scale_log2 = sc * 1.4426950408889634f;
  p.err = duo::device_error_word();
  p.wait_ns = c->stall_ns > 0 ? (uint64_t)c->stall_ns : duo::kPrefillWaitNs;
  p.skip_loads = c->stall_ns > 0 ? 1 : 0;
  c->stall_ns = 0;  // one call only
  const int64_t q_row = (int64_t)C * d.n_q_heads * d.head_dim * 2;
  const int64_t kv_row = (int64_t)C * d.n_kv_heads * d.head_dim * 2;
  for (size_t g0 = 0; g0 < rows.size(); g0 += duo::kMaxLaunchRows) {
    const int nr = (int)std::min<size_t>(duo::kMaxLaunchRows, rows.size() - g0);
    p.rows.n = nr;
    for (int r = 0; r < nr; ++r) {
      p.rows.row[r] = rows[g0 + r];
      p.rows.len[r] = (int32_t)len_of(c, layer, rows[g0 + r]);
    }
    p.q = static_cast<const uint8_t *>(q) + (int64_t)g0 * q_row;
    p.k = static_cast<const uint8_t *>(k) + (int64_t)g0 * kv_row;
    p.v = static_cast<const uint8_t *>(v) + (int64_t)g0 * kv_row;
    p.out = static_cast<uint8_t *>(out) + (int64_t)g0 * q_row;
    if (q4) {
      dq.rows = p.rows;
      if ((st = cuda_status(duo::launch_dequant_history(dq, s))) != DUO_OK) return st;
    }
    if ((st = launch_status(duo::launch_prefill(p, s))) != DUO_OK) return st;
  }
  return DUO_OK;
}

}  // namespace

extern "C" {

const char *duo_status_string(duo_status s) {
  switch (s) {
    case DUO_OK: return "ok";
    case DUO_ERR_ARG: return "invalid argument";
    case DUO_ERR_CAPACITY: return "retrieval capacity or block pool exceeded";
    case DUO_ERR_LAYOUT: return "inconsistent head layout";
    case DUO_ERR_WORKSPACE: return "workspace missing or too small";
    case DUO_ERR_CUDA: return "CUDA error";
    case DUO_ERR_TIMEOUT: return "bounded device wait gave up";
    case DUO_ERR_UNSUPPORTED: return "unsupported configuration";
    case DUO_ERR_STATE: return "cache not bound or call out of order";
  }
  return "unknown status";
}

duo_status duo_cache_create(duo_cache **out, const duo_cache_desc *desc, const uint8_t *head_mask,
                            int32_t S, int32_t R, int32_t layout) {
  if (layout != DUO_LAYOUT_PACKED) {
    if (out) *out = nullptr;
    return DUO_ERR_ARG;
  }
  return create(out, desc, head_mask, S, R, layout, 0);
}

duo_status duo_cache_create_paged(duo_cache **out, const duo_cache_desc *desc,
                                  const uint8_t *head_mask, int32_t S, int32_t R,
                                  int64_t pool_blocks) {
  return create(out, desc, head_mask, S, R, DUO_LAYOUT_PAGED, pool_blocks);
}

void duo_cache_destroy(duo_cache *c) { delete c; }

duo_status duo_cache_required_bytes(const duo_cache *c, size_t *cache_bytes, size_t *ws_bytes) {
  if (!c) return DUO_ERR_ARG;
  if (cache_bytes) *cache_bytes = c->cache_bytes;
  if (ws_bytes) *ws_bytes = c->ws_bytes;
  return DUO_OK;
}

duo_status duo_cache_bind(duo_cache *c, void *mem, size_t bytes) {
  if (!c || !mem) return DUO_ERR_ARG;
  if ((reinterpret_cast<uintptr_t>(mem) % kAlign) != 0) return DUO_ERR_ARG;
  if (bytes < c->cache_bytes) return DUO_ERR_ARG;
  cudaError_t e = cudaMemset(mem, 0, c->cache_bytes);
  if (e != cudaSuccess) return DUO_ERR_CUDA;
  if ((e = cudaDeviceSynchronize()) != cudaSuccess) return DUO_ERR_CUDA;
  c->base = static_cast<uint8_t *>(mem);
  reset_lengths(c);
  return DUO_OK;
}

duo_status duo_cache_reset(duo_cache *c) {
  if (!c) return DUO_ERR_ARG;
  reset_lengths(c);
  return DUO_OK;
}

duo_status duo_append_kv(duo_cache *c, int32_t layer, const void *k, const void *v,
                         int32_t n_tokens, duo_stream stream) {
  return duo_append_kv_rows(c, layer, nullptr, 0, k, v, n_tokens, stream);
}

duo_status duo_append_kv_rows(duo_cache *c, int32_t layer, const int32_t *rows, int32_t n_rows,
                              const void *k, const void *v, int32_t n_tokens, duo_stream stream) {
  duo_status st = check_layer(c, layer);
  if (st != DUO_OK) return st;
  std::vector<int32_t> list;
  if ((st = make_rows(c, rows, n_rows, &list)) != DUO_OK) return st;
  return append_rows(c, layer, list, k, v, n_tokens, (cudaStream_t)stream);
}

duo_status duo_decode_attn(duo_cache *c, int32_t layer, const void *q, void *out, float scale,
                           void *ws, size_t ws_bytes, duo_stream stream) {
  return duo_decode_attn_rows(c, layer, nullptr, 0, q, out, scale, ws, ws_bytes, stream);
}

duo_status duo_decode_attn_rows(duo_cache *c, int32_t layer, const int32_t *rows, int32_t n_rows,
                                const void *q, void *out, float scale, void *ws, size_t ws_bytes,
                                duo_stream stream) {
  duo_status st = check_layer(c, layer);
  if (st != DUO_OK) return st;
  std::vector<int32_t> list;
  if ((st = make_rows(c, rows, n_rows, &list)) != DUO_OK) return st;
  return decode_rows(c, layer, list, q, nullptr, nullptr, out, scale, Scratch{ws, ws_bytes, false},
                     (cudaStream_t)stream);
}

duo_status duo_decode_step(duo_cache *c, int32_t layer, const void *q, const void *k_new,
                           const void *v_new, void *out, float scale, void *ws, size_t ws_bytes,
                           duo_stream stream) {
  return duo_decode_step_rows(c, layer, nullptr, 0, q, k_new, v_new, out, scale, ws, ws_bytes,
                              stream);
}

duo_status duo_decode_step_rows(duo_cache *c, int32_t layer, const int32_t *rows, int32_t n_rows,
                                const void *q, const void *k_new, const void *v_new, void *out,
                                float scale, void *ws, size_t ws_bytes, duo_stream stream) {
  duo_status st = check_layer(c, layer);
  if (st != DUO_OK) return st;
  std::vector<int32_t> list;
  if ((st = make_rows(c, rows, n_rows, &list)) != DUO_OK) return st;
  return step_rows(c, layer, list, q, k_new, v_new, out, scale, Scratch{ws, ws_bytes, false},
                   (cudaStream_t)stream);
}

duo_status duo_decode_attn_static(duo_cache *c, int32_t layer, const void *q, void *out,
                                  float scale, duo_stream stream) {
  duo_status st = check_layer(c, layer);
  if (st != DUO_OK) return st;
  std::vector<int32_t> list;
  if ((st = make_rows(c, nullptr, 0, &list)) != DUO_OK) return st;
  return decode_rows(c, layer, list, q, nullptr, nullptr, out, scale, Scratch{nullptr, 0, true},
                     (cudaStream_t)stream);
}

duo_status duo_prefill_attn(duo_cache *c, int32_t layer, const void *q, const void *k,
                            const void *v, int32_t C, void *out, float scale, void *ws,
                            size_t ws_bytes, duo_stream stream) {
  return duo_prefill_attn_rows(c, layer, nullptr, 0, q, k, v, C, out, scale, ws, ws_bytes, stream);
}

duo_status duo_prefill_attn_rows(duo_cache *c, int32_t layer, const int32_t *rows, int32_t n_rows,
                                 const void *q, const void *k, const void *v, int32_t C, void *out,
                                 float scale, void *ws, size_t ws_bytes, duo_stream stream) {
  duo_status st = check_layer(c, layer);
  if (st != DUO_OK) return st;
  std::vector<int32_t> list;
  if ((st = make_rows(c, rows, n_rows, &list)) != DUO_OK) return st;
  return prefill_rows(c, layer, list, q, k, v, C, out, scale, ws, ws_bytes, (cudaStream_t)stream);
}

duo_status duo_prefill_workspace_bytes(const duo_cache *c, size_t *bytes) {
  if (!c || !bytes) return DUO_ERR_ARG;
  *bytes = prefill_ws_bytes(c);
  return DUO_OK;
}

duo_status duo_release_rows(duo_cache *c, const int32_t *rows, int32_t n_rows) {
  if (!c) return DUO_ERR_ARG;
  std::vector<int32_t> list;
  duo_status st = make_rows(c, rows, n_rows, &list);
  if (st != DUO_OK) return st;
  for (int b : list) {
    for (int l = 0; l < c->desc.layers; ++l) len_of(c, l, b) = 0;
    release_blocks(c, b);
  }
  return DUO_OK;
}

duo_status duo_set_retrieval_shard(duo_cache *c, int64_t lo, int64_t hi) {
  if (!c || lo < 0 || hi <= lo) return DUO_ERR_ARG;
  if (!mma_path(c)) return DUO_ERR_UNSUPPORTED;
  for (int64_t n : c->seq_len)
    if (n != 0) return DUO_ERR_STATE;
  c->shard_lo = lo;
  c->shard_hi = std::min(hi, kNoShardEnd);
  return DUO_OK;
}

duo_status duo_decode_attn_partial(duo_cache *c, int32_t layer, const void *q, float *o_part,
                                   float *lse_part, int32_t owns_streaming, float scale, void *ws,
                                   size_t ws_bytes, duo_stream stream) {
  duo_status st = check_layer(c, layer);
  if (st != DUO_OK) return st;
  if (owns_streaming != 0 && owns_streaming != 1) return DUO_ERR_ARG;
  std::vector<int32_t> list;
  if ((st = make_rows(c, nullptr, 0, &list)) != DUO_OK) return st;
  const Partial part{o_part, lse_part, owns_streaming};
  return decode_rows(c, layer, list, q, nullptr, nullptr, nullptr, scale,
                     Scratch{ws, ws_bytes, false}, (cudaStream_t)stream, &part);
}

duo_status duo_merge_partials(int32_t n_parts, int64_t rows, int32_t head_dim, const float *o_parts,
                              const float *lse_parts, void *out, int32_t out_dtype,
                              duo_stream stream) {
  if (n_parts <= 0 || rows <= 0 || !o_parts || !lse_parts || !out) return DUO_ERR_ARG;
  if (head_dim != 64 && head_dim != 128) return DUO_ERR_ARG;
  if (out_dtype != DUO_F32 && out_dtype != DUO_BF16) return DUO_ERR_ARG;
  if (!aligned16(o_parts)) return DUO_ERR_ARG;
  return launch_status(duo::launch_merge_partials(n_parts, rows, head_dim, o_parts, lse_parts, out,
                                                  out_dtype == DUO_F32 ? duo::kF32 : duo::kBF16,
                                                  (cudaStream_t)stream));
}

duo_status duo_seq_len(const duo_cache *c, int32_t layer, int64_t *n) {
  if (!c || !n || layer < 0 || layer >= c->desc.layers) return DUO_ERR_ARG;
  int64_t m = 0;
  for (int b = 0; b < c->desc.batch; ++b) m = std::max(m, len_of(c, layer, b));
  *n = m;
  return DUO_OK;
}

duo_status duo_row_seq_len(const duo_cache *c, int32_t layer, int32_t row, int64_t *n) {
  if (!c || !n || layer < 0 || layer >= c->desc.layers || row < 0 || row >= c->desc.batch)
    return DUO_ERR_ARG;
  *n = len_of(c, layer, row);
  return DUO_OK;
}

duo_status duo_row_blocks(const duo_cache *c, int32_t row, int32_t *blocks, int32_t max_blocks,
                          int32_t *n_blocks) {
  if (!c || !n_blocks || row < 0 || row >= c->desc.batch) return DUO_ERR_ARG;
  if (c->layout != DUO_LAYOUT_PAGED) {
    *n_blocks = 0;
    return DUO_OK;
  }
  const int held = c->held[row];
  *n_blocks = held;
  if (blocks) {
    if (max_blocks < held) return DUO_ERR_ARG;
    std::memcpy(blocks, c->table.data() + (size_t)row * c->table_stride, (size_t)held * 4);
  }
  return DUO_OK;
}

duo_status duo_pool_free_blocks(const duo_cache *c, int64_t *free_blocks) {
  if (!c || !free_blocks) return DUO_ERR_ARG;
  *free_blocks = (int64_t)c->free_blocks.size();
  return DUO_OK;
}

duo_status duo_kv_bytes(const duo_cache *c, int64_t *kept, int64_t *full) {
  if (!c) return DUO_ERR_ARG;
  const duo_cache_desc &d = c->desc;
  const int64_t per = d.kv_dtype == DUO_INT4 ? 2 * (d.head_dim / 2 + 4)
                                             : 2 * (int64_t)d.head_dim * elem_bytes(d.kv_dtype);
  int64_t k = 0, f = 0;
  for (int l = 0; l < d.layers; ++l)
    for (int b = 0; b < d.batch; ++b) {
      const int64_t n = len_of(c, l, b);
      const int64_t win = n < c->W ? n : c->W;
      k += (c->layers[l].n_ret * ret_len(c, n) + c->layers[l].n_str * win) * per;
      f += (int64_t)d.n_kv_heads * n * per;
    }
  if (kept) *kept = k;
  if (full) *full = f;
  return DUO_OK;
}

duo_status duo_layout_info(const duo_cache *c, int32_t layer, duo_layout_view *o) {
  if (!c || !o || layer < 0 || layer >= c->desc.layers) return DUO_ERR_ARG;
  const auto &L = c->layers[layer];
  std::memset(o, 0, sizeof(*o));
  o->n_retrieval = L.n_ret;
  o->n_streaming = L.n_str;
  o->window = c->W;
  o->window_stride = c->Ws;
  o->row_bytes = c->row_bytes;
  o->capacity = c->desc.capacity;
  duo_seq_len(c, layer, &o->seq_len);
  o->ret_k = L.off_ret_k;
  o->ret_v = L.off_ret_v;
  o->str_k = L.off_str_k;
  o->str_v = L.off_str_v;
  o->ret_k_sz = L.off_ret_k_sz;
  o->ret_v_sz = L.off_ret_v_sz;
  o->str_k_sz = L.off_str_k_sz;
  o->str_v_sz = L.off_str_v_sz;
  for (int h = 0; h < c->desc.n_kv_heads; ++h) {
    o->kind[h] = L.h.kind[h];
    o->packed_index[h] = L.h.index[h];
  }
  o->layout = c->layout;
  o->page_tokens = c->layout == DUO_LAYOUT_PAGED ? duo::kPageTokens : 0;
  o->table_stride = c->table_stride;
  o->pool_blocks = c->pool_blocks;
  o->block_table = c->off_table;
  return DUO_OK;
}

duo_status duo_set_decode_splits(duo_cache *c, int32_t splits) {
  if (!c || splits < 0 || splits > DUO_MAX_SPLITS) return DUO_ERR_ARG;
  c->forced_splits = splits;
  return DUO_OK;
}

duo_status duo_test_stall_next_prefill(duo_cache *c, int64_t wait_ns) {
  if (!c || wait_ns < 1000 || wait_ns > 1000000000LL) return DUO_ERR_ARG;
  c->stall_ns = wait_ns;
  return DUO_OK;
}

duo_status duo_set_decode_output(duo_cache *c, int32_t dtype) {
  if (!c || (dtype != DUO_F32 && dtype != DUO_BF16)) return DUO_ERR_ARG;
  if (c->desc.kv_dtype == DUO_F32 && dtype != DUO_F32) return DUO_ERR_UNSUPPORTED;
  c->out_dtype = dtype;
  return DUO_OK;
}

duo_status duo_set_decode_reproducible(duo_cache *c, int32_t on) {
  if (!c || (on != 0 && on != 1)) return DUO_ERR_ARG;
  c->reproducible = on == 1;
  return DUO_OK;
}

// The plan of a tensor-core decode of every row at the current lengths: the
// largest split count a row gets and the largest streaming pack of a launch.
void decode_plan_all_rows(const duo_cache *c, int32_t layer, const duo::DecodeConfig &cfg,
                          int32_t *splits, int32_t *pack) {
  std::vector<int32_t> lens(c->desc.batch), rlen(c->desc.batch);
  std::vector<int16_t> sp(c->desc.batch);
  for (int b = 0; b < c->desc.batch; ++b) {
    lens[b] = (int32_t)std::max<int64_t>(1, len_of(c, layer, b));
    rlen[b] = (int32_t)ret_len(c, lens[b]);
  }
  *splits = 1;
  *pack = 1;
  for (int g0 = 0; g0 < c->desc.batch; g0 += duo::kMaxLaunchRows) {
    const int nr = std::min(duo::kMaxLaunchRows, c->desc.batch - g0);
    *pack = std::max<int32_t>(*pack, plan_launch(c, layer, rlen.data() + g0, lens.data() + g0, nr,
                                                 cfg, sp.data() + g0));
    for (int r = 0; r < nr; ++r) *splits = std::max<int32_t>(*splits, sp[g0 + r]);
  }
}

duo_status duo_decode_splits(const duo_cache *c, int32_t layer, int32_t *splits) {
  if (!c || !splits || layer < 0 || layer >= c->desc.layers) return DUO_ERR_ARG;
  duo::DecodeConfig cfg{};
  cudaError_t e = cached_decode_config(const_cast<duo_cache *>(c), &cfg);
  if (e != cudaSuccess) return launch_status(e);
  int64_t n_max = 1;
  for (int b = 0; b < c->desc.batch; ++b) n_max = std::max(n_max, len_of(c, layer, b));
  if (!mma_path(c)) {
    const int want = choose_splits(c, layer, n_max, cfg);
    const int64_t split_len = round_up((n_max + want - 1) / want, cfg.tile_rows);
    *splits = (int32_t)((n_max + split_len - 1) / split_len);
    return DUO_OK;
  }
  // the largest count an all-rows decode of the current lengths gives a row
  int32_t best = 1, pack = 1;
  decode_plan_all_rows(c, layer, cfg, &best, &pack);
  *splits = best;
  return DUO_OK;
}

duo_status duo_test_plan_decode(const duo_cache *c, int32_t layer, const int32_t *lens,
                                int32_t n_rows, int32_t num_sms, int32_t ctas_per_sm, int32_t *splits,
                                int32_t *pack) {
  if (!c || !lens || !splits || !pack || layer < 0 || layer >= c->desc.layers || n_rows <= 0 ||
      n_rows > duo::kMaxLaunchRows || num_sms <= 0 || ctas_per_sm <= 0)
    return DUO_ERR_ARG;
  if (!mma_path(c)) return DUO_ERR_UNSUPPORTED;
  duo::DecodeConfig cfg{};
  cfg.num_sms = num_sms;
  cfg.ctas_per_sm = ctas_per_sm;
  cfg.tile_rows = duo::decode_mma_tile_rows(c->desc.kv_dtype == DUO_INT4 ? duo::kINT4 : duo::kBF16);
  int32_t len[duo::kMaxLaunchRows], rlen[duo::kMaxLaunchRows];
  int16_t ns[duo::kMaxLaunchRows];
  for (int r = 0; r < n_rows; ++r) {
    if (lens[r] < 1) return DUO_ERR_ARG;
    len[r] = lens[r];
    rlen[r] = (int32_t)ret_len(c, lens[r]);
  }
  *pack = plan_launch(c, layer, rlen, len, n_rows, cfg, ns);
  for (int r = 0; r < n_rows; ++r) splits[r] = ns[r];
  return DUO_OK;
}

duo_status duo_decode_streaming_pack(const duo_cache *c, int32_t layer, int32_t *heads_per_cta) {
  if (!c || !heads_per_cta || layer < 0 || layer >= c->desc.layers) return DUO_ERR_ARG;
  if (!mma_path(c)) {
    *heads_per_cta = 1;
    return DUO_OK;
  }
  duo::DecodeConfig cfg{};
  cudaError_t e = cached_decode_config(const_cast<duo_cache *>(c), &cfg);
  if (e != cudaSuccess) return launch_status(e);
  int32_t best = 1, pack = 1;
  decode_plan_all_rows(c, layer, cfg, &best, &pack);
  *heads_per_cta = pack;
  return DUO_OK;
}

duo_status duo_poll_device_error(int32_t *code) {
  int *word = duo::device_error_word();
  int host = 0;
  cudaError_t e = cudaDeviceSynchronize();
  if (e != cudaSuccess) return DUO_ERR_CUDA;
  if ((e = cudaMemcpy(&host, word, sizeof(int), cudaMemcpyDeviceToHost)) != cudaSuccess)
    return DUO_ERR_CUDA;
  if (host != 0) {
    const int zero = 0;
    if (cudaMemcpy(word, &zero, sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess)
      return DUO_ERR_CUDA;
  }
  if (code) *code = host;
  return host ? DUO_ERR_TIMEOUT : DUO_OK;
}

}  // extern "C"
