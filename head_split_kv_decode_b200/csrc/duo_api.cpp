// C-ABI layer of libduo: validates arguments, plans the packed layout of the
// head-split KV cache, tracks per-layer lengths, and launches the kernels.
//
// Layout (DUO_LAYOUT_PACKED), per layer, each buffer 256-byte aligned:
//   retrieval K, V : [batch][n_retrieval][capacity][row]
//   streaming K, V : [batch][n_streaming][S + R][row]
//   int4 only      : (fp16 scale, fp16 zero) per row, same indexing, for each
// row = head_dim elements (f32 / bf16) or head_dim/2 bytes of 4-bit codes.
// Retrieval heads keep every token; streaming heads keep S sinks plus an
// R-slot ring ("DuoAttention: Efficient Long-Context LLM Inference with
// Retrieval and Streaming Heads" (hotpaper.ai), section "기술적 접근법": a
// full KV cache for retrieval heads and a fixed-length one for streaming
// heads in every layer).
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

struct duo_cache {
  duo_cache_desc desc;
  int S, R, W;
  int Ws;                     // rows per streaming head buffer
  std::vector<uint8_t> mask;  // [layers][Hkv]
  struct Layer {
    int n_ret, n_str;
    duo::HeadTables h;
    int64_t off_ret_k, off_ret_v, off_str_k, off_str_v;
    int64_t off_ret_k_sz, off_ret_v_sz, off_str_k_sz, off_str_v_sz;
  };
  std::vector<Layer> layers;
  std::vector<int64_t> seq_len;
  size_t cache_bytes;
  size_t ws_bytes;
  int n_ret_max;
  int row_bytes;
  uint8_t *base;
  int forced_splits;
  bool reproducible;       // decode splits take fixed key shares only
  bool have_cfg;           // decode launch facts, queried once per cache
  duo::DecodeConfig cfg;
};

namespace {

constexpr int64_t kAlign = 256;

int64_t round_up(int64_t x, int64_t a) { return (x + a - 1) / a * a; }

int elem_bytes(int kv) { return kv == DUO_F32 ? 4 : 2; }

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

duo::LayerPtrs layer_ptrs(const duo_cache *c, int layer) {
  const auto &L = c->layers[layer];
  auto at = [&](int64_t off) { return off < 0 ? nullptr : c->base + off; };
  return duo::LayerPtrs{at(L.off_ret_k),    at(L.off_ret_v),    at(L.off_str_k),
                        at(L.off_str_v),    at(L.off_ret_k_sz), at(L.off_ret_v_sz),
                        at(L.off_str_k_sz), at(L.off_str_v_sz)};
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

duo_status cuda_status(cudaError_t e) { return e == cudaSuccess ? DUO_OK : DUO_ERR_CUDA; }

// Splits per retrieval head: enough CTAs to occupy every SM once (the
// streaming heads' CTAs included), at least two tiles per split.
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

}  // namespace

extern "C" {

const char *duo_status_string(duo_status s) {
  switch (s) {
    case DUO_OK: return "ok";
    case DUO_ERR_ARG: return "invalid argument";
    case DUO_ERR_CAPACITY: return "retrieval page capacity exceeded";
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
  if (!out || !desc || !head_mask) return DUO_ERR_ARG;
  *out = nullptr;
  const duo_cache_desc d = *desc;
  if (d.layers <= 0 || d.batch <= 0 || d.n_q_heads <= 0 || d.n_kv_heads <= 0) return DUO_ERR_ARG;
  if (d.n_kv_heads > DUO_MAX_KV_HEADS || d.n_q_heads % d.n_kv_heads) return DUO_ERR_LAYOUT;
  if (d.head_dim != 64 && d.head_dim != 128) return DUO_ERR_ARG;
  if (d.kv_dtype != DUO_F32 && d.kv_dtype != DUO_BF16 && d.kv_dtype != DUO_INT4) return DUO_ERR_ARG;
  if (d.capacity <= 0 || S < 0 || R < 1) return DUO_ERR_ARG;
  if (layout != DUO_LAYOUT_PACKED) return DUO_ERR_ARG;
  for (int64_t i = 0; i < (int64_t)d.layers * d.n_kv_heads; ++i)
    if (head_mask[i] > 1) return DUO_ERR_LAYOUT;

  duo_cache *c = new (std::nothrow) duo_cache();
  if (!c) return DUO_ERR_ARG;
  c->desc = d;
  c->S = S;
  c->R = R;
  c->W = S + R;
  // INT4 keeps scale/zero rows in 16-byte groups of four tokens, so its row
  // counts per head are rounded up to a multiple of 4.
  c->Ws = d.kv_dtype == DUO_INT4 ? (int)round_up(c->W, 4) : c->W;
  if (d.kv_dtype == DUO_INT4) c->desc.capacity = round_up(d.capacity, 4);
  c->mask.assign(head_mask, head_mask + (size_t)d.layers * d.n_kv_heads);
  c->seq_len.assign(d.layers, 0);
  c->base = nullptr;
  c->forced_splits = 0;
  c->reproducible = false;
  c->have_cfg = false;
  c->row_bytes = d.kv_dtype == DUO_INT4 ? d.head_dim / 2 : d.head_dim * elem_bytes(d.kv_dtype);
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
    const int64_t ret_rows = (int64_t)d.batch * L.n_ret * c->desc.capacity;
    const int64_t str_rows = (int64_t)d.batch * L.n_str * c->Ws;
    L.off_ret_k = L.n_ret ? take(ret_rows * c->row_bytes) : -1;
    L.off_ret_v = L.n_ret ? take(ret_rows * c->row_bytes) : -1;
    L.off_str_k = L.n_str ? take(str_rows * c->row_bytes) : -1;
    L.off_str_v = L.n_str ? take(str_rows * c->row_bytes) : -1;
    L.off_ret_k_sz = (q4 && L.n_ret) ? take(ret_rows * 4) : -1;
    L.off_ret_v_sz = (q4 && L.n_ret) ? take(ret_rows * 4) : -1;
    L.off_str_k_sz = (q4 && L.n_str) ? take(str_rows * 4) : -1;
    L.off_str_v_sz = (q4 && L.n_str) ? take(str_rows * 4) : -1;
    if (L.n_ret > c->n_ret_max) c->n_ret_max = L.n_ret;
    c->layers.push_back(L);
  }
  c->cache_bytes = (size_t)off;
  c->ws_bytes = (size_t)ws_layout(c->desc, c->n_ret_max).total;
  *out = c;
  return DUO_OK;
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
  for (auto &n : c->seq_len) n = 0;
  return DUO_OK;
}

duo_status duo_cache_reset(duo_cache *c) {
  if (!c) return DUO_ERR_ARG;
  for (auto &n : c->seq_len) n = 0;
  return DUO_OK;
}

duo_status duo_append_kv(duo_cache *c, int32_t layer, const void *k, const void *v,
                         int32_t n_tokens, duo_stream stream) {
  if (!c || !k || !v || n_tokens < 0) return DUO_ERR_ARG;
  if (layer < 0 || layer >= c->desc.layers) return DUO_ERR_ARG;
  if (!c->base) return DUO_ERR_STATE;
  if (!aligned16(k) || !aligned16(v)) return DUO_ERR_ARG;
  const auto &L = c->layers[layer];
  const int64_t n_cur = c->seq_len[layer];
  if (L.n_ret > 0 && n_cur + n_tokens > c->desc.capacity) return DUO_ERR_CAPACITY;
  if (n_tokens == 0) return DUO_OK;
  duo::AppendParams a{};
  a.k = k;
  a.v = v;
  a.p = layer_ptrs(c, layer);
  a.h = L.h;
  a.B = c->desc.batch;
  a.Hkv = c->desc.n_kv_heads;
  a.D = c->desc.head_dim;
  a.n_ret = L.n_ret;
  a.n_str = L.n_str;
  a.S = c->S;
  a.R = c->R;
  a.W = c->W;
  a.Ws = c->Ws;
  a.cap = c->desc.capacity;
  a.n_cur = n_cur;
  a.n_tok = n_tokens;
  const duo_status st = cuda_status(duo::launch_append(a, c->desc.kv_dtype, (cudaStream_t)stream));
  if (st == DUO_OK) c->seq_len[layer] = n_cur + n_tokens;
  return st;
}

namespace {

// Everything a decode launch needs except the scratch pointers, for a layer
// holding n tokens (the query at position n-1).
duo_status plan_decode(duo_cache *c, int32_t layer, int64_t n, const void *q, void *out, float scale,
                       duo::DecodeParams *p) {
  const auto &L = c->layers[layer];
  const duo_cache_desc &d = c->desc;
  duo::DecodeConfig cfg{};
  cudaError_t e = cached_decode_config(c, &cfg);
  if (e == cudaErrorInvalidValue || e == cudaErrorNotSupported) return DUO_ERR_UNSUPPORTED;
  if (e != cudaSuccess) return DUO_ERR_CUDA;
  const int want = choose_splits(c, layer, n, cfg);
  const int64_t split_len = round_up((n + want - 1) / want, cfg.tile_rows);
  *p = duo::DecodeParams{};
  p->q = q;
  p->out = out;
  p->p = layer_ptrs(c, layer);
  p->h = L.h;
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
  p->n = n;
  p->nsplit = (int)((n + split_len - 1) / split_len);
  p->split_len = split_len;
  const float sc = scale > 0.f ? scale : 1.0f / std::sqrt((float)d.head_dim);
  p->scale_log2 = sc * 1.4426950408889634f;
  p->err = duo::device_error_word();
  p->pool = c->reproducible ? 0 : 1;
  return DUO_OK;
}

// Point the decode at the caller's workspace (layout of ws_layout).
duo_status use_workspace(const duo_cache *c, const duo::DecodeParams &p, void *ws, size_t ws_bytes,
                         duo::DecodeParams *out) {
  *out = p;
  if (p.n_ret == 0 || p.nsplit == 1) return DUO_OK;
  const WsLayout w = ws_layout(c->desc, c->n_ret_max);
  if (!ws || ws_bytes < (size_t)w.total) return DUO_ERR_WORKSPACE;
  if ((reinterpret_cast<uintptr_t>(ws) % kAlign) != 0) return DUO_ERR_ARG;
  uint8_t *wsb = static_cast<uint8_t *>(ws);
  out->ws_cnt = reinterpret_cast<unsigned *>(wsb + w.cnt);
  out->ws_next = reinterpret_cast<unsigned *>(wsb + w.next);
  out->ws_lse = reinterpret_cast<float *>(wsb + w.lse);
  out->ws_o = reinterpret_cast<float *>(wsb + w.o);
  return DUO_OK;
}

duo_status launch_status(cudaError_t e) {
  if (e == cudaErrorInvalidValue || e == cudaErrorNotSupported) return DUO_ERR_UNSUPPORTED;
  return cuda_status(e);
}

duo_status check_decode_args(const duo_cache *c, int32_t layer, const void *q, void *out, float scale) {
  if (!c || !q || !out) return DUO_ERR_ARG;
  if (layer < 0 || layer >= c->desc.layers) return DUO_ERR_ARG;
  if (!c->base) return DUO_ERR_STATE;
  if (!std::isfinite(scale)) return DUO_ERR_ARG;
  return DUO_OK;
}

}  // namespace

duo_status duo_decode_attn(duo_cache *c, int32_t layer, const void *q, void *out, float scale,
                           void *ws, size_t ws_bytes, duo_stream stream) {
  duo_status st = check_decode_args(c, layer, q, out, scale);
  if (st != DUO_OK) return st;
  const int64_t n = c->seq_len[layer];
  if (n <= 0) return DUO_ERR_STATE;
  duo::DecodeParams plan, p;
  if ((st = plan_decode(c, layer, n, q, out, scale, &plan)) != DUO_OK) return st;
  if ((st = use_workspace(c, plan, ws, ws_bytes, &p)) != DUO_OK) return st;
  return launch_status(duo::launch_decode(p, c->desc.kv_dtype, (cudaStream_t)stream));
}

duo_status duo_decode_step(duo_cache *c, int32_t layer, const void *q, const void *k_new,
                           const void *v_new, void *out, float scale, void *ws, size_t ws_bytes,
                           duo_stream stream) {
  duo_status st = check_decode_args(c, layer, q, out, scale);
  if (st != DUO_OK) return st;
  if (!k_new || !v_new || !aligned16(k_new) || !aligned16(v_new)) return DUO_ERR_ARG;
  const duo_cache_desc &d = c->desc;
  const int64_t n_cur = c->seq_len[layer];
  if (c->layers[layer].n_ret > 0 && n_cur + 1 > d.capacity) return DUO_ERR_CAPACITY;
  if (!duo::decode_can_fuse_append(d.kv_dtype, d.head_dim, d.n_q_heads / d.n_kv_heads)) {
    // no fused kernel for this configuration: append, then attend
    if ((st = duo_append_kv(c, layer, k_new, v_new, 1, stream)) != DUO_OK) return st;
    return duo_decode_attn(c, layer, q, out, scale, ws, ws_bytes, stream);
  }
  const int64_t n = n_cur + 1;
  duo::DecodeParams plan, p;
  if ((st = plan_decode(c, layer, n, q, out, scale, &plan)) != DUO_OK) return st;
  if ((st = use_workspace(c, plan, ws, ws_bytes, &p)) != DUO_OK) return st;
  p.knew = k_new;
  p.vnew = v_new;
  p.new_slot = n_cur < c->S ? n_cur : c->S + (n_cur - c->S) % c->R;
  p.pdl = 1;
  st = launch_status(duo::launch_decode(p, d.kv_dtype, (cudaStream_t)stream));
  if (st == DUO_OK) c->seq_len[layer] = n;
  return st;
}

duo_status duo_decode_attn_static(duo_cache *c, int32_t layer, const void *q, void *out,
                                  float scale, duo_stream stream) {
  duo_status st = check_decode_args(c, layer, q, out, scale);
  if (st != DUO_OK) return st;
  const int64_t n = c->seq_len[layer];
  if (n <= 0) return DUO_ERR_STATE;
  const auto &L = c->layers[layer];
  const duo_cache_desc &d = c->desc;
  duo::DecodeParams p;
  if ((st = plan_decode(c, layer, n, q, out, scale, &p)) != DUO_OK) return st;
  const int G = p.G, nsplit = p.nsplit;
  // Compact scratch layout for exactly this launch: tickets, chunk counters,
  // lse, partial O.
  const int64_t units = (int64_t)d.batch * L.n_ret;
  const int64_t off_next = round_up(units * 4, kAlign);
  const int64_t off_lse = off_next + round_up(units * duo::kChunkCounterStride * 4, kAlign);
  const int64_t off_o = off_lse + round_up(units * nsplit * G * 4, kAlign);
  const int64_t need = off_o + units * nsplit * G * (int64_t)d.head_dim * 4;
  const bool need_ws = L.n_ret > 0 && nsplit > 1;
  if (need_ws && need > (int64_t)duo::decode_static_scratch_bytes()) return DUO_ERR_WORKSPACE;
  if (need_ws) {
    void *ptr = nullptr;
    if (duo::decode_static_scratch(&ptr) != cudaSuccess) return DUO_ERR_CUDA;
    uint8_t *scratch = static_cast<uint8_t *>(ptr);
    // tickets and counters start at zero for this launch (the array keeps
    // earlier calls' bytes)
    if (cudaMemsetAsync(scratch, 0, (size_t)off_lse, (cudaStream_t)stream) != cudaSuccess)
      return DUO_ERR_CUDA;
    p.ws_cnt = reinterpret_cast<unsigned *>(scratch);
    p.ws_next = reinterpret_cast<unsigned *>(scratch + off_next);
    p.ws_lse = reinterpret_cast<float *>(scratch + off_lse);
    p.ws_o = reinterpret_cast<float *>(scratch + off_o);
  }
  return launch_status(duo::launch_decode(p, d.kv_dtype, (cudaStream_t)stream));
}

duo_status duo_prefill_attn(duo_cache *c, int32_t layer, const void *q, const void *k,
                            const void *v, int32_t C, void *out, float scale, void *ws,
                            size_t ws_bytes, duo_stream stream) {
  (void)ws;
  (void)ws_bytes;
  if (!c || !q || !k || !v || !out || C <= 0) return DUO_ERR_ARG;
  if (layer < 0 || layer >= c->desc.layers) return DUO_ERR_ARG;
  if (!c->base) return DUO_ERR_STATE;
  if (!std::isfinite(scale)) return DUO_ERR_ARG;
  const duo_cache_desc &d = c->desc;
  if (d.kv_dtype != DUO_BF16 || d.head_dim != 128) return DUO_ERR_UNSUPPORTED;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)) return DUO_ERR_ARG;
  const auto &L = c->layers[layer];
  const int64_t c0 = c->seq_len[layer];
  if (L.n_ret > 0 && c0 + C > d.capacity) return DUO_ERR_CAPACITY;
  duo::PrefillParams p{};
  p.q = q;
  p.k = k;
  p.v = v;
  p.out = out;
  p.p = layer_ptrs(c, layer);
  p.h = L.h;
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
  p.cap = d.capacity;
  p.c0 = c0;
  const float sc = scale > 0.f ? scale : 1.0f / std::sqrt((float)d.head_dim);
  p.scale_log2 = sc * 1.4426950408889634f;
  p.err = duo::device_error_word();
  cudaError_t e = duo::launch_prefill(p, (cudaStream_t)stream);
  if (e == cudaErrorInvalidValue || e == cudaErrorNotSupported) return DUO_ERR_UNSUPPORTED;
  return cuda_status(e);
}

duo_status duo_seq_len(const duo_cache *c, int32_t layer, int64_t *n) {
  if (!c || !n || layer < 0 || layer >= c->desc.layers) return DUO_ERR_ARG;
  *n = c->seq_len[layer];
  return DUO_OK;
}

duo_status duo_kv_bytes(const duo_cache *c, int64_t *kept, int64_t *full) {
  if (!c) return DUO_ERR_ARG;
  const duo_cache_desc &d = c->desc;
  const int64_t per = d.kv_dtype == DUO_INT4 ? 2 * (d.head_dim / 2 + 4)
                                             : 2 * (int64_t)d.head_dim * elem_bytes(d.kv_dtype);
  int64_t k = 0, f = 0;
  for (int l = 0; l < d.layers; ++l) {
    const int64_t n = c->seq_len[l];
    const int64_t win = n < c->W ? n : c->W;
    k += (int64_t)d.batch * (c->layers[l].n_ret * n + c->layers[l].n_str * win) * per;
    f += (int64_t)d.batch * d.n_kv_heads * n * per;
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
  o->seq_len = c->seq_len[layer];
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
  return DUO_OK;
}

duo_status duo_set_decode_splits(duo_cache *c, int32_t splits) {
  if (!c || splits < 0 || splits > DUO_MAX_SPLITS) return DUO_ERR_ARG;
  c->forced_splits = splits;
  return DUO_OK;
}

duo_status duo_set_decode_reproducible(duo_cache *c, int32_t on) {
  if (!c || (on != 0 && on != 1)) return DUO_ERR_ARG;
  c->reproducible = on == 1;
  return DUO_OK;
}

duo_status duo_decode_splits(const duo_cache *c, int32_t layer, int32_t *splits) {
  if (!c || !splits || layer < 0 || layer >= c->desc.layers) return DUO_ERR_ARG;
  duo::DecodeConfig cfg{};
  cudaError_t e = cached_decode_config(const_cast<duo_cache *>(c), &cfg);
  if (e != cudaSuccess) return e == cudaErrorInvalidValue ? DUO_ERR_UNSUPPORTED : DUO_ERR_CUDA;
  const int64_t n = c->seq_len[layer] > 0 ? c->seq_len[layer] : 1;
  const int want = choose_splits(c, layer, n, cfg);
  int64_t split_len = round_up((n + want - 1) / want, cfg.tile_rows);
  *splits = (int32_t)((n + split_len - 1) / split_len);
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
