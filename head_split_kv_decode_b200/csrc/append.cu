// Cache append/evict: write the K/V of new tokens into the two layouts.
//
// Retrieval KV heads keep every token (full KV cache); streaming KV heads keep
// S sink slots and an R-slot ring of the most recent tokens, so writing a
// token into its ring slot evicts the token R positions older.  Pages:
// "What is DuoAttention" (nav.superapi.store), section "Technical principles of
// DuoAttention"; "DuoAttention: Efficient Long-Context LLM Inference with
// Retrieval and Streaming Heads" (hotpaper.ai), section "기술적 접근법".
//
// For a chunk of n_tok tokens a streaming head writes only the positions that
// survive the chunk: p < S (sinks) and the last R positions.  Those land in
// distinct slots, so the result equals appending token by token.
#include "common.cuh"
#include "quant_int4.cuh"

namespace duo {

// One thread per 16-byte chunk of one (token, KV head) row of K and of V.
__global__ void append_kernel(const __grid_constant__ AppendParams a, int row_bytes) {
  const int ch = row_bytes / 16;
  const int64_t total = (int64_t)a.rows.n * a.n_tok * a.Hkv * ch;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int c = (int)(i % ch);
    int64_t r = i / ch;
    const int h = (int)(r % a.Hkv);
    r /= a.Hkv;
    const int64_t t = r % a.n_tok;
    const int lr = (int)(r / a.n_tok);  // launch row
    const int b = a.rows.row[lr];
    const int64_t p = a.rows.len[lr] + t;
    const int64_t end = a.rows.len[lr] + a.n_tok;
    const int idx = a.h.index[h];
    int64_t off;
    uint8_t *dk, *dv;
    if (a.h.kind[h]) {
      if (p < a.shard_lo || p >= a.shard_hi) continue;  // another shard's position
      off = ret_row(a.ret, b, idx, p - a.shard_lo) * row_bytes;
      dk = a.p.ret_k;
      dv = a.p.ret_v;
    } else {
      if (!(p < a.S || p >= end - a.R)) continue;
      off = (((int64_t)b * a.n_str + idx) * a.Ws + ring_slot(p, a.S, a.R)) * row_bytes;
      dk = a.p.str_k;
      dv = a.p.str_v;
    }
    // The input is [rows][n_tok][Hkv][row], so chunk i of the input is chunk i.
    const uint4 kk = __ldg(reinterpret_cast<const uint4 *>(a.k) + i);
    const uint4 vv = __ldg(reinterpret_cast<const uint4 *>(a.v) + i);
    reinterpret_cast<uint4 *>(dk + off)[c] = kk;
    reinterpret_cast<uint4 *>(dv + off)[c] = vv;
  }
}

// INT4: one warp per (token, KV head, K or V) row of D bf16 channels.  Lane l
// owns channels [l*CPL, l*CPL + CPL); quantize_row_int4 performs the encoder's
// correctly rounded fp32 operations.
template <int D>
__global__ void append_int4_kernel(const __grid_constant__ AppendParams a) {
  constexpr int CPL = D / 32;
  static_assert(CPL == 2 || CPL == 4, "head_dim 64 or 128");
  const int lane = threadIdx.x & 31;
  const int64_t warps = (int64_t)a.rows.n * a.n_tok * a.Hkv * 2;
  const int64_t gw = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 5;
  const int64_t nw = ((int64_t)gridDim.x * blockDim.x) >> 5;
  for (int64_t w = gw; w < warps; w += nw) {
    const int which = (int)(w & 1);  // 0 = K, 1 = V
    int64_t r = w >> 1;
    const int h = (int)(r % a.Hkv);
    r /= a.Hkv;
    const int64_t t = r % a.n_tok;
    const int lr = (int)(r / a.n_tok);  // launch row
    const int b = a.rows.row[lr];
    const int64_t p = a.rows.len[lr] + t;
    const int64_t end = a.rows.len[lr] + a.n_tok;
    const int idx = a.h.index[h];
    int64_t row;
    uint8_t *codes, *sz;
    if (a.h.kind[h]) {
      if (p < a.shard_lo || p >= a.shard_hi) continue;  // another shard's position
      row = ret_row(a.ret, b, idx, p - a.shard_lo);
      codes = which ? a.p.ret_v : a.p.ret_k;
      sz = which ? a.p.ret_v_sz : a.p.ret_k_sz;
    } else {
      if (!(p < a.S || p >= end - a.R)) continue;
      row = ((int64_t)b * a.n_str + idx) * a.Ws + ring_slot(p, a.S, a.R);
      codes = which ? a.p.str_v : a.p.str_k;
      sz = which ? a.p.str_v_sz : a.p.str_k_sz;
    }
    const __nv_bfloat16 *src = reinterpret_cast<const __nv_bfloat16 *>(which ? a.v : a.k) +
                               (((int64_t)lr * a.n_tok + t) * a.Hkv + h) * D + lane * CPL;
    float x[CPL];
#pragma unroll
    for (int j = 0; j < CPL; ++j) x[j] = __bfloat162float(src[j]);
    __half sch, zph;
    const uint32_t packed = quantize_row_int4<CPL>(x, &sch, &zph);
    uint8_t *dst = codes + row * (D / 2) + lane * (CPL / 2);
    if (CPL == 4)
      *reinterpret_cast<uint16_t *>(dst) = (uint16_t)packed;
    else
      *dst = (uint8_t)packed;
    if (lane == 0) {
      __half2 pair;
      pair.x = sch;
      pair.y = zph;
      reinterpret_cast<__half2 *>(sz)[row] = pair;
    }
  }
}

// Block-table writes of the paged layout: one thread per entry.
__global__ void table_write_kernel(int32_t *table, const __grid_constant__ TableWrites w) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < w.n) table[w.index[i]] = w.block[i];
}

cudaError_t launch_table_writes(int32_t *table, const TableWrites &w, cudaStream_t s) {
  if (w.n <= 0) return cudaSuccess;
  table_write_kernel<<<1, kMaxTableWrites, 0, s>>>(table, w);
  return cudaGetLastError();
}

cudaError_t launch_append(const AppendParams &a, int kv_type, cudaStream_t s) {
  if (a.n_tok <= 0 || a.rows.n <= 0) return cudaSuccess;
  if (kv_type == kINT4) {
    const int64_t warps = (int64_t)a.rows.n * a.n_tok * a.Hkv * 2;
    const int threads = 256;
    const int64_t blocks = (warps * 32 + threads - 1) / threads;
    const int grid = (int)(blocks < 148 * 64 ? blocks : 148 * 64);
    if (a.D == 128)
      append_int4_kernel<128><<<grid, threads, 0, s>>>(a);
    else
      append_int4_kernel<64><<<grid, threads, 0, s>>>(a);
    return cudaGetLastError();
  }
  const int row_bytes = a.D * (kv_type == kF32 ? 4 : 2);
  const int64_t total = (int64_t)a.rows.n * a.n_tok * a.Hkv * (row_bytes / 16);
  const int threads = 256;
  const int64_t blocks = (total + threads - 1) / threads;
  const int grid = (int)(blocks < 148 * 32 ? blocks : 148 * 32);
  append_kernel<<<grid, threads, 0, s>>>(a, row_bytes);
  return cudaGetLastError();
}

}  // namespace duo
