// History of a 4-bit cache as bf16 rows, for the chunked pre-fill.
//
// The pre-fill's tensor-core products take bf16 operands, so before a chunk
// attends to a 4-bit cache, the part of the cache it reads (each launch row's
// retrieval keys below its length, and the filled slots of its streaming
// heads) is expanded into a bf16 scratch laid out like a bf16 cache: retrieval
// rows at the same storage rows as the codes (packed or paged), streaming
// rows [batch][n_streaming][S + R][d].  The pre-fill then reads the scratch
// exactly as it reads a bf16 cache.  Its key tiles are 128 rows, so it also
// reads the rows past a row's length up to the end of that tile, and the
// unfilled slots of a streaming buffer; their probabilities are 0, and the
// expansion writes zeros there so that 0 * value stays 0 whatever the scratch
// held before.  (The packed layout of a 4-bit cache gives each retrieval head
// a whole number of 128-row tiles, and a paged block holds two, so those rows
// belong to the same head and row.)  Each value is x = sc * u + zp of its
// (token, head) group, in fp32, rounded to bf16.  Pages: "DuoAttention:
// Efficient Long-Context LLM Inference with Retrieval and Streaming Heads"
// (hotpaper.ai), section "기술적 접근법" (the method combines with a 4-bit KV
// cache).
#include "common.cuh"

namespace duo {

namespace {

// One thread per 8 channels (4 bytes of codes -> 16 bytes of bf16) of one
// (token, head) row of K or V; blockIdx.y = (launch row, head, K or V).
__global__ void dequant_history_kernel(const __grid_constant__ DequantParams d) {
  const int heads = d.n_ret + d.n_str;
  const int y = blockIdx.y;
  const int which = y & 1;  // 0 = K, 1 = V
  const int hh = (y >> 1) % heads;
  const int r = (y >> 1) / heads;
  const int b = d.rows.row[r];
  const int n = d.rows.len[r];
  const bool ret = hh < d.n_ret;
  const int pidx = ret ? hh : hh - d.n_ret;
  const int keys = ret ? n : min(n, d.W);
  // rows written: the keys, then zeros up to the end of the last 128-row
  // tile (retrieval) or of the slot buffer (streaming)
  const int rows = ret ? (n + 127) / 128 * 128 : (keys > 0 ? d.W : 0);
  constexpr int CH = 8;               // channels per thread
  const int per_row = d.D / CH;       // threads per key row
  const int64_t total = (int64_t)rows * per_row;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int key = (int)(i / per_row);
    const int c = (int)(i % per_row) * CH;
    int64_t src_row, dst_row;
    const uint8_t *codes, *sz;
    __nv_bfloat16 *dst;
    if (ret) {
      src_row = dst_row = ret_row(d.ret, b, pidx, key);
      codes = which ? d.p.ret_v : d.p.ret_k;
      sz = which ? d.p.ret_v_sz : d.p.ret_k_sz;
      dst = which ? d.ret_v : d.ret_k;
    } else {
      // slot `key` of the ring buffer (every filled slot is read)
      src_row = ((int64_t)b * d.n_str + pidx) * d.Ws + key;
      dst_row = ((int64_t)b * d.n_str + pidx) * d.W + key;
      codes = which ? d.p.str_v : d.p.str_k;
      sz = which ? d.p.str_v_sz : d.p.str_k_sz;
      dst = which ? d.str_v : d.str_k;
    }
    if (key >= keys) {  // past the row's length: zeros
      *reinterpret_cast<uint4 *>(dst + dst_row * d.D + c) = make_uint4(0, 0, 0, 0);
      continue;
    }
    const uint32_t w = *reinterpret_cast<const uint32_t *>(codes + src_row * (d.D / 2) + c / 2);
    const __half2 p = *reinterpret_cast<const __half2 *>(sz + src_row * 4);
    const float scale = __low2float(p), zero = __high2float(p);
    uint32_t out[CH / 2];
#pragma unroll
    for (int j = 0; j < CH / 2; ++j) {  // low nibble = even channel
      const float lo = __fmaf_rn(scale, (float)((w >> (8 * j)) & 0xF), zero);
      const float hi = __fmaf_rn(scale, (float)((w >> (8 * j + 4)) & 0xF), zero);
      const __nv_bfloat162 h2 = __floats2bfloat162_rn(lo, hi);
      out[j] = *reinterpret_cast<const uint32_t *>(&h2);
    }
    *reinterpret_cast<uint4 *>(dst + dst_row * d.D + c) = make_uint4(out[0], out[1], out[2], out[3]);
  }
}

}  // namespace

cudaError_t launch_dequant_history(const DequantParams &d, cudaStream_t s) {
  if (d.rows.n <= 0 || d.D % 8) return d.D % 8 ? cudaErrorInvalidValue : cudaSuccess;
  int max_rows = 0;  // rows one (launch row, head) writes at most
  for (int r = 0; r < d.rows.n; ++r)
    max_rows = max(max_rows, max((d.rows.len[r] + 127) / 128 * 128, d.rows.len[r] > 0 ? d.W : 0));
  if (max_rows == 0) return cudaSuccess;
  const int threads = 256;
  const int64_t need = ((int64_t)max_rows * (d.D / 8) + threads - 1) / threads;
  dim3 grid((unsigned)(need < 1024 ? need : 1024), (unsigned)(d.rows.n * (d.n_ret + d.n_str) * 2));
  dequant_history_kernel<<<grid, threads, 0, s>>>(d);
  return cudaGetLastError();
}

}  // namespace duo
