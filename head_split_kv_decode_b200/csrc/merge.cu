// Merge of decode partials from several sequence shards.
//
// Each shard (a GPU holding a contiguous range of a long sequence's retrieval
// positions) leaves, per (row, query head), its normalised output o_i and the
// log-sum-exp lse_i of its scores.  The attention over the union of the keys
// is the log-sum-exp weighted mean: with L = log sum_i exp(lse_i),
// out = sum_i exp(lse_i - L) o_i.  A shard that saw no key has lse = -inf
// and weight 0.  This is the same merge the split-K decode does across the
// splits of one GPU, here across shards after the partials are gathered.
#include "common.cuh"

namespace duo {

namespace {

// One warp per (row, query head); lane l owns channels [4l, 4l+4) (D <= 128).
template <typename T>
__global__ void merge_partials_kernel(int n_parts, int64_t rows, int D, const float *o,
                                      const float *lse, T *out) {
  const int64_t row = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  float M = -INFINITY;
  for (int i = 0; i < n_parts; ++i) M = fmaxf(M, lse[(int64_t)i * rows + row]);
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  float den = 0.f;
  const bool owns = 4 * lane < D;
  for (int i = 0; i < n_parts; ++i) {
    const float x = lse[(int64_t)i * rows + row];
    const float w = (x == -INFINITY) ? 0.f : __expf(x - M);
    den += w;
    if (owns && w != 0.f) {
      const float4 v = *reinterpret_cast<const float4 *>(o + ((int64_t)i * rows + row) * D + 4 * lane);
      acc.x += w * v.x;
      acc.y += w * v.y;
      acc.z += w * v.z;
      acc.w += w * v.w;
    }
  }
  if (!owns) return;
  const float inv = den > 0.f ? 1.f / den : 0.f;  // no shard saw a key: zeros
  T *dst = out + row * D + 4 * lane;
  store_out(dst + 0, acc.x * inv);
  store_out(dst + 1, acc.y * inv);
  store_out(dst + 2, acc.z * inv);
  store_out(dst + 3, acc.w * inv);
}

}  // namespace

cudaError_t launch_merge_partials(int n_parts, int64_t rows, int D, const float *o,
                                  const float *lse, void *out, int out_type, cudaStream_t s) {
  if (n_parts <= 0 || rows <= 0 || D % 4 || D > 128) return cudaErrorInvalidValue;
  const int warps = 8;
  const int64_t grid = (rows + warps - 1) / warps;
  if (out_type == kF32)
    merge_partials_kernel<float><<<(unsigned)grid, warps * 32, 0, s>>>(n_parts, rows, D, o, lse,
                                                                       static_cast<float *>(out));
  else
    merge_partials_kernel<__nv_bfloat16><<<(unsigned)grid, warps * 32, 0, s>>>(
        n_parts, rows, D, o, lse, static_cast<__nv_bfloat16 *>(out));
  return cudaGetLastError();
}

}  // namespace duo
