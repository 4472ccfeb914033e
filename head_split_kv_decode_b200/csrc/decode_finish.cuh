// Epilogue shared by the decode kernels: combine the per-lane-group online
// softmax states of a CTA, write the output (single split) or a normalised
// partial plus its log-sum-exp (split-K), and let the last split of each head
// merge all partials.  The last CTA is found with an atomic ticket, so no CTA
// ever waits for another.
#pragma once

#include "common.cuh"

namespace duo {

// Second half of the epilogue: the per-warp states of the CTA are staged in
// shared memory as red_m [NWARPS][G], red_l [NWARPS][G] (log2 units) and
// red_o [NWARPS][G][D] (unnormalised), all starting at `smem`.  Combines them,
// writes the result of this KV head's G query heads (rows out_row ..
// out_row + G - 1 of the output, or of P.part_o / P.part_lse in partial mode)
// when `direct`, or else this split's normalised partial and log-sum-exp
// into slot part0 + split, and lets the last of the nsplit splits of the head
// (merge ticket `unit`) merge slots part0 .. part0 + nsplit - 1.
template <typename T, int D, int G, int NWARPS>
__device__ __forceinline__ void decode_reduce_store(const DecodeParams &P, uint8_t *smem,
                                                    int *s_last_p, bool direct, int64_t out_row,
                                                    int64_t unit, int64_t part0, int nsplit,
                                                    int split) {
  constexpr float kLn2 = 0.6931471805599453f;  // log-sum-exps leave in natural log
  // output element i of this head's rows, as T or (P.out_f32) as float
  auto put = [&](int i, float v) {
    if (P.out_f32) reinterpret_cast<float *>(P.out)[out_row * D + i] = v;
    else store_out(reinterpret_cast<T *>(P.out) + out_row * D + i, v);
  };
  constexpr int NT = NWARPS * 32;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  int &s_last = *s_last_p;
  const float *red_m = reinterpret_cast<const float *>(smem);
  const float *red_l = red_m + NWARPS * G;
  const float *red_o = red_l + NWARPS * G;
  const int64_t part = part0 + split;
  // One output element per thread and step; D is a multiple of 32, so the
  // query head g is the same across a warp and lane w < NWARPS can hold warp
  // w's weight 2^(m_w - M) for all lanes to fetch.
  static_assert(D % 32 == 0 && NWARPS <= 32, "warp-uniform query head");
  for (int idx = tid; idx < G * D; idx += NT) {
    const int g = idx / D, c = idx % D;
    const float mw = lane < NWARPS ? red_m[lane * G + g] : -INFINITY;
    float M = mw;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
    const float sw = (mw == -INFINITY) ? 0.f : fast_exp2(mw - M);
    float L = lane < NWARPS ? red_l[lane * G + g] * sw : 0.f;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) L += __shfl_xor_sync(0xffffffffu, L, off);
    float O = 0.f;
#pragma unroll
    for (int w = 0; w < NWARPS; ++w) O += red_o[(w * G + g) * D + c] * __shfl_sync(0xffffffffu, sw, w);
    if (direct && P.part_o) {
      const bool empty = L == 0.f;  // this shard holds no key of the head
      P.part_o[(out_row + g) * D + c] = empty ? 0.f : O / L;
      if (c == 0) P.part_lse[out_row + g] = empty ? -INFINITY : (M + fast_log2(L)) * kLn2;
    } else if (direct) {
      put(g * D + c, O / L);
    } else {
      // a split whose CTA claimed no keys leaves weight zero (lse -inf)
      const bool empty = L == 0.f;
      P.ws_o[(part * G + g) * D + c] = empty ? 0.f : O / L;
      if (c == 0) P.ws_lse[part * G + g] = empty ? -INFINITY : M + fast_log2(L);
    }
  }
  if (direct) return;

  // ---- the last split of this head to finish merges all splits.  The
  // barrier orders the CTA's partial stores before thread 0's ticket, an
  // atomic with release and acquire semantics at GPU scope: the release
  // (cumulative over what the barrier ordered before it) publishes the
  // partials with the ticket, and the acquire by the CTA that draws the last
  // ticket, followed by the barrier below, orders its threads' reads of the
  // other splits' partials after their release.  (One atomic in place of a
  // fence, the atomic and a second fence.)
  __syncthreads();
  unsigned *cnt = P.ws_cnt + unit;
  if (tid == 0) {
    unsigned prev;
    asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], 1;" : "=r"(prev) : "l"(cnt) : "memory");
    s_last = (prev == (unsigned)(nsplit - 1));
  }
  __syncthreads();
  if (!s_last) return;
  // Each warp produces 32 output channels of one query head (one per lane)
  // from all splits: the lanes load every split's partial at their channel
  // and the splits' log-sum-exps in one burst, so the merge costs one round
  // trip to L2, with the weights 2^(lse_s - max) formed by shuffles (no
  // shared memory, no barrier).  Splits are taken kHeld at a time, the
  // running sum rescaled to each chunk's maximum (one chunk up to kHeld).
  constexpr int SL = D / 32;     // 32-channel slices of a query head
  constexpr int kHeld = 64;      // partials a lane holds at once
  for (int sl = warp; sl < G * SL; sl += NWARPS) {
    const int g = sl / SL, c = (sl % SL) * 32 + lane;
    const float *po = P.ws_o + (part0 * G + g) * D + c;  // split s at po[s * G * D]
    const float *pl = P.ws_lse + part0 * G + g;          // split s at pl[s * G]
    float M = -INFINITY, den = 0.f, acc = 0.f;
    for (int s0 = 0; s0 < nsplit; s0 += kHeld) {
      const int ns = min(nsplit - s0, kHeld);
      float x[kHeld / 32], v[kHeld];
#pragma unroll
      for (int i = 0; i < kHeld / 32; ++i)
        x[i] = 32 * i + lane < ns ? __ldcg(pl + (int64_t)(s0 + 32 * i + lane) * G) : -INFINITY;
#pragma unroll
      for (int i = 0; i < kHeld; ++i) v[i] = i < ns ? __ldcg(po + (int64_t)(s0 + i) * G * D) : 0.f;
      float m = x[0];
#pragma unroll
      for (int i = 1; i < kHeld / 32; ++i) m = fmaxf(m, x[i]);
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
      const float Mn = fmaxf(M, m);
      if (Mn == -INFINITY) continue;  // no split of this chunk (or before) saw a key
      const float a = M == -INFINITY ? 0.f : fast_exp2(M - Mn);
      acc *= a;
      den *= a;
      M = Mn;
      float w[kHeld / 32], d = 0.f;
#pragma unroll
      for (int i = 0; i < kHeld / 32; ++i) {
        w[i] = x[i] == -INFINITY ? 0.f : fast_exp2(x[i] - M);  // a split that claimed no keys: 0
        d += w[i];
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) d += __shfl_xor_sync(0xffffffffu, d, off);
      den += d;
      // four independent chains, and nothing past the chunk's splits
      float a4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int i = 0; i < kHeld; i += 4) {
        if (i < ns) {
#pragma unroll
          for (int k = 0; k < 4; ++k) a4[k] += __shfl_sync(0xffffffffu, w[(i + k) / 32], (i + k) % 32) * v[i + k];
        }
      }
      acc += (a4[0] + a4[1]) + (a4[2] + a4[3]);
    }
    const bool empty = den == 0.f;
    if (P.part_o) {
      P.part_o[(out_row + g) * D + c] = empty ? 0.f : acc / den;
      if (c == 0) P.part_lse[out_row + g] = empty ? -INFINITY : (M + fast_log2(den)) * kLn2;
    } else {
      put(g * D + c, acc / den);
    }
  }
  if (tid == 0) {  // leave the ticket (and chunk counter) ready for the next call
    *cnt = 0u;
    if (P.ws_next) P.ws_next[unit * kChunkCounterStride] = 0u;
  }
}

// Epilogue of a streaming CTA that holds several streaming heads of launch
// row r (heads pidx0, pidx0 + 1, ... of the row), each on a group of wph
// consecutive warps.  The per-warp states are staged as for
// decode_reduce_store; group h combines warps h*wph .. h*wph + wph - 1 and
// writes its G query heads directly (or, in partial mode, their normalised
// rows and log-sum-exps).  Groups past the row's last streaming head write
// nothing.
template <typename T, int D, int G, int NWARPS>
__device__ __forceinline__ void decode_store_groups(const DecodeParams &P, uint8_t *smem, int wph,
                                                    int r, int pidx0) {
  constexpr float kLn2 = 0.6931471805599453f;
  constexpr int NT = NWARPS * 32;
  const int tid = threadIdx.x, lane = tid & 31;
  const float *red_m = reinterpret_cast<const float *>(smem);
  const float *red_l = red_m + NWARPS * G;
  const float *red_o = red_l + NWARPS * G;
  const int groups = min(NWARPS / wph, P.n_str - pidx0);
  // one output element per thread and step; D is a multiple of 32, so the
  // group and query head are the same across a warp, and lane w < wph holds
  // the weight of the group's warp w
  static_assert(D % 32 == 0, "warp-uniform query head");
  for (int idx = tid; idx < groups * G * D; idx += NT) {
    const int h = idx / (G * D), g = (idx / D) % G, c = idx % D;
    const int w0 = h * wph;
    const float mw = lane < wph ? red_m[(w0 + lane) * G + g] : -INFINITY;
    float M = mw;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
    const float sw = (mw == -INFINITY) ? 0.f : fast_exp2(mw - M);
    float L = lane < wph ? red_l[(w0 + lane) * G + g] * sw : 0.f;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) L += __shfl_xor_sync(0xffffffffu, L, off);
    float O = 0.f;
    for (int w = 0; w < wph; ++w) O += red_o[((w0 + w) * G + g) * D + c] * __shfl_sync(0xffffffffu, sw, w);
    const int64_t row = (int64_t)r * P.Hq + (int64_t)P.h.str_heads[pidx0 + h] * G + g;
    if (P.part_o) {
      const bool empty = L == 0.f;
      P.part_o[row * D + c] = empty ? 0.f : O / L;
      if (c == 0) P.part_lse[row] = empty ? -INFINITY : (M + fast_log2(L)) * kLn2;
    } else if (P.out_f32) {
      reinterpret_cast<float *>(P.out)[row * D + c] = O / L;
    } else {
      store_out(reinterpret_cast<T *>(P.out) + row * D + c, O / L);
    }
  }
}

// State layout expected: each 8-lane group of a warp holds m[g], l[g] and NP
// fp32 pairs of the output row of query head g; chan(li, j) gives the channel
// of pair j's first element for lane li of the group.
template <typename T, int D, int G, int NWARPS, int NP, typename ChanFn>
__device__ __forceinline__ void decode_finish(const DecodeParams &P, uint8_t *smem, int *s_last_p,
                                              float (&m)[G], float (&l)[G], float2 (&of)[G][NP],
                                              ChanFn chan, bool retrieval, int b, int kvh, int pidx,
                                              int split) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int grp = lane >> 3, li = lane & 7;
  // ---- combine the four 8-lane groups of each warp
#pragma unroll
  for (int off = 8; off <= 16; off <<= 1)
#pragma unroll
    for (int g = 0; g < G; ++g) {
      const float mo = __shfl_xor_sync(0xffffffffu, m[g], off);
      const float lo = __shfl_xor_sync(0xffffffffu, l[g], off);
      const float mn = fmaxf(m[g], mo);
      const float a = (m[g] == -INFINITY) ? 0.f : fast_exp2(m[g] - mn);
      const float c = (mo == -INFINITY) ? 0.f : fast_exp2(mo - mn);
      l[g] = l[g] * a + lo * c;
#pragma unroll
      for (int j = 0; j < NP; ++j) {
        const float ox = __shfl_xor_sync(0xffffffffu, of[g][j].x, off);
        const float oy = __shfl_xor_sync(0xffffffffu, of[g][j].y, off);
        of[g][j].x = of[g][j].x * a + ox * c;
        of[g][j].y = of[g][j].y * a + oy * c;
      }
      m[g] = mn;
    }

  // ---- combine warps through shared memory (the pipeline stages are idle now)
  float *red_m = reinterpret_cast<float *>(smem);       // [NWARPS][G]
  float *red_l = red_m + NWARPS * G;                    // [NWARPS][G]
  float *red_o = red_l + NWARPS * G;                    // [NWARPS][G][D]
  if (grp == 0) {
#pragma unroll
    for (int g = 0; g < G; ++g) {
      if (li == 0) {
        red_m[warp * G + g] = m[g];
        red_l[warp * G + g] = l[g];
      }
#pragma unroll
      for (int j = 0; j < NP; ++j) {
        const int e = chan(li, j);
        red_o[(warp * G + g) * D + e] = of[g][j].x;
        red_o[(warp * G + g) * D + e + 1] = of[g][j].y;
      }
    }
  }
  __syncthreads();

  // CUDA-core decode: packed layout, every batch row at length P.n, the
  // retrieval CTAs enumerated as ((b*n_ret + head)*nsplit + split).
  const int64_t unit = (int64_t)b * P.n_ret + (retrieval ? pidx : 0);
  decode_reduce_store<T, D, G, NWARPS>(P, smem, s_last_p, !retrieval || P.nsplit == 1,
                                       (int64_t)b * P.Hq + (int64_t)kvh * G, unit,
                                       unit * P.nsplit, P.nsplit, split);
}

}  // namespace duo
