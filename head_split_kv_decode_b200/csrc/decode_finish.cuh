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
// writes the output (single split) or this split's normalised partial and
// log-sum-exp, and lets the last split of the head merge every partial.
template <typename T, int D, int G, int NWARPS>
__device__ __forceinline__ void decode_reduce_store(const DecodeParams &P, uint8_t *smem,
                                                    int *s_last_p, bool retrieval, int b, int kvh,
                                                    int pidx, int split) {
  constexpr int NT = NWARPS * 32;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  int &s_last = *s_last_p;
  const float *red_m = reinterpret_cast<const float *>(smem);
  const float *red_l = red_m + NWARPS * G;
  const float *red_o = red_l + NWARPS * G;
  const bool direct = !retrieval || P.nsplit == 1;
  T *out = reinterpret_cast<T *>(P.out) + ((int64_t)b * P.Hq + (int64_t)kvh * G) * D;
  const int64_t part = ((int64_t)b * P.n_ret + (retrieval ? pidx : 0)) * P.nsplit + split;
  for (int idx = tid; idx < G * D; idx += NT) {
    const int g = idx / D, c = idx % D;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < NWARPS; ++w) M = fmaxf(M, red_m[w * G + g]);
    float L = 0.f, O = 0.f;
#pragma unroll
    for (int w = 0; w < NWARPS; ++w) {
      const float mw = red_m[w * G + g];
      const float sw = (mw == -INFINITY) ? 0.f : fast_exp2(mw - M);
      L += red_l[w * G + g] * sw;
      O += red_o[(w * G + g) * D + c] * sw;
    }
    if (direct) {
      store_out(out + g * D + c, O / L);
    } else {
      P.ws_o[(part * G + g) * D + c] = O / L;
      if (c == 0) P.ws_lse[part * G + g] = M + fast_log2(L);
    }
  }
  if (direct) return;

  // ---- the last split of this head to finish merges all splits
  __threadfence();
  __syncthreads();
  unsigned *cnt = P.ws_cnt + (int64_t)b * P.n_ret + pidx;
  if (tid == 0) s_last = (atomicAdd(cnt, 1u) == (unsigned)(P.nsplit - 1));
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  const int64_t part0 = ((int64_t)b * P.n_ret + pidx) * P.nsplit;
  // weights w_s = 2^(lse_s - max) per (split, query head)
  float *s_w = reinterpret_cast<float *>(smem);     // [nsplit][G]
  float *s_den = s_w + P.nsplit * G;                // [G]
  float *s_acc = s_w + ((P.nsplit * G + G + 3) & ~3);  // [NWARPS][G][D], 16-byte aligned
  for (int i = tid; i < P.nsplit * G; i += NT) s_w[i] = __ldcg(P.ws_lse + part0 * G + i);
  __syncthreads();
  if (tid < G) {
    float M = -INFINITY;
    for (int sp = 0; sp < P.nsplit; ++sp) M = fmaxf(M, s_w[sp * G + tid]);
    float den = 0.f;
    for (int sp = 0; sp < P.nsplit; ++sp) {
      const float w = fast_exp2(s_w[sp * G + tid] - M);
      s_w[sp * G + tid] = w;
      den += w;
    }
    s_den[tid] = den;
  }
  __syncthreads();
  // warp w sums splits w, w+NWARPS, ...; lane l owns channels [4l, 4l+4) of
  // every query head (D/4 float4 per head row, so lanes cover D = 128; for
  // D = 64 the upper lanes idle).  Four splits' loads are kept in flight.
  constexpr int L4 = D / 4;
  float4 acc[G];
#pragma unroll
  for (int g = 0; g < G; ++g) acc[g] = make_float4(0.f, 0.f, 0.f, 0.f);
  if (lane < L4) {
    const float4 *src = reinterpret_cast<const float4 *>(P.ws_o + part0 * G * D) + lane;
    int sp = warp;
    for (; sp + 3 * NWARPS < P.nsplit; sp += 4 * NWARPS) {
      float4 v[4][G];
#pragma unroll
      for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int g = 0; g < G; ++g) v[u][g] = __ldcg(src + ((sp + u * NWARPS) * G + g) * L4);
#pragma unroll
      for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int g = 0; g < G; ++g) {
          const float w = s_w[(sp + u * NWARPS) * G + g];
          acc[g].x += w * v[u][g].x;
          acc[g].y += w * v[u][g].y;
          acc[g].z += w * v[u][g].z;
          acc[g].w += w * v[u][g].w;
        }
    }
    for (; sp < P.nsplit; sp += NWARPS)
#pragma unroll
      for (int g = 0; g < G; ++g) {
        const float4 v = __ldcg(src + (sp * G + g) * L4);
        const float w = s_w[sp * G + g];
        acc[g].x += w * v.x;
        acc[g].y += w * v.y;
        acc[g].z += w * v.z;
        acc[g].w += w * v.w;
      }
#pragma unroll
    for (int g = 0; g < G; ++g)
      reinterpret_cast<float4 *>(s_acc + (warp * G + g) * D)[lane] = acc[g];
  }
  __syncthreads();
  for (int idx = tid; idx < G * D; idx += NT) {
    const int g = idx / D, c = idx % D;
    float num = 0.f;
#pragma unroll
    for (int w = 0; w < NWARPS; ++w) num += s_acc[(w * G + g) * D + c];
    store_out(out + g * D + c, num / s_den[g]);
  }
  if (tid == 0) *cnt = 0u;  // leave the ticket ready for the next call
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

  decode_reduce_store<T, D, G, NWARPS>(P, smem, s_last_p, retrieval, b, kvh, pidx, split);
}

}  // namespace duo
