// Single-token decode attention over a 4-bit KV cache.
//
// Same work split and pipeline as the bf16 decode kernel (split-K over the
// retrieval pages, one pass over each streaming slot buffer, last-split merge),
// reading packed 4-bit codes plus one fp16 (scale, zero) pair per token and
// head.  Pages: "DuoAttention: Efficient Long-Context LLM Inference with
// Retrieval and Streaming Heads" (hotpaper.ai), abstract (with quantisation,
// 3.3M-token decoding on one GPU) and section "기술적 접근법" (compatible with
// a 4-bit KV cache).
//
// Dequantisation never materialises k_hat = sc * u + zp.  With q' the scaled
// query, sum_c q'_c k_hat_c = sc * (q' . u) + zp * sum_c q'_c, and for the values
// sum_j p_j v_hat_j = sum_j (p_j sc_j) u_j + (sum_j p_j zp_j) * 1.  So the inner
// loops work on the integer codes u in [0, 15] only:
//  * a lane takes 8 code bytes (16 channels); for each byte, the low nibble is
//    (byte & 0x0F) and the high nibble is kept in place as 16 * u_hi
//    ((byte & 0xF0)); the query's odd channels are pre-divided by 16 (exact);
//  * a byte b becomes the fp32 2^23 + b by placing it under the exponent bits
//    of 2^23 (one byte permute), and 2^23 is then subtracted (exact);
//  * products use packed fp32x2 FMAs.
#include "common.cuh"
#include "decode_finish.cuh"

namespace duo {

template <int D>
struct Int4Shape {
  static constexpr int kCodeBytes = D / 2;  // bytes of codes per token row
  static constexpr int kTile = 64;          // rows per pipeline stage
  static constexpr int kStages = 6;
  static constexpr int kWarps = 4;
  static constexpr int kStage = 2 * kTile * kCodeBytes + 2 * kTile * 4;  // K, V codes; K, V sz
  static constexpr int kSmem = kStages * kStage + kStages * 8;
};

__device__ __forceinline__ float2 nib_pair(uint32_t lo, uint32_t hi, uint32_t sel) {
  // byte `sel` of lo / hi placed under the exponent of 2^23, minus 2^23
  const float a = __uint_as_float(__byte_perm(lo, 0x4B000000u, 0x7540u | sel));
  const float b = __uint_as_float(__byte_perm(hi, 0x4B000000u, 0x7540u | sel));
  return __fadd2_rn(make_float2(a, b), make_float2(-8388608.f, -8388608.f));
}

template <int NWORD>
__device__ __forceinline__ void load_codes(uint32_t addr, uint32_t (&w)[NWORD]) {
  if constexpr (NWORD == 2) {
    asm volatile("ld.shared.v2.u32 {%0,%1}, [%2];" : "=r"(w[0]), "=r"(w[1]) : "r"(addr));
  } else {
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(w[0]) : "r"(addr));
  }
}

template <int D, int G>
__global__ void __launch_bounds__(128) decode_int4_kernel(const __grid_constant__ DecodeParams P) {
  using Sh = Int4Shape<D>;
  constexpr int CB = Sh::kCodeBytes;
  constexpr int TILE = Sh::kTile;
  constexpr int STAGES = Sh::kStages;
  constexpr int NWARPS = Sh::kWarps;
  constexpr int NWORD = D / 64;          // 32-bit code words per lane per row
  constexpr int NP = NWORD * 4;          // channel pairs per lane (one per byte)
  constexpr int RW = TILE / NWARPS;
  constexpr int U = RW / 4;
  constexpr int CPL = D / 8;             // channels per lane
  static_assert(NWORD == 1 || NWORD == 2, "head_dim 64 or 128");

  extern __shared__ __align__(128) uint8_t smem[];
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + STAGES * Sh::kStage);
  __shared__ int s_last;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int grp = lane >> 3, li = lane & 7;

  const int n_ret_ctas = P.B * P.n_ret * P.nsplit;
  int b, kvh, pidx, split;
  bool retrieval;
  const uint8_t *Kc, *Vc, *Ks, *Vs;
  int64_t k0, k1;
  if ((int)blockIdx.x < n_ret_ctas) {
    split = blockIdx.x % P.nsplit;
    const int r = blockIdx.x / P.nsplit;
    pidx = r % P.n_ret;
    b = r / P.n_ret;
    kvh = P.h.ret_heads[pidx];
    retrieval = true;
    const int64_t row0 = ((int64_t)b * P.n_ret + pidx) * P.cap;
    Kc = P.p.ret_k + row0 * CB;
    Vc = P.p.ret_v + row0 * CB;
    Ks = P.p.ret_k_sz + row0 * 4;
    Vs = P.p.ret_v_sz + row0 * 4;
    k0 = (int64_t)split * P.split_len;
    k1 = min(P.n, k0 + P.split_len);
  } else {
    const int r = blockIdx.x - n_ret_ctas;
    pidx = r % P.n_str;
    b = r / P.n_str;
    kvh = P.h.str_heads[pidx];
    retrieval = false;
    split = 0;
    const int64_t row0 = ((int64_t)b * P.n_str + pidx) * P.Ws;
    Kc = P.p.str_k + row0 * CB;
    Vc = P.p.str_v + row0 * CB;
    Ks = P.p.str_k_sz + row0 * 4;
    Vs = P.p.str_v_sz + row0 * 4;
    k0 = 0;
    k1 = min(P.n, (int64_t)P.W);
  }
  const int ntiles = (int)((k1 - k0 + TILE - 1) / TILE);

  if (tid == 0) {
    for (int s = 0; s < STAGES; ++s) mbar_init(smem_u32(&bars[s]), 1);
    fence_barrier_init();
  }
  __syncthreads();

  // stage s: [K codes][V codes][K sz][V sz]; tiles start at multiples of TILE
  // and the sz rows of every head are padded to a multiple of 4, so copying
  // whole 16-byte groups of sz never leaves the head's rows.
  auto issue = [&](int t) {
    const int s = t % STAGES;
    const int64_t r0 = k0 + (int64_t)t * TILE;
    const uint32_t nrow = (uint32_t)min((int64_t)TILE, k1 - r0);
    const uint32_t cbytes = nrow * CB;
    const uint32_t sbytes = ((nrow + 3u) & ~3u) * 4u;
    const uint32_t bar = smem_u32(&bars[s]);
    const uint32_t dst = smem_u32(smem + s * Sh::kStage);
    mbar_arrive_expect_tx(bar, 2 * cbytes + 2 * sbytes);
    bulk_g2s(dst, Kc + r0 * CB, cbytes, bar);
    bulk_g2s(dst + TILE * CB, Vc + r0 * CB, cbytes, bar);
    bulk_g2s(dst + 2 * TILE * CB, Ks + r0 * 4, sbytes, bar);
    bulk_g2s(dst + 2 * TILE * CB + TILE * 4, Vs + r0 * 4, sbytes, bar);
  };
  if (tid == 0)
    for (int t = 0; t < min(STAGES, ntiles); ++t) issue(t);

  // queries, scaled to log2 units; the odd channel of each pair divided by 16
  float2 q2[G][NP];
  float qsum[G];
  {
    const __nv_bfloat16 *qb =
        reinterpret_cast<const __nv_bfloat16 *>(P.q) + ((int64_t)b * P.Hq + (int64_t)kvh * G) * D;
#pragma unroll
    for (int g = 0; g < G; ++g) {
      float part = 0.f;
#pragma unroll
      for (int j = 0; j < NP; ++j) {
        const int c = li * CPL + 2 * j;
        const float a = __bfloat162float(qb[g * D + c]) * P.scale_log2;
        const float bb = __bfloat162float(qb[g * D + c + 1]) * P.scale_log2;
        q2[g][j] = make_float2(a, bb * 0.0625f);
        part += a + bb;
      }
      part += __shfl_xor_sync(0xffffffffu, part, 1);
      part += __shfl_xor_sync(0xffffffffu, part, 2);
      part += __shfl_xor_sync(0xffffffffu, part, 4);
      qsum[g] = part;
    }
  }

  float m[G], l[G], z[G];
  float2 of[G][NP];
#pragma unroll
  for (int g = 0; g < G; ++g) {
    m[g] = -INFINITY;
    l[g] = 0.f;
    z[g] = 0.f;
#pragma unroll
    for (int j = 0; j < NP; ++j) of[g][j] = make_float2(0.f, 0.f);
  }

  bool failed = false;
  int t = 0;
  for (; t < ntiles; ++t) {
    const int s = t % STAGES;
    const bool got = mbar_wait(smem_u32(&bars[s]), (uint32_t)((t / STAGES) & 1), P.err,
                               kErrWaitTileLoad);
    const uint32_t kc = smem_u32(smem + s * Sh::kStage);
    const uint32_t vc = kc + TILE * CB;
    const uint8_t *ksz = smem + s * Sh::kStage + 2 * TILE * CB;
    const uint8_t *vsz = ksz + TILE * 4;
    const int nrow = (int)min((int64_t)TILE, k1 - (k0 + (int64_t)t * TILE));

    float sc[U][G];
    bool valid[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int row = warp * RW + u * 4 + grp;
      valid[u] = row < nrow;
      uint32_t w[NWORD];
      load_codes<NWORD>(kc + row * CB + li * 4 * NWORD, w);
      float2 acc[G];
#pragma unroll
      for (int g = 0; g < G; ++g) acc[g] = make_float2(0.f, 0.f);
#pragma unroll
      for (int k = 0; k < NWORD; ++k) {
        const uint32_t lo = w[k] & 0x0F0F0F0Fu, hi = w[k] & 0xF0F0F0F0u;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float2 f = nib_pair(lo, hi, (uint32_t)i);
#pragma unroll
          for (int g = 0; g < G; ++g) acc[g] = ffma2(q2[g][4 * k + i], f, acc[g]);
        }
      }
#pragma unroll
      for (int g = 0; g < G; ++g) sc[u][g] = acc[g].x + acc[g].y;
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int row = warp * RW + u * 4 + grp;
      const __half2 szp = *reinterpret_cast<const __half2 *>(ksz + row * 4);
      const float ks = __low2float(szp), kz = __high2float(szp);
#pragma unroll
      for (int g = 0; g < G; ++g) {
        float x = sc[u][g];
        x += __shfl_xor_sync(0xffffffffu, x, 1);
        x += __shfl_xor_sync(0xffffffffu, x, 2);
        x += __shfl_xor_sync(0xffffffffu, x, 4);
        sc[u][g] = valid[u] ? (ks * x + kz * qsum[g]) : -INFINITY;
      }
    }
#pragma unroll
    for (int g = 0; g < G; ++g) {
      float mx = sc[0][g];
#pragma unroll
      for (int u = 1; u < U; ++u) mx = fmaxf(mx, sc[u][g]);
      if (mx > m[g]) {
        const float a = (m[g] == -INFINITY) ? 0.f : fast_exp2(m[g] - mx);
        l[g] *= a;
        z[g] *= a;
        const float2 a2 = make_float2(a, a);
#pragma unroll
        for (int j = 0; j < NP; ++j) of[g][j] = fmul2(of[g][j], a2);
        m[g] = mx;
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      if (!valid[u]) continue;
      const int row = warp * RW + u * 4 + grp;
      const __half2 szp = *reinterpret_cast<const __half2 *>(vsz + row * 4);
      const float vs = __low2float(szp), vz = __high2float(szp);
      float ps[G];
#pragma unroll
      for (int g = 0; g < G; ++g) {
        const float p = fast_exp2(sc[u][g] - m[g]);
        l[g] += p;
        z[g] += p * vz;
        ps[g] = p * vs;
      }
      uint32_t w[NWORD];
      load_codes<NWORD>(vc + row * CB + li * 4 * NWORD, w);
#pragma unroll
      for (int k = 0; k < NWORD; ++k) {
        const uint32_t lo = w[k] & 0x0F0F0F0Fu, hi = w[k] & 0xF0F0F0F0u;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float2 f = nib_pair(lo, hi, (uint32_t)i);
#pragma unroll
          for (int g = 0; g < G; ++g)
            of[g][4 * k + i] = ffma2(make_float2(ps[g], ps[g] * 0.0625f), f, of[g][4 * k + i]);
        }
      }
    }
    if (!__syncthreads_and(got)) {
      failed = true;
      break;
    }
    if (tid == 0 && t + STAGES < ntiles) issue(t + STAGES);
  }
  if (failed) {
    if (tid == 0)
      for (int tt = t; tt < min(ntiles, t + STAGES); ++tt)
        mbar_wait(smem_u32(&bars[tt % STAGES]), (uint32_t)((tt / STAGES) & 1), P.err,
                  kErrWaitTileLoad);
    __syncthreads();  // every thread saw the failure (the barrier above)
    // Leave this split empty (weight zero) but still take its merge ticket
    // below, so that the workspace counters return to zero; the error word
    // tells the caller the output is not valid.
#pragma unroll
    for (int g = 0; g < G; ++g) {
      m[g] = -INFINITY;
      l[g] = 0.f;
      z[g] = 0.f;
#pragma unroll
      for (int j = 0; j < NP; ++j) of[g][j] = make_float2(0.f, 0.f);
    }
  }
  // the zero-point term adds the same amount to every channel
#pragma unroll
  for (int g = 0; g < G; ++g)
#pragma unroll
    for (int j = 0; j < NP; ++j) {
      of[g][j].x += z[g];
      of[g][j].y += z[g];
    }
  decode_finish<__nv_bfloat16, D, G, NWARPS, NP>(
      P, smem, &s_last, m, l, of, [](int li_, int j) { return li_ * CPL + 2 * j; }, retrieval, b,
      kvh, pidx, split);
}

template <int D, int G>
static cudaError_t run_int4(const DecodeParams &d, cudaStream_t s, DecodeConfig *cfg) {
  using Sh = Int4Shape<D>;
  auto kern = decode_int4_kernel<D, G>;
  static bool attr_done = false;
  if (!attr_done) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Sh::kSmem);
    if (e != cudaSuccess) return e;
    attr_done = true;
  }
  if (cfg) {
    int occ = 0, dev = 0, sms = 0;
    cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, 128, Sh::kSmem);
    if (e != cudaSuccess) return e;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
    if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
    cfg->tile_rows = Sh::kTile;
    cfg->ctas_per_sm = occ;
    cfg->num_sms = sms;
    return cudaSuccess;
  }
  const int grid = d.B * d.n_ret * d.nsplit + d.B * d.n_str;
  if (grid == 0) return cudaSuccess;
  kern<<<grid, 128, Sh::kSmem, s>>>(d);
  return cudaGetLastError();
}

template <int D>
static cudaError_t dispatch_int4(const DecodeParams &d, int G, cudaStream_t s, DecodeConfig *cfg) {
  switch (G) {
    case 1: return run_int4<D, 1>(d, s, cfg);
    case 2: return run_int4<D, 2>(d, s, cfg);
    case 4: return run_int4<D, 4>(d, s, cfg);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t decode_int4_config(int D, int G, DecodeConfig *cfg) {
  DecodeParams dummy{};
  if (D == 128) return dispatch_int4<128>(dummy, G, nullptr, cfg);
  if (D == 64) return dispatch_int4<64>(dummy, G, nullptr, cfg);
  return cudaErrorInvalidValue;
}

cudaError_t launch_decode_int4(const DecodeParams &d, cudaStream_t s) {
  if (d.D == 128) return dispatch_int4<128>(d, d.G, s, nullptr);
  if (d.D == 64) return dispatch_int4<64>(d, d.G, s, nullptr);
  return cudaErrorInvalidValue;
}

}  // namespace duo
