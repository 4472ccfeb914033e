// Single-token decode attention over the head-split KV cache.
//
// One launch covers a whole layer:
//  * retrieval KV heads (full KV cache, causal attention over every token) run
//    split-K flash decoding: CTA (b, head, split) streams its key range of the
//    page into its own shared memory with 1-D bulk copies (the TMA engine),
//    computes the G query heads' logits and an online softmax, and
//    writes a (normalised partial output, log-sum-exp) pair; the CTA that
//    finishes last for a head merges all splits (an atomic ticket; no CTA ever
//    waits for another);
//  * streaming KV heads (sinks plus recent tokens, constant length) run the
//    same pipeline over their S + R slot buffer in one CTA each.  After the
//    append the buffer holds exactly the visible set, and softmax does not
//    depend on the order of its terms, so slot order is irrelevant.
// Pages: "DuoAttention: Efficient Long-Context LLM Inference with Retrieval
// and Streaming Heads" (hotpaper.ai), abstract and section "기술적 접근법";
// "韩松团队长上下文LLM推理高效框架" (cn.bg3.co), section "研究背景" (decode cost
// linear in the context: this kernel is bound by HBM bandwidth).
//
// Work split inside a CTA (NWARPS warps): a warp owns TILE/NWARPS consecutive
// rows of each tile; a row is read by a group of 8 lanes, lane li holding the
// 16-byte chunks li, li+8, ... of the row (so each quarter-warp reads 128
// contiguous bytes of shared memory: no bank conflicts).  Dot products use
// packed fp32x2 FMAs; the 8 partial sums of a row meet through 3 xor shuffles.
#include "common.cuh"
#include "decode_finish.cuh"

namespace duo {

template <typename T, int D>
struct DecodeShape {
  static constexpr int kRowBytes = D * (int)sizeof(T);
  static constexpr int kTile = 16384 / kRowBytes;  // rows per pipeline stage
  static constexpr int kStages = 3;
  static constexpr int kWarps = 4;
  static constexpr int kTileBytes = kTile * kRowBytes;
  static constexpr int kSmem = kStages * 2 * kTileBytes + kStages * 8;
};

template <typename T, int D, int G>
__global__ void __launch_bounds__(128) decode_kernel(const __grid_constant__ DecodeParams P) {
  using Sh = DecodeShape<T, D>;
  constexpr int ROW_BYTES = Sh::kRowBytes;
  constexpr int TILE = Sh::kTile;
  constexpr int STAGES = Sh::kStages;
  constexpr int NWARPS = Sh::kWarps;
  constexpr int TILE_BYTES = Sh::kTileBytes;
  constexpr int CH = ROW_BYTES / 16;   // 16-byte chunks per row
  constexpr int NV = CH / 8;           // chunks per lane
  constexpr int EC = 16 / (int)sizeof(T);
  constexpr int PPC = EC / 2;          // fp32 pairs per chunk
  constexpr int NP = NV * PPC;         // fp32 pairs per lane
  constexpr int RW = TILE / NWARPS;    // rows per warp per tile
  constexpr int U = RW / 4;            // rows per 8-lane group per tile
  static_assert(CH % 8 == 0 && RW % 4 == 0, "tile shape");

  extern __shared__ __align__(128) uint8_t smem[];
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + STAGES * 2 * TILE_BYTES);
  __shared__ int s_last;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int grp = lane >> 3, li = lane & 7;

  // ---- which (batch, KV head, key range) this CTA owns
  const int n_ret_ctas = P.B * P.n_ret * P.nsplit;
  int b, kvh, pidx, split;
  bool retrieval;
  const uint8_t *Kb, *Vb;
  int64_t k0, k1;
  if ((int)blockIdx.x < n_ret_ctas) {
    split = blockIdx.x % P.nsplit;
    const int r = blockIdx.x / P.nsplit;
    pidx = r % P.n_ret;
    b = r / P.n_ret;
    kvh = P.h.ret_heads[pidx];
    retrieval = true;
    const int64_t base = ((int64_t)b * P.n_ret + pidx) * P.cap * ROW_BYTES;
    Kb = P.p.ret_k + base;
    Vb = P.p.ret_v + base;
    k0 = (int64_t)split * P.split_len;
    k1 = min(P.n, k0 + P.split_len);
  } else {
    const int r = blockIdx.x - n_ret_ctas;
    pidx = r % P.n_str;
    b = r / P.n_str;
    kvh = P.h.str_heads[pidx];
    retrieval = false;
    split = 0;
    const int64_t base = ((int64_t)b * P.n_str + pidx) * (int64_t)P.Ws * ROW_BYTES;
    Kb = P.p.str_k + base;
    Vb = P.p.str_v + base;
    k0 = 0;
    k1 = min(P.n, (int64_t)P.W);
  }
  const int ntiles = (int)((k1 - k0 + TILE - 1) / TILE);

  if (tid == 0) {
    for (int s = 0; s < STAGES; ++s) mbar_init(smem_u32(&bars[s]), 1);
    fence_barrier_init();
  }
  __syncthreads();

  auto issue = [&](int t) {
    const int s = t % STAGES;
    const int64_t r0 = k0 + (int64_t)t * TILE;
    const uint32_t nrow = (uint32_t)min((int64_t)TILE, k1 - r0);
    const uint32_t bytes = nrow * ROW_BYTES;
    const uint32_t bar = smem_u32(&bars[s]);
    const uint32_t dst = smem_u32(smem + s * 2 * TILE_BYTES);
    mbar_arrive_expect_tx(bar, 2 * bytes);
    bulk_g2s(dst, Kb + r0 * ROW_BYTES, bytes, bar);
    bulk_g2s(dst + TILE_BYTES, Vb + r0 * ROW_BYTES, bytes, bar);
  };
  if (tid == 0)
    for (int t = 0; t < min(STAGES, ntiles); ++t) issue(t);

  // ---- queries of the G heads sharing this KV head, pre-scaled to log2 units
  float2 qf[G][NP];
  {
    const T *qb = reinterpret_cast<const T *>(P.q) + ((int64_t)b * P.Hq + (int64_t)kvh * G) * D;
#pragma unroll
    for (int g = 0; g < G; ++g)
#pragma unroll
      for (int v = 0; v < NV; ++v)
#pragma unroll
        for (int j = 0; j < PPC; ++j) {
          const int e = (v * 8 + li) * EC + 2 * j;
          qf[g][v * PPC + j] = make_float2(load_in(qb + g * D + e) * P.scale_log2,
                                           load_in(qb + g * D + e + 1) * P.scale_log2);
        }
  }

  float m[G], l[G];
  float2 of[G][NP];
#pragma unroll
  for (int g = 0; g < G; ++g) {
    m[g] = -INFINITY;
    l[g] = 0.f;
#pragma unroll
    for (int j = 0; j < NP; ++j) of[g][j] = make_float2(0.f, 0.f);
  }

  bool failed = false;
  int t = 0;
  for (; t < ntiles; ++t) {
    const int s = t % STAGES;
    const bool got = mbar_wait(smem_u32(&bars[s]), (uint32_t)((t / STAGES) & 1), P.err,
                               kErrWaitTileLoad);
    const uint32_t kbase = smem_u32(smem + s * 2 * TILE_BYTES);
    const uint32_t vbase = kbase + TILE_BYTES;
    const int nrow = (int)min((int64_t)TILE, k1 - (k0 + (int64_t)t * TILE));

    float sc[U][G];
    bool valid[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int row = warp * RW + u * 4 + grp;
      valid[u] = row < nrow;
      float2 acc[G];
#pragma unroll
      for (int g = 0; g < G; ++g) acc[g] = make_float2(0.f, 0.f);
#pragma unroll
      for (int v = 0; v < NV; ++v) {
        const uint4 c = lds128(kbase + row * ROW_BYTES + (v * 8 + li) * 16);
        float2 f[PPC];
        Chunk<T>::unpack(c, f);
#pragma unroll
        for (int g = 0; g < G; ++g)
#pragma unroll
          for (int j = 0; j < PPC; ++j) acc[g] = ffma2(qf[g][v * PPC + j], f[j], acc[g]);
      }
#pragma unroll
      for (int g = 0; g < G; ++g) sc[u][g] = acc[g].x + acc[g].y;
    }
#pragma unroll
    for (int u = 0; u < U; ++u)
#pragma unroll
      for (int g = 0; g < G; ++g) {
        float x = sc[u][g];
        x += __shfl_xor_sync(0xffffffffu, x, 1);
        x += __shfl_xor_sync(0xffffffffu, x, 2);
        x += __shfl_xor_sync(0xffffffffu, x, 4);
        sc[u][g] = valid[u] ? x : -INFINITY;
      }
#pragma unroll
    for (int g = 0; g < G; ++g) {
      float mx = sc[0][g];
#pragma unroll
      for (int u = 1; u < U; ++u) mx = fmaxf(mx, sc[u][g]);
      if (mx > m[g]) {
        const float a = (m[g] == -INFINITY) ? 0.f : fast_exp2(m[g] - mx);
        l[g] *= a;
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
      float p[G];
#pragma unroll
      for (int g = 0; g < G; ++g) {
        p[g] = fast_exp2(sc[u][g] - m[g]);
        l[g] += p[g];
      }
#pragma unroll
      for (int v = 0; v < NV; ++v) {
        const uint4 c = lds128(vbase + row * ROW_BYTES + (v * 8 + li) * 16);
        float2 f[PPC];
        Chunk<T>::unpack(c, f);
#pragma unroll
        for (int g = 0; g < G; ++g) {
          const float2 p2 = make_float2(p[g], p[g]);
#pragma unroll
          for (int j = 0; j < PPC; ++j) of[g][v * PPC + j] = ffma2(p2, f[j], of[g][v * PPC + j]);
        }
      }
    }
    // every thread is done with stage s; refill it (or stop on a failed wait)
    if (!__syncthreads_and(got)) {
      failed = true;
      break;
    }
    if (tid == 0 && t + STAGES < ntiles) issue(t + STAGES);
  }
  if (failed) {
    // Let the copies already in flight land before shared memory is reused
    // below (and before the CTA's shared memory can go to another CTA).
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
#pragma unroll
      for (int j = 0; j < NP; ++j) of[g][j] = make_float2(0.f, 0.f);
    }
  }

  decode_finish<T, D, G, NWARPS, NP>(
      P, smem, &s_last, m, l, of, [](int li_, int j) { return ((j / PPC) * 8 + li_) * EC + 2 * (j % PPC); },
      retrieval, b, kvh, pidx, split);
}

// ------------------------------------------------------------------ dispatch

template <typename T, int D, int G>
static cudaError_t run(const DecodeParams &d, cudaStream_t s, DecodeConfig *cfg) {
  using Sh = DecodeShape<T, D>;
  auto kern = decode_kernel<T, D, G>;
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

template <typename T, int D>
static cudaError_t run_g(const DecodeParams &d, int G, cudaStream_t s, DecodeConfig *cfg) {
  switch (G) {
    case 1: return run<T, D, 1>(d, s, cfg);
    case 2: return run<T, D, 2>(d, s, cfg);
    case 4: return run<T, D, 4>(d, s, cfg);
    default: return cudaErrorInvalidValue;
  }
}

static cudaError_t dispatch(const DecodeParams &d, int kv_type, int D, int G, cudaStream_t s,
                            DecodeConfig *cfg) {
  if (kv_type == kF32) {
    if (D == 64) return run_g<float, 64>(d, G, s, cfg);
    if (D == 128) return run_g<float, 128>(d, G, s, cfg);
  } else if (kv_type == kBF16) {
    if (D == 64) return run_g<__nv_bfloat16, 64>(d, G, s, cfg);
    if (D == 128) return run_g<__nv_bfloat16, 128>(d, G, s, cfg);
  }
  return cudaErrorInvalidValue;
}

cudaError_t decode_int4_config(int D, int G, DecodeConfig *cfg);
cudaError_t launch_decode_int4(const DecodeParams &d, cudaStream_t s);
bool decode_mma_supported(int kv_type, int D, int G);
cudaError_t decode_mma_config(int kv_type, int G, DecodeConfig *cfg);
cudaError_t launch_decode_mma(const DecodeParams &d, int kv_type, cudaStream_t s);

// head_dim 128 with a bf16 or 4-bit cache runs the tensor-core decode
// (decode_mma.cu); fp32 caches and head_dim 64 run the CUDA-core kernels.
cudaError_t decode_config(int kv_type, int D, int G, DecodeConfig *cfg) {
  if (decode_mma_supported(kv_type, D, G)) return decode_mma_config(kv_type, G, cfg);
  if (kv_type == kINT4) return decode_int4_config(D, G, cfg);
  DecodeParams dummy{};
  return dispatch(dummy, kv_type, D, G, nullptr, cfg);
}

cudaError_t launch_decode(const DecodeParams &d, int kv_type, cudaStream_t s) {
  if (decode_mma_supported(kv_type, d.D, d.G)) return launch_decode_mma(d, kv_type, s);
  if (kv_type == kINT4) return launch_decode_int4(d, s);
  return dispatch(d, kv_type, d.D, d.G, s, nullptr);
}

}  // namespace duo
