// Single-token decode attention with warp-level tensor-core MMAs
// (mma.sync m16n8k16, bf16 in, fp32 accumulate), for head_dim 128 and a bf16
// or 4-bit KV cache.
//
// Same work split as the CUDA-core decode (split-K over retrieval pages, one
// CTA per streaming slot buffer, last split merges); what changes is the inner
// product.  Per warp and per 16 keys:
//   S[16 x 8]  = Q[16 x 128] . K^T      two key tiles of 8, 8 k-steps each
//   O[16 x 8] += P[16 x 16] . V         one per 8-channel output tile (16)
// Rows 0..G-1 of the 16-row operands are the G query heads sharing the KV head
// (the rest are zero).  The accumulator fragment of S is, element for element,
// the A fragment of P for the next product, so probabilities never leave
// registers.  Because a dot product does not depend on the order of its terms,
// the head-dim positions behind each k-slot are chosen so that every thread's
// B fragment of K is one contiguous 16-byte load of its key row (the query
// fragment follows the same order), and output channels are assigned so that
// a thread's V operand comes from 32 contiguous bytes per key.  K and V are
// loaded straight from global memory into registers; nothing is staged in
// shared memory except the final cross-warp combine.
//
// 4-bit cache: a nibble u becomes the bf16 128 + u by masking it under the bf16
// pattern of 128 and is then reduced by 128 (exact), and the per-token scale
// and zero are applied outside the products: s = sc*(q.u) + zp*sum(q),
// sum p*v_hat = sum (p*sc)*u + (sum p*zp).
//
// Pages: "DuoAttention: Efficient Long-Context LLM Inference with Retrieval and
// Streaming Heads" (hotpaper.ai), abstract and section "기술적 접근법".
#include "common.cuh"
#include "decode_finish.cuh"

namespace duo {

namespace dm {

constexpr int D = 128;
constexpr int NWARPS = 16;
// Key groups of 16 per warp iteration: the 4-bit rows are 4x smaller, so a
// warp takes two groups to keep as many bytes in flight as the bf16 path.
template <bool Q4>
struct Keys {
  static constexpr int KG = Q4 ? 2 : 1;
  static constexpr int STEP = NWARPS * 16 * KG;  // keys per CTA iteration
};

__device__ __forceinline__ void mma16816(float (&d)[4], uint32_t a0, uint32_t a2, uint32_t b0,
                                         uint32_t b1) {
  // rows g+8 of A are zero (a1 = a3 = 0)
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(0u), "r"(a2), "r"(0u), "r"(b0), "r"(b1));
}

template <bool B>
struct BoolC {
  static constexpr bool value = B;
};

__device__ __forceinline__ uint4 ldg128(const void *p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

__device__ __forceinline__ uint2 ldg64(const void *p) {
  uint2 v;
  asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0,%1}, [%2];" : "=r"(v.x), "=r"(v.y) : "l"(p));
  return v;
}

// Fetch [ptr, ptr + bytes) into L2 (16-byte aligned, bytes a multiple of 16).
__device__ __forceinline__ void prefetch_l2(const void *ptr, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(ptr), "r"(bytes) : "memory");
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t *>(&h);
}

// Two 4-bit codes u (at bit s and bit s+16 of x) -> bf16x2 of 128 + u (exact):
// the code is masked under the bit pattern of 128.0, whose mantissa is zero.
// The offset of 128 is removed after the products (see the callers).
__device__ __forceinline__ uint32_t nib2(uint32_t x, int s) {
  return ((x >> s) & 0x000F000Fu) | 0x43004300u;
}

__device__ __forceinline__ void mma16816_full(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                              uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

template <bool Q4, int G>
__global__ void __launch_bounds__(NWARPS * 32, 1) decode_mma_kernel(const __grid_constant__ DecodeParams P) {
  extern __shared__ __align__(16) uint8_t smem[];
  __shared__ int s_last;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, t = lane & 3;  // mma fragment coordinates

  // ---- work item: retrieval CTAs first (launch row r, head, split), then
  // one CTA per (launch row, streaming head)
  const int n_ret_ctas = P.cta0[P.rows.n];
  int r, kvh, pidx, split, nsplit;
  bool retrieval;
  if ((int)blockIdx.x < n_ret_ctas) {
    int lo = 0, hi = P.rows.n;  // the last r with cta0[r] <= blockIdx.x
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (P.cta0[mid] <= (int)blockIdx.x) lo = mid; else hi = mid;
    }
    r = lo;
    nsplit = P.nsplit_r[r];
    const int local = (int)blockIdx.x - P.cta0[r];
    pidx = local / nsplit;
    split = local % nsplit;
    kvh = P.h.ret_heads[pidx];
    retrieval = true;
  } else {
    const int x = (int)blockIdx.x - n_ret_ctas;
    r = x / P.n_str;
    pidx = x % P.n_str;
    kvh = P.h.str_heads[pidx];
    retrieval = false;
    split = 0;
    nsplit = 1;
  }
  const int b = P.rows.row[r];
  // Key indices and tile counts are 32-bit (a row holds fewer than 2^31
  // tokens); byte offsets are formed in 64 bits.
  const int n = P.rows.len[r];  // tokens incl. the new one; the query is at n-1
  // A sequence shard's retrieval heads hold positions [shard_lo, shard_hi)
  // at page rows from 0; `keys` of them are below n.  Streaming heads hold
  // the whole window.
  const int keys = retrieval ? (int)max((int64_t)0, min((int64_t)n, P.shard_hi) - P.shard_lo)
                             : min(n, P.W);
  const bool new_here_shard = !retrieval || (n - 1 >= P.shard_lo && n - 1 < P.shard_hi);
  constexpr int RB = Q4 ? D / 2 : D * 2;  // bytes per key row
  // Streaming heads: one slot buffer, first storage row srow0.  Retrieval
  // heads: key tiles are addressed block by block (a tile never crosses a
  // block of the paged layout), with key indices local to the block.
  auto srow0 = [&]() { return ((int64_t)b * P.n_str + pidx) * P.Ws; };
  const int k0 = 0, k1 = keys;
  constexpr int KG = Keys<Q4>::KG;
  constexpr int T = 16 * KG;  // keys per warp tile
  constexpr int kBlockMask = ~(kPageTokens - 1);
  // A retrieval head with several splits is cut into tiles of T keys.  Each
  // split walks a fixed share of them; with P.pool the shares cover 7/8 of
  // the tiles and the rest is claimed one tile at a time by warps that have
  // finished (see below), so a CTA that gets less memory bandwidth takes
  // fewer tiles and the splits finish together.  Each CTA leaves one
  // partial.  Streaming heads and single-split heads walk [k0, k1).
  const bool split_head = retrieval && nsplit > 1;
  const bool pooled = split_head && P.pool;
  const int tiles = (keys + T - 1) / T;
  const int ts = !split_head ? 0
                 : pooled    ? (tiles - tiles / 8) / nsplit
                             : (tiles + nsplit - 1) / nsplit;  // tiles per split share
  const int t1 = min(tiles, (split + 1) * ts);                 // end of this split's share
  // this warp's first two tiles, [first, first + T) and the one NWARPS tiles on
  const int first = split_head ? (split * ts + warp) * T : k0 + warp * T;
  const int last = split_head ? min(keys, t1 * T) : k1;

  // Launched with programmatic dependent launch, so this may run while the
  // previous kernel in the stream finishes.  Bring this warp's first two
  // tiles into L2 meanwhile: every global write lands in L2, so a line
  // fetched now cannot be stale when the loads below (after the wait) use it.
  // A block-table entry read now may be stale; it only aims a prefetch, and
  // is clamped to the pool so the address stays valid.
  if (lane == 0) {
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const int kb = first + i * NWARPS * T;
      if (kb < last) {
        const int rows = min(T, last - kb);
        int64_t row = srow0() + kb;
        const uint8_t *pk = P.p.str_k, *pv = P.p.str_v, *psk = P.p.str_k_sz, *psv = P.p.str_v_sz;
        if (retrieval) {
          pk = P.p.ret_k;
          pv = P.p.ret_v;
          psk = P.p.ret_k_sz;
          psv = P.p.ret_v_sz;
          if (P.ret.table) {
            int64_t blk = P.ret.table[(int64_t)b * P.ret.stride + (kb >> kPageShift)];
            blk = blk < 0 ? 0 : (blk >= P.ret.blocks ? P.ret.blocks - 1 : blk);
            row = ((blk * P.n_ret + pidx) << kPageShift) + (kb & (kPageTokens - 1));
          } else {
            row = ret_row(P.ret, b, pidx, kb);
          }
        }
        prefetch_l2(pk + row * RB, (uint32_t)(rows * RB));
        prefetch_l2(pv + row * RB, (uint32_t)(rows * RB));
        if (Q4) {  // 4-byte (scale, zero) rows; buffers hold a multiple of 4 rows
          const uint32_t sz = (uint32_t)(((rows + 3) & ~3) * 4);
          prefetch_l2(psk + row * 4, sz);
          prefetch_l2(psv + row * 4, sz);
        }
      }
    }
  }
  // Nothing the previous kernel may have written is read before this.
  asm volatile("griddepcontrol.wait;" ::: "memory");

  // Fused append (bf16 cache): the token at position n-1 is not in the cache
  // yet.  The warp whose tile holds its row writes it there, skips that row,
  // and adds the key at the end from the inputs.
  // In partial mode a rank that does not own the streaming heads leaves
  // their rows empty (another shard contributes them).
  if (P.part_o && !retrieval && !P.own_str) {
    const int64_t row0 = (int64_t)r * P.Hq + (int64_t)kvh * G;
    for (int i = tid; i < G * D; i += NWARPS * 32) P.part_o[row0 * D + i] = 0.f;
    if (tid < G) P.part_lse[row0 + tid] = -INFINITY;
    return;
  }
  const bool fused = !Q4 && P.knew != nullptr && new_here_shard;
  const int newk = retrieval ? n - 1 - (int)P.shard_lo : (int)ring_slot(n - 1, P.S, P.R);  // its row
  const bool owns_new = fused && !split_head && newk >= k0 && newk < k1;
  auto write_new = [&]() {  // one warp copies the new K and V rows into the cache
    const int64_t off = ((int64_t)r * P.Hkv + kvh) * (int64_t)RB;
    const int c = lane & 15;  // 16 lanes x 16 bytes = one 256-byte row
    const uint8_t *src = reinterpret_cast<const uint8_t *>(lane < 16 ? P.knew : P.vnew) + off;
    const int64_t row = retrieval ? ret_row(P.ret, b, pidx, newk) : srow0() + newk;
    uint8_t *dst = const_cast<uint8_t *>(lane < 16 ? (retrieval ? P.p.ret_k : P.p.str_k)
                                                   : (retrieval ? P.p.ret_v : P.p.str_v)) + row * RB;
    reinterpret_cast<uint4 *>(dst)[c] = ldg128(src + 16 * c);
  };
  if (owns_new && warp == 0) write_new();

  // ---- query fragments (rows g < G), k-step order matching the K loads
  uint32_t qa[8][2];
  float qsum = 0.f;  // sum of the query's channels (4-bit zero-point term)
  const bool live = g < G;
  {
    const __nv_bfloat16 *qrow =
        reinterpret_cast<const __nv_bfloat16 *>(P.q) + ((int64_t)r * P.Hq + (int64_t)kvh * G + g) * D;
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      int c0, c1, c2, c3;  // channels behind k-slots 2t, 2t+1, 2t+8, 2t+9
      if (Q4) {
        const int w = k >> 1, tt = k & 1;
        c0 = 32 * t + 8 * w + 2 * tt;
        c1 = c0 + 4;
        c2 = c0 + 1;
        c3 = c0 + 5;
      } else {
        const int s = k >> 1, tt = k & 1;
        c0 = 32 * s + 8 * t + 4 * tt;
        c1 = c0 + 1;
        c2 = c0 + 2;
        c3 = c0 + 3;
      }
      const float q0 = live ? __bfloat162float(qrow[c0]) : 0.f;
      const float q1 = live ? __bfloat162float(qrow[c1]) : 0.f;
      const float q2 = live ? __bfloat162float(qrow[c2]) : 0.f;
      const float q3 = live ? __bfloat162float(qrow[c3]) : 0.f;
      qa[k][0] = pack_bf16(q0, q1);  // exact: the inputs are bf16
      qa[k][1] = pack_bf16(q2, q3);
      qsum += (q0 + q1) + (q2 + q3);
    }
    qsum += __shfl_xor_sync(0xffffffffu, qsum, 1);
    qsum += __shfl_xor_sync(0xffffffffu, qsum, 2);
  }
  const float sl2 = P.scale_log2;

  // O^T accumulators: tile mt holds channels vchan(mt) (rows g) and
  // vchan(mt) + 1 (rows g+8) for queries 2t and 2t+1.  bf16: the thread's V
  // channels are the 16-byte chunks g and 8+g of a row (so the eight lanes of
  // a key read 128 contiguous bytes); 4-bit: code bytes 8g..8g+7.
  auto vchan = [&](int mt) {
    return Q4 ? 16 * g + 2 * mt : 64 * (mt >> 2) + 8 * g + 2 * (mt & 3);
  };
  float o[8][4];
#pragma unroll
  for (int i = 0; i < 8; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
  // softmax state of query g (identical in the four threads of a row); for the
  // 4-bit cache z = sum p*zp and cs = sum p*sc (as multiplied, see below)
  float m = -INFINITY, l = 0.f, z = 0.f, cs = 0.f;

  // One warp, keys [kb0, kb0 + 16*KG) below hi of the buffers Kx/Vx (and, for
  // the 4-bit cache, the (scale, zero) rows Ksx/Vsx), row index = key, except
  // `skip_key`.
  // `full` (a compile-time flag) promises that all keys of the tile lie below
  // hi and none is skip_key, so no load or score needs a bounds test.
  auto tile = [&](auto full, const uint8_t *Kx, const uint8_t *Vx, const uint8_t *Ksx,
                  const uint8_t *Vsx, int kb0, int hi, int skip_key) {
    constexpr bool FULL = decltype(full)::value;
    // ------------------------------------------------------------ loads (all up front)
    // group kg covers keys kb = kb0 + 16*kg ..: K of key kb + 8*nt + g (this
    // thread's column of S); V of keys kb + {2t, 2t+1, 8+2t, 9+2t} (the k-slots
    // of the P^T fragment) at this thread's channels (see vchan below).
    uint4 kr[KG][2][Q4 ? 1 : 4];
    uint2 ksz[KG][2], vsz[KG][2];
    uint4 vr[KG][4][Q4 ? 1 : 2];
#pragma unroll
    for (int kg = 0; kg < KG; ++kg) {
      const int kb = kb0 + 16 * kg;
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
        const int key = kb + 8 * nt + g;
        const bool ok = FULL || (key < hi && key != skip_key);
        if (Q4) {
          kr[kg][nt][0] = ok ? ldg128(Kx + key * RB + 16 * t) : make_uint4(0, 0, 0, 0);
          const int key2 = kb + 8 * nt + 2 * t;
          ksz[kg][nt] = (FULL || key2 < hi) ? ldg64(Ksx + key2 * 4) : make_uint2(0, 0);
          vsz[kg][nt] = (FULL || key2 < hi) ? ldg64(Vsx + key2 * 4) : make_uint2(0, 0);
        } else {
#pragma unroll
          for (int sp = 0; sp < 4; ++sp)
            kr[kg][nt][sp] = ok ? ldg128(Kx + key * RB + (32 * sp + 8 * t) * 2) : make_uint4(0, 0, 0, 0);
        }
      }
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int key = kb + 2 * t + (i & 1) + 8 * (i >> 1);
        const bool ok = FULL || (key < hi && key != skip_key);
        if (Q4) {
          const uint2 x = ok ? ldg64(Vx + key * RB + 8 * g) : make_uint2(0, 0);
          vr[kg][i][0] = make_uint4(x.x, x.y, 0, 0);
        } else {
#pragma unroll
          for (int h = 0; h < 2; ++h)
            vr[kg][i][h] = ok ? ldg128(Vx + key * RB + 16 * (8 * h + g)) : make_uint4(0, 0, 0, 0);
        }
      }
    }
    // ------------------------------------------------------------ S = Q K^T
    float sc[KG][2][2];
#pragma unroll
    for (int kg = 0; kg < KG; ++kg) {
      const int kb = kb0 + 16 * kg;
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
        float s[4] = {0.f, 0.f, 0.f, 0.f};
        if (Q4) {
          const uint32_t w4[4] = {kr[kg][nt][0].x, kr[kg][nt][0].y, kr[kg][nt][0].z, kr[kg][nt][0].w};
#pragma unroll
          for (int w = 0; w < 4; ++w) {
            mma16816(s, qa[2 * w][0], qa[2 * w][1], nib2(w4[w], 0), nib2(w4[w], 4));
            mma16816(s, qa[2 * w + 1][0], qa[2 * w + 1][1], nib2(w4[w], 8), nib2(w4[w], 12));
          }
        } else {
#pragma unroll
          for (int sp = 0; sp < 4; ++sp) {
            mma16816(s, qa[2 * sp][0], qa[2 * sp][1], kr[kg][nt][sp].x, kr[kg][nt][sp].y);
            mma16816(s, qa[2 * sp + 1][0], qa[2 * sp + 1][1], kr[kg][nt][sp].z, kr[kg][nt][sp].w);
          }
        }
        // scores of query g at keys kb + 8*nt + 2t + e
        const int key = kb + 8 * nt + 2 * t;
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          float raw = s[e];
          if (Q4) {
            const __half2 kp = *reinterpret_cast<const __half2 *>(e ? &ksz[kg][nt].y : &ksz[kg][nt].x);
            // q.(128 + u) = q.u + 128*sum(q):  s = sc*q.u + zp*sum(q)
            const float ksc = __low2float(kp);
            raw = ksc * raw + (__high2float(kp) - 128.f * ksc) * qsum;
          }
          sc[kg][nt][e] =
              (live && (FULL || (key + e < hi && key + e != skip_key))) ? raw * sl2 : -INFINITY;
        }
      }
    }
    // ------------------------------------------------------------ online softmax
    float mx = -INFINITY;
#pragma unroll
    for (int kg = 0; kg < KG; ++kg)
      mx = fmaxf(mx, fmaxf(fmaxf(sc[kg][0][0], sc[kg][0][1]), fmaxf(sc[kg][1][0], sc[kg][1][1])));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
    // Rescale only when the running max grows by more than 2^8 (numerator and
    // denominator scale together, so the result is unchanged).
    const bool grow = mx > m + 8.f || (m == -INFINITY && mx > -INFINITY);
    float alpha = 1.f;
    if (grow) {
      alpha = (m == -INFINITY) ? 0.f : fast_exp2(m - mx);
      l *= alpha;
      z *= alpha;
      cs *= alpha;
      m = mx;
    }
    if (__any_sync(0xffffffffu, grow)) {
      // O^T columns are queries 2t and 2t+1: take their factors from the
      // threads that own those rows of S.
      const float a0 = __shfl_sync(0xffffffffu, alpha, (2 * t) << 2);
      const float a1 = __shfl_sync(0xffffffffu, alpha, (2 * t + 1) << 2);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        o[i][0] *= a0;
        o[i][2] *= a0;
        o[i][1] *= a1;
        o[i][3] *= a1;
      }
    }
#pragma unroll
    for (int kg = 0; kg < KG; ++kg) {
      float p[2][2];
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          p[nt][e] = (sc[kg][nt][e] == -INFINITY) ? 0.f : fast_exp2(sc[kg][nt][e] - m);
          l += p[nt][e];
          if (Q4) {  // the key's V (scale, zero), unpacked where used
            const __half2 vp = *reinterpret_cast<const __half2 *>(e ? &vsz[kg][nt].y : &vsz[kg][nt].x);
            z += p[nt][e] * __high2float(vp);
            p[nt][e] *= __low2float(vp);
          }
        }
      // P^T fragment: b0 = keys 2t, 2t+1 (tile 0), b1 = keys 8+2t, 9+2t (tile 1)
      const uint32_t pb0 = pack_bf16(p[0][0], p[0][1]);
      const uint32_t pb1 = pack_bf16(p[1][0], p[1][1]);
      // 4-bit cache: p*sc multiplies codes up to 15 whose sum is offset by the
      // zero point, so bf16's 8-bit mantissa alone is too coarse; the residual
      // p*sc - bf16(p*sc) goes through a second product (16 mantissa bits).
      uint32_t pl0 = 0u, pl1 = 0u;
      if (Q4) {
        const __nv_bfloat162 h0 = *reinterpret_cast<const __nv_bfloat162 *>(&pb0);
        const __nv_bfloat162 h1 = *reinterpret_cast<const __nv_bfloat162 *>(&pb1);
        pl0 = pack_bf16(p[0][0] - __low2float(h0), p[0][1] - __high2float(h0));
        pl1 = pack_bf16(p[1][0] - __low2float(h1), p[1][1] - __high2float(h1));
        // The V codes enter as 128 + u: remember exactly what was multiplied
        // so that 128 * sum(p*sc) can be removed from O afterwards.
        const __nv_bfloat162 l0 = *reinterpret_cast<const __nv_bfloat162 *>(&pl0);
        const __nv_bfloat162 l1 = *reinterpret_cast<const __nv_bfloat162 *>(&pl1);
        cs += ((__low2float(h0) + __low2float(l0)) + (__high2float(h0) + __high2float(l0))) +
              ((__low2float(h1) + __low2float(l1)) + (__high2float(h1) + __high2float(l1)));
      }
      // ---------------------------------------------------------- O^T += V^T P^T
      if (Q4) {
#pragma unroll
        for (int wi = 0; wi < 2; ++wi) {
          const uint32_t xa = wi ? vr[kg][0][0].y : vr[kg][0][0].x, xb = wi ? vr[kg][1][0].y : vr[kg][1][0].x;
          const uint32_t xc = wi ? vr[kg][2][0].y : vr[kg][2][0].x, xd = wi ? vr[kg][3][0].y : vr[kg][3][0].x;
#pragma unroll
          for (int j = 0; j < 4; j += 2) {
            const uint32_t sel = j ? 0x7632u : 0x5410u;
            const uint32_t ab = __byte_perm(xa, xb, sel);  // [A_j, A_j+1, B_j, B_j+1]
            const uint32_t cd = __byte_perm(xc, xd, sel);
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const int mt = 4 * wi + j + h;  // code byte 8g + mt: channels 16g + 2mt, +1
              const uint32_t a0 = nib2(ab, 8 * h), a1 = nib2(ab, 8 * h + 4);
              const uint32_t a2 = nib2(cd, 8 * h), a3 = nib2(cd, 8 * h + 4);
              mma16816_full(o[mt], a0, a1, a2, a3, pb0, pb1);
              mma16816_full(o[mt], a0, a1, a2, a3, pl0, pl1);
            }
          }
        }
      } else {
        const uint4 *va = vr[kg][0], *vb = vr[kg][1], *vc = vr[kg][2], *vd = vr[kg][3];
        const uint32_t wa[8] = {va[0].x, va[0].y, va[0].z, va[0].w, va[1].x, va[1].y, va[1].z, va[1].w};
        const uint32_t wb[8] = {vb[0].x, vb[0].y, vb[0].z, vb[0].w, vb[1].x, vb[1].y, vb[1].z, vb[1].w};
        const uint32_t wc[8] = {vc[0].x, vc[0].y, vc[0].z, vc[0].w, vc[1].x, vc[1].y, vc[1].z, vc[1].w};
        const uint32_t wd[8] = {vd[0].x, vd[0].y, vd[0].z, vd[0].w, vd[1].x, vd[1].y, vd[1].z, vd[1].w};
#pragma unroll
        for (int mt = 0; mt < 8; ++mt)  // word mt holds channels vchan(mt), +1
          mma16816_full(o[mt], __byte_perm(wa[mt], wb[mt], 0x5410u), __byte_perm(wa[mt], wb[mt], 0x7632u),
                        __byte_perm(wc[mt], wd[mt], 0x5410u), __byte_perm(wc[mt], wd[mt], 0x7632u), pb0,
                        pb1);
      }
    }
  };
  // A tile of keys [kb0, kb0 + T) below hi: retrieval keys through the block
  // that holds them (indices local to the block), streaming keys in the slot
  // buffer.
  auto run_tile = [&](int kb0, int hi, int skip_key) {
    int64_t row;
    int base = 0;
    const uint8_t *pk, *pv, *psk, *psv;
    if (retrieval) {
      base = kb0 & kBlockMask;
      row = ret_row(P.ret, b, pidx, base);
      pk = P.p.ret_k, pv = P.p.ret_v, psk = P.p.ret_k_sz, psv = P.p.ret_v_sz;
    } else {
      row = srow0();
      pk = P.p.str_k, pv = P.p.str_v, psk = P.p.str_k_sz, psv = P.p.str_v_sz;
    }
    // 4-bit only: on the bf16 path a second copy of the tile costs more in
    // registers than the bounds tests it saves
    if constexpr (Q4) {
      const int lo_k = kb0 - base, hi_k = hi - base, sk = skip_key < 0 ? -1 : skip_key - base;
      if (lo_k + T <= hi_k && (sk < lo_k || sk >= lo_k + T)) {
        tile(BoolC<true>{}, pk + row * RB, pv + row * RB, psk + row * 4, psv + row * 4, lo_k, hi_k, sk);
        return;
      }
    }
    tile(BoolC<false>{}, pk + row * RB, pv + row * RB, Q4 ? psk + row * 4 : nullptr,
         Q4 ? psv + row * 4 : nullptr, kb0 - base, hi - base, skip_key < 0 ? -1 : skip_key - base);
  };
  bool new_here = owns_new && warp == 0;  // this warp adds the new token at the end
  if (split_head) {
    // The first pool claim is issued during the warp's last tile of its
    // share, so that its latency overlaps that tile.
    const int pool0 = pooled ? nsplit * ts : tiles;
    unsigned *next = P.ws_next + ((int64_t)r * P.n_ret + pidx) * kChunkCounterStride;
    auto visit = [&](int tt) {
      const int kb0 = tt * T;
      const bool has_new = fused && newk >= kb0 && newk < kb0 + T;
      if (has_new) {
        write_new();
        new_here = true;
      }
      run_tile(kb0, keys, has_new ? newk : -1);
    };
    unsigned c = 0;
    int tt = split * ts + warp;
    if (pooled && tt >= t1 && lane == 0) c = atomicAdd(next, 1u);
    for (; tt < t1; tt += NWARPS) {
      if (pooled && tt + NWARPS >= t1 && lane == 0) c = atomicAdd(next, 1u);
      visit(tt);
    }
    c = __shfl_sync(0xffffffffu, c, 0);
    while (pool0 + (int)c < tiles) {
      unsigned nx = 0;  // claim the following tile now; needed only after this one
      if (lane == 0) nx = atomicAdd(next, 1u);
      visit(pool0 + (int)c);
      c = __shfl_sync(0xffffffffu, nx, 0);
    }
  } else {
    for (int kb0 = k0 + warp * T; kb0 < k1; kb0 += Keys<Q4>::STEP)
      run_tile(kb0, k1, owns_new ? newk : -1);
  }
  if (new_here) {
    // the new token, straight from the inputs (key 0 of a one-row buffer)
    const int64_t off = ((int64_t)r * P.Hkv + kvh) * (int64_t)RB;
    tile(BoolC<false>{}, reinterpret_cast<const uint8_t *>(P.knew) + off,
         reinterpret_cast<const uint8_t *>(P.vnew) + off,
         nullptr, nullptr, 0, 1, -1);
  }

  // the next kernel in the stream may start its set-up now
  asm volatile("griddepcontrol.launch_dependents;");

  // ---- per-warp state -> shared memory (queries < G only)
  l += __shfl_xor_sync(0xffffffffu, l, 1);
  l += __shfl_xor_sync(0xffffffffu, l, 2);
  if (Q4) {
    z += __shfl_xor_sync(0xffffffffu, z, 1);
    z += __shfl_xor_sync(0xffffffffu, z, 2);
    cs += __shfl_xor_sync(0xffffffffu, cs, 1);
    cs += __shfl_xor_sync(0xffffffffu, cs, 2);
    z -= 128.f * cs;  // the codes were multiplied as 128 + u
  }
  float *red_m = reinterpret_cast<float *>(smem);
  float *red_l = red_m + NWARPS * G;
  float *red_o = red_l + NWARPS * G;
  // the zero-point sums of this thread's two O^T columns (queries 2t, 2t+1)
  const float z0 = __shfl_sync(0xffffffffu, z, (2 * t) << 2);
  const float z1 = __shfl_sync(0xffffffffu, z, (2 * t + 1) << 2);
  if (live && t == 0) {
    red_m[warp * G + g] = m;
    red_l[warp * G + g] = l;
  }
  const int q0 = 2 * t, q1 = 2 * t + 1;
#pragma unroll
  for (int mt = 0; mt < 8; ++mt) {
    const int ch = vchan(mt);
    if (q0 < G) {
      red_o[(warp * G + q0) * D + ch] = o[mt][0] + z0;
      red_o[(warp * G + q0) * D + ch + 1] = o[mt][2] + z0;
    }
    if (q1 < G) {
      red_o[(warp * G + q1) * D + ch] = o[mt][1] + z1;
      red_o[(warp * G + q1) * D + ch + 1] = o[mt][3] + z1;
    }
  }
  __syncthreads();
  decode_reduce_store<__nv_bfloat16, D, G, NWARPS>(
      P, smem, &s_last, nsplit == 1, (int64_t)r * P.Hq + (int64_t)kvh * G,
      (int64_t)r * P.n_ret + pidx, (int64_t)(retrieval ? P.cta0[r] : 0) + (int64_t)pidx * nsplit,
      nsplit, split);
}

template <bool Q4, int G>
cudaError_t run(const DecodeParams &d, cudaStream_t s, DecodeConfig *cfg) {
  auto kern = decode_mma_kernel<Q4, G>;
  // staging: 2*NWARPS*G + NWARPS*G*D floats; merge: nsplit*G + G (+align) + NWARPS*G*D floats
  const int smem = (int)sizeof(float) * (kMaxSplits * G + 8 + NWARPS * G * D + 2 * NWARPS * G);
  static bool attr_done = false;
  if (!attr_done) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    attr_done = true;
  }
  if (cfg) {
    int occ = 0, dev = 0, sms = 0;
    cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, NWARPS * 32, smem);
    if (e != cudaSuccess) return e;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
    if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
    cfg->tile_rows = Keys<Q4>::STEP;
    cfg->ctas_per_sm = occ;
    cfg->num_sms = sms;
    return cudaSuccess;
  }
  const int grid = d.cta0[d.rows.n] + d.rows.n * d.n_str;
  if (grid == 0) return cudaSuccess;
  if (!d.pdl) {
    kern<<<grid, NWARPS * 32, smem, s>>>(d);
    return cudaGetLastError();
  }
  cudaLaunchConfig_t lc = {};
  lc.gridDim = dim3(grid);
  lc.blockDim = dim3(NWARPS * 32);
  lc.dynamicSmemBytes = smem;
  lc.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  lc.attrs = attr;
  lc.numAttrs = 1;
  return cudaLaunchKernelEx(&lc, kern, d);
}

template <bool Q4>
cudaError_t dispatch(const DecodeParams &d, int G, cudaStream_t s, DecodeConfig *cfg) {
  switch (G) {
    case 1: return run<Q4, 1>(d, s, cfg);
    case 2: return run<Q4, 2>(d, s, cfg);
    case 4: return run<Q4, 4>(d, s, cfg);
    case 8: return run<Q4, 8>(d, s, cfg);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace dm

// head_dim 128, bf16 or 4-bit cache: the tensor-core decode.
bool decode_mma_supported(int kv_type, int D, int G) {
  return D == 128 && (kv_type == kBF16 || kv_type == kINT4) && (G == 1 || G == 2 || G == 4 || G == 8);
}

bool decode_can_fuse_append(int kv_type, int D, int G) {
  return kv_type == kBF16 && decode_mma_supported(kv_type, D, G);
}

cudaError_t decode_mma_config(int kv_type, int G, DecodeConfig *cfg) {
  DecodeParams dummy{};
  return kv_type == kINT4 ? dm::dispatch<true>(dummy, G, nullptr, cfg)
                          : dm::dispatch<false>(dummy, G, nullptr, cfg);
}

cudaError_t launch_decode_mma(const DecodeParams &d, int kv_type, cudaStream_t s) {
  return kv_type == kINT4 ? dm::dispatch<true>(d, d.G, s, nullptr)
                          : dm::dispatch<false>(d, d.G, s, nullptr);
}

}  // namespace duo
