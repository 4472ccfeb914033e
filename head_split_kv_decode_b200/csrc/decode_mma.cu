// Single-token decode attention with warp-level tensor-core MMAs
// (mma.sync m16n8k16, fp32 accumulate), for head_dim 128 and a bf16 or 4-bit
// KV cache.
//
// Work split: split-K over retrieval pages (the last split of a head merges
// the partials), streaming slot buffers one per CTA or several per CTA on
// groups of warps (DecodeParams::str_pack); what changes against the
// CUDA-core decode is the inner product.  Per warp and per 16 keys:
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
// loaded straight from global memory into registers (each warp's next tile
// is prefetched into L2 meanwhile); shared memory holds only the query
// fragments (reloaded per tile rather than held in registers) and the final
// cross-warp combine.
//
// 4-bit cache (f16 operands): a nibble masked into the low bits of a 16-bit
// half, all other bits zero, is the f16 subnormal u * 2^-24 exactly, and one
// at bits 4..7 is 16u * 2^-24; so one AND per register turns packed codes into
// MMA operands, with no offset to remove.  The scores are computed transposed,
// S^T[16 x 8] = K[16 x 128] . Q^T, so that the codes fill the whole A operand
// (16 keys per product) and Q is the two-register B operand; each thread then
// holds two keys for its queries 2t and 2t+1, and P^T for the V product comes
// from S^T by an 8x8 transpose (movmatrix) per 8 keys.  The factor 16 is taken out of the
// query (K side, q/16 on those k-slots) or out of the output channel (V
// side), both exact.  Scale and zero are applied outside the products:
//   s = sc * (q . u) + zp * sum(q),   sum p*x_hat = sum (p*sc) * u + sum p*zp.
// p*sc enters the V product as an f16 pair, high part plus residual (22
// significant bits; one f16 alone, 11 bits, would leave up to 2^-11 of a V
// row's range in the output), relative to a reference m - f: f is a
// power-of-two headroom chosen from the largest V scale seen, so that
// p*sc < 2^15 whatever the data (f16 overflows at 65504); lowering f rescales
// the state exactly.  With the fused step the warp that owns the new token
// quantises it (the append kernel's encoder), writes it to the cache and
// attends to it from shared memory.
//
// Pages: "DuoAttention: Efficient Long-Context LLM Inference with Retrieval and
// Streaming Heads" (hotpaper.ai), abstract and section "기술적 접근법".
#include "common.cuh"
#include "decode_finish.cuh"
#include "quant_int4.cuh"

namespace duo {

namespace dm {

constexpr int D = 128;
constexpr int NWARPS = 16;
// Key groups of 16 per warp iteration: the 4-bit rows are 4x smaller, so a
// warp takes two groups to keep as many bytes in flight as the bf16 path
// (measured: one group plus bulk L2 prefetches of the warp's later tiles is
// slower than two groups in registers).
template <bool Q4>
struct Keys {
  static constexpr int KG = Q4 ? 2 : 1;
  static constexpr int STEP = NWARPS * 16 * KG;  // keys per CTA iteration
};

// 4-bit codes as f16 subnormals: masks of the nibbles at bits 0..3 (value
// u * 2^-24) and 4..7 (16u * 2^-24) of both 16-bit halves.
constexpr uint32_t kNib0 = 0x000F000Fu, kNib1 = 0x00F000F0u;
constexpr float kTwo24 = 16777216.f, kTwo20 = 1048576.f;

__device__ __forceinline__ void mma16816(float (&d)[4], uint32_t a0, uint32_t a2, uint32_t b0,
                                         uint32_t b1) {
  // rows g+8 of A are zero (a1 = a3 = 0)
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(0u), "r"(a2), "r"(0u), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void mma16816_f16(float (&d)[4], uint32_t a0, uint32_t a2, uint32_t b0,
                                             uint32_t b1) {
  // f16 operands; rows g+8 of A are zero
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
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

// Loads of the 4-bit tile: read-only global memory, or (GEN) any address
// space through a generic pointer (the new token staged in shared memory).
template <bool GEN>
__device__ __forceinline__ uint4 ld16(const uint8_t *p) {
  if constexpr (GEN) return *reinterpret_cast<const uint4 *>(p);
  else return ldg128(p);
}

template <bool GEN>
__device__ __forceinline__ uint2 ld8(const uint8_t *p) {
  if constexpr (GEN) return *reinterpret_cast<const uint2 *>(p);
  else return ldg64(p);
}

template <bool GEN>
__device__ __forceinline__ uint32_t ld4(const uint8_t *p) {
  if constexpr (GEN) return *reinterpret_cast<const uint32_t *>(p);
  uint32_t v;
  asm volatile("ld.global.nc.L1::no_allocate.u32 %0, [%1];" : "=r"(v) : "l"(p));
  return v;
}

template <int N>
struct IntC {
  static constexpr int value = N;
};

// Transpose of an 8x8 matrix of 16-bit elements held as the warp's
// fragments (thread 4i+j holds row i, columns 2j and 2j+1).
__device__ __forceinline__ uint32_t movm_trans(uint32_t a) {
  uint32_t d;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(d) : "r"(a));
  return d;
}

// Fetch [ptr, ptr + bytes) into L2 (16-byte aligned, bytes a multiple of 16).
__device__ __forceinline__ void prefetch_l2(const void *ptr, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(ptr), "r"(bytes) : "memory");
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t *>(&h);
}

__device__ __forceinline__ uint32_t pack_f16(float lo, float hi) {
  __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t *>(&h);
}

__device__ __forceinline__ float2 half2_bits_to_f2(uint32_t w) {
  return __half22float2(*reinterpret_cast<const __half2 *>(&w));
}

// 2^e for an integer e in [-126, 127], exactly.
__device__ __forceinline__ float exp2i(int e) { return __int_as_float((127 + e) << 23); }

__device__ __forceinline__ void mma16816_full(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                              uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void mma16816_full_f16(float (&d)[4], uint32_t a0, uint32_t a1,
                                                  uint32_t a2, uint32_t a3, uint32_t b0,
                                                  uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

template <bool Q4, int G>
__global__ void __launch_bounds__(NWARPS * 32, 1) decode_mma_kernel(const __grid_constant__ DecodeParams P) {
  extern __shared__ __align__(16) uint8_t smem[];
  __shared__ int s_last;
  // 4-bit fused step: the new token of the head as quantised by its owning
  // warp: K codes [0, 64), V codes [64, 128), K (scale, zero) at 128 and V's
  // at 136, each padded to 8 bytes
  __shared__ __align__(16) uint8_t s_new[Q4 ? kMaxStrPack * 144 : 16];  // one slot per warp group
  // The query fragments of each warp group's head, the same in every warp of
  // the group (they depend on the lane only), as [group][4][32 lanes][4
  // words]: the tile reloads them instead of holding 16 registers through it
  // (on the bf16 path that removed every register spill of the kernel)
  __shared__ __align__(16) uint32_t s_q[kMaxStrPack * 4 * 32 * 4];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, t = lane & 3;  // mma fragment coordinates

  // ---- work item: retrieval CTAs first (launch row r, head, split), then
  // per launch row the streaming CTAs, each holding str_pack streaming heads
  // (heads i*str_pack .. i*str_pack + str_pack - 1 of the row), one per group
  // of wph = NWARPS/str_pack warps.  A warp's head (pidx, kvh) is the same
  // across its group; wsub is the warp's rank in the group.
  const int n_ret_ctas = P.cta0[P.rows.n];
  // (recomputed in the epilogue rather than held through the main loop)
  auto str_group = [&](int &r_, int &pidx0_, int &wph_) {
    const int x = (int)blockIdx.x - n_ret_ctas;
    const int hp = max(P.str_pack, 1);
    const int per_row = (P.n_str + hp - 1) / hp;
    r_ = x / per_row;
    pidx0_ = (x % per_row) * hp;
    wph_ = NWARPS / hp;
  };
  int r, kvh, pidx, split, nsplit;
  int wph = NWARPS, wsub = warp;
  bool retrieval, idle = false;
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
    int pidx0;
    str_group(r, pidx0, wph);
    wsub = warp % wph;
    pidx = pidx0 + warp / wph;
    idle = pidx >= P.n_str;  // a group past the row's last head: no keys, no output
    if (idle) pidx = P.n_str - 1;
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
                             : (idle ? 0 : min(n, P.W));
  const bool new_here_shard = !retrieval || (n - 1 >= P.shard_lo && n - 1 < P.shard_hi);
  constexpr int RB = Q4 ? D / 2 : D * 2;  // bytes per key row
  // this lane's query fragments in s_q, and (4-bit) the offset of the
  // new-token slot in s_new, of its group's head
  const uint32_t sq = smem_u32(s_q) + (uint32_t)(((warp / wph) * 128 + lane) * 16);
  const int snew = Q4 ? (warp / wph) * 144 : 0;
  // Streaming heads: one slot buffer, first storage row srow0.  Retrieval
  // heads: key tiles are addressed block by block (a tile never crosses a
  // block of the paged layout), with key indices local to the block.
  auto srow0 = [&]() { return ((int64_t)b * P.n_str + pidx) * P.Ws; };
  const int k0 = 0, k1 = keys;
  constexpr int KG = Keys<Q4>::KG;
  constexpr int T = 16 * KG;  // keys per warp tile
  constexpr int kBlockMask = ~(kPageTokens - 1);
  // A retrieval head with several splits is cut into tiles of T keys.  Each
  // split walks a fixed share of them; with P.pool the shares cover 13/16 of
  // the tiles (4-bit: 7/8) and the rest is claimed one tile at a time by
  // warps that have finished (see below), so a CTA that gets less memory
  // bandwidth takes fewer tiles and the splits finish together.  (The 4-bit
  // path keeps the smaller pool: its pool tiles miss the register-pipelined
  // walk of the fixed share.)  Each CTA leaves one partial.  Streaming heads
  // and single-split heads walk [k0, k1).
  const bool split_head = retrieval && nsplit > 1;
  const bool pooled = split_head && P.pool;
  const int tiles = (keys + T - 1) / T;
  const int ts = !split_head ? 0
                 : pooled    ? (tiles - (Q4 ? tiles / 8 : 3 * tiles / 16)) / nsplit
                             : (tiles + nsplit - 1) / nsplit;  // tiles per split share
  const int t1 = min(tiles, (split + 1) * ts);                 // end of this split's share
  // this warp's first two tiles, [first, first + T) and the one NWARPS (a
  // streaming group: wph) tiles on
  const int first = split_head ? (split * ts + warp) * T : k0 + wsub * T;
  const int last = split_head ? min(keys, t1 * T) : k1;

  // Bring rows [kb, min(kb + T, last)) of this head (one tile, inside one
  // block) into L2 with bulk prefetches (lane 0 of the calling warp).  A
  // block-table entry may be read here before the wait below; it only aims a
  // prefetch, and is clamped to the pool so the address stays valid.
  auto prefetch_tile = [&](int kb) {
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
  };
  // Launched with programmatic dependent launch, so this may run while the
  // previous kernel in the stream finishes.  Bring this warp's first two
  // tiles into L2 meanwhile: every global write lands in L2, so a line
  // fetched now cannot be stale when the loads below (after the wait) use it.
  if (lane == 0) {
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const int kb = first + i * wph * T;
      if (kb < last) prefetch_tile(kb);
    }
  }
  // Nothing the previous kernel may have written is read before this.
  asm volatile("griddepcontrol.wait;" ::: "memory");

  // Fused append: the token at position n-1 is not in the cache yet.  One
  // warp (see owns_new) writes it there and adds the key at the end from the
  // inputs (bf16) or from its shared-memory copy (4-bit); the tile walk skips
  // that row.
  // In partial mode a rank that does not own the streaming heads leaves
  // their rows empty (another shard contributes them).
  if (P.part_o && !retrieval && !P.own_str) {
    int r_, pidx0, wph_;
    str_group(r_, pidx0, wph_);
    for (int hs = 0; hs < NWARPS / wph_ && pidx0 + hs < P.n_str; ++hs) {
      const int64_t row0 = (int64_t)r * P.Hq + (int64_t)P.h.str_heads[pidx0 + hs] * G;
      for (int i = tid; i < G * D; i += NWARPS * 32) P.part_o[row0 * D + i] = 0.f;
      if (tid < G) P.part_lse[row0 + tid] = -INFINITY;
    }
    return;
  }
  const bool fused = P.knew != nullptr && new_here_shard;
  const int newk = retrieval ? n - 1 - (int)P.shard_lo : (int)ring_slot(n - 1, P.S, P.R);  // its row
  // The new token is written and attended by warp 0 of the CTA (of the
  // head's group) that walks its row, or for a split head by warp 0 of split
  // 0, at the start: the tile
  // that holds the row comes last and is claimed from the pool, so doing the
  // work (4-bit: quantisation) there would put it on the launch's critical
  // path.  Whichever warp visits that tile skips the row.
  const bool owns_new = fused && (split_head ? split == 0 : (newk >= k0 && newk < k1));
  // its K/V in the inputs (bf16); recomputed where used rather than held
  // through the main loop
  auto in_off = [&]() { return ((int64_t)r * P.Hkv + kvh) * (int64_t)(D * 2); };
  auto write_new = [&]() {  // one warp writes the new K and V rows into the cache
    const int64_t row = retrieval ? ret_row(P.ret, b, pidx, newk) : srow0() + newk;
    if constexpr (Q4) {
      // lane l quantises channels 4l .. 4l+3 of each row, as the append does
#pragma unroll
      for (int which = 0; which < 2; ++which) {
        const uint2 raw = ldg64(reinterpret_cast<const uint8_t *>(which ? P.vnew : P.knew) + in_off() + 8 * lane);
        const float x[4] = {__uint_as_float(raw.x << 16), __uint_as_float(raw.x & 0xffff0000u),
                            __uint_as_float(raw.y << 16), __uint_as_float(raw.y & 0xffff0000u)};
        __half sch, zph;
        const uint32_t packed = quantize_row_int4<4>(x, &sch, &zph);
        uint8_t *codes = which ? (retrieval ? P.p.ret_v : P.p.str_v) : (retrieval ? P.p.ret_k : P.p.str_k);
        uint8_t *sz = which ? (retrieval ? P.p.ret_v_sz : P.p.str_v_sz)
                            : (retrieval ? P.p.ret_k_sz : P.p.str_k_sz);
        *reinterpret_cast<uint16_t *>(codes + row * RB + 2 * lane) = (uint16_t)packed;
        *reinterpret_cast<uint16_t *>(s_new + snew + 64 * which + 2 * lane) = (uint16_t)packed;
        if (lane == 0) {
          __half2 pair;
          pair.x = sch;
          pair.y = zph;
          reinterpret_cast<__half2 *>(sz)[row] = pair;
          *reinterpret_cast<uint2 *>(s_new + snew + 128 + 8 * which) =
              make_uint2(*reinterpret_cast<const uint32_t *>(&pair), 0u);
        }
      }
      __syncwarp();
    } else {
      const int c = lane & 15;  // 16 lanes x 16 bytes = one 256-byte row
      const uint8_t *src = reinterpret_cast<const uint8_t *>(lane < 16 ? P.knew : P.vnew) + in_off();
      uint8_t *dst = (lane < 16 ? (retrieval ? P.p.ret_k : P.p.str_k)
                                : (retrieval ? P.p.ret_v : P.p.str_v)) + row * RB;
      reinterpret_cast<uint4 *>(dst)[c] = ldg128(src + 16 * c);
    }
  };
  if (owns_new && wsub == 0) write_new();

  // ---- query fragments (rows g < G), k-step order matching the K loads
  uint32_t qa[8][2];
  float qsum = 0.f;  // sum of the query's channels (4-bit zero-point term)
  const bool live = g < G;
  const float sl2 = P.scale_log2;
  // 4-bit: score (log2 units) = raw * (sc * c1) + zp * c2, raw = the MMA sum;
  // c2q: c2 of the queries 2t, 2t+1 this thread scores
  float c1 = sl2, c2 = 0.f, c2q[2] = {0.f, 0.f};
  {
    const __nv_bfloat16 *qrow =
        reinterpret_cast<const __nv_bfloat16 *>(P.q) + ((int64_t)r * P.Hq + (int64_t)kvh * G + g) * D;
    if constexpr (Q4) {
      // Thread column t holds channels 32t .. 32t+31 of its key rows: word w
      // of the 16-byte load covers 32t + 8w .. +7, and k-steps 2w and 2w+1
      // take its four registers: (c0, c4), (c1, c5)x16, (c2, c6), (c3, c7)x16
      // (see kNib0 / kNib1); the x16 slots get q/16.
      float qv[32];
      float amax = 0.f;
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        qv[i] = live ? __bfloat162float(qrow[32 * t + i]) : 0.f;
        amax = fmaxf(amax, fabsf(qv[i]));
        qsum += qv[i];
      }
      qsum += __shfl_xor_sync(0xffffffffu, qsum, 1);
      qsum += __shfl_xor_sync(0xffffffffu, qsum, 2);
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
      // one power of two for all the CTA's queries keeps |q| below 2^15 in
      // f16 (taken back in c1)
      const int ex = ((__float_as_int(amax) >> 23) & 0xff) - 127;
      const int eq = ex > 14 ? ex - 14 : 0;
      const float qs = exp2i(-eq), qs16 = qs * 0.0625f;
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        const float *c = qv + 8 * w;
        qa[2 * w][0] = pack_f16(c[0] * qs, c[4] * qs);
        qa[2 * w][1] = pack_f16(c[1] * qs16, c[5] * qs16);
        qa[2 * w + 1][0] = pack_f16(c[2] * qs, c[6] * qs);
        qa[2 * w + 1][1] = pack_f16(c[3] * qs16, c[7] * qs16);
      }
      c1 = sl2 * kTwo24 * exp2i(eq);
      c2 = qsum * sl2;
      // S^T: this thread scores queries 2t and 2t+1
      c2q[0] = __shfl_sync(0xffffffffu, c2, (2 * t) << 2);
      c2q[1] = __shfl_sync(0xffffffffu, c2, (2 * t + 1) << 2);
      if (wsub == 0) {
#pragma unroll
        for (int j = 0; j < 4; ++j)
          *reinterpret_cast<uint4 *>(&s_q[((warp / wph) * 128 + j * 32 + lane) * 4]) =
              make_uint4(qa[2 * j][0], qa[2 * j][1], qa[2 * j + 1][0], qa[2 * j + 1][1]);
      }
      __syncthreads();
    } else {
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        // channels behind k-slots 2t, 2t+1, 2t+8, 2t+9
        const int s = k >> 1, tt = k & 1;
        const int c0 = 32 * s + 8 * t + 4 * tt;
        const float q0 = live ? __bfloat162float(qrow[c0]) : 0.f;
        const float q1 = live ? __bfloat162float(qrow[c0 + 1]) : 0.f;
        const float q2 = live ? __bfloat162float(qrow[c0 + 2]) : 0.f;
        const float q3 = live ? __bfloat162float(qrow[c0 + 3]) : 0.f;
        qa[k][0] = pack_bf16(q0, q1);  // exact: the inputs are bf16
        qa[k][1] = pack_bf16(q2, q3);
      }
      if (wsub == 0) {
#pragma unroll
        for (int j = 0; j < 4; ++j)
          *reinterpret_cast<uint4 *>(&s_q[((warp / wph) * 128 + j * 32 + lane) * 4]) =
              make_uint4(qa[2 * j][0], qa[2 * j][1], qa[2 * j + 1][0], qa[2 * j + 1][1]);
      }
      __syncthreads();
    }
  }

  // O^T accumulators: tile mt holds channels vchan(mt) (rows g) and
  // vchan(mt) + 1 (rows g+8) for queries 2t and 2t+1.  bf16: the thread's V
  // channels are the 16-byte chunks g and 8+g of a row (so the eight lanes of
  // a key read 128 contiguous bytes); 4-bit: code bytes 8g..8g+7, and the
  // rows g+8 accumulate 16x (the nibble at bits 4..7).
  auto vchan = [&](int mt) {
    return Q4 ? 16 * g + 2 * mt : 64 * (mt >> 2) + 8 * g + 2 * (mt & 3);
  };
  float o[8][4];
#pragma unroll
  for (int i = 0; i < 8; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
  // bf16: softmax state of query g (identical in the four threads of a row).
  // 4-bit: state of queries 2t and 2t+1 (m the same in the eight threads of a
  // column; l and the zero-point sums z partial over this thread's keys), p
  // taken relative to m - f (f: headroom exponent, the same in every lane; at
  // most 20, which the smallest scales allow)
  float m = -INFINITY, l = 0.f;
  float mq[2] = {-INFINITY, -INFINITY}, lq[2] = {0.f, 0.f}, zq[2] = {0.f, 0.f};
  int f = 20;
  // 4-bit with at most 4 queries per KV head: the residual of p*sc rides in the
  // idle query columns 4..7 of the V product (see q4_update)
  constexpr bool kLoInN = Q4 && G <= 4;

  // bf16 cache, one warp: keys [kb0, kb0 + 16) below hi of the buffers Kx/Vx,
  // row index = key, except `skip_key`.  `full` (a compile-time flag)
  // promises that all keys of the tile lie below hi and none is skip_key, so
  // no load or score needs a bounds test.
  auto tile = [&](auto full, const uint8_t *Kx, const uint8_t *Vx, int kb0, int hi, int skip_key) {
    constexpr bool FULL = decltype(full)::value;
    // ------------------------------------------------------------ loads (all up front)
    // K of key kb0 + 8*nt + g (this thread's column of S); V of keys
    // kb0 + {2t, 2t+1, 8+2t, 9+2t} (the k-slots of the P^T fragment) at this
    // thread's channels (see vchan).
    uint4 kr[2][4];
    uint4 vr[4][2];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
      const int key = kb0 + 8 * nt + g;
      const bool ok = FULL || (key < hi && key != skip_key);
#pragma unroll
      for (int sp = 0; sp < 4; ++sp)
        kr[nt][sp] = ok ? ldg128(Kx + key * RB + (32 * sp + 8 * t) * 2) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int key = kb0 + 2 * t + (i & 1) + 8 * (i >> 1);
      const bool ok = FULL || (key < hi && key != skip_key);
#pragma unroll
      for (int h = 0; h < 2; ++h)
        vr[i][h] = ok ? ldg128(Vx + key * RB + 16 * (8 * h + g)) : make_uint4(0, 0, 0, 0);
    }
    // ------------------------------------------------------------ S = Q K^T
    // (query fragments from s_q, one 16-byte load per two k-steps for both
    // halves of the tile)
    float sc[2][2];
    float s2[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
    for (int sp = 0; sp < 4; ++sp) {
      const uint4 qf = lds128(sq + 512u * sp);  // k-steps 2sp, 2sp+1
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
        mma16816(s2[nt], qf.x, qf.y, kr[nt][sp].x, kr[nt][sp].y);
        mma16816(s2[nt], qf.z, qf.w, kr[nt][sp].z, kr[nt][sp].w);
      }
    }
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
      float(&s)[4] = s2[nt];
      // scores of query g at keys kb0 + 8*nt + 2t + e
      const int key = kb0 + 8 * nt + 2 * t;
#pragma unroll
      for (int e = 0; e < 2; ++e)
        sc[nt][e] = (live && (FULL || (key + e < hi && key + e != skip_key))) ? s[e] * sl2 : -INFINITY;
    }
    // ------------------------------------------------------------ online softmax
    float mx = fmaxf(fmaxf(sc[0][0], sc[0][1]), fmaxf(sc[1][0], sc[1][1]));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
    // Rescale only when the running max grows by more than 2^8 (numerator and
    // denominator scale together, so the result is unchanged).
    const bool grow = mx > m + 8.f || (m == -INFINITY && mx > -INFINITY);
    float alpha = 1.f;
    if (grow) {
      alpha = (m == -INFINITY) ? 0.f : fast_exp2(m - mx);
      l *= alpha;
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
    float p[2][2];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        p[nt][e] = (sc[nt][e] == -INFINITY) ? 0.f : fast_exp2(sc[nt][e] - m);
        l += p[nt][e];
      }
    // P^T fragment: b0 = keys 2t, 2t+1 (tile 0), b1 = keys 8+2t, 9+2t (tile 1)
    const uint32_t pb0 = pack_bf16(p[0][0], p[0][1]);
    const uint32_t pb1 = pack_bf16(p[1][0], p[1][1]);
    // ---------------------------------------------------------- O^T += V^T P^T
    const uint4 *va = vr[0], *vb = vr[1], *vc = vr[2], *vd = vr[3];
    const uint32_t wa[8] = {va[0].x, va[0].y, va[0].z, va[0].w, va[1].x, va[1].y, va[1].z, va[1].w};
    const uint32_t wb[8] = {vb[0].x, vb[0].y, vb[0].z, vb[0].w, vb[1].x, vb[1].y, vb[1].z, vb[1].w};
    const uint32_t wc[8] = {vc[0].x, vc[0].y, vc[0].z, vc[0].w, vc[1].x, vc[1].y, vc[1].z, vc[1].w};
    const uint32_t wd[8] = {vd[0].x, vd[0].y, vd[0].z, vd[0].w, vd[1].x, vd[1].y, vd[1].z, vd[1].w};
#pragma unroll
    for (int mt = 0; mt < 8; ++mt)  // word mt holds channels vchan(mt), +1
      mma16816_full(o[mt], __byte_perm(wa[mt], wb[mt], 0x5410u), __byte_perm(wa[mt], wb[mt], 0x7632u),
                    __byte_perm(wc[mt], wd[mt], 0x5410u), __byte_perm(wc[mt], wd[mt], 0x7632u), pb0,
                    pb1);
  };

  // 4-bit cache, one warp: keys [kb0, kb0 + 32) below hi, except `skip_key`.
  // The pointers are this thread's own starting points in the tile: K codes
  // at the tile's first row + g rows + 16t bytes, V codes at + 2t rows + 8g
  // bytes, (scale, zero) rows at + g rows; every load of the tile is then an
  // immediate offset from one of them.  `full` as above; `gen` reads through
  // generic pointers (the staged new token).
  // Registers of one 4-bit tile: K codes and (scale, zero) of keys
  // kb + 8*h + g (this thread's rows of S^T; codes at bytes 16t..16t+15,
  // channels 32t..32t+31); V codes of keys kb + {2t, 2t+1, 8+2t, 9+2t} at
  // bytes 8g..8g+7 (channels 16g..16g+15); group kg covers keys
  // kb = kb0 + 16*kg.  The K part is dead once the scores are computed, the
  // V part once O is updated, so a pipelined walk refills each as it dies.
  uint4 kr[KG][2];
  uint32_t ksz[KG][2], vsz[KG][2];
  uint2 vr[KG][4];
  // Loads of a 4-bit tile, keys [kb0, kb0 + 32) below hi except `skip_key`.
  // The pointers are this thread's own starting points in the tile: K codes
  // at the tile's first row + g rows + 16t bytes, V codes at + 2t rows + 8g
  // bytes, (scale, zero) rows at + g rows; every load of the tile is then an
  // immediate offset from one of them.  `full` promises that all keys lie
  // below hi and none is skip_key; `src` 1 reads through generic pointers
  // (the staged new token), 0 through the read-only global path.
  auto q4_load_k = [&](auto full, auto src, const uint8_t *Kt, const uint8_t *Kst, int kb0, int hi,
                       int skip_key) {
    constexpr bool FULL = decltype(full)::value;
    constexpr bool GEN = decltype(src)::value == 1;
#pragma unroll
    for (int kg = 0; kg < KG; ++kg)
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int r0 = 16 * kg + 8 * h;  // tile row of this thread's group
        const int key = kb0 + r0 + g;
        const bool ok = FULL || (key < hi && key != skip_key);
        kr[kg][h] = ok ? ld16<GEN>(Kt + r0 * RB) : make_uint4(0, 0, 0, 0);
        ksz[kg][h] = (FULL || key < hi) ? ld4<GEN>(Kst + r0 * 4) : 0u;
      }
  };
  auto q4_load_v = [&](auto full, auto src, const uint8_t *Vt, const uint8_t *Vst, int kb0, int hi,
                       int skip_key) {
    constexpr bool FULL = decltype(full)::value;
    constexpr bool GEN = decltype(src)::value == 1;
#pragma unroll
    for (int kg = 0; kg < KG; ++kg) {
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int r0 = 16 * kg + 8 * h;
        vsz[kg][h] = (FULL || kb0 + r0 + g < hi) ? ld4<GEN>(Vst + r0 * 4) : 0u;
      }
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int r0 = 16 * kg + (i & 1) + 8 * (i >> 1);
        const int key = kb0 + 16 * kg + 2 * t + (i & 1) + 8 * (i >> 1);
        const bool ok = FULL || (key < hi && key != skip_key);
        vr[kg][i] = ok ? ld8<GEN>(Vt + r0 * RB) : make_uint2(0, 0);
      }
    }
  };
  // Scores of the loaded tile (S^T = K Q^T, log2 units; -inf where not
  // visible) and the tile's headroom exponent.
  float sc[KG][2][2];  // [group][key g / 8+g][query 2t / 2t+1]
  int ftile = 0;
  auto q4_scores = [&](auto full, int kb0, int hi, int skip_key) {
    constexpr bool FULL = decltype(full)::value;
    // ------------------------------------------------------------ headroom
    // The largest V scale of the tile bounds p*sc: with p < 2^(8+f) (the lazy
    // rescale below) and sc < 2^(E-14) for an fp16 exponent field E >= 1,
    // f = 21 - E keeps p*sc < 2^15.  Positive fp16 values order as integers.
    // The warp-wide maximum is needed only when some lane's own scales ask
    // for less headroom than f has (rare after the first tiles).
    uint32_t vm = 0;
#pragma unroll
    for (int kg = 0; kg < KG; ++kg) vm = max(vm, max(vsz[kg][0] & 0xffffu, vsz[kg][1] & 0xffffu));
    ftile = f;
    if (__any_sync(0xffffffffu, 21 - max((int)(vm >> 10), 1) < f)) {
#pragma unroll
      for (int off = 4; off < 32; off <<= 1) vm = max(vm, __shfl_xor_sync(0xffffffffu, vm, off));
      ftile = 21 - max((int)(vm >> 10), 1);
    }
    // ------------------------------------------------------------ S^T = K Q^T
    // A rows g / g+8 are keys kb + g / kb + 8 + g; k-slots follow the channel
    // order of the query fragments (see the set-up)
    // Per key group two accumulators (channels 32t..32t+15 and +16..+31)
    // halve the chains of dependent products; each query fragment is loaded
    // once for both groups.
    float acc[KG][2][4];
#pragma unroll
    for (int kg = 0; kg < KG; ++kg)
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[kg][0][i] = acc[kg][1][i] = 0.f;
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      const uint4 qf = lds128(sq + 512u * w);  // k-steps 2w, 2w+1
#pragma unroll
      for (int kg = 0; kg < KG; ++kg) {
        const uint32_t x0 = (&kr[kg][0].x)[w], x1 = (&kr[kg][1].x)[w], y0 = x0 >> 8, y1 = x1 >> 8;
        float(&a)[4] = acc[kg][w >> 1];
        mma16816_full_f16(a, x0 & kNib0, x1 & kNib0, x0 & kNib1, x1 & kNib1, qf.x, qf.y);
        mma16816_full_f16(a, y0 & kNib0, y1 & kNib0, y0 & kNib1, y1 & kNib1, qf.z, qf.w);
      }
    }
#pragma unroll
    for (int kg = 0; kg < KG; ++kg) {
      const int kb = kb0 + 16 * kg;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const float2 kp = half2_bits_to_f2(ksz[kg][h]);  // (scale, zero)
        const float a = kp.x * c1;
        const int key = kb + 8 * h + g;
        const bool valid = FULL || (key < hi && key != skip_key);
#pragma unroll
        for (int e = 0; e < 2; ++e)
          sc[kg][h][e] =
              valid ? fmaf(acc[kg][0][2 * h + e] + acc[kg][1][2 * h + e], a, kp.y * c2q[e]) : -INFINITY;
      }
    }
  };
  // Online softmax of the scored tile, then O^T += V^T P^T.
  auto q4_update = [&](auto full) {
    constexpr bool FULL = decltype(full)::value;
    // Rescale when a running max grows by more than 2^8 or the headroom must
    // shrink (numerator and denominator scale together).  A column's maximum
    // over its eight key rows is needed only if some lane's own maximum
    // passes m + 8 (with m = -inf, any finite score does).
    float mx[2];
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      float x = -INFINITY;
#pragma unroll
      for (int kg = 0; kg < KG; ++kg) x = fmaxf(x, fmaxf(sc[kg][0][e], sc[kg][1][e]));
      mx[e] = x;
    }
    const bool shrink = ftile < f;  // the same in every lane
    if (__any_sync(0xffffffffu, mx[0] > mq[0] + 8.f || mx[1] > mq[1] + 8.f) || shrink) {
      bool grow[2];
#pragma unroll
      for (int e = 0; e < 2; ++e) {
#pragma unroll
        for (int off = 4; off < 32; off <<= 1) mx[e] = fmaxf(mx[e], __shfl_xor_sync(0xffffffffu, mx[e], off));
        grow[e] = mx[e] > mq[e] + 8.f;
      }
      float alpha[2];
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        alpha[e] = 1.f;
        if (grow[e]) {
          alpha[e] = (mq[e] == -INFINITY) ? 0.f : fast_exp2(mq[e] - mx[e]);
          mq[e] = mx[e];
        }
        if (shrink) alpha[e] *= exp2i(ftile - f);
        lq[e] *= alpha[e];
        zq[e] *= alpha[e];
        // the residual columns (lanes t >= 2) scale with their live columns
        if (kLoInN) {
          const float other = __shfl_xor_sync(0xffffffffu, alpha[e], 2);
          if (t >= 2) alpha[e] = other;
        }
      }
      if (shrink) f = ftile;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        o[i][0] *= alpha[0];
        o[i][2] *= alpha[0];
        o[i][1] *= alpha[1];
        o[i][3] *= alpha[1];
      }
    }
    const float ref[2] = {mq[0] - (float)f, mq[1] - (float)f};
#pragma unroll
    for (int kg = 0; kg < KG; ++kg) {
      // p*sc per (key, query) as an f16 high part and residual, packed per key
      // row of P (queries 2t, 2t+1), then transposed to P^T fragments.  With
      // G <= 4 the query columns 4..7 are idle, so lanes t = 2, 3 take the
      // live columns' p*sc from lanes t = 0, 1 and contribute the residuals
      // there: one product gives the high sums in columns 0..3 and the
      // residual sums in 4..7, added once at the end.
      uint32_t ph[2], pl[2] = {0u, 0u};
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const float2 vp = half2_bits_to_f2(vsz[kg][h]);  // (scale, zero)
        float pv[2];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const float x = sc[kg][h][e];
          // a full tile has finite scores in every column, so ref is finite
          const float p = (FULL || x != -INFINITY) ? fast_exp2(x - ref[e]) : 0.f;
          lq[e] += p;
          zq[e] = fmaf(p, vp.y, zq[e]);
          pv[e] = p * vp.x;
        }
        if constexpr (kLoInN) {
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const float other = __shfl_xor_sync(0xffffffffu, pv[e], 2);
            if (t >= 2) pv[e] = other;
          }
          const uint32_t hi = pack_f16(pv[0], pv[1]);
          const float2 hf = half2_bits_to_f2(hi);
          const uint32_t lo = pack_f16(pv[0] - hf.x, pv[1] - hf.y);
          ph[h] = t < 2 ? hi : lo;
        } else {
          ph[h] = pack_f16(pv[0], pv[1]);
          const float2 hf = half2_bits_to_f2(ph[h]);
          pl[h] = pack_f16(pv[0] - hf.x, pv[1] - hf.y);
        }
      }
      // P^T fragment: b0 = keys 2t, 2t+1, b1 = keys 8+2t, 9+2t, of column g
      const uint32_t pb0 = movm_trans(ph[0]), pb1 = movm_trans(ph[1]);
      uint32_t pl0 = 0u, pl1 = 0u;
      (void)pl;
      if constexpr (!kLoInN) {
        pl0 = movm_trans(pl[0]);
        pl1 = movm_trans(pl[1]);
      }
      // ---------------------------------------------------------- O^T += V^T P^T
      // A rows g / g+8 are channels vchan(mt) / vchan(mt)+1; cols are keys
      // (2t, 2t+1) from ab and (8+2t, 9+2t) from cd, two bytes (4 channels)
      // of each key per byte_perm.
#pragma unroll
      for (int wi = 0; wi < 2; ++wi) {
        const uint32_t xa = wi ? vr[kg][0].y : vr[kg][0].x, xb = wi ? vr[kg][1].y : vr[kg][1].x;
        const uint32_t xc = wi ? vr[kg][2].y : vr[kg][2].x, xd = wi ? vr[kg][3].y : vr[kg][3].x;
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          const uint32_t sel = hh ? 0x7632u : 0x5410u;
          const uint32_t ab = __byte_perm(xa, xb, sel), cd = __byte_perm(xc, xd, sel);
          const uint32_t ab8 = ab >> 8, cd8 = cd >> 8;
          const int mt = 4 * wi + 2 * hh;
          const uint32_t a0 = ab & kNib0, a1 = ab & kNib1, a2 = cd & kNib0, a3 = cd & kNib1;
          mma16816_full_f16(o[mt], a0, a1, a2, a3, pb0, pb1);
          if (!kLoInN) mma16816_full_f16(o[mt], a0, a1, a2, a3, pl0, pl1);
          const uint32_t b0 = ab8 & kNib0, b1 = ab8 & kNib1, b2 = cd8 & kNib0, b3 = cd8 & kNib1;
          mma16816_full_f16(o[mt + 1], b0, b1, b2, b3, pb0, pb1);
          if (!kLoInN) mma16816_full_f16(o[mt + 1], b0, b1, b2, b3, pl0, pl1);
        }
      }
    }
  };
  // One 4-bit tile (pointers as for the loads).
  auto tile_q4 = [&](auto full, auto src, const uint8_t *Kt, const uint8_t *Vt, const uint8_t *Kst,
                     const uint8_t *Vst, int kb0, int hi, int skip_key) {
    q4_load_k(full, src, Kt, Kst, kb0, hi, skip_key);
    q4_load_v(full, src, Vt, Vst, kb0, hi, skip_key);
    q4_scores(full, kb0, hi, skip_key);
    q4_update(full);
  };

  // A tile of keys [kb0, kb0 + T) below hi: retrieval keys through the block
  // that holds them (indices local to the block), streaming keys in the slot
  // buffer.
  // this thread's offsets within a 4-bit tile (see tile_q4)
  const int k_off = g * RB + 16 * t, v_off = 2 * t * RB + 8 * g, s_off = 4 * g;
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
    const int lo_k = kb0 - base, hi_k = hi - base, sk = skip_key < 0 ? -1 : skip_key - base;
    if constexpr (Q4) {
      // tiles wholly inside the visible range skip every bounds test (4-bit
      // only: on the bf16 path a second copy costs more in registers than the
      // tests it saves)
      const int64_t r = row + lo_k;  // the tile's first storage row
      const uint8_t *Kt = pk + r * RB + k_off, *Vt = pv + r * RB + v_off;
      const uint8_t *Kst = psk + r * 4 + s_off, *Vst = psv + r * 4 + s_off;
      if (lo_k + T <= hi_k && (sk < lo_k || sk >= lo_k + T))
        tile_q4(BoolC<true>{}, IntC<0>{}, Kt, Vt, Kst, Vst, lo_k, hi_k, sk);
      else
        tile_q4(BoolC<false>{}, IntC<0>{}, Kt, Vt, Kst, Vst, lo_k, hi_k, sk);
    } else {
      tile(BoolC<false>{}, pk + row * RB, pv + row * RB, lo_k, hi_k, sk);
    }
  };
  bool new_here = owns_new && wsub == 0;  // this warp adds the new token at the end
  if (split_head) {
    // The first pool claim is issued during the warp's last tile of its
    // share, so that its latency overlaps that tile.
    const int pool0 = pooled ? nsplit * ts : tiles;
    unsigned *next = P.ws_next + ((int64_t)r * P.n_ret + pidx) * kChunkCounterStride;
    auto visit = [&](int tt) {
      const int kb0 = tt * T;
      const bool has_new = fused && newk >= kb0 && newk < kb0 + T;
      run_tile(kb0, keys, has_new ? newk : -1);
    };
    unsigned c = 0;
    int tt = split * ts + warp;
    if (pooled && tt >= t1 && lane == 0) c = atomicAdd(next, 1u);
    if constexpr (Q4) {
      if (!P.ret.table) {
        // Packed layout: the warp's tiles of its share lie NWARPS tiles apart
        // in one contiguous page, so the walk only advances four pointers.
        // Its full tiles (all but one holding the new token or the page's
        // ragged end, which take the general path) are software-pipelined
        // in the tile's own registers: the next tile's K part is loaded as
        // soon as this tile's scores are computed, its V part as soon as O
        // is updated, so each load has half a tile of work to arrive.
        const int tend = min(t1, (keys - (fused ? 1 : 0)) / T);  // tiles below are full
        const int64_t r0 = ret_row(P.ret, b, pidx, (int64_t)tt * T);
        const uint8_t *Kt = P.p.ret_k + r0 * RB + k_off, *Vt = P.p.ret_v + r0 * RB + v_off;
        const uint8_t *Kst = P.p.ret_k_sz + r0 * 4 + s_off, *Vst = P.p.ret_v_sz + r0 * 4 + s_off;
        constexpr int kStep = NWARPS * T;  // rows between a warp's tiles
        if (tt < tend) {
          q4_load_k(BoolC<true>{}, IntC<0>{}, Kt, Kst, 0, 0, -1);
          q4_load_v(BoolC<true>{}, IntC<0>{}, Vt, Vst, 0, 0, -1);
          for (; tt < tend; tt += NWARPS) {
            // (the pool claim belongs to the last tile of the share: only
            // then can the condition hold)
            if (pooled && tt + NWARPS >= t1) {
              if (lane == 0) c = atomicAdd(next, 1u);
            }
            const bool more = tt + NWARPS < tend;
            q4_scores(BoolC<true>{}, tt * T, keys, -1);
            Kt += kStep * RB;
            Kst += kStep * 4;
            if (more) q4_load_k(BoolC<true>{}, IntC<0>{}, Kt, Kst, 0, 0, -1);
            q4_update(BoolC<true>{});
            Vt += kStep * RB;
            Vst += kStep * 4;
            if (more) q4_load_v(BoolC<true>{}, IntC<0>{}, Vt, Vst, 0, 0, -1);
          }
        }
      }
    }
    for (; tt < t1; tt += NWARPS) {
      if (pooled && tt + NWARPS >= t1 && lane == 0) c = atomicAdd(next, 1u);
      // bf16, packed layout: the warp's next tile goes to L2 while this one
      // is loaded and multiplied (one bulk prefetch; no registers held), so
      // each warp keeps two tiles in flight.  With a block table the
      // prefetch would wait on a table load, and the 4-bit path keeps its
      // next tile in registers instead.
      if (!Q4 && !P.ret.table && lane == 0 && tt + NWARPS < t1) prefetch_tile((tt + NWARPS) * T);
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
    for (int kb0 = k0 + wsub * T; kb0 < k1; kb0 += wph * T)
      run_tile(kb0, k1, owns_new ? newk : -1);
  }
  if (new_here) {
    // the new token: key 0 of a one-row buffer, the inputs (bf16) or the
    // warp's quantised copy in shared memory (4-bit)
    if constexpr (Q4)
      tile_q4(BoolC<false>{}, IntC<1>{}, s_new + snew + k_off, s_new + snew + 64 + v_off,
              s_new + snew + 128 + s_off, s_new + snew + 136 + s_off, 0, 1, -1);
    else
      tile(BoolC<false>{}, reinterpret_cast<const uint8_t *>(P.knew) + in_off(),
           reinterpret_cast<const uint8_t *>(P.vnew) + in_off(), 0, 1, -1);
  }

  // The epilogue's parameter fields (output and workspace pointers), read
  // once after a loop of tens of microseconds and by then out of the uniform
  // cache, are fetched back into it by one thread while the warps stage their
  // states; reading them cold delayed the partial store by up to 3 us.
  if (tid == 0) {
    const char *pp = reinterpret_cast<const char *>(&P);
    asm volatile("prefetchu.L1 [%0];" ::"l"(pp + offsetof(DecodeParams, out)));
    asm volatile("prefetchu.L1 [%0];" ::"l"(pp + offsetof(DecodeParams, Hq)));
    asm volatile("prefetchu.L1 [%0];" ::"l"(pp + offsetof(DecodeParams, part_o)));
    asm volatile("prefetchu.L1 [%0];" ::"l"(pp + offsetof(DecodeParams, ws_o)));
    asm volatile("prefetchu.L1 [%0];" ::"l"(pp + offsetof(DecodeParams, ws_next)));
    asm volatile("prefetchu.L1 [%0];" ::"l"(pp + offsetof(DecodeParams, out_f32)));
  }
  // the next kernel in the stream may start its set-up now
  asm volatile("griddepcontrol.launch_dependents;");

  // ---- per-warp state -> shared memory (queries < G only)
  float *red_m = reinterpret_cast<float *>(smem);
  float *red_l = red_m + NWARPS * G;
  float *red_o = red_l + NWARPS * G;
  // the zero-point sums of this thread's two O^T columns (queries 2t, 2t+1)
  float z0 = 0.f, z1 = 0.f;
  if constexpr (kLoInN) {
    // columns 4..7 (lanes t >= 2) hold the residual sums of columns 0..3
#pragma unroll
    for (int mt = 0; mt < 8; ++mt)
#pragma unroll
      for (int i = 0; i < 4; ++i) o[mt][i] += __shfl_xor_sync(0xffffffffu, o[mt][i], 2);
  }
  if constexpr (Q4) {
    // sums over the eight key rows g of each query column
#pragma unroll
    for (int e = 0; e < 2; ++e)
#pragma unroll
      for (int off = 4; off < 32; off <<= 1) {
        lq[e] += __shfl_xor_sync(0xffffffffu, lq[e], off);
        zq[e] += __shfl_xor_sync(0xffffffffu, zq[e], off);
      }
    z0 = zq[0];
    z1 = zq[1];
    if (g == 0) {
#pragma unroll
      for (int e = 0; e < 2; ++e)
        if (2 * t + e < G) {
          red_m[warp * G + 2 * t + e] = mq[e] - (float)f;  // the reference of l and O
          red_l[warp * G + 2 * t + e] = lq[e];
        }
    }
  } else {
    l += __shfl_xor_sync(0xffffffffu, l, 1);
    l += __shfl_xor_sync(0xffffffffu, l, 2);
    if (live && t == 0) {
      red_m[warp * G + g] = m;
      red_l[warp * G + g] = l;
    }
  }
  // 4-bit: rows g carry u * 2^-24, rows g+8 16u * 2^-24, plus the zero-point
  // term; bf16: the accumulators as they are
  auto fin = [&](float x, float e, float zz) { return Q4 ? fmaf(x, e, zz) : x; };
  const int q0 = 2 * t, q1 = 2 * t + 1;
#pragma unroll
  for (int mt = 0; mt < 8; ++mt) {
    const int ch = vchan(mt);
    if (q0 < G) {
      red_o[(warp * G + q0) * D + ch] = fin(o[mt][0], kTwo24, z0);
      red_o[(warp * G + q0) * D + ch + 1] = fin(o[mt][2], kTwo20, z0);
    }
    if (q1 < G) {
      red_o[(warp * G + q1) * D + ch] = fin(o[mt][1], kTwo24, z1);
      red_o[(warp * G + q1) * D + ch + 1] = fin(o[mt][3], kTwo20, z1);
    }
  }
  __syncthreads();
  if ((int)blockIdx.x >= n_ret_ctas && P.str_pack > 1) {  // several streaming heads, one per warp group
    int r_, pidx0, wph_;
    str_group(r_, pidx0, wph_);
    decode_store_groups<__nv_bfloat16, D, G, NWARPS>(P, smem, wph_, r_, pidx0);
    return;
  }
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
  const int hp = d.str_pack > 1 ? d.str_pack : 1;
  const int grid = d.cta0[d.rows.n] + d.rows.n * ((d.n_str + hp - 1) / hp);
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

// Both the bf16 and the 4-bit tensor-core decode take the new token themselves.
bool decode_can_fuse_append(int kv_type, int D, int G) { return decode_mma_supported(kv_type, D, G); }

int decode_mma_tile_rows(int kv_type) {
  return kv_type == kINT4 ? dm::Keys<true>::STEP : dm::Keys<false>::STEP;
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
