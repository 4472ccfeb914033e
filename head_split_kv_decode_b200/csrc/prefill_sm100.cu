// Chunked pre-fill attention on the sm_100a tensor cores (tcgen05 + TMEM + TMA).
//
// The C queries of a chunk (positions c0 .. c0+C-1) attend to the cache as it
// stands (positions < c0) and to the chunk's own keys.  Retrieval heads use
// the causal set; streaming heads the Lambda set {j <= i : j < S or i-j < R}
// (sinks plus recent tokens), so their key tiles outside the band are never
// loaded or multiplied.  Pages: "DuoAttention: Efficient Long-Context LLM
// Inference with Retrieval and Streaming Heads" (hotpaper.ai), abstract (the
// constant-length cache of streaming heads also cuts pre-filling latency);
// "韩松团队长上下文LLM推理高效框架" (cn.bg3.co), section "研究背景" (pre-fill cost
// quadratic in the context under full attention).
//
// One CTA = one (batch row, query head, pair of 128-row query tiles A and B).
// Warps 0-3 run the softmax of tile A, warps 4-7 of tile B, warp 8 issues TMA
// loads, warp 9 issues tcgen05.mma.  Per key tile j (128 keys):
//   S_X = Q_X K_j^T   (M=128, N=128, K=128; operands in 128B-swizzled smem)
//   P_X = exp2(S_X * scale*log2e - m_X)   written back over S_X as bf16 in TMEM
//   O_X += P_X V_j    (A operand from TMEM, V read MN-major from smem)
// S, P and O live in tensor memory (4 x 128 columns); O is rescaled in TMEM only
// when a row's running max grows by more than 2^8 (the ratio stays exact).
// Both query tiles share every K/V tile; K/V are double buffered.
#include <cuda.h>

#include <cstring>

#include "common.cuh"

namespace duo {

namespace pf {

constexpr int BM = 128;           // query rows per tile
constexpr int BN = 128;           // keys per tile
constexpr int HD = 128;           // head dim
constexpr int BOX = 16384;        // one 64-column x 128-row swizzled box (bytes)
constexpr int TILE = 2 * BOX;     // a 128 x 128 bf16 tile
constexpr int kThreads = 384;       // 3 warpgroups: softmax A, softmax B, TMA + MMA (+2 idle)
// Register split (setmaxnreg): the TMA/MMA warpgroup drops to kRegsLow and the
// softmax warpgroups rise to kRegsHigh.  The sum must fit what the CTA was
// launched with (kThreads x launch registers); the host checks it.
constexpr int kRegsHigh = 200;
constexpr int kRegsLow = 96;
constexpr float kRescaleLog2 = 8.0f;

// shared memory map (offsets from a 1024-aligned base)
constexpr int kQA = 0, kQB = TILE;
constexpr int kK0 = 2 * TILE, kV0 = 3 * TILE, kK1 = 4 * TILE, kV1 = 5 * TILE;
constexpr int kBars = 6 * TILE;
enum Bar { Q_FULL = 0, K_FULL0, K_FULL1, V_FULL0, V_FULL1, K_EMPTY0, K_EMPTY1, V_EMPTY0,
           V_EMPTY1, S_FULL_A, S_FULL_B, P_FULL_A, P_FULL_B, O_FULL_A, O_FULL_B, DRAIN, NBARS };
constexpr int kTmemSlot = kBars + NBARS * 8;
constexpr int kAbort = kTmemSlot + 4;
constexpr int kSmemBytes = kAbort + 4 + 1024;  // + alignment slack

// instruction descriptors (kind::f16): D f32, A/B bf16, M=128, N=128
constexpr uint32_t kIdescS = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) |
                             ((uint32_t)(BM >> 4) << 24);
constexpr uint32_t kIdescPV = (1u << 4) | (1u << 7) | (1u << 10) | (1u << 16) |
                              ((uint32_t)(HD >> 3) << 17) | ((uint32_t)(BM >> 4) << 24);

// Shared-memory matrix descriptor, 128-byte swizzle, split in two words.  The
// high word (stride between 8-row groups 1024 B, version 1, swizzle mode 128 B)
// is the same for every operand here; the low word holds the start address
// (>> 4, 14 bits) and the leading-byte offset.  Operands are passed as low
// words (advancing a k-step adds to the address field, which stays below 2^14
// since shared memory is < 256 KB) and joined to the high word in the MMA, so
// the issuing thread does 32-bit instead of 64-bit arithmetic per product.
constexpr uint32_t kDescHi = (1024u >> 4) | (1u << 14) | (2u << 29);
__device__ __forceinline__ uint32_t sdesc_lo(uint32_t addr, uint32_t lbo_bytes) {
  return ((addr & 0x3FFFFu) >> 4) | (((lbo_bytes >> 4) & 0x3FFFu) << 16);
}

// D (TMEM) (+)= A (smem) * B (smem)
__device__ __forceinline__ void mma_ss(uint32_t d_tmem, uint32_t a_lo, uint32_t b_lo, uint32_t idesc,
                                       uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t.reg .b64 da, db;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "mov.b64 da, {%1, %5};\n\t"
      "mov.b64 db, {%2, %5};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], da, db, %3, {%6, %7, %8, %9}, p;\n\t}\n" ::"r"(d_tmem),
      "r"(a_lo), "r"(b_lo), "r"(idesc), "r"(acc), "n"(kDescHi), "r"(0u), "r"(0u), "r"(0u), "r"(0u));
}

// D (TMEM) (+)= A (TMEM) * B (smem)
__device__ __forceinline__ void mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint32_t b_lo, uint32_t idesc,
                                       uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t.reg .b64 db;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "mov.b64 db, {%2, %5};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], db, %3, {%6, %7, %8, %9}, p;\n\t}\n" ::"r"(d_tmem),
      "r"(a_tmem), "r"(b_lo), "r"(idesc), "r"(acc), "n"(kDescHi), "r"(0u), "r"(0u), "r"(0u), "r"(0u));
}

__device__ __forceinline__ void mma_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
               : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]),
        "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]),
        "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

// Same load without the completion wait: issue several, then tmem_wait_ld().
__device__ __forceinline__ void tmem_ld32_async(uint32_t taddr, float *v) {
  uint32_t *r = reinterpret_cast<uint32_t *>(v);
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]),
        "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]),
        "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}

__device__ __forceinline__ void tmem_wait_ld() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ float max3f(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// Bits c in [0,32) set where first + 32*ch + c lies in [lo, hi).
__device__ __forceinline__ uint32_t range_bits(int64_t lo, int64_t hi, int64_t first, int ch) {
  const int64_t a = max(lo - (first + 32 * ch), (int64_t)0);
  const int64_t b = min(hi - (first + 32 * ch), (int64_t)32);
  if (b <= a) return 0u;
  const uint32_t upto_b = b >= 32 ? 0xffffffffu : ((1u << b) - 1u);
  const uint32_t below_a = (1u << a) - 1u;
  return upto_b & ~below_a;
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const float (&v)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,"
      "%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
      "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
      "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])), "r"(__float_as_uint(v[8])),
      "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
      "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])),
      "r"(__float_as_uint(v[15])), "r"(__float_as_uint(v[16])), "r"(__float_as_uint(v[17])),
      "r"(__float_as_uint(v[18])), "r"(__float_as_uint(v[19])), "r"(__float_as_uint(v[20])),
      "r"(__float_as_uint(v[21])), "r"(__float_as_uint(v[22])), "r"(__float_as_uint(v[23])),
      "r"(__float_as_uint(v[24])), "r"(__float_as_uint(v[25])), "r"(__float_as_uint(v[26])),
      "r"(__float_as_uint(v[27])), "r"(__float_as_uint(v[28])), "r"(__float_as_uint(v[29])),
      "r"(__float_as_uint(v[30])), "r"(__float_as_uint(v[31]))
      : "memory");
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&v)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,"
      "%15,%16};" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
      "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15])
      : "memory");
}

__device__ __forceinline__ void tmem_wait_st() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// 3-D tiled TMA load into this CTA's shared memory.  x must be a multiple of
// 8 elements (16 bytes); it is 0 or 64 here.
__device__ __forceinline__ void tma_load3(uint32_t dst, const CUtensorMap *map, int x, int y, int z,
                                          uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, "
      "%4}], [%5];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(bar)
      : "memory");
}

// ---------------------------------------------------------------- tile schedule
//
// The key tiles one query pair visits, in order: tiles of the cache prefix
// (segment 0: the retrieval page, or the streaming slot buffer), then tiles of
// the chunk itself (segment 1).  Every role of the CTA walks the same sequence.
struct Sched {
  bool ret;
  int64_t c0;       // tokens in the cache before the chunk
  int C, S, R, W;
  int q0;           // first chunk row of the pair
  int n_pre;        // candidate prefix tiles
  int filled;       // streaming: filled slots
  int kt_max;       // last chunk tile any row of the pair can see
  int ks_max;       // streaming: last chunk tile holding a sink position (-1: none)
  int kb_lo;        // streaming: first chunk tile reaching the band

  __device__ void init(bool retrieval, int64_t c0_, int C_, int S_, int R_, int W_, int q0_) {
    ret = retrieval;
    c0 = c0_;
    C = C_;
    S = S_;
    R = R_;
    W = W_;
    q0 = q0_;
    const int last_row = min(C - 1, q0 + 2 * BM - 1);
    kt_max = last_row / BN;
    if (ret) {
      n_pre = (int)((c0 + BN - 1) / BN);
      filled = 0;
      ks_max = -1;
      kb_lo = 0;
    } else {
      filled = (int)min(c0, (int64_t)W);
      n_pre = (filled + BN - 1) / BN;
      ks_max = (c0 < S) ? (int)((S - 1 - c0) / BN) : -1;
      const int need = q0 - R - (BN - 2);  // tile kt reaches the band iff BN*kt >= need
      kb_lo = need <= 0 ? 0 : (need + BN - 1) / BN;
    }
  }
  __device__ bool pre_needed(int t) const {
    if (ret) return true;
    const int lo = t * BN;
    if (lo < min(S, filled)) return true;                          // holds sinks
    return (q0 < R - 1) && (lo + BN - 1 >= S) && (lo < filled);    // ring may be visible
  }
  __device__ bool chunk_needed(int kt) const {
    if (ret) return true;
    return kt <= ks_max || kt >= kb_lo;
  }
  __device__ int count() const {
    if (ret) return n_pre + kt_max + 1;
    int n = 0;
    for (int t = 0; t < n_pre; ++t) n += pre_needed(t);
    for (int kt = 0; kt <= kt_max; ++kt) n += chunk_needed(kt);
    return n;
  }
  // j-th visited tile -> (segment, tile index); retrieval heads visit every
  // tile, streaming heads walk their short candidate list.
  __device__ void get(int j, int &seg, int &idx) const {
    if (ret) {
      seg = j < n_pre ? 0 : 1;
      idx = j < n_pre ? j : j - n_pre;
      return;
    }
    for (int t = 0; t < n_pre; ++t)
      if (pre_needed(t)) {
        if (j == 0) { seg = 0; idx = t; return; }
        --j;
      }
    for (int kt = 0; kt <= kt_max; ++kt)
      if (chunk_needed(kt)) {
        if (j == 0) { seg = 1; idx = kt; return; }
        --j;
      }
    seg = 1;
    idx = 0;
  }
};

struct Maps {
  CUtensorMap q;       // [B*C][Hq][D]
  CUtensorMap kc, vc;  // [B*C][Hkv][D]     (chunk K/V)
  CUtensorMap kr, vr;  // [B*n_ret][cap][D] (retrieval pages)
  CUtensorMap ks, vs;  // [B*n_str][W][D]   (streaming slot buffers)
};

__device__ __forceinline__ bool abort_set(volatile int *flag) { return *flag != 0; }

__global__ void __launch_bounds__(kThreads, 1)
    prefill_kernel(const __grid_constant__ PrefillParams P, const __grid_constant__ Maps M) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t *sm = smem_raw + (base - raw);
  auto bar = [&](int i) { return base + kBars + 8u * i; };
  volatile int *abort_flag = reinterpret_cast<volatile int *>(sm + kAbort);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  // ---- work item: retrieval query heads first, heaviest pairs first
  const int n_pairs = (P.C + 2 * BM - 1) / (2 * BM);
  const int ret_q = P.n_ret * P.G, str_q = P.n_str * P.G;
  int blk = blockIdx.x;
  bool retrieval;
  int b, hq, kvh, pidx, pair;  // b: launch row (indexes the inputs and outputs)
  if (blk < P.rows.n * ret_q * n_pairs) {
    retrieval = true;
    const int per = P.rows.n * ret_q;
    pair = n_pairs - 1 - blk / per;
    const int r = blk % per;
    b = r / ret_q;
    const int rr = r % ret_q;
    pidx = rr / P.G;
    kvh = P.h.ret_heads[pidx];
    hq = kvh * P.G + rr % P.G;
  } else {
    retrieval = false;
    blk -= P.rows.n * ret_q * n_pairs;
    const int per = P.rows.n * str_q;
    pair = n_pairs - 1 - blk / per;
    const int r = blk % per;
    b = r / str_q;
    const int rr = r % str_q;
    pidx = rr / P.G;
    kvh = P.h.str_heads[pidx];
    hq = kvh * P.G + rr % P.G;
  }
  const int brow = P.rows.row[b];       // its batch row in the cache
  const int64_t c0 = P.rows.len[b];     // tokens of that row already in the cache
  const int q0 = pair * 2 * BM;
  Sched sc;
  sc.init(retrieval, c0, P.C, P.S, P.R, P.W, q0);
  const int n_tiles = sc.count();

  // ---- set-up: barriers, tensor memory
  if (tid == 0) {
    for (int i = 0; i < NBARS; ++i) {
      const uint32_t cnt = (i == P_FULL_A || i == P_FULL_B) ? 4u : 1u;
      mbar_init(bar(i), cnt);
    }
    // once a bounded wait of this kernel has given up, later CTAs do no work
    *abort_flag = (P.err && (*(volatile int *)P.err & kErrWaitPrefillLoad)) ? 1 : 0;
    fence_barrier_init();
  }
  if (warp == 9) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(base + kTmemSlot),
                 "r"(512u));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(sm + kTmemSlot);

  if (warp >= 8) {
    // third warpgroup: one TMA warp, one MMA warp, two spare warps
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsLow));
  if (warp == 8) {
    // =============================================================== TMA producer
    // (testing hook: with P.skip_loads nothing is loaded, so every wait of
    // the other roles runs out and the CTA unwinds)
    if (lane == 0 && !P.skip_loads) {
      const int qz = b * P.C + q0;
      mbar_arrive_expect_tx(bar(Q_FULL), 2 * TILE);
      tma_load3(base + kQA, &M.q, 0, hq, qz, bar(Q_FULL));
      tma_load3(base + kQA + BOX, &M.q, 64, hq, qz, bar(Q_FULL));
      tma_load3(base + kQB, &M.q, 0, hq, qz + BM, bar(Q_FULL));
      tma_load3(base + kQB + BOX, &M.q, 64, hq, qz + BM, bar(Q_FULL));
      const CUtensorMap *pk = retrieval ? &M.kr : &M.ks;
      const CUtensorMap *pv = retrieval ? &M.vr : &M.vs;
      const int pz = brow * P.n_str + pidx;  // streaming slot buffer
      int issued_k = 0, issued_v = 0;
      auto issue = [&](int j, bool is_v) -> bool {
        const int st = j & 1;
        if (j >= 2 && !mbar_wait(bar((is_v ? V_EMPTY0 : K_EMPTY0) + st), (uint32_t)(((j - 2) >> 1) & 1),
                                 P.err, kErrWaitPrefillLoad, P.wait_ns))
          return false;
        int seg, idx;
        sc.get(j, seg, idx);
        const uint32_t dst = base + (is_v ? (st ? kV1 : kV0) : (st ? kK1 : kK0));
        const uint32_t fb = bar((is_v ? V_FULL0 : K_FULL0) + st);
        mbar_arrive_expect_tx(fb, TILE);
        if (seg == 0) {
          // retrieval: the storage row of the tile's first key (a tile of BN
          // keys never crosses a block of the paged layout); streaming: slot
          const CUtensorMap *m = is_v ? pv : pk;
          const int y = retrieval ? (int)ret_row(P.ret, brow, pidx, (int64_t)idx * BN) : idx * BN;
          const int z = retrieval ? 0 : pz;
          tma_load3(dst, m, 0, y, z, fb);
          tma_load3(dst + BOX, m, 64, y, z, fb);
        } else {
          const CUtensorMap *m = is_v ? &M.vc : &M.kc;
          const int z = b * P.C + idx * BN;
          tma_load3(dst, m, 0, kvh, z, fb);
          tma_load3(dst + BOX, m, 64, kvh, z, fb);
        }
        return true;
      };
      for (int j = 0; j <= n_tiles; ++j) {
        if (abort_set(abort_flag)) break;
        if (j < n_tiles) {
          if (!issue(j, false)) { *abort_flag = 1; break; }
          issued_k = j + 1;
        }
        if (j >= 1) {
          if (!issue(j - 1, true)) { *abort_flag = 1; break; }
          issued_v = j;
        }
      }
      // Copies still in flight land before the CTA can exit (bounded waits;
      // an already completed phase returns at once).
      for (int jj = max(0, issued_k - 2); jj < issued_k; ++jj)
        mbar_wait(bar(K_FULL0 + (jj & 1)), (uint32_t)((jj >> 1) & 1), P.err, kErrWaitPrefillLoad,
                  P.wait_ns);
      for (int jj = max(0, issued_v - 2); jj < issued_v; ++jj)
        mbar_wait(bar(V_FULL0 + (jj & 1)), (uint32_t)((jj >> 1) & 1), P.err, kErrWaitPrefillLoad,
                  P.wait_ns);
    }
  } else if (warp == 9) {
    // =============================================================== MMA issuer
    if (lane == 0) {
      const uint32_t tS[2] = {tmem + 0u, tmem + 128u};
      const uint32_t tO[2] = {tmem + 256u, tmem + 384u};
      // Descriptor low words are built once.  K-major Q and K: step k of 16
      // columns is 32 bytes into a 64-column box, the second box 16 KB on; V
      // is MN-major: 16 keys are 16 rows of 128 bytes.
      const uint32_t dq[2] = {sdesc_lo(base + kQA, 16), sdesc_lo(base + kQB, 16)};
      const uint32_t dk[2] = {sdesc_lo(base + kK0, 16), sdesc_lo(base + kK1, 16)};
      const uint32_t dv[2] = {sdesc_lo(base + kV0, BOX), sdesc_lo(base + kV1, BOX)};
      auto issue_s = [&](int x, int st) {
#pragma unroll
        for (int k = 0; k < HD / 16; ++k) {
          const uint32_t off = (uint32_t)(((k >> 2) * BOX + (k & 3) * 32) >> 4);
          mma_ss(tS[x], dq[x] + off, dk[st] + off, kIdescS, k > 0);
        }
      };
      auto issue_pv = [&](int x, int st, int j) {
#pragma unroll
        for (int k = 0; k < BN / 16; ++k)
          mma_ts(tO[x], tS[x] + 8u * k, dv[st] + (uint32_t)((k * 2048) >> 4), kIdescPV, (j > 0 || k > 0));
      };
      bool ok = mbar_wait(bar(Q_FULL), 0, P.err, kErrWaitMma, P.wait_ns) &&
                mbar_wait(bar(K_FULL0), 0, P.err, kErrWaitMma, P.wait_ns);
      if (ok) {
        tc_fence_after();
        issue_s(0, 0);
        mma_commit(bar(S_FULL_A));
        issue_s(1, 0);
        mma_commit(bar(S_FULL_B));
        mma_commit(bar(K_EMPTY0));
      }
      for (int j = 0; ok && j < n_tiles; ++j) {
        const int st = j & 1;
        const bool more = j + 1 < n_tiles;
        ok = mbar_wait(bar(V_FULL0 + st), (uint32_t)((j >> 1) & 1), P.err, kErrWaitMma, P.wait_ns) &&
             mbar_wait(bar(P_FULL_A), (uint32_t)(j & 1), P.err, kErrWaitMma, P.wait_ns);
        if (!ok) break;
        tc_fence_after();
        issue_pv(0, st, j);
        if (more) {
          ok = mbar_wait(bar(K_FULL0 + (st ^ 1)), (uint32_t)(((j + 1) >> 1) & 1), P.err, kErrWaitMma,
                         P.wait_ns);
          if (!ok) break;
          tc_fence_after();
          issue_s(0, st ^ 1);
          mma_commit(bar(S_FULL_A));
        } else {
          mma_commit(bar(O_FULL_A));
        }
        ok = mbar_wait(bar(P_FULL_B), (uint32_t)(j & 1), P.err, kErrWaitMma, P.wait_ns);
        if (!ok) break;
        tc_fence_after();
        issue_pv(1, st, j);
        mma_commit(bar(V_EMPTY0 + st));
        if (more) {
          issue_s(1, st ^ 1);
          mma_commit(bar(S_FULL_B));
          mma_commit(bar(K_EMPTY0 + (st ^ 1)));
        } else {
          mma_commit(bar(O_FULL_B));
        }
      }
      if (!ok) *abort_flag = 1;
      // nothing may still be writing tensor memory when it is freed
      mma_commit(bar(DRAIN));
      mbar_wait(bar(DRAIN), 0, P.err, kErrWaitMma, P.wait_ns);
    }
  }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsHigh));
    // =============================================================== softmax (A: warps 0-3, B: 4-7)
    const int x = warp >> 2;
    const int wq = warp & 3;
    const int row = wq * 32 + lane;                 // row of the query tile = TMEM lane
    const int crow = q0 + x * BM + row;             // chunk row
    const int64_t ipos = c0 + crow;                 // absolute query position
    const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
    const uint32_t tS = tmem + (x ? 128u : 0u) + lane_off;
    const uint32_t tO = tmem + (x ? 384u : 256u) + lane_off;
    const int s_bar = x ? S_FULL_B : S_FULL_A;
    const int p_bar = x ? P_FULL_B : P_FULL_A;
    const int o_bar = x ? O_FULL_B : O_FULL_A;
    const float sl2 = P.scale_log2;
    float m = -INFINITY;
    float2 l2[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
    bool ok = true;
    for (int j = 0; j < n_tiles; ++j) {
      ok = mbar_wait(bar(s_bar), (uint32_t)(j & 1), P.err, kErrWaitMma, P.wait_ns);
      if (!__all_sync(0xffffffffu, ok) || abort_set(abort_flag)) {
        ok = false;
        break;
      }
      tc_fence_after();
      int seg, idx;
      sc.get(j, seg, idx);

      // Visible columns of this row as bit masks, one per 32 columns.  Every
      // visible set here is a union of at most three position ranges.
      const int64_t first = (int64_t)idx * BN;
      uint32_t vis[BN / 32];
      if (seg == 1) {
        // chunk keys: kr in [0, C), kr <= crow, and (streaming) sink or band
        const int64_t hi = min((int64_t)P.C, (int64_t)crow + 1);
#pragma unroll
        for (int ch = 0; ch < BN / 32; ++ch) {
          if (retrieval) {
            vis[ch] = range_bits(0, hi, first, ch);
          } else {
            vis[ch] = range_bits(0, min(hi, (int64_t)P.S - c0), first, ch) |
                      range_bits((int64_t)crow - P.R + 1, hi, first, ch);
          }
        }
      } else if (retrieval) {
        // page rows are positions; all below c0 are visible
#pragma unroll
        for (int ch = 0; ch < BN / 32; ++ch) vis[ch] = range_bits(0, c0, first, ch);
      } else {
        // slot buffer: sinks, plus the ring slots of positions in
        // [max(S, ipos-R+1), c0) (a cyclic slot range)
        const int64_t filled = sc.filled;
        const int64_t p_lo = max((int64_t)P.S, ipos - P.R + 1), p_hi = c0;  // [p_lo, p_hi)
        int64_t r1lo = 0, r1hi = 0, r2lo = 0, r2hi = 0;
        if (p_lo < p_hi) {
          const int64_t cnt = p_hi - p_lo;
          const int64_t s_lo = P.S + (p_lo - P.S) % P.R;
          r1lo = s_lo;
          r1hi = min(s_lo + cnt, (int64_t)P.S + P.R);
          const int64_t spill = s_lo + cnt - ((int64_t)P.S + P.R);
          if (spill > 0) {
            r2lo = P.S;
            r2hi = P.S + spill;
          }
        }
#pragma unroll
        for (int ch = 0; ch < BN / 32; ++ch)
          vis[ch] = (range_bits(0, min((int64_t)P.S, filled), first, ch) |
                     range_bits(r1lo, min(r1hi, filled), first, ch) |
                     range_bits(r2lo, min(r2hi, filled), first, ch));
      }
      // The whole S row in registers: four loads in flight, one wait.
      float v[BN];
#pragma unroll
      for (int cc = 0; cc < BN / 32; ++cc) tmem_ld32_async(tS + 32u * cc, v + 32 * cc);
      tmem_wait_ld();
#pragma unroll
      for (int k = 0; k < BN / 32; ++k) {
        const uint32_t bits = vis[k];
        if (bits != 0xffffffffu) {
#pragma unroll
          for (int i = 0; i < 32; ++i)
            if (!((bits >> i) & 1u)) v[32 * k + i] = -INFINITY;
        }
      }
      float mx;
      {
        float t[16];
#pragma unroll
        for (int i = 0; i < 16; ++i)
          t[i] = max3f(max3f(v[8 * i], v[8 * i + 1], v[8 * i + 2]),
                       max3f(v[8 * i + 3], v[8 * i + 4], v[8 * i + 5]), fmaxf(v[8 * i + 6], v[8 * i + 7]));
        const float u0 = max3f(t[0], t[1], t[2]), u1 = max3f(t[3], t[4], t[5]);
        const float u2 = max3f(t[6], t[7], t[8]), u3 = max3f(t[9], t[10], t[11]);
        const float u4 = max3f(t[12], t[13], t[14]);
        mx = max3f(max3f(u0, u1, u2), max3f(u3, u4, t[15]), -INFINITY) * sl2;
      }
      const float m_new = fmaxf(m, mx);
      const bool grow = m_new > m + kRescaleLog2 || (m == -INFINITY && m_new > -INFINITY);
      if (__any_sync(0xffffffffu, grow)) {
        const float alpha = grow ? (m == -INFINITY ? 0.f : fast_exp2(m - m_new)) : 1.f;
        if (j > 0) {
#pragma unroll 1
          for (int cc = 0; cc < HD / 32; ++cc) {
            float o[32];
            tmem_ld32(tO + 32u * cc, o);
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] *= alpha;
            tmem_st32(tO + 32u * cc, o);
          }
          tmem_wait_st();
        }
        if (grow) {
          l2[0].x *= alpha;
          l2[0].y *= alpha;
          l2[1].x *= alpha;
          l2[1].y *= alpha;
          m = m_new;
        }
      }
      // probabilities 2^(s*scale*log2e - m), summed in fp32 and written over S
      // as packed bf16 (column c/2 holds keys c, c+1)
      const float mu = (m == -INFINITY) ? 0.f : m;
      const float2 sc2 = make_float2(sl2, sl2), nm2 = make_float2(-mu, -mu);
#pragma unroll
      for (int cc = 0; cc < BN / 32; ++cc) {
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          float2 t = ffma2(make_float2(v[32 * cc + 2 * i], v[32 * cc + 2 * i + 1]), sc2, nm2);
          t.x = fast_exp2(t.x);
          t.y = fast_exp2(t.y);
          l2[i & 1] = __fadd2_rn(l2[i & 1], t);
          __nv_bfloat162 h2 = __floats2bfloat162_rn(t.x, t.y);
          pk[i] = *reinterpret_cast<uint32_t *>(&h2);
        }
        tmem_st16(tS + 16u * cc, pk);
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(p_bar));
    }
    const float l = (l2[0].x + l2[0].y) + (l2[1].x + l2[1].y);
    if (ok) ok = mbar_wait(bar(o_bar), 0, P.err, kErrWaitMma, P.wait_ns);
    if (__all_sync(0xffffffffu, ok) && !abort_set(abort_flag)) {
      tc_fence_after();
      const float inv = l > 0.f ? 1.f / l : 0.f;
      __nv_bfloat16 *out = reinterpret_cast<__nv_bfloat16 *>(P.out) +
                           (((int64_t)b * P.C + crow) * P.Hq + hq) * HD;
      float o[HD];
#pragma unroll
      for (int cc = 0; cc < HD / 32; ++cc) tmem_ld32_async(tO + 32u * cc, o + 32 * cc);
      tmem_wait_ld();
      if (crow < P.C) {
        uint4 *dst = reinterpret_cast<uint4 *>(out);
#pragma unroll
        for (int i = 0; i < HD / 8; ++i) {
          uint4 pk;
          uint32_t *w = reinterpret_cast<uint32_t *>(&pk);
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            __nv_bfloat162 h2 = __floats2bfloat162_rn(o[8 * i + 2 * k] * inv, o[8 * i + 2 * k + 1] * inv);
            w[k] = *reinterpret_cast<uint32_t *>(&h2);
          }
          dst[i] = pk;
        }
      }
    } else {
      *abort_flag = 1;
    }
  }

  // ---- tear-down: every role has left its loop; free tensor memory
  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(512u));
  }
}

// ---------------------------------------------------------------- host side

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return nullptr;
    fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// 3-D bf16 map over [d2][d1][128] with a box of (64, b1, b2), 128-byte swizzle.
static bool make_map(CUtensorMap *m, const void *ptr, uint64_t d1, uint64_t d2, uint64_t stride1,
                     uint64_t stride2, uint32_t b1, uint32_t b2) {
  EncodeTiledFn enc = encode_fn();
  if (!enc || !ptr) return false;
  const cuuint64_t dims[3] = {HD, d1, d2};
  const cuuint64_t strides[2] = {stride1, stride2};
  const cuuint32_t box[3] = {64, b1, b2};
  const cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(ptr), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace pf

cudaError_t launch_prefill(const PrefillParams &p, cudaStream_t s) {
  using namespace pf;
  if (p.D != HD || p.C <= 0) return cudaErrorInvalidValue;
  Maps maps;
  std::memset(&maps, 0, sizeof(maps));
  const uint64_t row = HD * 2;
  if (p.rows.n <= 0) return cudaSuccess;
  const uint64_t BC = (uint64_t)p.rows.n * p.C;  // inputs and outputs: the launch rows
  bool ok = make_map(&maps.q, p.q, p.Hq, BC, row, row * p.Hq, 1, BM) &&
            make_map(&maps.kc, p.k, p.Hkv, BC, row, row * p.Hkv, 1, BN) &&
            make_map(&maps.vc, p.v, p.Hkv, BC, row, row * p.Hkv, 1, BN);
  // A kind with no heads in this layer keeps zeroed maps: no CTA reads them.
  // Retrieval buffers are addressed by storage row (packed or paged), so
  // their maps are flat; TMA coordinates are 32-bit.
  if (ok && p.n_ret > 0) {
    if (p.retrieval_rows >= (1LL << 31)) return cudaErrorInvalidValue;
    const uint64_t rr = (uint64_t)p.retrieval_rows;
    ok = make_map(&maps.kr, p.p.ret_k, rr, 1, row, row * rr, BN, 1) &&
         make_map(&maps.vr, p.p.ret_v, rr, 1, row, row * rr, BN, 1);
  }
  if (ok && p.n_str > 0)
    ok = make_map(&maps.ks, p.p.str_k, p.W, (uint64_t)p.B * p.n_str, row, row * p.W, BN, 1) &&
         make_map(&maps.vs, p.p.str_v, p.W, (uint64_t)p.B * p.n_str, row, row * p.W, BN, 1);
  if (!ok) return cudaErrorInvalidValue;
  static bool attr = false;
  if (!attr) {
    cudaError_t e = cudaFuncSetAttribute(prefill_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         kSmemBytes);
    if (e != cudaSuccess) return e;
    // The register split must fit the registers the CTA is launched with, or
    // setmaxnreg.inc would wait for registers that never come.
    cudaFuncAttributes fa;
    if ((e = cudaFuncGetAttributes(&fa, prefill_kernel)) != cudaSuccess) return e;
    if (128 * (2 * kRegsHigh + kRegsLow) > kThreads * fa.numRegs) return cudaErrorInvalidConfiguration;
    attr = true;
  }
  const int n_pairs = (p.C + 2 * BM - 1) / (2 * BM);
  const int grid = p.rows.n * (p.n_ret + p.n_str) * p.G * n_pairs;
  prefill_kernel<<<grid, kThreads, kSmemBytes, s>>>(p, maps);
  return cudaGetLastError();
}

}  // namespace duo
