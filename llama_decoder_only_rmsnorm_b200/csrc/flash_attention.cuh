// flash_attention.cuh -- causal grouped-query attention for prefill on tcgen05.
//
// What it computes ("Build your own Llama 3 from scratch" §3.4 Attention.forward,
// "从0开发大模型—译llama3-from-scratch" §6.11-§8): for the token at position
// p = start_pos + t and query head h,
//     o[t, h] = sum_{j <= p} softmax_j(q[t,h] . k[j, h/n_rep] / sqrt(hd)) v[j, h/n_rep]
// with k, v read from the caller's cache [B, cap, KV, hd] (rotated keys), and
// optionally the document mask of 附 1 (keys before the token's document start
// are invisible).
//
// Design (B200):
//  * A CTA owns one KV group g of one sequence b, 128 query positions, and TWO
//    query heads of that group ("slots").  Each K/V tile is loaded once by TMA
//    and used by both heads' MMAs, so repeat_kv is never formed and a KV head
//    is read ceil(n_rep/2) times per query tile instead of n_rep times.
//  * S = Q K^T (M=128 queries, N=128 keys, K=hd) and O += P V (M=128, N=hd,
//    K=128 keys) run on tcgen05 with fp32 accumulators in TMEM: slot s uses
//    columns [256s, 256s+128) for S and [256s+128, 256s+128+hd) for O.
//  * One softmax thread per query row (its TMEM lane), one warpgroup per slot.
//    The warpgroups trade registers at start-up (setmaxnreg): the producer /
//    MMA warpgroup drops to 104 per thread and the two softmax warpgroups rise
//    to 200, so a thread holds its row's 128 scores of a tile at once and
//    reads them from TMEM a single time (one max pass, one exponent pass, both
//    from registers).  Scores stay in the log2 domain; O is rescaled in TMEM
//    only when a row maximum grows by more than 2^8 (exact: the same reference
//    maximum serves numerator and denominator).
//  * P (bf16, two per 32-bit column) is written back into TMEM over the
//    scores just read (keys 0-127 -> columns 0-63) and P.V takes its A operand
//    from TMEM, so P never goes through shared memory; K and V are both
//    double-buffered in shared memory.  P is handed over in two halves (keys
//    0-63, then 64-127), so the first half's P.V runs on the tensor core
//    while the softmax is still on the second half's exponentials.
//  * A whole warp runs the MMA loop (warp-uniform addresses and descriptors)
//    and one elected lane issues; a head's next S goes right behind the P.V
//    that reads its columns, since the MMAs of one thread run in issue order.
//  * The softmax never waits for a P.V before its exponentials: the S commit
//    it waits for covers every MMA issued before that S, the P.V included.
//  * Q and K/V tiles come through 4-D TMA maps whose extents stop at `seq`
//    and `start_pos + seq`, so rows past the valid range read as zeros and no
//    unwritten cache entry is ever touched.
//  * Causal tile skipping: a query tile visits only key tiles up to its last
//    position; work units are issued longest first, in snake order.
//  * The epilogue goes through 2 KB of shared memory per softmax warp, 32
//    columns at a time, so the global stores write 64 contiguous bytes per
//    row instead of one 16-byte piece in each of 32 rows.
// The split of registers is only valid for a launch of 384 threads at 168
// registers each (128*104 + 256*200 = 384*168); the host checks the compiled
// register count before every launch.
#pragma once
#include "common.cuh"

namespace l3 {

struct FlashShape {
  int B, S, P, H, KV, n_rep, pairs, qtiles, units;
  int ldo;            // H * hd (output row length)
  float scale_log2;   // log2(e) / sqrt(hd)
  // Optional document mask: doc_start[b * S + t] is the position where the
  // document of token t begins (non-decreasing in t, <= start_pos + t); keys
  // before it are invisible ("Build your own Llama 3 from scratch" 附 1).
  const int32_t* doc_start;
  // Failure-detection test hook (0 in every normal launch): 2 = the softmax
  // thread of row 0 leaves out its P arrival on its first key tile, so the
  // MMA issuer's bounded wait for P gives up.
  int withhold;
};

__device__ __forceinline__ void flash_unit(const FlashShape& fs, int u, int& b, int& g, int& pair, int& qt) {
  const int per_qt = fs.B * fs.KV * fs.pairs;
  qt = fs.qtiles - 1 - u / per_qt;   // longest (latest) query tiles first
  int r = u % per_qt;
  pair = r % fs.pairs; r /= fs.pairs;
  g = r % fs.KV;
  b = r / fs.KV;
}
// The k-th unit of this CTA.  Units are numbered longest first; taking them
// in rows of gridDim.x, alternately left to right and right to left, evens out
// the per-CTA totals (for the 8B prefill the busiest CTA gets 229 key tiles
// instead of 256 with a plain stride, against a mean of 225).
__device__ __forceinline__ int flash_snake(int k) {
  const int G = gridDim.x, c = blockIdx.x;
  return k * G + ((k & 1) ? G - 1 - c : c);
}
__device__ __forceinline__ int flash_ntiles(const FlashShape& fs, int qt) {
  const int last_key = min(fs.P + qt * 128 + 127, fs.P + fs.S - 1);
  return last_key / 128 + 1;
}
// Lowest visible key of query row t (document mask), clamped so that a row
// always keeps its own key.
__device__ __forceinline__ int flash_row_lo(const FlashShape& fs, int b, int t) {
  if (!fs.doc_start) return 0;
  const int tt = min(t, fs.S - 1);
  return max(0, min(fs.doc_start[(size_t)b * fs.S + tt], fs.P + tt));
}
// First key tile a query tile needs: the tile of its first row's document start.
__device__ __forceinline__ int flash_first_tile(const FlashShape& fs, int b, int qt) {
  return flash_row_lo(fs, b, qt * 128) / 128;
}

// D[tmem] (+)= A[tmem] * B[smem desc]^T, kind::f16; A is K-major in TMEM
// (row m in lane m, two bf16 per 32-bit column).
__device__ __forceinline__ void tc_mma_f16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc,
                                              uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

constexpr int kFlashThreads = 384;
constexpr int kFlashLowRegs = 104, kFlashHighRegs = 200;

template <int HD>
struct FlashCfg {
  static constexpr int CHUNKS = (HD + 63) / 64;
  static constexpr int TILE_BYTES = 128 * 128;
  static constexpr int Q_BYTES = CHUNKS * TILE_BYTES;
  static constexpr int KV_BYTES = CHUNKS * TILE_BYTES;
  static constexpr int KST = 2, VST = 2;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + 2 * Q_BYTES;
  static constexpr int OFF_V = OFF_K + KST * KV_BYTES;
  static constexpr int OFF_BAR = OFF_V + VST * KV_BYTES;
  static constexpr int N_BARS = 2 + 2 + 2 * KST + 2 * VST + 2 + 2 + 2 + 2;
  // output staging: 2 KB (32 rows x 32 bf16) per softmax warp
  static constexpr int OFF_STAGE = (OFF_BAR + N_BARS * 8 + 16 + 127) / 128 * 128;
  static constexpr int SMEM_BYTES = 1024 + OFF_STAGE + 8 * 2048;
  static_assert(SMEM_BYTES <= 232448, "shared memory");
  static_assert(HD % 32 == 0 && HD <= 128, "head_dim");
};

// The 128 scores of one row (this thread's TMEM lane), 32 columns at a time.
__device__ __forceinline__ void flash_load_row(uint32_t taddr, uint32_t (&a)[32], uint32_t (&b)[32],
                                                uint32_t (&c)[32], uint32_t (&d)[32]) {
  tmem_ld32(taddr, a);
  tmem_ld32(taddr + 32, b);
  tmem_ld32(taddr + 64, c);
  tmem_ld32(taddr + 96, d);
  tc_wait_ld();
}

// p = 2^(s*scl - m) for 32 scores of the row, in place (as fp32 bits), and
// their sum in (sa, sb).  Exponentials in fp32: on unmasked tiles 4 of every
// 16 pairs go to the FMA pipe (exp2_poly2), the rest to the MUFU; masked tiles
// use the MUFU only, which gives exactly 0 for the -inf scores.
template <bool MASKED>
__device__ __forceinline__ void flash_exp_inplace(uint32_t (&r)[32], float scl, float neg_m, float& sa, float& sb) {
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    float x0, x1, p0, p1;
    fma2(x0, x1, __uint_as_float(r[2 * i]), __uint_as_float(r[2 * i + 1]), scl, scl, neg_m, neg_m);
    if (!MASKED && (i & 7) < 2) {
      exp2_poly2(x0, x1, p0, p1);
    } else {
      p0 = ex2_approx(x0);
      p1 = ex2_approx(x1);
    }
    add2(sa, sb, p0, p1);
    r[2 * i] = __float_as_uint(p0);
    r[2 * i + 1] = __float_as_uint(p1);
  }
}
__device__ __forceinline__ void flash_pack_store(uint32_t (&r)[32], uint32_t taddr) {
  uint32_t pk[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) pk[i] = pack_bf16x2(__uint_as_float(r[2 * i]), __uint_as_float(r[2 * i + 1]));
  tmem_st16(taddr, pk);
}
// Half a row (64 scores): both chunks' exponentials before any pack or store,
// so that they overlap; then the bf16 pairs go to the 32 TMEM columns at
// taddr.  Returns the half row's sum.
template <bool MASKED>
__device__ __forceinline__ float flash_exp_half(uint32_t (&ra)[32], uint32_t (&rb)[32], float scl, float neg_m,
                                                 uint32_t taddr) {
  float s0 = 0.f, s1 = 0.f, s2 = 0.f, s3 = 0.f;
  flash_exp_inplace<MASKED>(ra, scl, neg_m, s0, s1);
  flash_exp_inplace<MASKED>(rb, scl, neg_m, s2, s3);
  flash_pack_store(ra, taddr);
  flash_pack_store(rb, taddr + 16);
  return (s0 + s1) + (s2 + s3);
}

template <bool MASKED>
__device__ __forceinline__ float flash_row_max(uint32_t (&r)[32], int key0, int qpos, int lo) {
  float mx = -INFINITY;
  if (MASKED) {
#pragma unroll
    for (int i = 0; i < 32; ++i)
      if (key0 + i > qpos || key0 + i < lo) r[i] = __float_as_uint(-INFINITY);
  }
#pragma unroll
  for (int i = 0; i < 32; i += 2) mx = max3f(mx, __uint_as_float(r[i]), __uint_as_float(r[i + 1]));
  return mx;
}

// The barriers the three roles share (all in shared memory).
struct FlashBars {
  uint64_t *q_full, *q_empty, *k_full, *k_empty, *v_full, *v_empty, *s_full, *p_full, *o_done, *p_half;
};

// Producer (one thread): per work unit the Q tiles of its one or two heads,
// then K and V of every visible key tile, through the K and V rings.
template <int HD>
__device__ __forceinline__ void flash_produce(const CUtensorMap& mapQ, const CUtensorMap& mapK, const CUtensorMap& mapV,
                                               uint8_t* smem, const FlashBars& B, const FlashShape& fs,
                                               unsigned long long wait_ns) {
  using C = FlashCfg<HD>;
  uint64_t *q_full = B.q_full, *q_empty = B.q_empty, *k_full = B.k_full, *k_empty = B.k_empty;
  uint64_t *v_full = B.v_full, *v_empty = B.v_empty;
  int ks = 0, vs = 0;
  uint32_t kph = 0, vph = 0, qph = 0;   // qph: phase bit per Q slot
  bool ok = true;
  uint32_t kiss = 0, kpar = 0, viss = 0, vpar = 0, qiss = 0, qpar = 0;
  for (int k_ = 0, u = flash_snake(0); u < fs.units && ok; u = flash_snake(++k_)) {
    int b, g, pair, qt;
    flash_unit(fs, u, b, g, pair, qt);
    const int nt = flash_ntiles(fs, qt);
    const bool has1 = pair * 2 + 1 < fs.n_rep;
    for (int s = 0; s < 2 && ok; ++s) {
      if (s == 1 && !has1) break;
      if (!mbar_wait(&q_empty[s], ((qph >> s) & 1u) ^ 1u, wait_ns)) { ok = false; break; }
      mbar_arrive_expect_tx(&q_full[s], C::Q_BYTES);
      const int h = g * fs.n_rep + pair * 2 + s;
      for (int c = 0; c < C::CHUNKS; ++c)
        tma_load_4d(smem + C::OFF_Q + s * C::Q_BYTES + c * C::TILE_BYTES, &mapQ, &q_full[s], c * 64, h,
                    qt * 128, b);
      qiss |= 1u << s; qpar = (qpar & ~(1u << s)) | (qph & (1u << s));
      qph ^= 1u << s;
    }
    const int jt0 = flash_first_tile(fs, b, qt);
    for (int j = jt0; j < nt && ok; ++j) {
      if (!mbar_wait(&k_empty[ks], kph ^ 1u, wait_ns)) { ok = false; break; }
      mbar_arrive_expect_tx(&k_full[ks], C::KV_BYTES);
      for (int c = 0; c < C::CHUNKS; ++c)
        tma_load_4d(smem + C::OFF_K + ks * C::KV_BYTES + c * C::TILE_BYTES, &mapK, &k_full[ks], c * 64, g,
                    j * 128, b);
      kiss |= 1u << ks; kpar = (kpar & ~(1u << ks)) | (kph << ks);
      if (++ks == C::KST) { ks = 0; kph ^= 1u; }
      if (!mbar_wait(&v_empty[vs], vph ^ 1u, wait_ns)) { ok = false; break; }
      mbar_arrive_expect_tx(&v_full[vs], C::KV_BYTES);
      for (int c = 0; c < C::CHUNKS; ++c)
        tma_load_4d(smem + C::OFF_V + vs * C::KV_BYTES + c * C::TILE_BYTES, &mapV, &v_full[vs], c * 64, g,
                    j * 128, b);
      viss |= 1u << vs; vpar = (vpar & ~(1u << vs)) | (vph << vs);
      if (++vs == C::VST) { vs = 0; vph ^= 1u; }
    }
  }
  for (int s = 0; s < 2; ++s)
    if (qiss & (1u << s)) mbar_wait(&q_full[s], (qpar >> s) & 1u, wait_ns);
  for (int s = 0; s < C::KST; ++s)
    if (kiss & (1u << s)) mbar_wait(&k_full[s], (kpar >> s) & 1u, wait_ns);
  for (int s = 0; s < C::VST; ++s)
    if (viss & (1u << s)) mbar_wait(&v_full[s], (vpar >> s) & 1u, wait_ns);
}

// MMA issuer (one whole warp; one elected lane issues).  Per key tile and head:
// S = Q K^T into the head's S columns, and, once the softmax has written P over
// them, O += P V (P from TMEM, V MN-major from shared memory).
template <int HD>
__device__ __forceinline__ void flash_issue_mma(uint8_t* smem, const FlashBars& B, uint32_t tmem_base,
                                                 const FlashShape& fs, unsigned long long wait_ns) {
  using C = FlashCfg<HD>;
  constexpr uint32_t IDESC_S = idesc_bf16_f32(128, 128, 0, 0);
  constexpr uint32_t IDESC_O = idesc_bf16_f32(128, HD, 0, 1);   // A = P (TMEM), B = V MN-major
  uint64_t *q_full = B.q_full, *q_empty = B.q_empty, *k_full = B.k_full, *k_empty = B.k_empty;
  uint64_t *v_full = B.v_full, *v_empty = B.v_empty, *s_full = B.s_full, *p_full = B.p_full, *o_done = B.o_done;
  const bool leader = elect_one_sync();
  int ks = 0, vs = 0;
  // phase bits per slot (bit s) of the Q and P barriers as this thread sees them
  uint32_t kph = 0, vph = 0, qph = 0, pph = 0;
  bool ok = true;
  // S of the next tile overwrites the TMEM columns that hold P.  It is
  // issued right behind the P.V that reads them, without waiting for that
  // P.V to complete: the MMAs one thread issues execute in issue order, so
  // every read of P precedes the first write of the next S (the tcgen05
  // attention mainloops of CUTLASS rely on the same order).
  const uint32_t q_addr = smem_u32(smem + C::OFF_Q);
  auto issue_s = [&](int s, int kst) {
    const uint32_t d = tmem_base + s * 256;
    const uint32_t qa = q_addr + s * C::Q_BYTES;
    const uint32_t ka = smem_u32(smem + C::OFF_K + kst * C::KV_BYTES);
    if (leader) {
#pragma unroll
      for (int k = 0; k < HD / 16; ++k) {
        const uint32_t off = (k >> 2) * C::TILE_BYTES + (k & 3) * 32;
        tc_mma_f16_ss(d, sw128_desc(qa + off, 1024, 16), sw128_desc(ka + off, 1024, 16), IDESC_S, k > 0);
      }
      tc_commit(&s_full[s]);
    }
    __syncwarp();
  };
  // keys 16k.. for k in [k0, k1): P in columns 8k.., V rows 16k..
  auto issue_pv = [&](int s, int vst, bool accumulate, int k0, int k1) {
    const uint32_t d = tmem_base + s * 256 + 128;
    const uint32_t pa = tmem_base + s * 256;
    const uint32_t va = smem_u32(smem + C::OFF_V + vst * C::KV_BYTES);
    if (leader) {
#pragma unroll
      for (int k = k0; k < k1; ++k)
        tc_mma_f16_ts(d, pa + k * 8, sw128_desc(va + k * 2048, 1024, C::TILE_BYTES), IDESC_O,
                      (accumulate || k > 0) ? 1u : 0u);
      if (k1 == 8) tc_commit(&o_done[s]);
    }
    __syncwarp();
  };
  for (int k_ = 0, u = flash_snake(0); u < fs.units && ok; u = flash_snake(++k_)) {
    int b, g, pair, qt;
    flash_unit(fs, u, b, g, pair, qt);
    const int nt = flash_ntiles(fs, qt);
    const int nslots = (pair * 2 + 1 < fs.n_rep) ? 2 : 1;
    for (int s = 0; s < nslots; ++s) {
      if (!mbar_wait_warp(&q_full[s], (qph >> s) & 1u, wait_ns)) ok = false;
      qph ^= 1u << s;
    }
    if (!ok) break;
    tc_fence_after();
    const int jt0 = flash_first_tile(fs, b, qt);
    if (!mbar_wait_warp(&k_full[ks], kph, wait_ns)) break;
    tc_fence_after();
    for (int s = 0; s < nslots; ++s) issue_s(s, ks);
    if (leader) tc_commit(&k_empty[ks]);
    if (++ks == C::KST) { ks = 0; kph ^= 1u; }
    for (int j = jt0; j < nt && ok; ++j) {
      if (!mbar_wait_warp(&v_full[vs], vph, wait_ns)) { ok = false; break; }
      const bool more = j + 1 < nt;
      bool k_ready = false;
      for (int s = 0; s < nslots; ++s) {
        // keys 0-63 of P.V as soon as the softmax has written their P,
        // while it works on keys 64-127; then the rest and the next S
        if (!mbar_wait_warp(&B.p_half[s], (pph >> s) & 1u, wait_ns)) { ok = false; break; }
        tc_fence_after();
        issue_pv(s, vs, j > jt0, 0, 4);
        if (!mbar_wait_warp(&p_full[s], (pph >> s) & 1u, wait_ns)) { ok = false; break; }
        pph ^= 1u << s;
        tc_fence_after();
        issue_pv(s, vs, true, 4, 8);
        if (more) {
          if (!k_ready && !mbar_wait_warp(&k_full[ks], kph, wait_ns)) { ok = false; break; }
          k_ready = true;
          issue_s(s, ks);
        }
      }
      if (!ok) break;
      if (leader) tc_commit(&v_empty[vs]);
      if (++vs == C::VST) { vs = 0; vph ^= 1u; }
      if (more) {
        if (leader) tc_commit(&k_empty[ks]);
        if (++ks == C::KST) { ks = 0; kph ^= 1u; }
      }
    }
    if (leader)
      for (int s = 0; s < nslots; ++s) tc_commit(&q_empty[s]);
    __syncwarp();
  }
}

template <int HD>
__global__ void __launch_bounds__(kFlashThreads, 1)
    flash_attention_kernel(const __grid_constant__ CUtensorMap mapQ, const __grid_constant__ CUtensorMap mapK,
                            const __grid_constant__ CUtensorMap mapV, bf16* __restrict__ out, const FlashShape fs,
                            const unsigned long long wait_ns) {
  using C = FlashCfg<HD>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* q_full = bars;
  uint64_t* q_empty = q_full + 2;
  uint64_t* k_full = q_empty + 2;
  uint64_t* k_empty = k_full + C::KST;
  uint64_t* v_full = k_empty + C::KST;
  uint64_t* v_empty = v_full + C::VST;
  uint64_t* s_full = v_empty + C::VST;
  uint64_t* p_full = s_full + 2;
  uint64_t* o_done = p_full + 2;
  uint64_t* p_half = o_done + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(p_half + 2);
  const FlashBars fbars{q_full, q_empty, k_full, k_empty, v_full, v_empty, s_full, p_full, o_done, p_half};

  // warp index through a shuffle: the compiler then treats it as uniform
  // across the warp, so the whole-warp MMA issuer below keeps its addresses
  // and descriptors in uniform registers
  const int warp = __shfl_sync(0xffffffffu, (int)(threadIdx.x >> 5), 0), lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < 2; ++s) {
      mbar_init(&q_full[s], 1); mbar_init(&q_empty[s], 1);
      mbar_init(&s_full[s], 1); mbar_init(&p_full[s], 128); mbar_init(&o_done[s], 1);
      mbar_init(&p_half[s], 128);
    }
    for (int s = 0; s < C::KST; ++s) { mbar_init(&k_full[s], 1); mbar_init(&k_empty[s], 1); }
    for (int s = 0; s < C::VST; ++s) { mbar_init(&v_full[s], 1); mbar_init(&v_empty[s], 1); }
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&mapQ); prefetch_tensormap(&mapK); prefetch_tensormap(&mapV);
  }
  if (warp == 1) tmem_alloc(tmem_slot, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = __shfl_sync(0xffffffffu, *tmem_slot, 0);
  // Each warpgroup takes its register share (all threads of a warpgroup
  // execute it).  The two roles stay in separate branches up to the final
  // barrier, so the register limit of one never applies to the other's code.
  if (warp < 4) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;\n" ::"n"(kFlashLowRegs));
    griddep_wait_and_release();
  if (warp == 0) {
    // ---------------------------------------------------------------- producer
    if (lane == 0) flash_produce<HD>(mapQ, mapK, mapV, smem, fbars, fs, wait_ns);
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    flash_issue_mma<HD>(smem, fbars, tmem_base, fs, wait_ns);
  }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;\n" ::"n"(kFlashHighRegs));
    griddep_wait_and_release();
    // ---------------------------------------------------------------- softmax (one thread per row)
    const int slot = (warp - 4) >> 2;
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;            // query row in the tile == TMEM lane
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const uint32_t s_tmem = tmem_base + lane_off + slot * 256;
    const uint32_t o_tmem = s_tmem + 128;
    uint32_t sph = 0, oph = 0;
    for (int k_ = 0, u = flash_snake(0); u < fs.units; u = flash_snake(++k_)) {
      int b, g, pair, qt;
      flash_unit(fs, u, b, g, pair, qt);
      if (slot == 1 && !(pair * 2 + 1 < fs.n_rep)) continue;
      const int nt = flash_ntiles(fs, qt);
      const int jt0 = flash_first_tile(fs, b, qt);
      const int qpos = fs.P + qt * 128 + row;
      const int lo = flash_row_lo(fs, b, qt * 128 + row);
      const int lo_last = flash_row_lo(fs, b, qt * 128 + 127);   // largest lower bound in the tile
      float m_ref = -INFINITY, l = 0.f;
      bool ok = true;
      for (int j = jt0; j < nt; ++j) {
        if (!mbar_wait_warp(&s_full[slot], sph, wait_ns)) { ok = false; break; }
        sph ^= 1u;
        tc_fence_after();
        const bool need_mask = j * 128 + 127 > fs.P + qt * 128 || j * 128 < lo_last;
        const int key0 = j * 128;
        uint32_t ra[32], rb[32], rc[32], rd[32];
        flash_load_row(s_tmem, ra, rb, rc, rd);
        float m0, m1, m2, m3;   // four independent chains
        if (need_mask) {
          m0 = flash_row_max<true>(ra, key0, qpos, lo);
          m1 = flash_row_max<true>(rb, key0 + 32, qpos, lo);
          m2 = flash_row_max<true>(rc, key0 + 64, qpos, lo);
          m3 = flash_row_max<true>(rd, key0 + 96, qpos, lo);
        } else {
          m0 = flash_row_max<false>(ra, key0, qpos, lo);
          m1 = flash_row_max<false>(rb, key0 + 32, qpos, lo);
          m2 = flash_row_max<false>(rc, key0 + 64, qpos, lo);
          m3 = flash_row_max<false>(rd, key0 + 96, qpos, lo);
        }
        const float mx = fmaxf(fmaxf(m0, m1), fmaxf(m2, m3));
        const float m_tile = mx * fs.scale_log2;   // scale_log2 > 0: max commutes with the scale
        // The previous tile's P.V is complete here: the s_full commit just
        // waited for tracks every MMA issued before it, that P.V included.
        // So O may be rescaled without waiting on o_done; only its phase is
        // counted (one per P.V), for the epilogue's wait on the last one.
        if (j > jt0) oph ^= 1u;
        const bool grow = m_tile > m_ref + 8.0f;
        float alpha = 1.f;
        if (grow) {
          alpha = exp2f(m_ref - m_tile);   // 0 on the first tile
          l *= alpha;
          m_ref = m_tile;
        }
        if (j > jt0 && __any_sync(0xffffffffu, grow)) {
#pragma unroll 1
          for (int c = 0; c < HD / 16; ++c) {
            uint32_t o[16];
            tmem_ld16(o_tmem + c * 16, o);
            tc_wait_ld();
#pragma unroll
            for (int i = 0; i < 16; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
            tmem_st16(o_tmem + c * 16, o);
          }
          tc_wait_st();
        }
        const float scl = fs.scale_log2;
        const float neg_m = m_ref == -INFINITY ? 0.f : -m_ref;   // a row with no visible key yet: p = 0
        // P in two hand-offs: keys 0-63 (columns 0-31), then keys 64-127
        // (columns 32-63), so that the first half's P.V overlaps the second
        // half's exponentials
        float la, lb;
        if (need_mask)
          la = flash_exp_half<true>(ra, rb, scl, neg_m, s_tmem);
        else
          la = flash_exp_half<false>(ra, rb, scl, neg_m, s_tmem);
        tc_wait_st();
        tc_fence_before();
        mbar_arrive(&p_half[slot]);
        if (need_mask)
          lb = flash_exp_half<true>(rc, rd, scl, neg_m, s_tmem + 32);
        else
          lb = flash_exp_half<false>(rc, rd, scl, neg_m, s_tmem + 32);
        l += la + lb;
        tc_wait_st();
        tc_fence_before();
        if (!(fs.withhold == 2 && k_ == 0 && j == jt0 && row == 0 && slot == 0)) mbar_arrive(&p_full[slot]);
      }
      if (!ok) break;
      // epilogue: wait for the last P.V, out = O / l
      if (!mbar_wait_warp(&o_done[slot], oph, wait_ns)) break;
      oph ^= 1u;
      tc_fence_after();
      const int h = g * fs.n_rep + pair * 2 + slot;
      const float inv = 1.f / l;
      // 32 columns at a time through this warp's 2 KB of shared memory
      // (row r at 64 r bytes, its 16-byte piece k in slot k ^ ((r >> 1) & 3),
      // so neither the row-wise writes nor the piece-wise reads conflict),
      // then stored with four lanes per row: 64 contiguous bytes per row
      uint8_t* stage = smem + C::OFF_STAGE + (warp - 4) * 2048;
      const int t0 = qt * 128 + quarter * 32;
      bf16* obase = out + ((size_t)b * fs.S + t0) * fs.ldo + (size_t)h * HD;
#pragma unroll 1
      for (int c = 0; c < HD / 32; ++c) {
        uint32_t r[32];
        tmem_ld32(o_tmem + c * 32, r);
        tc_wait_ld();
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          uint4 o;
          o.x = pack_bf16x2(__uint_as_float(r[8 * k + 0]) * inv, __uint_as_float(r[8 * k + 1]) * inv);
          o.y = pack_bf16x2(__uint_as_float(r[8 * k + 2]) * inv, __uint_as_float(r[8 * k + 3]) * inv);
          o.z = pack_bf16x2(__uint_as_float(r[8 * k + 4]) * inv, __uint_as_float(r[8 * k + 5]) * inv);
          o.w = pack_bf16x2(__uint_as_float(r[8 * k + 6]) * inv, __uint_as_float(r[8 * k + 7]) * inv);
          *reinterpret_cast<uint4*>(stage + lane * 64 + ((k ^ ((lane >> 1) & 3)) << 4)) = o;
        }
        __syncwarp();
#pragma unroll
        for (int m = 0; m < 4; ++m) {
          const int rr = m * 8 + (lane >> 2), k = lane & 3;
          const uint4 o = *reinterpret_cast<const uint4*>(stage + rr * 64 + ((k ^ ((rr >> 1) & 3)) << 4));
          if (t0 + rr < fs.S)
            *reinterpret_cast<uint4*>(obase + (size_t)rr * fs.ldo + c * 32 + k * 8) = o;
        }
        __syncwarp();
      }
      tc_fence_before();
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 512);
  }
}

}  // namespace l3
