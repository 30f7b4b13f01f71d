// flash_attention.cuh -- causal grouped-query attention for prefill on tcgen05.
//
// What it computes ("Build your own Llama 3 from scratch" §3.4 Attention.forward,
// "从0开发大模型—译llama3-from-scratch" §6.11-§8): for the token at position
// p = start_pos + t and query head h,
//     o[t, h] = sum_{j <= p} softmax_j(q[t,h] . k[j, h/n_rep] / sqrt(hd)) v[j, h/n_rep]
// with k, v read from the caller's cache [B, cap, KV, hd] (rotated keys).
//
// Design (B200):
//  * A CTA owns one KV group g of one sequence b, 128 query positions, and TWO
//    query heads of that group ("slots").  Each K/V tile is loaded once by TMA
//    and used by both heads' MMAs, so repeat_kv is never formed and a KV head
//    is read ceil(n_rep/2) times per query tile instead of n_rep times.
//  * S = Q K^T (M=128 queries, N=128 keys, K=hd) and O += P V (M=128, N=hd,
//    K=128 keys) run on tcgen05 with fp32 accumulators in TMEM:
//    slot s uses columns [256s, 256s+128) for S and [256s+128, 256s+128+hd) for O.
//  * One warpgroup per slot does the online softmax, one thread per query row
//    (its TMEM lane).  While one slot's warpgroup exponentiates, the tensor
//    core runs the other slot's MMAs (ping-pong).  Scores are kept in the
//    log2 domain; O is rescaled in TMEM only when a row maximum grows by more
//    than 2^8 (exact: the same reference maximum is used for numerator and
//    denominator).
//  * P (bf16) is written to shared memory in the 128-byte-swizzled K-major
//    layout the MMA reads; V is consumed directly as an MN-major operand.
//  * Q and K/V tiles come through 4-D TMA maps whose extents stop at `seq`
//    and `start_pos + seq`, so rows past the valid range read as zeros and no
//    unwritten cache entry is ever touched.
//  * Causal tile skipping: a query tile visits only key tiles up to its last
//    position; work units are issued longest first.
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
};

template <int HD>
struct FlashCfg {
  static constexpr int CHUNKS = (HD + 63) / 64;     // 64-element (128-byte) slabs of a head
  static constexpr int TILE_BYTES = 128 * 128;      // one [128 rows x 64 elems] bf16 slab
  static constexpr int Q_BYTES = CHUNKS * TILE_BYTES;
  static constexpr int KV_BYTES = CHUNKS * TILE_BYTES;
  static constexpr int P_BYTES = 2 * TILE_BYTES;    // 128 rows x 128 keys
  static constexpr int KST = 1, VST = 2;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + 2 * Q_BYTES;
  static constexpr int OFF_V = OFF_K + KST * KV_BYTES;
  static constexpr int OFF_P = OFF_V + VST * KV_BYTES;
  static constexpr int OFF_BAR = OFF_P + 2 * P_BYTES;
  static constexpr int N_BARS = 2 /*q_full*/ + 2 /*q_empty*/ + 2 * KST + 2 * VST + 2 /*s_full*/ +
                                2 /*p_full*/ + 2 /*o_done*/;
  static constexpr int SMEM_BYTES = 1024 + OFF_BAR + N_BARS * 8 + 16;
  static constexpr int KSTEPS_QK = HD / 16;   // MMA K-steps over the head dimension
  static_assert(SMEM_BYTES <= 232448, "shared memory");
  static_assert(HD % 32 == 0 && HD <= 128, "head_dim");
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

template <int HD>
__global__ void __launch_bounds__(384, 1)
    flash_attention_kernel(const __grid_constant__ CUtensorMap mapQ, const __grid_constant__ CUtensorMap mapK,
                           const __grid_constant__ CUtensorMap mapV, bf16* __restrict__ out, const FlashShape fs,
                           const unsigned long long wait_ns) {
  using C = FlashCfg<HD>;
  constexpr uint32_t IDESC_S = idesc_bf16_f32(128, 128, 0, 0);
  constexpr uint32_t IDESC_O = idesc_bf16_f32(128, HD, 0, 1);   // V is MN-major (hd contiguous)

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
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(o_done + 2);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < 2; ++s) {
      mbar_init(&q_full[s], 1); mbar_init(&q_empty[s], 1);
      mbar_init(&s_full[s], 1); mbar_init(&p_full[s], 128); mbar_init(&o_done[s], 1);
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
  const uint32_t tmem_base = *tmem_slot;
  griddep_wait_and_release();

  if (warp == 0) {
    // ---------------------------------------------------------------- producer
    if (lane == 0) {
      int ks = 0, vs = 0;
      uint32_t kph = 0, vph = 0, qph[2] = {0, 0};
      bool ok = true;
      uint32_t kiss = 0, kpar = 0, viss = 0, vpar = 0, qiss = 0, qpar = 0;
      for (int k_ = 0, u = flash_snake(0); u < fs.units && ok; u = flash_snake(++k_)) {
        int b, g, pair, qt;
        flash_unit(fs, u, b, g, pair, qt);
        const int nt = flash_ntiles(fs, qt);
        const bool has1 = pair * 2 + 1 < fs.n_rep;
        for (int s = 0; s < 2 && ok; ++s) {
          if (s == 1 && !has1) break;
          if (!mbar_wait(&q_empty[s], qph[s] ^ 1u, wait_ns)) { ok = false; break; }
          mbar_arrive_expect_tx(&q_full[s], C::Q_BYTES);
          const int h = g * fs.n_rep + pair * 2 + s;
          for (int c = 0; c < C::CHUNKS; ++c)
            tma_load_4d(smem + C::OFF_Q + s * C::Q_BYTES + c * C::TILE_BYTES, &mapQ, &q_full[s], c * 64, h,
                        qt * 128, b);
          qiss |= 1u << s; qpar = (qpar & ~(1u << s)) | (qph[s] << s);
          qph[s] ^= 1u;
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
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      int ks = 0, vs = 0;
      uint32_t kph = 0, vph = 0, qph[2] = {0, 0};
      uint32_t pph[2] = {0, 0};
      bool ok = true;
      const uint32_t q_addr = smem_u32(smem + C::OFF_Q);
      const uint32_t p_addr = smem_u32(smem + C::OFF_P);
      auto issue_s = [&](int s, int kst) {
        const uint32_t d = tmem_base + s * 256;
        const uint32_t qa = q_addr + s * C::Q_BYTES;
        const uint32_t ka = smem_u32(smem + C::OFF_K + kst * C::KV_BYTES);
#pragma unroll
        for (int k = 0; k < C::KSTEPS_QK; ++k) {
          const uint32_t off = (k >> 2) * C::TILE_BYTES + (k & 3) * 32;
          tc_mma_f16_ss(d, sw128_desc(qa + off, 1024, 16), sw128_desc(ka + off, 1024, 16), IDESC_S, k > 0);
        }
        tc_commit(&s_full[s]);
      };
      auto issue_pv = [&](int s, int vst, bool accumulate) {
        const uint32_t d = tmem_base + s * 256 + 128;
        const uint32_t pa = p_addr + s * C::P_BYTES;
        const uint32_t va = smem_u32(smem + C::OFF_V + vst * C::KV_BYTES);
#pragma unroll
        for (int k = 0; k < 8; ++k) {   // 128 keys, 16 per MMA
          const uint64_t adesc = sw128_desc(pa + (k >> 2) * C::TILE_BYTES + (k & 3) * 32, 1024, 16);
          const uint64_t bdesc = sw128_desc(va + k * 2048, 1024, C::TILE_BYTES);
          tc_mma_f16_ss(d, adesc, bdesc, IDESC_O, (accumulate || k > 0) ? 1u : 0u);
        }
        tc_commit(&o_done[s]);
      };
      for (int k_ = 0, u = flash_snake(0); u < fs.units && ok; u = flash_snake(++k_)) {
        int b, g, pair, qt;
        flash_unit(fs, u, b, g, pair, qt);
        const int nt = flash_ntiles(fs, qt);
        const int nslots = (pair * 2 + 1 < fs.n_rep) ? 2 : 1;
        for (int s = 0; s < nslots; ++s) {
          if (!mbar_wait(&q_full[s], qph[s], wait_ns)) ok = false;
          qph[s] ^= 1u;
        }
        if (!ok) break;
        tc_fence_after();
        const int jt0 = flash_first_tile(fs, b, qt);
        // S of the first key tile for every slot
        if (!mbar_wait(&k_full[ks], kph, wait_ns)) break;
        tc_fence_after();
        for (int s = 0; s < nslots; ++s) issue_s(s, ks);
        tc_commit(&k_empty[ks]);
        if (++ks == C::KST) { ks = 0; kph ^= 1u; }
        for (int j = jt0; j < nt && ok; ++j) {
          if (!mbar_wait(&v_full[vs], vph, wait_ns)) { ok = false; break; }
          const bool more = j + 1 < nt;
          bool k_ready = false;
          for (int s = 0; s < nslots; ++s) {
            if (!mbar_wait(&p_full[s], pph[s], wait_ns)) { ok = false; break; }
            pph[s] ^= 1u;
            tc_fence_after();
            issue_pv(s, vs, j > jt0);
            if (more) {
              // K of the next tile is only needed from here on: P.V above does not wait for it
              if (!k_ready && !mbar_wait(&k_full[ks], kph, wait_ns)) { ok = false; break; }
              k_ready = true;
              tc_fence_after();
              issue_s(s, ks);
            }
          }
          if (!ok) break;
          tc_commit(&v_empty[vs]);
          if (++vs == C::VST) { vs = 0; vph ^= 1u; }
          if (more) {
            tc_commit(&k_empty[ks]);
            if (++ks == C::KST) { ks = 0; kph ^= 1u; }
          }
        }
        for (int s = 0; s < nslots; ++s) tc_commit(&q_empty[s]);
      }
    }
  } else if (warp >= 4) {
    // ---------------------------------------------------------------- softmax
    const int slot = (warp - 4) >> 2;
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;            // query row in the tile == TMEM lane
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const uint32_t s_tmem = tmem_base + lane_off + slot * 256;
    const uint32_t o_tmem = s_tmem + 128;
    uint8_t* p_smem = smem + C::OFF_P + slot * C::P_BYTES;
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
        if (!mbar_wait(&s_full[slot], sph, wait_ns)) { ok = false; break; }
        sph ^= 1u;
        tc_fence_after();
        const bool need_mask = j * 128 + 127 > fs.P + qt * 128 || j * 128 < lo_last;
        // pass 1: row maximum of the raw scores (the next chunk's TMEM load is
        // in flight while the current one is reduced)
        float mx = -INFINITY;
        {
          uint32_t ra[32], rb[32];
          tmem_ld32(s_tmem, ra);
          tc_wait_ld();
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            uint32_t(&cur)[32] = (c & 1) ? rb : ra;
            uint32_t(&nxt)[32] = (c & 1) ? ra : rb;
            if (c + 1 < 4) tmem_ld32(s_tmem + (c + 1) * 32, nxt);
            if (need_mask) {
#pragma unroll
              for (int i = 0; i < 32; ++i)
                if (j * 128 + c * 32 + i > qpos || j * 128 + c * 32 + i < lo) cur[i] = __float_as_uint(-INFINITY);
            }
#pragma unroll
            for (int i = 0; i < 32; i += 2) mx = max3f(mx, __uint_as_float(cur[i]), __uint_as_float(cur[i + 1]));
            if (c + 1 < 4) tc_wait_ld();
          }
        }
        const float m_tile = mx * fs.scale_log2;   // scale_log2 > 0: max commutes with the scale
        // the O written by the previous tile's P.V must be complete before P
        // (single buffer) is overwritten or O is rescaled
        if (j > jt0) {
          if (!mbar_wait(&o_done[slot], oph, wait_ns)) { ok = false; break; }
          oph ^= 1u;
          tc_fence_after();
        }
        const bool grow = m_tile > m_ref + 8.0f;
        float alpha = 1.f;
        if (grow) {
          alpha = exp2f(m_ref - m_tile);   // 0 on the first tile
          l *= alpha;
          m_ref = m_tile;
        }
        // rescale this warp's rows of O in TMEM when any of them grew (the
        // TMEM accesses are warp-collective; rows that did not grow use 1)
        if (j > jt0 && __any_sync(0xffffffffu, grow)) {
#pragma unroll 1
          for (int c = 0; c < HD / 16; ++c) {
            uint32_t r[16];
            tmem_ld16(o_tmem + c * 16, r);
            tc_wait_ld();
#pragma unroll
            for (int i = 0; i < 16; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * alpha);
            tmem_st16(o_tmem + c * 16, r);
          }
          tc_wait_st();
        }
        // pass 2: p = 2^(s*scale - m_ref), row sum, bf16 P into shared memory
        // (again with the next chunk's TMEM load overlapping this chunk's math)
        const float scl = fs.scale_log2;
        const float neg_m = m_ref == -INFINITY ? 0.f : -m_ref;   // a row with no visible key yet: p = 0
        float sum_a = 0.f, sum_b = 0.f;
        {
          uint32_t ra[32], rb[32];
          tmem_ld32(s_tmem, ra);
          tc_wait_ld();
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            uint32_t(&r)[32] = (c & 1) ? rb : ra;
            uint32_t(&nxt)[32] = (c & 1) ? ra : rb;
            if (c + 1 < 4) tmem_ld32(s_tmem + (c + 1) * 32, nxt);
            if (need_mask) {
#pragma unroll
              for (int i = 0; i < 32; ++i)
                if (j * 128 + c * 32 + i > qpos || j * 128 + c * 32 + i < lo) r[i] = __float_as_uint(-INFINITY);
            }
            uint32_t pk[16];
            if (need_mask) {   // masked keys must give exactly 0: MUFU path only
#pragma unroll
              for (int i = 0; i < 16; ++i) {
                float x0, x1;
                fma2(x0, x1, __uint_as_float(r[2 * i]), __uint_as_float(r[2 * i + 1]), scl, scl, neg_m, neg_m);
                const float p0 = ex2_approx(x0), p1 = ex2_approx(x1);
                add2(sum_a, sum_b, p0, p1);
                pk[i] = pack_bf16x2(p0, p1);
              }
            } else {           // 6 of every 16 pairs on the FMA pipe, the rest on MUFU
#pragma unroll
              for (int i = 0; i < 16; ++i) {
                float x0, x1, p0, p1;
                fma2(x0, x1, __uint_as_float(r[2 * i]), __uint_as_float(r[2 * i + 1]), scl, scl, neg_m, neg_m);
                if ((i & 7) < 3) {
                  exp2_poly2(x0, x1, p0, p1);
                } else {
                  p0 = ex2_approx(x0);
                  p1 = ex2_approx(x1);
                }
                add2(sum_a, sum_b, p0, p1);
                pk[i] = pack_bf16x2(p0, p1);
              }
            }
            // chunk c covers keys 32c..32c+31: slab c/2, 16-byte pieces (c%2)*4 .. +3
            uint8_t* slab = p_smem + (c >> 1) * C::TILE_BYTES + row * 128;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const int piece = (c & 1) * 4 + q;
              *reinterpret_cast<uint4*>(slab + ((piece ^ (row & 7)) << 4)) =
                  make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
            }
            if (c + 1 < 4) tc_wait_ld();
          }
        }
        const float sum = sum_a + sum_b;
        l += sum;
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(&p_full[slot]);
      }
      if (!ok) break;
      // epilogue: wait for the last P.V, out = O / l
      if (!mbar_wait(&o_done[slot], oph, wait_ns)) break;
      oph ^= 1u;
      tc_fence_after();
      const int t = qt * 128 + row;
      const int h = g * fs.n_rep + pair * 2 + slot;
      const float inv = 1.f / l;
      bf16* orow = out + ((size_t)b * fs.S + t) * fs.ldo + (size_t)h * HD;
#pragma unroll 1
      for (int c = 0; c < HD / 32; ++c) {
        uint32_t r[32];
        tmem_ld32(o_tmem + c * 32, r);
        tc_wait_ld();
        if (t < fs.S) {
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            uint4 o;
            o.x = pack_bf16x2(__uint_as_float(r[8 * q + 0]) * inv, __uint_as_float(r[8 * q + 1]) * inv);
            o.y = pack_bf16x2(__uint_as_float(r[8 * q + 2]) * inv, __uint_as_float(r[8 * q + 3]) * inv);
            o.z = pack_bf16x2(__uint_as_float(r[8 * q + 4]) * inv, __uint_as_float(r[8 * q + 5]) * inv);
            o.w = pack_bf16x2(__uint_as_float(r[8 * q + 6]) * inv, __uint_as_float(r[8 * q + 7]) * inv);
            *reinterpret_cast<uint4*>(orow + c * 32 + q * 8) = o;
          }
        }
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
