// flash_attention2.cuh -- causal GQA prefill attention, tcgen05, second design.
//
// Computes the same thing as flash_attention.cuh ("Build your own Llama 3 from
// scratch" §3.4; document mask of 附 1), with three changes aimed at the
// softmax, which bounds the first design:
//  * every query row is shared by two softmax warps from two warpgroups
//    (TMEM lanes can be read by the warps of any warpgroup that sit in the
//    same lane quarter), each taking 64 of the tile's 128 scores; the two
//    exchange their partial row maxima (and, at the end, row sums) through
//    shared memory behind a bounded mbarrier;
//  * P is written back into TMEM over scores already consumed (keys 0-63 into
//    columns 0-31, keys 64-127 into columns 64-95, two bf16 per column) and
//    P.V reads its A operand from TMEM, so P never touches shared memory;
//  * with shared memory freed, K and V tiles are both double-buffered.
// Two query heads of a KV group share every K/V tile, as before.
#pragma once
#include "flash_attention.cuh"

namespace l3 {

template <int HD>
struct Flash2Cfg {
  static constexpr int CHUNKS = (HD + 63) / 64;
  static constexpr int TILE_BYTES = 128 * 128;
  static constexpr int Q_BYTES = CHUNKS * TILE_BYTES;
  static constexpr int KV_BYTES = CHUNKS * TILE_BYTES;
  static constexpr int KST = 2, VST = 2;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + 2 * Q_BYTES;
  static constexpr int OFF_V = OFF_K + KST * KV_BYTES;
  static constexpr int OFF_X = OFF_V + VST * KV_BYTES;     // exchange [slot][quarter][half][parity][32] floats
  static constexpr int X_BYTES = 2 * 4 * 2 * 2 * 32 * 4;
  static constexpr int OFF_BAR = OFF_X + X_BYTES;
  static constexpr int N_BARS = 2 + 2 + 2 * KST + 2 * VST + 2 + 2 + 2 + 16;
  static constexpr int SMEM_BYTES = 1024 + OFF_BAR + N_BARS * 8 + 16;
  static constexpr int OCOLS = HD / 2;                    // O columns per softmax half
  static_assert(SMEM_BYTES <= 232448, "shared memory");
  static_assert(HD % 32 == 0 && HD <= 128, "head_dim");
};

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

template <int HD>
__global__ void __launch_bounds__(640, 1)
    flash_attention2_kernel(const __grid_constant__ CUtensorMap mapQ, const __grid_constant__ CUtensorMap mapK,
                            const __grid_constant__ CUtensorMap mapV, bf16* __restrict__ out, const FlashShape fs,
                            const unsigned long long wait_ns) {
  using C = Flash2Cfg<HD>;
  constexpr uint32_t IDESC_S = idesc_bf16_f32(128, 128, 0, 0);
  constexpr uint32_t IDESC_O = idesc_bf16_f32(128, HD, 0, 1);   // A = P (TMEM), B = V MN-major

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  float* xch = reinterpret_cast<float*>(smem + C::OFF_X);
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
  uint64_t* xbar = o_done + 2;    // [slot][quarter][parity]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(xbar + 16);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < 2; ++s) {
      mbar_init(&q_full[s], 1); mbar_init(&q_empty[s], 1);
      mbar_init(&s_full[s], 1); mbar_init(&p_full[s], 256); mbar_init(&o_done[s], 1);
    }
    for (int s = 0; s < C::KST; ++s) { mbar_init(&k_full[s], 1); mbar_init(&k_empty[s], 1); }
    for (int s = 0; s < C::VST; ++s) { mbar_init(&v_full[s], 1); mbar_init(&v_empty[s], 1); }
    for (int i = 0; i < 16; ++i) mbar_init(&xbar[i], 2);
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
      // S of the next tile overwrites the TMEM columns that hold P.  It is
      // issued right behind the P.V that reads them, without waiting for that
      // P.V to complete: the MMAs one thread issues execute in issue order, so
      // every read of P precedes the first write of the next S.
      const uint32_t q_addr = smem_u32(smem + C::OFF_Q);
      auto issue_s = [&](int s, int kst) {
        const uint32_t d = tmem_base + s * 256;
        const uint32_t qa = q_addr + s * C::Q_BYTES;
        const uint32_t ka = smem_u32(smem + C::OFF_K + kst * C::KV_BYTES);
#pragma unroll
        for (int k = 0; k < HD / 16; ++k) {
          const uint32_t off = (k >> 2) * C::TILE_BYTES + (k & 3) * 32;
          tc_mma_f16_ss(d, sw128_desc(qa + off, 1024, 16), sw128_desc(ka + off, 1024, 16), IDESC_S, k > 0);
        }
        tc_commit(&s_full[s]);
      };
      auto issue_pv = [&](int s, int vst, bool accumulate) {
        const uint32_t d = tmem_base + s * 256 + 128;
        const uint32_t pa = tmem_base + s * 256;
        const uint32_t va = smem_u32(smem + C::OFF_V + vst * C::KV_BYTES);
#pragma unroll
        for (int k = 0; k < 8; ++k) {   // 16 keys per MMA: P keys 16k.. sit in columns (k<4 ? 8k : 64+8(k-4))
          const uint32_t a = pa + (k < 4 ? k * 8 : 64 + (k - 4) * 8);
          const uint64_t bdesc = sw128_desc(va + k * 2048, 1024, C::TILE_BYTES);
          tc_mma_f16_ts(d, a, bdesc, IDESC_O, (accumulate || k > 0) ? 1u : 0u);
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
              if (!k_ready && !mbar_wait(&k_full[ks], kph, wait_ns)) { ok = false; break; }
              k_ready = true;
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
    // ---------------------------------------------------------------- softmax halves
    const int idx = warp - 4;
    const int slot = idx >> 3, half = (idx >> 2) & 1, quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const uint32_t s_tmem = tmem_base + lane_off + slot * 256;
    const uint32_t o_tmem = s_tmem + 128 + half * C::OCOLS;
    uint32_t sph = 0, oph = 0, xph = 0;   // xph: phase bit of each exchange barrier
    int xpar = 0;
    // swap one float per row with the partner warp (other half, same lanes)
    auto exchange = [&](float mine, float& theirs) -> bool {
      float* base = xch + (((slot * 4 + quarter) * 2) * 2 + xpar) * 32;   // [..][half][parity][32]
      base[half * 64 + lane] = mine;
      __syncwarp();
      uint64_t* bar = &xbar[(slot * 4 + quarter) * 2 + xpar];
      if (lane == 0) mbar_arrive(bar);
      const bool done = mbar_wait(bar, (xph >> xpar) & 1u, wait_ns);
      xph ^= 1u << xpar;
      theirs = base[(1 - half) * 64 + lane];
      xpar ^= 1;
      return done;
    };
    for (int k_ = 0, u = flash_snake(0); u < fs.units; u = flash_snake(++k_)) {
      int b, g, pair, qt;
      flash_unit(fs, u, b, g, pair, qt);
      if (slot == 1 && !(pair * 2 + 1 < fs.n_rep)) continue;
      const int nt = flash_ntiles(fs, qt);
      const int jt0 = flash_first_tile(fs, b, qt);
      const int qpos = fs.P + qt * 128 + row;
      const int lo = flash_row_lo(fs, b, qt * 128 + row);
      const int lo_last = flash_row_lo(fs, b, qt * 128 + 127);
      float m_ref = -INFINITY, l = 0.f;
      bool ok = true;
      for (int j = jt0; j < nt; ++j) {
        if (!mbar_wait(&s_full[slot], sph, wait_ns)) { ok = false; break; }
        sph ^= 1u;
        tc_fence_after();
        const bool need_mask = j * 128 + 127 > fs.P + qt * 128 || j * 128 < lo_last;
        const int key0 = j * 128 + half * 64;
        // pass 1: maximum of this half's 64 raw scores
        float mx = -INFINITY;
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          uint32_t r[32];
          tmem_ld32(s_tmem + half * 64 + c * 32, r);
          tc_wait_ld();
          if (need_mask) {
#pragma unroll
            for (int i = 0; i < 32; ++i)
              if (key0 + c * 32 + i > qpos || key0 + c * 32 + i < lo) r[i] = __float_as_uint(-INFINITY);
          }
#pragma unroll
          for (int i = 0; i < 32; i += 2) mx = max3f(mx, __uint_as_float(r[i]), __uint_as_float(r[i + 1]));
        }
        float other;
        if (!exchange(mx, other)) { ok = false; break; }
        const float m_tile = fmaxf(mx, other) * fs.scale_log2;
        if (j > jt0) {   // the previous P.V (same slot) is complete: O may be rescaled
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
        if (j > jt0 && __any_sync(0xffffffffu, grow)) {
#pragma unroll 1
          for (int c = 0; c < C::OCOLS / 16; ++c) {
            uint32_t o[16];
            tmem_ld16(o_tmem + c * 16, o);
            tc_wait_ld();
#pragma unroll
            for (int i = 0; i < 16; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
            tmem_st16(o_tmem + c * 16, o);
          }
          tc_wait_st();
        }
        // pass 2: p = 2^(s*scale - m_ref) -> bf16 pairs back into TMEM over the
        // scores just read (keys 64h + 32c.. -> columns 64h + 16c..)
        const float scl = fs.scale_log2;
        const float neg_m = m_ref == -INFINITY ? 0.f : -m_ref;   // a row with no visible key yet: p = 0
        float sum_a = 0.f, sum_b = 0.f;
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          uint32_t r[32];
          tmem_ld32(s_tmem + half * 64 + c * 32, r);
          tc_wait_ld();
          if (need_mask) {
#pragma unroll
            for (int i = 0; i < 32; ++i)
              if (key0 + c * 32 + i > qpos || key0 + c * 32 + i < lo) r[i] = __float_as_uint(-INFINITY);
          }
          uint32_t pk[16];
          if (need_mask) {
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              float x0, x1;
              fma2(x0, x1, __uint_as_float(r[2 * i]), __uint_as_float(r[2 * i + 1]), scl, scl, neg_m, neg_m);
              const float p0 = ex2_approx(x0), p1 = ex2_approx(x1);
              add2(sum_a, sum_b, p0, p1);
              pk[i] = pack_bf16x2(p0, p1);
            }
          } else {
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
          tmem_st16(s_tmem + half * 64 + c * 16, pk);
        }
        l += sum_a + sum_b;
        tc_wait_st();
        tc_fence_before();
        mbar_arrive(&p_full[slot]);
      }
      if (!ok) break;
      // epilogue: last P.V, the row sum over both halves, out = O / l
      if (!mbar_wait(&o_done[slot], oph, wait_ns)) break;
      oph ^= 1u;
      tc_fence_after();
      float l_other;
      if (!exchange(l, l_other)) break;
      const float inv = 1.f / (l + l_other);
      const int t = qt * 128 + row;
      const int h = g * fs.n_rep + pair * 2 + slot;
      bf16* orow = out + ((size_t)b * fs.S + t) * fs.ldo + (size_t)h * HD + half * C::OCOLS;
#pragma unroll 1
      for (int c = 0; c < C::OCOLS / 16; ++c) {
        uint32_t r[16];
        tmem_ld16(o_tmem + c * 16, r);
        tc_wait_ld();
        if (t < fs.S) {
#pragma unroll
          for (int q = 0; q < 2; ++q) {
            uint4 o;
            o.x = pack_bf16x2(__uint_as_float(r[8 * q + 0]) * inv, __uint_as_float(r[8 * q + 1]) * inv);
            o.y = pack_bf16x2(__uint_as_float(r[8 * q + 2]) * inv, __uint_as_float(r[8 * q + 3]) * inv);
            o.z = pack_bf16x2(__uint_as_float(r[8 * q + 4]) * inv, __uint_as_float(r[8 * q + 5]) * inv);
            o.w = pack_bf16x2(__uint_as_float(r[8 * q + 6]) * inv, __uint_as_float(r[8 * q + 7]) * inv);
            *reinterpret_cast<uint4*>(orow + c * 16 + q * 8) = o;
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
