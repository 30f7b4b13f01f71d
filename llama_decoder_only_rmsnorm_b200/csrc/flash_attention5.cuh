// flash_attention5.cuh -- causal GQA prefill attention, tcgen05, fifth design.
//
// Computes the same thing as flash_attention.cuh ("Build your own Llama 3 from
// scratch" §3.4; document mask of 附 1), with the producer, MMA issuer, TMEM
// layout and register split of the third design.  What changes is who runs
// the softmax of a key tile: in the third design each softmax warpgroup owns
// one head and sits idle while its head's P.V and next S run, so on every
// SM sub-partition only one softmax warp is busy at a time.  Here both
// warpgroups work on the same tile -- the first on keys 0-63, the second on
// keys 64-127 of every query row -- and then together on the other head's
// tile.  A row's two halves meet twice per tile and head: their partial
// maxima are exchanged through shared memory behind a bounded mbarrier (one
// per lane quarter and parity), and at the end of a work unit their partial
// row sums.  Each half writes its P pairs into its own 32 TMEM columns (keys
// 0-63 -> columns 0-31, keys 64-127 -> columns 32-63, the layout P.V reads)
// and rescales and stores its half of O's columns.
#pragma once
#include "flash_attention3.cuh"

namespace l3 {

template <int HD>
struct Flash5Cfg {
  using B3 = Flash3Cfg<HD>;   // same Q/K/V ring layout as the third design
  static constexpr int OFF_X = B3::OFF_V + B3::VST * B3::KV_BYTES;   // [parity][half][128 rows] floats
  static constexpr int X_BYTES = 2 * 2 * 128 * 4;
  static constexpr int OFF_BAR = OFF_X + X_BYTES;
  static constexpr int N_BARS = B3::N_BARS + 8;                       // + exchange [quarter][parity]
  static constexpr int SMEM_BYTES = 1024 + OFF_BAR + N_BARS * 8 + 16;
  static_assert(SMEM_BYTES <= 232448, "shared memory");
  static_assert(HD % 32 == 0 && HD <= 128, "head_dim");
};

template <int HD>
__global__ void __launch_bounds__(kFlash3Threads, 1)
    flash_attention5_kernel(const __grid_constant__ CUtensorMap mapQ, const __grid_constant__ CUtensorMap mapK,
                            const __grid_constant__ CUtensorMap mapV, bf16* __restrict__ out, const FlashShape fs,
                            const unsigned long long wait_ns) {
  using C = Flash5Cfg<HD>;
  using C3 = Flash3Cfg<HD>;
  constexpr int OH = HD / 2;   // O columns per half

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* q_full = bars;
  uint64_t* q_empty = q_full + 2;
  uint64_t* k_full = q_empty + 2;
  uint64_t* k_empty = k_full + C3::KST;
  uint64_t* v_full = k_empty + C3::KST;
  uint64_t* v_empty = v_full + C3::VST;
  uint64_t* s_full = v_empty + C3::VST;
  uint64_t* p_full = s_full + 2;
  uint64_t* o_done = p_full + 2;
  uint64_t* xbar = o_done + 2;   // [quarter][parity]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(xbar + 8);
  const Flash3Bars bars3{q_full, q_empty, k_full, k_empty, v_full, v_empty, s_full, p_full, o_done};

  const int warp = __shfl_sync(0xffffffffu, (int)(threadIdx.x >> 5), 0), lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < 2; ++s) {
      mbar_init(&q_full[s], 1); mbar_init(&q_empty[s], 1);
      mbar_init(&s_full[s], 1); mbar_init(&p_full[s], 256); mbar_init(&o_done[s], 1);
    }
    for (int s = 0; s < C3::KST; ++s) { mbar_init(&k_full[s], 1); mbar_init(&k_empty[s], 1); }
    for (int s = 0; s < C3::VST; ++s) { mbar_init(&v_full[s], 1); mbar_init(&v_empty[s], 1); }
    for (int i = 0; i < 8; ++i) mbar_init(&xbar[i], 64);
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
  if (warp < 4) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;\n" ::"n"(kFlash3LowRegs));
    griddep_wait_and_release();
    if (warp == 0) {
      if (lane == 0) flash3_produce<HD>(mapQ, mapK, mapV, smem, bars3, fs, wait_ns);
    } else if (warp == 1) {
      flash3_issue_mma<HD>(smem, bars3, tmem_base, fs, wait_ns);
    }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;\n" ::"n"(kFlash3HighRegs));
    griddep_wait_and_release();
    // ---------------------------------------------------------------- softmax (two threads per row)
    const int half = (warp - 4) >> 2;               // keys [64*half, 64*half + 64) of every tile
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;            // query row in the tile == TMEM lane
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    float* xch = reinterpret_cast<float*>(smem + C::OFF_X);
    uint32_t xs = 0;   // exchanges done (the same count in both halves)
    // Hand v to the other half of this row and take its value back.
    auto exchange = [&](float v, float& other) -> bool {
      const uint32_t par = xs & 1u;
      xch[(par * 2 + half) * 128 + row] = v;
      tc_fence_before();   // this thread's TMEM reads come before the partner's writes
      mbar_arrive(&xbar[quarter * 2 + par]);
      const bool r = mbar_wait_warp(&xbar[quarter * 2 + par], (xs >> 1) & 1u, wait_ns);
      tc_fence_after();
      other = xch[(par * 2 + (half ^ 1)) * 128 + row];
      ++xs;
      return r;
    };
    uint32_t sph = 0, oph = 0;   // phase bit per head slot
    bool ok = true;
    for (int k_ = 0, u = flash_snake(0); u < fs.units && ok; u = flash_snake(++k_)) {
      int b, g, pair, qt;
      flash_unit(fs, u, b, g, pair, qt);
      const int nslots = (pair * 2 + 1 < fs.n_rep) ? 2 : 1;
      const int nt = flash_ntiles(fs, qt);
      const int jt0 = flash_first_tile(fs, b, qt);
      const int qpos = fs.P + qt * 128 + row;
      const int lo = flash_row_lo(fs, b, qt * 128 + row);
      const int lo_last = flash_row_lo(fs, b, qt * 128 + 127);   // largest lower bound in the tile
      float m_ref[2] = {-INFINITY, -INFINITY}, l[2] = {0.f, 0.f};
      for (int j = jt0; j < nt && ok; ++j) {
        const bool need_mask = j * 128 + 127 > fs.P + qt * 128 || j * 128 < lo_last;
        const int key0 = j * 128 + half * 64;
#pragma unroll
        for (int s = 0; s < 2; ++s) {
          if (s >= nslots) break;
          const uint32_t s_tmem = tmem_base + lane_off + s * 256;
          const uint32_t o_tmem = s_tmem + 128 + half * OH;
          if (!mbar_wait_warp(&s_full[s], (sph >> s) & 1u, wait_ns)) { ok = false; break; }
          sph ^= 1u << s;
          tc_fence_after();
          uint32_t ra[32], rb[32];
          tmem_ld32(s_tmem + half * 64, ra);
          tmem_ld32(s_tmem + half * 64 + 32, rb);
          tc_wait_ld();
          float m0, m1;
          if (need_mask) {
            m0 = flash3_row_max<true>(ra, key0, qpos, lo);
            m1 = flash3_row_max<true>(rb, key0 + 32, qpos, lo);
          } else {
            m0 = flash3_row_max<false>(ra, key0, qpos, lo);
            m1 = flash3_row_max<false>(rb, key0 + 32, qpos, lo);
          }
          const float mine = fmaxf(m0, m1);
          float theirs;
          // Both halves have read their S columns once this exchange is
          // through, so from here on the second half may write P over
          // columns 32-63, which held keys 32-63 of the first half.
          if (!exchange(mine, theirs)) { ok = false; break; }
          const float m_tile = fmaxf(mine, theirs) * fs.scale_log2;   // scale_log2 > 0
          // The previous tile's P.V is complete (the s_full commit tracks it);
          // only its o_done phase is counted, for the epilogue's wait.
          if (j > jt0) oph ^= 1u << s;
          const bool grow = m_tile > m_ref[s] + 8.0f;
          float alpha = 1.f;
          if (grow) {
            alpha = exp2f(m_ref[s] - m_tile);   // 0 on the first tile
            l[s] *= alpha;
            m_ref[s] = m_tile;
          }
          if (j > jt0 && __any_sync(0xffffffffu, grow)) {
#pragma unroll 1
            for (int c = 0; c < OH / 16; ++c) {
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
          const float neg_m = m_ref[s] == -INFINITY ? 0.f : -m_ref[s];   // no visible key yet: p = 0
          float s0 = 0.f, s1 = 0.f, s2 = 0.f, s3 = 0.f;
          if (need_mask) {
            flash3_exp_inplace<true>(ra, scl, neg_m, s0, s1);
            flash3_exp_inplace<true>(rb, scl, neg_m, s2, s3);
          } else {
            flash3_exp_inplace<false>(ra, scl, neg_m, s0, s1);
            flash3_exp_inplace<false>(rb, scl, neg_m, s2, s3);
          }
          flash3_pack_store(ra, s_tmem + half * 32);
          flash3_pack_store(rb, s_tmem + half * 32 + 16);
          l[s] += (s0 + s1) + (s2 + s3);
          tc_wait_st();
          tc_fence_before();
          mbar_arrive(&p_full[s]);
        }
      }
      if (!ok) break;
      // epilogue per head: wait for its last P.V, out = O / (l_first + l_second)
#pragma unroll
      for (int s = 0; s < 2; ++s) {
        if (s >= nslots) break;
        if (!mbar_wait_warp(&o_done[s], (oph >> s) & 1u, wait_ns)) { ok = false; break; }
        oph ^= 1u << s;
        tc_fence_after();
        float l_other;
        if (!exchange(l[s], l_other)) { ok = false; break; }
        const float inv = 1.f / (half == 0 ? l[s] + l_other : l_other + l[s]);
        const int t = qt * 128 + row;
        const int h = g * fs.n_rep + pair * 2 + s;
        const uint32_t o_tmem = tmem_base + lane_off + s * 256 + 128 + half * OH;
        bf16* orow = out + ((size_t)b * fs.S + t) * fs.ldo + (size_t)h * HD + half * OH;
#pragma unroll 1
        for (int c = 0; c < OH / 16; ++c) {
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
