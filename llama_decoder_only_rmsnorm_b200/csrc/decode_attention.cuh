// decode_attention.cuh -- one new query token per sequence against the KV cache
// ("Build your own Llama 3 from scratch" §3.3 KV Cache and 六 inference: the
// step's single query attends to every cached position 0..start_pos).
//
// Memory-bound: every cached K and V row is read exactly once per step.  A CTA
// owns (sequence b, KV head g, key range) and serves all n_rep query heads of
// group g from the same K/V rows (GQA, §3.4: head h reads KV head h / n_rep),
// so repeat_kv is never formed.  Key ranges ("splits") spread one sequence
// over many SMs; a second kernel merges the per-split softmax partials.
#pragma once
#include "common.cuh"

namespace l3 {

// Partial record per (b, h, slot): m (running max of the scores, log2 domain),
// l (sum of 2^(s - m)), acc[hd] (sum of 2^(s - m) * v).  Stored as floats
// [B][H][slots][hd + 2] and merged by the combine kernel:
// out[b, h, :] = sum_s e^(m_s - M) acc_s / sum_s e^(m_s - M) l_s over the
// first `used` slots of (b, h) (records_used below).
template <int HD>
__global__ void decode_attention_combine_kernel(const float* __restrict__ part, bf16* __restrict__ out,
                                                int slots, int H, int nrep, int tiles, int per) {
  griddep_wait_and_release();
  const int bh = blockIdx.x;  // b * H + h
  const int seg = (bh / H) * (H / nrep) + (bh % H) / nrep;   // (b, KV head h / nrep)
  const int used = per > 0 ? 2 * ((seg * tiles + tiles - 1) / per - (seg * tiles) / per + 1) : slots;
  const float* p = part + (size_t)bh * slots * (HD + 2);
  float mx = -INFINITY;
  for (int s = 0; s < used; ++s) mx = fmaxf(mx, p[s * (HD + 2)]);
  for (int d = threadIdx.x; d < HD; d += blockDim.x) {
    float num = 0.f, den = 0.f;
    for (int s = 0; s < used; ++s) {
      const float ms = p[s * (HD + 2)];
      const float f = ms == -INFINITY ? 0.f : exp2f(ms - mx);
      den += f * p[s * (HD + 2) + 1];
      num += f * p[s * (HD + 2) + 2 + d];
    }
    out[(size_t)bh * HD + d] = __float2bfloat16_rn(num / den);
  }
}

// ===========================================================================
// Tensor-core kernel.  K/V tiles of 128 keys arrive by TMA (3-stage ring of
// 64 KB for head_dim 128); per tile two tcgen05 MMAs:
//   S^T[key, head] = K_tile[128 x hd] . Q^T          (M = 128 keys, N = 16)
//   O^T[dim, head] += V_tile^T[hd x 128] . P^T       (M = 128 dims, N = 16)
// Keys sit on the MMA's 128-row side, so the n_rep query heads of a group
// (padded to 16 columns) share every K/V byte read.  Two softmax warpgroups
// take alternate tiles, each with its own running (m, l, O^T), so one tile's
// softmax overlaps the next one's; a piece of work therefore yields two
// partial records (slot 2*piece + warpgroup) that the combine kernel merges.
//
// Schedule: the key tiles of all (sequence, KV head) segments, laid end to
// end (segment s = b*KV + g holds tiles s*tiles .. s*tiles + tiles - 1), are
// cut into equal runs of `per` tiles, one per CTA, so every CTA streams the
// same number of K/V bytes.  A run that crosses segment boundaries is split
// there into pieces; piece j of a segment is the part of it that the
// segment's j-th CTA (in run order) covers.
// ===========================================================================
struct DecodeShape {
  int B, H, KV, nrep, n_keys;
  int tiles;      // key tiles per segment: ceil(n_keys / 128)
  int per;        // tiles per CTA run
  int slots;      // records per (b, h): 2 x the most pieces any segment has
  float scale_log2;
  // Optional per-sequence positions (device, [B]): sequence b's token sits at
  // positions[b] and sees keys 0..positions[b] (at most n_keys of them).
  const int32_t* positions;
};

template <int HD>
struct DecodeTcCfg {
  static constexpr int SLAB = 128 * 128;            // 128 rows x 64 bf16
  static constexpr int CHUNKS_K = (HD + 63) / 64;   // slabs holding a K tile
  static constexpr int K_BYTES = CHUNKS_K * SLAB;
  static constexpr int V_BYTES = 2 * SLAB;          // always 128 dims (zero beyond hd)
  static constexpr int STAGE_BYTES = K_BYTES + V_BYTES;
  static constexpr int STAGES = 3;
  static constexpr int Q_SLAB = 16 * 128;           // 16 rows x 64 bf16
  static constexpr int Q_BYTES = CHUNKS_K * Q_SLAB;
  static constexpr int P_BYTES = 2 * Q_SLAB;        // 16 heads x 128 keys
  static constexpr int OFF_STAGE = 0;
  static constexpr int OFF_Q = STAGES * STAGE_BYTES;              // 2 buffers
  static constexpr int OFF_P = OFF_Q + 2 * Q_BYTES;               // [warpgroup][2] buffers
  static constexpr int OFF_RED = OFF_P + 4 * P_BYTES;             // [warpgroup][2][4][16] floats
  static constexpr int OFF_BAR = OFF_RED + 2 * 2 * 4 * 16 * 4;
  // kv full/empty, q full/empty [2], per warpgroup: s_full[2], p_full[2], o_done, red[2]
  static constexpr int N_BARS = 2 * STAGES + 4 + 2 * 7;
  static constexpr int SMEM_BYTES = 1024 + OFF_BAR + N_BARS * 8 + 16;
  static_assert(SMEM_BYTES <= 232448, "shared memory");
};

// Piece `it` of CTA c's run -> sequence b, KV head g, piece index j within
// the segment, key tiles [t0, t1) and the number of keys sequence b sees (nk:
// n_keys, or positions[b] + 1 clamped to [1, n_keys]); false once the run is
// exhausted.  Tiles past a short sequence's last one are dropped, so a piece
// may be empty (t1 == t0): it still writes its (empty) records.
__device__ __forceinline__ bool decode_piece(const DecodeShape& ds, int c, int it, int& b, int& g, int& j, int& t0,
                                             int& t1, int& nk) {
  const long long total = (long long)ds.B * ds.KV * ds.tiles;
  const long long a = (long long)c * ds.per, e = min(a + ds.per, total);
  if (a >= e) return false;
  const long long seg = a / ds.tiles + it;
  const long long s0 = seg * ds.tiles;
  if (s0 >= e) return false;
  g = (int)(seg % ds.KV);
  b = (int)(seg / ds.KV);
  j = c - (int)(s0 / ds.per);
  nk = ds.positions ? max(1, min(ds.positions[b] + 1, ds.n_keys)) : ds.n_keys;
  const int own = (nk + 127) / 128;
  t0 = (int)max(a - s0, 0LL);
  t1 = (int)min(e - s0, (long long)ds.tiles);
  t1 = max(t0, min(t1, own));
  return true;
}

template <int HD, int NREP>
__global__ void __launch_bounds__(384, 1)
    decode_attention_tc_kernel(const __grid_constant__ CUtensorMap mapQ, const __grid_constant__ CUtensorMap mapK,
                               const __grid_constant__ CUtensorMap mapV, float* __restrict__ part,
                               const DecodeShape ds, const unsigned long long wait_ns) {
  using C = DecodeTcCfg<HD>;
  static_assert(NREP >= 1 && NREP <= 16, "query heads per KV head (upper bound)");
  const int nrep = ds.nrep;   // <= NREP
  constexpr uint32_t IDESC_S = idesc_bf16_f32(128, 16, 0, 0);
  constexpr uint32_t IDESC_O = idesc_bf16_f32(128, 16, 1, 0);   // V^T: dims contiguous (MN-major A)

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* kv_full = bars;
  uint64_t* kv_empty = kv_full + C::STAGES;
  uint64_t* q_full = kv_empty + C::STAGES;   // [2]
  uint64_t* q_empty = q_full + 2;            // [2]
  uint64_t* wg_bars = q_empty + 2;           // [warpgroup][7]: s_full[2], p_full[2], o_done, red[2]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(wg_bars + 14);
  auto s_full = [&](int wg, int i) { return &wg_bars[wg * 7 + i]; };
  auto p_full = [&](int wg, int i) { return &wg_bars[wg * 7 + 2 + i]; };
  auto o_done = [&](int wg) { return &wg_bars[wg * 7 + 4]; };
  auto red_bar = [&](int wg, int i) { return &wg_bars[wg * 7 + 5 + i]; };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) { mbar_init(&kv_full[s], 1); mbar_init(&kv_empty[s], 1); }
    for (int s = 0; s < 2; ++s) { mbar_init(&q_full[s], 1); mbar_init(&q_empty[s], 1); }
    for (int wg = 0; wg < 2; ++wg) {
      for (int s = 0; s < 2; ++s) {
        mbar_init(s_full(wg, s), 1);
        mbar_init(p_full(wg, s), 128);
        mbar_init(red_bar(wg, s), 4);
      }
      mbar_init(o_done(wg), 1);
    }
    fence_mbar_init();
  }
  // P rows >= n_rep stay zero for the whole kernel; dims >= hd of the V slabs
  // that TMA never writes (head_dim 64) stay zero as well.
  for (int i = threadIdx.x; i < 4 * C::P_BYTES / 16; i += blockDim.x)
    reinterpret_cast<uint4*>(smem + C::OFF_P)[i] = make_uint4(0, 0, 0, 0);
  if (HD <= 64) {
    for (int s = 0; s < C::STAGES; ++s)
      for (int i = threadIdx.x; i < C::SLAB / 16; i += blockDim.x)
        reinterpret_cast<uint4*>(smem + C::OFF_STAGE + s * C::STAGE_BYTES + C::K_BYTES + C::SLAB)[i] =
            make_uint4(0, 0, 0, 0);
  }
  fence_proxy_async_smem();
  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&mapQ); prefetch_tensormap(&mapK); prefetch_tensormap(&mapV);
  }
  if (warp == 1) tmem_alloc(tmem_slot, 128);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // TMEM columns: warpgroup w owns S buffers [64w, 64w+16), [64w+16, 64w+32) and O^T [64w+32, 64w+48)
  const uint32_t tmem_base = *tmem_slot;
  griddep_wait_and_release();

  if (warp == 0) {
    // ---------------------------------------------------------------- producer
    if (lane == 0) {
      int st = 0, kq = 0;
      uint32_t ph = 0, qph[2] = {0, 0};
      uint32_t iss = 0, par = 0, qiss = 0, qpar = 0;
      bool ok = true;
      int b, g, piece, t0, t1, nk;
      for (int it = 0; ok && decode_piece(ds, blockIdx.x, it, b, g, piece, t0, t1, nk); ++it, ++kq) {
        const int qb = kq & 1;
        if (!mbar_wait(&q_empty[qb], qph[qb] ^ 1u, wait_ns)) break;
        mbar_arrive_expect_tx(&q_full[qb], C::Q_BYTES);
        for (int c = 0; c < C::CHUNKS_K; ++c)
          tma_load_2d(smem + C::OFF_Q + qb * C::Q_BYTES + c * C::Q_SLAB, &mapQ, &q_full[qb], c * 64,
                      b * ds.H + g * nrep);
        qiss |= 1u << qb; qpar = (qpar & ~(1u << qb)) | (qph[qb] << qb);
        qph[qb] ^= 1u;
        for (int t = t0; t < t1; ++t) {
          if (!mbar_wait(&kv_empty[st], ph ^ 1u, wait_ns)) { ok = false; break; }
          uint8_t* base = smem + C::OFF_STAGE + st * C::STAGE_BYTES;
          mbar_arrive_expect_tx(&kv_full[st], C::K_BYTES + C::CHUNKS_K * C::SLAB);
          for (int c = 0; c < C::CHUNKS_K; ++c) {
            tma_load_4d(base + c * C::SLAB, &mapK, &kv_full[st], c * 64, g, t * 128, b);
            tma_load_4d(base + C::K_BYTES + c * C::SLAB, &mapV, &kv_full[st], c * 64, g, t * 128, b);
          }
          iss |= 1u << st; par = (par & ~(1u << st)) | (ph << st);
          if (++st == C::STAGES) { st = 0; ph ^= 1u; }
        }
      }
      for (int s = 0; s < 2; ++s)
        if (qiss & (1u << s)) mbar_wait(&q_full[s], (qpar >> s) & 1u, wait_ns);
      for (int s = 0; s < C::STAGES; ++s)
        if (iss & (1u << s)) mbar_wait(&kv_full[s], (par >> s) & 1u, wait_ns);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      int st = 0, kq = 0;
      uint32_t ph = 0, qph[2] = {0, 0};
      uint32_t pph[2][2] = {{0, 0}, {0, 0}};
      bool ok = true;
      int b, g, piece, t0, t1, nk;
      for (int it = 0; ok && decode_piece(ds, blockIdx.x, it, b, g, piece, t0, t1, nk); ++it, ++kq) {
        const int qb = kq & 1;
        const uint32_t q_addr = smem_u32(smem + C::OFF_Q + qb * C::Q_BYTES);
        if (!mbar_wait(&q_full[qb], qph[qb], wait_ns)) break;
        qph[qb] ^= 1u;
        tc_fence_after();
        const int n = t1 - t0;
        // tile i: warpgroup wg = i & 1, its (i >> 1)-th tile, S buffer (i >> 1) & 1
        int st_s = st;
        uint32_t ph_s = ph;
        auto issue_s = [&](int i) -> bool {
          if (!mbar_wait(&kv_full[st_s], ph_s, wait_ns)) return false;
          tc_fence_after();
          const uint32_t ka = smem_u32(smem + C::OFF_STAGE + st_s * C::STAGE_BYTES);
          const int wg = i & 1, sb = (i >> 1) & 1;
#pragma unroll
          for (int k = 0; k < HD / 16; ++k) {
            const uint64_t a = sw128_desc(ka + (k >> 2) * C::SLAB + (k & 3) * 32, 1024, 16);
            const uint64_t bq = sw128_desc(q_addr + (k >> 2) * C::Q_SLAB + (k & 3) * 32, 1024, 16);
            tc_mma_f16_ss(tmem_base + wg * 64 + sb * 16, a, bq, IDESC_S, k > 0);
          }
          tc_commit(s_full(wg, sb));
          if (++st_s == C::STAGES) { st_s = 0; ph_s ^= 1u; }
          return true;
        };
        if (n > 0 && !issue_s(0)) break;
        if (n > 1 && !issue_s(1)) break;
        for (int i = 0; i < n && ok; ++i) {
          const int wg = i & 1, sb = (i >> 1) & 1;
          // O^T += V^T P^T for tile i once its warpgroup has written P
          if (!mbar_wait(p_full(wg, sb), pph[wg][sb], wait_ns)) { ok = false; break; }
          pph[wg][sb] ^= 1u;
          tc_fence_after();
          const uint32_t va = smem_u32(smem + C::OFF_STAGE + st * C::STAGE_BYTES + C::K_BYTES);
          const uint32_t pa = smem_u32(smem + C::OFF_P + (wg * 2 + sb) * C::P_BYTES);
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            const uint64_t a = sw128_desc(va + k * 2048, 1024, C::SLAB);
            const uint64_t bp = sw128_desc(pa + (k >> 2) * C::Q_SLAB + (k & 3) * 32, 1024, 16);
            tc_mma_f16_ss(tmem_base + wg * 64 + 32, a, bp, IDESC_O, (i > 1 || k > 0) ? 1u : 0u);
          }
          tc_commit(&kv_empty[st]);
          tc_commit(o_done(wg));
          if (++st == C::STAGES) { st = 0; ph ^= 1u; }
          // S for tile i + 2 (same warpgroup, its other S buffer)
          if (i + 2 < n && !issue_s(i + 2)) { ok = false; break; }
        }
        tc_commit(&q_empty[qb]);
      }
    }
  } else if (warp >= 4) {
    // ---------------------------------------------------------------- softmax + epilogue
    const int wg = (warp - 4) >> 2;                 // 0 or 1: takes tiles i with i % 2 == wg
    const int w4 = warp & 3;                        // quarter of the TMEM lanes
    const int row = w4 * 32 + lane;                 // TMEM lane: key of the tile / dim of O^T
    const uint32_t lane_off = (uint32_t)(w4 * 32) << 16;
    const uint32_t wg_tmem = tmem_base + lane_off + wg * 64;
    float* red = reinterpret_cast<float*>(smem + C::OFF_RED) + wg * 128;
    uint32_t sph[2] = {0, 0}, oph = 0, rph[2] = {0, 0};
    int rpar = 0;
    // the four warps of this warpgroup meet here (bounded: a warp that gave up
    // makes the others give up too instead of hanging)
    auto exchange = [&]() -> bool {
      __syncwarp();
      if (lane == 0) mbar_arrive(red_bar(wg, rpar));
      const bool done = mbar_wait(red_bar(wg, rpar), rph[rpar], wait_ns);
      rph[rpar] ^= 1u;
      return done;
    };
    int b, g, piece, t0, t1, nk;
    for (int it = 0; decode_piece(ds, blockIdx.x, it, b, g, piece, t0, t1, nk); ++it) {
      const int n = t1 - t0;
      const int mine = n > wg ? (n - wg + 1) / 2 : 0;   // tiles wg, wg+2, ...
      float m_ref[NREP], l_part[NREP];
#pragma unroll
      for (int h = 0; h < NREP; ++h) { m_ref[h] = -INFINITY; l_part[h] = 0.f; }
      bool ok = true;
      for (int k = 0; k < mine; ++k) {
        const int i = wg + 2 * k, sb = k & 1;
        if (!mbar_wait(s_full(wg, sb), sph[sb], wait_ns)) { ok = false; break; }
        sph[sb] ^= 1u;
        tc_fence_after();
        uint32_t r[16];
        tmem_ld16(wg_tmem + sb * 16, r);
        tc_wait_ld();
        const int key = (t0 + i) * 128 + row;
        const bool valid = key < nk;
        float s[NREP];
#pragma unroll
        for (int h = 0; h < NREP; ++h)
          s[h] = (valid && h < nrep) ? __uint_as_float(r[h]) * ds.scale_log2 : -INFINITY;
        // tile maximum per head over the 128 keys
        float* rb = red + rpar * 64;
#pragma unroll
        for (int h = 0; h < NREP; ++h) {
          const float mx = warp_max(s[h]);
          if (lane == 0) rb[w4 * 16 + h] = mx;
        }
        if (!exchange()) { ok = false; break; }
        rpar ^= 1;
        bool grow = false;
        float alpha[NREP];
#pragma unroll
        for (int h = 0; h < NREP; ++h) {
          const float tm = fmaxf(fmaxf(rb[h], rb[16 + h]), fmaxf(rb[32 + h], rb[48 + h]));
          alpha[h] = 1.f;
          if (tm > m_ref[h] + 8.0f) {
            alpha[h] = exp2f(m_ref[h] - tm);
            m_ref[h] = tm;
            l_part[h] *= alpha[h];
            grow = true;
          }
        }
        // this warpgroup's previous P.V must be done before P is rewritten or O rescaled
        if (k > 0) {
          if (!mbar_wait(o_done(wg), oph, wait_ns)) { ok = false; break; }
          oph ^= 1u;
          tc_fence_after();
          if (grow) {   // uniform across the warpgroup (all threads hold the same maxima)
            uint32_t o[16];
            tmem_ld16(wg_tmem + 32, o);
            tc_wait_ld();
#pragma unroll
            for (int h = 0; h < NREP; ++h) o[h] = __float_as_uint(__uint_as_float(o[h]) * alpha[h]);
            tmem_st16(wg_tmem + 32, o);
            tc_wait_st();
          }
        }
        // P^T[head][key] in bf16, 128-byte-swizzled K-major rows of 128 keys;
        // even lanes store the (key, key+1) pair as one 32-bit word
        uint8_t* pbuf = smem + C::OFF_P + (wg * 2 + sb) * C::P_BYTES + (row >> 6) * C::Q_SLAB;
        const int kin = row & 63;
#pragma unroll
        for (int h = 0; h < NREP; ++h) {
          const float p = (h < nrep) ? exp2f(s[h] - m_ref[h]) : 0.f;
          l_part[h] += p;
          const float p_next = __shfl_down_sync(0xffffffffu, p, 1);
          if ((lane & 1) == 0 && h < nrep)
            *reinterpret_cast<uint32_t*>(pbuf + h * 128 + ((((kin >> 3) ^ (h & 7))) << 4) + (kin & 7) * 2) =
                pack_bf16x2(p, p_next);
        }
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(p_full(wg, sb));
      }
      if (!ok) break;
      // epilogue: last P.V of this warpgroup, then its (m, l, acc) record
      float o_val[NREP];
      if (mine > 0) {
        if (!mbar_wait(o_done(wg), oph, wait_ns)) break;
        oph ^= 1u;
        tc_fence_after();
        uint32_t o[16];
        tmem_ld16(wg_tmem + 32, o);
        tc_wait_ld();
        tc_fence_before();
#pragma unroll
        for (int h = 0; h < NREP; ++h) o_val[h] = __uint_as_float(o[h]);
      } else {
#pragma unroll
        for (int h = 0; h < NREP; ++h) o_val[h] = 0.f;
      }
      float* rb = red + rpar * 64;
#pragma unroll
      for (int h = 0; h < NREP; ++h) {
        const float sum = warp_sum(l_part[h]);
        if (lane == 0) rb[w4 * 16 + h] = sum;
      }
      if (!exchange()) break;
      rpar ^= 1;
      const int slot = 2 * piece + wg;
#pragma unroll
      for (int h = 0; h < NREP; ++h) {
        if (h >= nrep) break;
        float* rec = part + (((size_t)b * ds.H + g * nrep + h) * ds.slots + slot) * (HD + 2);
        if (row < HD) rec[2 + row] = o_val[h];
        if (row == 0) {
          rec[0] = m_ref[h];
          rec[1] = rb[h] + rb[16 + h] + rb[32 + h] + rb[48 + h];
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 128);
  }
}

}  // namespace l3
