// tc_gemm.cuh -- persistent tcgen05 GEMM, D[a, b] = sum_k A[a, k] * B[b, k],
// bf16 operands in shared memory (TMA, 128-byte swizzle), fp32 accumulators in
// TMEM, with the decoder's epilogues fused into the TMEM read-back.
//
// The dense contractions of the block are Linear layers y = x W^T with
// weights stored [out, in] ("从0开发大模型—译llama3-from-scratch" §6.5 / §9.1,
// "Build your own Llama 3 from scratch" §3.4 nn.Linear), i.e. both operands
// are K-major: A and B are each read as rows of K contiguous elements.
//
// Roles (192 threads, one CTA per SM, persistent over work units):
//   warp 0      TMA producer: fills a STAGES-deep ring of (A, B[, B2]) tiles
//   warp 1      allocates TMEM; one lane issues tcgen05.mma (M=128, N=BN, K=16)
//   warps 2..5  epilogue: tcgen05.ld 32 lanes x 32 columns, fused op, global store
// The accumulator is double-buffered in TMEM so the epilogue of one tile
// overlaps the main loop of the next.
//
// Work unit = (split, m-tile, n-tile), visited in groups of m-tiles (see
// gemm_unit) so that the tiles in flight share their operands through L2.
//
// "A" may consist of two tensors stacked along rows (tiles of the second one
// come after those of the first; their output rows are offset by
// `out_row_offset2`), which lets one launch stream W1 and W3 for the decode
// SwiGLU.  With DUAL, every tile multiplies A by two B tensors into two
// accumulators (W1 and W3 for the prefill SwiGLU).
#pragma once
#include "common.cuh"

namespace l3 {

enum EpiKind {
  EPI_STORE = 0,     // out[a, b] = acc                      (bf16)
  EPI_RESIDUAL = 1,  // out[a, b] = res[a, b] + acc          (bf16, out may == res)
  EPI_QKV_ROPE = 2,  // RoPE on q/k columns, q -> q_out, k/v -> caches
  EPI_SWIGLU = 3,    // DUAL: out[a, b] = silu(acc1) * acc3
  EPI_PARTIAL = 4,   // swapped: P[split][b][a] = acc        (fp32 split-K partials)
  EPI_ARGMAX = 5     // swapped: logits[b][a] = acc, argmax over a per column b
};

struct GemmShape {
  int rows_a;          // rows of A (first tensor)
  int rows_a2;         // rows of the second stacked A tensor (0 = none)
  int rows_b;          // rows of B (= valid output columns for non-swapped epilogues)
  int k;               // reduction length
  int tiles_m1;        // m-tiles of the first A tensor
  int tiles_m;         // all m-tiles
  int tiles_n;
  int kblocks;         // ceil(k / 64)
  int kb_per_split;
  int splits;
  int units;           // splits * tiles_m * tiles_n (stream-K: the CTAs of the schedule)
  int group_m;         // raster: m-tiles per group (tiles of a group share A rows and B columns)
  // Stream-K (one n-tile only): CTA c takes k-blocks [c*sk_per, (c+1)*sk_per)
  // of the (m-tile, k-block) space in m-major order; 0 = split-K units.
  int sk_per;
  // Failure-detection test hook (0 in every normal launch): 1 = the first
  // epilogue warp leaves out its release of the accumulator after the CTA's
  // first unit, so the MMA issuer's bounded wait for that buffer gives up.
  int withhold;
};

// Work unit -> (split, m-tile, n-tile).  Within a split, tiles are visited in
// groups of `group_m` m-tiles: n varies across the group, m fastest inside it,
// so the CTAs running at the same time touch group_m A row-blocks and a few B
// column-blocks, which stay in L2.
__device__ __forceinline__ void gemm_unit(const GemmShape& sh, int u, int& split, int& mt, int& nt) {
  const int per_split = sh.tiles_m * sh.tiles_n;
  split = u / per_split;
  const int r = u % per_split;
  const int per_group = sh.group_m * sh.tiles_n;
  const int group = r / per_group;
  const int first_m = group * sh.group_m;
  const int gm = min(sh.group_m, sh.tiles_m - first_m);
  const int q = r % per_group;
  mt = first_m + q % gm;
  nt = q / gm;
}

// One unit of a CTA's work: an output tile and a k-block range of it.  slab:
// the partial-sum slab it writes (EPI_PARTIAL).  zero_from > 0: this CTA is the
// tile's last contributor and also zeroes slabs [zero_from, splits).
struct GemmUnit {
  int mt, nt, kb0, kb1, slab, zero_from;
};

// Unit `it` of CTA `c` (of `ctas`); false once the CTA has no more.
__device__ __forceinline__ bool cta_unit(const GemmShape& sh, int c, int ctas, int it, GemmUnit& g) {
  if (sh.sk_per == 0) {
    const int u = c + it * ctas;
    if (u >= sh.units) return false;
    int split;
    gemm_unit(sh, u, split, g.mt, g.nt);
    g.kb0 = split * sh.kb_per_split;
    g.kb1 = min(g.kb0 + sh.kb_per_split, sh.kblocks);
    g.slab = split;
    g.zero_from = 0;
    return true;
  }
  const int total = sh.tiles_m * sh.kblocks;
  const int start = c * sh.sk_per, end = min(start + sh.sk_per, total);
  const int tile = start / sh.kblocks + it;
  const int tstart = tile * sh.kblocks;
  if (tstart >= end) return false;
  g.mt = tile;
  g.nt = 0;
  g.kb0 = max(start - tstart, 0);
  g.kb1 = min(end - tstart, sh.kblocks);
  const int first = tstart / sh.sk_per;                     // CTAs that share the tile, in k order
  const int last = (tstart + sh.kblocks - 1) / sh.sk_per;
  g.slab = c - first;
  g.zero_from = c == last ? last - first + 1 : 0;
  return true;
}

struct EpiParams {
  void* out;           // STORE/RESIDUAL/SWIGLU: bf16 [rows_a, ldo]; PARTIAL: float
  long long ldo;
  const void* res;     // RESIDUAL: bf16 [rows_a, ldo]
  long long split_stride;  // PARTIAL: elements between split slabs
  int out_row_offset2;     // PARTIAL: output-row offset of the second A tensor
  // EPI_QKV_ROPE
  int seq, start_pos, n_heads, n_kv, head_dim, cache_cap;
  const float* rope;
  void* q_out;
  void* k_cache;
  void* v_cache;
  // EPI_ARGMAX
  float* logits;       // nullable, [rows_b, vocab]
  unsigned long long* keys;  // [rows_b]
};

template <int BN, int STAGES, bool DUAL>
struct TcGemmCfg {
  static constexpr int BM = 128, BK = 64;
  static constexpr int NB = DUAL ? 2 : 1;
  static constexpr int A_BYTES = BM * BK * 2;
  static constexpr int B_BYTES = BN * BK * 2;
  static constexpr int STAGE_BYTES = A_BYTES + NB * B_BYTES;
  static constexpr int ACC_COLS = BN * NB;
  static constexpr int ACC_BUFS = (2 * ACC_COLS <= 512) ? 2 : 1;
  static constexpr int TMEM_NEED = ACC_COLS * ACC_BUFS;
  static constexpr int TMEM_COLS = TMEM_NEED <= 32 ? 32 : TMEM_NEED <= 64 ? 64 : TMEM_NEED <= 128 ? 128
                                 : TMEM_NEED <= 256 ? 256 : 512;
  static constexpr int CW = BN < 32 ? BN : 32;  // epilogue chunk width (columns)
  static constexpr int BAR_BYTES = (2 * STAGES + 2 * ACC_BUFS) * 8 + 16;
  static constexpr int SMEM_BYTES = 1024 /*alignment slack*/ + STAGES * STAGE_BYTES + BAR_BYTES;
  static_assert(BN % 16 == 0 && BN >= 16 && BN <= 256, "MMA N for M=128");
  static_assert(B_BYTES % 1024 == 0, "swizzle atoms");
  static_assert(SMEM_BYTES <= 232448, "shared memory");
};

// Swap a 32-column slab of (value, index) pairs across the warp so that lane L
// ends with the best pair of column L (highest value, lowest index on ties).
__device__ __forceinline__ void better_pair(float& v, uint32_t& i, float v2, uint32_t i2) {
  if (v2 > v || (v2 == v && i2 < i)) { v = v2; i = i2; }
}
__device__ __forceinline__ void warp_column_argmax(float (&v)[32], uint32_t (&id)[32], int lane) {
#pragma unroll
  for (int half = 16; half >= 1; half >>= 1) {
    const bool upper = (lane & half) != 0;
#pragma unroll
    for (int c = 0; c < half; ++c) {
      float send_v = upper ? v[c] : v[c + half];
      uint32_t send_i = upper ? id[c] : id[c + half];
      float keep_v = upper ? v[c + half] : v[c];
      uint32_t keep_i = upper ? id[c + half] : id[c];
      float rv = __shfl_xor_sync(0xffffffffu, send_v, half);
      uint32_t ri = __shfl_xor_sync(0xffffffffu, send_i, half);
      better_pair(keep_v, keep_i, rv, ri);
      v[c] = keep_v;
      id[c] = keep_i;
    }
  }
}

template <int EPI, int CW>
__device__ __forceinline__ void epilogue_chunk(const EpiParams& ep, const GemmShape& sh,
                                               const float (&acc)[32], const float (&acc3)[32],
                                               int arow, bool arow_ok, int out_row, int bcol0,
                                               int split, int lane, int zero_from = 0) {
  if constexpr (EPI == EPI_STORE || EPI == EPI_RESIDUAL || EPI == EPI_SWIGLU) {
    if (!arow_ok) return;
    bf16* out = reinterpret_cast<bf16*>(ep.out) + (size_t)arow * ep.ldo + bcol0;
    const bf16* res = EPI == EPI_RESIDUAL ? reinterpret_cast<const bf16*>(ep.res) + (size_t)arow * ep.ldo + bcol0
                                          : nullptr;
    float v[32];
#pragma unroll
    for (int j = 0; j < CW; ++j) {
      if constexpr (EPI == EPI_SWIGLU) {
        float a = acc[j];
        v[j] = a / (1.f + expf(-a)) * acc3[j];
      } else {
        v[j] = acc[j];
      }
    }
    if (bcol0 + CW <= sh.rows_b) {
#pragma unroll
      for (int q = 0; q < CW / 8; ++q) {
        if constexpr (EPI == EPI_RESIDUAL) {
          uint4 r = *reinterpret_cast<const uint4*>(res + q * 8);
          v[q * 8 + 0] += bf16lo(r.x); v[q * 8 + 1] += bf16hi(r.x);
          v[q * 8 + 2] += bf16lo(r.y); v[q * 8 + 3] += bf16hi(r.y);
          v[q * 8 + 4] += bf16lo(r.z); v[q * 8 + 5] += bf16hi(r.z);
          v[q * 8 + 6] += bf16lo(r.w); v[q * 8 + 7] += bf16hi(r.w);
        }
        uint4 o;
        o.x = pack_bf16x2(v[q * 8 + 0], v[q * 8 + 1]);
        o.y = pack_bf16x2(v[q * 8 + 2], v[q * 8 + 3]);
        o.z = pack_bf16x2(v[q * 8 + 4], v[q * 8 + 5]);
        o.w = pack_bf16x2(v[q * 8 + 6], v[q * 8 + 7]);
        *reinterpret_cast<uint4*>(out + q * 8) = o;
      }
    } else {
#pragma unroll
      for (int j = 0; j < CW; ++j) {
        if (bcol0 + j < sh.rows_b) {
          float x = v[j];
          if constexpr (EPI == EPI_RESIDUAL) x += __bfloat162float(res[j]);
          out[j] = __float2bfloat16_rn(x);
        }
      }
    }
  } else if constexpr (EPI == EPI_QKV_ROPE) {
    // Columns bcol0..bcol0+CW-1 lie inside one head (head_dim is a multiple of 32).
    if (!arow_ok || bcol0 >= sh.rows_b) return;
    const int hd = ep.head_dim, H = ep.n_heads, KV = ep.n_kv;
    const int head = bcol0 / hd, d0 = bcol0 % hd;
    const int b = arow / ep.seq, t = arow % ep.seq, pos = ep.start_pos + t;
    float v[32];
#pragma unroll
    for (int j = 0; j < CW; ++j) v[j] = acc[j];
    if (head < H + KV) {
      const float4* cs = reinterpret_cast<const float4*>(ep.rope + ((size_t)pos * (hd / 2) + d0 / 2) * 2);
#pragma unroll
      for (int p = 0; p < CW / 4; ++p) {
        float4 c = cs[p];  // (cos_i, sin_i, cos_{i+1}, sin_{i+1})
        float a0 = v[4 * p], b0 = v[4 * p + 1], a1 = v[4 * p + 2], b1 = v[4 * p + 3];
        v[4 * p] = a0 * c.x - b0 * c.y;
        v[4 * p + 1] = a0 * c.y + b0 * c.x;
        v[4 * p + 2] = a1 * c.z - b1 * c.w;
        v[4 * p + 3] = a1 * c.w + b1 * c.z;
      }
    }
    bf16* dst;
    if (head < H) {
      dst = reinterpret_cast<bf16*>(ep.q_out) + (size_t)arow * H * hd + bcol0;
    } else {
      const bool is_k = head < H + KV;
      const int kvh = head - (is_k ? H : H + KV);
      dst = reinterpret_cast<bf16*>(is_k ? ep.k_cache : ep.v_cache) +
            (((size_t)b * ep.cache_cap + pos) * KV + kvh) * hd + d0;
    }
#pragma unroll
    for (int q = 0; q < CW / 8; ++q) {
      uint4 o;
      o.x = pack_bf16x2(v[q * 8 + 0], v[q * 8 + 1]);
      o.y = pack_bf16x2(v[q * 8 + 2], v[q * 8 + 3]);
      o.z = pack_bf16x2(v[q * 8 + 4], v[q * 8 + 5]);
      o.w = pack_bf16x2(v[q * 8 + 6], v[q * 8 + 7]);
      *reinterpret_cast<uint4*>(dst + q * 8) = o;
    }
  } else if constexpr (EPI == EPI_PARTIAL) {
    // Swapped: A rows are output features, B rows are tokens.
    if (!arow_ok) return;
    float* P = reinterpret_cast<float*>(ep.out) + (size_t)split * ep.split_stride + out_row;
#pragma unroll
    for (int j = 0; j < CW; ++j)
      if (bcol0 + j < sh.rows_b) P[(size_t)(bcol0 + j) * ep.ldo] = acc[j];
    // stream-K: the tile's last contributor zeroes the slabs no CTA writes
    if (zero_from > 0) {
      for (int z = zero_from; z < sh.splits; ++z) {
        float* Z = reinterpret_cast<float*>(ep.out) + (size_t)z * ep.split_stride + out_row;
#pragma unroll
        for (int j = 0; j < CW; ++j)
          if (bcol0 + j < sh.rows_b) Z[(size_t)(bcol0 + j) * ep.ldo] = 0.f;
      }
    }
  } else if constexpr (EPI == EPI_ARGMAX) {
    // Swapped: A rows are vocabulary entries, B rows are hidden rows.
    float v[32];
    uint32_t id[32];
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      v[j] = (j < CW && arow_ok) ? acc[j] : -INFINITY;
      id[j] = (uint32_t)arow;
    }
    if (ep.logits && arow_ok) {
#pragma unroll
      for (int j = 0; j < CW; ++j)
        if (bcol0 + j < sh.rows_b) ep.logits[(size_t)(bcol0 + j) * sh.rows_a + arow] = acc[j];
    }
    warp_column_argmax(v, id, lane);
    const int col = bcol0 + lane;
    if (lane < CW && col < sh.rows_b && v[0] != -INFINITY)
      atomicMax(&ep.keys[col], argmax_pack(v[0], id[0]));
  }
}

template <int BN, int STAGES, int EPI, bool DUAL>
__global__ void __launch_bounds__(192, 1)
    tc_gemm_kernel(const __grid_constant__ CUtensorMap mapA, const __grid_constant__ CUtensorMap mapA2,
                   const __grid_constant__ CUtensorMap mapB, const __grid_constant__ CUtensorMap mapB2,
                   const GemmShape sh, const EpiParams ep, const unsigned long long wait_ns) {
  using C = TcGemmCfg<BN, STAGES, DUAL>;
  constexpr uint32_t IDESC = idesc_bf16_f32(128, BN, 0, 0);
  constexpr uint32_t IDESC_DUAL = idesc_bf16_f32(128, DUAL ? 2 * BN : BN, 0, 0);
  static_assert(!DUAL || 2 * BN <= 256, "one MMA covers both B tiles");

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES * C::A_BYTES;
  uint64_t* full = reinterpret_cast<uint64_t*>(sB + STAGES * C::NB * C::B_BYTES);
  uint64_t* empty = full + STAGES;
  uint64_t* acc_full = empty + STAGES;
  uint64_t* acc_empty = acc_full + C::ACC_BUFS;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_empty + C::ACC_BUFS);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
    for (int s = 0; s < C::ACC_BUFS; ++s) { mbar_init(&acc_full[s], 1); mbar_init(&acc_empty[s], 4); }
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&mapA);
    if (sh.rows_a2) prefetch_tensormap(&mapA2);
    prefetch_tensormap(&mapB);
    if (DUAL) prefetch_tensormap(&mapB2);
  }
  if (warp == 1) tmem_alloc(tmem_slot, C::TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // In the swapped launches A is a weight matrix, which no earlier kernel
  // writes: the producer starts streaming it before waiting for the previous
  // kernel (programmatic launch) and waits only before loading B.  Every other
  // thread waits here, before its first global access.
  constexpr bool kEarlyA = (EPI == EPI_PARTIAL || EPI == EPI_ARGMAX);
  if (!(kEarlyA && warp == 0)) griddep_wait_and_release();

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued_mask = 0, issued_parity = 0;
      bool ok = true;
      int pre = 0;   // k-blocks of the first unit whose A tile went out before the dependency wait
      if constexpr (kEarlyA) {
        GemmUnit g0;
        if (cta_unit(sh, blockIdx.x, gridDim.x, 0, g0)) {
          const int mt = g0.mt, nt = g0.nt;
          const bool second = mt >= sh.tiles_m1;
          const int arow = (second ? mt - sh.tiles_m1 : mt) * C::BM;
          const int kb0 = g0.kb0;
          pre = min(STAGES, g0.kb1 - kb0);
          for (int i = 0; i < pre; ++i) {   // fresh ring: these stages are free
            mbar_arrive_expect_tx(&full[i], C::STAGE_BYTES);
            tma_load_2d(sA + i * C::A_BYTES, second ? &mapA2 : &mapA, &full[i], (kb0 + i) * C::BK, arow);
          }
          griddep_wait_and_release();
          for (int i = 0; i < pre; ++i) {
            tma_load_2d(sB + (i * C::NB) * C::B_BYTES, &mapB, &full[i], (kb0 + i) * C::BK, nt * BN);
            if constexpr (DUAL)
              tma_load_2d(sB + (i * C::NB + 1) * C::B_BYTES, &mapB2, &full[i], (kb0 + i) * C::BK, nt * BN);
            issued_mask |= 1u << i;
          }
          stage = pre % STAGES;
          phase = pre == STAGES ? 1u : 0u;
        } else {
          griddep_wait_and_release();
        }
      }
      GemmUnit g;
      for (int it = 0; ok && cta_unit(sh, blockIdx.x, gridDim.x, it, g); ++it) {
        const int mt = g.mt, nt = g.nt;
        const bool second = mt >= sh.tiles_m1;
        const CUtensorMap* ma = second ? &mapA2 : &mapA;
        const int arow = (second ? mt - sh.tiles_m1 : mt) * C::BM;
        const int kb0 = g.kb0 + (it == 0 ? pre : 0);
        const int kb1 = g.kb1;
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, wait_ns)) { ok = false; break; }
          mbar_arrive_expect_tx(&full[stage], C::STAGE_BYTES);
          tma_load_2d(sA + stage * C::A_BYTES, ma, &full[stage], kb * C::BK, arow);
          tma_load_2d(sB + (stage * C::NB) * C::B_BYTES, &mapB, &full[stage], kb * C::BK, nt * BN);
          if constexpr (DUAL)
            tma_load_2d(sB + (stage * C::NB + 1) * C::B_BYTES, &mapB2, &full[stage], kb * C::BK, nt * BN);
          issued_mask |= 1u << stage;
          issued_parity = (issued_parity & ~(1u << stage)) | (phase << stage);
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
      }
      // Let every copy this thread started land before the CTA may exit.
      for (int s = 0; s < STAGES; ++s)
        if (issued_mask & (1u << s)) mbar_wait(&full[s], (issued_parity >> s) & 1u, wait_ns);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int stage = 0, abuf = 0;
      uint32_t phase = 0, aphase = 0;
      int last_buf = -1;
      uint32_t last_parity = 0;
      bool ok = true;
      GemmUnit g;
      for (int it = 0; ok && cta_unit(sh, blockIdx.x, gridDim.x, it, g); ++it) {
        const int kb0 = g.kb0, kb1 = g.kb1;
        if (!mbar_wait(&acc_empty[abuf], aphase ^ 1u, wait_ns)) break;
        tc_fence_after();
        const uint32_t d = tmem_base + abuf * C::ACC_COLS;
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait(&full[stage], phase, wait_ns)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(sA + stage * C::A_BYTES);
          const uint32_t b_addr = smem_u32(sB + (stage * C::NB) * C::B_BYTES);
#pragma unroll
          for (int k = 0; k < C::BK / 16; ++k) {
            const uint64_t adesc = sw128_desc(a_addr + k * 32, 1024, 16);
            const uint64_t bdesc = sw128_desc(b_addr + k * 32, 1024, 16);
            const uint32_t accum = (kb > kb0 || k > 0) ? 1u : 0u;
            // DUAL: the two B tiles sit back to back in shared memory (same
            // swizzle atoms), so one N = 2*BN MMA covers both and writes the
            // first operand's columns at d and the second's at d + BN.
            tc_mma_f16_ss(d, adesc, bdesc, DUAL ? IDESC_DUAL : IDESC, accum);
          }
          tc_commit(&empty[stage]);
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        tc_commit(&acc_full[abuf]);
        last_buf = abuf;
        last_parity = aphase;
        if (++abuf == C::ACC_BUFS) { abuf = 0; aphase ^= 1u; }
      }
      // Wait for the last accumulator's MMAs before TMEM may be released.
      if (last_buf >= 0) mbar_wait(&acc_full[last_buf], last_parity, wait_ns);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int quarter = warp & 3;  // TMEM lanes this warp may access
    const int row_in_tile = quarter * 32 + lane;
    int abuf = 0;
    uint32_t aphase = 0;
    GemmUnit g;
    for (int it = 0; cta_unit(sh, blockIdx.x, gridDim.x, it, g); ++it) {
      const int mt = g.mt, nt = g.nt, split = g.slab;
      const bool second = mt >= sh.tiles_m1;
      const int local_row = (second ? mt - sh.tiles_m1 : mt) * C::BM + row_in_tile;
      const bool arow_ok = local_row < (second ? sh.rows_a2 : sh.rows_a);
      const int out_row = second ? ep.out_row_offset2 + local_row : local_row;
      if (!mbar_wait(&acc_full[abuf], aphase, wait_ns)) break;
      tc_fence_after();
      const uint32_t tbase = tmem_base + ((uint32_t)(quarter * 32) << 16) + abuf * C::ACC_COLS;
#pragma unroll 1
      for (int c = 0; c < BN / C::CW; ++c) {
        float acc[32], acc3[32];
        if constexpr (C::CW == 32) {
          uint32_t r[32];
          tmem_ld32(tbase + c * 32, r);
          uint32_t r3[32];
          if constexpr (DUAL) tmem_ld32(tbase + BN + c * 32, r3);
          tc_wait_ld();
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            acc[j] = __uint_as_float(r[j]);
            acc3[j] = DUAL ? __uint_as_float(r3[j]) : 0.f;
          }
        } else {
          uint32_t r[16];
          tmem_ld16(tbase + c * 16, r);
          uint32_t r3[16];
          if constexpr (DUAL) tmem_ld16(tbase + BN + c * 16, r3);
          tc_wait_ld();
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            acc[j] = j < 16 ? __uint_as_float(r[j]) : 0.f;
            acc3[j] = (DUAL && j < 16) ? __uint_as_float(r3[j & 15]) : 0.f;
          }
        }
        epilogue_chunk<EPI, C::CW>(ep, sh, acc, acc3, local_row, arow_ok, out_row,
                                   nt * BN + c * C::CW, split, lane, g.zero_from);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0 && !(sh.withhold == 1 && it == 0 && warp == 2)) mbar_arrive(&acc_empty[abuf]);
      if (++abuf == C::ACC_BUFS) { abuf = 0; aphase ^= 1u; }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
}

}  // namespace l3
