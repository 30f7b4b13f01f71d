// tc_gemm_pair.cuh -- the prefill Linear layers (y = x W^T, "Build your own
// Llama 3 from scratch" §3.4-§3.5) on a CTA pair: tcgen05 cta_group::2.
//
// Same contraction and epilogues as tc_gemm.cuh, but a work tile is 256 rows
// of A by one n-tile and is computed by the two CTAs of a cluster on
// neighbouring SMs.  CTA r loads rows [128r, 128r + 128) of the A tile and its
// half of every B tile; the leader (r = 0) issues M = 256 MMAs that read both
// CTAs' shared memory and write each CTA's 128 accumulator rows into that
// CTA's TMEM.  Per CTA and k-block this fills 32 KB of shared memory from L2
// instead of 48 KB for the same tensor work, which leaves room for a 6-stage
// ring and cuts the L2 -> SM traffic of the prefill GEMMs by a third.
//
// B halves and accumulator columns.  Without DUAL (BN = 256) CTA r holds B
// rows [128r, 128r + 128) of the tile and accumulator column j is output
// column j.  With DUAL (w1 | w3, BN = 128 per weight) CTA r holds 64 rows of
// w1 and then the same 64 rows of w3, back to back, so one N = 256 MMA covers
// both weights: accumulator columns 0-63 are w1 columns 0-63, 64-127 their w3
// partners, 128-191 w1 columns 64-127, 192-255 their w3 partners.
//
// Synchronisation (every mbarrier wait bounded; both CTAs execute the same
// two cluster barriers, after set-up and before exit):
//   full[s]      leader only: expect_tx of both CTAs' bytes, completed by both
//                CTAs' TMA loads
//   empty[s]     in each CTA: the leader's commit after the stage's MMAs
//   acc_full[b]  in each CTA: the leader's commit after a tile's last MMA
//   acc_empty[b] leader only: 8 arrivals (the 4 epilogue warps of each CTA)
// No load carries a multicast qualifier: each CTA loads its own halves.
#pragma once
#include "tc_gemm.cuh"

namespace l3 {

template <int BN, int STAGES, bool DUAL>
struct TcGemmPairCfg {
  static constexpr int BK = 64;
  static constexpr int NB = DUAL ? 2 : 1;
  static constexpr int BH = BN / 2;                  // rows of each B operand per CTA
  static constexpr int A_BYTES = 128 * BK * 2;       // this CTA's 128 rows of A
  static constexpr int B_BYTES = BH * BK * 2;        // this CTA's half of one B operand
  static constexpr int STAGE_BYTES = A_BYTES + NB * B_BYTES;
  static constexpr int NMMA = BN * NB;               // MMA N (both weights with DUAL)
  static constexpr int ACC_COLS = NMMA;
  static constexpr int ACC_BUFS = 2;
  static constexpr int OFF_A = 0;
  static constexpr int OFF_B = STAGES * A_BYTES;
  // 16 KB of spare shared memory after the B ring: a margin kept from the
  // first version of this kernel; the MMAs read only the ring itself.
  static constexpr int SLACK = 16384;
  static constexpr int OFF_BAR = OFF_B + STAGES * NB * B_BYTES + SLACK;
  static constexpr int BAR_BYTES = (2 * STAGES + 2 * ACC_BUFS) * 8 + 16;
  static constexpr int SMEM_BYTES = 1024 + OFF_BAR + BAR_BYTES;
  static_assert(NMMA == 256, "one M = 256, N = 256 MMA per k-step");
  static_assert(2 * ACC_COLS <= 512, "two accumulators in TMEM");
  static_assert(B_BYTES % 1024 == 0, "swizzle atoms");
  static_assert(SMEM_BYTES <= 232448, "shared memory");
};

// Accumulator column of output column `col` (0 <= col < BN) of the tile; the
// w3 partner of a DUAL column is 64 further on.
template <int BN, bool DUAL>
__device__ __forceinline__ int pair_acc_col(int col) {
  return DUAL ? col + (col >= BN / 2 ? BN / 2 : 0) : col;
}

// `sh` describes tiles of 256 rows (tiles_m = ceil(rows_a / 256), one split,
// no stream-K); a pair of CTAs takes units pair, pair + pairs, ... in the
// grouped raster of cta_unit.  Non-swapped epilogues only (STORE, RESIDUAL,
// SWIGLU, QKV_ROPE): A is the activation, B the weight.
template <int BN, int STAGES, int EPI, bool DUAL>
__global__ void __launch_bounds__(192, 1)
    tc_gemm_pair_kernel(const __grid_constant__ CUtensorMap mapA, const __grid_constant__ CUtensorMap mapB,
                        const __grid_constant__ CUtensorMap mapB2, const GemmShape sh, const EpiParams ep,
                        const unsigned long long wait_ns) {
  using C = TcGemmPairCfg<BN, STAGES, DUAL>;
  constexpr uint32_t IDESC = idesc_bf16_f32(256, C::NMMA, 0, 0);
  static_assert(EPI == EPI_STORE || EPI == EPI_RESIDUAL || EPI == EPI_SWIGLU || EPI == EPI_QKV_ROPE,
                "non-swapped epilogues");

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem + C::OFF_A;
  uint8_t* sB = smem + C::OFF_B;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* empty = full + STAGES;
  uint64_t* acc_full = empty + STAGES;
  uint64_t* acc_empty = acc_full + C::ACC_BUFS;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_empty + C::ACC_BUFS);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int pair = blockIdx.x >> 1, pairs = gridDim.x >> 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
    for (int s = 0; s < C::ACC_BUFS; ++s) { mbar_init(&acc_full[s], 1); mbar_init(&acc_empty[s], 8); }
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&mapA);
    prefetch_tensormap(&mapB);
    if (DUAL) prefetch_tensormap(&mapB2);
  }
  if (warp == 1) tmem_alloc_pair(tmem_slot, 512);
  tc_fence_before();
  __syncthreads();
  cluster_sync();   // the partner's barriers are initialised before anyone signals them
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  griddep_wait_and_release();

  if (warp == 0) {
    // ------------------------------------------------------------ producer (both CTAs)
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued_mask = 0, issued_parity = 0;
      bool ok = true;
      GemmUnit g;
      for (int it = 0; ok && cta_unit(sh, pair, pairs, it, g); ++it) {
        const int arow = g.mt * 256 + (int)rank * 128;
        const int brow = g.nt * BN + (int)rank * C::BH;
        for (int kb = g.kb0; kb < g.kb1; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, wait_ns)) { ok = false; break; }
          const uint32_t full_leader = cluster_map(smem_u32(&full[stage]), 0);
          if (leader) mbar_arrive_expect_tx(&full[stage], 2 * C::STAGE_BYTES);
          tma_load_2d_pair(sA + stage * C::A_BYTES, &mapA, full_leader, kb * C::BK, arow);
          tma_load_2d_pair(sB + (stage * C::NB) * C::B_BYTES, &mapB, full_leader, kb * C::BK, brow);
          if constexpr (DUAL)
            tma_load_2d_pair(sB + (stage * C::NB + 1) * C::B_BYTES, &mapB2, full_leader, kb * C::BK, brow);
          issued_mask |= 1u << stage;
          issued_parity = (issued_parity & ~(1u << stage)) | (phase << stage);
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
      }
      // The leader's full barriers count both CTAs' copies: let them all land
      // before the final cluster barrier lets either CTA go.
      if (leader)
        for (int s = 0; s < STAGES; ++s)
          if (issued_mask & (1u << s)) mbar_wait(&full[s], (issued_parity >> s) & 1u, wait_ns);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (leader)
    if (leader && lane == 0) {
      int stage = 0, abuf = 0;
      uint32_t phase = 0, aphase = 0;
      int last_buf = -1;
      uint32_t last_parity = 0;
      bool ok = true;
      GemmUnit g;
      for (int it = 0; ok && cta_unit(sh, pair, pairs, it, g); ++it) {
        if (!mbar_wait(&acc_empty[abuf], aphase ^ 1u, wait_ns)) break;
        tc_fence_after();
        const uint32_t d = tmem_base + abuf * C::ACC_COLS;
        for (int kb = g.kb0; kb < g.kb1; ++kb) {
          if (!mbar_wait(&full[stage], phase, wait_ns)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(sA + stage * C::A_BYTES);
          const uint32_t b_addr = smem_u32(sB + (stage * C::NB) * C::B_BYTES);
#pragma unroll
          for (int k = 0; k < C::BK / 16; ++k) {
            const uint64_t adesc = sw128_desc(a_addr + k * 32, 1024, 16);
            const uint64_t bdesc = sw128_desc(b_addr + k * 32, 1024, 16);
            tc_mma_f16_pair(d, adesc, bdesc, IDESC, (kb > g.kb0 || k > 0) ? 1u : 0u);
          }
          tc_commit_pair(&empty[stage]);
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        tc_commit_pair(&acc_full[abuf]);
        last_buf = abuf;
        last_parity = aphase;
        if (++abuf == C::ACC_BUFS) { abuf = 0; aphase ^= 1u; }
      }
      // the last accumulator's MMAs complete before TMEM may be released
      if (last_buf >= 0) mbar_wait(&acc_full[last_buf], last_parity, wait_ns);
    }
  } else {
    // ------------------------------------------------------------ epilogue (both CTAs)
    const int quarter = warp & 3;   // TMEM lanes this warp may access
    const int row_in_tile = (int)rank * 128 + quarter * 32 + lane;
    int abuf = 0;
    uint32_t aphase = 0;
    GemmUnit g;
    for (int it = 0; cta_unit(sh, pair, pairs, it, g); ++it) {
      const int row = g.mt * 256 + row_in_tile;
      const bool row_ok = row < sh.rows_a;
      if (!mbar_wait(&acc_full[abuf], aphase, wait_ns)) break;
      tc_fence_after();
      const uint32_t tbase = tmem_base + ((uint32_t)(quarter * 32) << 16) + abuf * C::ACC_COLS;
#pragma unroll 1
      for (int c = 0; c < BN / 32; ++c) {
        const int col = pair_acc_col<BN, DUAL>(c * 32);
        float acc[32], acc3[32];
        uint32_t r[32];
        tmem_ld32(tbase + col, r);
        uint32_t r3[32];
        if constexpr (DUAL) tmem_ld32(tbase + col + BN / 2, r3);
        tc_wait_ld();
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          acc[j] = __uint_as_float(r[j]);
          acc3[j] = DUAL ? __uint_as_float(r3[j]) : 0.f;
        }
        epilogue_chunk<EPI, 32>(ep, sh, acc, acc3, row, row_ok, row, g.nt * BN + c * 32, 0, lane);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0 && !(sh.withhold == 1 && it == 0 && warp == 2 && leader))
        mbar_arrive_cluster(cluster_map(smem_u32(&acc_empty[abuf]), 0));
      if (++abuf == C::ACC_BUFS) { abuf = 0; aphase ^= 1u; }
    }
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync();   // neither CTA leaves while its partner may still touch its shared memory or TMEM
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, 512);
  }
}

}  // namespace l3
