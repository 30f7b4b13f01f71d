// tc_gemm_pair.cuh -- the prefill GEMM on a CTA pair (tcgen05 cta_group::2).
//
// Same contraction and epilogues as tc_gemm.cuh (Linear layers y = x W^T of
// the decoder block), but each work tile is 256 rows of A x BN columns and is
// computed by two CTAs on neighbouring SMs: CTA r of the pair loads rows
// [128r, 128r+128) of the A tile and rows [r*BN/2, (r+1)*BN/2) of the B tile;
// the leader CTA issues M=256 MMAs that read both CTAs' shared memory and
// write each CTA's 128 accumulator rows into that CTA's TMEM.  Per CTA and
// k-block this moves 32 KB from L2 instead of 48 KB for the same tensor work,
// and leaves room for a 6-stage ring.
//
// Synchronisation (all mbarrier waits bounded; both CTAs execute the same
// two cluster barriers, at set-up and before exit):
//   full[s]      leader only: expect_tx of both CTAs' bytes, completed by
//                both CTAs' TMA loads
//   empty[s]     in each CTA: the leader's commit after the stage's MMAs
//   acc_full[b]  in each CTA: the leader's commit after a tile's last MMA
//   acc_empty[b] leader only: 8 arrivals (4 epilogue warps of each CTA)
#pragma once
#include "tc_gemm.cuh"

namespace l3 {

template <int BN, int STAGES, bool DUAL>
struct TcGemmPairCfg {
  static constexpr int BK = 64;
  static constexpr int NB = DUAL ? 2 : 1;
  static constexpr int BH = BN / 2;                  // B rows per CTA (per B operand)
  static constexpr int A_BYTES = 128 * BK * 2;       // this CTA's 128 rows of A
  static constexpr int B_BYTES = BH * BK * 2;        // this CTA's half of one B operand
  static constexpr int STAGE_BYTES = A_BYTES + NB * B_BYTES;
  static constexpr int ACC_COLS = BN * NB;
  static constexpr int ACC_BUFS = (2 * ACC_COLS <= 512) ? 2 : 1;
  static constexpr int OFF_A = 0;
  static constexpr int OFF_B = STAGES * A_BYTES;
  static constexpr int SLACK = 16384;                // keeps any operand read inside the allocation
  static constexpr int OFF_BAR = OFF_B + STAGES * NB * B_BYTES + SLACK;
  static constexpr int BAR_BYTES = (2 * STAGES + 2 * ACC_BUFS) * 8 + 16;
  static constexpr int SMEM_BYTES = 1024 + OFF_BAR + BAR_BYTES;
  static_assert(BN % 32 == 0 && BN >= 32 && BN <= 256, "MMA N for M=256");
  static_assert(B_BYTES % 1024 == 0, "swizzle atoms");
  static_assert(SMEM_BYTES <= 232448, "shared memory");
};

template <int BN, int STAGES, int EPI, bool DUAL>
__global__ void __launch_bounds__(192, 1)
    tc_gemm_pair_kernel(const __grid_constant__ CUtensorMap mapA, const __grid_constant__ CUtensorMap mapB,
                        const __grid_constant__ CUtensorMap mapB2, const GemmShape sh, const EpiParams ep,
                        const unsigned long long wait_ns) {
  using C = TcGemmPairCfg<BN, STAGES, DUAL>;
  constexpr uint32_t IDESC = idesc_bf16_f32(256, BN, 0, 0);

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
  const int pair = blockIdx.x >> 1, n_pairs = gridDim.x >> 1;

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
  cluster_sync();   // the peer's barriers are initialised before anyone signals them
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
      for (int u = pair; u < sh.units && ok; u += n_pairs) {
        int split, mt, nt;
        gemm_unit(sh, u, split, mt, nt);
        const int arow = mt * 256 + (int)rank * 128;
        const int brow = nt * BN + (int)rank * C::BH;
        for (int kb = 0; kb < sh.kblocks; ++kb) {
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
      // the leader's full barriers count both CTAs' copies: let them land
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
      for (int u = pair; u < sh.units && ok; u += n_pairs) {
        if (!mbar_wait(&acc_empty[abuf], aphase ^ 1u, wait_ns)) break;
        tc_fence_after();
        const uint32_t d = tmem_base + abuf * C::ACC_COLS;
        for (int kb = 0; kb < sh.kblocks; ++kb) {
          if (!mbar_wait(&full[stage], phase, wait_ns)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(sA + stage * C::A_BYTES);
          const uint32_t b_addr = smem_u32(sB + (stage * C::NB) * C::B_BYTES);
#pragma unroll
          for (int k = 0; k < C::BK / 16; ++k) {
            const uint64_t adesc = sw128_desc(a_addr + k * 32, 1024, 16);
            const uint64_t bdesc = sw128_desc(b_addr + k * 32, 1024, 16);
            const uint32_t accum = (kb > 0 || k > 0) ? 1u : 0u;
            tc_mma_f16_pair(d, adesc, bdesc, IDESC, accum);
            if constexpr (DUAL) {
              const uint64_t bdesc2 = sw128_desc(b_addr + C::B_BYTES + k * 32, 1024, 16);
              tc_mma_f16_pair(d + BN, adesc, bdesc2, IDESC, accum);
            }
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
      if (last_buf >= 0) mbar_wait(&acc_full[last_buf], last_parity, wait_ns);
    }
  } else {
    // ------------------------------------------------------------ epilogue (both CTAs)
    const int quarter = warp & 3;
    const int row_in_tile = (int)rank * 128 + quarter * 32 + lane;
    int abuf = 0;
    uint32_t aphase = 0;
    for (int u = pair; u < sh.units; u += n_pairs) {
      int split, mt, nt;
      gemm_unit(sh, u, split, mt, nt);
      const int row = mt * 256 + row_in_tile;
      const bool row_ok = row < sh.rows_a;
      if (!mbar_wait(&acc_full[abuf], aphase, wait_ns)) break;
      tc_fence_after();
      const uint32_t tbase = tmem_base + ((uint32_t)(quarter * 32) << 16) + abuf * C::ACC_COLS;
#pragma unroll 1
      for (int c = 0; c < BN / 32; ++c) {
        float acc[32], acc3[32];
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
        epilogue_chunk<EPI, 32>(ep, sh, acc, acc3, row, row_ok, row, nt * BN + c * 32, split, lane);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(cluster_map(smem_u32(&acc_empty[abuf]), 0));
      if (++abuf == C::ACC_BUFS) { abuf = 0; aphase ^= 1u; }
    }
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync();   // no CTA leaves while its partner may still touch its shared memory
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, 512);
  }
}

}  // namespace l3
