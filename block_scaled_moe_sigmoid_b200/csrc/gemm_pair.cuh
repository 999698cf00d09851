// Routed block-scaled grouped GEMM on CTA pairs (tcgen05 .cta_group::2).
//
// Same product as gemm_kernel<KIND_MX, EPI> in swap-AB form (weights on the MMA's M side,
// token rows on N), but a cluster of two CTAs on two SMs works on one pair tile: 512 weight
// rows (two 256-row m-tiles, one per CTA, each as two 128-row halves) x up to BN_MAX token
// rows.  Each MMA instruction is M=256 (128 rows from each CTA's shared memory) x N (the
// token tile, whose first N/2 rows sit in the even CTA's shared memory and the rest in the
// odd CTA's) x K=32, and each CTA's TMEM receives its own 128 rows x N.  So each SM holds
// its 256 weight rows but only half the token rows per stage: 42 KB instead of 54 KB of
// tiles for the same tensor work (five stages instead of four), and each SM fetches only
// half of each token tile from L2.  The single-CTA routed GEMM moves about as many bytes
// from L2 into shared memory as the GPU delivers to TMA loads on all SMs, and the token
// rows, re-read by every m-tile, are half of them: halving those is the point.
// Measured on the Kimi-K3 prefill shapes, it is nonetheless slower than gemm_kernel's
// single-CTA tiles (each stage now waits for both SMs' loads), so it runs only when the
// 160-row tile configuration is selected explicitly.  Its outputs are bit-identical to the
// single-CTA kernel's: the fp32 accumulation order over K is the same.
//
// Roles per CTA (384 threads), rank 0 = leader, rank 1 = peer:
//   warp 0   weight rows of its own m-tile (TMA .cta_group::2: the completed bytes count on
//            the leader's full barrier) and their scale atoms (bulk copy, local barrier);
//            the leader's also arms its full barrier with both CTAs' weight bytes;
//   warp 10  its half of the token rows (TMA .cta_group::2, leader's barrier) and the whole
//            tile's token scale atoms (bulk copy, local barrier); the leader's also arms
//            its full barrier with the whole tile's token bytes;
//   warp 11  leader: once both CTAs' scale atoms of a stage are in shared memory (the peer
//            forwards its local completion with a remote arrive), copies them into both
//            CTAs' TMEM (tcgen05.cp .cta_group::2) and commits to the stage's full barrier;
//            peer: forwards;
//   warp 1   owns TMEM (allocated for the pair); the leader's lane 0 issues the MMAs and
//            commits each stage's release to both CTAs' empty barriers (multicast) and each
//            tile's accumulator to both CTAs' acc_full;
//   warps 2..9  the swap-AB epilogue on the CTA's own TMEM rows; the accumulator is free
//            again when all 16 epilogue warps of the pair have arrived on the leader's
//            acc_empty.
// Only the leader's producers arrive on its full barrier, each expecting both CTAs' bytes;
// the peer's copies only complete bytes on it (no remote arrivals, which measured 15-18%
// slower).  A stage is full when both CTAs' tiles and the leader's scale copies are done;
// the peer arms nothing before its own empty barrier has released the stage, so its bytes
// always land in the phase the leader is arming.
#pragma once
#include "gemm.cuh"

namespace moe {

template <int BN_MAX, int STAGES>
struct PairCfg {
  static constexpr int BM = 256;                    // weight rows per CTA (two 128-row halves)
  static constexpr int BK = 128;                    // K elements per stage
  static constexpr int A_BYTES = BM * 128;          // FP4 padded to a byte per element
  static constexpr int B_ROWS = BN_MAX / 2;         // this CTA's token rows at most
  static constexpr int B_BYTES = B_ROWS * 128;
  static constexpr int SFA_BYTES = 1024;
  static constexpr int SFB_ATOMS = (BN_MAX + 127) / 128;
  static constexpr int SFB_BYTES = SFB_ATOMS * 512;  // the whole tile's token scales
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int SF_STAGE_BYTES = SFA_BYTES + SFB_BYTES;
  static constexpr int SF_OFFSET = STAGES * STAGE_BYTES;
  static constexpr int CTRL_OFFSET = SF_OFFSET + STAGES * SF_STAGE_BYTES;
  static constexpr int A_TX = BM * BK / 2;          // global bytes of one weight tile
  static constexpr int SMEM_BYTES = CTRL_OFFSET + 1024 /*barriers*/ + 1024 /*align*/;
  static constexpr int TMEM_SF = 2 * BN_MAX;        // after the two accumulator halves
  static constexpr int TMEM_COLS = 512;
  static constexpr int NUM_THREADS = 384;
  static_assert(BN_MAX % 32 == 0 && BN_MAX <= 256, "each CTA holds a multiple of 16 token rows");
  static_assert(SFB_ATOMS <= 2, "two token scale atoms at most");
  static_assert(STAGE_BYTES % 1024 == 0, "stage alignment");
  static_assert(SF_STAGE_BYTES % 128 == 0, "scale atom alignment");
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
  static_assert(TMEM_SF + 16 * STAGES <= TMEM_COLS, "TMEM budget");
  static_assert(STAGES < 8, "barrier block");
};

// Pair tiles: t = group-tile * (m_tiles / 2) + m-tile pair.  CTA `rank` of the pair takes
// m-tile 2 * pair + rank; the MMA's N is the tile's rows rounded up to 32 (16 per CTA).
__device__ __forceinline__ int pair_num_tiles(const GemmArgs& a) {
  return __ldg(a.tile_prefix + a.num_groups) * (a.m_tiles >> 1);
}
__device__ __forceinline__ void pair_decode_tile(const GemmArgs& a, int bn_max, int t, int rank, TileInfo& ti) {
  const int mp_tiles = a.m_tiles >> 1;
  const int gt = t / mp_tiles;
  const int mp = t - gt * mp_tiles;
  gemm_decode_tile(a, bn_max, gt * a.m_tiles + 2 * mp + rank, ti);
  ti.n_mma = (ti.n_valid + 31) & ~31;
}

template <int EPI, int BN_MAX, int STAGES>
__global__ void __launch_bounds__(384, 1)
    gemm_pair_kernel(const __grid_constant__ GemmArgs args, const __grid_constant__ CUtensorMap tmA,
                     const __grid_constant__ BMaps tmB) {
  using C = PairCfg<BN_MAX, STAGES>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* ctrl = smem + C::CTRL_OFFSET;
  uint64_t* full_bar = (uint64_t*)ctrl;           // [STAGES] leader: the stage is ready for MMAs
  uint64_t* empty_bar = full_bar + 8;             // [STAGES] both: the stage may be refilled
  uint64_t* sf_full = empty_bar + 8;              // [STAGES] both: local scale atoms landed
  uint64_t* sf_peer = sf_full + 8;                // [STAGES] leader: the peer's scale atoms landed
  uint64_t* acc_full = sf_peer + 8;               // both: the tile's accumulator is complete
  uint64_t* acc_empty = acc_full + 1;             // leader: all 16 epilogue warps drained it
  uint64_t* drain_bar = acc_empty + 1;
  uint64_t* drain_sf = drain_bar + 1;
  uint32_t* tmem_holder = (uint32_t*)(drain_sf + 1);
  volatile int* abort_flag = (volatile int*)(tmem_holder + 1);
  // Abort cleanup counters: [0] weight producer, [1] token producer (stages issued; the
  // leader's also armed them),
  // [2] leader scale warp (stages committed), [3] leader MMA (full phases consumed),
  // [4] scale warp (sf_full phases consumed).
  int* fills = (int*)(tmem_holder + 2);
  int* stage_n = fills + 8;                       // [STAGES] leader: MMA N of the stage's tile

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int rank = (int)(cluster_ctarank() & 1u);
  const bool leader = rank == 0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      // the leader's weight and token producers (each arming both CTAs' bytes), plus the
      // leader's scale-copy commit
      mbar_init(smem_u32(full_bar + s), 3);
      mbar_init(smem_u32(empty_bar + s), 1);
      mbar_init(smem_u32(sf_full + s), 2);
      mbar_init(smem_u32(sf_peer + s), 1);
    }
    mbar_init(smem_u32(acc_full), 1);
    mbar_init(smem_u32(acc_empty), 16);
    mbar_init(smem_u32(drain_bar), 1);
    mbar_init(smem_u32(drain_sf), 1);
    *abort_flag = 0;
    for (int r = 0; r < 8; ++r) fills[r] = 0;
    fence_mbar_init_cluster();
    prefetch_tmap(&tmA);
  }
  if (warp == 1) {
    tmem_alloc2(smem_u32(tmem_holder), C::TMEM_COLS);
    tmem_relinquish2();
  }
  tc_fence_before();
  cluster_sync();   // both CTAs' barriers are initialised before any remote arrival
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  griddep_wait();
  griddep_launch_dependents();

  const int num_tiles = pair_num_tiles(args);
  const int pair = (int)blockIdx.x >> 1, npairs = (int)gridDim.x >> 1;
  // the leader's barriers as seen from this CTA
  auto leader_addr = [&](const void* p) -> uint32_t { return mapa_shared(smem_u32(p), 0); };

  if (warp == 0) {
    // ------------------------------------------------------------- producer: weights
    const uint64_t pol_a = policy_evict_first();
    int stage = 0;
    uint32_t phase = 0;
    bool ok = true;
    int nfill = 0;
    for (int t = pair; t < num_tiles && ok; t += npairs) {
      TileInfo ti;
      pair_decode_tile(args, BN_MAX, t, rank, ti);
      for (int kt = ti.kb; kt < ti.ke; ++kt) {
        if (lane == 0) {
          ok = mbar_wait_cluster(smem_u32(empty_bar + stage), phase ^ 1, args.status, abort_flag);
          if (ok) {
            const size_t blk = ((size_t)ti.grp * args.m_tiles + ti.mt) * args.k_tiles + kt;
            // the scale atoms first: the leader's copies into TMEM then overlap the tile
            const uint32_t sb = smem_u32(sf_full + stage);
            mbar_arrive_expect_tx(sb, C::SFA_BYTES);
            asm volatile(
                "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], 1024, [%2];" ::"r"(
                    smem_u32(smem + C::SF_OFFSET + stage * C::SF_STAGE_BYTES)),
                "l"(args.sfa + blk * 1024), "r"(sb)
                : "memory");
            const uint32_t fb = leader_addr(full_bar + stage);
            if (leader) mbar_arrive_expect_tx(smem_u32(full_bar + stage), 2 * C::A_TX);
            tma_load_2d_pair(smem_u32(smem + stage * C::STAGE_BYTES), &tmA, fb, 0, (int)(blk * C::BM), pol_a);
          }
        }
        ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
        if (!ok) break;
        ++nfill;
        if (++stage == STAGES) { stage = 0; phase ^= 1; }
      }
    }
    if (lane == 0) fills[0] = nfill;
  } else if (warp == 10) {
    // ------------------------------------------------------------- producer: token rows
    const uint64_t pol_b = policy_evict_last();
    int stage = 0;
    uint32_t phase = 0;
    bool ok = true;
    int nfill = 0;
    for (int t = pair; t < num_tiles && ok; t += npairs) {
      TileInfo ti;
      pair_decode_tile(args, BN_MAX, t, rank, ti);
      const int half = ti.n_mma >> 1;   // this CTA's rows: row0 + rank * half, a multiple of 16
      const int nB = half / BOX_ROWS;
      for (int kt = ti.kb; kt < ti.ke; ++kt) {
        if (lane == 0) ok = mbar_wait_cluster(smem_u32(empty_bar + stage), phase ^ 1, args.status, abort_flag);
        ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
        if (!ok) break;
        if (lane == 0) {
          if (leader) stage_n[stage] = ti.n_mma;
          const int sfb_bytes = ((ti.n_mma + 127) >> 7) * 512;
          const uint32_t sb = smem_u32(sf_full + stage);
          mbar_arrive_expect_tx(sb, sfb_bytes);
          asm volatile(
              "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                  smem_u32(smem + C::SF_OFFSET + stage * C::SF_STAGE_BYTES + C::SFA_BYTES)),
              "l"(args.sfb + ((size_t)ti.gt * args.k_tiles + kt) * SF_TILE_BYTES), "r"(sfb_bytes), "r"(sb)
              : "memory");
          const uint32_t fb = leader_addr(full_bar + stage);
          if (leader) mbar_arrive_expect_tx(smem_u32(full_bar + stage), ti.n_mma * 128);
          tma_load_2d_pair(smem_u32(smem + stage * C::STAGE_BYTES + C::A_BYTES), &tmB.box[nB - 1], fb,
                           (kt % args.kb_wrap) * C::BK, ti.row0 + rank * half, pol_b);
        }
        __syncwarp();
        ++nfill;
        if (++stage == STAGES) { stage = 0; phase ^= 1; }
      }
    }
    if (lane == 0) fills[1] = nfill;
  } else if (warp == 11) {
    // ------------------------------------------------------------- scale atoms -> TMEM
    if (lane == 0) {
      const uint64_t sf_desc0 = smem_desc(smem_u32(smem) + C::SF_OFFSET, 16, 128, 0);
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      int nsf = 0, ncommit = 0;
      for (int t = pair; t < num_tiles && ok; t += npairs) {
        TileInfo ti;
        pair_decode_tile(args, BN_MAX, t, rank, ti);
        const bool h1 = ti.mt * C::BM + 128 < args.M_total;
        const int atoms = (ti.n_mma + 127) >> 7;
        for (int kt = ti.kb; kt < ti.ke; ++kt) {
          ok = mbar_wait(smem_u32(sf_full + stage), phase, args.status, abort_flag);
          if (!ok) break;
          ++nsf;
          if (!leader) {
            mbar_arrive_cluster(leader_addr(sf_peer + stage));   // the peer's atoms are in place
          } else {
            ok = mbar_wait_cluster(smem_u32(sf_peer + stage), phase, args.status, abort_flag);
            if (!ok) break;
            tc_fence_after();
            const uint64_t sfa_desc = sf_desc0 + (uint64_t)((stage * C::SF_STAGE_BYTES) >> 4);
            const uint64_t sfb_desc = sfa_desc + (uint64_t)(C::SFA_BYTES >> 4);
            const uint32_t tsf = tmem_base + C::TMEM_SF + 16 * stage;
            tc_cp2_32x128b_warpx4(tsf, sfa_desc);
            if (h1) tc_cp2_32x128b_warpx4(tsf + 4, sfa_desc + (uint64_t)(512 >> 4));
            tc_cp2_32x128b_warpx4(tsf + 8, sfb_desc);
            if (atoms > 1) tc_cp2_32x128b_warpx4(tsf + 12, sfb_desc + (uint64_t)(512 >> 4));
            tc_commit2(smem_u32(full_bar + stage));
            ++ncommit;
          }
          if (++stage == STAGES) { stage = 0; phase ^= 1; }
        }
      }
      if (leader) {
        // every scale copy this warp issued lands before TMEM is released
        tc_commit2(smem_u32(drain_sf));
        mbar_wait_drain(smem_u32(drain_sf), 0);
      }
      fills[2] = ncommit;
      fills[4] = nsf;
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------- MMA issuer (leader)
    if (leader && lane == 0) {
      const uint64_t desc0 = smem_desc(smem_u32(smem), 16, 1024, 2);
      const int mp_tiles = args.m_tiles >> 1;
      int stage = 0;
      uint32_t phase = 0, acc_phase = 0;
      bool ok = true;
      int nfill = 0;
      for (int t = pair; t < num_tiles && ok; t += npairs) {
        const int mt = 2 * (t % mp_tiles);   // the leader's m-tile (the peer's is mt + 1)
        const bool h1 = mt * C::BM + 128 < args.M_total;
        const int kb = 0, ke = args.k_tiles;
        uint32_t idesc[4];
        bool first = true;
        auto issue_stage = [&](int st, uint32_t acc0) {
          const uint64_t a_desc = desc0 + (uint64_t)((st * C::STAGE_BYTES) >> 4);
          const uint64_t b_desc = a_desc + (uint64_t)(C::A_BYTES >> 4);
          const uint32_t tsf = tmem_base + C::TMEM_SF + 16 * st;
#pragma unroll
          for (int j = 0; j < 4; ++j) {
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              if (h == 1 && !h1) continue;
              mma2_mxf8f6f4(tmem_base + h * BN_MAX, a_desc + (uint64_t)((h * 16384 + 32 * j) >> 4),
                            b_desc + (uint64_t)((32 * j) >> 4), idesc[j], (tsf + 4 * h) | ((uint32_t)j << 30),
                            (tsf + 8) | ((uint32_t)j << 30), j > 0 ? 1u : acc0);
            }
          }
        };
        // one or two K tiles per round, as in gemm_kernel (the second only if it has
        // already landed); each stage released to both CTAs
        for (int kt = kb; kt < ke;) {
          const int kt0 = kt;
          const int stage2 = stage + 1 == STAGES ? 0 : stage + 1;
          const uint32_t phase2 = stage + 1 == STAGES ? phase ^ 1u : phase;
          ok = mbar_wait_cluster(smem_u32(full_bar + stage), phase, args.status, abort_flag);
          if (ok) ++nfill;
          const bool two = ok && kt + 1 < ke && mbar_try_wait_cluster(smem_u32(full_bar + stage2), phase2);
          if (two) ++nfill;
          kt += two ? 2 : 1;
          if (!ok) break;
          if (first) {
            const int n_mma = stage_n[stage];
#pragma unroll
            for (int j = 0; j < 4; ++j) idesc[j] = idesc_mx_e2m1_e4m3(256, n_mma, j, j);
            // the accumulator is free once both CTAs' epilogues drained the previous tile
            ok = mbar_wait_cluster(smem_u32(acc_empty), acc_phase ^ 1, args.status, abort_flag);
            if (!ok) break;
            first = false;
          }
          tc_fence_after();
          issue_stage(stage, kt0 > kb ? 1u : 0u);
          tc_commit2_mc(smem_u32(empty_bar + stage), 0x3);
          if (two) {
            issue_stage(stage2, 1u);
            tc_commit2_mc(smem_u32(empty_bar + stage2), 0x3);
          }
          stage = stage2;
          phase = phase2;
          if (two && ++stage == STAGES) { stage = 0; phase ^= 1; }
        }
        if (!ok) break;
        tc_commit2_mc(smem_u32(acc_full), 0x3);
        acc_phase ^= 1;
      }
      // every MMA issued has finished (it reads the peer's shared memory) before either
      // CTA goes on to release anything
      tc_commit2(smem_u32(drain_bar));
      mbar_wait_drain(smem_u32(drain_bar), 0);
      fills[3] = nfill;
    }
    __syncwarp();
  } else if (warp >= 2 && warp <= 9) {
    // ------------------------------------------------------------- epilogue
    const int q = warp & 3;
    const int sub = (warp - 2) >> 2;
    const uint32_t lane_base = tmem_base + ((uint32_t)(q * 32) << 16);
    const uint32_t acc_empty_leader = leader_addr(acc_empty);
    uint32_t acc_phase = 0;
    for (int t = pair; t < num_tiles; t += npairs) {
      TileInfo ti;
      pair_decode_tile(args, BN_MAX, t, rank, ti);
      bool ok = true;
      if (lane == 0) ok = mbar_wait_cluster(smem_u32(acc_full), acc_phase, args.status, abort_flag);
      ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
      if (!ok) break;
      tc_fence_after();
      auto release_tmem = [&]() {
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(acc_empty_leader);
      };
      epilogue_swapab<KIND_MX, EPI, BN_MAX>(args, ti, lane_base, q, sub, lane, release_tmem);
      acc_phase ^= 1;
    }
  }

  __syncthreads();
  cluster_sync();   // both CTAs' roles have stopped; their counters are final
  if (threadIdx.x == 0) {
    // Abort cleanup (nothing is pending on the normal path): let every copy still in
    // flight into either CTA's shared memory land, supplying the arrivals of roles that
    // stopped early.  The leader's full ring counts both CTAs' producers.
    if (leader) {
      const int arrived[3] = {fills[0], fills[1], fills[2]};
      drain_ring(full_bar, STAGES, arrived, 3, fills[3]);
    }
    drain_ring(sf_full, STAGES, fills, 2, fills[4]);
  }
  __syncthreads();
  cluster_sync();   // the peer's shared memory outlives every access from the leader
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc2(tmem_base, C::TMEM_COLS);
  }
}

}  // namespace moe
