// The fused NVFP4 linear on CTA pairs (tcgen05 cta_group::2), for tiles of 256 rows x 256 weight rows.
//
// A cluster of two CTAs on neighbouring SMs owns a 256 x 256 output tile.  CTA r holds rows
// [128r, 128r+128) of A and rows [128r, 128r+128) of the tile's 256 B rows in its shared memory.  The
// leader's (rank 0) MMA warp issues tcgen05.mma.cta_group::2 with M = 256, N = 256, which
// reads both CTAs' shared memory and writes each CTA's 128 rows of D into that CTA's TMEM.  Each SM
// therefore receives half of the B codes it would load for a one-CTA 128 x 256 tile: a third less
// TMA and shared-memory traffic per FLOP, and a stage of 38 KB instead of 54 KB (5 stages).
//
// Roles per CTA:
//   warp 0     producer: its A box, its half of B and its scale atoms (A's for its own rows, B's for
//              all 256 rows), all with the paired TMA form, whose bytes are counted on the leader's
//              `full` barrier (the leader arms it for both CTAs' bytes).  No multicast loads.
//   warp 1     leader only: the MMA issuer, the whole warp converged with one elected lane issuing.
//              Per stage it copies the stage's twelve scale atoms from both CTAs' shared memory into
//              their TMEM scale slot (tcgen05.cp, which the tensor pipe runs in order with the MMAs
//              that follow), then issues the four MMAs; commits go to both CTAs' `empty` / `acc_full`.
//   warp 2     TMEM allocation (paired form) before the roles start and release after they end.
//   warps 2-7  idle while the roles run.
//   warps 8-15 epilogue of this CTA's 128 rows; the accumulator release is an arrival on the
//              leader's `acc_empty` (16 arrivals: 8 warps per CTA).
// 128-wide tiles stay on the one-CTA kernel.  Split-K units exchange partial sums per (pair tile,
// rank) exactly as the one-CTA kernel does per tile.
#pragma once

#include "gemm.cuh"

namespace nvfp4 {

struct GemmPairCfg {
  static constexpr int BM = 128;                         // rows of A per CTA
  static constexpr int BN = 256;                         // B rows per pair tile
  static constexpr int THREADS = 512;
  static constexpr int KSTEPS = kStageKSteps;
  static constexpr int BK_BYTES = kStageRowBytes;
  static constexpr int A_BYTES = BM * BK_BYTES;
  static constexpr int B_BYTES = (BN / 2) * BK_BYTES;    // this CTA's half of B
  static constexpr int SF_ATOM_BYTES = 512;
  static constexpr int SFA_BYTES = KSTEPS * SF_ATOM_BYTES;
  static constexpr int SFB_BYTES = (BN / 128) * KSTEPS * SF_ATOM_BYTES;  // both 128-row blocks of B
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES + SFA_BYTES + SFB_BYTES;
  static constexpr int SF_COL0 = BN;                     // TMEM columns after the accumulator
  static constexpr int SFA_COLS = KSTEPS * 4;
  static constexpr int SFB_COLS = KSTEPS * (BN / 32);
  static constexpr int SF_COLS = SFA_COLS + SFB_COLS;
  static constexpr int TMEM_COLS = 512;
  static constexpr int EPI_WARPS = 8;
  static constexpr int XPOSE_BYTES = 2048;             // per epilogue warp: 32 rows x 64 bytes
  static constexpr int AUX_BYTES = 1536;
  static constexpr int SS_OFFSET = 512;
  static constexpr int SMEM_LIMIT = 232448;
  static constexpr int STAGES_SMEM = (SMEM_LIMIT - AUX_BYTES - 1023 - EPI_WARPS * XPOSE_BYTES) / STAGE_BYTES;
  static constexpr int STAGES_TMEM = (TMEM_COLS - SF_COL0) / SF_COLS;
  static constexpr int STAGES = STAGES_SMEM < STAGES_TMEM ? STAGES_SMEM : STAGES_TMEM;
  static constexpr int SMEM_BYTES = AUX_BYTES + 1023 + STAGES * STAGE_BYTES + EPI_WARPS * XPOSE_BYTES;
  static constexpr uint32_t IDESC = idesc_nvf4(2 * BM, BN);
  static_assert(SF_COL0 + STAGES * SF_COLS <= TMEM_COLS, "TMEM budget");
  static_assert(SF_COLS % 4 == 0, "a scale atom fills four TMEM columns");
  static_assert(SMEM_BYTES <= SMEM_LIMIT, "shared memory budget");
  static_assert(STAGE_BYTES % 1024 == 0, "swizzle atoms stay 1024-byte aligned");
  static_assert((3 * STAGES + 5) * 8 + 16 <= SS_OFFSET, "barrier area");
  static_assert((SMEM_LIMIT >> 4) < (1 << 14), "operand descriptors advance by adds inside the 14-bit address field");
  // the epilogue and its column split are those of the one-CTA 256-wide tile
  static_assert(GemmCfg<256>::EPI_WARPS == EPI_WARPS, "epilogue");
};

// TMA maps over the block-scale bytes viewed as rows of one 512-byte atom (128 x uint32): a box of
// four rows is the four atoms of one 128-row block for one stage.
struct ScaleMaps {
  CUtensorMap sfa, sfb;
};

struct PairUnit {
  int tile, mp, nb;  // pair tile = 256-row block pair x 256-wide B block
  int kb0, kb1;      // this unit's range of stages along K (split-K)
};

// As in the one-CTA kernel, the `splits` units of one tile are adjacent in the grid-stride order, so
// they run in the same wave on neighbouring clusters.
__device__ __forceinline__ PairUnit pair_unit(const GemmArgs& a, int u, int num_kb) {
  PairUnit w;
  const int split = u % a.splits;
  w.tile = u / a.splits;
  if (a.n_fastest) {
    w.nb = w.tile % a.num_n_blocks;
    w.mp = w.tile / a.num_n_blocks;
  } else {
    w.mp = w.tile % a.num_m_pairs;
    w.nb = w.tile / a.num_m_pairs;
  }
  w.kb0 = split * num_kb / a.splits;
  w.kb1 = (split + 1) * num_kb / a.splits;
  return w;
}

// kSplit: the instantiation with the split-K exchange (the host uses it when splits > 1)
template <int KIND, bool kSplit>
__global__ void __launch_bounds__(512, 1) __cluster_dims__(2, 1, 1)
    nvfp4_gemm_pair_kernel(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_b,
                           const __grid_constant__ ScaleMaps sf_maps, const __grid_constant__ OutMaps out_maps,
                           const __grid_constant__ GemmArgs args) {
  using C = GemmPairCfg;
  using E = Epilogue<256, KIND, C::XPOSE_BYTES>;
  extern __shared__ uint8_t smem_raw[];
  uint64_t* full = reinterpret_cast<uint64_t*>(smem_raw);
  uint64_t* empty = full + C::STAGES;
  uint64_t* acc_full = empty + C::STAGES;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* drain = acc_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* never_abort = abort_flag + 1;
  volatile int* split_role = never_abort + 1;
  float* ss_x = reinterpret_cast<float*>(smem_raw + C::SS_OFFSET);
  uint8_t* ring = smem_raw + C::AUX_BYTES;
  ring += (1024u - (smem_u32(ring) & 1023u)) & 1023u;
  uint8_t* xpose_all = ring + C::STAGES * C::STAGE_BYTES;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const int cluster = blockIdx.x >> 1;
  const int num_clusters = gridDim.x >> 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      // leader's copy: its expect-tx arrival for both CTAs' bytes
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 2 * C::EPI_WARPS);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    *never_abort = 0;
    fence_mbarrier_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&tmap_a);
    prefetch_tensormap(&tmap_b);
    prefetch_tensormap(&sf_maps.sfa);
    prefetch_tensormap(&sf_maps.sfb);
    if (args.out != nullptr) prefetch_tensormap(&out_maps.out);
    if (args.q_codes != nullptr) prefetch_tensormap(&out_maps.q_codes);
  }
  if (warp == 2) {
    tmem_alloc_pair(tmem_slot, C::TMEM_COLS);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // both CTAs' barriers are initialised before any remote arrival
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int num_kb = (args.k_steps + C::KSTEPS - 1) / C::KSTEPS;

  if (warp < 4) {
    regs_decrease<56>();
    if (warp == 0) {
      if (lane == 0) {
        // ---------------------------------------------------------------- TMA producer (both CTAs)
        int stage = 0;
        uint32_t phase = 0;
        bool ok = true;
        for (int u = cluster; ok && u < args.num_units; u += num_clusters) {
          const PairUnit pu = pair_unit(args, u, num_kb);
          // this CTA's 128-row block of A; a block wholly past M reads zeros (codes and scales)
          const int mb = 2 * pu.mp + static_cast<int>(rank);
          for (int kb = pu.kb0; kb < pu.kb1; ++kb) {
            if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag, args.timeout_ns)) {
              ok = false;
              break;
            }
            uint8_t* sa = ring + stage * C::STAGE_BYTES;
            uint8_t* sb = sa + C::A_BYTES;
            uint8_t* ssfa = sb + C::B_BYTES;
            uint8_t* ssfb = ssfa + C::SFA_BYTES;
            const uint32_t leader_full = cluster_addr(&full[stage], 0);
            if (rank == 0) mbar_arrive_expect_tx(&full[stage], 2 * C::STAGE_BYTES);
            tma_load_2d_pair(sa, &tmap_a, leader_full, kb * C::BK_BYTES, mb * C::BM);
            tma_load_2d_pair(sb, &tmap_b, leader_full, kb * C::BK_BYTES,
                             b_row0<256, KIND>(args, pu.nb, static_cast<int>(rank)));
            // scale atoms: rows of the scale maps are atoms, ordered along K within a 128-row block;
            // a K tail loads the next atoms too, which no MMA reads
            tma_load_2d_pair(ssfa, &sf_maps.sfa, leader_full, 0, mb * args.k_atoms + kb * C::KSTEPS);
#pragma unroll
            for (int j = 0; j < C::BN / 128; ++j)
              tma_load_2d_pair(ssfb + j * C::KSTEPS * C::SF_ATOM_BYTES, &sf_maps.sfb, leader_full, 0,
                               (b_row0<256, KIND>(args, pu.nb, j) / 128) * args.k_atoms + kb * C::KSTEPS);
            if (++stage == C::STAGES) {
              stage = 0;
              phase ^= 1u;
            }
          }
        }
        // every box this CTA loads is counted on the leader's `full`, which the leader's MMA thread
        // consumes before the final cluster barrier
        if (!ok) raise_device_error(args.error_word, kErrTimeout, abort_flag);
      }
      __syncwarp();
    } else if (warp == 1) {
      if (rank == 0) {
        // ---------------------------------------------------------------- MMA issuer (leader)
        // The whole warp runs this loop converged and one elected lane issues each tcgen05 instruction;
        // every operand is warp-uniform (the TMEM base is broadcast from lane 0 so that the compiler
        // can prove it), and each wait's outcome is agreed by a vote.
        const uint32_t t_base = __shfl_sync(0xFFFFFFFFu, tmem_base, 0);
        constexpr uint64_t kStageDesc = C::STAGE_BYTES >> 4;
        const uint64_t a_desc0 = desc_kmajor_swizzled<C::BK_BYTES>(smem_u32(ring));
        const uint64_t b_desc_off = C::A_BYTES >> 4;
        const uint64_t sf_desc0 = desc_scale_atom(smem_u32(ring + C::A_BYTES + C::B_BYTES));
        const uint32_t sf_col0 = t_base + C::SF_COL0;
        int stage = 0;
        uint32_t phase = 0;
        uint64_t a_desc = a_desc0;
        uint64_t sf_desc = sf_desc0;
        uint32_t sfa_t = sf_col0;
        uint32_t aphase = 0;
        bool ok = true;
        for (int u = cluster; ok && u < args.num_units; u += num_clusters) {
          const PairUnit pu = pair_unit(args, u, num_kb);
          if (!__all_sync(0xFFFFFFFFu, mbar_wait(&acc_empty[0], aphase ^ 1u, abort_flag, args.timeout_ns))) {
            ok = false;
            break;
          }
          tc_fence_after();
          uint32_t accumulate = 0;
          for (int kb = pu.kb0; kb < pu.kb1; ++kb) {
            if (!__all_sync(0xFFFFFFFFu, mbar_wait(&full[stage], phase, abort_flag, args.timeout_ns))) {
              ok = false;
              break;
            }
            tc_fence_after();
            // scale slot: atom v (A's atoms k = 0..3, then B's atoms k = 0..3 of both 128-row blocks,
            // interleaved by block) to columns 4v..4v+3, where the MMAs below read them
#pragma unroll
            for (int v = 0; v < C::SF_COLS / 4; ++v) {
              const int off = v < C::KSTEPS ? v * C::SF_ATOM_BYTES
                                            : C::SFA_BYTES + ((v - C::KSTEPS) % (C::BN / 128)) * C::KSTEPS * C::SF_ATOM_BYTES +
                                                  ((v - C::KSTEPS) / (C::BN / 128)) * C::SF_ATOM_BYTES;
              tc_cp_pair_32x128b_warpx4_warp(sfa_t + 4 * v, sf_desc + (off >> 4));
            }
            const uint64_t b_desc = a_desc + b_desc_off;
            const uint32_t sfb_t = sfa_t + C::SFA_COLS;
            if (kb * C::KSTEPS + C::KSTEPS <= args.k_steps) {
#pragma unroll
              for (int k = 0; k < C::KSTEPS; ++k)
                tc_mma_nvf4_pair_warp(t_base, a_desc + 2 * k, b_desc + 2 * k, C::IDESC, accumulate | k, sfa_t + k * 4,
                                      sfb_t + k * (C::BN / 32));
            } else {
              const int ks = args.k_steps - kb * C::KSTEPS;
              for (int k = 0; k < ks; ++k)
                tc_mma_nvf4_pair_warp(t_base, a_desc + 2 * k, b_desc + 2 * k, C::IDESC, accumulate | k, sfa_t + k * 4,
                                      sfb_t + k * (C::BN / 32));
            }
            accumulate = 1;
            tc_commit_pair_warp(&empty[stage], 0x3);
            if (++stage == C::STAGES) {
              stage = 0;
              phase ^= 1u;
              a_desc = a_desc0;
              sf_desc = sf_desc0;
              sfa_t = sf_col0;
            } else {
              a_desc += kStageDesc;
              sf_desc += kStageDesc;
              sfa_t += C::SF_COLS;
            }
          }
          if (!ok) break;
          tc_commit_pair_warp(&acc_full[0], 0x3);
          aphase ^= 1u;
        }
        if (!ok && lane == 0) raise_device_error(args.error_word, kErrTimeout, abort_flag);
        tc_commit_pair_warp(drain, 0x1);
        mbar_wait(drain, 0, never_abort, args.timeout_ns);
      }
      __syncwarp();
    }
  } else if (warp < 8) {
    regs_decrease<64>();  // idle: the scale atoms reach TMEM through the MMA thread's copies
  } else {
    regs_increase<192>();
    // ------------------------------------------------------------------ epilogue (both CTAs)
    const int e = (warp - 8) >> 2;
    const int q = warp & 3;
    uint8_t* xpose = xpose_all + (warp - 8) * C::XPOSE_BYTES;
    const float alpha = __fmul_rn(*args.ga, *args.gb);
    const float qg = args.q_codes != nullptr ? *args.q_g : 1.0f;
    const uint32_t leader_acc_empty = cluster_addr(&acc_empty[0], 0);
    uint32_t aphase = 0;
    uint32_t amax_bits = 0;
    for (int u = cluster; u < args.num_units; u += num_clusters) {
      const PairUnit pu = pair_unit(args, u, num_kb);
      const int mb = 2 * pu.mp + static_cast<int>(rank);
      const int nb = pu.nb;
      const __nv_bfloat16* gamma = nullptr;
      if constexpr (KIND == kEpiQkNorm) {
        const int col_base = nb * 256;
        if (col_base >= args.q_col0 && col_base < args.q_col0 + args.qk_cols) gamma = args.gamma_q;
        else if (col_base >= args.k_col0 && col_base < args.k_col0 + args.qk_cols) gamma = args.gamma_k;
      }
      const bool got = mbar_wait(&acc_full[0], aphase, abort_flag, args.timeout_ns);
      if (!__all_sync(0xFFFFFFFFu, got)) {
        if (lane == 0) raise_device_error(args.error_word, kErrTimeout, abort_flag);
        break;
      }
      tc_fence_after();
      const int row0 = mb * C::BM + q * 32;
      const uint32_t t_acc = tmem_base + (static_cast<uint32_t>(q * 32) << 16);
      float acc[E::COLS];
      E::load(t_acc, e, acc);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(leader_acc_empty);
      aphase ^= 1u;
      // split-K: the unit that finishes first parks its partial sums and moves on; the second adds
      // them and runs the epilogue (exchange slot = this CTA's half of the pair tile)
      if constexpr (kSplit && KIND != kEpiQkNorm) {
        if (!split_exchange<E::COLS>(args, 2 * pu.tile + static_cast<int>(rank), e, q * 32 + lane, acc,
                                     split_role, abort_flag))
          continue;
      }
      float ss = 0.0f;
      if (KIND == kEpiQkNorm && gamma != nullptr) ss = E::head_sumsq(args, e, nb, q * 32 + lane, alpha, acc, ss_x);
      E::finish(args, &out_maps, xpose, row0, row0 + lane, e, nb, alpha, qg, gamma, ss, acc, amax_bits);
    }
    publish_amax(args.out_amax_bits, amax_bits);
    if (lane == 0) bulk_wait_group_all();
    __syncwarp();
  }

  // the leader's MMAs read both CTAs' shared memory and write both TMEMs, and each CTA arrives on the
  // other's barriers: neither CTA frees TMEM or exits before both are done
  tc_fence_before();
  __syncthreads();
  cluster_sync();
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, C::TMEM_COLS);
  }
}

}  // namespace nvfp4
