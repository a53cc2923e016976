// Block-scaled NVFP4 GEMM with the DiT's follow-on ops fused into the epilogue, for sm_100a.
//
// One persistent CTA per SM walks output tiles of 128 rows x BN weight rows.  Warp roles:
//   warp 0      TMA producer: A/B code tiles (128-byte swizzle) and their scale atoms into a ring of
//               shared-memory stages, completion counted on the stage's "full" mbarrier.
//   warp 1      MMA issuer (one thread): per stage, tcgen05.cp of the scale atoms into a TMEM slot
//               owned by that stage, then four tcgen05.mma.kind::mxf4nvf4 (K = 64 each) accumulating
//               in TMEM; tcgen05.commit frees the stage and, after the last K step, publishes the
//               accumulator to the epilogue.
//   warp 2      TMEM allocation / release.
//   warps 4..7  epilogue: thread i of warp 4+q owns accumulator row 32q+i (TMEM lane = row), so every
//               row-wise reduction (the 256-wide head RMSNorm, the 16-element requant blocks) is
//               thread-local: a 256-column tile holds a whole head, there is no cross-fragment
//               exchange and no revisit of the output.
// The per-stage scale slots in TMEM are safe to overwrite without extra waits: the producer only
// refills stage s after the commit of the MMAs that read stage s (and so its TMEM scale slot).
#pragma once

#include "ptx.cuh"
#include "quantize.cuh"

namespace nvfp4 {

enum EpiKind : int { kEpiBias = 0, kEpiQkNorm = 1, kEpiGatedSilu = 2, kEpiResidGate = 3 };

enum DeviceError : unsigned int { kErrNone = 0, kErrTimeout = 5 };

struct GemmArgs {
  int32_t M, N, K;
  int32_t num_m_blocks, num_n_blocks, num_tiles;
  int32_t k_steps;      // K / 64
  int32_t k_atoms;      // scale atoms along K (= K / 64)
  const uint8_t* sfa;
  const uint8_t* sfb;
  const float* ga;
  const float* gb;
  const __nv_bfloat16* bias;
  const __nv_bfloat16* gamma_q;
  const __nv_bfloat16* gamma_k;
  float eps;
  int32_t q_col0, k_col0, qk_cols;
  const __nv_bfloat16* residual;
  int64_t ld_res;
  const float* gate;
  __nv_bfloat16* out;
  int64_t ld_out;
  uint8_t* q_codes;     // NVFP4 re-quantised output, or nullptr
  int64_t ld_q_codes;
  uint8_t* q_scales;
  const float* q_g;
  int32_t q_k_atoms;
  unsigned int* error_word;
  uint64_t timeout_ns;
};

template <int BN>
struct GemmCfg {
  static constexpr int BM = 128;
  static constexpr int BK_BYTES = 128;                  // 256 E2M1 elements per stage and row
  static constexpr int KSTEPS = 4;                      // MMAs of K = 64 per stage
  static constexpr int A_BYTES = BM * BK_BYTES;
  static constexpr int B_BYTES = BN * BK_BYTES;
  static constexpr int SFA_BYTES = 4 * 512;             // 128 rows x 16 blocks
  static constexpr int SFB_BYTES = (BN / 128) * 4 * 512;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES + SFA_BYTES + SFB_BYTES;
  static constexpr int STAGES = BN == 256 ? 4 : 6;
  static constexpr int ACC_BUFS = BN == 256 ? 1 : 2;
  static constexpr int SF_COL0 = ACC_BUFS * BN;         // TMEM columns after the accumulator(s)
  static constexpr int SFA_COLS = KSTEPS * 4;
  static constexpr int SFB_COLS = KSTEPS * (BN / 32);
  static constexpr int SF_COLS = SFA_COLS + SFB_COLS;
  static constexpr int TMEM_COLS = 512;
  static constexpr int BAR_BYTES = 256;
  static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + BAR_BYTES + 1024;
  static constexpr uint32_t IDESC = idesc_nvf4(BM, BN);
  static_assert(SF_COL0 + STAGES * SF_COLS <= TMEM_COLS, "TMEM budget");
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
  static_assert((2 * STAGES + 5) * 8 + 8 <= BAR_BYTES, "barrier area");
};

__device__ __forceinline__ void raise_device_error(unsigned int* word, unsigned int code, volatile int* abort) {
  *abort = 1;
  atomicCAS(word, 0u, code);
}

// First weight row of the j-th 128-row box of tile column block nb.  For the gated SiLU the tile
// pairs the a-rows [128 nb, 128 nb + 128) with the b-rows N/2 + [128 nb, 128 nb + 128).
template <int BN, int KIND>
__device__ __forceinline__ int b_row0(const GemmArgs& a, int nb, int j) {
  if (KIND == kEpiGatedSilu) return (j == 0 ? 0 : a.N / 2) + nb * 128;
  return nb * BN + j * 128;
}

__device__ __forceinline__ void load_bf16x32(const __nv_bfloat16* p, float (&f)[32]) {
  const uint4* q = reinterpret_cast<const uint4*>(p);
#pragma unroll
  for (int v = 0; v < 4; ++v) {
    const uint4 u = __ldg(q + v);
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      f[8 * v + 2 * i] = __uint_as_float(w[i] << 16);
      f[8 * v + 2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
  }
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  return static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(lo))) |
         (static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(hi))) << 16);
}

// Write 32 consecutive output values of one row: bf16 (RNE) and, when requested, their NVFP4
// re-quantisation with the caller's tensor scale (the quantiser's block rule applied to the
// bf16-rounded values).  Rows past M write nothing except zero scales in the padding rows.
__device__ __forceinline__ void emit_row32(const GemmArgs& a, int row, int col0, const float (&o)[32], float qg) {
  uint32_t packed[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) packed[i] = pack_bf16x2(o[2 * i], o[2 * i + 1]);
  if (row < a.M && a.out != nullptr) {
    uint4* dst = reinterpret_cast<uint4*>(a.out + static_cast<int64_t>(row) * a.ld_out + col0);
#pragma unroll
    for (int v = 0; v < 4; ++v) dst[v] = make_uint4(packed[4 * v], packed[4 * v + 1], packed[4 * v + 2], packed[4 * v + 3]);
  }
  if (a.q_codes != nullptr) {
    const int64_t soff = scale_offset(row, col0 / 16, a.q_k_atoms);
    if (row >= a.M) {
      *reinterpret_cast<uint16_t*>(a.q_scales + soff) = 0;
      return;
    }
    uint32_t words[4];
    uint32_t sc[2];
#pragma unroll
    for (int blk = 0; blk < 2; ++blk) {
      float f[16];
      uint32_t mb = 0;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const uint32_t w = packed[8 * blk + i];
        f[2 * i] = __uint_as_float(w << 16);
        f[2 * i + 1] = __uint_as_float(w & 0xFFFF0000u);
        mb = max(mb, bf16x2_absmax_bits(w));
      }
      float inv;
      sc[blk] = block_scale(__uint_as_float(mb << 16), qg, inv);
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        float q[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) q[i] = __fmul_rn(f[8 * h + i], inv);
        words[2 * blk + h] = (inv == 0.0f) ? 0u : e2m1x8(q);
      }
    }
    *reinterpret_cast<uint4*>(a.q_codes + static_cast<int64_t>(row) * a.ld_q_codes + col0 / 2) =
        make_uint4(words[0], words[1], words[2], words[3]);
    *reinterpret_cast<uint16_t*>(a.q_scales + soff) = static_cast<uint16_t>(sc[0] | (sc[1] << 8));
  }
}

__device__ __forceinline__ void tmem_load_f32x32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  tmem_ld_32x32b_x32(taddr, r);
  tmem_ld_wait();
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

// Epilogue for one tile; t_acc addresses this warp's 32 lanes at the tile's first column.
template <int BN, int KIND>
__device__ __forceinline__ void epilogue_tile(const GemmArgs& a, uint32_t t_acc, int row, int nb, float alpha,
                                              float qg) {
  if constexpr (KIND == kEpiGatedSilu) {
    static_assert(BN == 256, "gated SiLU pairs two 128-row weight boxes");
#pragma unroll 1
    for (int c = 0; c < 4; ++c) {
      const int ocol = nb * 128 + c * 32;
      float ya[32], yb[32];
      tmem_load_f32x32(t_acc + c * 32, ya);
      tmem_load_f32x32(t_acc + 128 + c * 32, yb);
#pragma unroll
      for (int i = 0; i < 32; ++i) { ya[i] *= alpha; yb[i] *= alpha; }
      if (a.bias != nullptr) {
        float ba[32], bb[32];
        load_bf16x32(a.bias + ocol, ba);
        load_bf16x32(a.bias + a.N / 2 + ocol, bb);
#pragma unroll
        for (int i = 0; i < 32; ++i) { ya[i] += ba[i]; yb[i] += bb[i]; }
      }
      float o[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) o[i] = ya[i] / (1.0f + __expf(-ya[i])) * yb[i];
      emit_row32(a, row, ocol, o, qg);
    }
  } else {
    const int col_base = nb * BN;
    const __nv_bfloat16* gamma = nullptr;
    if constexpr (KIND == kEpiQkNorm) {
      if (col_base >= a.q_col0 && col_base < a.q_col0 + a.qk_cols) gamma = a.gamma_q;
      else if (col_base >= a.k_col0 && col_base < a.k_col0 + a.qk_cols) gamma = a.gamma_k;
    }
    float rs = 1.0f;
    if (KIND == kEpiQkNorm && gamma != nullptr) {
      // pass 1 over TMEM: sum of squares of the biased head (the tile is exactly one 256-wide head)
      float ss = 0.0f;
#pragma unroll 1
      for (int c = 0; c < BN / 32; ++c) {
        float y[32];
        tmem_load_f32x32(t_acc + c * 32, y);
        float b[32];
        if (a.bias != nullptr) load_bf16x32(a.bias + col_base + c * 32, b);
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const float v = y[i] * alpha + (a.bias != nullptr ? b[i] : 0.0f);
          ss = fmaf(v, v, ss);
        }
      }
      rs = rsqrtf(ss * (1.0f / BN) + a.eps);
    }
#pragma unroll 1
    for (int c = 0; c < BN / 32; ++c) {
      const int col0 = col_base + c * 32;
      float y[32];
      tmem_load_f32x32(t_acc + c * 32, y);
#pragma unroll
      for (int i = 0; i < 32; ++i) y[i] *= alpha;
      if (a.bias != nullptr) {
        float b[32];
        load_bf16x32(a.bias + col0, b);
#pragma unroll
        for (int i = 0; i < 32; ++i) y[i] += b[i];
      }
      if (KIND == kEpiQkNorm && gamma != nullptr) {
        float gm[32];
        load_bf16x32(gamma + c * 32, gm);
#pragma unroll
        for (int i = 0; i < 32; ++i) y[i] = y[i] * rs * gm[i];
      }
      if constexpr (KIND == kEpiResidGate) {
        float r[32];
        if (row < a.M) load_bf16x32(a.residual + static_cast<int64_t>(row) * a.ld_res + col0, r);
        else {
#pragma unroll
          for (int i = 0; i < 32; ++i) r[i] = 0.0f;
        }
        const float4* gp = reinterpret_cast<const float4*>(a.gate + col0);
#pragma unroll
        for (int v = 0; v < 8; ++v) {
          const float4 gg = __ldg(gp + v);
          y[4 * v + 0] = fmaf(gg.x, y[4 * v + 0], r[4 * v + 0]);
          y[4 * v + 1] = fmaf(gg.y, y[4 * v + 1], r[4 * v + 1]);
          y[4 * v + 2] = fmaf(gg.z, y[4 * v + 2], r[4 * v + 2]);
          y[4 * v + 3] = fmaf(gg.w, y[4 * v + 3], r[4 * v + 3]);
        }
      }
      emit_row32(a, row, col0, y, qg);
    }
  }
}

template <int BN, int KIND>
__global__ void __launch_bounds__(256, 1)
    nvfp4_gemm_kernel(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_b,
                      const __grid_constant__ GemmArgs args) {
  using C = GemmCfg<BN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::STAGES * C::STAGE_BYTES);
  uint64_t* empty = full + C::STAGES;
  uint64_t* acc_full = empty + C::STAGES;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* drain = acc_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* never_abort = abort_flag + 1;  // stays 0: drains must not be cut short by an abort

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 4);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    *never_abort = 0;
    fence_mbarrier_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&tmap_a);
    prefetch_tensormap(&tmap_b);
  }
  if (warp == 2) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int num_kb = (args.k_steps + C::KSTEPS - 1) / C::KSTEPS;

  if (warp == 0) {
    if (lane == 0) {
    // ------------------------------------------------------------------ TMA producer
    int stage = 0;
    uint32_t phase = 0;
    uint32_t armed_mask = 0, armed_parity = 0;
    bool ok = true;
    for (int tile = blockIdx.x; ok && tile < args.num_tiles; tile += gridDim.x) {
      const int mb = tile % args.num_m_blocks, nb = tile / args.num_m_blocks;
      for (int kb = 0; kb < num_kb; ++kb) {
        if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag, args.timeout_ns)) {
          ok = false;
          break;
        }
        const int ks = min(C::KSTEPS, args.k_steps - kb * C::KSTEPS);
        const uint32_t sf_bytes = static_cast<uint32_t>(ks) * 512u;
        mbar_arrive_expect_tx(&full[stage], C::A_BYTES + C::B_BYTES + sf_bytes * (1 + BN / 128));
        uint8_t* sa = smem + stage * C::STAGE_BYTES;
        uint8_t* sb = sa + C::A_BYTES;
        uint8_t* ssfa = sb + C::B_BYTES;
        uint8_t* ssfb = ssfa + C::SFA_BYTES;
        tma_load_2d(sa, &tmap_a, &full[stage], kb * C::BK_BYTES, mb * C::BM);
#pragma unroll
        for (int j = 0; j < BN / 128; ++j)
          tma_load_2d(sb + j * 128 * C::BK_BYTES, &tmap_b, &full[stage], kb * C::BK_BYTES,
                      b_row0<BN, KIND>(args, nb, j));
        bulk_load(ssfa, args.sfa + (static_cast<int64_t>(mb) * args.k_atoms + kb * 4) * 512, sf_bytes, &full[stage]);
#pragma unroll
        for (int j = 0; j < BN / 128; ++j)
          bulk_load(ssfb + j * 2048,
                    args.sfb + (static_cast<int64_t>(b_row0<BN, KIND>(args, nb, j) / 128) * args.k_atoms + kb * 4) * 512,
                    sf_bytes, &full[stage]);
        armed_mask |= 1u << stage;
        armed_parity = (armed_parity & ~(1u << stage)) | (phase << stage);
        if (++stage == C::STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
    }
    if (!ok) raise_device_error(args.error_word, kErrTimeout, abort_flag);
    // every copy this thread started must land before the CTA's shared memory is released
    for (int s = 0; s < C::STAGES; ++s)
      if (armed_mask & (1u << s)) mbar_wait(&full[s], (armed_parity >> s) & 1u, never_abort, args.timeout_ns);
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
    // ------------------------------------------------------------------ MMA issuer
    int stage = 0;
    uint32_t phase = 0;
    int abuf = 0;
    uint32_t aphase = 0;
    bool ok = true;
    for (int tile = blockIdx.x; ok && tile < args.num_tiles; tile += gridDim.x) {
      if (!mbar_wait(&acc_empty[abuf], aphase ^ 1u, abort_flag, args.timeout_ns)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(abuf * BN);
      for (int kb = 0; kb < num_kb; ++kb) {
        if (!mbar_wait(&full[stage], phase, abort_flag, args.timeout_ns)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const int ks = min(C::KSTEPS, args.k_steps - kb * C::KSTEPS);
        const uint8_t* sa = smem + stage * C::STAGE_BYTES;
        const uint8_t* sb = sa + C::A_BYTES;
        const uint8_t* ssfa = sb + C::B_BYTES;
        const uint8_t* ssfb = ssfa + C::SFA_BYTES;
        const uint32_t sfa_t = tmem_base + C::SF_COL0 + stage * C::SF_COLS;
        const uint32_t sfb_t = sfa_t + C::SFA_COLS;
        for (int k = 0; k < ks; ++k) tc_cp_32x128b_warpx4(sfa_t + k * 4, desc_scale_block(smem_u32(ssfa + k * 512)));
#pragma unroll
        for (int j = 0; j < BN / 128; ++j)
          for (int k = 0; k < ks; ++k)
            tc_cp_32x128b_warpx4(sfb_t + k * (BN / 32) + j * 4, desc_scale_block(smem_u32(ssfb + j * 2048 + k * 512)));
        const uint32_t a_addr = smem_u32(sa), b_addr = smem_u32(sb);
        for (int k = 0; k < ks; ++k)
          tc_mma_nvf4(d_tmem, desc_kmajor_sw128(a_addr + k * 32), desc_kmajor_sw128(b_addr + k * 32), C::IDESC,
                      (kb | k) != 0 ? 1u : 0u, sfa_t + k * 4, sfb_t + k * (BN / 32));
        tc_commit(&empty[stage]);
        if (++stage == C::STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (!ok) break;
      tc_commit(&acc_full[abuf]);
      if (++abuf == C::ACC_BUFS) {
        abuf = 0;
        aphase ^= 1u;
      }
    }
    if (!ok) raise_device_error(args.error_word, kErrTimeout, abort_flag);
    // every tcgen05 operation this thread issued must finish before TMEM and smem are released
    tc_commit(drain);
    mbar_wait(drain, 0, never_abort, args.timeout_ns);
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ------------------------------------------------------------------ epilogue
    const int q = warp & 3;
    const float alpha = __fmul_rn(*args.ga, *args.gb);
    const float qg = args.q_codes != nullptr ? *args.q_g : 1.0f;
    int abuf = 0;
    uint32_t aphase = 0;
    for (int tile = blockIdx.x; tile < args.num_tiles; tile += gridDim.x) {
      const int mb = tile % args.num_m_blocks, nb = tile / args.num_m_blocks;
      const bool got = mbar_wait(&acc_full[abuf], aphase, abort_flag, args.timeout_ns);
      if (!__all_sync(0xFFFFFFFFu, got)) {  // the tcgen05.ld below needs the whole warp
        if (lane == 0) raise_device_error(args.error_word, kErrTimeout, abort_flag);
        break;
      }
      tc_fence_after();
      const int row = mb * C::BM + q * 32 + lane;
      const uint32_t t_acc = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(abuf * BN);
      epilogue_tile<BN, KIND>(args, t_acc, row, nb, alpha, qg);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[abuf]);
      if (++abuf == C::ACC_BUFS) {
        abuf = 0;
        aphase ^= 1u;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
}

}  // namespace nvfp4
