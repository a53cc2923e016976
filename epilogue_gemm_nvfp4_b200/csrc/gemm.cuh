// Block-scaled NVFP4 GEMM with the DiT's follow-on ops fused into the epilogue, for sm_100a.
//
// One persistent CTA per SM walks output tiles of 128 rows x BN weight rows (512 threads):
//   warp 0        TMA producer: per stage, first the scale atoms (bulk copies, counted on `sf_landed`),
//                 then the A/B code tiles (TMA, 128-byte swizzle, bytes counted on `full`), into a ring
//                 of shared-memory stages.
//   warp 1        MMA issuer (one thread): four tcgen05.mma.kind::mxf4nvf4 (K = 64 each) per stage,
//                 accumulating in TMEM; tcgen05.commit frees the stage (`empty`) and, after the last
//                 K step of a tile, hands the accumulator to the epilogue (`acc_full`).
//   warp 2        TMEM allocation / release.
//   warps 4..7    scale stagers: move each stage's scale atoms from shared memory into that stage's
//                 TMEM scale slot with tcgen05.st (replicated into the four 32-lane sub-partitions the
//                 MMA reads), then arrive on the stage's `full` barrier too, so that the MMA thread
//                 waits once per stage: that thread issues an MMA only every ~128 cycles and spends
//                 about 100 of them issuing it, so a second wait per stage would idle the tensor pipe.
//                 This keeps scale traffic off the tensor pipe, and since the atoms land before the
//                 code tiles it overlaps their copy.
//   warps 8..15   epilogue, two warpgroups over the same 128 rows: thread i of warp 8+4e+q owns
//                 accumulator row 32q+i (TMEM lane = row) and half of the tile's columns.  It copies its
//                 columns into registers, releases TMEM at once (`acc_empty`) so the next tile's MMAs
//                 start, then applies bias / head RMSNorm / gated SiLU / residual+gate and the NVFP4
//                 requantisation from registers.  Row-wise reductions stay within the two threads that
//                 hold a row: for the 256-wide head each adds the squares of its 128 columns and the
//                 two partial sums meet in shared memory, so the head is never revisited.
//                 Each warp writes its 32 rows of a 16- or 32-column slice into its own shared-memory
//                 box in the TMA swizzle, and one lane hands the box to a TMA bulk tensor store.
// The per-stage TMEM scale slot is safe to rewrite without extra waits: the producer refills stage s
// only after the commit of the MMAs that read stage s.
#pragma once

#include "ptx.cuh"
#include "quantize.cuh"

namespace nvfp4 {

enum EpiKind : int { kEpiBias = 0, kEpiQkNorm = 1, kEpiGatedSilu = 2, kEpiResidGate = 3 };

enum DeviceError : unsigned int { kErrNone = 0, kErrTimeout = 5 };

// MMAs of K = 64 per pipeline stage: 2 (64-byte rows, 64-byte swizzle) or 4 (128-byte rows).
#ifndef NVFP4_STAGE_KSTEPS
#define NVFP4_STAGE_KSTEPS 4
#endif
constexpr int kStageKSteps = NVFP4_STAGE_KSTEPS;
constexpr int kStageRowBytes = 32 * kStageKSteps;  // code bytes of one row per stage
static_assert(kStageKSteps == 2 || kStageKSteps == 4, "stage depth");

struct GemmArgs {
  int32_t M, N, K;
  int32_t n_out;         // output columns: N, or N / 2 for the gated SiLU
  int32_t num_m_blocks, num_n_blocks, num_tiles;
  int32_t num_m_pairs;   // 256-row blocks (CTA-pair kernel)
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
  unsigned int* out_amax_bits;  // raised to max |bf16 output| (fp32 bit pattern), or nullptr
  // tile order of the persistent walk: 0 = row blocks fastest (a wave shares few weight blocks and
  // keeps A resident in L2), 1 = column blocks fastest (a wave shares few row blocks and keeps W resident)
  int32_t n_fastest;
  const float* row_scale;       // INT8 form: decode scale of each row of A [M]
  const float* col_scale;       // INT8 form: decode scale of each row of W [N]
  unsigned int* error_word;
  uint64_t timeout_ns;
  // split-K: `splits` consecutive work units share one output tile, each summing a contiguous range
  // of K blocks; the first to finish parks its fp32 partial, the second adds it and runs the epilogue.
  int32_t splits;
  int32_t num_units;     // num_tiles * splits
  float* split_partials; // [num_tiles][2][128][cols per thread] fp32
  unsigned int* split_flags;  // [num_tiles], zero before the launch
#ifdef NVFP4_TEST_HOOKS
  // test builds only: the first unit of each split tile parks its partial but never publishes it, so the
  // second unit's bounded wait runs out and the call reports a device timeout
  int32_t test_withhold_split_ready;
#endif
};

struct WorkUnit {
  int tile, mb, nb, kb0, kb1;
};

__device__ __forceinline__ WorkUnit work_unit(const GemmArgs& a, int u, int num_kb) {
  WorkUnit w;
  const int split = u % a.splits;
  w.tile = u / a.splits;
  if (a.n_fastest) {
    w.nb = w.tile % a.num_n_blocks;
    w.mb = w.tile / a.num_n_blocks;
  } else {
    w.mb = w.tile % a.num_m_blocks;
    w.nb = w.tile / a.num_m_blocks;
  }
  w.kb0 = split * num_kb / a.splits;
  w.kb1 = (split + 1) * num_kb / a.splits;
  return w;
}

// kI8: the W8A8 INT8 form of the same kernel (tcgen05.mma.kind::i8, s32 accumulators): no block
// scales to stage, so no scale slots in shared memory or TMEM, and two accumulators even at BN = 256.
template <int BN, bool kI8 = false>
struct GemmCfg {
  static constexpr int BM = 128;
  static constexpr int THREADS = 512;
  static constexpr int KSTEPS = kStageKSteps;           // MMAs of K = 64 per stage
  static constexpr int BK_BYTES = kStageRowBytes;       // 64 * KSTEPS E2M1 elements per stage and row
  static constexpr int A_BYTES = BM * BK_BYTES;
  static constexpr int B_BYTES = BN * BK_BYTES;
  static constexpr int SF_ATOM_BYTES = 512;             // 128 rows x 4 blocks
  static constexpr int SFA_BYTES = kI8 ? 0 : KSTEPS * SF_ATOM_BYTES;
  static constexpr int SFB_BYTES = kI8 ? 0 : (BN / 128) * KSTEPS * SF_ATOM_BYTES;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES + SFA_BYTES + SFB_BYTES;
  static constexpr int ACC_BUFS = (BN == 256 && !kI8) ? 1 : 2;
  static constexpr int SF_COL0 = ACC_BUFS * BN;         // TMEM columns after the accumulator(s)
  static constexpr int SFA_COLS = kI8 ? 0 : KSTEPS * 4;
  static constexpr int SFB_COLS = kI8 ? 0 : KSTEPS * (BN / 32);
  static constexpr int SF_COLS = SFA_COLS + SFB_COLS;
  static constexpr int TMEM_COLS = 512;
  static constexpr int EPI_WARPS = 8;
  static constexpr int XPOSE_BYTES = 1024;              // per epilogue warp: 32 rows x 32 bytes
  static constexpr int AUX_BYTES = 1536;                // barriers, flags, head-norm partial sums
  static constexpr int SS_OFFSET = 512;                 // float [2][128] partial sums of squares
  static constexpr int SMEM_LIMIT = 232448;
  // as many stages as shared memory and the TMEM scale slots allow
  static constexpr int STAGES_SMEM = (SMEM_LIMIT - AUX_BYTES - 1023 - EPI_WARPS * XPOSE_BYTES) / STAGE_BYTES;
  static constexpr int STAGES_TMEM = kI8 ? STAGES_SMEM : (TMEM_COLS - SF_COL0) / (SF_COLS > 0 ? SF_COLS : 1);
  static constexpr int STAGES = STAGES_SMEM < STAGES_TMEM ? STAGES_SMEM : STAGES_TMEM;
  static constexpr int SMEM_BYTES = AUX_BYTES + 1023 + STAGES * STAGE_BYTES + EPI_WARPS * XPOSE_BYTES;
  static constexpr uint32_t IDESC = kI8 ? idesc_i8(BM, BN) : idesc_nvf4(BM, BN);
  static_assert(SF_COL0 + STAGES * SF_COLS <= TMEM_COLS, "TMEM budget");
  static_assert(SF_COLS % 8 == 0, "scale slot is written 8 columns at a time");
  static_assert(SMEM_BYTES <= SMEM_LIMIT, "shared memory budget");
  static_assert(STAGE_BYTES % 1024 == 0, "swizzle atoms stay 1024-byte aligned");
  static_assert((3 * STAGES + 5) * 8 + 16 <= SS_OFFSET, "barrier area");
  static_assert(BM == 128, "the split-K partial layout assumes 128 rows per tile");
  static_assert((SMEM_LIMIT >> 4) < (1 << 14), "operand descriptors advance by adds inside the 14-bit address field");
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

__device__ __forceinline__ void load_bf16x16(const __nv_bfloat16* p, float (&f)[16]) {
  const uint4* q = reinterpret_cast<const uint4*>(p);
#pragma unroll
  for (int v = 0; v < 2; ++v) {
    const uint4 u = __ldg(q + v);
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      f[8 * v + 2 * i] = __uint_as_float(w[i] << 16);
      f[8 * v + 2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
  }
}

// Two floats -> two bf16 (round to nearest even) in one 32-bit word, `lo` in the low half.
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  const __nv_bfloat162 p = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&p);
}

// silu(a) = a / (1 + exp(-a)), with the fast exponential and division intrinsics: a few fp32 ulps of
// relative error for every a.  (The form h + h * tanh(h), h = a / 2, cancels for negative a: there
// tanh is near -1, and the hardware tanh's 2^-11 relative error became several percent of silu(a)
// at a = -5.)  For a below about -88 the exponential overflows and the quotient is -0.
__device__ __forceinline__ float silu(float a) { return __fdividef(a, 1.0f + __expf(-a)); }

__device__ __forceinline__ void tmem_load32(uint32_t taddr, float* v) {
  uint32_t r[32];
  tmem_ld_32x32b_x32(taddr, r);
  tmem_ld_wait();
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

// TMA store maps of the outputs (built on the host; a map is all zeros when its output is absent):
//   out      bf16 [M][ld_out], box 16 columns x 32 rows, 32-byte swizzle
//   q_codes  E2M1 bytes [M][ld_q_codes], box 16 bytes x 32 rows, no swizzle
// The epilogue writes each 32-row block into its warp's 1 KB shared-memory buffer and one lane hands
// it to the TMA engine: row segments 9 KB apart would otherwise cost the load/store unit one line
// transaction each, and that unit also carries the MMA thread's barrier traffic.  The map's row count
// is M, so the engine drops rows at or past M.
struct OutMaps {
  CUtensorMap out;
  CUtensorMap q_codes;
};

// Wait until the TMA engine has read this warp's buffer (the previous store from it), so that it can
// be rewritten.  Lane 0 issues all of the warp's bulk stores.
__device__ __forceinline__ void xpose_acquire() {
  if ((threadIdx.x & 31) == 0) bulk_wait_group_read<0>();
  __syncwarp();
}

// Hand the warp's buffer to the TMA engine as the box at (x, y) of `map`.  `live` is false when the box
// starts at or past the last row or the last column of the output: nothing is stored then (a box that
// starts inside the output and reaches past its edge is clipped by the engine).
__device__ __forceinline__ void xpose_release(const CUtensorMap* map, const uint8_t* xpose, int x, int y, bool live) {
  fence_proxy_async_smem();  // this thread's shared-memory writes become visible to the TMA engine
  __syncwarp();
  if ((threadIdx.x & 31) == 0 && live) {
    tma_store_2d(map, xpose, x, y);
    bulk_commit_group();
  }
}

// Store 16 bf16 values of this lane's row at column col0: lane i writes row i of the 32 x 32-byte box
// in the 32-byte swizzle (the two 16-byte halves swap every 4 rows, which also keeps the shared-memory
// writes free of bank conflicts), then the box goes out with one TMA store.
__device__ __forceinline__ void store_row16_bf16(const OutMaps* om, uint8_t* xpose, int row0, int col0, bool live,
                                                 const uint32_t* w) {
  const int lane = threadIdx.x & 31;
  const int sw = (lane >> 2) & 1;
  xpose_acquire();
  uint4* mine = reinterpret_cast<uint4*>(xpose + lane * 32);
  mine[sw] = make_uint4(w[0], w[1], w[2], w[3]);
  mine[sw ^ 1] = make_uint4(w[4], w[5], w[6], w[7]);
  xpose_release(&om->out, xpose, col0, row0, live);
}

// Store 32 bf16 values of this lane's row at column col0 as one 32-row x 64-byte box in the 64-byte
// swizzle (16-byte chunk j of row r sits at chunk j ^ ((r >> 1) & 3), which keeps the shared-memory
// writes at four wavefronts): half the TMA store operations of two 16-column boxes.  Needs a 2 KB box.
__device__ __forceinline__ void store_row32_bf16(const OutMaps* om, uint8_t* xpose, int row0, int col0, bool live,
                                                 const uint32_t* w) {
  const int lane = threadIdx.x & 31;
  const int sw = (lane >> 1) & 3;
  xpose_acquire();
  uint4* mine = reinterpret_cast<uint4*>(xpose + lane * 64);
#pragma unroll
  for (int j = 0; j < 4; ++j) mine[j ^ sw] = make_uint4(w[4 * j], w[4 * j + 1], w[4 * j + 2], w[4 * j + 3]);
  xpose_release(&om->out, xpose, col0, row0, live);
}

// 32 consecutive output values of one row: bf16 (RNE) output and, when requested, the NVFP4
// re-quantisation of those bf16 values with the caller's tensor scale (the quantiser's block rule).
template <int kBoxBytes>
__device__ __forceinline__ void emit_row32(const GemmArgs& a, const OutMaps* om, uint8_t* xpose, int row0, int row,
                                           int col0, const float* o, float qg, uint32_t& amax_bits) {
  uint32_t packed[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) packed[i] = pack_bf16x2(o[2 * i], o[2 * i + 1]);
  if (a.out_amax_bits != nullptr && row < a.M) {
    uint32_t m = amax_bits;
#pragma unroll
    for (int i = 0; i < 16; ++i) m = max(m, bf16x2_absmax_bits(packed[i]));
    amax_bits = m;
  }
  if (a.out != nullptr) {
    if constexpr (kBoxBytes >= 2048) {
      store_row32_bf16(om, xpose, row0, col0, row0 < a.M && col0 < a.n_out, packed);
    } else {
      store_row16_bf16(om, xpose, row0, col0, row0 < a.M && col0 < a.n_out, packed);
      store_row16_bf16(om, xpose, row0, col0 + 16, row0 < a.M && col0 + 16 < a.n_out, packed + 8);
    }
  }
  if (a.q_codes != nullptr) {
    // codes and scales of this row's two 16-blocks; rows at or past M get zero scales (the padding
    // rows of the scale layout) and zero codes, which the TMA store drops
    uint32_t words[4] = {0u, 0u, 0u, 0u};
    uint32_t sc[2] = {0u, 0u};
    if (row < a.M) {
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
    }
    const int lane = threadIdx.x & 31;
    xpose_acquire();
    *reinterpret_cast<uint4*>(xpose + lane * 16) = make_uint4(words[0], words[1], words[2], words[3]);
    xpose_release(&om->q_codes, xpose, col0 / 2, row0, row0 < a.M && col0 < a.n_out);
    // the scale layout's rows end at the 128-row padding and its blocks at the 4-block padding of a row
    // (a ragged N's last tile reaches past both; its blocks up to the padding get zero scales)
    if (row < a.num_m_blocks * 128 && col0 / 16 < 4 * a.q_k_atoms)
      *reinterpret_cast<uint16_t*>(a.q_scales + scale_offset(row, col0 / 16, a.q_k_atoms)) =
          static_cast<uint16_t>(sc[0] | (sc[1] << 8));
  }
}

// Publish a warp's largest output magnitude (bf16 magnitude bits) with one atomic max on the fp32
// bit pattern; every lane of the warp calls this.
__device__ __forceinline__ void publish_amax(unsigned int* out_bits, uint32_t m) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
  if ((threadIdx.x & 31) == 0 && out_bits != nullptr && m != 0) atomicMax(out_bits, m << 16);
}

// ------------------------------------------------------------------------------------------
// epilogue: registers <- TMEM, release, then math and stores
// ------------------------------------------------------------------------------------------

// kBoxBytes: the per-warp shared-memory store box, 1 KB (32 x 16 bf16) or 2 KB (32 x 32 bf16).
template <int BN, int KIND, int kBoxBytes = 1024>
struct Epilogue {
  static constexpr int COLS = (KIND == kEpiGatedSilu) ? 128 : BN / 2;  // accumulator columns per thread

  // Copy this thread's accumulator columns into `acc` (gated SiLU: its 64 a columns, then the 64
  // matching b columns).
  static __device__ __forceinline__ void load(uint32_t t_acc, int e, float* acc) {
    if constexpr (KIND == kEpiGatedSilu) {
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        tmem_load32(t_acc + 64 * e + 32 * c, acc + 32 * c);              // a
        tmem_load32(t_acc + 128 + 64 * e + 32 * c, acc + 64 + 32 * c);   // b
      }
    } else {
#pragma unroll
      for (int c = 0; c < COLS / 32; ++c) tmem_load32(t_acc + COLS * e + 32 * c, acc + 32 * c);
    }
  }

  // Sum of squares of the biased 256-wide head of this row: each of the row's two threads adds its
  // 128 columns, and the partial sums meet in shared memory (both epilogue warpgroups take part).
  static __device__ __forceinline__ float head_sumsq(const GemmArgs& a, int e, int nb, int row_local, float alpha,
                                                     const float* acc, float* ss_x) {
    float ss = 0.0f;
    const int col_e = nb * BN + COLS * e;
#pragma unroll
    for (int g = 0; g < COLS / 16; ++g) {
      float b[16];
      if (a.bias != nullptr) load_bf16x16(a.bias + col_e + 16 * g, b);
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const float v = acc[16 * g + i] * alpha + (a.bias != nullptr ? b[i] : 0.0f);
        ss = fmaf(v, v, ss);
      }
    }
    ss_x[e * 128 + row_local] = ss;
    named_barrier_sync(2, 256);
    ss += ss_x[(1 - e) * 128 + row_local];
    named_barrier_sync(2, 256);  // the next tile may overwrite the slots only after both reads
    return ss;
  }

  static __device__ __forceinline__ void finish(const GemmArgs& a, const OutMaps* om, uint8_t* xpose, int row0, int row,
                                                int e, int nb,
                                                float alpha, float qg, const __nv_bfloat16* gamma, float ss,
                                                float* acc, uint32_t& amax_bits) {
    if constexpr (KIND == kEpiGatedSilu) {
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        const int ocol = nb * 128 + 64 * e + 32 * c;
        float o[32];
#pragma unroll
        for (int g = 0; g < 2; ++g) {
          float ba[16], bb[16];
          if (a.bias != nullptr) {
            load_bf16x16(a.bias + ocol + 16 * g, ba);
            load_bf16x16(a.bias + a.N / 2 + ocol + 16 * g, bb);
          }
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            float ya = acc[32 * c + 16 * g + i] * alpha, yb = acc[64 + 32 * c + 16 * g + i] * alpha;
            if (a.bias != nullptr) {
              ya += ba[i];
              yb += bb[i];
            }
            o[16 * g + i] = silu(ya) * yb;
          }
        }
        emit_row32<kBoxBytes>(a, om, xpose, row0, row, ocol, o, qg, amax_bits);
      }
    } else {
      const int col_e = nb * BN + COLS * e;
      float rs = 1.0f;
      if (KIND == kEpiQkNorm && gamma != nullptr) rs = rsqrtf(ss * (1.0f / BN) + a.eps);
#pragma unroll
      for (int c = 0; c < COLS / 32; ++c) {
        const int col0 = col_e + 32 * c;
        float* y = acc + 32 * c;
#pragma unroll
        for (int g = 0; g < 2; ++g) {
          // N is a multiple of 16, so a 16-column group lies wholly inside or wholly past it; the last
          // 128-wide tile of a ragged N reads no bias, residual or gate past N (its accumulator columns
          // there are 0: the weight's TMA box fills the rows past N with zeros) and the store map drops
          // those columns
          const bool in_n = col0 + 16 * g < a.N;
          float b[16];
          if (a.bias != nullptr && in_n) {
            load_bf16x16(a.bias + col0 + 16 * g, b);
          } else {
#pragma unroll
            for (int i = 0; i < 16; ++i) b[i] = 0.0f;
          }
#pragma unroll
          for (int i = 0; i < 16; ++i) y[16 * g + i] = y[16 * g + i] * alpha + b[i];
          if (KIND == kEpiQkNorm && gamma != nullptr) {
            float gm[16];
            load_bf16x16(gamma + COLS * e + 32 * c + 16 * g, gm);
#pragma unroll
            for (int i = 0; i < 16; ++i) y[16 * g + i] = y[16 * g + i] * rs * gm[i];
          }
          if constexpr (KIND == kEpiResidGate) {
            float r[16];
            if (row < a.M && in_n) {
              load_bf16x16(a.residual + static_cast<int64_t>(row) * a.ld_res + col0 + 16 * g, r);
            } else {
#pragma unroll
              for (int i = 0; i < 16; ++i) r[i] = 0.0f;
            }
            const float4* gp = reinterpret_cast<const float4*>(a.gate + col0 + 16 * g);
#pragma unroll
            for (int v = 0; v < 4; ++v) {
              const float4 gg = in_n ? __ldg(gp + v) : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
              y[16 * g + 4 * v + 0] = fmaf(gg.x, y[16 * g + 4 * v + 0], r[4 * v + 0]);
              y[16 * g + 4 * v + 1] = fmaf(gg.y, y[16 * g + 4 * v + 1], r[4 * v + 1]);
              y[16 * g + 4 * v + 2] = fmaf(gg.z, y[16 * g + 4 * v + 2], r[4 * v + 2]);
              y[16 * g + 4 * v + 3] = fmaf(gg.w, y[16 * g + 4 * v + 3], r[4 * v + 3]);
            }
          }
        }
        emit_row32<kBoxBytes>(a, om, xpose, row0, row, col0, y, qg, amax_bits);
      }
    }
  }
};

// INT8 form: the accumulator columns hold s32 sums (their bits, as loaded); turn each into fp32 and
// multiply it by its weight row's decode scale.  The row's activation scale enters as the epilogue's
// alpha.  Columns of the gated SiLU: this thread's 64 a columns, then the matching 64 b columns.
template <int BN, int KIND>
__device__ __forceinline__ void i8_scale_columns(const GemmArgs& a, int e, int nb, float* acc) {
  auto scale32 = [&](float* v, int col0) {
    const float4* cs = reinterpret_cast<const float4*>(a.col_scale + col0);
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const float4 c = __ldg(cs + q);
      v[4 * q + 0] = __fmul_rn(__int2float_rn(__float_as_int(v[4 * q + 0])), c.x);
      v[4 * q + 1] = __fmul_rn(__int2float_rn(__float_as_int(v[4 * q + 1])), c.y);
      v[4 * q + 2] = __fmul_rn(__int2float_rn(__float_as_int(v[4 * q + 2])), c.z);
      v[4 * q + 3] = __fmul_rn(__int2float_rn(__float_as_int(v[4 * q + 3])), c.w);
    }
  };
  if constexpr (KIND == kEpiGatedSilu) {
#pragma unroll
    for (int c = 0; c < 2; ++c) {
      scale32(acc + 32 * c, nb * 128 + 64 * e + 32 * c);
      scale32(acc + 64 + 32 * c, a.N / 2 + nb * 128 + 64 * e + 32 * c);
    }
  } else {
    constexpr int COLS = Epilogue<BN, KIND>::COLS;
#pragma unroll
    for (int c = 0; c < COLS / 32; ++c) scale32(acc + 32 * c, nb * BN + COLS * e + 32 * c);
  }
}

constexpr unsigned int kSplitReady = 0x100u;

// Split-K hand-off for one tile (two work units).  Returns true when this CTA now holds the full sum
// in `acc` and must run the epilogue; false when it parked its partial for the other unit (or the
// wait for the other unit's partial ran out of time).  fp32 addition is commutative, so the sum is
// the same bits whichever unit finishes first; the split depends on K only, never on M.
template <int COLS>
__device__ __forceinline__ bool split_exchange(const GemmArgs& a, int tile, int e, int row_local, float* acc,
                                               volatile int* role_slot, volatile int* abort_flag) {
  const int et = threadIdx.x - 256;  // epilogue thread 0..255
  if (et == 0) *role_slot = static_cast<int>(atomicAdd(&a.split_flags[tile], 1u));
  named_barrier_sync(1, 256);
  const int role = *role_slot;
  float4* part = reinterpret_cast<float4*>(a.split_partials +
                                           ((static_cast<int64_t>(tile) * 2 + e) * 128 + row_local) * COLS);
  if ((role & 0xFF) == 0) {
#pragma unroll
    for (int i = 0; i < COLS / 4; ++i) part[i] = make_float4(acc[4 * i], acc[4 * i + 1], acc[4 * i + 2], acc[4 * i + 3]);
    __threadfence();
    named_barrier_sync(1, 256);
#ifdef NVFP4_TEST_HOOKS
    if (et == 0 && !a.test_withhold_split_ready) atomicOr(&a.split_flags[tile], kSplitReady);
#else
    if (et == 0) atomicOr(&a.split_flags[tile], kSplitReady);
#endif
    return false;
  }
  if (et == 0) {
    const uint64_t t0 = global_timer_ns();
    int ok = 1;
    while ((atomicAdd(&a.split_flags[tile], 0u) & kSplitReady) == 0) {
      if (*abort_flag || global_timer_ns() - t0 > a.timeout_ns) {
        ok = 0;
        break;
      }
      __nanosleep(64);
    }
    if (!ok) raise_device_error(a.error_word, kErrTimeout, abort_flag);
    *role_slot = ok ? 1 : -1;
  }
  named_barrier_sync(1, 256);
  if (*role_slot < 0) return false;
  __threadfence();
#pragma unroll
  for (int i = 0; i < COLS / 4; ++i) {
    const float4 p = __ldcg(part + i);
    acc[4 * i] += p.x;
    acc[4 * i + 1] += p.y;
    acc[4 * i + 2] += p.z;
    acc[4 * i + 3] += p.w;
  }
  return true;
}

template <int BN, int KIND, bool kI8 = false>
__global__ void __launch_bounds__(512, 1)
    nvfp4_gemm_kernel(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_b,
                      const __grid_constant__ OutMaps out_maps, const __grid_constant__ GemmArgs args) {
  using C = GemmCfg<BN, kI8>;
  using E = Epilogue<BN, KIND>;
  extern __shared__ uint8_t smem_raw[];
  // small state first, then the 1024-aligned stage ring (128-byte swizzle atoms), then the transposes
  uint64_t* full = reinterpret_cast<uint64_t*>(smem_raw);
  uint64_t* empty = full + C::STAGES;
  uint64_t* sf_landed = empty + C::STAGES;
  uint64_t* acc_full = sf_landed + C::STAGES;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* drain = acc_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* never_abort = abort_flag + 1;  // stays 0: drains must not be cut short by an abort
  volatile int* split_role = never_abort + 1;
  float* ss_x = reinterpret_cast<float*>(smem_raw + C::SS_OFFSET);
  uint8_t* ring = smem_raw + C::AUX_BYTES;
  ring += (1024u - (smem_u32(ring) & 1023u)) & 1023u;
  uint8_t* xpose_all = ring + C::STAGES * C::STAGE_BYTES;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&full[s], kI8 ? 1 : 1 + 4);  // the producer's expect-tx arrival + one per scale-stager warp
      mbar_init(&empty[s], 1);
      mbar_init(&sf_landed[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], C::EPI_WARPS);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    *never_abort = 0;
    fence_mbarrier_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&tmap_a);
    prefetch_tensormap(&tmap_b);
    if (args.out != nullptr) prefetch_tensormap(&out_maps.out);
    if (args.q_codes != nullptr) prefetch_tensormap(&out_maps.q_codes);
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

  if (warp < 4) {
    regs_decrease<56>();
    if (warp == 0) {
      if (lane == 0) {
        // ---------------------------------------------------------------- TMA producer
        int stage = 0;
        uint32_t phase = 0;
        uint32_t armed_mask = 0, armed_parity = 0;
        bool ok = true;
        for (int u = blockIdx.x; ok && u < args.num_units; u += gridDim.x) {
          const WorkUnit wu = work_unit(args, u, num_kb);
          const int mb = wu.mb, nb = wu.nb;
          for (int kb = wu.kb0; kb < wu.kb1; ++kb) {
            if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag, args.timeout_ns)) {
              ok = false;
              break;
            }
            uint8_t* sa = ring + stage * C::STAGE_BYTES;
            uint8_t* sb = sa + C::A_BYTES;
            if constexpr (!kI8) {
              const int ks = min(C::KSTEPS, args.k_steps - kb * C::KSTEPS);
              const uint32_t sf_bytes = static_cast<uint32_t>(ks) * 512u;
              uint8_t* ssfa = sb + C::B_BYTES;
              uint8_t* ssfb = ssfa + C::SFA_BYTES;
              mbar_arrive_expect_tx(&sf_landed[stage], sf_bytes * (1 + BN / 128));
              bulk_load(ssfa, args.sfa + (static_cast<int64_t>(mb) * args.k_atoms + kb * C::KSTEPS) * 512, sf_bytes,
                        &sf_landed[stage]);
#pragma unroll
              for (int j = 0; j < BN / 128; ++j)
                bulk_load(ssfb + j * C::KSTEPS * C::SF_ATOM_BYTES,
                          args.sfb + (static_cast<int64_t>(b_row0<BN, KIND>(args, nb, j) / 128) * args.k_atoms +
                                      kb * C::KSTEPS) * 512,
                          sf_bytes, &sf_landed[stage]);
            }
            mbar_arrive_expect_tx(&full[stage], C::A_BYTES + C::B_BYTES);
            tma_load_2d(sa, &tmap_a, &full[stage], kb * C::BK_BYTES, mb * C::BM);
#pragma unroll
            for (int j = 0; j < BN / 128; ++j)
              tma_load_2d(sb + j * 128 * C::BK_BYTES, &tmap_b, &full[stage], kb * C::BK_BYTES,
                          b_row0<BN, KIND>(args, nb, j));
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
        // (`full` also counts the stagers' arrivals: if they stopped on an error, this wait ends at
        // its time limit instead)
        for (int s = 0; s < C::STAGES; ++s)
          if (armed_mask & (1u << s)) {
            if (!kI8) mbar_wait(&sf_landed[s], (armed_parity >> s) & 1u, never_abort, args.timeout_ns);
            mbar_wait(&full[s], (armed_parity >> s) & 1u, never_abort, args.timeout_ns);
          }
      }
      __syncwarp();
    } else if (warp == 1) {
      if (lane == 0) {
        // ---------------------------------------------------------------- MMA issuer
        // The tensor pipe queues only about two MMAs ahead of this thread, so every instruction
        // spent here between MMAs is lost tensor time: descriptors and TMEM scale addresses are
        // formed once and advanced by adds, and a full stage issues its MMAs fully unrolled.
        constexpr uint64_t kStageDesc = C::STAGE_BYTES >> 4;  // descriptor address units per stage
        const uint64_t a_desc0 = desc_kmajor_swizzled<C::BK_BYTES>(smem_u32(ring));
        const uint64_t b_desc_off = C::A_BYTES >> 4;
        const uint32_t sf_col0 = tmem_base + C::SF_COL0;
        int stage = 0;
        uint32_t phase = 0;
        uint64_t a_desc = a_desc0;
        uint32_t sfa_t = sf_col0;
        int abuf = 0;
        uint32_t aphase = 0;
        bool ok = true;
        for (int u = blockIdx.x; ok && u < args.num_units; u += gridDim.x) {
          const WorkUnit wu = work_unit(args, u, num_kb);
          if (!mbar_wait(&acc_empty[abuf], aphase ^ 1u, abort_flag, args.timeout_ns)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(abuf * BN);
          uint32_t accumulate = 0;
          for (int kb = wu.kb0; kb < wu.kb1; ++kb) {
            if (!mbar_wait(&full[stage], phase, abort_flag, args.timeout_ns)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint64_t b_desc = a_desc + b_desc_off;
            const uint32_t sfb_t = sfa_t + C::SFA_COLS;
            if (kb * C::KSTEPS + C::KSTEPS <= args.k_steps) {
#pragma unroll
              for (int k = 0; k < C::KSTEPS; ++k) {
                if constexpr (kI8)
                  tc_mma_i8(d_tmem, a_desc + 2 * k, b_desc + 2 * k, C::IDESC, accumulate | k);
                else
                  tc_mma_nvf4(d_tmem, a_desc + 2 * k, b_desc + 2 * k, C::IDESC, accumulate | k, sfa_t + k * 4,
                              sfb_t + k * (BN / 32));
              }
            } else {
              const int ks = args.k_steps - kb * C::KSTEPS;  // K tail: 1 .. KSTEPS-1 steps
              for (int k = 0; k < ks; ++k) {
                if constexpr (kI8)
                  tc_mma_i8(d_tmem, a_desc + 2 * k, b_desc + 2 * k, C::IDESC, accumulate | k);
                else
                  tc_mma_nvf4(d_tmem, a_desc + 2 * k, b_desc + 2 * k, C::IDESC, accumulate | k, sfa_t + k * 4,
                              sfb_t + k * (BN / 32));
              }
            }
            accumulate = 1;
            tc_commit(&empty[stage]);
            if (++stage == C::STAGES) {
              stage = 0;
              phase ^= 1u;
              a_desc = a_desc0;
              sfa_t = sf_col0;
            } else {
              a_desc += kStageDesc;
              sfa_t += C::SF_COLS;
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
    }
  } else if (warp < 8) {
    regs_decrease<64>();
    if constexpr (!kI8) {  // the INT8 form has no block scales to stage
      // ------------------------------------------------------------------ scale stagers
      // Lane i of warp 4+q writes TMEM lane 32q+i.  The MMA reads, for row r of a 128-row block, the
      // 4 scales of one K step from column r / 32 of that step's group of 4 columns, identically in
      // every sub-partition; 16-byte row i of a 512-byte scale atom is exactly those 4 columns of lane i.
      const int q = warp & 3;
      constexpr int NV = C::SF_COLS / 4;  // 16-byte vectors per lane and stage
      int stage = 0;
      uint32_t phase = 0;
      for (int u = blockIdx.x; u < args.num_units; u += gridDim.x) {
        const WorkUnit wu = work_unit(args, u, num_kb);
        bool ok = true;
        for (int kb = wu.kb0; kb < wu.kb1; ++kb) {
          const bool got = mbar_wait(&sf_landed[stage], phase, abort_flag, args.timeout_ns);
          if (!__all_sync(0xFFFFFFFFu, got)) {
            ok = false;
            break;
          }
          const uint8_t* ssfa = ring + stage * C::STAGE_BYTES + C::A_BYTES + C::B_BYTES;
          const uint8_t* ssfb = ssfa + C::SFA_BYTES;
          const int ks = min(C::KSTEPS, args.k_steps - kb * C::KSTEPS);
          const uint32_t t_sf = tmem_base + (static_cast<uint32_t>(32 * q) << 16) + C::SF_COL0 + stage * C::SF_COLS;
          // slot column order: A steps 0..KSTEPS-1 (4 columns each), then for each step k the weight's
          // 128-row blocks j = 0 .. BN/128-1 (4 columns each).  The slot's NV vectors (16 bytes each) are
          // gathered, then written with the widest stores (one 32- and one 16-column tcgen05.st for a
          // 48-column slot, one 32-column store for a 32-column slot).
          uint32_t v[4 * NV];
#pragma unroll
          for (int idx = 0; idx < NV; ++idx) {
            int k;
            const uint8_t* src;
            if (idx < C::KSTEPS) {
              k = idx;
              src = ssfa + k * C::SF_ATOM_BYTES;
            } else {
              k = (idx - C::KSTEPS) / (BN / 128);
              src = ssfb + ((idx - C::KSTEPS) % (BN / 128)) * C::KSTEPS * C::SF_ATOM_BYTES + k * C::SF_ATOM_BYTES;
            }
            uint4 x = make_uint4(0, 0, 0, 0);
            if (k < ks) x = *reinterpret_cast<const uint4*>(src + lane * 16);
            v[4 * idx + 0] = x.x;
            v[4 * idx + 1] = x.y;
            v[4 * idx + 2] = x.z;
            v[4 * idx + 3] = x.w;
          }
          static_assert(NV == 12 || NV == 8, "a slot is 48 or 32 columns");
          tmem_st_32x32b_x32(t_sf, v);
          if constexpr (NV == 12) tmem_st_32x32b_x16(t_sf + 32, v + 32);
          tmem_st_wait();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&full[stage]);
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) {
          if (lane == 0) raise_device_error(args.error_word, kErrTimeout, abort_flag);
          break;
        }
      }
    }
  } else {
    regs_increase<192>();
    // ------------------------------------------------------------------ epilogue
    const int e = (warp - 8) >> 2;
    const int q = warp & 3;
    uint8_t* xpose = xpose_all + (warp - 8) * C::XPOSE_BYTES;
    const float alpha_t = kI8 ? 1.0f : __fmul_rn(*args.ga, *args.gb);
    const float qg = args.q_codes != nullptr ? *args.q_g : 1.0f;
    int abuf = 0;
    uint32_t aphase = 0;
    uint32_t amax_bits = 0;
    for (int u = blockIdx.x; u < args.num_units; u += gridDim.x) {
      const WorkUnit wu = work_unit(args, u, num_kb);
      const int mb = wu.mb, nb = wu.nb;
      const __nv_bfloat16* gamma = nullptr;
      if constexpr (KIND == kEpiQkNorm) {
        const int col_base = nb * BN;
        if (col_base >= args.q_col0 && col_base < args.q_col0 + args.qk_cols) gamma = args.gamma_q;
        else if (col_base >= args.k_col0 && col_base < args.k_col0 + args.qk_cols) gamma = args.gamma_k;
      }
      const bool got = mbar_wait(&acc_full[abuf], aphase, abort_flag, args.timeout_ns);
      if (!__all_sync(0xFFFFFFFFu, got)) {  // the tcgen05.ld below needs the whole warp
        if (lane == 0) raise_device_error(args.error_word, kErrTimeout, abort_flag);
        break;
      }
      tc_fence_after();
      const int row0 = mb * C::BM + q * 32;
      const uint32_t t_acc = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(abuf * BN);
      float acc[E::COLS];
      E::load(t_acc, e, acc);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[abuf]);
      if (++abuf == C::ACC_BUFS) {
        abuf = 0;
        aphase ^= 1u;
      }
      // the dequantisation factor of this row: ga * gb, or the INT8 form's activation scale of the row
      // (0 for the padding rows past M, whose outputs the store drops)
      float alpha = alpha_t;
      if constexpr (kI8) {
        alpha = row0 + lane < args.M ? __ldg(args.row_scale + row0 + lane) : 0.0f;
        i8_scale_columns<BN, KIND>(args, e, nb, acc);
      }
      // (the head norm's sum of squares is taken while loading, so the host never splits QK-norm GEMMs)
      if (KIND != kEpiQkNorm && args.splits > 1 &&
          !split_exchange<E::COLS>(args, wu.tile, e, q * 32 + lane, acc, split_role, abort_flag))
        continue;
      float ss = 0.0f;
      if (KIND == kEpiQkNorm && gamma != nullptr) ss = E::head_sumsq(args, e, nb, q * 32 + lane, alpha, acc, ss_x);
      E::finish(args, &out_maps, xpose, row0, row0 + lane, e, nb, alpha, qg, gamma, ss, acc, amax_bits);
    }
    publish_amax(args.out_amax_bits, amax_bits);
    // the TMA stores read this warp's buffer and write the outputs asynchronously: both must be done
    // before the CTA's shared memory is released
    if (lane == 0) bulk_wait_group_all();
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
}

}  // namespace nvfp4
