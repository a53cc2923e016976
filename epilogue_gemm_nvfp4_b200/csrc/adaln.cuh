// The quantiser with the adaLN prologue of a DiT block fused in front of it:
//
//   rstd[r] = 1 / sqrt(mean_k x[r,k]^2 + eps)
//   u[r,k]  = bf16( x[r,k] * rstd[r] * (1 + scale[b,k]) + shift[b,k] ),   b = r / rows_per_sample
//   codes, scales = the NVFP4 block rule on u with the tensor decode scale g
//
// so the normalised, modulated activation never makes a round trip through memory before the QKV or
// FFN-up GEMM.  One warp owns one row at a time: the row's 16-element blocks are spread over the
// lanes (lane l holds blocks l, l + 32, ...; 512 elements per warp step), the sum of squares is a
// per-lane fp32 sum reduced by a butterfly (every lane ends with the same bits), and each lane then
// modulates, rounds to bf16 and quantises its own blocks with the quantiser's block code.
//
// The row is walked in chunks of kAdalnChunkSteps warp steps, twice: the first sweep streams it from
// memory for the sum of squares, the second reads it again (from L2, where the first sweep just left
// it) to modulate and quantise.  Holding a whole 4608-wide row in registers instead needs 124-167
// registers per thread and leaves 12-16 warps per SM; the kernel is bound by instruction issue and
// dependent arithmetic, not by memory, so it ran slower (81-86 us against 77 us for [16896, 4608]).
//
// With a dynamic tensor scale there are two launches of the same kernel: the amax pass computes u for
// every row and reduces max |u| (its last CTA writes g), then the quantise pass recomputes u (the same
// instructions on the same inputs, so the same bits) and encodes it, walking the rows back to front so
// that its first rows are still in L2.
#pragma once

#include "quantize.cuh"

namespace nvfp4 {

constexpr int kAdalnChunkSteps = 2;  // warp steps (512 elements each) per chunk of a row

struct AdalnArgs {
  const __nv_bfloat16* x;
  int64_t rows, cols, ldx;
  const __nv_bfloat16* shift;  // [samples, ld_mod] or null (no shift)
  const __nv_bfloat16* scale;  // [samples, ld_mod] or null (multiplier 1)
  int64_t ld_mod;
  int64_t rows_per_sample;     // 0: every row uses sample 0
  float eps;
  // quantise pass
  const float* g_src;
  uint8_t* codes;
  int64_t ld_codes;
  uint8_t* scales;
  int64_t k_atoms;
  float* rstd;                 // [rows] or null
  __nv_bfloat16* u;            // [rows, ld_u] or null
  int64_t ld_u;
  // amax pass
  unsigned int* state;
  float* tensor_scale;
};

__device__ __forceinline__ void ld_mod16(const __nv_bfloat16* p, uint32_t (&v)[8]) {
  const uint4 a = __ldg(reinterpret_cast<const uint4*>(p));
  const uint4 b = __ldg(reinterpret_cast<const uint4*>(p) + 1);
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
  v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}

// u = bf16(x * rstd * (1 + scale) + shift) for one 16-element block (8 bf16x2 words each): the
// product x * rstd rounded to fp32, the multiplier 1 + scale rounded to fp32, then one fused
// multiply-add and one rounding to bf16.
__device__ __forceinline__ void modulate_block16(const uint32_t (&w)[8], float rstd, const __nv_bfloat16* sh,
                                                 const __nv_bfloat16* sc, uint32_t (&u)[8]) {
  uint32_t shw[8], scw[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) shw[i] = scw[i] = 0u;
  if (sh) ld_mod16(sh, shw);
  if (sc) ld_mod16(sc, scw);
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float lo = __fmaf_rn(__fmul_rn(__uint_as_float(w[i] << 16), rstd),
                               __fadd_rn(1.0f, __uint_as_float(scw[i] << 16)), __uint_as_float(shw[i] << 16));
    const float hi = __fmaf_rn(__fmul_rn(__uint_as_float(w[i] & 0xFFFF0000u), rstd),
                               __fadd_rn(1.0f, __uint_as_float(scw[i] & 0xFFFF0000u)),
                               __uint_as_float(shw[i] & 0xFFFF0000u));
    const __nv_bfloat162 p = __floats2bfloat162_rn(lo, hi);  // lo in the low half
    u[i] = *reinterpret_cast<const uint32_t*>(&p);
  }
}

// The modulation of a single sample as a shared-memory table: for bf16x2 word i of the block a lane
// holds in warp step st, entry (st * 8 + i) * 32 + lane is {1 + scale, shift} of the word's two
// columns, in fp32.  A warp step's read of one word index is 32 consecutive 16-byte entries, so the
// reads are free of bank conflicts, and the per-element unpacking and the 1 + scale add happen once
// per CTA instead of once per row.
constexpr int kAdalnTableMaxSteps = 11;  // up to 5632 columns: 44 KB of table, under the 48 KB default with the static reduction buffer

__device__ __forceinline__ int adaln_table_index(int col) {
  const int blk = col >> 4, i = (col & 15) >> 1;
  return ((blk >> 5) * 8 + i) * 32 + (blk & 31);
}

__device__ void fill_adaln_table(float4* tab, const AdalnArgs& a) {
  for (int c = 2 * static_cast<int>(threadIdx.x); c < a.cols; c += 2 * static_cast<int>(blockDim.x)) {
    float m0 = 1.0f, m1 = 1.0f, s0 = 0.0f, s1 = 0.0f;
    if (a.scale) {
      const uint32_t w = *reinterpret_cast<const uint32_t*>(a.scale + c);
      m0 = __fadd_rn(1.0f, __uint_as_float(w << 16));
      m1 = __fadd_rn(1.0f, __uint_as_float(w & 0xFFFF0000u));
    }
    if (a.shift) {
      const uint32_t w = *reinterpret_cast<const uint32_t*>(a.shift + c);
      s0 = __uint_as_float(w << 16);
      s1 = __uint_as_float(w & 0xFFFF0000u);
    }
    tab[adaln_table_index(c)] = make_float4(m0, s0, m1, s1);
  }
}

// modulate_block16 from the table (the same operations on the same fp32 values, so the same bits).
__device__ __forceinline__ void modulate_block16_tab(const uint32_t (&w)[8], float rstd, const float4* tab, int st,
                                                     int lane, uint32_t (&u)[8]) {
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float4 t = tab[(st * 8 + i) * 32 + lane];
    const float lo = __fmaf_rn(__fmul_rn(__uint_as_float(w[i] << 16), rstd), t.x, t.y);
    const float hi = __fmaf_rn(__fmul_rn(__uint_as_float(w[i] & 0xFFFF0000u), rstd), t.z, t.w);
    const __nv_bfloat162 p = __floats2bfloat162_rn(lo, hi);
    u[i] = *reinterpret_cast<const uint32_t*>(&p);
  }
}

// Steps [c0, c0 + kAdalnChunkSteps) of a row into registers (zeros outside the row).
template <bool kVec32>
__device__ __forceinline__ void ld_row_chunk(const __nv_bfloat16* xrow, int c0, int steps, int bpr, int lane,
                                             uint32_t (&w)[kAdalnChunkSteps][8]) {
#pragma unroll
  for (int s = 0; s < kAdalnChunkSteps; ++s) {
    const int blk = (c0 + s) * 32 + lane;
#pragma unroll
    for (int i = 0; i < 8; ++i) w[s][i] = 0u;
    if (c0 + s < steps && blk < bpr) ld_block32(xrow + blk * 16, kVec32, w[s]);
  }
}

// kTable: one sample for every row and at most kAdalnTableMaxSteps warp steps per row; the modulation
// then comes from the shared-memory table (dynamic shared memory of steps * 4 KB).
template <bool kAmaxPass, bool kReverse, bool kVec32, bool kTable>
__global__ void __launch_bounds__(256, 4) adaln_quantize_kernel(const AdalnArgs a) {
  extern __shared__ float4 adaln_tab[];
  if constexpr (kTable) {
    fill_adaln_table(adaln_tab, a);
    __syncthreads();
  }
  const int lane = threadIdx.x & 31;
  const int64_t nwarps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  const int64_t gwarp = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int bpr = static_cast<int>(a.cols / 16);
  const int steps = (bpr + 31) / 32;
  const float g = kAmaxPass ? 1.0f : *a.g_src;
  uint32_t umax = 0;  // amax pass: largest bf16 magnitude field of u seen by this lane

  for (int64_t t = gwarp; t < a.rows; t += nwarps) {
    const int64_t row = kReverse ? a.rows - 1 - t : t;
    const __nv_bfloat16* xrow = a.x + row * a.ldx;
    uint32_t w[kAdalnChunkSteps][8];

    // sweep 1: sum of squares (each square of a bf16 is exact in fp32)
    float ss = 0.0f;
    for (int c0 = 0; c0 < steps; c0 += kAdalnChunkSteps) {
      ld_row_chunk<kVec32>(xrow, c0, steps, bpr, lane, w);
#pragma unroll
      for (int s = 0; s < kAdalnChunkSteps; ++s) {
        float p = 0.0f;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const float lo = __uint_as_float(w[s][i] << 16), hi = __uint_as_float(w[s][i] & 0xFFFF0000u);
          p = __fmaf_rn(lo, lo, p);
          p = __fmaf_rn(hi, hi, p);
        }
        ss = __fadd_rn(ss, p);
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss = __fadd_rn(ss, __shfl_xor_sync(0xFFFFFFFFu, ss, o));
    const float ms = __fdiv_rn(ss, static_cast<float>(a.cols));
    const float rstd = __fdiv_rn(1.0f, __fsqrt_rn(__fadd_rn(ms, a.eps)));
    if (!kAmaxPass && a.rstd != nullptr && lane == 0) a.rstd[row] = rstd;

    const int64_t b = a.rows_per_sample ? row / a.rows_per_sample : 0;
    const __nv_bfloat16* shrow = a.shift ? a.shift + b * a.ld_mod : nullptr;
    const __nv_bfloat16* scrow = a.scale ? a.scale + b * a.ld_mod : nullptr;
    uint8_t* crow = kAmaxPass ? nullptr : a.codes + row * a.ld_codes;
    uint8_t* srow = kAmaxPass ? nullptr
                              : a.scales + ((row >> 7) * a.k_atoms) * 512 + (row & 31) * 16 + ((row >> 5) & 3) * 4;
    __nv_bfloat16* urow = (!kAmaxPass && a.u != nullptr) ? a.u + row * a.ld_u : nullptr;

    // sweep 2: modulate, round to bf16, then reduce (amax pass) or quantise
    for (int c0 = 0; c0 < steps; c0 += kAdalnChunkSteps) {
      ld_row_chunk<kVec32>(xrow, c0, steps, bpr, lane, w);
#pragma unroll
      for (int s = 0; s < kAdalnChunkSteps; ++s) {
        if (c0 + s >= steps) break;  // warp-uniform
        const int blk = (c0 + s) * 32 + lane;
        const bool valid = blk < bpr;
        uint32_t u[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) u[i] = 0u;
        if (valid) {
          if constexpr (kTable)
            modulate_block16_tab(w[s], rstd, adaln_tab, c0 + s, lane, u);
          else
            modulate_block16(w[s], rstd, shrow ? shrow + blk * 16 : nullptr, scrow ? scrow + blk * 16 : nullptr, u);
        }
        if (kAmaxPass) {
#pragma unroll
          for (int i = 0; i < 8; ++i) umax = max(umax, max(u[i] & 0x7FFFu, (u[i] >> 16) & 0x7FFFu));
        } else {
          if (urow != nullptr && valid) {
            uint4* dst = reinterpret_cast<uint4*>(urow + blk * 16);
            dst[0] = make_uint4(u[0], u[1], u[2], u[3]);
            dst[1] = make_uint4(u[4], u[5], u[6], u[7]);
          }
          store_block16(u, g, blk, valid, lane, crow, srow);
        }
      }
    }
  }

  if (kAmaxPass) {
    const uint32_t m = cta_max_u32(umax);
    if (threadIdx.x == 0) finish_tensor_scale(m, a.state, a.tensor_scale);
  } else {
    // zero the scale rows that pad the tensor to a multiple of 128 rows
    const int64_t pad_words = (((a.rows + 127) & ~int64_t(127)) - a.rows) * a.k_atoms;
    const int64_t nthr = static_cast<int64_t>(gridDim.x) * blockDim.x;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < pad_words; i += nthr) {
      const int64_t r = a.rows + i / a.k_atoms, at = i % a.k_atoms;
      *reinterpret_cast<uint32_t*>(a.scales + scale_offset(r, at * 4, a.k_atoms)) = 0u;
    }
  }
}

}  // namespace nvfp4
