// Per-row symmetric INT8 quantiser of the W8A8 linear: per-token activations and per-output-row
// weights, with the SmoothQuant channel migration as a per-column multiplier ("Quantizing a Dual-Branch
// Flow-Matching Diffusion Transformer for Consumer GPUs", method section).  For row r:
//
//   x'[k] = x[r,k] * col_mult[k]            (1 / lambda for activations, lambda for weights)
//   s[r]  = max_k |x'| / 127                (1 for an all-zero row)
//   q[r,k] = clamp(RNE(x'[k] * (127 / max_k |x'|)), -127, 127)
//
// each step one binary32 operation rounded to nearest even.  One warp owns one row at a time; lane l
// holds the 16-element blocks l, l + 32, ... and the row is walked twice in chunks of two warp steps
// (1024 elements): first for the row's max, then, re-reading it from L2, for the codes.
#pragma once

#include "quantize.cuh"

namespace nvfp4 {

constexpr int kInt8ChunkSteps = 2;  // warp steps (512 elements each) per chunk of a row

// x' of one 16-element block (8 bf16x2 words) as floats, element 2i from the low half of word i.
__device__ __forceinline__ void scaled_block16(const uint32_t (&w)[8], const float* mult, float (&v)[16]) {
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    v[2 * i] = __uint_as_float(w[i] << 16);
    v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
  if (mult != nullptr) {
    const float4* m4 = reinterpret_cast<const float4*>(mult);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float4 m = __ldg(m4 + j);
      v[4 * j + 0] = __fmul_rn(v[4 * j + 0], m.x);
      v[4 * j + 1] = __fmul_rn(v[4 * j + 1], m.y);
      v[4 * j + 2] = __fmul_rn(v[4 * j + 2], m.z);
      v[4 * j + 3] = __fmul_rn(v[4 * j + 3], m.w);
    }
  }
}

template <bool kVec32>
__global__ void __launch_bounds__(256, 4) int8_quantize_kernel(const __nv_bfloat16* __restrict__ x, int64_t rows,
                                                            int64_t cols, int64_t ldx,
                                                            const float* __restrict__ col_mult,
                                                            int8_t* __restrict__ q, int64_t ld_q,
                                                            float* __restrict__ row_scale) {
  const int lane = threadIdx.x & 31;
  const int64_t nwarps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  const int64_t gwarp = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int bpr = static_cast<int>(cols / 16);
  const int steps = (bpr + 31) / 32;

  for (int64_t row = gwarp; row < rows; row += nwarps) {
    const __nv_bfloat16* xrow = x + row * ldx;
    uint32_t w[kInt8ChunkSteps][8];

    // sweep 1: max |x'| (a max is exact in any order)
    float amax = 0.0f;
    for (int c0 = 0; c0 < steps; c0 += kInt8ChunkSteps) {
#pragma unroll
      for (int s = 0; s < kInt8ChunkSteps; ++s) {
        const int blk = (c0 + s) * 32 + lane;
#pragma unroll
        for (int i = 0; i < 8; ++i) w[s][i] = 0u;
        if (c0 + s < steps && blk < bpr) ld_block32(xrow + blk * 16, kVec32, w[s]);
      }
#pragma unroll
      for (int s = 0; s < kInt8ChunkSteps; ++s) {
        const int blk = (c0 + s) * 32 + lane;
        if (c0 + s >= steps || blk >= bpr) continue;
        float v[16];
        scaled_block16(w[s], col_mult != nullptr ? col_mult + blk * 16 : nullptr, v);
#pragma unroll
        for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(v[i]));
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o));
    const float inv = amax == 0.0f ? 0.0f : __fdiv_rn(127.0f, amax);
    if (lane == 0) row_scale[row] = amax == 0.0f ? 1.0f : __fdiv_rn(amax, 127.0f);

    // sweep 2: codes
    int8_t* qrow = q + row * ld_q;
    for (int c0 = 0; c0 < steps; c0 += kInt8ChunkSteps) {
#pragma unroll
      for (int s = 0; s < kInt8ChunkSteps; ++s) {
        const int blk = (c0 + s) * 32 + lane;
#pragma unroll
        for (int i = 0; i < 8; ++i) w[s][i] = 0u;
        if (c0 + s < steps && blk < bpr) ld_block32(xrow + blk * 16, kVec32, w[s]);
      }
#pragma unroll
      for (int s = 0; s < kInt8ChunkSteps; ++s) {
        const int blk = (c0 + s) * 32 + lane;
        if (c0 + s >= steps || blk >= bpr) continue;
        float v[16];
        scaled_block16(w[s], col_mult != nullptr ? col_mult + blk * 16 : nullptr, v);
        uint32_t packed[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          uint32_t word = 0;
#pragma unroll
          for (int b = 0; b < 4; ++b) {
            const int qi = min(127, max(-127, __float2int_rn(__fmul_rn(v[4 * j + b], inv))));
            word |= (static_cast<uint32_t>(qi) & 0xFFu) << (8 * b);
          }
          packed[j] = word;
        }
        *reinterpret_cast<uint4*>(qrow + blk * 16) = make_uint4(packed[0], packed[1], packed[2], packed[3]);
      }
    }
  }
}

}  // namespace nvfp4
