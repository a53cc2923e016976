// Bandwidth-bound NVFP4 kernels: the amax pass, the quantiser, its one-thread finalise step, and the
// dequantiser.  All loads and stores are 16-byte vectors; a warp covers 256 consecutive elements of
// a row (16 blocks of 16) per step, so every load and every code store is coalesced.
#pragma once

#include "ptx.cuh"

namespace nvfp4 {

constexpr float kTensorScaleDivisor = 2688.0f;  // 6 (largest E2M1) * 448 (largest E4M3)

// Byte offset of the scale of row r, block c in the padded tensor-core layout (k_atoms = blocks per
// row / 4, rounded up): 512-byte atoms of 128 rows x 4 blocks, K-major atom order.
__host__ __device__ __forceinline__ int64_t scale_offset(int64_t r, int64_t c, int64_t k_atoms) {
  return ((r >> 7) * k_atoms + (c >> 2)) * 512 + (r & 31) * 16 + ((r >> 5) & 3) * 4 + (c & 3);
}

__device__ __forceinline__ uint4 ld_stream(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

__device__ __forceinline__ uint32_t bf16x2_absmax_bits(uint32_t w) {
  return max(w & 0x7FFFu, (w >> 16) & 0x7FFFu);
}

// ------------------------------------------------------------------------------------------
// amax: max |x| over a bf16 matrix.  For finite bf16, |x| orders like its 15-bit magnitude field,
// so the reduction runs on integers and one atomicMax per CTA publishes the fp32 bit pattern.
// ------------------------------------------------------------------------------------------

// max of one value per thread over the CTA (valid in thread 0); blockDim.x <= 1024
__device__ __forceinline__ uint32_t cta_max_u32(uint32_t m) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
  __shared__ uint32_t red[32];
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x == 0)
    for (int w = 1; w < static_cast<int>(blockDim.x >> 5); ++w) m = max(m, red[w]);
  return m;
}

// max over this CTA's share of the matrix of the bf16 magnitude bits (valid in thread 0)
__device__ __forceinline__ uint32_t block_absmax_bits(const __nv_bfloat16* __restrict__ x, int64_t rows, int64_t cols,
                                                      int64_t ldx) {
  uint32_t m = 0;
  const int64_t nthreads = static_cast<int64_t>(gridDim.x) * blockDim.x;
  const int64_t tid = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (ldx == cols) {
    const int64_t groups = rows * cols / 8;  // 8 bf16 per 16-byte load
    const uint4* p = reinterpret_cast<const uint4*>(x);
    int64_t g = tid;
    for (; g + 3 * nthreads < groups; g += 4 * nthreads) {
      uint4 v[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) v[u] = ld_stream(p + g + u * nthreads);
#pragma unroll
      for (int u = 0; u < 4; ++u)
        m = max(m, max(max(bf16x2_absmax_bits(v[u].x), bf16x2_absmax_bits(v[u].y)),
                       max(bf16x2_absmax_bits(v[u].z), bf16x2_absmax_bits(v[u].w))));
    }
    for (; g < groups; g += nthreads) {
      const uint4 v = ld_stream(p + g);
      m = max(m, max(max(bf16x2_absmax_bits(v.x), bf16x2_absmax_bits(v.y)),
                     max(bf16x2_absmax_bits(v.z), bf16x2_absmax_bits(v.w))));
    }
  } else {
    const int64_t gpr = cols / 8;
    for (int64_t r = blockIdx.x; r < rows; r += gridDim.x) {
      const uint4* p = reinterpret_cast<const uint4*>(x + r * ldx);
      for (int64_t g = threadIdx.x; g < gpr; g += blockDim.x) {
        const uint4 v = ld_stream(p + g);
        m = max(m, max(max(bf16x2_absmax_bits(v.x), bf16x2_absmax_bits(v.y)),
                       max(bf16x2_absmax_bits(v.z), bf16x2_absmax_bits(v.w))));
      }
    }
  }
  return cta_max_u32(m);
}

__global__ void __launch_bounds__(256) amax_kernel(const __nv_bfloat16* __restrict__ x, int64_t rows,
                                                   int64_t cols, int64_t ldx, unsigned int* __restrict__ out_bits) {
  const uint32_t m = block_absmax_bits(x, rows, cols, ldx);
  if (threadIdx.x == 0 && m) atomicMax(out_bits, m << 16);  // bf16 magnitude -> fp32 bit pattern
}

// Thread 0 of every CTA of a grid: publish the CTA's max (bf16 magnitude bits), then take a ticket;
// the CTA with the last ticket writes g = amax / 2688 (1 for an all-zero tensor) and puts the
// per-stream state {amax bits, CTAs done} back to zero for the next call on the stream.
__device__ __forceinline__ void finish_tensor_scale(uint32_t m, unsigned int* state, float* tensor_scale) {
  if (m) atomicMax(&state[0], m << 16);  // bf16 magnitude -> fp32 bit pattern
  __threadfence();
  if (atomicAdd(&state[1], 1u) == gridDim.x - 1) {
    __threadfence();
    const float amax = __uint_as_float(atomicOr(&state[0], 0u));
    *tensor_scale = (amax == 0.0f) ? 1.0f : __fdiv_rn(amax, kTensorScaleDivisor);
    state[0] = 0u;
    state[1] = 0u;
  }
}

// The same reduction, finished in place: the last CTA to finish writes the tensor decode scale
// g = amax / 2688 (1 for an all-zero tensor).  `state` is the caller's per-stream pair {amax bits,
// CTAs done}, zero on entry; the last CTA puts it back to zero for the next call on the stream.  Each
// CTA publishes its max before it takes its ticket (atomicMax, fence, atomicAdd), so the CTA that draws
// the last ticket sees every CTA's max.
__global__ void __launch_bounds__(256) amax_scale_kernel(const __nv_bfloat16* __restrict__ x, int64_t rows,
                                                         int64_t cols, int64_t ldx, unsigned int* __restrict__ state,
                                                         float* __restrict__ tensor_scale) {
  const uint32_t m = block_absmax_bits(x, rows, cols, ldx);
  if (threadIdx.x == 0) finish_tensor_scale(m, state, tensor_scale);
}

// The block rule for one 16-element block, given its amax and the tensor decode scale g:
// returns the E4M3 byte and the fp32 reciprocal of d = e4m3(s) * g (0 when d == 0).
__device__ __forceinline__ uint32_t block_scale(float amax_b, float g, float& inv) {
  const float r = __fdiv_rn(amax_b, g);
  const float sf = __fdiv_rn(r, 6.0f);
  const uint32_t s = e4m3_satfinite(sf);
  const float d = __fmul_rn(e4m3_to_float(s), g);
  inv = (d == 0.0f) ? 0.0f : __frcp_rn(d);
  return s;
}

// The block rule on one 16-element block held as 8 bf16x2 words (element 2i in the low half of word
// i): returns the E4M3 scale byte and writes the 16 codes two per byte, element 2i in the low nibble
// (all codes 0 when d == 0).  `inv` is 1/d, 0 when d == 0.
__device__ __forceinline__ uint32_t quantize_block16(const uint32_t (&w)[8], float g, uint32_t (&packed)[2],
                                                     float& inv) {
  uint32_t m2 = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) m2 = __vmaxu2(m2, w[i] & 0x7FFF7FFFu);
  const uint32_t mb = max(m2 & 0xFFFFu, m2 >> 16);
  const uint32_t sc = block_scale(__uint_as_float(mb << 16), g, inv);
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    float q[8];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      q[2 * i] = __fmul_rn(__uint_as_float(w[4 * h + i] << 16), inv);
      q[2 * i + 1] = __fmul_rn(__uint_as_float(w[4 * h + i] & 0xFFFF0000u), inv);
    }
    packed[h] = (inv == 0.0f) ? 0u : e2m1x8(q);
  }
  return sc;
}

// Quantise one block per lane and store it: lane `lane` of the warp holds block `blk` of a row whose
// codes start at `crow` and whose scales start at `srow` (the row's first scale word in the atom
// layout).  Every lane of the warp takes part (the scale bytes of four lanes form one 32-bit word);
// lanes with valid == false store nothing.
__device__ __forceinline__ void store_block16(const uint32_t (&w)[8], float g, int blk, bool valid, int lane,
                                              uint8_t* crow, uint8_t* srow) {
  uint32_t packed[2];
  float inv;
  uint32_t sc = quantize_block16(w, g, packed, inv);
  if (!valid) sc = 0;
  if (valid) *reinterpret_cast<uint2*>(crow + static_cast<int64_t>(blk) * 8) = make_uint2(packed[0], packed[1]);
  const uint32_t s1 = __shfl_down_sync(0xFFFFFFFFu, sc, 1);
  const uint32_t s2 = __shfl_down_sync(0xFFFFFFFFu, sc, 2);
  const uint32_t s3 = __shfl_down_sync(0xFFFFFFFFu, sc, 3);
  if ((lane & 3) == 0 && valid)
    *reinterpret_cast<uint32_t*>(srow + static_cast<int64_t>(blk >> 2) * 512) = sc | (s1 << 8) | (s2 << 16) | (s3 << 24);
}

// ------------------------------------------------------------------------------------------
// quantise.  Lane l of a warp step owns one 16-element block (32 bytes, one 256-bit load); a warp
// step covers 32 consecutive blocks of a row and a task up to kQuantStepsPerTask steps of one row.
// The block rule runs once per block in its own lane; four lanes' scale bytes form one aligned
// 32-bit word of the scale layout.  With kReverse the tasks run from the end of the tensor
// backwards, so right after the amax pass (which streams the tensor front to back) the first tasks
// re-read from L2 what that pass left there.
// ------------------------------------------------------------------------------------------

constexpr int kQuantStepsPerTask = 16;  // up to 16 x 512 elements of one row per warp task
constexpr int kQuantUnroll = 2;         // 32-byte loads in flight per lane

__device__ __forceinline__ void ld_block32(const __nv_bfloat16* p, bool vec32, uint32_t (&w)[8]) {
  if (vec32) {
    asm volatile("ld.global.L1::no_allocate.v8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : "=r"(w[0]), "=r"(w[1]), "=r"(w[2]), "=r"(w[3]), "=r"(w[4]), "=r"(w[5]), "=r"(w[6]), "=r"(w[7])
                 : "l"(p));
  } else {
    const uint4 a = ld_stream(p), b = ld_stream(p + 8);
    w[0] = a.x; w[1] = a.y; w[2] = a.z; w[3] = a.w;
    w[4] = b.x; w[5] = b.y; w[6] = b.z; w[7] = b.w;
  }
}

template <bool kReverse, bool kVec32>
__global__ void __launch_bounds__(256, 6) quantize_kernel(const __nv_bfloat16* __restrict__ x, int64_t rows,
                                                       int64_t cols, int64_t ldx, const float* __restrict__ scale_src,
                                                       uint8_t* __restrict__ codes, int64_t ld_codes,
                                                       uint8_t* __restrict__ scales, int64_t k_atoms) {
  const float g = *scale_src;
  const int lane = threadIdx.x & 31;
  const int64_t nwarps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  const int64_t gwarp = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int bpr = static_cast<int>(cols / 16);                 // blocks per row
  const int steps = (bpr + 31) / 32;
  const int chunks = (steps + kQuantStepsPerTask - 1) / kQuantStepsPerTask;
  const int per_chunk = (steps + chunks - 1) / chunks;  // equal chunks of at most kQuantStepsPerTask steps
  const int64_t total = rows * chunks;

  for (int64_t t = gwarp; t < total; t += nwarps) {
    const int64_t tt = kReverse ? total - 1 - t : t;
    const int64_t row = tt / chunks;
    const int chunk = static_cast<int>(tt - row * chunks);
    const int st_begin = chunk * per_chunk;
    const int st_end = min(steps, st_begin + per_chunk);
    const __nv_bfloat16* xrow = x + row * ldx;
    uint8_t* crow = codes + row * ld_codes;
    uint8_t* srow = scales + ((row >> 7) * k_atoms) * 512 + (row & 31) * 16 + ((row >> 5) & 3) * 4;
    for (int st = st_begin; st < st_end; st += kQuantUnroll) {
      uint32_t w[kQuantUnroll][8];
#pragma unroll
      for (int u = 0; u < kQuantUnroll; ++u) {
        const int blk = (st + u) * 32 + lane;
#pragma unroll
        for (int i = 0; i < 8; ++i) w[u][i] = 0;
        if (st + u < st_end && blk < bpr) ld_block32(xrow + blk * 16, kVec32, w[u]);
      }
#pragma unroll
      for (int u = 0; u < kQuantUnroll; ++u) {
        if (st + u >= st_end) break;  // warp-uniform
        const int blk = (st + u) * 32 + lane;
        store_block16(w[u], g, blk, blk < bpr, lane, crow, srow);
      }
    }
  }

  // zero the scale rows that pad the tensor to a multiple of 128 rows
  const int64_t pad_rows = ((rows + 127) & ~int64_t(127)) - rows;
  const int64_t pad_words = pad_rows * k_atoms;
  const int64_t nthr = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < pad_words; i += nthr) {
    const int64_t r = rows + i / k_atoms, a = i % k_atoms;
    *reinterpret_cast<uint32_t*>(scales + scale_offset(r, a * 4, k_atoms)) = 0u;
  }
}

// ------------------------------------------------------------------------------------------
// dequantise: one thread per 16-element block.
// ------------------------------------------------------------------------------------------

// ------------------------------------------------------------------------------------------
// fake quantisation: y = dequantise(quantise(x, g)) in bf16, one pass, no codes kept (the forward of
// quantisation-aware training).  Per block: the quantiser's block rule and codes, then the
// dequantiser's decode (e2m1(code) * (e4m3(s) * g), each product in fp32, then bf16 RNE), so y equals
// nvfp4_quantize followed by nvfp4_dequantize bit for bit.  Same task layout as quantize_kernel.
// ------------------------------------------------------------------------------------------

template <bool kReverse, bool kVec32>
__global__ void __launch_bounds__(256, 6) fake_quantize_kernel(const __nv_bfloat16* __restrict__ x, int64_t rows,
                                                            int64_t cols, int64_t ldx,
                                                            const float* __restrict__ scale_src,
                                                            __nv_bfloat16* __restrict__ y, int64_t ldy) {
  const float g = *scale_src;
  const int lane = threadIdx.x & 31;
  const int64_t nwarps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  const int64_t gwarp = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int bpr = static_cast<int>(cols / 16);
  const int steps = (bpr + 31) / 32;
  const int chunks = (steps + kQuantStepsPerTask - 1) / kQuantStepsPerTask;
  const int per_chunk = (steps + chunks - 1) / chunks;
  const int64_t total = rows * chunks;

  for (int64_t t = gwarp; t < total; t += nwarps) {
    const int64_t tt = kReverse ? total - 1 - t : t;
    const int64_t row = tt / chunks;
    const int chunk = static_cast<int>(tt - row * chunks);
    const int st_begin = chunk * per_chunk;
    const int st_end = min(steps, st_begin + per_chunk);
    const __nv_bfloat16* xrow = x + row * ldx;
    __nv_bfloat16* yrow = y + row * ldy;
    for (int st = st_begin; st < st_end; st += kQuantUnroll) {
      uint32_t w[kQuantUnroll][8];
#pragma unroll
      for (int u = 0; u < kQuantUnroll; ++u) {
        const int blk = (st + u) * 32 + lane;
#pragma unroll
        for (int i = 0; i < 8; ++i) w[u][i] = 0;
        if (st + u < st_end && blk < bpr) ld_block32(xrow + blk * 16, kVec32, w[u]);
      }
#pragma unroll
      for (int u = 0; u < kQuantUnroll; ++u) {
        if (st + u >= st_end) break;  // warp-uniform
        const int blk = (st + u) * 32 + lane;
        if (blk >= bpr) continue;
        uint32_t packed[2];
        float inv;
        const uint32_t sc = quantize_block16(w[u], g, packed, inv);
        const float d = __fmul_rn(e4m3_to_float(sc), g);
        uint32_t o[8];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const uint32_t byte = (packed[h] >> (8 * i)) & 0xFFu;
            const __nv_bfloat16 lo = __float2bfloat16_rn(__fmul_rn(e2m1_to_float(byte & 0xFu), d));
            const __nv_bfloat16 hi = __float2bfloat16_rn(__fmul_rn(e2m1_to_float(byte >> 4), d));
            o[4 * h + i] = static_cast<uint32_t>(__bfloat16_as_ushort(lo)) |
                           (static_cast<uint32_t>(__bfloat16_as_ushort(hi)) << 16);
          }
        }
        uint4* dst = reinterpret_cast<uint4*>(yrow + blk * 16);
        dst[0] = make_uint4(o[0], o[1], o[2], o[3]);
        dst[1] = make_uint4(o[4], o[5], o[6], o[7]);
      }
    }
  }
}

__global__ void __launch_bounds__(256) dequantize_kernel(const uint8_t* __restrict__ codes, int64_t ld_codes,
                                                         const uint8_t* __restrict__ scales,
                                                         const float* __restrict__ gptr, int64_t rows, int64_t cols,
                                                         int64_t k_atoms, __nv_bfloat16* __restrict__ out,
                                                         int64_t ld_out) {
  const float g = *gptr;
  const int64_t bpr = cols / 16;
  const int64_t total = rows * bpr;
  const int64_t nthr = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total; i += nthr) {
    const int64_t r = i / bpr, b = i - r * bpr;
    const uint2 c = *reinterpret_cast<const uint2*>(codes + r * ld_codes + b * 8);
    const float d = __fmul_rn(e4m3_to_float(scales[scale_offset(r, b, k_atoms)]), g);
    uint32_t o[8];
#pragma unroll
    for (int i2 = 0; i2 < 8; ++i2) {
      const uint32_t byte = ((i2 < 4 ? c.x : c.y) >> (8 * (i2 & 3))) & 0xFFu;
      const __nv_bfloat16 lo = __float2bfloat16_rn(__fmul_rn(e2m1_to_float(byte & 0xFu), d));
      const __nv_bfloat16 hi = __float2bfloat16_rn(__fmul_rn(e2m1_to_float(byte >> 4), d));
      o[i2] = static_cast<uint32_t>(__bfloat16_as_ushort(lo)) | (static_cast<uint32_t>(__bfloat16_as_ushort(hi)) << 16);
    }
    uint4* dst = reinterpret_cast<uint4*>(out + r * ld_out + b * 16);
    dst[0] = make_uint4(o[0], o[1], o[2], o[3]);
    dst[1] = make_uint4(o[4], o[5], o[6], o[7]);
  }
}

}  // namespace nvfp4
