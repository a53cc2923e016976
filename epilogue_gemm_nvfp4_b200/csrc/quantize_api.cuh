// Entry points of the bandwidth-bound NVFP4 ops: amax, quantise (static or dynamic tensor scale), fake
// quantise, the adaLN-prologue quantiser and dequantise.  Included at the end of nvfp4_api.cu, whose
// helpers (argument checks, per-device and per-stream state, grid sizing) they use.
#pragma once

#include "adaln.cuh"
#include "quantize.cuh"

extern "C" {

nvfp4_status nvfp4_amax(const void* x, int64_t rows, int64_t cols, int64_t ldx, float* amax, nvfp4_stream_t stream) {
  if (!x || !amax || rows < 0 || cols <= 0 || ldx < cols) return NVFP4_ERR_INVALID_ARG;
  if (cols % 8) return NVFP4_ERR_UNSUPPORTED_SHAPE;
  if (!aligned16(x) || (ldx * 2) % 16 || !aligned4(amax)) return NVFP4_ERR_MISALIGNED;
  DeviceState* st;
  if (nvfp4_status e = device_state(&st)) return e;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(amax, 0, sizeof(float), s) != cudaSuccess) return NVFP4_ERR_CUDA;
  if (rows == 0) return NVFP4_OK;
  const int grid = resident_grid(amax_kernel, 256, rows * cols / 8, 256 * 4, st->sm_count);
  amax_kernel<<<grid, 256, 0, s>>>(static_cast<const __nv_bfloat16*>(x), rows, cols, ldx,
                                   reinterpret_cast<unsigned int*>(amax));
  return launch_status();
}

nvfp4_status nvfp4_quantize(const void* x, int64_t rows, int64_t cols, int64_t ldx, int32_t compute_scale,
                            const nvfp4_tensor* out, nvfp4_stream_t stream) {
  if (!x || !out || rows < 0 || cols <= 0 || ldx < cols) return NVFP4_ERR_INVALID_ARG;
  if (nvfp4_status e = check_tensor(out, true, 8)) return e;
  if (out->rows != rows || out->cols != cols) return NVFP4_ERR_INVALID_ARG;
  if (!aligned16(x) || (ldx * 2) % 16) return NVFP4_ERR_MISALIGNED;
  DeviceState* st;
  if (nvfp4_status e = device_state(&st)) return e;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const auto* xb = static_cast<const __nv_bfloat16*>(x);
  auto* codes = static_cast<uint8_t*>(out->codes);
  auto* scales = static_cast<uint8_t*>(out->scales);
  const int64_t ld = ld_codes_of(out), ka = k_atoms_of(cols);
  const int64_t steps = (cols / 16 + 31) / 32;
  const int64_t tasks = rows * ((steps + kQuantStepsPerTask - 1) / kQuantStepsPerTask) + 1;
  // one 256-bit load per block when every block starts on a 32-byte boundary
  const bool vec32 = (reinterpret_cast<uintptr_t>(x) & 31u) == 0 && (ldx * 2) % 32 == 0;
  // dynamic scale: the amax pass (which also writes g) streams the tensor front to back, then the
  // quantiser walks it back to front so that its first tasks re-read from L2 what that pass left there
  auto qk = compute_scale ? (vec32 ? quantize_kernel<true, true> : quantize_kernel<true, false>)
                          : (vec32 ? quantize_kernel<false, true> : quantize_kernel<false, false>);
  const int qgrid = resident_grid(qk, 256, tasks, 8, st->sm_count);
  if (compute_scale) {
    unsigned int* state = nullptr;
    if (nvfp4_status e = amax_state_for(s, &state)) return e;
    const int agrid = resident_grid(amax_scale_kernel, 256, rows * cols / 8, 256 * 4, st->sm_count);
    amax_scale_kernel<<<agrid, 256, 0, s>>>(xb, rows, cols, ldx, state, out->tensor_scale);
  }
  qk<<<qgrid, 256, 0, s>>>(xb, rows, cols, ldx, out->tensor_scale, codes, ld, scales, ka);
  return launch_status();
}

nvfp4_status nvfp4_fake_quantize(const void* x, int64_t rows, int64_t cols, int64_t ldx, int32_t compute_scale,
                                 float* tensor_scale, void* y, int64_t ldy, nvfp4_stream_t stream) {
  if (!x || !y || !tensor_scale || rows < 0 || cols <= 0 || ldx < cols || ldy < cols) return NVFP4_ERR_INVALID_ARG;
  if (cols % 16) return NVFP4_ERR_UNSUPPORTED_SHAPE;
  if (!aligned16(x) || (ldx * 2) % 16 || !aligned16(y) || (ldy * 2) % 16 || !aligned4(tensor_scale))
    return NVFP4_ERR_MISALIGNED;
  DeviceState* st;
  if (nvfp4_status e = device_state(&st)) return e;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const auto* xb = static_cast<const __nv_bfloat16*>(x);
  const int64_t steps = (cols / 16 + 31) / 32;
  const int64_t tasks = rows * ((steps + kQuantStepsPerTask - 1) / kQuantStepsPerTask) + 1;
  const bool vec32 = (reinterpret_cast<uintptr_t>(x) & 31u) == 0 && (ldx * 2) % 32 == 0;
  // as in nvfp4_quantize: after the amax pass, walk the tensor back to front
  auto fk = compute_scale ? (vec32 ? fake_quantize_kernel<true, true> : fake_quantize_kernel<true, false>)
                          : (vec32 ? fake_quantize_kernel<false, true> : fake_quantize_kernel<false, false>);
  if (compute_scale) {
    unsigned int* state = nullptr;
    if (nvfp4_status e = amax_state_for(s, &state)) return e;
    const int agrid = resident_grid(amax_scale_kernel, 256, rows * cols / 8, 256 * 4, st->sm_count);
    amax_scale_kernel<<<agrid, 256, 0, s>>>(xb, rows, cols, ldx, state, tensor_scale);
  }
  if (rows > 0) {
    const int grid = resident_grid(fk, 256, tasks, 8, st->sm_count);
    fk<<<grid, 256, 0, s>>>(xb, rows, cols, ldx, tensor_scale, static_cast<__nv_bfloat16*>(y), ldy);
  }
  return launch_status();
}

}  // extern "C"

namespace {

using AdalnKernel = void (*)(const AdalnArgs);

AdalnKernel adaln_kernel_for(bool amax_pass, bool reverse, bool vec32, bool table) {
#define NVFP4_ADALN_PICK(T)                                                                                   \
  if (amax_pass) return vec32 ? adaln_quantize_kernel<true, false, true, T> : adaln_quantize_kernel<true, false, false, T>; \
  if (reverse) return vec32 ? adaln_quantize_kernel<false, true, true, T> : adaln_quantize_kernel<false, true, false, T>;    \
  return vec32 ? adaln_quantize_kernel<false, false, true, T> : adaln_quantize_kernel<false, false, false, T>;
  if (table) {
    NVFP4_ADALN_PICK(true)
  }
  NVFP4_ADALN_PICK(false)
#undef NVFP4_ADALN_PICK
}

// One resident wave of 256-thread CTAs (one row per warp at a time), at most one warp per row.
int adaln_grid(AdalnKernel k, size_t smem, int64_t rows, int sm_count) {
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k, 256, smem) != cudaSuccess || per_sm < 1) per_sm = 1;
  int64_t g = (rows + 7) / 8;
  const int64_t cap = static_cast<int64_t>(sm_count) * per_sm;
  if (g > cap) g = cap;
  if (g < 1) g = 1;
  return static_cast<int>(g);
}

}  // namespace

extern "C" {

nvfp4_status nvfp4_adaln_quantize(const void* x, int64_t rows, int64_t cols, int64_t ldx, const nvfp4_adaln_desc* ada,
                                  int32_t compute_scale, const nvfp4_tensor* out, nvfp4_stream_t stream) {
  if (!x || !ada || !out || rows < 0 || cols <= 0 || ldx < cols) return NVFP4_ERR_INVALID_ARG;
  if (!(ada->eps > 0.0f) || ada->eps > 3.0e38f || ada->rows_per_sample < 0) return NVFP4_ERR_INVALID_ARG;
  const bool per_sample = ada->rows_per_sample > 0 && ada->rows_per_sample < rows;
  if (per_sample && (ada->shift || ada->scale) && ada->ld_mod < cols) return NVFP4_ERR_INVALID_ARG;
  if (ada->u_out && ada->ld_u < cols) return NVFP4_ERR_INVALID_ARG;
  if (nvfp4_status e = check_tensor(out, true, 8)) return e;
  if (out->rows != rows || out->cols != cols) return NVFP4_ERR_INVALID_ARG;
  if (!aligned16(x) || (ldx * 2) % 16) return NVFP4_ERR_MISALIGNED;
  if ((ada->shift && !aligned16(ada->shift)) || (ada->scale && !aligned16(ada->scale)) ||
      (per_sample && (ada->ld_mod * 2) % 16) || (ada->rstd && !aligned4(ada->rstd)) ||
      (ada->u_out && (!aligned16(ada->u_out) || (ada->ld_u * 2) % 16)))
    return NVFP4_ERR_MISALIGNED;
  DeviceState* st;
  if (nvfp4_status e = device_state(&st)) return e;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  AdalnArgs a{};
  a.x = static_cast<const __nv_bfloat16*>(x);
  a.rows = rows;
  a.cols = cols;
  a.ldx = ldx;
  a.shift = static_cast<const __nv_bfloat16*>(ada->shift);
  a.scale = static_cast<const __nv_bfloat16*>(ada->scale);
  a.ld_mod = ada->ld_mod;
  a.rows_per_sample = per_sample ? ada->rows_per_sample : 0;
  a.eps = ada->eps;
  a.g_src = out->tensor_scale;
  a.codes = static_cast<uint8_t*>(out->codes);
  a.ld_codes = ld_codes_of(out);
  a.scales = static_cast<uint8_t*>(out->scales);
  a.k_atoms = k_atoms_of(cols);
  a.rstd = ada->rstd;
  a.u = static_cast<__nv_bfloat16*>(ada->u_out);
  a.ld_u = ada->ld_u;
  a.tensor_scale = out->tensor_scale;
  const bool vec32 = (reinterpret_cast<uintptr_t>(x) & 31u) == 0 && (ldx * 2) % 32 == 0;
  // one sample and rows of at most 5632 elements: the modulation comes from a shared-memory table
  const int64_t steps = (cols / 16 + 31) / 32;
  const bool table = a.rows_per_sample == 0 && steps <= kAdalnTableMaxSteps;
  const size_t smem = table ? static_cast<size_t>(steps) * 8 * 32 * sizeof(float4) : 0;
  // dynamic scale: the amax pass walks the rows front to back, the quantise pass back to front
  if (compute_scale) {
    if (nvfp4_status e = amax_state_for(s, &a.state)) return e;
    const AdalnKernel ak = adaln_kernel_for(true, false, vec32, table);
    ak<<<adaln_grid(ak, smem, rows, st->sm_count), 256, smem, s>>>(a);
  }
  const AdalnKernel qk = adaln_kernel_for(false, compute_scale != 0, vec32, table);
  qk<<<adaln_grid(qk, smem, rows + 1, st->sm_count), 256, smem, s>>>(a);
  return launch_status();
}

nvfp4_status nvfp4_dequantize(const nvfp4_tensor* t, void* out_bf16, int64_t ld_out, nvfp4_stream_t stream) {
  if (!out_bf16) return NVFP4_ERR_INVALID_ARG;
  if (nvfp4_status e = check_tensor(t, true, 8)) return e;
  if (ld_out < t->cols) return NVFP4_ERR_INVALID_ARG;
  if (!aligned16(out_bf16) || (ld_out * 2) % 16) return NVFP4_ERR_MISALIGNED;
  if (t->rows == 0) return NVFP4_OK;
  DeviceState* st;
  if (nvfp4_status e = device_state(&st)) return e;
  const int grid = resident_grid(dequantize_kernel, 256, t->rows * (t->cols / 16), 256, st->sm_count);
  dequantize_kernel<<<grid, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      static_cast<const uint8_t*>(t->codes), ld_codes_of(t), static_cast<const uint8_t*>(t->scales), t->tensor_scale,
      t->rows, t->cols, k_atoms_of(t->cols), static_cast<__nv_bfloat16*>(out_bf16), ld_out);
  return launch_status();
}

}  // extern "C"
