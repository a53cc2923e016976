// Entry points of the W8A8 INT8 path: the per-row quantiser and the fused linear on the INT8 form of the
// one-CTA GEMM kernel.  Included at the end of nvfp4_api.cu, whose helpers (argument checks, per-device
// state, TMA store maps, tile choice) they use.
#pragma once

#include "gemm.cuh"
#include "int8.cuh"

namespace {

int64_t ld_q_of(const nvfp4_int8_tensor* t) { return t->ld ? t->ld : t->cols; }

nvfp4_status check_int8_tensor(const nvfp4_int8_tensor* t) {
  if (!t || !t->q || !t->scale || t->rows < 0 || t->cols <= 0) return NVFP4_ERR_INVALID_ARG;
  if (ld_q_of(t) < t->cols) return NVFP4_ERR_INVALID_ARG;
  if (!aligned16(t->q) || ld_q_of(t) % 16 || !aligned4(t->scale)) return NVFP4_ERR_MISALIGNED;
  return NVFP4_OK;
}

// TMA map of an INT8 GEMM operand: 128-byte (128-element) boxes of 128 rows, 128-byte swizzle, the
// same shared-memory layout the FP4 kernel's code tiles have.
nvfp4_status make_i8_map(CUtensorMap* map, const nvfp4_int8_tensor* t) {
  auto encode = tensor_map_encoder();
  if (!encode) return NVFP4_ERR_CUDA;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(t->cols), static_cast<cuuint64_t>(t->rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(ld_q_of(t))};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(kStageRowBytes), 128};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = encode(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, t->q, dims, strides, box, estr,
                      CU_TENSOR_MAP_INTERLEAVE_NONE,
                      kStageRowBytes == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B,
                      CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? NVFP4_OK : NVFP4_ERR_CUDA;
}

template <int BN, int KIND>
nvfp4_status launch_gemm_i8(DeviceState* st, const CUtensorMap& ma, const CUtensorMap& mb, const OutMaps& om,
                            const GemmArgs& args, cudaStream_t stream) {
  using C = GemmCfg<BN, true>;
  auto kernel = nvfp4_gemm_kernel<BN, KIND, true>;
  {
    std::lock_guard<std::mutex> lock(g_mutex);
    bool& attr = st->smem_attr_set_i8[BN == 256 ? 1 : 0][KIND];
    if (!attr) {
      if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES) != cudaSuccess)
        return NVFP4_ERR_CUDA;
      attr = true;
    }
  }
  const int grid = args.num_units < st->sm_count ? args.num_units : st->sm_count;
  kernel<<<grid, C::THREADS, C::SMEM_BYTES, stream>>>(ma, mb, om, args);
  return launch_status();
}

}  // namespace

extern "C" {

nvfp4_status nvfp4_int8_quantize(const void* x, int64_t rows, int64_t cols, int64_t ldx, const float* col_mult,
                                 const nvfp4_int8_tensor* out, nvfp4_stream_t stream) {
  if (!x || !out || rows < 0 || cols <= 0 || ldx < cols) return NVFP4_ERR_INVALID_ARG;
  if (nvfp4_status e = check_int8_tensor(out)) return e;
  if (out->rows != rows || out->cols != cols) return NVFP4_ERR_INVALID_ARG;
  if (cols % 16) return NVFP4_ERR_UNSUPPORTED_SHAPE;
  if (!aligned16(x) || (ldx * 2) % 16 || (col_mult && !aligned16(col_mult))) return NVFP4_ERR_MISALIGNED;
  if (rows == 0) return NVFP4_OK;
  DeviceState* st;
  if (nvfp4_status e = device_state(&st)) return e;
  const bool vec32 = (reinterpret_cast<uintptr_t>(x) & 31u) == 0 && (ldx * 2) % 32 == 0;
  auto k = vec32 ? int8_quantize_kernel<true> : int8_quantize_kernel<false>;
  const int grid = resident_grid(k, 256, rows, 8, st->sm_count);
  k<<<grid, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(static_cast<const __nv_bfloat16*>(x), rows, cols, ldx,
                                                              col_mult, static_cast<int8_t*>(out->q), ld_q_of(out),
                                                              out->scale);
  return launch_status();
}

nvfp4_status nvfp4_int8_linear(const nvfp4_int8_tensor* a, const nvfp4_int8_tensor* w,
                               const nvfp4_epilogue_desc* epi, void* out_bf16, int64_t ld_out,
                               const nvfp4_tensor* out_fp4, nvfp4_stream_t stream) {
  if (!epi) return NVFP4_ERR_INVALID_ARG;
  if (nvfp4_status e = check_int8_tensor(a)) return e;
  if (nvfp4_status e = check_int8_tensor(w)) return e;
  const int64_t M = a->rows, N = w->rows, K = a->cols;
  if (w->cols != K) return NVFP4_ERR_INVALID_ARG;
  if (epi->kind < NVFP4_EPI_BIAS || epi->kind > NVFP4_EPI_RESID_GATE) return NVFP4_ERR_INVALID_ARG;
  if (K % 32 || K > 131072) return NVFP4_ERR_UNSUPPORTED_SHAPE;
  // tile width as in the FP4 linear (the FP4 rule on K is in elements of 64; here K counts bytes); the
  // INT8 epilogue reads a weight scale for every column of a tile, so N stays a multiple of 128
  const int BN = tile_n_for(N, 64, epi->kind);
  if (BN == 0 || N % 128) return NVFP4_ERR_UNSUPPORTED_SHAPE;
  if (M > (int64_t(1) << 30) || N > (int64_t(1) << 30)) return NVFP4_ERR_UNSUPPORTED_SHAPE;
  if (!aligned16(a->scale) || !aligned16(w->scale)) return NVFP4_ERR_MISALIGNED;
  const int64_t n_out = epi->kind == NVFP4_EPI_GATED_SILU ? N / 2 : N;
  if (epi->bias && !aligned16(epi->bias)) return NVFP4_ERR_MISALIGNED;
  if (epi->kind == NVFP4_EPI_QKNORM) {
    if (!epi->gamma_q || !epi->gamma_k || epi->head_dim != 256 || !(epi->eps > 0.0f)) return NVFP4_ERR_INVALID_ARG;
    if (epi->q_col0 % 256 || epi->k_col0 % 256 || epi->qk_cols % 256 || epi->q_col0 < 0 || epi->k_col0 < 0 ||
        epi->qk_cols < 0 || epi->q_col0 + epi->qk_cols > N || epi->k_col0 + epi->qk_cols > N)
      return NVFP4_ERR_UNSUPPORTED_SHAPE;
    if (!aligned16(epi->gamma_q) || !aligned16(epi->gamma_k)) return NVFP4_ERR_MISALIGNED;
  }
  if (epi->kind == NVFP4_EPI_RESID_GATE) {
    if (!epi->residual || !epi->gate || epi->ld_residual < n_out) return NVFP4_ERR_INVALID_ARG;
    if (!aligned16(epi->residual) || (epi->ld_residual * 2) % 16 || !aligned16(epi->gate)) return NVFP4_ERR_MISALIGNED;
  }
  if (epi->out_amax && !aligned4(epi->out_amax)) return NVFP4_ERR_MISALIGNED;
  if (epi->out_nvfp4) {
    if (nvfp4_status e = check_tensor(out_fp4, true, 16)) return e;
    if (out_fp4->rows != M || out_fp4->cols != n_out) return NVFP4_ERR_INVALID_ARG;
  } else if (!out_bf16) {
    return NVFP4_ERR_INVALID_ARG;
  }
  if (out_bf16) {
    if (ld_out < n_out) return NVFP4_ERR_INVALID_ARG;
    if (!aligned16(out_bf16) || (ld_out * 2) % 16) return NVFP4_ERR_MISALIGNED;
  }
  if (M == 0) return NVFP4_OK;
  DeviceState* st;
  if (nvfp4_status e = device_state(&st)) return e;

  CUtensorMap ma, mb;
  if (nvfp4_status e = make_i8_map(&ma, a)) return e;
  if (nvfp4_status e = make_i8_map(&mb, w)) return e;
  OutMaps om;
  if (nvfp4_status e = make_store_maps(&om, out_bf16, ld_out, epi->out_nvfp4 ? out_fp4 : nullptr, M, n_out, 16))
    return e;

  GemmArgs g{};
  g.M = static_cast<int32_t>(M);
  g.N = static_cast<int32_t>(N);
  g.K = static_cast<int32_t>(K);
  g.n_out = static_cast<int32_t>(n_out);
  g.num_m_blocks = static_cast<int32_t>((M + 127) / 128);
  g.num_n_blocks = static_cast<int32_t>(epi->kind == NVFP4_EPI_GATED_SILU ? (N / 2) / 128 : N / BN);
  g.num_tiles = g.num_m_blocks * g.num_n_blocks;
  g.num_m_pairs = static_cast<int32_t>((M + 255) / 256);
  g.k_steps = static_cast<int32_t>(K / 32);  // 32-byte MMA steps
  g.row_scale = a->scale;
  g.col_scale = w->scale;
  g.bias = static_cast<const __nv_bfloat16*>(epi->bias);
  g.gamma_q = static_cast<const __nv_bfloat16*>(epi->gamma_q);
  g.gamma_k = static_cast<const __nv_bfloat16*>(epi->gamma_k);
  g.eps = epi->eps;
  g.q_col0 = static_cast<int32_t>(epi->q_col0);
  g.k_col0 = static_cast<int32_t>(epi->k_col0);
  g.qk_cols = static_cast<int32_t>(epi->qk_cols);
  g.residual = static_cast<const __nv_bfloat16*>(epi->residual);
  g.ld_res = epi->ld_residual;
  g.gate = epi->gate;
  g.out = static_cast<__nv_bfloat16*>(out_bf16);
  g.ld_out = ld_out;
  if (epi->out_nvfp4) {
    g.q_codes = static_cast<uint8_t*>(out_fp4->codes);
    g.ld_q_codes = ld_codes_of(out_fp4);
    g.q_scales = static_cast<uint8_t*>(out_fp4->scales);
    g.q_g = out_fp4->tensor_scale;
    g.q_k_atoms = static_cast<int32_t>(k_atoms_of(n_out));
  }
  g.out_amax_bits = reinterpret_cast<unsigned int*>(epi->out_amax);
  g.error_word = st->error_word;
  g.timeout_ns = wait_timeout_ns();
  g.n_fastest = N <= M ? 1 : 0;  // keep the smaller operand resident in L2 (as nvfp4_linear does)
  g.splits = 1;
  g.num_units = g.num_tiles;

  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  switch (epi->kind) {
    case NVFP4_EPI_BIAS:
      return BN == 256 ? launch_gemm_i8<256, kEpiBias>(st, ma, mb, om, g, s)
                       : launch_gemm_i8<128, kEpiBias>(st, ma, mb, om, g, s);
    case NVFP4_EPI_RESID_GATE:
      return BN == 256 ? launch_gemm_i8<256, kEpiResidGate>(st, ma, mb, om, g, s)
                       : launch_gemm_i8<128, kEpiResidGate>(st, ma, mb, om, g, s);
    case NVFP4_EPI_QKNORM: return launch_gemm_i8<256, kEpiQkNorm>(st, ma, mb, om, g, s);
    case NVFP4_EPI_GATED_SILU: return launch_gemm_i8<256, kEpiGatedSilu>(st, ma, mb, om, g, s);
  }
  return NVFP4_ERR_INVALID_ARG;
}

}  // extern "C"
