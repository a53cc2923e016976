/*
 * nvfp4.h - C ABI of libnvfp4: the NVFP4 quantised linear layer of a flow-matching diffusion
 * transformer, with the small op that follows each product fused into the GEMM epilogue.
 *
 * What is computed comes from "Serving sub-second Ideogram v4 without quality loss" (fal, via
 * tldrocket.com): the DiT's matrix products run in NVFP4, the 4-bit floating-point format that
 * Blackwell tensor cores execute natively, and the RMSNorm over 256-wide attention heads or the
 * gated SiLU that follows a product runs inside the same kernel instead of after a round trip of
 * the product through memory.  The text-conditioning projection (53248 -> 4608 with a bias) and
 * the rule that a linear must treat its rows independently come from "Faster Ideogram 4 with Less
 * Prompt Compute" (sections "Most of the Tensor Was Zero" and "The NF4 Exactness Problem").
 *
 * Encoding (the pages do not spell it out; this is the reading the library implements):
 *   - element: E2M1 code in 4 bits, sign in bit 3, magnitudes {0,.5,1,1.5,2,3,4,6};
 *   - block:   one unsigned E4M3 scale byte per 16 consecutive elements of a row;
 *   - tensor:  one fp32 decode scale g; value = e2m1(code) * e4m3(scale) * g.
 *   Quantisation of a block: r = amax_b / g; s = E4M3(r / 6); d = s * g; code_i = E2M1(x_i * (1/d)),
 *   each step one binary32 operation rounded to nearest even, E4M3 and E2M1 rounding to nearest even
 *   and saturating (448, 6).  A block with d == 0 gets codes 0.  The tensor scale computed by
 *   nvfp4_quantize is g = amax / 2688 (2688 = 6 * 448), or 1 when the tensor is all zero.
 *
 * Conventions for every entry point:
 *   - All pointers inside the structs and all data pointers are DEVICE pointers, owned by the caller.
 *     The library allocates no memory the caller sees; its only allocation is the split-K scratch of
 *     nvfp4_linear for K >= 32768 (see nvfp4_linear_split_k).
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL = the legacy default stream).  Host-side
 *     argument checks run before anything is launched; when one fails nothing is launched and the
 *     status says why.  Nothing throws, prints or traps.
 *   - NVFP4_ERR_CUDA means a CUDA runtime call failed (the launch, or the device has no sm_100a).
 *   - Device-side failures (a pipeline wait that ran out of time) are recorded in a sticky per-device
 *     word and reported by nvfp4_get_device_error().
 */
#ifndef NVFP4_H_
#define NVFP4_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define NVFP4_API __attribute__((visibility("default")))
#else
#define NVFP4_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* nvfp4_stream_t; /* same type as cudaStream_t */

typedef enum {
  NVFP4_OK = 0,
  NVFP4_ERR_INVALID_ARG = 1,       /* NULL where a pointer is required, negative size, bad enum      */
  NVFP4_ERR_UNSUPPORTED_SHAPE = 2, /* a size rule below is not met                                   */
  NVFP4_ERR_MISALIGNED = 3,        /* a pointer or leading dimension is not 16-byte aligned           */
  NVFP4_ERR_CUDA = 4,              /* a CUDA runtime call failed                                      */
  NVFP4_ERR_DEVICE_TIMEOUT = 5,    /* a kernel's pipeline wait ran out of time and the kernel gave up */
  NVFP4_ERR_SCRATCH_LIMIT = 6      /* nvfp4_linear_noalloc: the problem needs more split-K scratch than
                                      its fixed buffer holds                                          */
} nvfp4_status;

/*
 * An NVFP4 tensor of `rows` x `cols` logical elements (cols = the reduction dimension K for GEMM
 * operands).
 *   codes:        uint8, row r starts at codes + r * ld_codes; element k of the row is the low nibble
 *                 of byte k/2 when k is even, the high nibble when k is odd.  ld_codes >= cols/2
 *                 (0 means cols/2); a multiple of 8 for nvfp4_quantize / nvfp4_dequantize and of 16
 *                 for the operands and the NVFP4 output of nvfp4_linear.
 *   scales:       uint8 E4M3 block scales in the tensor-core scale layout, nvfp4_scale_bytes(rows, cols)
 *                 bytes: 512-byte atoms of 128 rows x 4 blocks, atoms ordered along K first, then along
 *                 rows; inside an atom row r, block c is at (r%32)*16 + ((r/32)%4)*4 + c%4 (see
 *                 nvfp4_scale_offset).  Rows are padded to a multiple of 128 and blocks per row to a
 *                 multiple of 4; nvfp4_quantize writes 0 into the padding.
 *   tensor_scale: one fp32, the decode scale g.
 */
typedef struct {
  void* codes;
  void* scales;
  float* tensor_scale;
  int64_t rows;
  int64_t cols;
  int64_t ld_codes;
} nvfp4_tensor;

typedef enum {
  NVFP4_EPI_BIAS = 0,       /* y = acc + bias                                                      */
  NVFP4_EPI_QKNORM = 1,     /* y = acc + bias; RMSNorm of every 256-wide head in the q and k ranges */
  NVFP4_EPI_GATED_SILU = 2, /* y = acc + bias; out = silu(y[:, :N/2]) * y[:, N/2:]                  */
  NVFP4_EPI_RESID_GATE = 3  /* out = residual + gate[n] * (acc + bias)                              */
} nvfp4_epilogue_kind;

/*
 * The op fused after the product acc[m,n] = sum_k a[m,k] * w[n,k] (dequantised operands, fp32
 * accumulation).  N is w->rows.  The output has N columns, or N/2 for NVFP4_EPI_GATED_SILU.
 *   bias:          bf16 [N] or NULL (no bias).  Added before any norm or activation.
 *   QKNORM:        gamma_q, gamma_k bf16 [head_dim]; head_dim must be 256; eps > 0.  Columns
 *                  [q_col0, q_col0 + qk_cols) are normalised per head with gamma_q, columns
 *                  [k_col0, k_col0 + qk_cols) with gamma_k: y_h / sqrt(mean(y_h^2) + eps) * gamma.
 *                  q_col0, k_col0 and qk_cols are multiples of 256; other columns get bias only.
 *   GATED_SILU:    rows [0, N/2) of w give a, rows [N/2, N) give b; out = a / (1 + exp(-a)) * b.
 *   RESID_GATE:    residual bf16 [M, ld_residual] (row stride in elements), gate fp32 [N].
 *   out_nvfp4:     1 = also re-quantise the bf16-rounded output to NVFP4 into `out_fp4` with the
 *                  caller's static decode scale already stored in out_fp4->tensor_scale (the rule of
 *                  nvfp4_quantize, so the codes equal nvfp4_quantize of the bf16 output bit for bit).
 *   out_amax:      device fp32, or NULL.  When given, the kernel raises *out_amax to the largest |y| of
 *                  the bf16-rounded output (the values out_nvfp4 quantises; rows < M only), as an
 *                  atomic max on the bit pattern, so *out_amax must hold a non-negative float (0 to
 *                  start, or a running max over calls).  amax / 2688 is then the decode scale that
 *                  nvfp4_quantize would compute for this output: a delayed scale for the next call's
 *                  out_fp4, available without a separate pass over the output.
 */
typedef struct {
  int32_t kind;
  const void* bias;
  const void* gamma_q;
  const void* gamma_k;
  float eps;
  int32_t head_dim;
  int64_t q_col0;
  int64_t k_col0;
  int64_t qk_cols;
  const void* residual;
  int64_t ld_residual;
  const float* gate;
  int32_t out_nvfp4;
  float* out_amax;
} nvfp4_epilogue_desc;

/*
 * Quantise a bf16 matrix x [rows, cols] (row stride ldx elements) to NVFP4 into `out`
 * (out->rows == rows, out->cols == cols).
 * Passage: "Serving sub-second Ideogram v4 without quality loss", the paragraph on the 6x speed-up and
 * NVFP4: the DiT's products run on 4-bit floats that Blackwell's tensor cores take natively, so every
 * activation entering a product is first put in that format (the encoding above is the reading of it).
 *   compute_scale = 1: compute g = amax(|x|) / 2688 (1 when x is all zeros or empty) on the device and
 *                      store it in *out->tensor_scale: two stream-ordered kernels, an amax pass whose
 *                      last CTA writes g, then the quantise pass.  The first such call on a stream
 *                      allocates 256 bytes of per-stream reduction state, so it must not be the first
 *                      call made under CUDA graph capture.
 *   compute_scale = 0: use the g already stored in *out->tensor_scale (a calibrated static scale).
 * Rules: cols % 16 == 0; x, ldx*2, codes and scales 16-byte aligned; ld_codes a multiple of 8.
 * rows == 0 writes no codes.
 */
NVFP4_API nvfp4_status nvfp4_quantize(const void* x, int64_t rows, int64_t cols, int64_t ldx, int32_t compute_scale,
                            const nvfp4_tensor* out, nvfp4_stream_t stream);

/*
 * The fused NVFP4 linear: out = epilogue(a x w^T) on one GPU.
 * Passages: "Serving sub-second Ideogram v4 without quality loss", the paragraph on kernel fusion (the
 * small ops that follow a product, RMSNorm over 256-wide attention heads that straddle two tile fragments
 * and the gated SiLU, run inside the GEMM instead of after a round trip of its output through memory);
 * "Faster Ideogram 4 with Less Prompt Compute", "Most of the Tensor Was Zero" (the 53248 -> 4608 text
 * projection with a bias, and a linear treats its rows independently) and "The NF4 Exactness Problem"
 * (a kernel chosen by row count changes the bits, so nothing here depends on M).
 *   a:        NVFP4 [M, K] activation.  w: NVFP4 [N, K] weight (nn.Linear layout).
 *   out_bf16: bf16 [M, ld_out] (row stride in elements) or NULL when only out_fp4 is wanted.
 *   out_fp4:  NVFP4 [M, n_out] when epi->out_nvfp4 == 1, else ignored (may be NULL).
 * Rules: K % 64 == 0, K >= 64; N % 16 == 0 (N % 256 == 0 for QKNORM and GATED_SILU); M >= 1 (any);
 * all pointers and ld_out * 2 16-byte aligned; the scale padding of w (rows past N up to a multiple of
 * 128) holds zeros, as nvfp4_quantize writes it.  The per-row arithmetic does not depend on M: row m of
 * the output is bitwise the same whatever rows accompany it.
 * Kernels: 256-wide tiles (N % 256 == 0) run on two-CTA clusters with the paired tensor-core MMA;
 * other tiles on single CTAs.  The environment variable NVFP4_GEMM_PAIR=0, read once per process,
 * keeps every tile on single CTAs; the results are the same bits.  K >= 32768 splits the reduction
 * in two halves summed in a fixed order, using per-stream scratch that the library allocates on
 * first use (nvfp4_linear_noalloc uses a fixed array instead).
 */
NVFP4_API nvfp4_status nvfp4_linear(const nvfp4_tensor* a, const nvfp4_tensor* w, const nvfp4_epilogue_desc* epi,
                          void* out_bf16, int64_t ld_out, const nvfp4_tensor* out_fp4, nvfp4_stream_t stream);

/*
 * nvfp4_linear for callers that cannot allocate device memory.  The paper has no counterpart to this
 * entry point; it exists for how the library is called, not for what it computes.  Some callers must not call cudaMalloc from inside this library: code that
 * runs while a serving runtime or framework owns all device memory through its own pool, code on a
 * latency-critical path where cudaMalloc / cudaFree would synchronise the device, and code that records
 * work for later replay.  This entry point computes exactly what nvfp4_linear computes, with the same
 * arguments and rules, but the split-K scratch of long-K calls (K >= 32768, see nvfp4_linear_split_k)
 * lives in a fixed device array of nvfp4_linear_noalloc_scratch_bytes() bytes (64 MiB) built into the
 * library instead of a buffer it allocates; calls without split-K need no scratch at all.
 *   - It calls no cudaMalloc, cudaFree or allocating routine.  The array is part of the library's
 *     device image: every GPU that loads the library holds it until the process exits.
 *   - The first call on a device looks up the array's device address (cudaGetSymbolAddress) with that
 *     device current; make that first call before any stream capture.
 *   - A call whose scratch would not fit returns NVFP4_ERR_SCRATCH_LIMIT and launches nothing.  The
 *     scratch of a split-K call is 4 bytes per output tile plus 128 KiB per 128 x 256 tile.
 *   - All calls on a device share the one array, which keeps the previous call's contents; each call
 *     clears the part that must start at zero.  Calls that overlap on the GPU (different streams without
 *     ordering between them) race on the array and give wrong results: order them.
 */
NVFP4_API nvfp4_status nvfp4_linear_noalloc(const nvfp4_tensor* a, const nvfp4_tensor* w,
                                            const nvfp4_epilogue_desc* epi, void* out_bf16, int64_t ld_out,
                                            const nvfp4_tensor* out_fp4, nvfp4_stream_t stream);

/* Size in bytes of the fixed split-K scratch array used by nvfp4_linear_noalloc. */
NVFP4_API size_t nvfp4_linear_noalloc_scratch_bytes(void);

/*
 * Fake quantisation (the forward of quantisation-aware training): y = dequantise(quantise(x)) as bf16
 * [rows, ldy], in one pass that keeps no codes.  y equals nvfp4_quantize followed by nvfp4_dequantize
 * with the same scale, bit for bit.
 *   compute_scale = 1: g = amax(|x|) / 2688 (1 for an all-zero or empty x) is computed on the device
 *                      and written to *tensor_scale (the amax pass of nvfp4_quantize, with the same
 *                      per-stream state and the same rule on graph capture).
 *   compute_scale = 0: *tensor_scale holds g.
 * Rules: cols % 16 == 0; x, y, ldx*2 and ldy*2 16-byte aligned; ldy >= cols; tensor_scale 4-byte
 * aligned.  rows == 0 writes nothing to y.
 */
NVFP4_API nvfp4_status nvfp4_fake_quantize(const void* x, int64_t rows, int64_t cols, int64_t ldx,
                                           int32_t compute_scale, float* tensor_scale, void* y, int64_t ldy,
                                           nvfp4_stream_t stream);

/*
 * The adaLN prologue of a DiT block, fused into the quantiser.  RMSNorm is one of the small ops that
 * follow the big products ("Serving sub-second Ideogram v4 without quality loss", paragraph on kernel
 * fusion); adaLN modulates the hidden state with vectors generated at run time ("Quantizing a
 * Dual-Branch Flow-Matching Diffusion Transformer for Consumer GPUs", related-work paragraph on W8A8).
 * For row r of x and its sample b = r / rows_per_sample:
 *   rstd[r] = 1 / sqrt(mean_k x[r,k]^2 + eps)
 *   u[r,k]  = bf16( x[r,k] * rstd[r] * (1 + scale[b,k]) + shift[b,k] )
 * and u is quantised by the rule of nvfp4_quantize, so the codes equal nvfp4_quantize(u) bit for bit.
 *   shift, scale:     bf16 vectors of `cols` elements per sample, sample b at element offset b * ld_mod,
 *                     ceil(rows / rows_per_sample) samples (one when rows_per_sample is 0);
 *                     NULL = no shift / multiplier 1.
 *   ld_mod:           elements between samples (>= cols; read only when rows_per_sample > 0).
 *   rows_per_sample:  rows [b * L, (b + 1) * L) use sample b; 0 (or >= rows) = sample 0 for every row.
 *   eps:              > 0.
 *   rstd:             device fp32 [rows] or NULL: receives rstd[r].
 *   u_out, ld_u:      bf16 [rows, ld_u] or NULL: receives u (the values that were quantised).
 * Arithmetic: the sum of squares is an fp32 sum in a fixed order (it does not depend on `rows`); then
 * rstd = 1 / sqrt(sum / cols + eps), x * rstd and 1 + scale each rounded to fp32, one fused
 * multiply-add with shift, and one rounding to bf16.
 */
typedef struct {
  const void* shift;
  const void* scale;
  int64_t ld_mod;
  int64_t rows_per_sample;
  float eps;
  float* rstd;
  void* u_out;
  int64_t ld_u;
} nvfp4_adaln_desc;

/*
 * Quantise adaLN(x) (see nvfp4_adaln_desc) to NVFP4 into `out` (out->rows == rows, out->cols == cols).
 *   compute_scale = 1: g = amax(|u|) / 2688 (1 for an all-zero or empty u) is computed on the device
 *                      and stored in *out->tensor_scale: two stream-ordered launches of one kernel, an
 *                      amax pass that computes u and reduces its max (its last CTA writes g), then the
 *                      quantise pass.  The per-stream state and the rule on graph capture are those of
 *                      nvfp4_quantize.
 *   compute_scale = 0: the g already stored in *out->tensor_scale is used; one launch.
 * Rules: cols % 16 == 0; x, ldx*2, shift, scale, ld_mod*2 (when read), u_out, ld_u*2, codes and scales
 * 16-byte aligned; rstd 4-byte aligned; ld_codes a multiple of 8.  Each pass walks a row twice (sum of
 * squares, then modulate and quantise); the second walk reads it from L2, so x crosses HBM once per pass.
 */
NVFP4_API nvfp4_status nvfp4_adaln_quantize(const void* x, int64_t rows, int64_t cols, int64_t ldx,
                                            const nvfp4_adaln_desc* ada, int32_t compute_scale,
                                            const nvfp4_tensor* out, nvfp4_stream_t stream);

/*
 * W8A8 INT8 operands ("Quantizing a Dual-Branch Flow-Matching Diffusion Transformer for Consumer GPUs",
 * method section: per-output-row INT8 weights, per-token dynamic INT8 activations, SmoothQuant channel
 * migration).  A `rows` x `cols` tensor:
 *   q:      int8 [rows, ld] (row stride ld bytes; 0 means cols), values in [-127, 127];
 *   scale:  fp32 [rows], the decode scale of each row: value = q * scale[row].
 */
typedef struct {
  void* q;
  float* scale;
  int64_t rows;
  int64_t cols;
  int64_t ld;
} nvfp4_int8_tensor;

/*
 * Quantise bf16 x [rows, cols] (row stride ldx elements) to per-row INT8 into `out` (out->rows == rows,
 * out->cols == cols).  For each row, each step one binary32 operation rounded to nearest even:
 *   x'[k] = x[k] * col_mult[k]   (col_mult = NULL: x' = x)
 *   s     = max_k |x'| / 127     (1 for an all-zero row), stored in out->scale[row]
 *   q[k]  = clamp(RNE(x'[k] * (127 / max_k |x'|)), -127, 127)   (0 for an all-zero row)
 * col_mult carries the SmoothQuant migration: 1 / lambda for activations, lambda for the weight (whose
 * rows are the output channels).  Rules: cols % 16 == 0; x, ldx * 2, col_mult, out->q and out->ld 16-byte
 * aligned; out->scale 4-byte aligned.
 */
NVFP4_API nvfp4_status nvfp4_int8_quantize(const void* x, int64_t rows, int64_t cols, int64_t ldx,
                                           const float* col_mult, const nvfp4_int8_tensor* out,
                                           nvfp4_stream_t stream);

/*
 * The fused W8A8 linear: out = epilogue(y) with y[m,n] = (sum_k a.q[m,k] * w.q[n,k]) * a.scale[m] *
 * w.scale[n], the products summed exactly in s32 on the tensor cores (tcgen05.mma.kind::i8), then
 * converted to fp32 and scaled.  `epi`, out_bf16, ld_out and out_fp4 mean what they mean for
 * nvfp4_linear, every epilogue kind included.  Rules: K % 32 == 0; N % 128 == 0 (N % 256 == 0 for QKNORM
 * and GATED_SILU); a.q, w.q and their ld 16-byte aligned; a.scale and w.scale 16-byte aligned.  There
 * is no split of K: the s32 sums of K <= 131072 cannot overflow.
 */
NVFP4_API nvfp4_status nvfp4_int8_linear(const nvfp4_int8_tensor* a, const nvfp4_int8_tensor* w,
                                         const nvfp4_epilogue_desc* epi, void* out_bf16, int64_t ld_out,
                                         const nvfp4_tensor* out_fp4, nvfp4_stream_t stream);

/* Dequantise t to bf16 [t->rows, ld_out]: value = e2m1(code) * (e4m3(scale) * g), each product in fp32
 * rounded to nearest even, then rounded to bf16.  Rules as for nvfp4_quantize.
 * Passage: the decode of the 4-bit format of "Serving sub-second Ideogram v4 without quality loss"
 * (paragraph on NVFP4), in the reading above: a value is its E2M1 element times its block's E4M3 scale
 * times the tensor's fp32 scale. */
NVFP4_API nvfp4_status nvfp4_dequantize(const nvfp4_tensor* t, void* out_bf16, int64_t ld_out, nvfp4_stream_t stream);

/* max |x| over a bf16 matrix into *amax (device fp32), overwriting it.  The first pass of
 * nvfp4_quantize(compute_scale = 1), exported so it can be timed and used on its own. */
NVFP4_API nvfp4_status nvfp4_amax(const void* x, int64_t rows, int64_t cols, int64_t ldx, float* amax,
                        nvfp4_stream_t stream);

/* Size in bytes of the padded block-scale buffer of a rows x cols NVFP4 tensor. */
NVFP4_API size_t nvfp4_scale_bytes(int64_t rows, int64_t cols);

/* Byte offset of the scale of row r, 16-element block kb, in a tensor with `cols` columns
 * (host helper). */
NVFP4_API int64_t nvfp4_scale_offset(int64_t r, int64_t kb, int64_t cols);

/* Wait for `stream`, then return and clear the sticky device-side error of the current device
 * (NVFP4_OK when none). */
NVFP4_API nvfp4_status nvfp4_get_device_error(nvfp4_stream_t stream);

/* Column tile width the GEMM uses for a weight of N rows and K columns and an epilogue kind; it
 * depends on (N, K, kind) only, never on M.  0 when the shape is unsupported. */
NVFP4_API int32_t nvfp4_linear_tile_n(int64_t N, int64_t K, int32_t kind);

/* Number of K splits the GEMM uses for a weight of N rows and K columns and an epilogue kind: 2 when
 * K >= 32768 (except the head-norm epilogue), else 1; it depends on (N, K, kind) only, never on M.
 * A split GEMM keeps per-stream scratch in device memory that the library allocates on first use
 * (and regrows when a larger problem needs more); make the first such call on a stream outside
 * stream capture.  0 when the shape is unsupported. */
NVFP4_API int32_t nvfp4_linear_split_k(int64_t N, int64_t K, int32_t kind);

/* Static string naming a status code. */
NVFP4_API const char* nvfp4_status_string(nvfp4_status status);

/* Library version, major * 10000 + minor * 100 + patch. */
NVFP4_API int32_t nvfp4_version(void);

#ifdef __cplusplus
}
#endif

#endif /* NVFP4_H_ */
