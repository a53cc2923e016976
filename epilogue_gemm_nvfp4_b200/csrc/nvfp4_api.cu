// Host side of libnvfp4: argument checks, TMA descriptors, tile configuration and launches.
// Device state the library owns: one sticky error word per device (a module-scope __device__
// variable) and the per-stream split-K scratch of long-K GEMMs.
#include <cudaTypedefs.h>

#include <atomic>
#include <cstdlib>
#include <cstring>
#include <map>
#include <mutex>
#include <utility>

#include "nvfp4.h"
#include "gemm.cuh"
#include "gemm_pair.cuh"
#include "ptx.cuh"
#include "quantize.cuh"

using namespace nvfp4;

namespace {

__device__ unsigned int g_device_error;

constexpr int kMaxDevices = 64;

struct DeviceState {
  bool ready = false;
  int sm_count = 0;
  unsigned int* error_word = nullptr;
  bool smem_attr_set[2][4] = {};
  bool smem_attr_set_i8[2][4] = {};  // the INT8 form of the one-CTA kernel
  int pair_clusters[2][4] = {};  // resident CTA pairs per (split-K, epilogue kind), 0 until first use
};

std::mutex g_mutex;
DeviceState g_devices[kMaxDevices];

// Fixed split-K scratch for nvfp4_linear_noalloc: a file-scope device array, so that entry point
// never allocates.  Every device that loads the library holds it until the process exits.
constexpr size_t kNoAllocScratchBytes = size_t(64) << 20;
static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];
void* g_noalloc_scratch_addr[kMaxDevices] = {};

// Device address of g_noalloc_scratch on the current device, looked up once per device.  In host
// code the array's name is only a host-side handle, so kernels must be given this address.
nvfp4_status noalloc_scratch(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return NVFP4_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mutex);
  if (g_noalloc_scratch_addr[dev] == nullptr) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || ptr == nullptr) return NVFP4_ERR_CUDA;
    g_noalloc_scratch_addr[dev] = ptr;
  }
  *out = g_noalloc_scratch_addr[dev];
  return NVFP4_OK;
}

// Split-K scratch, one buffer per (device, stream) so that calls on different streams never share
// it.  Grown on demand; growing frees the old buffer (cudaFree waits for the device).
struct Scratch {
  void* ptr = nullptr;
  size_t bytes = 0;
};
std::map<std::pair<int, uintptr_t>, Scratch> g_scratch;

nvfp4_status scratch_for(cudaStream_t s, size_t need, void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return NVFP4_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mutex);
  Scratch& w = g_scratch[{dev, reinterpret_cast<uintptr_t>(s)}];
  if (w.bytes < need) {
    if (w.ptr != nullptr && cudaFree(w.ptr) != cudaSuccess) return NVFP4_ERR_CUDA;
    w.ptr = nullptr;
    w.bytes = 0;
    const size_t sz = (need + (size_t(16) << 20) - 1) & ~((size_t(16) << 20) - 1);
    if (cudaMalloc(&w.ptr, sz) != cudaSuccess) return NVFP4_ERR_CUDA;
    w.bytes = sz;
  }
  *out = w.ptr;
  return NVFP4_OK;
}

// Per-(device, stream) state of the dynamic-scale quantiser's amax reduction: {amax bits, CTAs done},
// zero between calls (each call's last CTA clears it).  Allocated and cleared on the stream's first
// dynamic-scale call, which therefore must not run under graph capture.
std::map<std::pair<int, uintptr_t>, unsigned int*> g_amax_state;

nvfp4_status amax_state_for(cudaStream_t s, unsigned int** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return NVFP4_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mutex);
  unsigned int*& p = g_amax_state[{dev, reinterpret_cast<uintptr_t>(s)}];
  if (p == nullptr) {
    void* q = nullptr;
    if (cudaMalloc(&q, 256) != cudaSuccess) return NVFP4_ERR_CUDA;
    if (cudaMemsetAsync(q, 0, 256, s) != cudaSuccess) {
      cudaFree(q);
      return NVFP4_ERR_CUDA;
    }
    p = static_cast<unsigned int*>(q);
  }
  *out = p;
  return NVFP4_OK;
}

// Per-device set-up, done once with that device current: SM count and the address of the error word.
nvfp4_status device_state(DeviceState** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return NVFP4_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mutex);
  DeviceState& st = g_devices[dev];
  if (!st.ready) {
    if (cudaDeviceGetAttribute(&st.sm_count, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return NVFP4_ERR_CUDA;
    if (cudaGetSymbolAddress(reinterpret_cast<void**>(&st.error_word), g_device_error) != cudaSuccess)
      return NVFP4_ERR_CUDA;
    st.ready = true;
  }
  *out = &st;
  return NVFP4_OK;
}

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

uint64_t wait_timeout_ns() {
  static uint64_t ns = [] {
    const char* e = std::getenv("NVFP4_WAIT_TIMEOUT_MS");
    long ms = e ? std::strtol(e, nullptr, 10) : 1000;
    if (ms <= 0) ms = 1000;
    return static_cast<uint64_t>(ms) * 1000000ull;
  }();
  return ns;
}

#ifdef NVFP4_TEST_HOOKS
// Test builds only (libnvfp4_testhooks.so): see nvfp4_test_withhold_split_ready.
std::atomic<int> g_test_withhold_split_ready{0};
#endif

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

int64_t k_atoms_of(int64_t cols) { return (cols / 16 + 3) / 4; }

int64_t ld_codes_of(const nvfp4_tensor* t) { return t->ld_codes ? t->ld_codes : t->cols / 2; }

// Checks shared by every NVFP4 tensor argument.  The quantiser and dequantiser move codes in 4- and
// 8-byte words, so their code rows need 8-byte alignment; the GEMM reads them with TMA (16 bytes).
nvfp4_status check_tensor(const nvfp4_tensor* t, bool need_scale, int64_t ld_align) {
  if (!t || !t->codes || !t->scales || (need_scale && !t->tensor_scale)) return NVFP4_ERR_INVALID_ARG;
  if (t->rows < 0 || t->cols <= 0) return NVFP4_ERR_INVALID_ARG;
  if (t->cols % 16) return NVFP4_ERR_UNSUPPORTED_SHAPE;
  const int64_t ld = ld_codes_of(t);
  if (ld < t->cols / 2) return NVFP4_ERR_INVALID_ARG;
  if (!aligned16(t->codes) || (ld % ld_align) || !aligned16(t->scales) ||
      (t->tensor_scale && !aligned4(t->tensor_scale)))
    return NVFP4_ERR_MISALIGNED;
  return NVFP4_OK;
}

nvfp4_status launch_status() { return cudaGetLastError() == cudaSuccess ? NVFP4_OK : NVFP4_ERR_CUDA; }

// Grid for a grid-stride kernel: enough CTAs for the work, at most one resident wave.
template <typename Kernel>
int resident_grid(Kernel kernel, int threads, int64_t work_items, int items_per_cta, int sm_count) {
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, threads, 0) != cudaSuccess || per_sm < 1)
    per_sm = 1;
  int64_t g = (work_items + items_per_cta - 1) / items_per_cta;
  const int64_t cap = static_cast<int64_t>(sm_count) * per_sm;
  if (g > cap) g = cap;
  if (g < 1) g = 1;
  return static_cast<int>(g);
}

// 2-D TMA descriptor over packed E2M1 codes viewed as bytes: [rows][cols/2], box of 128 rows x one
// stage's row bytes, swizzled by that width (the layout the tensor-core descriptors expect).
nvfp4_status make_code_map(CUtensorMap* map, const nvfp4_tensor* t) {
  auto encode = tensor_map_encoder();
  if (!encode) return NVFP4_ERR_CUDA;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(t->cols / 2), static_cast<cuuint64_t>(t->rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(ld_codes_of(t))};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(kStageRowBytes), 128};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = encode(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, t->codes, dims, strides, box, estr,
                      CU_TENSOR_MAP_INTERLEAVE_NONE,
                      kStageRowBytes == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B,
                      CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                      CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? NVFP4_OK : NVFP4_ERR_CUDA;
}

// 2-D TMA descriptor over a tensor's block-scale bytes viewed as rows of one 512-byte atom (128 x
// uint32, unswizzled): row b * k_atoms + k is atom k of 128-row block b.  A box is four atoms, the
// scales of one 128-row block for one stage of K; rows past the last block read as zeros.
nvfp4_status make_scale_map(CUtensorMap* map, const nvfp4_tensor* t) {
  auto encode = tensor_map_encoder();
  if (!encode) return NVFP4_ERR_CUDA;
  const int64_t atoms = (t->rows + 127) / 128 * k_atoms_of(t->cols);
  cuuint64_t dims[2] = {128, static_cast<cuuint64_t>(atoms)};
  cuuint64_t strides[1] = {512};
  cuuint32_t box[2] = {128, static_cast<cuuint32_t>(kStageKSteps)};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = encode(map, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, t->scales, dims, strides, box, estr,
                      CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                      CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? NVFP4_OK : NVFP4_ERR_CUDA;
}

// TMA store maps of the fused linear's outputs, in the boxes the epilogue writes (32 rows of one warp):
// bf16 output `box_cols` (16 or 32) columns wide with the 32- or 64-byte swizzle of its shared-memory
// box, E2M1 codes 16 bytes wide unswizzled.  A map stays zeroed when its output is not requested (the
// kernel never uses it).
nvfp4_status make_store_maps(OutMaps* om, void* out_bf16, int64_t ld_out, const nvfp4_tensor* out_fp4, int64_t M,
                             int64_t n_out, int box_cols) {
  std::memset(om, 0, sizeof(*om));
  auto encode = tensor_map_encoder();
  if (!encode) return NVFP4_ERR_CUDA;
  cuuint32_t estr[2] = {1, 1};
  if (out_bf16) {
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(n_out), static_cast<cuuint64_t>(M)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(ld_out * 2)};
    cuuint32_t box[2] = {static_cast<cuuint32_t>(box_cols), 32};
    if (encode(&om->out, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, out_bf16, dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, box_cols == 32 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_32B,
               CU_TENSOR_MAP_L2_PROMOTION_NONE,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return NVFP4_ERR_CUDA;
  }
  if (out_fp4) {
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(n_out / 2), static_cast<cuuint64_t>(M)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(ld_codes_of(out_fp4))};
    cuuint32_t box[2] = {16, 32};
    if (encode(&om->q_codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, out_fp4->codes, dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return NVFP4_ERR_CUDA;
  }
  return NVFP4_OK;
}

// Two-way split of K for long reductions (the 53248-wide text projection): a function of K and the
// epilogue only, never of M, so every row's arithmetic is the same whatever M is.  The head norm takes
// its sum of squares while loading the accumulator and is never split.
int split_k_for(int64_t K, int32_t kind) { return (K >= 32768 && kind != NVFP4_EPI_QKNORM) ? 2 : 1; }

// Column tile width: 256 whenever N allows it (CTA pairs); otherwise 128-wide tiles on single CTAs, the
// last of which is ragged when N is not a multiple of 128 (the weight's TMA box fills its rows past N
// with zeros, the epilogue reads no bias, residual or gate there and the store map drops its columns).
// The head norm needs whole 256-wide heads and the gated SiLU pairs 128-row halves of a and b.
int tile_n_for(int64_t N, int64_t K, int32_t kind) {
  if (K < 64 || K % 64 || N <= 0) return 0;
  if (kind == NVFP4_EPI_QKNORM || kind == NVFP4_EPI_GATED_SILU) return N % 256 == 0 ? 256 : 0;
  if (kind == NVFP4_EPI_BIAS || kind == NVFP4_EPI_RESID_GATE) {
    if (N % 256 == 0) return 256;
    if (N % 16 == 0) return 128;
  }
  return 0;
}

// 256-wide tiles without split-K run on CTA pairs unless NVFP4_GEMM_PAIR=0.
bool pair_kernel_enabled() {
  static const bool on = [] {
    const char* v = std::getenv("NVFP4_GEMM_PAIR");
    return !(v && v[0] == '0');
  }();
  return on;
}

template <int KIND, bool kSplit>
nvfp4_status launch_gemm_pair_as(DeviceState* st, const CUtensorMap& ma, const CUtensorMap& mb, const ScaleMaps& sm,
                                 const OutMaps& om, const GemmArgs& args, cudaStream_t stream) {
  using C = GemmPairCfg;
  auto kernel = nvfp4_gemm_pair_kernel<KIND, kSplit>;
  int clusters = 0;
  {
    // first use on this device (under the library lock, so concurrent callers do it once)
    std::lock_guard<std::mutex> lock(g_mutex);
    int& cached = st->pair_clusters[kSplit ? 1 : 0][KIND];
    if (cached == 0) {
      if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES) != cudaSuccess)
        return NVFP4_ERR_CUDA;
      // clusters that can be resident at once: the persistent grid must not exceed one wave
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3(2 * (st->sm_count / 2));
      cfg.blockDim = dim3(C::THREADS);
      cfg.dynamicSmemBytes = C::SMEM_BYTES;
      int n = 0;
      if (cudaOccupancyMaxActiveClusters(&n, kernel, &cfg) != cudaSuccess || n < 1) return NVFP4_ERR_CUDA;
      cached = n;
    }
    clusters = cached;
  }
  const int grid_clusters = args.num_units < clusters ? args.num_units : clusters;
  kernel<<<2 * grid_clusters, C::THREADS, C::SMEM_BYTES, stream>>>(ma, mb, sm, om, args);
  return launch_status();
}

template <int KIND>
nvfp4_status launch_gemm_pair(DeviceState* st, const CUtensorMap& ma, const CUtensorMap& mb, const ScaleMaps& sm,
                              const OutMaps& om, const GemmArgs& args, cudaStream_t stream) {
  if constexpr (KIND == kEpiQkNorm) {
    return launch_gemm_pair_as<KIND, false>(st, ma, mb, sm, om, args, stream);  // never split
  } else {
    return args.splits > 1 ? launch_gemm_pair_as<KIND, true>(st, ma, mb, sm, om, args, stream)
                           : launch_gemm_pair_as<KIND, false>(st, ma, mb, sm, om, args, stream);
  }
}

template <int BN, int KIND>
nvfp4_status launch_gemm(DeviceState* st, const CUtensorMap& ma, const CUtensorMap& mb, const OutMaps& om,
                         const GemmArgs& args, cudaStream_t stream) {
  using C = GemmCfg<BN>;
  auto kernel = nvfp4_gemm_kernel<BN, KIND>;
  {
    std::lock_guard<std::mutex> lock(g_mutex);
    bool& attr = st->smem_attr_set[BN == 256 ? 1 : 0][KIND];
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

int32_t nvfp4_version(void) { return 100; }

const char* nvfp4_status_string(nvfp4_status s) {
  switch (s) {
    case NVFP4_OK: return "ok";
    case NVFP4_ERR_INVALID_ARG: return "invalid argument";
    case NVFP4_ERR_UNSUPPORTED_SHAPE: return "unsupported shape";
    case NVFP4_ERR_MISALIGNED: return "misaligned pointer or leading dimension";
    case NVFP4_ERR_CUDA: return "CUDA runtime error";
    case NVFP4_ERR_DEVICE_TIMEOUT: return "device-side pipeline wait timed out";
    case NVFP4_ERR_SCRATCH_LIMIT: return "split-K scratch needed exceeds the fixed buffer of nvfp4_linear_noalloc";
  }
  return "unknown status";
}

size_t nvfp4_scale_bytes(int64_t rows, int64_t cols) {
  if (rows < 0 || cols <= 0) return 0;
  const int64_t r = (rows + 127) / 128 * 128;
  return static_cast<size_t>(r * k_atoms_of(cols) * 4);
}

int64_t nvfp4_scale_offset(int64_t r, int64_t kb, int64_t cols) { return scale_offset(r, kb, k_atoms_of(cols)); }

int32_t nvfp4_linear_tile_n(int64_t N, int64_t K, int32_t kind) { return tile_n_for(N, K, kind); }

int32_t nvfp4_linear_split_k(int64_t N, int64_t K, int32_t kind) {
  return tile_n_for(N, K, kind) ? split_k_for(K, kind) : 0;
}

}  // extern "C"

namespace {

// The fused linear; `fixed_scratch` selects the split-K scratch: the library's per-stream buffer
// (nvfp4_linear) or the fixed file-scope array (nvfp4_linear_noalloc).
nvfp4_status linear_impl(const nvfp4_tensor* a, const nvfp4_tensor* w, const nvfp4_epilogue_desc* epi,
                         void* out_bf16, int64_t ld_out, const nvfp4_tensor* out_fp4, nvfp4_stream_t stream,
                         bool fixed_scratch) {
  if (!epi) return NVFP4_ERR_INVALID_ARG;
  if (nvfp4_status e = check_tensor(a, true, 16)) return e;
  if (nvfp4_status e = check_tensor(w, true, 16)) return e;
  const int64_t M = a->rows, N = w->rows, K = a->cols;
  if (w->cols != K) return NVFP4_ERR_INVALID_ARG;
  if (epi->kind < NVFP4_EPI_BIAS || epi->kind > NVFP4_EPI_RESID_GATE) return NVFP4_ERR_INVALID_ARG;
  const int BN = tile_n_for(N, K, epi->kind);
  if (BN == 0) return NVFP4_ERR_UNSUPPORTED_SHAPE;
  if (M > (int64_t(1) << 30) || N > (int64_t(1) << 30) || K > (int64_t(1) << 30)) return NVFP4_ERR_UNSUPPORTED_SHAPE;
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
  if (nvfp4_status e = make_code_map(&ma, a)) return e;
  if (nvfp4_status e = make_code_map(&mb, w)) return e;
  const bool pair = BN == 256 && pair_kernel_enabled();
  OutMaps om;
  if (nvfp4_status e = make_store_maps(&om, out_bf16, ld_out, epi->out_nvfp4 ? out_fp4 : nullptr, M, n_out,
                                       pair ? GemmPairCfg::XPOSE_BYTES / 64 : 16))
    return e;

  GemmArgs g{};
  g.M = static_cast<int32_t>(M);
  g.N = static_cast<int32_t>(N);
  g.K = static_cast<int32_t>(K);
  g.n_out = static_cast<int32_t>(n_out);
  g.num_m_blocks = static_cast<int32_t>((M + 127) / 128);
  g.num_n_blocks = static_cast<int32_t>(epi->kind == NVFP4_EPI_GATED_SILU ? (N / 2) / 128 : (N + BN - 1) / BN);
  g.num_tiles = g.num_m_blocks * g.num_n_blocks;
  g.num_m_pairs = static_cast<int32_t>((M + 255) / 256);
  g.k_steps = static_cast<int32_t>(K / 64);
  g.k_atoms = static_cast<int32_t>(k_atoms_of(K));
  g.sfa = static_cast<const uint8_t*>(a->scales);
  g.sfb = static_cast<const uint8_t*>(w->scales);
  g.ga = a->tensor_scale;
  g.gb = w->tensor_scale;
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
#ifdef NVFP4_TEST_HOOKS
  g.test_withhold_split_ready = g_test_withhold_split_ready.load();
#endif
  // Tile order: every wave of the persistent grid re-reads whichever operand the order sweeps, so the
  // order keeps the smaller operand (same K: fewer rows) resident in L2 and streams the larger one from
  // HBM once.  (Row blocks fastest re-read all of A every wave; for the 2048^2 down projection that is
  // 117 MB of A per wave against a 126 MB L2.)  Which CTA computes a tile never changes its bits.
  g.n_fastest = N <= M ? 1 : 0;
  g.splits = split_k_for(K, epi->kind);
  if (pair) g.num_tiles = g.num_m_pairs * g.num_n_blocks;  // 256 x 256 tiles of CTA pairs
  g.num_units = g.num_tiles * g.splits;
  // split-K exchange slots: one per tile, or one per CTA of each pair tile
  const int64_t exch_slots = static_cast<int64_t>(g.num_tiles) * (pair ? 2 : 1);

  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (g.splits > 1) {
    const int cols_per_thread = epi->kind == NVFP4_EPI_GATED_SILU ? 128 : BN / 2;
    const size_t flag_bytes = (static_cast<size_t>(exch_slots) * 4 + 255) & ~size_t(255);
    const size_t part_bytes = static_cast<size_t>(exch_slots) * 2 * 128 * cols_per_thread * 4;
    void* ws = nullptr;
    if (fixed_scratch) {
      if (flag_bytes + part_bytes > kNoAllocScratchBytes) return NVFP4_ERR_SCRATCH_LIMIT;
      if (nvfp4_status e = noalloc_scratch(&ws)) return e;
    } else if (nvfp4_status e = scratch_for(s, flag_bytes + part_bytes, &ws)) {
      return e;
    }
    g.split_flags = static_cast<unsigned int*>(ws);
    g.split_partials = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + flag_bytes);
    if (cudaMemsetAsync(ws, 0, static_cast<size_t>(exch_slots) * 4, s) != cudaSuccess) return NVFP4_ERR_CUDA;
  }
  if (pair) {
    ScaleMaps sm;
    if (nvfp4_status e = make_scale_map(&sm.sfa, a)) return e;
    if (nvfp4_status e = make_scale_map(&sm.sfb, w)) return e;
    switch (epi->kind) {
      case NVFP4_EPI_BIAS: return launch_gemm_pair<kEpiBias>(st, ma, mb, sm, om, g, s);
      case NVFP4_EPI_RESID_GATE: return launch_gemm_pair<kEpiResidGate>(st, ma, mb, sm, om, g, s);
      case NVFP4_EPI_QKNORM: return launch_gemm_pair<kEpiQkNorm>(st, ma, mb, sm, om, g, s);
      case NVFP4_EPI_GATED_SILU: return launch_gemm_pair<kEpiGatedSilu>(st, ma, mb, sm, om, g, s);
    }
    return NVFP4_ERR_INVALID_ARG;
  }
  switch (epi->kind) {
    case NVFP4_EPI_BIAS:
      return BN == 256 ? launch_gemm<256, kEpiBias>(st, ma, mb, om, g, s) : launch_gemm<128, kEpiBias>(st, ma, mb, om, g, s);
    case NVFP4_EPI_RESID_GATE:
      return BN == 256 ? launch_gemm<256, kEpiResidGate>(st, ma, mb, om, g, s)
                       : launch_gemm<128, kEpiResidGate>(st, ma, mb, om, g, s);
    case NVFP4_EPI_QKNORM: return launch_gemm<256, kEpiQkNorm>(st, ma, mb, om, g, s);
    case NVFP4_EPI_GATED_SILU: return launch_gemm<256, kEpiGatedSilu>(st, ma, mb, om, g, s);
  }
  return NVFP4_ERR_INVALID_ARG;
}

}  // namespace

extern "C" {

nvfp4_status nvfp4_linear(const nvfp4_tensor* a, const nvfp4_tensor* w, const nvfp4_epilogue_desc* epi,
                          void* out_bf16, int64_t ld_out, const nvfp4_tensor* out_fp4, nvfp4_stream_t stream) {
  return linear_impl(a, w, epi, out_bf16, ld_out, out_fp4, stream, false);
}

// Same computation as nvfp4_linear, for callers that must not allocate device memory: the split-K
// scratch of long-K calls lives in a fixed 64 MiB device array instead of a buffer the library
// allocates.  The array's address is looked up on the first call on each device.  Calls whose
// scratch would not fit return NVFP4_ERR_SCRATCH_LIMIT before launching anything.  All calls on a
// device share the array, so calls that overlap on the GPU race.
nvfp4_status nvfp4_linear_noalloc(const nvfp4_tensor* a, const nvfp4_tensor* w, const nvfp4_epilogue_desc* epi,
                                  void* out_bf16, int64_t ld_out, const nvfp4_tensor* out_fp4,
                                  nvfp4_stream_t stream) {
  return linear_impl(a, w, epi, out_bf16, ld_out, out_fp4, stream, true);
}

size_t nvfp4_linear_noalloc_scratch_bytes(void) { return kNoAllocScratchBytes; }

#ifdef NVFP4_TEST_HOOKS
// Test builds only, not declared in the public header: while `on` is non-zero, the split-K linears
// launched afterwards withhold the first unit's ready bit, so that the second unit's bounded wait runs
// out, the kernel gives up and nvfp4_get_device_error reports NVFP4_ERR_DEVICE_TIMEOUT.  This is how the
// device-timeout path is exercised without faulting or hanging anything.
NVFP4_API void nvfp4_test_withhold_split_ready(int32_t on) { g_test_withhold_split_ready.store(on != 0); }
#endif

nvfp4_status nvfp4_get_device_error(nvfp4_stream_t stream) {
  DeviceState* st;
  if (nvfp4_status e = device_state(&st)) return e;
  if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) return NVFP4_ERR_CUDA;
  unsigned int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_device_error, sizeof(v)) != cudaSuccess) return NVFP4_ERR_CUDA;
  if (v) {
    const unsigned int zero = 0;
    if (cudaMemcpyToSymbol(g_device_error, &zero, sizeof(zero)) != cudaSuccess) return NVFP4_ERR_CUDA;
  }
  return v == 0 ? NVFP4_OK : (v == kErrTimeout ? NVFP4_ERR_DEVICE_TIMEOUT : NVFP4_ERR_CUDA);
}

}  // extern "C"

// Entry points of the bandwidth-bound op family (amax, quantise, fake quantise, adaLN quantise,
// dequantise): they use the helpers above, so they are part of this translation unit.
#include "quantize_api.cuh"

// Entry points of the W8A8 INT8 linear and its quantiser.
#include "int8_api.cuh"
