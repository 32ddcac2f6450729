// Library-wide state: the per-device status word, error messages, version,
// debug hooks, and tensor-map encoding through the driver entry point.
#include <cuda.h>
#include <cuda_runtime.h>

#include <mutex>
#include <string>

#include "common.cuh"
#include "launch.h"
#include "tc_sm100.cuh"
#include "tmap.h"

#include <cstdlib>

namespace pbsa {

// One status word per device.  Kernels write PBSA_ERR_TIMEOUT into it with
// atomicCAS(0 -> code); pbsa_get_status reads and clears it.
__device__ int g_device_status = 0;

static thread_local std::string t_last_error;
static int g_debug_flags = 0;
static int64_t g_wait_limit_ns = 2000000000LL;

void set_error(const std::string& msg) { t_last_error = msg; }
int debug_flags() { return g_debug_flags; }
int64_t wait_limit_ns() { return g_wait_limit_ns; }

bool pdl_enabled() {
  static const bool on = [] {
    const char* e = std::getenv("PBSA_PDL");
    return !(e != nullptr && e[0] == '0');
  }();
  return on;
}

int sm_count() {
  static int counts[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  if (counts[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n < 1)
      n = 148;
    counts[dev] = n;
  }
  return counts[dev];
}

int* device_status_ptr() {
  static int* ptrs[64] = {nullptr};
  static std::mutex mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (ptrs[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_device_status) != cudaSuccess) return nullptr;
    ptrs[dev] = static_cast<int*>(p);
  }
  return ptrs[dev];
}

// ------------------------------------------------------------- tensor maps
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

int make_tmap_bf16_2d(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols,
                      uint32_t box_rows, uint32_t box_cols) {
  EncodeTiledFn fn = encode_fn();
  PBSA_CHECK_ARG(fn != nullptr, PBSA_ERR_CUDA, "cuTensorMapEncodeTiled is not available");
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 2};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  PBSA_CHECK_ARG(r == CUDA_SUCCESS, PBSA_ERR_CUDA,
                 "cuTensorMapEncodeTiled failed with code " + std::to_string(int(r)));
  return PBSA_OK;
}

// y_poly[i] = exp2_poly2(x[i]) (the FMA-pipe exponent of the attention
// softmax), y_hw[i] = ex2.approx (the special-function unit it replaces on
// three pairs in four), both on the device, for the unit test of the former.
__global__ void exp2_check_kernel(const float* __restrict__ x, float* __restrict__ y_poly,
                                  float* __restrict__ y_hw, int n) {
  const int i = 2 * (blockIdx.x * blockDim.x + threadIdx.x);
  if (i >= n) return;
  const float x0 = x[i], x1 = (i + 1 < n) ? x[i + 1] : 0.f;
  float p0, p1;
  tc::f2_split(tc::exp2_poly2(tc::f2(x0, x1)), p0, p1);
  y_poly[i] = p0;
  y_hw[i] = tc::ex2(x0);
  if (i + 1 < n) {
    y_poly[i + 1] = p1;
    y_hw[i + 1] = tc::ex2(x1);
  }
}

}  // namespace pbsa

extern "C" {

int pbsa_check_exp2(const float* x, float* y_poly, float* y_hw, int n, void* stream) {
  PBSA_CHECK_ARG(x && y_poly && y_hw && n >= 1, PBSA_ERR_ARG, "check_exp2: NULL buffer or n < 1");
  const int pairs = (n + 1) / 2;
  pbsa::exp2_check_kernel<<<(pairs + 255) / 256, 256, 0, static_cast<cudaStream_t>(stream)>>>(
      x, y_poly, y_hw, n);
  PBSA_CHECK_LAUNCH("exp2_check_kernel");
  return PBSA_OK;
}

int pbsa_get_status(void* stream) {
  int* p = pbsa::device_status_ptr();
  if (p == nullptr) {
    pbsa::set_error("cannot resolve the device status word");
    return PBSA_ERR_CUDA;
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int host = 0;
  cudaError_t e = cudaMemcpyAsync(&host, p, sizeof(int), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e == cudaSuccess) e = cudaMemsetAsync(p, 0, sizeof(int), s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) {
    pbsa::set_error(std::string("pbsa_get_status: ") + cudaGetErrorString(e));
    return PBSA_ERR_CUDA;
  }
  return host;
}

const char* pbsa_last_error(void) { return pbsa::t_last_error.c_str(); }

const char* pbsa_version(void) { return "pbsa-b200 0.1.0 (sm_100a)"; }

void pbsa_set_debug(int flags, int64_t wait_limit_ns) {
  pbsa::g_debug_flags = flags;
  pbsa::g_wait_limit_ns = wait_limit_ns > 0 ? wait_limit_ns : 2000000000LL;
}

}  // extern "C"
