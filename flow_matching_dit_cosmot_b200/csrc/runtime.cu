// Status strings, the device status word, tensor-map encoding and device
// queries shared by every entry point.
#include <cstdio>
#include <cstring>
#include <mutex>

#include "cosmot_internal.h"
#include "ptx.cuh"

namespace cosmot {

__device__ int g_status_word[2];

namespace {

constexpr int kMaxDevices = 64;
int* g_status_ptr[kMaxDevices] = {};
int g_sm_count[kMaxDevices] = {};
std::mutex g_mu;

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn g_encode = nullptr;

EncodeTiledFn encode_fn() {
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_encode) {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<EncodeTiledFn>(fn);
  }
  return g_encode;
}

}  // namespace

int* device_status_ptr() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_status_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_status_word) != cudaSuccess) return nullptr;
    g_status_ptr[dev] = static_cast<int*>(p);
  }
  return g_status_ptr[dev];
}

int num_sms() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 148;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_sm_count[dev]) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    g_sm_count[dev] = n;
  }
  return g_sm_count[dev];
}

cosmot_status make_tmap_bf16_2d(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols, uint64_t ld,
                                uint32_t box_rows, uint32_t box_cols) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return COSMOT_ERR_CUDA;
  if (!aligned16(base) || (ld * 2) % 16 != 0 || rows == 0 || cols == 0) return COSMOT_ERR_INVALID_ARG;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {ld * 2};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? COSMOT_OK : COSMOT_ERR_INVALID_ARG;
}

// Test-only: warp 0 is a producer that never arrives on the barrier; thread 32
// waits for it with the library's bounded wait, which gives up after
// kWaitLimitNs and latches COSMOT_ERR_TIMEOUT at kWhereSelftest.
__global__ void __launch_bounds__(64) selftest_timeout_kernel(int* status) {
  __shared__ alignas(8) uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 32) mbar_wait(smem_u32(&bar), 0, status, kWhereSelftest);
  __syncthreads();
}

// Test-only: a checked store one past its stated extent (index 1 of extent 1
// into a two-element array, so the store would stay in bounds even unchecked).
__device__ int g_selftest_bounds_target[2];

__global__ void selftest_bounds_kernel(int* status) {
  const int extent = 1, index = 1;
  if (dcheck(index < extent, status, kWhereSelftestBounds)) g_selftest_bounds_target[index] = 1;
}

}  // namespace cosmot

extern "C" {

int32_t cosmot_debug_checks(void) {
#if defined(COSMOT_DEBUG_CHECKS)
  return 1;
#else
  return 0;
#endif
}

cosmot_status cosmot_selftest_bounds_check(cosmot_stream_t stream) {
#if defined(COSMOT_DEBUG_CHECKS)
  int* st = cosmot::device_status_ptr();
  if (!st) return COSMOT_ERR_CUDA;
  cosmot::selftest_bounds_kernel<<<1, 1, 0, reinterpret_cast<cudaStream_t>(stream)>>>(st);
  return cosmot::launch_status();
#else
  (void)stream;
  return COSMOT_ERR_UNSUPPORTED;
#endif
}

cosmot_status cosmot_selftest_wait_timeout(cosmot_stream_t stream) {
  int* st = cosmot::device_status_ptr();
  if (!st) return COSMOT_ERR_CUDA;
  cosmot::selftest_timeout_kernel<<<1, 64, 0, reinterpret_cast<cudaStream_t>(stream)>>>(st);
  return cosmot::launch_status();
}

const char* cosmot_status_string(cosmot_status s) {
  switch (s) {
    case COSMOT_OK: return "COSMOT_OK";
    case COSMOT_ERR_INVALID_ARG: return "COSMOT_ERR_INVALID_ARG";
    case COSMOT_ERR_UNSUPPORTED: return "COSMOT_ERR_UNSUPPORTED";
    case COSMOT_ERR_CUDA: return "COSMOT_ERR_CUDA";
    case COSMOT_ERR_TIMEOUT: return "COSMOT_ERR_TIMEOUT";
    case COSMOT_ERR_WORKSPACE: return "COSMOT_ERR_WORKSPACE";
    case COSMOT_ERR_BOUNDS: return "COSMOT_ERR_BOUNDS";
    default: return "COSMOT_ERR_UNKNOWN";
  }
}

int32_t cosmot_version(void) { return 200; }

cosmot_status cosmot_get_device_status(cosmot_stream_t stream, cosmot_status* out, int32_t* where_out) {
  if (!out) return COSMOT_ERR_INVALID_ARG;
  int* p = cosmot::device_status_ptr();
  if (!p) return COSMOT_ERR_CUDA;
  int host[2] = {0, 0};
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (cudaMemcpyAsync(host, p, sizeof(host), cudaMemcpyDeviceToHost, s) != cudaSuccess) return COSMOT_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return COSMOT_ERR_CUDA;
  if (host[0] != 0) {
    if (cudaMemsetAsync(p, 0, sizeof(host), s) != cudaSuccess) return COSMOT_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return COSMOT_ERR_CUDA;
  }
  *out = host[0];
  if (where_out) *where_out = host[1];
  return COSMOT_OK;
}

}  // extern "C"
