// cosmot_layer_forward for callers that cannot allocate device memory.
//
// Some callers are not allowed to allocate at all once they are running: a
// robot or simulator control loop with a hard per-step deadline (cudaMalloc can
// synchronise the device and take unbounded time), or a host framework that
// hands out all device memory from its own pool and forbids anyone else from
// calling the CUDA allocator.  Such a caller still owns its inputs and outputs
// but cannot provide the layer's workspace.  This entry point takes the
// workspace from a fixed array compiled into the library instead.
//
// The array is a file-scope __device__ variable: every GPU that loads this
// library's device code holds kNoAllocScratchBytes for it until the process
// exits.  The CUDA driver reserves it when it loads this file's module on a
// device.  Under the default lazy module loading that happens at the first
// cudaGetSymbolAddress below, i.e. inside the first call on each device (with
// CUDA_MODULE_LOADING=EAGER, at context creation instead), so a caller with a
// deadline makes one warm-up call before its loop.  In host code the array's
// name only stands in for the symbol and is not a device address, so the
// address is looked up with cudaGetSymbolAddress, once per device, with that
// device current, the first time the entry point runs on it.  The cached
// address belongs to the device's current primary context: after a
// cudaDeviceReset the entry point must not be called again in that process.
#include <mutex>

#include "cosmot_internal.h"

namespace cosmot {
namespace {

// COSMOT_NOALLOC_SCRATCH_BYTES (64 MiB): enough for one full-width (d_model
// 4096, FFN 14336) DROID policy step (703 tokens, batch 1), which needs about
// 61 MB of workspace.
constexpr size_t kNoAllocScratchBytes = COSMOT_NOALLOC_SCRATCH_BYTES;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
void* g_scratch_ptr[kMaxDevices] = {};
std::mutex g_scratch_mu;

// Device address of g_noalloc_scratch on the current device (looked up once).
cosmot_status scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return COSMOT_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_scratch_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return COSMOT_ERR_CUDA;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return COSMOT_OK;
}

}  // namespace
}  // namespace cosmot

extern "C" {

cosmot_status cosmot_layer_forward_noalloc(const cosmot_dims* dims, const cosmot_layer_weights* w,
                                           const cosmot_seq_desc* seq, void* h, void* h_out, double sigma,
                                           double sigma_next, cosmot_stream_t stream) {
  if (!seq) return COSMOT_ERR_INVALID_ARG;
  // Every call starts from scratch contents left by the previous call; only
  // self-contained calls are accepted, where each scratch byte read is first
  // written by the same call.
  if (seq->n_cached != 0) return COSMOT_ERR_UNSUPPORTED;
  size_t need = 0;
  cosmot_status st = cosmot_layer_workspace_size(dims, seq, &need);
  if (st != COSMOT_OK) return st;
  if (need > cosmot::kNoAllocScratchBytes) return COSMOT_ERR_WORKSPACE;
  void* scratch = nullptr;
  st = cosmot::scratch_address(&scratch);
  if (st != COSMOT_OK) return st;
  return cosmot_layer_forward(dims, w, seq, h, h_out, sigma, sigma_next, scratch, cosmot::kNoAllocScratchBytes,
                              stream);
}

}  // extern "C"
