// Internal declarations shared by the libcosmot translation units.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "cosmot.h"

namespace cosmot {

// Device status site codes (reported through cosmot_get_device_status).
enum Where : int {
  kWhereGemmProducer = 100,
  kWhereGemmMma = 101,
  kWhereGemmEpilogue = 102,
  kWhereGemmDrain = 103,
  kWhereAttnProducer = 200,
  kWhereAttnMma = 201,
  kWhereAttnSoftmax = 202,
  kWhereAttnDrain = 203,
  // debug-build store checks (COSMOT_ERR_BOUNDS)
  kWhereGemmStore = 104,
  kWhereAttnStore = 204,
  kWhereNormStore = 300,
  kWhereEulerStore = 301,
  kWhereSelftest = COSMOT_SITE_SELFTEST,
  kWhereSelftestBounds = COSMOT_SITE_SELFTEST_BOUNDS,
};

// Encodes a 2D bf16 tensor map: `rows` x `cols` elements with row pitch
// `ld` elements, box of box_rows x box_cols (box_cols * 2 == 128 bytes for the
// 128-byte swizzle), out-of-bounds elements read as zero.
cosmot_status make_tmap_bf16_2d(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols, uint64_t ld,
                                uint32_t box_rows, uint32_t box_cols);

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline cosmot_status launch_status() {
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? COSMOT_OK : COSMOT_ERR_CUDA;
}

// The status of a launch call's own return code and of the runtime's last
// error, which is read (and so cleared) either way: a failed launch leaves
// nothing behind for the next call's check.
inline cosmot_status launch_status(cudaError_t launched) {
  const cudaError_t last = cudaGetLastError();
  return launched == cudaSuccess && last == cudaSuccess ? COSMOT_OK : COSMOT_ERR_CUDA;
}

int num_sms();

// Launches a kernel with programmatic stream serialization: it may be
// scheduled while the previous kernel of the stream drains, so its prologue
// (barrier setup, tensor-memory allocation, descriptor prefetch) overlaps that
// kernel's last wave.  The kernel must execute pdl_wait (ptx.cuh) in every
// thread before touching memory an earlier kernel writes or reads, and before
// it exits.  `extra` adds one more launch attribute (a cluster shape).
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                              const cudaLaunchAttribute* extra, Args&&... args) {
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  unsigned n = 1;
  if (extra != nullptr) attr[n++] = *extra;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = n;
  return cudaLaunchKernelEx(&cfg, kern, static_cast<Args&&>(args)...);
}

// cosmot_rmsnorm_routed with a float32 input when h_f32 (the layer's h1, the
// residual stream between the attention and FFN halves, is kept in float32).
cosmot_status rmsnorm_routed(const void* h, bool h_f32, int64_t ld_h, const cosmot_segment* segs, int32_t n_segs,
                             const void* g0, const void* g1, int64_t d, float eps, void* out, int64_t ld_out,
                             cosmot_stream_t stream);

// Key split of an attention call with dm_items DM work items (sequences x
// heads x query-tile pairs) over n_keys keys (see cosmot_attention_kv_split).
int32_t attention_kv_split(int64_t dm_items, int64_t n_keys);

// Per-device address of the status word that kernels latch failures into.
int* device_status_ptr();

}  // namespace cosmot
