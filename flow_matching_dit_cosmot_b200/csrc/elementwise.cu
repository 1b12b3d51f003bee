// HBM-bound kernels: routed RMSNorm, standalone mRoPE, the Euler sampler step
// and its guided form.
//
// All of them stream 16-byte vectors (8 bf16) per thread with fully coalesced
// warps; grids are sized in multiples of the SM count.
#include <cuda_bf16.h>

#include "cosmot_internal.h"
#include "ptx.cuh"

namespace cosmot {
namespace {

constexpr int kMaxSegs = 64;

struct SegTable {
  int64_t row_begin[kMaxSegs];
  int64_t out_row[kMaxSegs];
  int64_t prefix[kMaxSegs + 1];  // flattened row index where each segment starts
  int64_t out_extent;            // output rows the segments address (debug store checks)
  int32_t set[kMaxSegs];
  int32_t n;
};

bool fill_segs(const cosmot_segment* segs, int32_t n, SegTable* t) {
  if (!segs || n < 1 || n > kMaxSegs) return false;
  t->n = n;
  t->out_extent = 0;
  int64_t acc = 0;
  for (int i = 0; i < n; ++i) {
    if (segs[i].row_begin < 0 || segs[i].row_end < segs[i].row_begin || segs[i].out_row < 0) return false;
    if (segs[i].weight_set != 0 && segs[i].weight_set != 1) return false;
    t->row_begin[i] = segs[i].row_begin;
    t->out_row[i] = segs[i].out_row;
    t->set[i] = segs[i].weight_set;
    t->prefix[i] = acc;
    acc += segs[i].row_end - segs[i].row_begin;
    const int64_t end = segs[i].out_row + (segs[i].row_end - segs[i].row_begin);
    if (end > t->out_extent) t->out_extent = end;
  }
  t->prefix[n] = acc;
  return true;
}

// ---------------------------------------------------------------- RMSNorm
// One warp per row.  A bf16 row stays in registers between the two passes; a
// float32 row (a residual stream kept in float32) is read again in the second
// pass, from L1/L2, so that the registers hold no more than for bf16.
__device__ __forceinline__ void load8_f32(const float* p, float* f) {
  const float4 a = *reinterpret_cast<const float4*>(p);
  const float4 b = *reinterpret_cast<const float4*>(p + 4);
  f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w;
  f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
}

template <int kVecPerLane>
__global__ void __launch_bounds__(256) rmsnorm_f32in_kernel(const float* __restrict__ h, int64_t ld_h,
                                                            const SegTable segs, const __nv_bfloat16* __restrict__ g0,
                                                            const __nv_bfloat16* __restrict__ g1, int32_t d, float eps,
                                                            __nv_bfloat16* __restrict__ out, int64_t ld_out,
                                                            int* status) {
  pdl_trigger();
  pdl_wait();
  const int lane = threadIdx.x & 31;
  const int64_t warps_total = (int64_t)gridDim.x * (blockDim.x >> 5);
  const int nvec = d >> 3;
  for (int64_t gr = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); gr < segs.prefix[segs.n];
       gr += warps_total) {
    int s = 0;
    while (s + 1 < segs.n && gr >= segs.prefix[s + 1]) ++s;
    const int64_t local = gr - segs.prefix[s];
    const int64_t r = segs.row_begin[s] + local;
    const int64_t o = segs.out_row[s] + local;
    const __nv_bfloat16* g = segs.set[s] ? g1 : g0;
    const float* src = h + r * ld_h;
    float ss = 0.f;
#pragma unroll
    for (int j = 0; j < kVecPerLane; ++j) {
      const int c = lane + 32 * j;
      if (c < nvec) {
        float f[8];
        load8_f32(src + 8 * c, f);
#pragma unroll
        for (int q = 0; q < 8; ++q) ss = fmaf(f[q], f[q], ss);
      }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
    const float rstd = rsqrtf(ss / (float)d + eps);
    if (!dcheck(o >= 0 && o < segs.out_extent, status, kWhereNormStore)) continue;
    uint4* dst = reinterpret_cast<uint4*>(out + o * ld_out);
    const uint4* gv = reinterpret_cast<const uint4*>(g);
#pragma unroll
    for (int j = 0; j < kVecPerLane; ++j) {
      const int c = lane + 32 * j;
      if (c < nvec) {
        float f[8];
        load8_f32(src + 8 * c, f);
        uint4 gg = __ldg(gv + c);
        const uint32_t* gu = reinterpret_cast<const uint32_t*>(&gg);
        uint4 res;
        uint32_t* ru = reinterpret_cast<uint32_t*>(&res);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          float2 w = unpack_bf16x2(gu[q]);
          ru[q] = pack_bf16x2(f[2 * q] * rstd * w.x, f[2 * q + 1] * rstd * w.y);
        }
        dst[c] = res;
      }
    }
  }
}

// Wide rows (d >= 1024): one 128-thread block per row, up to kVecPerThread
// 16-byte vectors of 8 elements per thread held in registers across both
// passes (float32 rows as two float4 per vector), so a row is read once.  Small
// blocks keep up to 16 rows in flight per SM; the sum of squares is reduced by
// warp shuffles and a two-slot shared-memory exchange (one barrier per row).
constexpr int kNormBlock = 128;

template <typename TIn, int kVecPerThread>
__global__ void __launch_bounds__(kNormBlock) rmsnorm_block_kernel(const TIn* __restrict__ h, int64_t ld_h,
                                                                  const SegTable segs,
                                                                  const __nv_bfloat16* __restrict__ g0,
                                                                  const __nv_bfloat16* __restrict__ g1, int32_t d,
                                                                  float eps, __nv_bfloat16* __restrict__ out,
                                                                  int64_t ld_out, int* status) {
  pdl_trigger();
  pdl_wait();
  constexpr bool kF32 = sizeof(TIn) == 4;
  __shared__ float part[2][kNormBlock / 32];
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const int nvec = d >> 3;
  int slot = 0;
  for (int64_t gr = blockIdx.x; gr < segs.prefix[segs.n]; gr += gridDim.x, slot ^= 1) {
    int s = 0;
    while (s + 1 < segs.n && gr >= segs.prefix[s + 1]) ++s;
    const int64_t local = gr - segs.prefix[s];
    const TIn* src = h + (segs.row_begin[s] + local) * ld_h;
    float f[kVecPerThread][8];
    float ss = 0.f;
#pragma unroll
    for (int j = 0; j < kVecPerThread; ++j) {
      const int c = threadIdx.x + kNormBlock * j;
      if (c < nvec) {
        if (kF32) {
          const float4 a = *reinterpret_cast<const float4*>(reinterpret_cast<const float*>(src) + 8 * c);
          const float4 b = *reinterpret_cast<const float4*>(reinterpret_cast<const float*>(src) + 8 * c + 4);
          f[j][0] = a.x; f[j][1] = a.y; f[j][2] = a.z; f[j][3] = a.w;
          f[j][4] = b.x; f[j][5] = b.y; f[j][6] = b.z; f[j][7] = b.w;
        } else {
          const uint4 v = *reinterpret_cast<const uint4*>(reinterpret_cast<const __nv_bfloat16*>(src) + 8 * c);
          const uint32_t* u = reinterpret_cast<const uint32_t*>(&v);
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const float2 x = unpack_bf16x2(u[q]);
            f[j][2 * q] = x.x;
            f[j][2 * q + 1] = x.y;
          }
        }
#pragma unroll
        for (int q = 0; q < 8; ++q) ss = fmaf(f[j][q], f[j][q], ss);
      }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
    if (lane == 0) part[slot][wid] = ss;
    __syncthreads();  // also orders this row's reads of part[slot] before its reuse two rows later
    float tot = 0.f;
#pragma unroll
    for (int i = 0; i < kNormBlock / 32; ++i) tot += part[slot][i];
    const float rstd = rsqrtf(tot / (float)d + eps);
    const __nv_bfloat16* g = segs.set[s] ? g1 : g0;
    const int64_t orow = segs.out_row[s] + local;
    const bool store_ok = dcheck(orow >= 0 && orow < segs.out_extent, status, kWhereNormStore);
    uint4* dst = reinterpret_cast<uint4*>(out + orow * ld_out);
    const uint4* gv = reinterpret_cast<const uint4*>(g);
#pragma unroll
    for (int j = 0; j < kVecPerThread; ++j) {
      const int c = threadIdx.x + kNormBlock * j;
      if (c < nvec && store_ok) {
        const uint4 gg = __ldg(gv + c);
        const uint32_t* gu = reinterpret_cast<const uint32_t*>(&gg);
        uint4 res;
        uint32_t* ru = reinterpret_cast<uint32_t*>(&res);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float2 wq = unpack_bf16x2(gu[q]);
          ru[q] = pack_bf16x2(f[j][2 * q] * rstd * wq.x, f[j][2 * q + 1] * rstd * wq.y);
        }
        dst[c] = res;
      }
    }
  }
}

template <int kVecPerLane>
__global__ void __launch_bounds__(256) rmsnorm_kernel(const __nv_bfloat16* __restrict__ h, int64_t ld_h,
                                                      const SegTable segs, const __nv_bfloat16* __restrict__ g0,
                                                      const __nv_bfloat16* __restrict__ g1, int32_t d, float eps,
                                                      __nv_bfloat16* __restrict__ out, int64_t ld_out,
                                                      int* status) {
  pdl_trigger();
  pdl_wait();
  const int lane = threadIdx.x & 31;
  const int64_t warps_total = (int64_t)gridDim.x * (blockDim.x >> 5);
  const int nvec = d >> 3;
  for (int64_t gr = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); gr < segs.prefix[segs.n];
       gr += warps_total) {
    int s = 0;
    while (s + 1 < segs.n && gr >= segs.prefix[s + 1]) ++s;
    const int64_t local = gr - segs.prefix[s];
    const int64_t r = segs.row_begin[s] + local;
    const int64_t o = segs.out_row[s] + local;
    const __nv_bfloat16* g = segs.set[s] ? g1 : g0;
    const uint4* src = reinterpret_cast<const uint4*>(h + r * ld_h);
    uint4 v[kVecPerLane];
    float ss = 0.f;
#pragma unroll
    for (int j = 0; j < kVecPerLane; ++j) {
      const int c = lane + 32 * j;
      if (c < nvec) {
        v[j] = src[c];
        const uint32_t* u = reinterpret_cast<const uint32_t*>(&v[j]);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          float2 f = unpack_bf16x2(u[q]);
          ss = fmaf(f.x, f.x, ss);
          ss = fmaf(f.y, f.y, ss);
        }
      }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
    const float rstd = rsqrtf(ss / (float)d + eps);
    if (!dcheck(o >= 0 && o < segs.out_extent, status, kWhereNormStore)) continue;
    uint4* dst = reinterpret_cast<uint4*>(out + o * ld_out);
    const uint4* gv = reinterpret_cast<const uint4*>(g);
#pragma unroll
    for (int j = 0; j < kVecPerLane; ++j) {
      const int c = lane + 32 * j;
      if (c < nvec) {
        uint4 gg = __ldg(gv + c);
        const uint32_t* u = reinterpret_cast<const uint32_t*>(&v[j]);
        const uint32_t* gu = reinterpret_cast<const uint32_t*>(&gg);
        uint4 res;
        uint32_t* ru = reinterpret_cast<uint32_t*>(&res);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          float2 f = unpack_bf16x2(u[q]);
          float2 w = unpack_bf16x2(gu[q]);
          ru[q] = pack_bf16x2(f.x * rstd * w.x, f.y * rstd * w.y);
        }
        dst[c] = res;
      }
    }
  }
}

// ---------------------------------------------------------------- mRoPE
// One thread per (row, head, group of 8 pairs): reads x[i..i+7] and
// x[i+hd/2..+7], rotates them with the table and writes both back.
__global__ void __launch_bounds__(256) mrope_kernel(__nv_bfloat16* __restrict__ q, int64_t ld_q, int32_t n_q_heads,
                                                    __nv_bfloat16* __restrict__ k, int64_t ld_k, int32_t n_k_heads,
                                                    int64_t n_rows, int32_t head_dim,
                                                    const float2* __restrict__ cs) {
  pdl_trigger();
  pdl_wait();
  const int32_t half = head_dim >> 1;
  const int32_t groups = half >> 3;
  const int32_t per_row = (n_q_heads + n_k_heads) * groups;
  const int64_t total = n_rows * per_row;
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < total; e += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = e / per_row;
    const int32_t w = (int32_t)(e % per_row);
    const int32_t head = w / groups;
    const int32_t i0 = (w % groups) * 8;
    __nv_bfloat16* base = head < n_q_heads ? q + r * ld_q + (int64_t)head * head_dim
                                           : k + r * ld_k + (int64_t)(head - n_q_heads) * head_dim;
    uint4 lo = *reinterpret_cast<const uint4*>(base + i0);
    uint4 hi = *reinterpret_cast<const uint4*>(base + half + i0);
    const float4* t = reinterpret_cast<const float4*>(cs + r * half + i0);
    float c[8], s[8];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      float4 v = __ldg(t + j);  // (cos, sin) of pairs i0+2j and i0+2j+1
      c[2 * j] = v.x;
      s[2 * j] = v.y;
      c[2 * j + 1] = v.z;
      s[2 * j + 1] = v.w;
    }
    uint32_t* lu = reinterpret_cast<uint32_t*>(&lo);
    uint32_t* hu = reinterpret_cast<uint32_t*>(&hi);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      float2 a = unpack_bf16x2(lu[j]);
      float2 b = unpack_bf16x2(hu[j]);
      const float c0 = c[2 * j], s0 = s[2 * j], c1 = c[2 * j + 1], s1 = s[2 * j + 1];
      lu[j] = pack_bf16x2(a.x * c0 - b.x * s0, a.y * c1 - b.y * s1);
      hu[j] = pack_bf16x2(b.x * c0 + a.x * s0, b.y * c1 + a.y * s1);
    }
    *reinterpret_cast<uint4*>(base + i0) = lo;
    *reinterpret_cast<uint4*>(base + half + i0) = hi;
  }
}

// ---------------------------------------------------------------- Euler
__global__ void __launch_bounds__(256) euler_kernel(__nv_bfloat16* __restrict__ x, int64_t ld_x,
                                                    const __nv_bfloat16* __restrict__ v, int64_t ld_v,
                                                    int64_t row_begin, int64_t n_rows, int64_t n_cols, float dsigma,
                                                    int* status) {
  pdl_trigger();
  pdl_wait();
  const int64_t vec_per_row = n_cols >> 3;
  const int64_t total = n_rows * vec_per_row;
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < total; e += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = row_begin + e / vec_per_row;
    const int64_t c = (e % vec_per_row) << 3;
    if (!dcheck(r < row_begin + n_rows && c + 8 <= n_cols, status, kWhereEulerStore)) continue;
    uint4* xp = reinterpret_cast<uint4*>(x + r * ld_x + c);
    uint4 xv = *xp;
    uint4 vv = __ldg(reinterpret_cast<const uint4*>(v + r * ld_v + c));
    uint32_t* xu = reinterpret_cast<uint32_t*>(&xv);
    const uint32_t* vu = reinterpret_cast<const uint32_t*>(&vv);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      float2 a = unpack_bf16x2(xu[j]);
      float2 b = unpack_bf16x2(vu[j]);
      xu[j] = pack_bf16x2(fmaf(dsigma, b.x, a.x), fmaf(dsigma, b.y, a.y));
    }
    *xp = xv;
  }
}

// ---------------------------------------------------------------- guided Euler
// x' = x + dsigma * (v_base + w * (v_cond - v_base)), written to both states of
// a (conditioned, baseline) pair so they stay identical for the next step.
__global__ void __launch_bounds__(256) cfg_euler_kernel(__nv_bfloat16* x_cond, __nv_bfloat16* x_base,
                                                        int64_t ld_x,
                                                        const __nv_bfloat16* __restrict__ v_cond,
                                                        const __nv_bfloat16* __restrict__ v_base, int64_t ld_v,
                                                        int64_t n_rows, int64_t n_cols, float dsigma, float w) {
  pdl_trigger();
  pdl_wait();
  const int64_t vec_per_row = n_cols >> 3;
  const int64_t total = n_rows * vec_per_row;
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < total; e += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = e / vec_per_row;
    const int64_t c = (e % vec_per_row) << 3;
    uint4 xv = *reinterpret_cast<const uint4*>(x_cond + r * ld_x + c);
    const uint4 vc = __ldg(reinterpret_cast<const uint4*>(v_cond + r * ld_v + c));
    const uint4 vb = __ldg(reinterpret_cast<const uint4*>(v_base + r * ld_v + c));
    uint32_t* xu = reinterpret_cast<uint32_t*>(&xv);
    const uint32_t* cu = reinterpret_cast<const uint32_t*>(&vc);
    const uint32_t* bu = reinterpret_cast<const uint32_t*>(&vb);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float2 a = unpack_bf16x2(xu[j]);
      const float2 fc = unpack_bf16x2(cu[j]);
      const float2 fb = unpack_bf16x2(bu[j]);
      const float v0 = fmaf(w, fc.x - fb.x, fb.x);
      const float v1 = fmaf(w, fc.y - fb.y, fb.y);
      xu[j] = pack_bf16x2(fmaf(dsigma, v0, a.x), fmaf(dsigma, v1, a.y));
    }
    *reinterpret_cast<uint4*>(x_cond + r * ld_x + c) = xv;
    *reinterpret_cast<uint4*>(x_base + r * ld_x + c) = xv;
  }
}

unsigned grid_for(int64_t work_items, int threads) {
  const int64_t want = (work_items + threads - 1) / threads;
  const int64_t cap = (int64_t)num_sms() * 16;
  return (unsigned)(want < 1 ? 1 : (want < cap ? want : cap));
}

}  // namespace
}  // namespace cosmot

namespace cosmot {

cosmot_status rmsnorm_routed(const void* h, bool h_f32, int64_t ld_h, const cosmot_segment* segs, int32_t n_segs,
                             const void* g0, const void* g1, int64_t d, float eps, void* out, int64_t ld_out,
                             cosmot_stream_t stream) {
  SegTable t;
  if (!h || !out || !fill_segs(segs, n_segs, &t)) return COSMOT_ERR_INVALID_ARG;
  if (d <= 0 || d % 8 || ld_h % 8 || ld_out % 8 || ld_h < d || ld_out < d || !aligned16(h) || !aligned16(out))
    return COSMOT_ERR_INVALID_ARG;
  for (int i = 0; i < t.n; ++i) {
    const void* g = t.set[i] ? g1 : g0;
    if (!g || !aligned16(g)) return COSMOT_ERR_INVALID_ARG;
  }
  if (d > 8 * kNormBlock * 6) return COSMOT_ERR_UNSUPPORTED;  // d <= 6144: 6 vectors per thread of a block
  const int64_t rows = t.prefix[t.n];
  if (rows == 0) return COSMOT_OK;
  const int threads = 256;
  const unsigned grid = grid_for(rows * 32, threads);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const auto* hp = static_cast<const __nv_bfloat16*>(h);
  const auto* gp0 = static_cast<const __nv_bfloat16*>(g0);
  const auto* gp1 = static_cast<const __nv_bfloat16*>(g1);
  auto* op = static_cast<__nv_bfloat16*>(out);
  int* st = device_status_ptr();
  if (!st) return COSMOT_ERR_CUDA;
  cudaError_t e;
  if (d >= 1024) {  // one block per row
    const int64_t cap = (int64_t)num_sms() * 16;
    const unsigned bgrid = (unsigned)(rows < cap ? rows : cap);
    const int vpt = (int)((d / 8 + kNormBlock - 1) / kNormBlock);
    if (h_f32) {
      const auto* hf = static_cast<const float*>(h);
      if (vpt <= 4)
        e = launch_pdl(rmsnorm_block_kernel<float, 4>, dim3(bgrid), dim3(kNormBlock), 0, s, nullptr, hf, ld_h, t,
                         gp0, gp1, (int32_t)d, eps, op, ld_out, st);
      else
        e = launch_pdl(rmsnorm_block_kernel<float, 6>, dim3(bgrid), dim3(kNormBlock), 0, s, nullptr, hf, ld_h, t,
                         gp0, gp1, (int32_t)d, eps, op, ld_out, st);
    } else {
      if (vpt <= 4)
        e = launch_pdl(rmsnorm_block_kernel<__nv_bfloat16, 4>, dim3(bgrid), dim3(kNormBlock), 0, s, nullptr, hp,
                         ld_h, t, gp0, gp1, (int32_t)d, eps, op, ld_out, st);
      else
        e = launch_pdl(rmsnorm_block_kernel<__nv_bfloat16, 6>, dim3(bgrid), dim3(kNormBlock), 0, s, nullptr, hp,
                         ld_h, t, gp0, gp1, (int32_t)d, eps, op, ld_out, st);
    }
    return launch_status(e);
  }
  // narrow rows (d < 1024): one warp per row, at most 4 vectors per lane
  if (h_f32)
    e = launch_pdl(rmsnorm_f32in_kernel<4>, dim3(grid), dim3(threads), 0, s, nullptr, static_cast<const float*>(h),
                     ld_h, t, gp0, gp1, (int32_t)d, eps, op, ld_out, st);
  else
    e = launch_pdl(rmsnorm_kernel<4>, dim3(grid), dim3(threads), 0, s, nullptr, hp, ld_h, t, gp0, gp1, (int32_t)d,
                     eps, op, ld_out, st);
  return launch_status(e);
}

}  // namespace cosmot

extern "C" {

cosmot_status cosmot_rmsnorm_routed(const void* h, int64_t ld_h, const cosmot_segment* segs, int32_t n_segs,
                                    const void* g0, const void* g1, int64_t d, float eps, void* out,
                                    int64_t ld_out, cosmot_stream_t stream) {
  return cosmot::rmsnorm_routed(h, false, ld_h, segs, n_segs, g0, g1, d, eps, out, ld_out, stream);
}

cosmot_status cosmot_mrope_apply(void* q, int64_t ld_q, int32_t n_q_heads, void* k, int64_t ld_k,
                                 int32_t n_k_heads, int64_t n_rows, int32_t head_dim, const float* cs,
                                 cosmot_stream_t stream) {
  using namespace cosmot;
  if (!cs || n_rows < 0 || n_q_heads < 0 || n_k_heads < 0) return COSMOT_ERR_INVALID_ARG;
  if (head_dim <= 0 || head_dim % 16) return COSMOT_ERR_UNSUPPORTED;
  if (n_q_heads > 0 && (!q || !aligned16(q) || ld_q % 8 || ld_q < (int64_t)n_q_heads * head_dim))
    return COSMOT_ERR_INVALID_ARG;
  if (n_k_heads > 0 && (!k || !aligned16(k) || ld_k % 8 || ld_k < (int64_t)n_k_heads * head_dim))
    return COSMOT_ERR_INVALID_ARG;
  if (!aligned16(cs)) return COSMOT_ERR_INVALID_ARG;
  const int64_t items = n_rows * (n_q_heads + n_k_heads) * (head_dim / 16);
  if (items == 0) return COSMOT_OK;
  const int threads = 256;
  return launch_status(launch_pdl(mrope_kernel, dim3(grid_for(items, threads)), dim3(threads), 0,
                                  reinterpret_cast<cudaStream_t>(stream), nullptr, static_cast<__nv_bfloat16*>(q), ld_q,
                                  n_q_heads, static_cast<__nv_bfloat16*>(k), ld_k, n_k_heads, n_rows, head_dim,
                                  reinterpret_cast<const float2*>(cs)));
}

cosmot_status cosmot_flow_euler_step(void* x, int64_t ld_x, const void* v, int64_t ld_v, int64_t row_begin,
                                     int64_t row_end, int64_t n_cols, double sigma, double sigma_next,
                                     cosmot_stream_t stream) {
  using namespace cosmot;
  if (!x || !v || row_begin < 0 || row_end < row_begin || n_cols <= 0) return COSMOT_ERR_INVALID_ARG;
  if (n_cols % 8 || ld_x % 8 || ld_v % 8 || ld_x < n_cols || ld_v < n_cols || !aligned16(x) || !aligned16(v))
    return COSMOT_ERR_INVALID_ARG;
  const int64_t items = (row_end - row_begin) * (n_cols / 8);
  if (items == 0) return COSMOT_OK;
  const float dsigma = (float)(sigma_next - sigma);
  const int threads = 256;
  int* st = device_status_ptr();
  if (!st) return COSMOT_ERR_CUDA;
  return launch_status(launch_pdl(euler_kernel, dim3(grid_for(items, threads)), dim3(threads), 0,
                                  reinterpret_cast<cudaStream_t>(stream), nullptr, static_cast<__nv_bfloat16*>(x), ld_x,
                                  static_cast<const __nv_bfloat16*>(v), ld_v, row_begin, row_end - row_begin, n_cols,
                                  dsigma, st));
}

cosmot_status cosmot_flow_cfg_euler_step(void* x_cond, void* x_base, int64_t ld_x, const void* v_cond,
                                         const void* v_base, int64_t ld_v, int64_t n_rows, int64_t n_cols,
                                         double sigma, double sigma_next, double guidance, cosmot_stream_t stream) {
  using namespace cosmot;
  if (!x_cond || !x_base || !v_cond || !v_base || n_rows < 0 || n_cols <= 0) return COSMOT_ERR_INVALID_ARG;
  if (n_cols % 8 || ld_x % 8 || ld_v % 8 || ld_x < n_cols || ld_v < n_cols) return COSMOT_ERR_INVALID_ARG;
  if (!aligned16(x_cond) || !aligned16(x_base) || !aligned16(v_cond) || !aligned16(v_base)) return COSMOT_ERR_INVALID_ARG;
  const int64_t items = n_rows * (n_cols / 8);
  if (items == 0) return COSMOT_OK;
  const int threads = 256;
  return launch_status(launch_pdl(cfg_euler_kernel, dim3(grid_for(items, threads)), dim3(threads), 0,
                                  reinterpret_cast<cudaStream_t>(stream), nullptr, static_cast<__nv_bfloat16*>(x_cond),
                                  static_cast<__nv_bfloat16*>(x_base), ld_x, static_cast<const __nv_bfloat16*>(v_cond),
                                  static_cast<const __nv_bfloat16*>(v_base), ld_v, n_rows, n_cols,
                                  (float)(sigma_next - sigma), (float)guidance));
}

}  // extern "C"
