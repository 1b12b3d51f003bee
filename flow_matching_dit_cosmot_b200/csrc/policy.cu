// Sampler schedule and the action heads of a policy.
//
// "Cosmos 3 方法原理全解" §6.3: the flow shift sigma = s t_bar / (1 + (s - 1)
// t_bar), t_bar = 1 - t.  §4.2: normalised actions (clean conditions and the
// noisy variable alike) enter the Generator through a domain-specific W_in, and
// a domain-specific W_out returns the action velocity at the current sigma;
// the sampler integrates in the normalised action space.  §6.3 also gives every
// modality its own noise level, so the action state takes its own Euler step.
//
// Both action kernels are small (tens of rows): the embedding is a K = C_a
// contraction (C_a = 8 for DROID joint positions, 10 for a generic arm) done on
// the CUDA cores, one thread per 8 output columns; the head is one warp per
// action row (or per conditioned/baseline row pair under guidance) that forms
// the RMS of the row and the C_a dot products with W_out in one pass, in fp32.
#include <cuda_bf16.h>

#include <cmath>

#include "cosmot_internal.h"
#include "ptx.cuh"

namespace cosmot {
namespace {

constexpr int kMaxActSegs = 64;
constexpr int kMaxActionDim = 32;

struct ActSegs {
  int64_t row_begin[kMaxActSegs];  // first source row
  int64_t out_row[kMaxActSegs];    // first destination row
  int64_t prefix[kMaxActSegs + 1];
  int32_t n;
};

bool fill_act_segs(const cosmot_segment* segs, int32_t n, ActSegs* t) {
  if (!segs || n < 1 || n > kMaxActSegs) return false;
  t->n = n;
  int64_t acc = 0;
  for (int i = 0; i < n; ++i) {
    if (segs[i].row_begin < 0 || segs[i].row_end < segs[i].row_begin || segs[i].out_row < 0) return false;
    t->row_begin[i] = segs[i].row_begin;
    t->out_row[i] = segs[i].out_row;
    t->prefix[i] = acc;
    acc += segs[i].row_end - segs[i].row_begin;
  }
  t->prefix[n] = acc;
  return true;
}

__device__ __forceinline__ int seg_of(const ActSegs& s, int64_t r) {
  int i = 0;
  while (i + 1 < s.n && r >= s.prefix[i + 1]) ++i;
  return i;
}

// h[out] = bf16(x[row] . W_in^T): thread (row, 8-column chunk).
__global__ void __launch_bounds__(256) action_embed_kernel(const __nv_bfloat16* __restrict__ x, int64_t ld_x,
                                                           const ActSegs segs,
                                                           const __nv_bfloat16* __restrict__ w_in, int32_t ca,
                                                           int32_t d, __nv_bfloat16* __restrict__ h, int64_t ld_h) {
  pdl_trigger();
  pdl_wait();
  const int chunks = d >> 3;
  const int64_t total = segs.prefix[segs.n] * chunks;
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < total; e += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = e / chunks;
    const int c8 = (int)(e % chunks) << 3;
    const int s = seg_of(segs, r);
    const int64_t local = r - segs.prefix[s];
    const __nv_bfloat16* xr = x + (segs.row_begin[s] + local) * ld_x;
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    for (int c = 0; c < ca; ++c) {
      const float xv = __bfloat162float(xr[c]);
#pragma unroll
      for (int j = 0; j < 8; ++j) acc[j] = fmaf(xv, __bfloat162float(w_in[(int64_t)(c8 + j) * ca + c]), acc[j]);
    }
    uint4 o;
    o.x = pack_bf16x2(acc[0], acc[1]);
    o.y = pack_bf16x2(acc[2], acc[3]);
    o.z = pack_bf16x2(acc[4], acc[5]);
    o.w = pack_bf16x2(acc[6], acc[7]);
    *reinterpret_cast<uint4*>(h + (segs.out_row[s] + local) * ld_h + c8) = o;
  }
}

// Velocity of one action row in one pass: lane c (< ca) returns
// v_c = rstd * sum_j h_j g_j w_out[c, j] (the RMS scale factored out of the
// sums), fp32 throughout; 16-byte loads of h, g and each W_out row.
__device__ __forceinline__ float action_velocity_row(const __nv_bfloat16* __restrict__ hr,
                                                     const __nv_bfloat16* __restrict__ g,
                                                     const __nv_bfloat16* __restrict__ w_out, int32_t ca, int32_t d,
                                                     float eps, int lane) {
  float acc[kMaxActionDim];
#pragma unroll
  for (int c = 0; c < kMaxActionDim; ++c) acc[c] = 0.f;
  float ss = 0.f;
  for (int j8 = lane * 8; j8 < d; j8 += 256) {
    const uint4 hv = __ldg(reinterpret_cast<const uint4*>(hr + j8));
    const uint4 gv = __ldg(reinterpret_cast<const uint4*>(g + j8));
    const uint32_t* hu = reinterpret_cast<const uint32_t*>(&hv);
    const uint32_t* gu = reinterpret_cast<const uint32_t*>(&gv);
    float hg[8];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 hh = unpack_bf16x2(hu[e]);
      const float2 gg = unpack_bf16x2(gu[e]);
      ss = fmaf(hh.x, hh.x, fmaf(hh.y, hh.y, ss));
      hg[2 * e] = hh.x * gg.x;
      hg[2 * e + 1] = hh.y * gg.y;
    }
#pragma unroll
    for (int c = 0; c < kMaxActionDim; ++c) {
      if (c < ca) {
        const uint4 wv = __ldg(reinterpret_cast<const uint4*>(w_out + (int64_t)c * d + j8));
        const uint32_t* wu = reinterpret_cast<const uint32_t*>(&wv);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 ww = unpack_bf16x2(wu[e]);
          acc[c] = fmaf(hg[2 * e], ww.x, fmaf(hg[2 * e + 1], ww.y, acc[c]));
        }
      }
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
  const float rstd = rsqrtf(ss / (float)d + eps);
  float mine = 0.f;
#pragma unroll
  for (int c = 0; c < kMaxActionDim; ++c) {
    if (c < ca) {
      float v = acc[c];
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
      if (lane == c) mine = v * rstd;
    }
  }
  return mine;
}

// One warp per action row (unguided) or per conditioned/baseline pair of rows
// (guided: segments 2p and 2p+1 are the pair).  x[out] = bf16(x[out] + dsigma v).
__global__ void __launch_bounds__(256) action_head_kernel(const __nv_bfloat16* __restrict__ h, int64_t ld_h,
                                                          const ActSegs segs, const __nv_bfloat16* __restrict__ g,
                                                          float eps, const __nv_bfloat16* __restrict__ w_out,
                                                          int32_t ca, int32_t d, __nv_bfloat16* x, int64_t ld_x,
                                                          float dsigma, int32_t guided, float w) {
  pdl_trigger();
  pdl_wait();
  const int lane = threadIdx.x & 31;
  const int64_t warps_total = (int64_t)gridDim.x * (blockDim.x >> 5);
  // guided: one item per row of the even (conditioned) segments
  const int64_t items = guided ? segs.prefix[segs.n] / 2 : segs.prefix[segs.n];
  for (int64_t it = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); it < items; it += warps_total) {
    if (!guided) {
      const int s = seg_of(segs, it);
      const int64_t local = it - segs.prefix[s];
      const float v = action_velocity_row(h + (segs.row_begin[s] + local) * ld_h, g, w_out, ca, d, eps, lane);
      if (lane < ca) {
        __nv_bfloat16* xp = x + (segs.out_row[s] + local) * ld_x + lane;
        *xp = __float2bfloat16_rn(fmaf(dsigma, v, __bfloat162float(*xp)));
      }
    } else {
      // pair p covers segments 2p (cond) and 2p+1 (base) of equal length
      int64_t acc = 0;
      int p = 0;
      for (;; ++p) {
        const int64_t len = segs.prefix[2 * p + 1] - segs.prefix[2 * p];
        if (it < acc + len || 2 * p + 3 > segs.n) break;
        acc += len;
      }
      const int64_t local = it - acc;
      const int sc = 2 * p, sb = 2 * p + 1;
      const float vc = action_velocity_row(h + (segs.row_begin[sc] + local) * ld_h, g, w_out, ca, d, eps, lane);
      const float vb = action_velocity_row(h + (segs.row_begin[sb] + local) * ld_h, g, w_out, ca, d, eps, lane);
      if (lane < ca) {
        const float v = fmaf(w, vc - vb, vb);
        __nv_bfloat16* xc = x + (segs.out_row[sc] + local) * ld_x + lane;
        __nv_bfloat16* xb = x + (segs.out_row[sb] + local) * ld_x + lane;
        const __nv_bfloat16 r = __float2bfloat16_rn(fmaf(dsigma, v, __bfloat162float(*xc)));
        *xc = r;
        *xb = r;
      }
    }
  }
}

unsigned grid_cap(int64_t items, int per_block) {
  const int64_t want = (items + per_block - 1) / per_block;
  const int64_t cap = (int64_t)num_sms() * 8;
  return (unsigned)(want < 1 ? 1 : (want < cap ? want : cap));
}

}  // namespace
}  // namespace cosmot

extern "C" {

cosmot_status cosmot_flow_shift_sigmas(int32_t n_steps, double shift, double* sigmas) {
  if (n_steps < 1 || !(shift > 0.0) || !std::isfinite(shift) || !sigmas) return COSMOT_ERR_INVALID_ARG;
  for (int32_t k = 0; k <= n_steps; ++k) {
    const double t_bar = 1.0 - (double)k / (double)n_steps;
    sigmas[k] = shift * t_bar / (1.0 + (shift - 1.0) * t_bar);
  }
  return COSMOT_OK;
}

cosmot_status cosmot_action_embed(const void* x, int64_t ld_x, const cosmot_segment* segs, int32_t n_segs,
                                  const void* w_in, int32_t action_dim, int32_t d_model, void* h, int64_t ld_h,
                                  cosmot_stream_t stream) {
  using namespace cosmot;
  if (!x || !w_in || !h || action_dim < 1 || action_dim > kMaxActionDim || d_model < 8 || d_model % 8 ||
      ld_x < action_dim || ld_h < d_model || ld_h % 8 || !aligned16(h))
    return COSMOT_ERR_INVALID_ARG;
  ActSegs t;
  if (!fill_act_segs(segs, n_segs, &t)) return COSMOT_ERR_INVALID_ARG;
  if (t.prefix[t.n] == 0) return COSMOT_OK;
  const int64_t items = t.prefix[t.n] * (d_model / 8);
  return launch_status(launch_pdl(action_embed_kernel, dim3(grid_cap(items, 256)), dim3(256), 0,
                                  reinterpret_cast<cudaStream_t>(stream), nullptr, static_cast<const __nv_bfloat16*>(x),
                                  ld_x, t, static_cast<const __nv_bfloat16*>(w_in), action_dim, d_model,
                                  static_cast<__nv_bfloat16*>(h), ld_h));
}

cosmot_status cosmot_action_head(const void* h_last, int64_t ld_h, const cosmot_segment* segs, int32_t n_segs,
                                 const void* g_fin, float eps, const void* w_out, int32_t action_dim, int32_t d_model,
                                 void* x, int64_t ld_x, double sigma, double sigma_next, const double* guidance,
                                 cosmot_stream_t stream) {
  using namespace cosmot;
  if (!h_last || !g_fin || !w_out || !x || action_dim < 1 || action_dim > kMaxActionDim || d_model < 8 ||
      d_model % 8 || ld_h < d_model || ld_h % 8 || ld_x < action_dim || !(eps >= 0.f) || !aligned16(h_last) ||
      !aligned16(g_fin) || !aligned16(w_out))
    return COSMOT_ERR_INVALID_ARG;
  ActSegs t;
  if (!fill_act_segs(segs, n_segs, &t)) return COSMOT_ERR_INVALID_ARG;
  if (guidance) {
    if (t.n % 2) return COSMOT_ERR_INVALID_ARG;
    for (int p = 0; p < t.n / 2; ++p)
      if (t.prefix[2 * p + 1] - t.prefix[2 * p] != t.prefix[2 * p + 2] - t.prefix[2 * p + 1])
        return COSMOT_ERR_INVALID_ARG;
  }
  const int64_t items = guidance ? t.prefix[t.n] / 2 : t.prefix[t.n];
  if (items == 0) return COSMOT_OK;
  return launch_status(launch_pdl(action_head_kernel, dim3(grid_cap(items, 8)), dim3(256), 0,
                                  reinterpret_cast<cudaStream_t>(stream), nullptr,
                                  static_cast<const __nv_bfloat16*>(h_last), ld_h, t,
                                  static_cast<const __nv_bfloat16*>(g_fin), eps,
                                  static_cast<const __nv_bfloat16*>(w_out), action_dim, d_model,
                                  static_cast<__nv_bfloat16*>(x), ld_x, (float)(sigma_next - sigma), guidance ? 1 : 0,
                                  guidance ? (float)*guidance : 0.f));
}

}  // extern "C"
