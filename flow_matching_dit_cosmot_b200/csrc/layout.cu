// Packed-sequence layout (mRoPE coordinates, block ids) and the mRoPE cos/sin
// table.  "Cosmos 3 方法原理全解" §2 (token order) and §5 (t/h/w coordinates,
// dt = 6/TPS, TPS = FPS/4 for video, the 15000 AR->DM offset).
//
// Coordinates are formed in float64 with explicitly rounded operations (no
// contraction into FMA) in the order: T0 + tau*dt, then rounded once to
// float32, so the float32 result is reproducible bit for bit.
#include "cosmot_internal.h"

namespace cosmot {
namespace {

constexpr int kArDmTimeOffset = 15000;

struct LayoutParams {
  // Group boundaries (token index where each group starts), in packing order:
  // 0 AR | 1 clean video | 2 clean audio | 3 clean action | 4 proprio |
  // 5 noisy video | 6 noisy audio | 7 noisy action | 8 = end.
  int32_t start[9];
  int32_t n_ar;
  int32_t views, gh, gw, fps;
  int32_t clean_steps;
  int32_t audio_clean, audio_rate;
  int32_t action_clean, action_hz;
  int32_t tau_offset;
};

bool group_bounds(const cosmot_layout_spec& s, int32_t start[9]) {
  if (s.n_text < 0 || s.video_views < 0 || s.video_grid_h < 0 || s.video_grid_w < 0 || s.video_clean_steps < 0 ||
      s.video_noisy_steps < 0 || s.audio_clean < 0 || s.audio_noisy < 0 || s.action_clean < 0 ||
      s.action_noisy < 0 || s.proprio < 0 || s.tau_offset < 0)
    return false;
  const bool has_video = (s.video_clean_steps + s.video_noisy_steps) > 0;
  if (has_video && (s.video_views <= 0 || s.video_grid_h <= 0 || s.video_grid_w <= 0 || s.video_fps <= 0))
    return false;
  if ((s.audio_clean + s.audio_noisy) > 0 && s.audio_rate <= 0) return false;
  if ((s.action_clean + s.action_noisy) > 0 && s.action_hz <= 0) return false;
  const int64_t tps = has_video ? (int64_t)s.video_views * s.video_grid_h * s.video_grid_w : 0;
  int64_t sizes[8] = {(int64_t)s.n_text + 2,
                      tps * s.video_clean_steps,
                      s.audio_clean,
                      s.action_clean,
                      s.proprio,
                      tps * s.video_noisy_steps,
                      s.audio_noisy,
                      s.action_noisy};
  int64_t acc = 0;
  for (int g = 0; g < 8; ++g) {
    start[g] = (int32_t)acc;
    acc += sizes[g];
    if (acc > (int64_t)INT32_MAX / 4) return false;
  }
  start[8] = (int32_t)acc;
  return true;
}

__global__ void build_layout_kernel(LayoutParams p, float* __restrict__ pos, int32_t* __restrict__ chunk,
                                    int8_t* __restrict__ region) {
  const int32_t i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= p.start[8]) return;
  int g = 0;
#pragma unroll
  for (int k = 1; k < 8; ++k)
    if (i >= p.start[k]) g = k;
  const int32_t idx = i - p.start[g];

  const double T0 = (double)(p.n_ar + kArDmTimeOffset);
  const int fps = p.fps > 0 ? p.fps : 24;
  const double dt_v = __ddiv_rn(6.0, __ddiv_rn((double)fps, 4.0));
  const int32_t tau_a0 = p.tau_offset + p.clean_steps;
  const int32_t tau_p = p.tau_offset + (p.clean_steps > 0 ? p.clean_steps - 1 : 0);

  double t = 0.0, h = 0.0, w = 0.0;
  int32_t ch = -1;
  int8_t reg = (g == 0) ? 0 : (g <= 4 ? 1 : 2);
  if (g == 0) {  // AR: text, EOS, BOG -> (k, k, k)
    t = h = w = (double)idx;
  } else if (g == 1 || g == 5) {  // video: tau, view, y, x
    const int32_t per_view = p.gh * p.gw;
    const int32_t tps = p.views * per_view;
    const int32_t tau = p.tau_offset + (g == 5 ? p.clean_steps : 0) + idx / tps;
    const int32_t rem = idx % tps;
    const int32_t view = rem / per_view;
    const int32_t y = (rem % per_view) / p.gw;
    const int32_t x = rem % p.gw;
    t = __dadd_rn(T0, __dmul_rn((double)tau, dt_v));
    h = (double)y;
    w = (double)(x + view * p.gw);
    ch = tau;
  } else if (g == 2 || g == 6) {  // audio: counted over the clip, clean first
    const int64_t k = (g == 6 ? p.audio_clean : 0) + idx;
    const double dt_a = __ddiv_rn(6.0, (double)p.audio_rate);
    t = __dadd_rn(T0, __dmul_rn((double)k, dt_a));
    ch = p.tau_offset + (int32_t)((k * fps) / (4LL * p.audio_rate));
  } else if (g == 3 || g == 7) {  // actions: start at the first noisy video step
    const int64_t k = (g == 7 ? p.action_clean : 0) + idx;
    const double dt_act = __ddiv_rn(6.0, (double)p.action_hz);
    const double a0 = __dadd_rn(T0, __dmul_rn((double)tau_a0, dt_v));
    t = __dadd_rn(a0, __dmul_rn((double)k, dt_act));
    ch = tau_a0 + (int32_t)((k * fps) / (4LL * p.action_hz));
  } else {  // proprioception: at the last clean video step
    t = __dadd_rn(T0, __dmul_rn((double)tau_p, dt_v));
    ch = tau_p;
  }
  pos[3 * (int64_t)i + 0] = __double2float_rn(t);
  pos[3 * (int64_t)i + 1] = __double2float_rn(h);
  pos[3 * (int64_t)i + 2] = __double2float_rn(w);
  chunk[i] = ch;
  if (region) region[i] = reg;
}

// cs[r][i] = (cos theta, sin theta), theta = pos[r][axis(i)] * base^(-2i/hd),
// all in float64, rounded once to float32.
__global__ void mrope_table_kernel(const float* __restrict__ pos, int64_t n_rows, int32_t head_dim, int32_t s_t,
                                   int32_t s_h, double base, float2* __restrict__ cs) {
  const int32_t half = head_dim / 2;
  const int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= n_rows * half) return;
  const int64_t r = e / half;
  const int32_t i = (int32_t)(e % half);
  const int axis = i < s_t ? 0 : (i < s_t + s_h ? 1 : 2);
  const double expo = __ddiv_rn(__dmul_rn(-2.0, (double)i), (double)head_dim);
  const double inv_freq = pow(base, expo);
  const double theta = __dmul_rn((double)pos[3 * r + axis], inv_freq);
  double s, c;
  sincos(theta, &s, &c);
  cs[e] = make_float2(__double2float_rn(c), __double2float_rn(s));
}

}  // namespace
}  // namespace cosmot

extern "C" {

cosmot_status cosmot_layout_counts(const cosmot_layout_spec* spec, int32_t* n_tokens, int32_t* n_ar,
                                   int32_t* n_clean, int32_t* n_noisy) {
  if (!spec) return COSMOT_ERR_INVALID_ARG;
  int32_t st[9];
  if (!cosmot::group_bounds(*spec, st)) return COSMOT_ERR_INVALID_ARG;
  if (n_tokens) *n_tokens = st[8];
  if (n_ar) *n_ar = st[1];
  if (n_clean) *n_clean = st[5] - st[1];
  if (n_noisy) *n_noisy = st[8] - st[5];
  return COSMOT_OK;
}

cosmot_status cosmot_build_layout(const cosmot_layout_spec* spec, float* pos, int32_t* chunk, int8_t* region,
                                  cosmot_stream_t stream) {
  if (!spec || !pos || !chunk) return COSMOT_ERR_INVALID_ARG;
  cosmot::LayoutParams p{};
  if (!cosmot::group_bounds(*spec, p.start)) return COSMOT_ERR_INVALID_ARG;
  p.n_ar = p.start[1];
  p.views = spec->video_views;
  p.gh = spec->video_grid_h;
  p.gw = spec->video_grid_w;
  p.fps = spec->video_fps;
  p.clean_steps = spec->video_clean_steps;
  p.audio_clean = spec->audio_clean;
  p.audio_rate = spec->audio_rate;
  p.action_clean = spec->action_clean;
  p.action_hz = spec->action_hz;
  p.tau_offset = spec->tau_offset;
  const int n = p.start[8];
  const int threads = 256;
  cosmot::build_layout_kernel<<<(n + threads - 1) / threads, threads, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      p, pos, chunk, region);
  return cosmot::launch_status();
}

cosmot_status cosmot_mrope_table(const float* pos, int64_t n_rows, int32_t head_dim, const int32_t sections[3],
                                 double rope_base, float* cs, cosmot_stream_t stream) {
  if (!pos || !cs || !sections || n_rows <= 0 || head_dim <= 0 || (head_dim % 2) != 0 || rope_base <= 0.0)
    return COSMOT_ERR_INVALID_ARG;
  if (sections[0] < 0 || sections[1] < 0 || sections[2] < 0 ||
      sections[0] + sections[1] + sections[2] != head_dim / 2)
    return COSMOT_ERR_INVALID_ARG;
  const int64_t total = n_rows * (head_dim / 2);
  const int threads = 256;
  const int64_t blocks = (total + threads - 1) / threads;
  if (blocks > INT32_MAX) return COSMOT_ERR_UNSUPPORTED;
  cosmot::mrope_table_kernel<<<(unsigned)blocks, threads, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      pos, n_rows, head_dim, sections[0], sections[1], rope_base, reinterpret_cast<float2*>(cs));
  return cosmot::launch_status();
}

}  // extern "C"
