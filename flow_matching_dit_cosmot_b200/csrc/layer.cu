// One Mixture-of-Transformers layer forward plus the Euler sampler step.
//
// "Cosmos 3 方法原理全解" §3 (two weight sets, one shared attention under the
// MoT mask) and §7.2 (velocity output, x_next = x + (sigma_next - sigma) v).
// The driver only sequences kernels on the caller's stream; every step runs in
// the kernels of this library:
//   1 routed RMSNorm            h -> a                      (g1 of each set)
//   2 routed QKV GEMM + mRoPE    a -> qkv
//   3 MoT attention              qkv -> o
//   4 routed O GEMM + residual   o, h -> h1                 (h1 in float32)
//   5 routed RMSNorm             h1 -> a                     (g2)
//   6 routed gate/up + SiLU*mul  a -> u
//   7 routed down + residual     u, h1 -> h_out
//   8 RMSNorm (noisy rows)       h_out -> a (packed)         (g_fin)
//   9 velocity GEMM + Euler      a -> h[noisy rows] in place
//
// Cached prefix (seq.n_cached > 0): the first n_cached rows of every sequence
// keep the K and V that an earlier call left in the workspace's qkv region and
// are not recomputed; only rows [n_cached, N) go through the layer.  AR rows
// never read DM rows ("Cosmos 3 方法原理全解" §3), so a sampler reuses the AR
// K/V of its first step (§7.2: the Reasoner prompt is encoded once); a
// streaming rollout keeps AR + history-block K/V there ("流式生成如何工作":
// the key/value cache keeps attention information for the next prediction).
#include "cosmot_internal.h"

namespace cosmot {
namespace {

constexpr int kMaxBatch = 32;

struct WsLayout {
  size_t a, qkv, o, h1, u, part, part_bytes, total;
  int32_t kv_split;  // key split of a streaming-style call (queries = the noisy rows)
};

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

cosmot_status check_dims(const cosmot_dims* d) {
  if (!d) return COSMOT_ERR_INVALID_ARG;
  if (d->d_model <= 0 || d->d_model % 8 || d->ffn <= 0 || d->ffn % 8) return COSMOT_ERR_INVALID_ARG;
  if (d->n_heads <= 0 || d->n_kv_heads <= 0 || d->n_heads % d->n_kv_heads) return COSMOT_ERR_INVALID_ARG;
  if (d->head_dim != 64 && d->head_dim != 128) return COSMOT_ERR_UNSUPPORTED;
  if (d->rope_sections[0] < 0 || d->rope_sections[1] < 0 || d->rope_sections[2] < 0 ||
      d->rope_sections[0] + d->rope_sections[1] + d->rope_sections[2] != d->head_dim / 2)
    return COSMOT_ERR_INVALID_ARG;
  if (!(d->eps >= 0.f) || !(d->rope_base > 0.0)) return COSMOT_ERR_INVALID_ARG;
  return COSMOT_OK;
}

cosmot_status check_seq(const cosmot_seq_desc* s) {
  if (!s) return COSMOT_ERR_INVALID_ARG;
  if (s->n_ar < 0 || s->n_clean < 0 || s->n_noisy < 0 || s->n_ar + s->n_clean + s->n_noisy < 1)
    return COSMOT_ERR_INVALID_ARG;
  if (s->batch < 1 || s->batch > kMaxBatch) return COSMOT_ERR_UNSUPPORTED;
  if (s->mask_mode != COSMOT_MASK_FULL && s->mask_mode != COSMOT_MASK_BLOCK_CAUSAL) return COSMOT_ERR_INVALID_ARG;
  if (s->mask_mode == COSMOT_MASK_BLOCK_CAUSAL && !s->chunk) return COSMOT_ERR_INVALID_ARG;
  if (!s->rope_cs) return COSMOT_ERR_INVALID_ARG;
  if (s->n_cached < 0 || s->n_cached > s->n_ar + s->n_clean) return COSMOT_ERR_INVALID_ARG;
  return COSMOT_OK;
}

// Routed row segments over rows [lo, N) of each sequence: AR rows through set 0,
// DM rows through set 1; output row = input row + out_shift.
int make_segments(const cosmot_seq_desc& S, int64_t lo, int64_t out_shift, cosmot_segment* segs) {
  const int64_t N = (int64_t)S.n_ar + S.n_clean + S.n_noisy;
  int ns = 0;
  for (int b = 0; b < S.batch; ++b) {
    const int64_t r0 = b * N;
    if (lo < S.n_ar) segs[ns++] = cosmot_segment{r0 + lo, r0 + S.n_ar, r0 + lo + out_shift, 0, 0};
    const int64_t dm0 = lo > S.n_ar ? lo : S.n_ar;
    if (N > dm0) segs[ns++] = cosmot_segment{r0 + dm0, r0 + N, r0 + dm0 + out_shift, 1, 0};
  }
  return ns;
}

// The attention of a call that computes only the noisy rows of each sequence.
cosmot_attn_desc stream_attn_desc(const cosmot_dims& d, const cosmot_seq_desc& s) {
  const int64_t N = (int64_t)s.n_ar + s.n_clean + s.n_noisy;
  cosmot_attn_desc ad{};
  ad.n_q = s.n_noisy;
  ad.q_key_offset = N - s.n_noisy;
  ad.n_keys = N;
  ad.n_ar = s.n_ar;
  ad.n_heads = d.n_heads;
  ad.n_kv_heads = d.n_kv_heads;
  ad.head_dim = d.head_dim;
  ad.mask_mode = s.mask_mode;
  ad.chunk = s.chunk;
  ad.batch = s.batch;
  ad.flags = COSMOT_ATTN_NO_TILE_SKIP;
  ad.q_batch_stride = ad.kv_batch_stride = ad.o_batch_stride = N;
  return ad;
}

WsLayout ws_layout(const cosmot_dims& d, const cosmot_seq_desc& s) {
  const size_t rows = (size_t)s.batch * (size_t)(s.n_ar + s.n_clean + s.n_noisy);
  const size_t qkv_cols = (size_t)(d.n_heads + 2 * d.n_kv_heads) * d.head_dim;
  const size_t q_cols = (size_t)d.n_heads * d.head_dim;
  WsLayout w;
  size_t off = 0;
  // qkv first: cached K/V rows keep their addresses whatever the other sizes.
  w.qkv = off; off += align256(rows * qkv_cols * 2);
  w.a = off;   off += align256(rows * d.d_model * 2);
  w.o = off;   off += align256(rows * q_cols * 2);
  w.h1 = off;  off += align256(rows * d.d_model * 4);  // float32: the residual stream between the two halves
  w.u = off;   off += align256(rows * d.ffn * 2);
  // A call whose queries are the noisy rows alone behind a cached prefix of
  // AR and clean rows (a streaming step: the AR rows and the cache) may split
  // its keys across CTAs to fill the SMs; its float32 partials live here.
  cosmot_attn_desc ad = stream_attn_desc(d, s);
  w.kv_split = s.n_noisy > 0 && s.n_clean > 0 ? cosmot_attention_kv_split(&ad) : 1;
  w.part_bytes = 0;
  if (w.kv_split > 1) cosmot_attention_split_workspace(&ad, w.kv_split, &w.part_bytes);
  w.part = off;
  off += align256(w.part_bytes);
  w.total = off;
  return w;
}

}  // namespace
}  // namespace cosmot

extern "C" {

cosmot_status cosmot_layer_workspace_size(const cosmot_dims* dims, const cosmot_seq_desc* seq, size_t* bytes) {
  using namespace cosmot;
  if (!bytes) return COSMOT_ERR_INVALID_ARG;
  cosmot_status st = check_dims(dims);
  if (st != COSMOT_OK) return st;
  if (!seq || seq->batch < 1 || seq->batch > kMaxBatch || seq->n_ar < 0 || seq->n_clean < 0 || seq->n_noisy < 0)
    return COSMOT_ERR_INVALID_ARG;
  *bytes = ws_layout(*dims, *seq).total;
  return COSMOT_OK;
}

}  // extern "C"

namespace cosmot {
namespace {

// Records ev[i] (when the array and the entry are given) on the stream just
// before stage i starts.  A NULL entry leaves that boundary unmarked, so the
// kernels on either side keep their programmatic (overlapped) launch.
struct StageMarks {
  const cudaEvent_t* ev;
  cudaStream_t s;
  cosmot_status mark(int i) const {
    if (!ev || !ev[i]) return COSMOT_OK;
    return cudaEventRecord(ev[i], s) == cudaSuccess ? COSMOT_OK : COSMOT_ERR_CUDA;
  }
};

// Steps 1-7 for the rows [n_cached, N) of every sequence: x_in -> x_out.
// kv_cache (a stack's per-layer AR K/V store, or null): with n_cached == 0 the
// AR rows' q/k/v rows are copied there after the QKV projection; with
// n_cached > 0 they are copied back before the attention.
cosmot_status layer_body(const cosmot_dims& D, const cosmot_layer_weights* w, const cosmot_seq_desc& S,
                         const WsLayout& L, uint8_t* ws, const void* x_in, void* x_out, void* kv_cache,
                         cosmot_stream_t stream, const StageMarks& M) {
  cosmot_status st;
  const int64_t N = (int64_t)S.n_ar + S.n_clean + S.n_noisy;
  const int64_t d = D.d_model, F = D.ffn, hd = D.head_dim;
  const int64_t qc = (int64_t)D.n_heads * hd, kvc = (int64_t)D.n_kv_heads * hd, qkvc = qc + 2 * kvc;
  const int B = S.batch;
  void* a = ws + L.a;
  void* qkv = ws + L.qkv;
  void* o = ws + L.o;
  void* h1 = ws + L.h1;
  void* u = ws + L.u;

  // Row segments over the rows this call computes: AR rows through set 0, DM
  // rows through set 1; rows before n_cached keep their cached K/V.
  const int64_t c0 = S.n_cached;
  cosmot_segment segs[2 * kMaxBatch];
  const int ns = make_segments(S, c0, 0, segs);
  const cosmot_set_weights& R = w->set[0];
  const cosmot_set_weights& G = w->set[1];

  if ((st = M.mark(0)) != COSMOT_OK) return st;
  // 1. pre-attention norm
  st = cosmot_rmsnorm_routed(x_in, d, segs, ns, R.g1, G.g1, d, D.eps, a, d, stream);
  if (st != COSMOT_OK) return st;
  if ((st = M.mark(1)) != COSMOT_OK) return st;
  // 2. QKV projection with mRoPE on the Q and K heads
  cosmot_epilogue e{};
  e.kind = COSMOT_EPI_MROPE;
  e.head_dim = D.head_dim;
  e.rope_cols = qc + kvc;
  e.rope_cs = S.rope_cs;
  e.rope_period = N;
  st = cosmot_routed_linear(a, d, d, segs, ns, R.wqkv, G.wqkv, nullptr, nullptr, qkvc, qkv, qkvc, &e, stream);
  if (st != COSMOT_OK) return st;
  if (kv_cache && S.n_ar > 0) {
    // One strided copy per direction: the n_ar leading rows of every sequence.
    const size_t width = (size_t)S.n_ar * qkvc * 2, seq_pitch = (size_t)N * qkvc * 2;
    cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
    const cudaError_t ce = c0 == 0
        ? cudaMemcpy2DAsync(kv_cache, width, qkv, seq_pitch, width, B, cudaMemcpyDeviceToDevice, cs)
        : cudaMemcpy2DAsync(qkv, seq_pitch, kv_cache, width, width, B, cudaMemcpyDeviceToDevice, cs);
    if (ce != cudaSuccess) return COSMOT_ERR_CUDA;
  }
  if ((st = M.mark(2)) != COSMOT_OK) return st;
  // 3. attention
  cosmot_attn_desc ad{};
  ad.n_q = N - c0;
  ad.q_key_offset = c0;
  ad.n_keys = N;
  ad.n_ar = S.n_ar;
  ad.n_heads = D.n_heads;
  ad.n_kv_heads = D.n_kv_heads;
  ad.head_dim = D.head_dim;
  ad.mask_mode = S.mask_mode;
  ad.chunk = S.chunk;
  ad.batch = B;
  // A streaming step's queries are its newest block; its cache holds earlier
  // chunks only, so no key tile is hidden from every query.
  const bool noisy_only = c0 == (int64_t)S.n_ar + S.n_clean && S.n_noisy > 0;
  if (noisy_only) ad.flags = COSMOT_ATTN_NO_TILE_SKIP;
  ad.q_batch_stride = ad.kv_batch_stride = ad.o_batch_stride = N;
  uint16_t* qkvp = static_cast<uint16_t*>(qkv);
  // Few query tiles against a long cache (a streaming step: the cached prefix
  // holds clean or history rows): split the keys to fill the SMs.  A sampler
  // step that caches only the AR rows never splits, so it stays bit-identical
  // to a full recompute.
  if (noisy_only && S.n_clean > 0 && L.kv_split > 1)
    st = cosmot_mot_attention_split(&ad, qkvp + c0 * qkvc, qkvc, qkvp + qc, qkvp + qc + kvc, qkvc,
                                    static_cast<uint16_t*>(o) + c0 * qc, qc, L.kv_split, ws + L.part, L.part_bytes,
                                    stream);
  else
    st = cosmot_mot_attention(&ad, qkvp + c0 * qkvc, qkvc, qkvp + qc, qkvp + qc + kvc, qkvc,
                              static_cast<uint16_t*>(o) + c0 * qc, qc, stream);
  if (st != COSMOT_OK) return st;
  if ((st = M.mark(3)) != COSMOT_OK) return st;
  // 4. output projection + residual; h1 stays in float32 (it is read twice more:
  // by the pre-FFN norm and as the residual of the down projection)
  e = cosmot_epilogue{};
  e.kind = COSMOT_EPI_RESIDUAL;
  e.flags = COSMOT_EPI_OUT_F32;
  e.res = x_in;
  e.ld_res = d;
  st = cosmot_routed_linear(o, qc, qc, segs, ns, R.wo, G.wo, nullptr, nullptr, d, h1, d, &e, stream);
  if (st != COSMOT_OK) return st;
  if ((st = M.mark(4)) != COSMOT_OK) return st;
  // 5. pre-FFN norm
  st = rmsnorm_routed(h1, true, d, segs, ns, R.g2, G.g2, d, D.eps, a, d, stream);
  if (st != COSMOT_OK) return st;
  if ((st = M.mark(5)) != COSMOT_OK) return st;
  // 6. gate/up with SiLU * mul
  e = cosmot_epilogue{};
  e.kind = COSMOT_EPI_SILU_MUL;
  st = cosmot_routed_linear(a, d, d, segs, ns, R.wg, G.wg, R.wu, G.wu, F, u, F, &e, stream);
  if (st != COSMOT_OK) return st;
  if ((st = M.mark(6)) != COSMOT_OK) return st;
  // 7. down projection + residual
  e = cosmot_epilogue{};
  e.kind = COSMOT_EPI_RESIDUAL;
  e.flags = COSMOT_EPI_RES_F32;
  e.res = h1;
  e.ld_res = d;
  st = cosmot_routed_linear(u, F, F, segs, ns, R.wd, G.wd, nullptr, nullptr, d, x_out, d, &e, stream);
  if (st != COSMOT_OK) return st;
  return M.mark(7);
}

// Steps 8-9: final norm of the first nz noisy rows of h_last, velocity head,
// Euler step (or the guided step) into the same rows of `state`.
// io (or null): the float32 state and velocity output of the noisy rows, packed
// [batch][nz] (unguided steps only).
cosmot_status layer_head(const cosmot_dims& D, const cosmot_layer_weights* w, const cosmot_seq_desc& S,
                         const WsLayout& L, uint8_t* ws, const void* h_last, void* state, double sigma,
                         double sigma_next, cosmot_stream_t stream, const StageMarks& M, const double* guidance,
                         int64_t nz, const cosmot_step_io* io = nullptr) {
  cosmot_status st;
  const int64_t N = (int64_t)S.n_ar + S.n_clean + S.n_noisy;
  const int64_t d = D.d_model;
  const int B = S.batch;
  void* a = ws + L.a;
  void* u = ws + L.u;
  uint16_t* hb = static_cast<uint16_t*>(state);
  if (nz == 0) {
    if ((st = M.mark(8)) != COSMOT_OK) return st;
    return M.mark(9);
  }
  // 8. final norm of the noisy rows, packed into a
  cosmot_segment vs[kMaxBatch], ns_in[kMaxBatch];
  for (int b = 0; b < B; ++b) {
    const int64_t z0 = b * N + S.n_ar + S.n_clean;
    ns_in[b] = cosmot_segment{z0, z0 + nz, (int64_t)b * nz, 1, 0};
    vs[b] = cosmot_segment{(int64_t)b * nz, (int64_t)(b + 1) * nz, z0, 1, 0};
  }
  st = cosmot_rmsnorm_routed(h_last, d, ns_in, B, w->gfin, w->gfin, d, D.eps, a, d, stream);
  if (st != COSMOT_OK) return st;
  if ((st = M.mark(8)) != COSMOT_OK) return st;
  cosmot_epilogue e{};
  if (guidance) {
    // 9'. guided step: velocities of every sequence into the (now free) FFN
    // hidden region, then v_base + w (v_cond - v_base) and the Euler step for
    // each (conditioned, baseline) pair, written to both states of the pair.
    uint16_t* vbuf = static_cast<uint16_t*>(u);
    const cosmot_segment all{0, (int64_t)B * nz, 0, 1, 0};
    e.kind = COSMOT_EPI_NONE;
    st = cosmot_routed_linear(a, d, d, &all, 1, w->wvel, w->wvel, nullptr, nullptr, d, vbuf, d, &e, stream);
    if (st != COSMOT_OK) return st;
    for (int pr = 0; pr < B / 2; ++pr) {
      const int64_t zc = (int64_t)(2 * pr) * N + S.n_ar + S.n_clean;
      const int64_t zb = (int64_t)(2 * pr + 1) * N + S.n_ar + S.n_clean;
      st = cosmot_flow_cfg_euler_step(hb + zc * d, hb + zb * d, d, vbuf + (int64_t)(2 * pr) * nz * d,
                                      vbuf + (int64_t)(2 * pr + 1) * nz * d, d, nz, d, sigma, sigma_next, *guidance,
                                      stream);
      if (st != COSMOT_OK) return st;
    }
    return M.mark(9);
  }
  // 9. velocity head with the Euler step, in place on the noisy rows of the state
  e.kind = COSMOT_EPI_EULER;
  e.x = state;
  e.ld_x = d;
  e.dsigma = (float)(sigma_next - sigma);
  if (io) {  // the velocity GEMM's input rows are the packed noisy rows b * nz + i
    e.x_state = io->x_state;
    e.ld_state = io->ld_state;
    e.state_from_x = io->state_from_h;
    e.vel = io->vel;
    e.ld_vel = io->ld_vel;
  }
  st = cosmot_routed_linear(a, d, d, vs, B, w->wvel, w->wvel, nullptr, nullptr, d, hb, d, &e, stream);
  if (st != COSMOT_OK) return st;
  return M.mark(9);
}

cosmot_status check_io(const cosmot_step_io* io, const cosmot_dims& D, const double* guidance) {
  if (!io) return COSMOT_OK;
  if (guidance) return COSMOT_ERR_UNSUPPORTED;
  if (io->x_state && (!aligned16(io->x_state) || io->ld_state < D.d_model || io->ld_state % 8))
    return COSMOT_ERR_INVALID_ARG;
  if (io->vel && (!aligned16(io->vel) || io->ld_vel < D.d_model || io->ld_vel % 8)) return COSMOT_ERR_INVALID_ARG;
  return COSMOT_OK;
}

cosmot_status layer_forward_impl(const cosmot_dims* dims, const cosmot_layer_weights* w, const cosmot_seq_desc* seq,
                                 void* h, void* h_out, double sigma, double sigma_next, void* workspace,
                                 size_t workspace_bytes, cosmot_stream_t stream, const cudaEvent_t* events,
                                 const double* guidance = nullptr, const cosmot_step_io* io = nullptr) {
  const StageMarks M{events, reinterpret_cast<cudaStream_t>(stream)};
  cosmot_status st = check_dims(dims);
  if (st != COSMOT_OK) return st;
  st = check_seq(seq);
  if (st != COSMOT_OK) return st;
  st = check_io(io, *dims, guidance);
  if (st != COSMOT_OK) return st;
  if (!w || !h || !h_out || !workspace) return COSMOT_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return COSMOT_ERR_INVALID_ARG;
  const WsLayout L = ws_layout(*dims, *seq);
  if (workspace_bytes < L.total) return COSMOT_ERR_WORKSPACE;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  st = layer_body(*dims, w, *seq, L, ws, h, h_out, nullptr, stream, M);
  if (st != COSMOT_OK) return st;
  return layer_head(*dims, w, *seq, L, ws, h_out, h, sigma, sigma_next, stream, M, guidance, seq->n_noisy, io);
}

// Stack workspace: one layer's working set, a second hidden-state buffer for
// the layer outputs, and the AR rows' q/k/v of every layer.
struct StackWs {
  WsLayout layer;
  size_t tmp, cache, cache_per_layer, total;
};

StackWs stack_ws_layout(const cosmot_dims& d, int32_t n_layers, const cosmot_seq_desc& s) {
  StackWs w;
  w.layer = ws_layout(d, s);
  size_t off = w.layer.total;
  const size_t rows = (size_t)s.batch * (size_t)(s.n_ar + s.n_clean + s.n_noisy);
  const size_t qkv_cols = (size_t)(d.n_heads + 2 * d.n_kv_heads) * d.head_dim;
  w.tmp = off;
  off += align256(rows * d.d_model * 2);
  w.cache_per_layer = align256((size_t)s.batch * (size_t)s.n_ar * qkv_cols * 2);
  w.cache = off;
  off += (size_t)n_layers * w.cache_per_layer;
  w.total = off;
  return w;
}

constexpr int32_t kMaxLayers = 1024;

// Checks shared by the stack entries; fills W.
cosmot_status stack_check(const cosmot_dims* dims, const cosmot_layer_weights* layers, int32_t n_layers,
                          const cosmot_seq_desc* seq, const void* h, const void* h_out, const void* workspace,
                          size_t workspace_bytes, StackWs* W) {
  cosmot_status st = check_dims(dims);
  if (st != COSMOT_OK) return st;
  st = check_seq(seq);
  if (st != COSMOT_OK) return st;
  if (!layers || n_layers < 1 || n_layers > kMaxLayers || !h || !h_out || !workspace || h == h_out)
    return COSMOT_ERR_INVALID_ARG;
  // Clean DM rows read the noisy rows from the second layer on, so only the AR
  // prefix has step-invariant K/V in a stack.
  if (seq->n_cached != 0 && seq->n_cached != seq->n_ar) return COSMOT_ERR_UNSUPPORTED;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return COSMOT_ERR_INVALID_ARG;
  *W = stack_ws_layout(*dims, n_layers, *seq);
  if (workspace_bytes < W->total) return COSMOT_ERR_WORKSPACE;
  return COSMOT_OK;
}

// The layer bodies of a stack: h -> h_out.  events (or null): 8 per layer
// (layer l records events[8l + i] before its stage i, i < 7, and
// events[8l + 7] after its last stage).
cosmot_status stack_bodies(const cosmot_dims* dims, const cosmot_layer_weights* layers, int32_t n_layers,
                           const cosmot_seq_desc* seq, const StackWs& W, uint8_t* ws, const void* h, void* h_out,
                           cosmot_stream_t stream, const cudaEvent_t* events) {
  const cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  // Layer outputs alternate between h_out and the workspace buffer so that the
  // last one lands in h_out; the state h is only read until the final step.
  for (int32_t l = 0; l < n_layers; ++l) {
    void* out = ((n_layers - 1 - l) % 2 == 0) ? h_out : static_cast<void*>(ws + W.tmp);
    const void* in = l == 0 ? h : (((n_layers - l) % 2 == 0) ? h_out : static_cast<const void*>(ws + W.tmp));
    const StageMarks M{events ? events + 8 * l : nullptr, cs};
    cosmot_status st = layer_body(*dims, &layers[l], *seq, W.layer, ws, in, out,
                                  ws + W.cache + (size_t)l * W.cache_per_layer, stream, M);
    if (st != COSMOT_OK) return st;
  }
  return COSMOT_OK;
}

// events: as stack_bodies, then 2 for the head (before the velocity stage and
// after it).
cosmot_status stack_forward_impl(const cosmot_dims* dims, const cosmot_layer_weights* layers, int32_t n_layers,
                                 const cosmot_seq_desc* seq, void* h, void* h_out, double sigma, double sigma_next,
                                 void* workspace, size_t workspace_bytes, cosmot_stream_t stream,
                                 const cudaEvent_t* events, const cosmot_step_io* io = nullptr) {
  StackWs W;
  cosmot_status st = stack_check(dims, layers, n_layers, seq, h, h_out, workspace, workspace_bytes, &W);
  if (st != COSMOT_OK) return st;
  st = check_io(io, *dims, nullptr);
  if (st != COSMOT_OK) return st;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  st = stack_bodies(dims, layers, n_layers, seq, W, ws, h, h_out, stream, events);
  if (st != COSMOT_OK) return st;
  // the head's marks 8 and 9 land at events[8 n_layers] and [8 n_layers + 1]
  const StageMarks MH{events ? events + 8 * (n_layers - 1) : nullptr, reinterpret_cast<cudaStream_t>(stream)};
  return layer_head(*dims, &layers[n_layers - 1], *seq, W.layer, ws, h_out, h, sigma, sigma_next, stream, MH,
                    nullptr, seq->n_noisy, io);
}

// ---------------------------------------------------------------- row shards
// Rows [row0, row1) of one sequence held by one rank of a sequence-parallel
// layer, in local buffers indexed from row0 (global row row0 + i is local
// row i).  Routing follows the global index: AR rows through set 0.
int make_shard_segments(const cosmot_seq_desc& S, int64_t row0, int64_t row1, cosmot_segment* segs) {
  int ns = 0;
  const int64_t ar_end = row1 < S.n_ar ? row1 : S.n_ar;
  if (row0 < ar_end) segs[ns++] = cosmot_segment{0, ar_end - row0, 0, 0, 0};
  const int64_t dm0 = row0 > S.n_ar ? row0 : S.n_ar;
  if (row1 > dm0) segs[ns++] = cosmot_segment{dm0 - row0, row1 - row0, dm0 - row0, 1, 0};
  return ns;
}

cosmot_status check_shard(const cosmot_dims* dims, const cosmot_seq_desc* seq, int64_t row0, int64_t row1,
                          const void* workspace, size_t workspace_bytes, WsLayout* L) {
  cosmot_status st = check_dims(dims);
  if (st != COSMOT_OK) return st;
  st = check_seq(seq);
  if (st != COSMOT_OK) return st;
  const int64_t N = (int64_t)seq->n_ar + seq->n_clean + seq->n_noisy;
  if (seq->batch != 1 || seq->n_cached != 0) return COSMOT_ERR_UNSUPPORTED;
  if (row0 < 0 || row1 <= row0 || row1 > N || !workspace) return COSMOT_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return COSMOT_ERR_INVALID_ARG;
  cosmot_seq_desc local = *seq;  // a shard's working set is that of a row1 - row0 row sequence
  local.n_ar = (int32_t)(row1 - row0);
  local.n_clean = local.n_noisy = 0;
  *L = ws_layout(*dims, local);
  if (workspace_bytes < L->total) return COSMOT_ERR_WORKSPACE;
  return COSMOT_OK;
}

cosmot_status shard_pre(const cosmot_dims* dims, const cosmot_layer_weights* w, const cosmot_seq_desc* seq,
                        int64_t row0, int64_t row1, const void* h_local, void* qkv_local, void* workspace,
                        size_t workspace_bytes, cosmot_stream_t stream) {
  WsLayout L;
  cosmot_status st = check_shard(dims, seq, row0, row1, workspace, workspace_bytes, &L);
  if (st != COSMOT_OK) return st;
  if (!w || !h_local || !qkv_local) return COSMOT_ERR_INVALID_ARG;
  const cosmot_dims& D = *dims;
  const int64_t d = D.d_model, hd = D.head_dim;
  const int64_t qc = (int64_t)D.n_heads * hd, kvc = (int64_t)D.n_kv_heads * hd, qkvc = qc + 2 * kvc;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  cosmot_segment segs[2];
  const int ns = make_shard_segments(*seq, row0, row1, segs);
  const cosmot_set_weights& R = w->set[0];
  const cosmot_set_weights& G = w->set[1];
  st = cosmot_rmsnorm_routed(h_local, d, segs, ns, R.g1, G.g1, d, D.eps, ws + L.a, d, stream);
  if (st != COSMOT_OK) return st;
  cosmot_epilogue e{};
  e.kind = COSMOT_EPI_MROPE;
  e.head_dim = D.head_dim;
  e.rope_cols = qc + kvc;
  e.rope_cs = seq->rope_cs + row0 * hd;  // (cos, sin) pairs of the shard's global rows
  e.rope_period = 0;
  return cosmot_routed_linear(ws + L.a, d, d, segs, ns, R.wqkv, G.wqkv, nullptr, nullptr, qkvc, qkv_local, qkvc, &e,
                              stream);
}

cosmot_status shard_post(const cosmot_dims* dims, const cosmot_layer_weights* w, const cosmot_seq_desc* seq,
                         int64_t row0, int64_t row1, void* h_local, const void* o_local, void* h_out_local,
                         double sigma, double sigma_next, void* workspace, size_t workspace_bytes,
                         cosmot_stream_t stream) {
  WsLayout L;
  cosmot_status st = check_shard(dims, seq, row0, row1, workspace, workspace_bytes, &L);
  if (st != COSMOT_OK) return st;
  if (!w || !h_local || !o_local || !h_out_local || h_local == h_out_local) return COSMOT_ERR_INVALID_ARG;
  const cosmot_dims& D = *dims;
  const cosmot_seq_desc& S = *seq;
  const int64_t d = D.d_model, F = D.ffn, qc = (int64_t)D.n_heads * D.head_dim;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  cosmot_segment segs[2];
  const int ns = make_shard_segments(S, row0, row1, segs);
  const cosmot_set_weights& R = w->set[0];
  const cosmot_set_weights& G = w->set[1];
  cosmot_epilogue e{};
  e.kind = COSMOT_EPI_RESIDUAL;
  e.flags = COSMOT_EPI_OUT_F32;  // h1 in float32, as in layer_body
  e.res = h_local;
  e.ld_res = d;
  st = cosmot_routed_linear(o_local, qc, qc, segs, ns, R.wo, G.wo, nullptr, nullptr, d, ws + L.h1, d, &e, stream);
  if (st != COSMOT_OK) return st;
  st = rmsnorm_routed(ws + L.h1, true, d, segs, ns, R.g2, G.g2, d, D.eps, ws + L.a, d, stream);
  if (st != COSMOT_OK) return st;
  e = cosmot_epilogue{};
  e.kind = COSMOT_EPI_SILU_MUL;
  st = cosmot_routed_linear(ws + L.a, d, d, segs, ns, R.wg, G.wg, R.wu, G.wu, F, ws + L.u, F, &e, stream);
  if (st != COSMOT_OK) return st;
  e = cosmot_epilogue{};
  e.kind = COSMOT_EPI_RESIDUAL;
  e.flags = COSMOT_EPI_RES_F32;
  e.res = ws + L.h1;
  e.ld_res = d;
  st = cosmot_routed_linear(ws + L.u, F, F, segs, ns, R.wd, G.wd, nullptr, nullptr, d, h_out_local, d, &e, stream);
  if (st != COSMOT_OK) return st;
  // the noisy rows of the shard: final norm, velocity head and the Euler step
  const int64_t z0 = (int64_t)S.n_ar + S.n_clean;
  const int64_t nz0 = row0 > z0 ? row0 : z0;
  if (row1 <= nz0) return COSMOT_OK;
  const int64_t nz = row1 - nz0;
  const cosmot_segment ns_in{nz0 - row0, row1 - row0, 0, 1, 0};
  st = cosmot_rmsnorm_routed(h_out_local, d, &ns_in, 1, w->gfin, w->gfin, d, D.eps, ws + L.a, d, stream);
  if (st != COSMOT_OK) return st;
  const cosmot_segment vs{0, nz, nz0 - row0, 1, 0};
  e = cosmot_epilogue{};
  e.kind = COSMOT_EPI_EULER;
  e.x = h_local;
  e.ld_x = d;
  e.dsigma = (float)(sigma_next - sigma);
  return cosmot_routed_linear(ws + L.a, d, d, &vs, 1, w->wvel, w->wvel, nullptr, nullptr, d, h_local, d, &e, stream);
}

cosmot_status policy_step_impl(const cosmot_dims* dims, const cosmot_layer_weights* layers, int32_t n_layers,
                               const cosmot_seq_desc* seq, const cosmot_action_desc* act, void* h, void* h_out,
                               double sigma, double sigma_next, const double* guidance, void* workspace,
                               size_t workspace_bytes, cosmot_stream_t stream, const cudaEvent_t* events) {
  StackWs W;
  cosmot_status st = stack_check(dims, layers, n_layers, seq, h, h_out, workspace, workspace_bytes, &W);
  if (st != COSMOT_OK) return st;
  const cosmot_seq_desc& S = *seq;
  if (!act || !act->w_in || !act->w_out || !act->x || act->n_clean < 0 || act->n_noisy < 0 ||
      act->n_noisy > S.n_noisy || act->ld_x < act->action_dim)
    return COSMOT_ERR_INVALID_ARG;
  if (act->n_clean > 0 && (act->clean_row < S.n_ar || act->clean_row + act->n_clean > S.n_ar + S.n_clean))
    return COSMOT_ERR_INVALID_ARG;
  if (guidance) {
    if (S.batch < 2 || S.batch % 2) return COSMOT_ERR_INVALID_ARG;
    if ((int64_t)dims->ffn * (S.n_ar + S.n_clean + S.n_noisy) < (int64_t)dims->d_model * S.n_noisy)
      return COSMOT_ERR_UNSUPPORTED;
  }
  const int64_t N = (int64_t)S.n_ar + S.n_clean + S.n_noisy;
  const int64_t na = act->n_clean + act->n_noisy;
  const int32_t d = dims->d_model;
  // 0. action rows of the layer input: x W_in^T (clean conditions and the noisy
  // variable alike); the noisy action rows close the noisy group.
  cosmot_segment es[2 * kMaxBatch], hs[kMaxBatch];
  int ne = 0;
  for (int b = 0; b < S.batch; ++b) {
    if (act->n_clean > 0)
      es[ne++] = cosmot_segment{b * na, b * na + act->n_clean, b * N + act->clean_row, 0, 0};
    if (act->n_noisy > 0)
      es[ne++] = cosmot_segment{b * na + act->n_clean, (b + 1) * na, b * N + N - act->n_noisy, 0, 0};
    hs[b] = cosmot_segment{b * N + N - act->n_noisy, (b + 1) * N, b * na + act->n_clean, 0, 0};
  }
  if (ne > 0) {
    st = cosmot_action_embed(act->x, act->ld_x, es, ne, act->w_in, act->action_dim, d, h, d, stream);
    if (st != COSMOT_OK) return st;
  }
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  st = stack_bodies(dims, layers, n_layers, seq, W, ws, h, h_out, stream, events);
  if (st != COSMOT_OK) return st;
  const cosmot_layer_weights* last = &layers[n_layers - 1];
  // the noisy action rows: W_out velocity and the action's own Euler step (it
  // reads h^L and writes the action state only; timed with the final norm)
  if (act->n_noisy > 0) {
    st = cosmot_action_head(h_out, d, hs, S.batch, last->gfin, dims->eps, act->w_out, act->action_dim, d, act->x,
                            act->ld_x, act->sigma, act->sigma_next, guidance, stream);
    if (st != COSMOT_OK) return st;
  }
  // the other noisy rows: hidden-space velocity head and their Euler step
  const StageMarks MH{events ? events + 8 * (n_layers - 1) : nullptr, reinterpret_cast<cudaStream_t>(stream)};
  return layer_head(*dims, last, S, W.layer, ws, h_out, h, sigma, sigma_next, stream, MH, guidance,
                    S.n_noisy - act->n_noisy);
}

}  // namespace
}  // namespace cosmot

extern "C" {

cosmot_status cosmot_layer_forward(const cosmot_dims* dims, const cosmot_layer_weights* w,
                                   const cosmot_seq_desc* seq, void* h, void* h_out, double sigma,
                                   double sigma_next, void* workspace, size_t workspace_bytes,
                                   cosmot_stream_t stream) {
  return cosmot::layer_forward_impl(dims, w, seq, h, h_out, sigma, sigma_next, workspace, workspace_bytes, stream,
                                    nullptr);
}

cosmot_status cosmot_layer_forward_io(const cosmot_dims* dims, const cosmot_layer_weights* w,
                                      const cosmot_seq_desc* seq, void* h, void* h_out, double sigma,
                                      double sigma_next, const cosmot_step_io* io, void* workspace,
                                      size_t workspace_bytes, cosmot_stream_t stream) {
  return cosmot::layer_forward_impl(dims, w, seq, h, h_out, sigma, sigma_next, workspace, workspace_bytes, stream,
                                    nullptr, nullptr, io);
}

cosmot_status cosmot_layer_forward_cfg(const cosmot_dims* dims, const cosmot_layer_weights* w,
                                       const cosmot_seq_desc* seq, void* h, void* h_out, double sigma,
                                       double sigma_next, double guidance, void* workspace, size_t workspace_bytes,
                                       cosmot_stream_t stream) {
  if (!seq || !dims || seq->batch < 2 || seq->batch % 2) return COSMOT_ERR_INVALID_ARG;
  // the velocities of all sequences reuse the FFN hidden region of the workspace
  if ((int64_t)dims->ffn * (seq->n_ar + seq->n_clean + seq->n_noisy) < (int64_t)dims->d_model * seq->n_noisy)
    return COSMOT_ERR_UNSUPPORTED;
  return cosmot::layer_forward_impl(dims, w, seq, h, h_out, sigma, sigma_next, workspace, workspace_bytes, stream,
                                    nullptr, &guidance);
}

cosmot_status cosmot_layer_commit_kv(const cosmot_dims* dims, const cosmot_layer_weights* w,
                                     const cosmot_seq_desc* seq, const void* h, int64_t dst_row, void* workspace,
                                     size_t workspace_bytes, cosmot_stream_t stream) {
  using namespace cosmot;
  cosmot_status st = check_dims(dims);
  if (st != COSMOT_OK) return st;
  st = check_seq(seq);
  if (st != COSMOT_OK) return st;
  if (!w || !h || !workspace) return COSMOT_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return COSMOT_ERR_INVALID_ARG;
  const WsLayout L = ws_layout(*dims, *seq);
  if (workspace_bytes < L.total) return COSMOT_ERR_WORKSPACE;
  const cosmot_dims& D = *dims;
  const cosmot_seq_desc& S = *seq;
  const int64_t N = (int64_t)S.n_ar + S.n_clean + S.n_noisy;
  const int64_t c0 = S.n_cached;
  if (dst_row < 0 || dst_row + (N - c0) > N) return COSMOT_ERR_INVALID_ARG;
  const int64_t d = D.d_model, hd = D.head_dim;
  const int64_t qc = (int64_t)D.n_heads * hd, kvc = (int64_t)D.n_kv_heads * hd, qkvc = qc + 2 * kvc;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  cosmot_segment segs[2 * kMaxBatch], dst[2 * kMaxBatch];
  const int ns = make_segments(S, c0, 0, segs);
  make_segments(S, c0, dst_row - c0, dst);
  const cosmot_set_weights& R = w->set[0];
  const cosmot_set_weights& G = w->set[1];
  st = cosmot_rmsnorm_routed(h, d, segs, ns, R.g1, G.g1, d, D.eps, ws + L.a, d, stream);
  if (st != COSMOT_OK) return st;
  cosmot_epilogue e{};
  e.kind = COSMOT_EPI_MROPE;
  e.head_dim = D.head_dim;
  e.rope_cols = qc + kvc;
  e.rope_cs = S.rope_cs;
  e.rope_period = N;
  return cosmot_routed_linear(ws + L.a, d, d, dst, ns, R.wqkv, G.wqkv, nullptr, nullptr, qkvc, ws + L.qkv, qkvc, &e,
                              stream);
}

cosmot_status cosmot_stack_workspace_size(const cosmot_dims* dims, int32_t n_layers, const cosmot_seq_desc* seq,
                                          size_t* bytes) {
  using namespace cosmot;
  if (!bytes) return COSMOT_ERR_INVALID_ARG;
  cosmot_status st = check_dims(dims);
  if (st != COSMOT_OK) return st;
  if (!seq || seq->batch < 1 || seq->batch > kMaxBatch || seq->n_ar < 0 || seq->n_clean < 0 || seq->n_noisy < 0 ||
      n_layers < 1 || n_layers > kMaxLayers)
    return COSMOT_ERR_INVALID_ARG;
  *bytes = stack_ws_layout(*dims, n_layers, *seq).total;
  return COSMOT_OK;
}

cosmot_status cosmot_stack_forward(const cosmot_dims* dims, const cosmot_layer_weights* layers, int32_t n_layers,
                                   const cosmot_seq_desc* seq, void* h, void* h_out, double sigma, double sigma_next,
                                   void* workspace, size_t workspace_bytes, cosmot_stream_t stream) {
  return cosmot::stack_forward_impl(dims, layers, n_layers, seq, h, h_out, sigma, sigma_next, workspace,
                                    workspace_bytes, stream, nullptr);
}

cosmot_status cosmot_stack_forward_io(const cosmot_dims* dims, const cosmot_layer_weights* layers, int32_t n_layers,
                                      const cosmot_seq_desc* seq, void* h, void* h_out, double sigma,
                                      double sigma_next, const cosmot_step_io* io, void* workspace,
                                      size_t workspace_bytes, cosmot_stream_t stream) {
  return cosmot::stack_forward_impl(dims, layers, n_layers, seq, h, h_out, sigma, sigma_next, workspace,
                                    workspace_bytes, stream, nullptr, io);
}

cosmot_status cosmot_policy_step(const cosmot_dims* dims, const cosmot_layer_weights* layers, int32_t n_layers,
                                 const cosmot_seq_desc* seq, const cosmot_action_desc* act, void* h, void* h_out,
                                 double sigma, double sigma_next, const double* guidance, void* workspace,
                                 size_t workspace_bytes, cosmot_stream_t stream, void* const* stage_events,
                                 int32_t n_events) {
  if (stage_events && (n_layers < 1 || n_layers > cosmot::kMaxLayers || n_events != 8 * n_layers + 2))
    return COSMOT_ERR_INVALID_ARG;
  return cosmot::policy_step_impl(dims, layers, n_layers, seq, act, h, h_out, sigma, sigma_next, guidance, workspace,
                                  workspace_bytes, stream, reinterpret_cast<const cudaEvent_t*>(stage_events));
}

cosmot_status cosmot_shard_workspace_size(const cosmot_dims* dims, int64_t rows, size_t* bytes) {
  using namespace cosmot;
  if (!bytes || rows < 1 || rows > INT32_MAX) return COSMOT_ERR_INVALID_ARG;
  cosmot_status st = check_dims(dims);
  if (st != COSMOT_OK) return st;
  cosmot_seq_desc local{};
  local.n_ar = (int32_t)rows;
  local.batch = 1;
  *bytes = ws_layout(*dims, local).total;
  return COSMOT_OK;
}

cosmot_status cosmot_layer_shard_pre(const cosmot_dims* dims, const cosmot_layer_weights* w,
                                     const cosmot_seq_desc* seq, int64_t row0, int64_t row1, const void* h_local,
                                     void* qkv_local, void* workspace, size_t workspace_bytes,
                                     cosmot_stream_t stream) {
  return cosmot::shard_pre(dims, w, seq, row0, row1, h_local, qkv_local, workspace, workspace_bytes, stream);
}

cosmot_status cosmot_layer_shard_post(const cosmot_dims* dims, const cosmot_layer_weights* w,
                                      const cosmot_seq_desc* seq, int64_t row0, int64_t row1, void* h_local,
                                      const void* o_local, void* h_out_local, double sigma, double sigma_next,
                                      void* workspace, size_t workspace_bytes, cosmot_stream_t stream) {
  return cosmot::shard_post(dims, w, seq, row0, row1, h_local, o_local, h_out_local, sigma, sigma_next, workspace,
                            workspace_bytes, stream);
}

cosmot_status cosmot_copy_columns(const void* src, int64_t ld_src, void* dst, int64_t ld_dst, int64_t rows,
                                  int64_t n_cols, cosmot_stream_t stream) {
  if (!src || !dst || rows < 0 || n_cols < 0 || ld_src < n_cols || ld_dst < n_cols) return COSMOT_ERR_INVALID_ARG;
  if (rows == 0 || n_cols == 0) return COSMOT_OK;
  const cudaError_t e = cudaMemcpy2DAsync(dst, (size_t)ld_dst * 2, src, (size_t)ld_src * 2, (size_t)n_cols * 2,
                                          (size_t)rows, cudaMemcpyDeviceToDevice,
                                          reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? COSMOT_OK : COSMOT_ERR_CUDA;
}

cosmot_status cosmot_stack_forward_timed(const cosmot_dims* dims, const cosmot_layer_weights* layers,
                                         int32_t n_layers, const cosmot_seq_desc* seq, void* h, void* h_out,
                                         double sigma, double sigma_next, void* workspace, size_t workspace_bytes,
                                         cosmot_stream_t stream, void* const* stage_events, int32_t n_events,
                                         const cosmot_step_io* io) {
  if (!stage_events || n_layers < 1 || n_layers > cosmot::kMaxLayers || n_events != 8 * n_layers + 2)
    return COSMOT_ERR_INVALID_ARG;
  return cosmot::stack_forward_impl(dims, layers, n_layers, seq, h, h_out, sigma, sigma_next, workspace,
                                    workspace_bytes, stream, reinterpret_cast<const cudaEvent_t*>(stage_events), io);
}

cosmot_status cosmot_layer_forward_timed(const cosmot_dims* dims, const cosmot_layer_weights* w,
                                         const cosmot_seq_desc* seq, void* h, void* h_out, double sigma,
                                         double sigma_next, void* workspace, size_t workspace_bytes,
                                         cosmot_stream_t stream, void* const* stage_events, int32_t n_events,
                                         const double* guidance, const cosmot_step_io* io) {
  if (!stage_events || n_events != COSMOT_LAYER_STAGES + 1) return COSMOT_ERR_INVALID_ARG;
  if (guidance) {
    if (!seq || !dims || seq->batch < 2 || seq->batch % 2) return COSMOT_ERR_INVALID_ARG;
    if ((int64_t)dims->ffn * (seq->n_ar + seq->n_clean + seq->n_noisy) < (int64_t)dims->d_model * seq->n_noisy)
      return COSMOT_ERR_UNSUPPORTED;
  }
  return cosmot::layer_forward_impl(dims, w, seq, h, h_out, sigma, sigma_next, workspace, workspace_bytes, stream,
                                    reinterpret_cast<const cudaEvent_t*>(stage_events), guidance, io);
}

}  // extern "C"
