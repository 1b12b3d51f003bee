/*
 * libcosmot — the Cosmos 3 Mixture-of-Transformers (MoT) layer hot path on
 * NVIDIA B200 (sm_100a).  C ABI: plain pointers, sizes and small structs.
 *
 * What is computed, and where the pages define it:
 *   "Cosmos 3 方法原理全解" §2  packed sequence [AR..., EOS, BOG, DM clean..., DM noisy...]
 *   "Cosmos 3 方法原理全解" §3  two weight sets (Reasoner for AR rows, Generator for DM rows),
 *                               O_AR = Attn_causal(Q_AR,K_AR,V_AR),
 *                               O_DM = Attn_full(Q_DM,[K_AR;K_DM],[V_AR;V_DM])
 *   "Cosmos 3 方法原理全解" §5  unified 3D mRoPE (t,h,w), dt = 6/TPS, AR->DM offset 15000
 *   "Cosmos 3 方法原理全解" §7.2 Euler step x_next = x + (sigma_next - sigma) * v
 *   "NVIDIA 发布 Cosmos 3 系列四个开放权重世界模型", "流式生成如何工作":
 *                               time-causal block attention with a key/value cache
 *
 * Conventions for every entry point:
 *   - All compute runs asynchronously on `stream` (a cudaStream_t; NULL = legacy
 *     default stream).  Every pointer marked "device" must be device memory
 *     reachable from the current device.
 *   - The caller owns every buffer.  The library allocates no device memory on any
 *     path; scratch comes from the caller (see cosmot_layer_workspace_size).
 *   - Element types: activations and weights are bf16 (stored as 16-bit words),
 *     row-major.  Weights are [out_features, in_features] ("K-major").  Leading
 *     dimensions (`ld*`) count elements, not bytes.
 *   - Alignment: every bf16 matrix base pointer must be 16-byte aligned and every
 *     leading dimension a multiple of 8 elements (the 16-byte TMA stride rule).
 *   - Argument errors are reported synchronously as COSMOT_ERR_INVALID_ARG (or
 *     COSMOT_ERR_UNSUPPORTED for shapes the library does not handle) and nothing is
 *     launched.  Launch failures return COSMOT_ERR_CUDA.
 *   - Device-side failures (a bounded wait that ran out, recorded instead of
 *     hanging) are latched into a device status word; read and clear it with
 *     cosmot_get_device_status.
 *   - Results are deterministic: no atomics in any reduction, no split-K.
 */
#ifndef COSMOT_H_
#define COSMOT_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define COSMOT_API __attribute__((visibility("default")))
#else
#define COSMOT_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* cosmot_stream_t; /* same type as cudaStream_t */

typedef int32_t cosmot_status;
enum {
  COSMOT_OK = 0,
  COSMOT_ERR_INVALID_ARG = 1,
  COSMOT_ERR_UNSUPPORTED = 2,
  COSMOT_ERR_CUDA = 3,
  COSMOT_ERR_TIMEOUT = 4,
  COSMOT_ERR_WORKSPACE = 5,
  COSMOT_ERR_BOUNDS = 6     /* debug build only: a device-side store index check failed (store skipped) */
};

/* Human-readable name of a status code (static string, never NULL). */
COSMOT_API const char* cosmot_status_string(cosmot_status s);

/* Library version as MAJOR*10000 + MINOR*100 + PATCH. */
COSMOT_API int32_t cosmot_version(void);

/*
 * Reads the device status word on `stream` (synchronising that stream) into *out
 * and clears it.  COSMOT_OK if no kernel recorded a failure since the last call.
 * `where_out` (may be NULL) receives an internal site code of the first failure.
 */
COSMOT_API cosmot_status cosmot_get_device_status(cosmot_stream_t stream, cosmot_status* out, int32_t* where_out);

/* Site code that cosmot_selftest_wait_timeout latches with its timeout. */
#define COSMOT_SITE_SELFTEST 900
/* Site code that cosmot_selftest_bounds_check latches (debug build). */
#define COSMOT_SITE_SELFTEST_BOUNDS 901

/*
 * 1 in the debug build of the library (libcosmot_debug.so, compiled with
 * COSMOT_DEBUG_CHECKS), 0 in the release build.  The debug build checks the
 * index of every global store its kernels make (GEMM, attention, norm and
 * Euler outputs) against the extent the host side derived for that output; a
 * failed check latches COSMOT_ERR_BOUNDS with the kernel's site code into the
 * device status word and skips the store (no trap).  Results are otherwise
 * identical to the release build's.
 */
COSMOT_API int32_t cosmot_debug_checks(void);

/*
 * Test-only check of the debug build's store checks: one thread makes a
 * checked store whose index is one past the extent it states (the index still
 * lies inside the kernel's own buffer), so the check fails, latches
 * COSMOT_ERR_BOUNDS at COSMOT_SITE_SELFTEST_BOUNDS and skips the store.  The
 * release build returns COSMOT_ERR_UNSUPPORTED and launches nothing.
 */
COSMOT_API cosmot_status cosmot_selftest_bounds_check(cosmot_stream_t stream);

/*
 * Test-only check of the failure path.  One CTA whose consumer thread waits on
 * an mbarrier that its producer warp never arrives on, through the same bounded
 * wait every kernel of the library uses.  The wait gives up after its bound
 * (one second), latches COSMOT_ERR_TIMEOUT with site COSMOT_SITE_SELFTEST into
 * the device status word, and the kernel returns: nothing faults or traps, and
 * the context stays usable.  Returns the launch status; read the outcome with
 * cosmot_get_device_status.  If the status word already holds a failure, the
 * wait gives up at once and leaves that failure in place.
 */
COSMOT_API cosmot_status cosmot_selftest_wait_timeout(cosmot_stream_t stream);

/* ===================================================================== layout */

/*
 * Contents of one packed sequence ("Cosmos 3 方法原理全解" §2): n_text AR text
 * tokens, then EOS and BOG (both AR), then the clean DM group and the noisy DM
 * group, each ordered vision, audio, action.  Video: `video_views` views side by
 * side along w, grid_h x grid_w tokens per view per latent step, clean steps
 * first, then noisy steps, on one time axis starting at latent step tau_offset.
 * Proprioception tokens are clean and sit with the clean actions.
 */
typedef struct {
  int32_t n_text;
  int32_t video_views, video_grid_h, video_grid_w, video_fps;
  int32_t video_clean_steps, video_noisy_steps;
  int32_t audio_clean, audio_noisy, audio_rate;   /* audio_rate: tokens per second */
  int32_t action_clean, action_noisy, action_hz;
  int32_t proprio;
  int32_t tau_offset;                             /* first video latent step */
} cosmot_layout_spec;

/* Token counts of a layout (host only, no launch). */
COSMOT_API cosmot_status cosmot_layout_counts(const cosmot_layout_spec* spec, int32_t* n_tokens, int32_t* n_ar,
                                   int32_t* n_clean, int32_t* n_noisy);

/*
 * Builds the per-token mRoPE coordinates and block ids of one packed sequence
 * ("Cosmos 3 方法原理全解" §5).  Device outputs, N = n_tokens:
 *   pos    float32 [N][3]  (t, h, w).  Each value is computed in float64 and
 *                          rounded once to float32:
 *                          AR token k -> (k, k, k); T0 = n_ar + 15000;
 *                          video (step tau, view v, y, x) -> (T0 + tau*dt_v, y, x + v*grid_w),
 *                          dt_v = 6 / (fps/4); audio k -> (T0 + k*6/rate, 0, 0);
 *                          action k -> ((T0 + tau_a0*dt_v) + k*6/hz, 0, 0), tau_a0 =
 *                          first noisy step; proprio -> (T0 + tau_last_clean*dt_v, 0, 0).
 *   chunk  int32 [N]       -1 on AR rows, else the latent step of the token.
 *   region int8  [N]       0 AR, 1 clean DM, 2 noisy DM (may be NULL).
 */
COSMOT_API cosmot_status cosmot_build_layout(const cosmot_layout_spec* spec, float* pos, int32_t* chunk, int8_t* region,
                                  cosmot_stream_t stream);

/*
 * cos/sin table of the unified 3D mRoPE for rows with coordinates `pos`
 * ([n_rows][3] float32, device).  Pair i in [0, head_dim/2) takes its angle from
 * axis t, h or w by contiguous sections (sections[0] pairs on t, then
 * sections[1] on h, then sections[2] on w; their sum is head_dim/2):
 * theta = pos[axis] * base^(-2i/head_dim), evaluated in float64.
 * Output cs float32 [n_rows][head_dim/2][2] = (cos theta, sin theta), device.
 */
COSMOT_API cosmot_status cosmot_mrope_table(const float* pos, int64_t n_rows, int32_t head_dim, const int32_t sections[3],
                                 double rope_base, float* cs, cosmot_stream_t stream);

/* ===================================================================== kernels */

/* Row segment of a routed operation: rows [row_begin, row_end) of the input go
 * through weight set `weight_set` (0 = Reasoner, 1 = Generator); input row r
 * writes output row out_row + (r - row_begin). */
typedef struct {
  int64_t row_begin;
  int64_t row_end;
  int64_t out_row;
  int32_t weight_set;
  int32_t reserved;
} cosmot_segment;

/*
 * Routed RMSNorm ("Cosmos 3 方法原理全解" §3: each room has its own norm).
 * out[o] = bf16( h[r] * g_s / sqrt(mean(h[r]^2) + eps) ), fp32 arithmetic.
 * h: [rows, d] (ld_h), out: [rows, d] (ld_out), g0/g1: [d] gains of the two sets.
 */
COSMOT_API cosmot_status cosmot_rmsnorm_routed(const void* h, int64_t ld_h, const cosmot_segment* segs, int32_t n_segs,
                                    const void* g0, const void* g1, int64_t d, float eps, void* out,
                                    int64_t ld_out, cosmot_stream_t stream);

/* Epilogues of cosmot_routed_linear. */
enum {
  COSMOT_EPI_NONE = 0,      /* out = bf16(acc) */
  COSMOT_EPI_RESIDUAL = 1,  /* out = bf16(acc + res); res may alias out */
  COSMOT_EPI_SILU_MUL = 2,  /* out[:, j] = bf16(silu(a.Wg_j) * (a.Wu_j)); W = gate, W_up = up */
  COSMOT_EPI_MROPE = 3,     /* QKV projection: heads in columns [0, rope_cols) rotated by mRoPE */
  COSMOT_EPI_EULER = 4      /* out = bf16(x + dsigma * acc); x may alias out; see x_state below */
};

/* cosmot_epilogue.flags (RESIDUAL only): float32 instead of bf16 for the
 * output and/or the residual, so that a residual stream can stay in float32. */
#define COSMOT_EPI_OUT_F32 1
#define COSMOT_EPI_RES_F32 2

typedef struct {
  int32_t kind;
  int32_t head_dim;        /* MROPE: head width (64 or 128) */
  int64_t rope_cols;       /* MROPE: number of leading output columns rotated (Q and K heads) */
  const float* rope_cs;    /* MROPE: table of cosmot_mrope_table, row = input row mod rope_period */
  int64_t rope_period;     /* MROPE: rows per sequence in the table (0 = no wrap) */
  const void* res;         /* RESIDUAL: [rows, n_out] bf16, indexed by output row */
  int64_t ld_res;
  const void* x;           /* EULER: [rows, n_out] bf16, indexed by output row */
  int64_t ld_x;
  float dsigma;            /* EULER: sigma_next - sigma */
  float reserved;
  /* EULER, optional float32 sampler state: x_state [rows, ld_state] float32,
   * indexed by INPUT row.  When non-NULL, x is read from x_state (or from `x`
   * when state_from_x = 1), x' = x + dsigma * acc is written back to x_state
   * in float32, and bf16(x') still goes to `out`. */
  float* x_state;
  int64_t ld_state;
  void* vel;               /* EULER, optional: [rows, ld_vel] bf16, indexed by input row, receives bf16(acc) */
  int64_t ld_vel;
  int32_t state_from_x;
  int32_t flags;           /* COSMOT_EPI_OUT_F32 | COSMOT_EPI_RES_F32 (RESIDUAL only), else 0 */
} cosmot_epilogue;

/*
 * Routed projection on the 5th-generation tensor cores (tcgen05, fp32 TMEM
 * accumulation): for every segment s and input row r in it,
 *     acc[r, j] = sum_k a[r, k] * W_{set(s)}[j, k],   j in [0, n_out)
 * then the epilogue writes output row out_row(s) + (r - row_begin).
 *   a      device bf16 [*, k], ld_a            (rows addressed by the segments)
 *   w0/w1  device bf16 [n_out, k] (Reasoner / Generator); a set no segment uses
 *          may be NULL
 *   w0_up/w1_up  SILU_MUL only: the up projections, same shape; NULL otherwise
 *   out    device bf16 [*, n_out], ld_out
 * Requires k % 8 == 0, n_out % 8 == 0, ld_a/ld_out % 8 == 0; MROPE needs
 * head_dim in {64, 128} and rope_cols a multiple of head_dim; 1 <= n_segs <= 64.
 * With COSMOT_EPI_OUT_F32 (RESIDUAL) `out` is float32 [*, ld_out]; with
 * COSMOT_EPI_RES_F32 `res` is float32 [*, ld_res]; both 16-byte aligned.
 */
COSMOT_API cosmot_status cosmot_routed_linear(const void* a, int64_t ld_a, int64_t k, const cosmot_segment* segs,
                                   int32_t n_segs, const void* w0, const void* w1, const void* w0_up,
                                   const void* w1_up, int64_t n_out, void* out, int64_t ld_out,
                                   const cosmot_epilogue* epi, cosmot_stream_t stream);

/*
 * Standalone mRoPE ("Cosmos 3 方法原理全解" §5), in place on bf16 rows:
 * for each row r and head, pairs (i, i + head_dim/2) rotate by theta(r, i):
 *     x_i' = x_i cos - x_{i+hd/2} sin,   x_{i+hd/2}' = x_{i+hd/2} cos + x_i sin
 * q: [n_rows, ld_q] with n_q_heads heads from column 0; k likewise (may be NULL).
 * cs: table of cosmot_mrope_table for the same rows.
 */
COSMOT_API cosmot_status cosmot_mrope_apply(void* q, int64_t ld_q, int32_t n_q_heads, void* k, int64_t ld_k,
                                 int32_t n_k_heads, int64_t n_rows, int32_t head_dim, const float* cs,
                                 cosmot_stream_t stream);

/* Key visibility of cosmot_mot_attention. */
enum { COSMOT_MASK_FULL = 0, COSMOT_MASK_BLOCK_CAUSAL = 1 };

typedef struct {
  int64_t n_q;          /* query rows */
  int64_t q_key_offset; /* query row i is key row q_key_offset + i */
  int64_t n_keys;       /* key rows: [0, n_ar) AR, the rest DM */
  int64_t n_ar;
  int32_t n_heads, n_kv_heads, head_dim;
  int32_t mask_mode;    /* COSMOT_MASK_* */
  const int32_t* chunk; /* BLOCK_CAUSAL: device int32 [n_keys] latent step of each key row */
  int32_t batch;        /* independent sequences */
  int32_t flags;        /* COSMOT_ATTN_* hints, 0 = none */
  int64_t q_batch_stride, kv_batch_stride, o_batch_stride; /* rows between sequences */
  float softmax_scale;  /* 0 = 1/sqrt(head_dim) */
  float reserved2;
} cosmot_attn_desc;

/* BLOCK_CAUSAL hint: no DM query row can have a fully hidden key tile (a
 * streaming step, whose cache holds only earlier chunks), so the kernel need
 * not look for tiles to skip.  Results are the same either way: element masks
 * still apply; a wrong hint only costs the skipped work. */
#define COSMOT_ATTN_NO_TILE_SKIP 1

/*
 * MoT attention ("Cosmos 3 方法原理全解" §3 equations; block-causal variant from
 * "流式生成如何工作").  Per head h (kv head h / (n_heads/n_kv_heads)):
 *     o_i = sum_{j visible to i} softmax_j(q_i . k_j * scale) v_j
 * visible: AR query i sees AR keys j <= i; a DM query sees every AR key and, in
 * FULL mode, every DM key; in BLOCK_CAUSAL mode the DM keys with
 * chunk[j] <= chunk[query].  q: [n_q, ld_q] (heads of head_dim from column 0),
 * k, v: [n_keys, ld_kv], o: [n_q, ld_o], all bf16 device.  head_dim 128 or 64.
 * Key tiles that none of a CTA's query rows sees are skipped: causally hidden
 * AR tiles always, and in BLOCK_CAUSAL mode DM tiles of later chunks (unless
 * COSMOT_ATTN_NO_TILE_SKIP); block-causal calls need ceil(n_keys / 128) <= 65536.
 */
COSMOT_API cosmot_status cosmot_mot_attention(const cosmot_attn_desc* desc, const void* q, int64_t ld_q, const void* k,
                                   const void* v, int64_t ld_kv, void* o, int64_t ld_o, cosmot_stream_t stream);

/*
 * cosmot_mot_attention with the keys of every DM query item split kv_split
 * ways (1..8) across CTAs: split s of an item visits key tiles [s n_kt /
 * kv_split, (s + 1) n_kt / kv_split) of n_kt = ceil(n_keys / 128), writes its
 * O / l in float32 to the workspace with its running max m_s and sum l_s, and
 * a second kernel combines them in split order: O = sum_s w_s O_s / sum_s w_s,
 * w_s = l_s 2^(m_s - max m).  Fills the SMs when a call has few query tiles (a
 * streaming step's single block); AR query items are not split.  Results equal
 * cosmot_mot_attention's up to the summation order of the softmax sums.
 * Requires no tile skipping (FULL mask, or COSMOT_ATTN_NO_TILE_SKIP) and
 * kv_split <= n_kt (else UNSUPPORTED / INVALID_ARG); workspace: device, 256-byte
 * aligned, cosmot_attention_split_workspace bytes (WORKSPACE if shorter).
 */
COSMOT_API cosmot_status cosmot_mot_attention_split(const cosmot_attn_desc* desc, const void* q, int64_t ld_q,
                                                    const void* k, const void* v, int64_t ld_kv, void* o,
                                                    int64_t ld_o, int32_t kv_split, void* workspace,
                                                    size_t workspace_bytes, cosmot_stream_t stream);
/* Workspace bytes of cosmot_mot_attention_split (0 for kv_split = 1); host only. */
COSMOT_API cosmot_status cosmot_attention_split_workspace(const cosmot_attn_desc* desc, int32_t kv_split,
                                                          size_t* bytes);
/* The key split the layer uses for this call shape: among 1..4 (with at least
 * 8 key tiles a split), the one that keeps the SMs busiest over the waves of
 * DM work items, taken only when it beats no split by more than 5 points.  It
 * depends on the batch, heads, DM query tiles, key count and the device's SM
 * count only. */
COSMOT_API int32_t cosmot_attention_kv_split(const cosmot_attn_desc* desc);

/*
 * Debug export of the masking decisions cosmot_mot_attention takes for the
 * same descriptor (sequence 0; they depend on neither the sequence nor the
 * head).  The pages define the mask only element by element (the §3 equations);
 * this shows the kernel's tiling of it so that a test can hold both against
 * the definition.  Key tiles are 128 keys wide; n_kt = ceil(n_keys / 128).
 *   tile_codes  device uint8 [n_q][n_kt]: 0 = the query's CTA never visits the
 *               key tile, 1 = visited with no element mask (every key visible),
 *               2 = visited with per-element masks.  Required.
 *   visible     device uint8 [n_q][n_keys] or NULL: 1 where the kernel lets the
 *               query see the key, else 0.
 * Caller-owned buffers; every element of both is written.  Argument errors as
 * for cosmot_mot_attention (the q/k/v/o checks do not apply).
 */
COSMOT_API cosmot_status cosmot_mot_mask_export(const cosmot_attn_desc* desc, uint8_t* tile_codes, uint8_t* visible,
                                                cosmot_stream_t stream);

/*
 * Flow-matching Euler step ("Cosmos 3 方法原理全解" §7.2), in place:
 *     x[r, c] = bf16( x[r, c] + (sigma_next - sigma) * v[r, c] )  for r in [row_begin, row_end)
 * Rows outside the range are not touched (clean DM rows pass through bit-exact).
 * dsigma is formed in float64 and rounded to float32; the update is one fp32 FMA.
 */
COSMOT_API cosmot_status cosmot_flow_euler_step(void* x, int64_t ld_x, const void* v, int64_t ld_v, int64_t row_begin,
                                     int64_t row_end, int64_t n_cols, double sigma, double sigma_next,
                                     cosmot_stream_t stream);

/*
 * Guided Euler step for a (conditioned, baseline) pair of states
 * ("Cosmos 3 方法原理全解" §7.2 classifier-free guidance):
 *     x' = bf16( x + (sigma_next - sigma) * (v_base + w * (v_cond - v_base)) )
 * computed from x_cond and written to both x_cond and x_base (the two states
 * are equal on entry and stay equal).  All [n_rows, n_cols] bf16 device arrays;
 * x_cond/x_base share ld_x, v_cond/v_base share ld_v.  One fp32 FMA for the
 * guided velocity, one for the step.
 */
COSMOT_API cosmot_status cosmot_flow_cfg_euler_step(void* x_cond, void* x_base, int64_t ld_x, const void* v_cond,
                                                    const void* v_base, int64_t ld_v, int64_t n_rows, int64_t n_cols,
                                                    double sigma, double sigma_next, double guidance,
                                                    cosmot_stream_t stream);

/* ===================================================================== layer */

typedef struct {
  int32_t d_model, n_heads, n_kv_heads, head_dim, ffn;
  int32_t rope_sections[3];
  double rope_base;
  float eps;
  int32_t reserved;
} cosmot_dims;

typedef struct {
  const void* g1;   /* [d] pre-attention RMSNorm gain */
  const void* wqkv; /* [(n_heads + 2 n_kv_heads) head_dim, d]: Q heads, K heads, V heads */
  const void* wo;   /* [d, n_heads head_dim] */
  const void* g2;   /* [d] pre-FFN RMSNorm gain */
  const void* wg;   /* [ffn, d] gate */
  const void* wu;   /* [ffn, d] up */
  const void* wd;   /* [d, ffn] down */
} cosmot_set_weights;

typedef struct {
  cosmot_set_weights set[2]; /* 0 = Reasoner (AR rows), 1 = Generator (DM rows) */
  const void* gfin;          /* [d] final RMSNorm gain before the velocity head (noisy rows) */
  const void* wvel;          /* [d, d] velocity head */
} cosmot_layer_weights;

typedef struct {
  int32_t n_ar, n_clean, n_noisy; /* per sequence; N = n_ar + n_clean + n_noisy */
  int32_t batch;                  /* sequences laid out back to back: [batch][N][d] */
  int32_t mask_mode;              /* COSMOT_MASK_* among DM rows */
  int32_t n_cached;               /* leading rows of each sequence whose K/V are already in the
                                     workspace (0 <= n_cached <= n_ar + n_clean); see below */
  const float* rope_cs;           /* device table of cosmot_mrope_table for one sequence [N] */
  const int32_t* chunk;           /* device [N] (BLOCK_CAUSAL only; may be NULL for FULL) */
} cosmot_seq_desc;

/*
 * Key/value cache in the workspace.  The workspace starts with the layer's QKV
 * rows [batch][N][(n_heads + 2 n_kv_heads) head_dim] (K rotated by mRoPE).  With
 * seq.n_cached = c > 0, rows [0, c) of every sequence keep the K and V left there
 * by earlier calls on the same workspace with the same batch and N; they are not
 * recomputed, their h_out rows are not written, and only rows [c, N) are queries.
 * Because AR rows never read DM rows ("Cosmos 3 方法原理全解" §3), a sampler loop
 * reuses the AR K/V of its first step (c = n_ar, §7.2); a streaming rollout keeps
 * AR + history-block K/V there (c = n_ar + history rows, "流式生成如何工作").
 */

/* Bytes of scratch cosmot_layer_forward needs for these sizes (host only). */
COSMOT_API cosmot_status cosmot_layer_workspace_size(const cosmot_dims* dims, const cosmot_seq_desc* seq, size_t* bytes);

/*
 * One MoT layer forward plus the sampler step, for `batch` packed sequences:
 *   h      device bf16 [batch][N][d], in/out.  Its DM rows are the sampler state x;
 *          on return the noisy DM rows hold x' = x + (sigma_next - sigma) *
 *          (RMSNorm(h2; gfin) . Wvel^T).  AR and clean rows are not written.
 *   h_out  device bf16 [batch][N][d], out: the layer output h2 of every row.
 * Steps: routed RMSNorm -> routed QKV GEMM with mRoPE epilogue -> MoT attention ->
 * routed O GEMM + residual -> routed RMSNorm -> routed gate/up GEMM with SiLU*mul
 * epilogue -> routed down GEMM + residual -> final RMSNorm (noisy rows) ->
 * velocity GEMM with Euler epilogue.  `workspace` must hold
 * cosmot_layer_workspace_size bytes (256-byte aligned); it is clobbered.
 */
COSMOT_API cosmot_status cosmot_layer_forward(const cosmot_dims* dims, const cosmot_layer_weights* w,
                                   const cosmot_seq_desc* seq, void* h, void* h_out, double sigma,
                                   double sigma_next, void* workspace, size_t workspace_bytes,
                                   cosmot_stream_t stream);

/*
 * Sampler state and diagnostic outputs of one step (cosmot_layer_forward_io).
 * "Cosmos 3 方法原理全解" §7.2: the sampler integrates x_next = x + (sigma_next -
 * sigma) v over all steps; the layer reads x as its bf16 DM input rows, but the
 * running state need not be rounded to bf16 after every step.
 *   x_state       NULL, or device float32 [batch][n_noisy][ld_state]: the state
 *                 of the noisy rows, kept in float32 between steps.  The Euler
 *                 step reads x from here (from the bf16 noisy rows of h instead
 *                 when state_from_h = 1, as the first step of a sampling does),
 *                 writes x' here in float32, and writes bf16(x') into the noisy
 *                 rows of h, which the next step's layer reads as its input.
 *   vel           NULL, or device bf16 [batch][n_noisy][ld_vel]: receives the
 *                 velocity v = RMSNorm(h2; gfin) Wvel^T of the noisy rows (the
 *                 step itself uses v's fp32 accumulator, not this copy).
 *   ld_state, ld_vel: row pitches in elements, >= d_model, multiples of 8
 *                 (x_state and vel 16-byte aligned).
 */
typedef struct {
  float* x_state;
  int64_t ld_state;
  void* vel;
  int64_t ld_vel;
  int32_t state_from_h;
  int32_t reserved;
} cosmot_step_io;

/*
 * cosmot_layer_forward with the optional state and outputs of `io` (NULL = the
 * plain cosmot_layer_forward).  Unguided steps only; everything else, including
 * n_cached, as cosmot_layer_forward.
 */
COSMOT_API cosmot_status cosmot_layer_forward_io(const cosmot_dims* dims, const cosmot_layer_weights* w,
                                                 const cosmot_seq_desc* seq, void* h, void* h_out, double sigma,
                                                 double sigma_next, const cosmot_step_io* io, void* workspace,
                                                 size_t workspace_bytes, cosmot_stream_t stream);

/*
 * One guided sampler step ("Cosmos 3 方法原理全解" §7.2-7.3): seq->batch holds
 * (conditioned, baseline) pairs, sequences 2p and 2p+1, with equal layouts and
 * equal DM rows (the state x) but different AR rows (the prompt and the
 * baseline prompt).  Both passes run as one batch of the layer; then the
 * velocities give v = v_base + guidance * (v_cond - v_base) and x' is written
 * to the noisy rows of both sequences of every pair.  h_out holds each pass's
 * h2.  Requires an even batch and ffn * N >= d_model * n_noisy (the velocities
 * reuse the FFN hidden region of the workspace); otherwise as
 * cosmot_layer_forward, including n_cached.
 */
COSMOT_API cosmot_status cosmot_layer_forward_cfg(const cosmot_dims* dims, const cosmot_layer_weights* w,
                                                  const cosmot_seq_desc* seq, void* h, void* h_out, double sigma,
                                                  double sigma_next, double guidance, void* workspace,
                                                  size_t workspace_bytes, cosmot_stream_t stream);

/*
 * Streaming key/value cache update ("NVIDIA 发布 Cosmos 3 系列四个开放权重世界模型",
 * "流式生成如何工作": each finished block's keys and values stay in the cache for
 * the blocks that follow; "Cosmos 3 方法原理全解" §3 for the projection).
 * Commit K/V into the workspace's cache: rows [seq.n_cached, N) of every sequence
 * of h go through the pre-attention RMSNorm and the QKV projection with mRoPE
 * (positions of those rows from seq.rope_cs), and the resulting QKV rows are
 * written to rows [dst_row, dst_row + N - n_cached) of the cache.  Streaming: after
 * a block's last denoising step, its final x is committed over the ring slot of
 * the oldest history block; with n_cached = 0 and dst_row = 0 it fills the cache
 * (AR rows and a prefilled history) in place.  Requires dst_row + N - n_cached <= N.
 */
COSMOT_API cosmot_status cosmot_layer_commit_kv(const cosmot_dims* dims, const cosmot_layer_weights* w,
                                                const cosmot_seq_desc* seq, const void* h, int64_t dst_row,
                                                void* workspace, size_t workspace_bytes, cosmot_stream_t stream);

/*
 * A stack of MoT layers and one sampler step ("Cosmos 3 方法原理全解" §3 for the
 * layer, §12.4 for the released models, which stack 28, 36 or 64 of them; §7.2
 * for the step):
 *     h^0 = h;  h^l = layer_l(h^{l-1})  for l = 1 .. n_layers
 *     noisy rows:  v = RMSNorm(h^L; gfin) W_vel^T,  h <- h + (sigma_next - sigma) v
 * layers: host array of n_layers weight descriptors (device pointers inside),
 *         applied in order; the final norm and velocity head are the gfin and
 *         wvel of the last entry (the others' are not read).
 * h:      [batch, N, d] bf16 device, the stack input; its noisy rows are the
 *         state and receive x'.  Its other rows are not written.
 * h_out:  [batch, N, d] bf16 device, receives h^L (must not alias h).
 * seq:    as for cosmot_layer_forward, with n_cached 0 or n_ar only.  With 0
 *         every row is computed and the q/k/v rows of the AR prefix of every
 *         layer are kept in the workspace; with n_ar those are reused (a
 *         sampler's later steps: AR rows never read DM rows at any depth) and
 *         rows < n_ar of h_out are not written.  Clean DM rows read the noisy
 *         rows from the second layer on, so no longer prefix is step-invariant:
 *         other values return COSMOT_ERR_UNSUPPORTED.
 * workspace: cosmot_stack_workspace_size bytes, 256-byte aligned, owned by the
 *         caller and kept between the steps of one sampling.
 * Errors: INVALID_ARG for null pointers, h == h_out, n_layers outside
 * [1, 1024] or bad dims/seq; WORKSPACE if the workspace is too small.
 */
COSMOT_API cosmot_status cosmot_stack_workspace_size(const cosmot_dims* dims, int32_t n_layers,
                                                     const cosmot_seq_desc* seq, size_t* bytes);
COSMOT_API cosmot_status cosmot_stack_forward(const cosmot_dims* dims, const cosmot_layer_weights* layers,
                                              int32_t n_layers, const cosmot_seq_desc* seq, void* h, void* h_out,
                                              double sigma, double sigma_next, void* workspace,
                                              size_t workspace_bytes, cosmot_stream_t stream);
/* cosmot_stack_forward with the optional float32 state and velocity output of
 * cosmot_step_io (see cosmot_layer_forward_io); io = NULL is the plain call. */
COSMOT_API cosmot_status cosmot_stack_forward_io(const cosmot_dims* dims, const cosmot_layer_weights* layers,
                                                 int32_t n_layers, const cosmot_seq_desc* seq, void* h, void* h_out,
                                                 double sigma, double sigma_next, const cosmot_step_io* io,
                                                 void* workspace, size_t workspace_bytes, cosmot_stream_t stream);

/*
 * Sampler noise levels with the flow shift ("Cosmos 3 方法原理全解" §6.3:
 * t_bar = 1 - t, sigma = s t_bar / (1 + (s - 1) t_bar)) on the uniform grid
 * t_k = k / n_steps: sigmas[k] for k = 0 .. n_steps (n_steps + 1 host doubles,
 * sigmas[0] = 1, sigmas[n_steps] = 0).  Host arithmetic, no stream.  INVALID_ARG
 * for n_steps < 1, a shift that is not a positive finite number, or NULL.
 */
COSMOT_API cosmot_status cosmot_flow_shift_sigmas(int32_t n_steps, double shift, double* sigmas);

/*
 * Domain-specific action input projection ("Cosmos 3 方法原理全解" §4.2:
 * normalised actions, clean conditions and the noisy variable alike, enter the
 * Generator through W_in):  for every segment, rows [row_begin, row_end) of x
 * ([*, ld_x] bf16, action_dim <= 32 columns used) give rows out_row.. of h
 * ([*, ld_h] bf16, 16-byte aligned, ld_h % 8 == 0):
 *     h[out, n] = bf16( sum_c x[row, c] * w_in[n, c] ),  w_in [d_model, action_dim] bf16.
 * weight_set of the segments is ignored; at most 64 segments.
 */
COSMOT_API cosmot_status cosmot_action_embed(const void* x, int64_t ld_x, const cosmot_segment* segs, int32_t n_segs,
                                             const void* w_in, int32_t action_dim, int32_t d_model, void* h,
                                             int64_t ld_h, cosmot_stream_t stream);

/*
 * Action velocity head and the action's own Euler step (§4.2: W_out returns the
 * velocity at the current sigma in the normalised action space; §6.3: each
 * modality has its own noise level).  For every segment, row r of h_last
 * ([*, ld_h] bf16) and row o = out_row + (r - row_begin) of x ([*, ld_x] bf16):
 *     v = RMSNorm(h_last[r]; g_fin, eps) . w_out^T      (fp32; w_out [action_dim, d_model])
 *     x[o] = bf16( x[o] + (sigma_next - sigma) v )
 * With guidance != NULL the segments come in (conditioned, baseline) pairs of
 * equal length (segment 2p and 2p + 1): v = v_base + w (v_cond - v_base) and
 * both x rows receive the same result (they are equal on entry).  h_last, g_fin
 * and w_out 16-byte aligned, d_model and ld_h multiples of 8.
 */
COSMOT_API cosmot_status cosmot_action_head(const void* h_last, int64_t ld_h, const cosmot_segment* segs,
                                            int32_t n_segs, const void* g_fin, float eps, const void* w_out,
                                            int32_t action_dim, int32_t d_model, void* x, int64_t ld_x, double sigma,
                                            double sigma_next, const double* guidance, cosmot_stream_t stream);

/* Actions of a policy step (see cosmot_policy_step). */
typedef struct {
  int32_t action_dim; /* C_a, 1..32 (8 for DROID joint positions, 10 for a generic arm) */
  int32_t n_clean;    /* clean (conditioning) action rows per sequence */
  int32_t n_noisy;    /* noisy action rows per sequence: the last rows of each sequence */
  int32_t clean_row;  /* first clean action row within a sequence (inside the clean group) */
  const void* w_in;   /* [d_model, C_a] bf16 device */
  const void* w_out;  /* [C_a, d_model] bf16 device */
  void* x;            /* [batch * (n_clean + n_noisy), ld_x] bf16 device: per sequence its clean rows,
                         then its noisy rows (the action state, updated in place) */
  int64_t ld_x;
  double sigma, sigma_next; /* the action modality's noise levels for this step */
} cosmot_action_desc;

/*
 * One sampler step of a policy with an action head (§4.2, §6.3, §7.2-7.3):
 *   1. the action rows of h (clean and noisy) receive x W_in^T;
 *   2. the layer stack runs as in cosmot_stack_forward (h^L into h_out);
 *   3. the other noisy rows take the hidden-space head and the Euler step with
 *      (sigma, sigma_next) into h;
 *   4. the noisy action rows take v_a = RMSNorm(h^L; gfin) W_out^T and the Euler
 *      step with (act->sigma, act->sigma_next) into act->x.
 * guidance (NULL or a weight): sequences 2p and 2p + 1 are a (conditioned,
 * baseline) pair sharing their DM rows and action state; both steps use the
 * guided velocity and write both states.  Workspace, n_cached and errors as for
 * cosmot_stack_forward; INVALID_ARG also for a bad action descriptor.
 * stage_events: NULL, or n_events = 8 * n_layers + 2 CUDA events recorded as
 * for cosmot_stack_forward_timed (the action head falls in the final-norm
 * stage; NULL entries are skipped); the computation is the same either way.
 */
COSMOT_API cosmot_status cosmot_policy_step(const cosmot_dims* dims, const cosmot_layer_weights* layers,
                                            int32_t n_layers, const cosmot_seq_desc* seq,
                                            const cosmot_action_desc* act, void* h, void* h_out, double sigma,
                                            double sigma_next, const double* guidance, void* workspace,
                                            size_t workspace_bytes, cosmot_stream_t stream,
                                            void* const* stage_events, int32_t n_events);

/*
 * A layer split around its attention for sequence parallelism over P ranks
 * (one sequence, batch 1, no cached prefix).  A rank holds rows [row0, row1)
 * of the packed sequence in local buffers (global row row0 + i is local row i);
 * routing, positions and the noisy rows follow the global index.
 *   cosmot_layer_shard_pre:  qkv_local [row1 - row0, (H + 2 Hkv) hd] bf16 =
 *       routed RMSNorm and QKV projection with mRoPE of h_local's rows.
 *   (the caller trades rows for heads, runs cosmot_mot_attention on its heads
 *    over all rows, and trades back)
 *   cosmot_layer_shard_post: o_local [row1 - row0, H hd] (heads in order) ->
 *       O projection + residual, routed norm, gate/up, down + residual into
 *       h_out_local, and for the shard's noisy rows the velocity head and the
 *       Euler step into h_local.
 * Every output element is computed with the same arithmetic as in
 * cosmot_layer_forward.  Workspace: cosmot_shard_workspace_size(row1 - row0),
 * 256-byte aligned.  UNSUPPORTED for batch != 1 or n_cached != 0.
 */
COSMOT_API cosmot_status cosmot_shard_workspace_size(const cosmot_dims* dims, int64_t rows, size_t* bytes);
COSMOT_API cosmot_status cosmot_layer_shard_pre(const cosmot_dims* dims, const cosmot_layer_weights* w,
                                                const cosmot_seq_desc* seq, int64_t row0, int64_t row1,
                                                const void* h_local, void* qkv_local, void* workspace,
                                                size_t workspace_bytes, cosmot_stream_t stream);
COSMOT_API cosmot_status cosmot_layer_shard_post(const cosmot_dims* dims, const cosmot_layer_weights* w,
                                                 const cosmot_seq_desc* seq, int64_t row0, int64_t row1,
                                                 void* h_local, const void* o_local, void* h_out_local, double sigma,
                                                 double sigma_next, void* workspace, size_t workspace_bytes,
                                                 cosmot_stream_t stream);

/*
 * dst[r, 0:n_cols] = src[r, 0:n_cols] for r < rows (bf16, row pitches ld_src
 * and ld_dst in elements): packs and unpacks column blocks for the exchanges
 * of a sequence-parallel layer.  One strided device-to-device copy.
 */
COSMOT_API cosmot_status cosmot_copy_columns(const void* src, int64_t ld_src, void* dst, int64_t ld_dst, int64_t rows,
                                             int64_t n_cols, cosmot_stream_t stream);

/*
 * cosmot_stack_forward with CUDA events (cudaEvent_t, created by the caller on
 * the current device) recorded on the stream around every stage:
 * n_events = 8 * n_layers + 2.  Layer l records events[8l + i] before its stage
 * i (COSMOT_STAGE_NORM1 .. COSMOT_STAGE_DOWN_RESIDUAL) and events[8l + 7]
 * after its last one (where the final-norm stage starts); events[8 n_layers]
 * is recorded before the velocity stage and events[8 n_layers + 1] after it.
 * A NULL entry is skipped: that boundary is not marked, and the kernels on
 * either side keep overlapping their launch (a caller timing one stage passes
 * only the events around it).  The computation is identical to
 * cosmot_stack_forward_io with `io` (NULL: cosmot_stack_forward).
 */
COSMOT_API cosmot_status cosmot_stack_forward_timed(const cosmot_dims* dims, const cosmot_layer_weights* layers,
                                                    int32_t n_layers, const cosmot_seq_desc* seq, void* h,
                                                    void* h_out, double sigma, double sigma_next, void* workspace,
                                                    size_t workspace_bytes, cosmot_stream_t stream,
                                                    void* const* stage_events, int32_t n_events,
                                                    const cosmot_step_io* io);

/*
 * cosmot_layer_forward without a caller workspace, for callers that may not
 * allocate device memory while they run: a control loop with a hard per-step
 * deadline (cudaMalloc can synchronise the device and stall for an unbounded
 * time) or a host framework whose own pool owns all device memory.  The pages
 * have no counterpart; this is a deployment convenience of this library.
 *
 * The workspace is a fixed array of COSMOT_NOALLOC_SCRATCH_BYTES compiled into
 * the library; every GPU that loads the library's device code keeps it until
 * the process exits.  Inputs, outputs and semantics are those of
 * cosmot_layer_forward.
 *   - The CUDA driver reserves the array when it loads the module that holds
 *     it.  With the default lazy module loading that is inside the first call
 *     on each device (with CUDA_MODULE_LOADING=EAGER, at context creation), so
 *     make one warm-up call on every device before the deadline loop; later
 *     calls reserve nothing.
 *   - Sizes whose cosmot_layer_workspace_size exceeds the limit return
 *     COSMOT_ERR_WORKSPACE before any launch (64 MiB covers a full-width DROID
 *     policy step, 703 tokens at d_model 4096, batch 1).
 *   - seq->n_cached must be 0 (COSMOT_ERR_UNSUPPORTED otherwise): nothing may
 *     depend on the array's previous contents.  Every scratch byte a call reads
 *     is written earlier in the same call, so nothing needs clearing.
 *   - All calls on a device share its one array: calls that can run at the same
 *     time on that GPU (issued on different streams, or from several host
 *     threads) race on it and corrupt each other's results.  Issue them in order
 *     on one stream.
 *   - The first call on each device looks up the array's device address
 *     (cudaGetSymbolAddress, with that device current); make that first call
 *     before any stream capture.  The address is kept for the life of the
 *     process: after cudaDeviceReset on a device, do not call this entry point
 *     on that device again.
 * The library itself calls no allocator on any path (no cudaMalloc or
 * cudaFree); the only reservation is the driver's, at module load, above.
 */
#define COSMOT_NOALLOC_SCRATCH_BYTES ((size_t)64 << 20)
COSMOT_API cosmot_status cosmot_layer_forward_noalloc(const cosmot_dims* dims, const cosmot_layer_weights* w,
                                                      const cosmot_seq_desc* seq, void* h, void* h_out,
                                                      double sigma, double sigma_next, cosmot_stream_t stream);

/* Stages of cosmot_layer_forward, in launch order. */
enum {
  COSMOT_STAGE_NORM1 = 0,    /* routed RMSNorm before attention */
  COSMOT_STAGE_QKV = 1,      /* routed QKV GEMM + mRoPE epilogue */
  COSMOT_STAGE_ATTN = 2,     /* MoT attention */
  COSMOT_STAGE_OPROJ = 3,    /* routed O GEMM + residual */
  COSMOT_STAGE_NORM2 = 4,    /* routed RMSNorm before the FFN */
  COSMOT_STAGE_GATEUP = 5,   /* routed gate/up GEMM + SiLU*mul */
  COSMOT_STAGE_DOWN = 6,     /* routed down GEMM + residual */
  COSMOT_STAGE_NORMFIN = 7,  /* final RMSNorm of the noisy rows */
  COSMOT_STAGE_VEL = 8,      /* velocity GEMM + Euler step */
  COSMOT_LAYER_STAGES = 9
};

/*
 * cosmot_layer_forward with stage timing: stage_events[i] (i < COSMOT_LAYER_STAGES)
 * is recorded on `stream` just before stage i and stage_events[COSMOT_LAYER_STAGES]
 * after the last one, so cudaEventElapsedTime between consecutive events is the
 * device time of one stage.  The events are cudaEvent_t handles created by the
 * caller on the current device; n_events must be COSMOT_LAYER_STAGES + 1, and a
 * NULL entry is skipped (that boundary is not marked, so the kernels on either
 * side keep overlapping their launch: a caller timing one stage passes only the
 * two events around it).  With
 * guidance == NULL the computation is identical to cosmot_layer_forward_io with
 * `io` (which may be NULL); with a guidance weight it is that of
 * cosmot_layer_forward_cfg (the last stage then covers the velocity GEMM and the
 * guided Euler step), and io must be NULL.
 */
COSMOT_API cosmot_status cosmot_layer_forward_timed(const cosmot_dims* dims, const cosmot_layer_weights* w,
                                                    const cosmot_seq_desc* seq, void* h, void* h_out, double sigma,
                                                    double sigma_next, void* workspace, size_t workspace_bytes,
                                                    cosmot_stream_t stream, void* const* stage_events,
                                                    int32_t n_events, const double* guidance,
                                                    const cosmot_step_io* io);

#ifdef __cplusplus
}
#endif

#endif /* COSMOT_H_ */
