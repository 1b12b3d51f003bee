"""ctypes binding of libcosmot (include/cosmot.h).

Argument marshalling only: every function forwards to the C entry point of the
same name.  Pointers are plain integers (device addresses, e.g. a torch
tensor's data_ptr()), streams are cudaStream_t handles as integers.  Nothing
here computes; if the shared library is missing the import fails loudly.
"""

from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libcosmot.so")
LIB_DEBUG_PATH = os.path.join(_HERE, "libcosmot_debug.so")  # the same ABI, with device-side store checks

COSMOT_OK = 0
COSMOT_ERR_INVALID_ARG = 1
COSMOT_ERR_UNSUPPORTED = 2
COSMOT_ERR_CUDA = 3
COSMOT_ERR_TIMEOUT = 4
COSMOT_ERR_WORKSPACE = 5
COSMOT_ERR_BOUNDS = 6

COSMOT_EPI_NONE = 0
COSMOT_EPI_RESIDUAL = 1
COSMOT_EPI_SILU_MUL = 2
COSMOT_EPI_MROPE = 3
COSMOT_EPI_EULER = 4
COSMOT_EPI_OUT_F32 = 1
COSMOT_EPI_RES_F32 = 2

COSMOT_MASK_FULL = 0
COSMOT_MASK_BLOCK_CAUSAL = 1
COSMOT_ATTN_NO_TILE_SKIP = 1
COSMOT_SITE_SELFTEST = 900
COSMOT_SITE_SELFTEST_BOUNDS = 901

c_i32, c_i64, c_f32, c_f64, c_vp = ctypes.c_int32, ctypes.c_int64, ctypes.c_float, ctypes.c_double, ctypes.c_void_p


class LayoutSpec(ctypes.Structure):
    _fields_ = [("n_text", c_i32),
                ("video_views", c_i32), ("video_grid_h", c_i32), ("video_grid_w", c_i32), ("video_fps", c_i32),
                ("video_clean_steps", c_i32), ("video_noisy_steps", c_i32),
                ("audio_clean", c_i32), ("audio_noisy", c_i32), ("audio_rate", c_i32),
                ("action_clean", c_i32), ("action_noisy", c_i32), ("action_hz", c_i32),
                ("proprio", c_i32), ("tau_offset", c_i32)]


class Segment(ctypes.Structure):
    _fields_ = [("row_begin", c_i64), ("row_end", c_i64), ("out_row", c_i64),
                ("weight_set", c_i32), ("reserved", c_i32)]


class Epilogue(ctypes.Structure):
    _fields_ = [("kind", c_i32), ("head_dim", c_i32), ("rope_cols", c_i64), ("rope_cs", c_vp),
                ("rope_period", c_i64), ("res", c_vp), ("ld_res", c_i64), ("x", c_vp), ("ld_x", c_i64),
                ("dsigma", c_f32), ("reserved", c_f32), ("x_state", c_vp), ("ld_state", c_i64), ("vel", c_vp),
                ("ld_vel", c_i64), ("state_from_x", c_i32), ("flags", c_i32)]


class AttnDesc(ctypes.Structure):
    _fields_ = [("n_q", c_i64), ("q_key_offset", c_i64), ("n_keys", c_i64), ("n_ar", c_i64),
                ("n_heads", c_i32), ("n_kv_heads", c_i32), ("head_dim", c_i32), ("mask_mode", c_i32),
                ("chunk", c_vp), ("batch", c_i32), ("flags", c_i32),
                ("q_batch_stride", c_i64), ("kv_batch_stride", c_i64), ("o_batch_stride", c_i64),
                ("softmax_scale", c_f32), ("reserved2", c_f32)]


class Dims(ctypes.Structure):
    _fields_ = [("d_model", c_i32), ("n_heads", c_i32), ("n_kv_heads", c_i32), ("head_dim", c_i32),
                ("ffn", c_i32), ("rope_sections", c_i32 * 3), ("rope_base", c_f64), ("eps", c_f32),
                ("reserved", c_i32)]


class SetWeights(ctypes.Structure):
    _fields_ = [("g1", c_vp), ("wqkv", c_vp), ("wo", c_vp), ("g2", c_vp), ("wg", c_vp), ("wu", c_vp), ("wd", c_vp)]


class LayerWeights(ctypes.Structure):
    _fields_ = [("set", SetWeights * 2), ("gfin", c_vp), ("wvel", c_vp)]


class ActionDesc(ctypes.Structure):
    _fields_ = [("action_dim", c_i32), ("n_clean", c_i32), ("n_noisy", c_i32), ("clean_row", c_i32),
                ("w_in", c_vp), ("w_out", c_vp), ("x", c_vp), ("ld_x", c_i64), ("sigma", c_f64),
                ("sigma_next", c_f64)]


class StepIO(ctypes.Structure):
    _fields_ = [("x_state", c_vp), ("ld_state", c_i64), ("vel", c_vp), ("ld_vel", c_i64), ("state_from_h", c_i32),
                ("reserved", c_i32)]


class SeqDesc(ctypes.Structure):
    _fields_ = [("n_ar", c_i32), ("n_clean", c_i32), ("n_noisy", c_i32), ("batch", c_i32),
                ("mask_mode", c_i32), ("n_cached", c_i32), ("rope_cs", c_vp), ("chunk", c_vp)]


_P = ctypes.POINTER

# name -> (restype, argtypes); every entry is declared in include/cosmot.h
SIGNATURES = {
    "cosmot_status_string": (ctypes.c_char_p, [c_i32]),
    "cosmot_version": (c_i32, []),
    "cosmot_get_device_status": (c_i32, [c_vp, _P(c_i32), _P(c_i32)]),
    "cosmot_selftest_wait_timeout": (c_i32, [c_vp]),
    "cosmot_debug_checks": (c_i32, []),
    "cosmot_selftest_bounds_check": (c_i32, [c_vp]),
    "cosmot_layout_counts": (c_i32, [_P(LayoutSpec), _P(c_i32), _P(c_i32), _P(c_i32), _P(c_i32)]),
    "cosmot_build_layout": (c_i32, [_P(LayoutSpec), c_vp, c_vp, c_vp, c_vp]),
    "cosmot_mrope_table": (c_i32, [c_vp, c_i64, c_i32, _P(c_i32), c_f64, c_vp, c_vp]),
    "cosmot_rmsnorm_routed": (c_i32, [c_vp, c_i64, _P(Segment), c_i32, c_vp, c_vp, c_i64, c_f32, c_vp, c_i64, c_vp]),
    "cosmot_routed_linear": (c_i32, [c_vp, c_i64, c_i64, _P(Segment), c_i32, c_vp, c_vp, c_vp, c_vp, c_i64, c_vp,
                                     c_i64, _P(Epilogue), c_vp]),
    "cosmot_mrope_apply": (c_i32, [c_vp, c_i64, c_i32, c_vp, c_i64, c_i32, c_i64, c_i32, c_vp, c_vp]),
    "cosmot_mot_attention": (c_i32, [_P(AttnDesc), c_vp, c_i64, c_vp, c_vp, c_i64, c_vp, c_i64, c_vp]),
    "cosmot_mot_mask_export": (c_i32, [_P(AttnDesc), c_vp, c_vp, c_vp]),
    "cosmot_mot_attention_split": (c_i32, [_P(AttnDesc), c_vp, c_i64, c_vp, c_vp, c_i64, c_vp, c_i64, c_i32, c_vp,
                                           ctypes.c_size_t, c_vp]),
    "cosmot_attention_split_workspace": (c_i32, [_P(AttnDesc), c_i32, _P(ctypes.c_size_t)]),
    "cosmot_attention_kv_split": (c_i32, [_P(AttnDesc)]),
    "cosmot_flow_euler_step": (c_i32, [c_vp, c_i64, c_vp, c_i64, c_i64, c_i64, c_i64, c_f64, c_f64, c_vp]),
    "cosmot_flow_cfg_euler_step": (c_i32, [c_vp, c_vp, c_i64, c_vp, c_vp, c_i64, c_i64, c_i64, c_f64, c_f64, c_f64,
                                           c_vp]),
    "cosmot_layer_forward_cfg": (c_i32, [_P(Dims), _P(LayerWeights), _P(SeqDesc), c_vp, c_vp, c_f64, c_f64, c_f64,
                                         c_vp, ctypes.c_size_t, c_vp]),
    "cosmot_layer_workspace_size": (c_i32, [_P(Dims), _P(SeqDesc), _P(ctypes.c_size_t)]),
    "cosmot_layer_forward": (c_i32, [_P(Dims), _P(LayerWeights), _P(SeqDesc), c_vp, c_vp, c_f64, c_f64, c_vp,
                                     ctypes.c_size_t, c_vp]),
    "cosmot_layer_forward_io": (c_i32, [_P(Dims), _P(LayerWeights), _P(SeqDesc), c_vp, c_vp, c_f64, c_f64,
                                        _P(StepIO), c_vp, ctypes.c_size_t, c_vp]),
    "cosmot_flow_shift_sigmas": (c_i32, [c_i32, c_f64, _P(c_f64)]),
    "cosmot_action_embed": (c_i32, [c_vp, c_i64, _P(Segment), c_i32, c_vp, c_i32, c_i32, c_vp, c_i64, c_vp]),
    "cosmot_action_head": (c_i32, [c_vp, c_i64, _P(Segment), c_i32, c_vp, c_f32, c_vp, c_i32, c_i32, c_vp, c_i64, c_f64,
                                   c_f64, _P(c_f64), c_vp]),
    "cosmot_policy_step": (c_i32, [_P(Dims), _P(LayerWeights), c_i32, _P(SeqDesc), _P(ActionDesc), c_vp, c_vp, c_f64,
                                   c_f64, _P(c_f64), c_vp, ctypes.c_size_t, c_vp, _P(c_vp), c_i32]),
    "cosmot_shard_workspace_size": (c_i32, [_P(Dims), c_i64, _P(ctypes.c_size_t)]),
    "cosmot_layer_shard_pre": (c_i32, [_P(Dims), _P(LayerWeights), _P(SeqDesc), c_i64, c_i64, c_vp, c_vp, c_vp,
                                       ctypes.c_size_t, c_vp]),
    "cosmot_layer_shard_post": (c_i32, [_P(Dims), _P(LayerWeights), _P(SeqDesc), c_i64, c_i64, c_vp, c_vp, c_vp,
                                        c_f64, c_f64, c_vp, ctypes.c_size_t, c_vp]),
    "cosmot_copy_columns": (c_i32, [c_vp, c_i64, c_vp, c_i64, c_i64, c_i64, c_vp]),
    "cosmot_stack_workspace_size": (c_i32, [_P(Dims), c_i32, _P(SeqDesc), _P(ctypes.c_size_t)]),
    "cosmot_stack_forward": (c_i32, [_P(Dims), _P(LayerWeights), c_i32, _P(SeqDesc), c_vp, c_vp, c_f64, c_f64, c_vp,
                                     ctypes.c_size_t, c_vp]),
    "cosmot_stack_forward_io": (c_i32, [_P(Dims), _P(LayerWeights), c_i32, _P(SeqDesc), c_vp, c_vp, c_f64, c_f64,
                                        _P(StepIO), c_vp, ctypes.c_size_t, c_vp]),
    "cosmot_stack_forward_timed": (c_i32, [_P(Dims), _P(LayerWeights), c_i32, _P(SeqDesc), c_vp, c_vp, c_f64, c_f64,
                                           c_vp, ctypes.c_size_t, c_vp, _P(c_vp), c_i32, _P(StepIO)]),
    "cosmot_layer_commit_kv": (c_i32, [_P(Dims), _P(LayerWeights), _P(SeqDesc), c_vp, c_i64, c_vp, ctypes.c_size_t,
                                       c_vp]),
    "cosmot_layer_forward_noalloc": (c_i32, [_P(Dims), _P(LayerWeights), _P(SeqDesc), c_vp, c_vp, c_f64, c_f64,
                                             c_vp]),
    "cosmot_layer_forward_timed": (c_i32, [_P(Dims), _P(LayerWeights), _P(SeqDesc), c_vp, c_vp, c_f64, c_f64, c_vp,
                                           ctypes.c_size_t, c_vp, _P(c_vp), c_i32, _P(c_f64), _P(StepIO)]),
}

COSMOT_LAYER_STAGES = 9
COSMOT_NOALLOC_SCRATCH_BYTES = 64 << 20
STAGE_NAMES = ("norm1", "qkv_mrope", "attention", "oproj_residual", "norm2", "gateup_silu", "down_residual",
               "norm_final", "velocity_euler")

_lib = None
_lib_debug = None


def load(path: str) -> ctypes.CDLL:
    """Loads one build of the library and declares every entry's signature."""
    if not os.path.exists(path):
        raise ImportError(f"{os.path.basename(path)} not built at {path}; run "
                          f"`python -m flow_matching_dit_cosmot_b200.build`")
    L = ctypes.CDLL(path)
    for name, (res, args) in SIGNATURES.items():
        f = getattr(L, name)
        f.restype = res
        f.argtypes = args
    return L


def lib() -> ctypes.CDLL:
    """Loads libcosmot.so (built in-tree by flow_matching_dit_cosmot_b200.build)."""
    global _lib
    if _lib is None:
        _lib = load(LIB_PATH)
    return _lib


def lib_debug() -> ctypes.CDLL:
    """Loads libcosmot_debug.so: the debug build, whose kernels check the index
    of every global store and latch COSMOT_ERR_BOUNDS instead of writing out of
    place.  Call its entries directly (same names and signatures)."""
    global _lib_debug
    if _lib_debug is None:
        _lib_debug = load(LIB_DEBUG_PATH)
    return _lib_debug


class CosmotError(RuntimeError):
    def __init__(self, fn, code):
        super().__init__(f"{fn} failed: {status_string(code)} ({code})")
        self.code = code


def status_string(code: int) -> str:
    return lib().cosmot_status_string(code).decode()


def _check(fn, code):
    if code != COSMOT_OK:
        raise CosmotError(fn, code)
    return code


def _call(name, *args, check=True):
    code = getattr(lib(), name)(*args)
    return _check(name, code) if check else code


# ------------------------------------------------------------------ thin wrappers (same names as the C ABI)

def cosmot_version() -> int:
    return lib().cosmot_version()


def cosmot_get_device_status(stream: int = 0):
    st, where = c_i32(0), c_i32(0)
    _call("cosmot_get_device_status", c_vp(stream), ctypes.byref(st), ctypes.byref(where))
    return st.value, where.value


def cosmot_selftest_wait_timeout(stream: int = 0):
    """Test-only: a bounded wait that never completes; latches COSMOT_ERR_TIMEOUT."""
    _call("cosmot_selftest_wait_timeout", c_vp(stream))


def cosmot_layout_counts(spec: LayoutSpec):
    n, a, c, z = c_i32(), c_i32(), c_i32(), c_i32()
    _call("cosmot_layout_counts", ctypes.byref(spec), ctypes.byref(n), ctypes.byref(a), ctypes.byref(c), ctypes.byref(z))
    return n.value, a.value, c.value, z.value


def cosmot_build_layout(spec: LayoutSpec, pos: int, chunk: int, region: int = 0, stream: int = 0, check=True):
    return _call("cosmot_build_layout", ctypes.byref(spec), c_vp(pos), c_vp(chunk), c_vp(region or None),
                 c_vp(stream), check=check)


def cosmot_mrope_table(pos: int, n_rows: int, head_dim: int, sections, rope_base: float, cs: int, stream: int = 0,
                       check=True):
    sec = (c_i32 * 3)(*sections)
    return _call("cosmot_mrope_table", c_vp(pos), n_rows, head_dim, sec, rope_base, c_vp(cs), c_vp(stream),
                 check=check)


def _segs(segs):
    """(row_begin, row_end, out_row, weight_set[, reserved]) tuples -> Segment array."""
    arr = (Segment * len(segs))(*[Segment(int(t[0]), int(t[1]), int(t[2]), int(t[3]), 0) for t in segs])
    return arr, len(segs)


def cosmot_rmsnorm_routed(h: int, ld_h: int, segs, g0: int, g1: int, d: int, eps: float, out: int, ld_out: int,
                          stream: int = 0, check=True):
    arr, n = _segs(segs)
    return _call("cosmot_rmsnorm_routed", c_vp(h), ld_h, arr, n, c_vp(g0), c_vp(g1), d, eps, c_vp(out), ld_out,
                 c_vp(stream), check=check)


def cosmot_routed_linear(a: int, ld_a: int, k: int, segs, w0: int, w1: int, n_out: int, out: int, ld_out: int,
                         epi: Epilogue | None = None, w0_up: int = 0, w1_up: int = 0, stream: int = 0, check=True):
    arr, n = _segs(segs)
    e = epi if epi is not None else Epilogue(kind=COSMOT_EPI_NONE)
    return _call("cosmot_routed_linear", c_vp(a), ld_a, k, arr, n, c_vp(w0 or None), c_vp(w1 or None),
                 c_vp(w0_up or None), c_vp(w1_up or None), n_out, c_vp(out), ld_out, ctypes.byref(e), c_vp(stream),
                 check=check)


def cosmot_mrope_apply(q: int, ld_q: int, n_q_heads: int, k: int, ld_k: int, n_k_heads: int, n_rows: int,
                       head_dim: int, cs: int, stream: int = 0, check=True):
    return _call("cosmot_mrope_apply", c_vp(q or None), ld_q, n_q_heads, c_vp(k or None), ld_k, n_k_heads, n_rows,
                 head_dim, c_vp(cs), c_vp(stream), check=check)


def cosmot_mot_attention(desc: AttnDesc, q: int, ld_q: int, k: int, v: int, ld_kv: int, o: int, ld_o: int,
                         stream: int = 0, check=True):
    return _call("cosmot_mot_attention", ctypes.byref(desc), c_vp(q), ld_q, c_vp(k), c_vp(v), ld_kv, c_vp(o), ld_o,
                 c_vp(stream), check=check)


def cosmot_mot_attention_split(desc: AttnDesc, q: int, ld_q: int, k: int, v: int, ld_kv: int, o: int, ld_o: int,
                               kv_split: int, workspace: int, workspace_bytes: int, stream: int = 0, check=True):
    return _call("cosmot_mot_attention_split", ctypes.byref(desc), c_vp(q), ld_q, c_vp(k), c_vp(v), ld_kv, c_vp(o),
                 ld_o, kv_split, c_vp(workspace or None), workspace_bytes, c_vp(stream), check=check)


def cosmot_attention_split_workspace(desc: AttnDesc, kv_split: int) -> int:
    n = ctypes.c_size_t(0)
    _call("cosmot_attention_split_workspace", ctypes.byref(desc), kv_split, ctypes.byref(n))
    return n.value


def cosmot_attention_kv_split(desc: AttnDesc) -> int:
    return lib().cosmot_attention_kv_split(ctypes.byref(desc))


def cosmot_mot_mask_export(desc: AttnDesc, tile_codes: int, visible: int = 0, stream: int = 0, check=True):
    """Tile codes [n_q][ceil(n_keys/128)] and element visibility [n_q][n_keys]
    (uint8 device buffers) of the attention kernel's masking."""
    return _call("cosmot_mot_mask_export", ctypes.byref(desc), c_vp(tile_codes), c_vp(visible or None),
                 c_vp(stream), check=check)


def cosmot_flow_euler_step(x: int, ld_x: int, v: int, ld_v: int, row_begin: int, row_end: int, n_cols: int,
                           sigma: float, sigma_next: float, stream: int = 0, check=True):
    return _call("cosmot_flow_euler_step", c_vp(x), ld_x, c_vp(v), ld_v, row_begin, row_end, n_cols, sigma,
                 sigma_next, c_vp(stream), check=check)


def cosmot_flow_cfg_euler_step(x_cond: int, x_base: int, ld_x: int, v_cond: int, v_base: int, ld_v: int, n_rows: int,
                               n_cols: int, sigma: float, sigma_next: float, guidance: float, stream: int = 0,
                               check=True):
    return _call("cosmot_flow_cfg_euler_step", c_vp(x_cond), c_vp(x_base), ld_x, c_vp(v_cond), c_vp(v_base), ld_v,
                 n_rows, n_cols, sigma, sigma_next, guidance, c_vp(stream), check=check)


def cosmot_layer_forward_cfg(dims: Dims, w: LayerWeights, seq: SeqDesc, h: int, h_out: int, sigma: float,
                             sigma_next: float, guidance: float, workspace: int, workspace_bytes: int, stream: int = 0,
                             check=True):
    return _call("cosmot_layer_forward_cfg", ctypes.byref(dims), ctypes.byref(w), ctypes.byref(seq), c_vp(h),
                 c_vp(h_out), sigma, sigma_next, guidance, c_vp(workspace), workspace_bytes, c_vp(stream), check=check)


def cosmot_layer_workspace_size(dims: Dims, seq: SeqDesc) -> int:
    n = ctypes.c_size_t(0)
    _call("cosmot_layer_workspace_size", ctypes.byref(dims), ctypes.byref(seq), ctypes.byref(n))
    return n.value


def cosmot_layer_forward(dims: Dims, w: LayerWeights, seq: SeqDesc, h: int, h_out: int, sigma: float,
                         sigma_next: float, workspace: int, workspace_bytes: int, stream: int = 0, check=True):
    return _call("cosmot_layer_forward", ctypes.byref(dims), ctypes.byref(w), ctypes.byref(seq), c_vp(h),
                 c_vp(h_out), sigma, sigma_next, c_vp(workspace), workspace_bytes, c_vp(stream), check=check)


def step_io(x_state: int = 0, ld_state: int = 0, vel: int = 0, ld_vel: int = 0, state_from_h: bool = False):
    """StepIO for cosmot_layer_forward_io / _timed (pointers as integers, 0 = absent)."""
    return StepIO(x_state or None, ld_state, vel or None, ld_vel, 1 if state_from_h else 0, 0)


def cosmot_layer_forward_io(dims: Dims, w: LayerWeights, seq: SeqDesc, h: int, h_out: int, sigma: float,
                            sigma_next: float, io: StepIO | None, workspace: int, workspace_bytes: int,
                            stream: int = 0, check=True):
    return _call("cosmot_layer_forward_io", ctypes.byref(dims), ctypes.byref(w), ctypes.byref(seq), c_vp(h),
                 c_vp(h_out), sigma, sigma_next, ctypes.byref(io) if io is not None else None, c_vp(workspace),
                 workspace_bytes, c_vp(stream), check=check)


def cosmot_layer_commit_kv(dims: Dims, w: LayerWeights, seq: SeqDesc, h: int, dst_row: int, workspace: int,
                           workspace_bytes: int, stream: int = 0, check=True):
    return _call("cosmot_layer_commit_kv", ctypes.byref(dims), ctypes.byref(w), ctypes.byref(seq), c_vp(h), dst_row,
                 c_vp(workspace), workspace_bytes, c_vp(stream), check=check)


def cosmot_flow_shift_sigmas(n_steps: int, shift: float) -> list:
    out = (c_f64 * (n_steps + 1))()
    _call("cosmot_flow_shift_sigmas", n_steps, shift, out)
    return list(out)


def cosmot_action_embed(x: int, ld_x: int, segs, w_in: int, action_dim: int, d_model: int, h: int, ld_h: int,
                        stream: int = 0, check=True):
    """`segs`: (row_begin, row_end, out_row, weight_set, reserved) tuples."""
    arr, n = _segs(segs)
    return _call("cosmot_action_embed", c_vp(x), ld_x, arr, n, c_vp(w_in), action_dim, d_model, c_vp(h), ld_h,
                 c_vp(stream), check=check)


def cosmot_action_head(h_last: int, ld_h: int, segs, g_fin: int, eps: float, w_out: int, action_dim: int,
                       d_model: int, x: int, ld_x: int, sigma: float, sigma_next: float, guidance=None,
                       stream: int = 0, check=True):
    arr, n = _segs(segs)
    g = ctypes.byref(c_f64(guidance)) if guidance is not None else None
    return _call("cosmot_action_head", c_vp(h_last), ld_h, arr, n, c_vp(g_fin), eps, c_vp(w_out), action_dim,
                 d_model, c_vp(x), ld_x, sigma, sigma_next, g, c_vp(stream), check=check)


def cosmot_policy_step(dims: Dims, layers, seq: SeqDesc, act: ActionDesc, h: int, h_out: int, sigma: float,
                       sigma_next: float, guidance, workspace: int, workspace_bytes: int, stream: int = 0,
                       events=None, check=True):
    """`events`: None, or 8 * len(layers) + 2 raw cudaEvent_t handles (ints; None skips that boundary)."""
    if not isinstance(layers, ctypes.Array):
        layers = (LayerWeights * len(layers))(*layers)
    g = ctypes.byref(c_f64(guidance)) if guidance is not None else None
    arr = (c_vp * len(events))(*[c_vp(e) for e in events]) if events else None
    return _call("cosmot_policy_step", ctypes.byref(dims), layers, len(layers), ctypes.byref(seq), ctypes.byref(act),
                 c_vp(h), c_vp(h_out), sigma, sigma_next, g, c_vp(workspace), workspace_bytes, c_vp(stream), arr,
                 len(events) if events else 0, check=check)


def cosmot_shard_workspace_size(dims: Dims, rows: int) -> int:
    n = ctypes.c_size_t(0)
    _call("cosmot_shard_workspace_size", ctypes.byref(dims), rows, ctypes.byref(n))
    return n.value


def cosmot_layer_shard_pre(dims: Dims, w: LayerWeights, seq: SeqDesc, row0: int, row1: int, h_local: int,
                           qkv_local: int, workspace: int, workspace_bytes: int, stream: int = 0, check=True):
    return _call("cosmot_layer_shard_pre", ctypes.byref(dims), ctypes.byref(w), ctypes.byref(seq), row0, row1,
                 c_vp(h_local), c_vp(qkv_local), c_vp(workspace), workspace_bytes, c_vp(stream), check=check)


def cosmot_layer_shard_post(dims: Dims, w: LayerWeights, seq: SeqDesc, row0: int, row1: int, h_local: int,
                            o_local: int, h_out_local: int, sigma: float, sigma_next: float, workspace: int,
                            workspace_bytes: int, stream: int = 0, check=True):
    return _call("cosmot_layer_shard_post", ctypes.byref(dims), ctypes.byref(w), ctypes.byref(seq), row0, row1,
                 c_vp(h_local), c_vp(o_local), c_vp(h_out_local), sigma, sigma_next, c_vp(workspace),
                 workspace_bytes, c_vp(stream), check=check)


def cosmot_copy_columns(src: int, ld_src: int, dst: int, ld_dst: int, rows: int, n_cols: int, stream: int = 0,
                        check=True):
    return _call("cosmot_copy_columns", c_vp(src), ld_src, c_vp(dst), ld_dst, rows, n_cols, c_vp(stream),
                 check=check)


def cosmot_stack_workspace_size(dims: Dims, n_layers: int, seq: SeqDesc) -> int:
    n = ctypes.c_size_t(0)
    _call("cosmot_stack_workspace_size", ctypes.byref(dims), n_layers, ctypes.byref(seq), ctypes.byref(n))
    return n.value


def cosmot_stack_forward(dims: Dims, layers, seq: SeqDesc, h: int, h_out: int, sigma: float, sigma_next: float,
                         workspace: int, workspace_bytes: int, stream: int = 0, check=True):
    """`layers`: a ctypes array of LayerWeights (or a sequence of them)."""
    if not isinstance(layers, ctypes.Array):
        layers = (LayerWeights * len(layers))(*layers)
    return _call("cosmot_stack_forward", ctypes.byref(dims), layers, len(layers), ctypes.byref(seq), c_vp(h),
                 c_vp(h_out), sigma, sigma_next, c_vp(workspace), workspace_bytes, c_vp(stream), check=check)


def cosmot_stack_forward_io(dims: Dims, layers, seq: SeqDesc, h: int, h_out: int, sigma: float, sigma_next: float,
                            io: StepIO | None, workspace: int, workspace_bytes: int, stream: int = 0, check=True):
    if not isinstance(layers, ctypes.Array):
        layers = (LayerWeights * len(layers))(*layers)
    return _call("cosmot_stack_forward_io", ctypes.byref(dims), layers, len(layers), ctypes.byref(seq), c_vp(h),
                 c_vp(h_out), sigma, sigma_next, ctypes.byref(io) if io is not None else None, c_vp(workspace),
                 workspace_bytes, c_vp(stream), check=check)


def cosmot_stack_forward_timed(dims: Dims, layers, seq: SeqDesc, h: int, h_out: int, sigma: float,
                               sigma_next: float, workspace: int, workspace_bytes: int, stream: int, events,
                               io: StepIO | None = None, check=True):
    """`events`: 8 * len(layers) + 2 raw cudaEvent_t handles (ints; None skips that boundary)."""
    if not isinstance(layers, ctypes.Array):
        layers = (LayerWeights * len(layers))(*layers)
    arr = (c_vp * len(events))(*[c_vp(e) for e in events])
    return _call("cosmot_stack_forward_timed", ctypes.byref(dims), layers, len(layers), ctypes.byref(seq), c_vp(h),
                 c_vp(h_out), sigma, sigma_next, c_vp(workspace), workspace_bytes, c_vp(stream), arr, len(events),
                 ctypes.byref(io) if io is not None else None, check=check)


def cosmot_layer_forward_noalloc(dims: Dims, w: LayerWeights, seq: SeqDesc, h: int, h_out: int, sigma: float,
                                 sigma_next: float, stream: int = 0, check=True):
    """Layer forward with the library's fixed scratch array instead of a caller workspace."""
    return _call("cosmot_layer_forward_noalloc", ctypes.byref(dims), ctypes.byref(w), ctypes.byref(seq), c_vp(h),
                 c_vp(h_out), sigma, sigma_next, c_vp(stream), check=check)


def cosmot_layer_forward_timed(dims: Dims, w: LayerWeights, seq: SeqDesc, h: int, h_out: int, sigma: float,
                               sigma_next: float, workspace: int, workspace_bytes: int, stream: int, events,
                               guidance: float | None = None, io: StepIO | None = None, check=True):
    """`events`: COSMOT_LAYER_STAGES + 1 raw cudaEvent_t handles (ints; None skips that boundary); `guidance`
    selects the guided step of cosmot_layer_forward_cfg; `io` the float32 state
    and velocity output of cosmot_layer_forward_io."""
    arr = (c_vp * len(events))(*[c_vp(e) for e in events])
    g = ctypes.byref(c_f64(guidance)) if guidance is not None else None
    return _call("cosmot_layer_forward_timed", ctypes.byref(dims), ctypes.byref(w), ctypes.byref(seq), c_vp(h),
                 c_vp(h_out), sigma, sigma_next, c_vp(workspace), workspace_bytes, c_vp(stream), arr, len(events), g,
                 ctypes.byref(io) if io is not None else None, check=check)
