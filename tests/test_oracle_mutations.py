"""Planted mistakes in the oracle must fail its pins.

Each case below plants one plausible error in the fp64 oracle on the CPU (a
flipped sign, a transposed index, a dropped term, a wrong constant; patched in
for one test only) and runs the pins of tests/test_oracle_pins.py that cover
that part.  At least one of them must fail: a pin set that passes a wrong
oracle would not be pinning it.
"""

import os

import numpy as np
import pytest

import test_oracle_pins as P
from oracle import layer, layout, mask, rope

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


# ---------------------------------------------------------------- mRoPE

def _rope_with(rotate):
    def apply(x, pos, head_dim, sections, base):
        x = np.asarray(x, dtype=np.float64)
        th = rope.angles(pos, head_dim, sections, base)
        return rotate(x, np.cos(th)[:, None, :], np.sin(th)[:, None, :], head_dim // 2)
    return apply


def _rotate_negative_angle(x, c, s, half):  # the rotation runs the other way
    x1, x2 = x[..., :half], x[..., half:]
    return np.concatenate([x1 * c + x2 * s, x2 * c - x1 * s], axis=-1)


def _rotate_interleaved(x, c, s, half):  # pairs (2i, 2i+1) instead of (i, i + hd/2)
    out = np.empty_like(x)
    xe, xo = x[..., 0::2], x[..., 1::2]
    out[..., 0::2] = xe * c - xo * s
    out[..., 1::2] = xo * c + xe * s
    return out


def _inv_freq_without_the_two(head_dim, base):
    return base ** (-np.arange(head_dim // 2, dtype=np.float64) / head_dim)


def _pair_axis_t_h_swapped(head_dim, sections):
    n_t, n_h, n_w = sections
    return np.concatenate([np.ones(n_t, np.int64), np.zeros(n_h, np.int64), np.full(n_w, 2, np.int64)])


# ---------------------------------------------------------------- mask

def _allow_with(ar_not_causal=False, ar_sees_all=False, strict_chunks=False):
    def allow_matrix(q_rows, region, chunk, mode, k_rows=None):
        region, chunk = np.asarray(region), np.asarray(chunk)
        q_rows = np.asarray(q_rows, dtype=np.int64)
        k_rows = np.arange(len(region), dtype=np.int64) if k_rows is None else np.asarray(k_rows, np.int64)
        q_ar = (region[q_rows] == layout.REGION_AR)[:, None]
        k_ar = (region[k_rows] == layout.REGION_AR)[None, :]
        causal = k_rows[None, :] <= q_rows[:, None]
        if ar_sees_all:
            ar_part = q_ar & np.ones_like(causal)
        elif ar_not_causal:
            ar_part = q_ar & k_ar
        else:
            ar_part = q_ar & k_ar & causal
        if mode == mask.FULL:
            dm_keys = np.ones((1, len(k_rows)), dtype=bool)
        elif strict_chunks:
            dm_keys = k_ar | (chunk[k_rows][None, :] < chunk[q_rows][:, None])
        else:
            dm_keys = k_ar | (chunk[k_rows][None, :] <= chunk[q_rows][:, None])
        return ar_part | (~q_ar & dm_keys)
    return allow_matrix


def _patch_allow(mp, fn):
    mp.setattr(mask, "allow_matrix", fn)
    mp.setattr(layer, "allow_matrix", fn)  # the layer holds its own reference


# ---------------------------------------------------------------- attention, norms, routing

def _attention_without_scale(orig):
    return lambda q, k, v, allow, scale, q_block=2048: orig(q, k, v, allow, 1.0, q_block)


def _attention_heads_modulo(q, k, v, allow, scale, q_block=2048):
    """Query head h reads kv head h % n_kv instead of h // (H / n_kv)."""
    nq, n_heads, _ = q.shape
    n_kv = k.shape[1]
    out = np.zeros((nq, n_heads, v.shape[2]))
    any_key = allow.any(axis=1)
    for hh in range(n_heads):
        g = hh % n_kv
        s = np.where(allow, (q[:, hh, :] @ k[:, g, :].T) * scale, -np.inf)
        m = np.max(s, axis=1, keepdims=True)
        p = np.exp(s - np.where(np.isfinite(m), m, 0.0))
        lsum = np.where(p.sum(axis=1, keepdims=True) > 0, p.sum(axis=1, keepdims=True), 1.0)
        out[:, hh, :] = np.where(any_key[:, None], (p / lsum) @ v[:, g, :], 0.0)
    return out


def _rms_norm_mean_abs(h, g, eps):
    h = np.asarray(h, dtype=np.float64)
    return h * g / (np.mean(np.abs(h), axis=-1, keepdims=True) + eps)


def _rms_norm_eps_outside(h, g, eps):
    h = np.asarray(h, dtype=np.float64)
    return h * g / (np.sqrt(np.mean(h * h, axis=-1, keepdims=True)) + eps)


def _routed_sets_swapped(orig):
    def routed(x, is_ar, fn):
        return orig(x, is_ar, lambda rows, s, sel: fn(rows, "G" if s == "R" else "R", sel))
    return routed


def _video_group_views_stacked(video, taus, t0, dt_v):
    """Views share the canvas columns instead of sitting side by side along w."""
    tau, view, y, x = np.meshgrid(np.asarray(taus, dtype=np.int64), np.arange(video.views),
                                  np.arange(video.grid_h), np.arange(video.grid_w), indexing="ij")
    tau, view, y, x = (a.reshape(-1) for a in (tau, view, y, x))
    pos = np.stack([t0 + tau.astype(np.float64) * dt_v, y.astype(np.float64), x.astype(np.float64)], axis=1)
    return pos, tau.astype(np.int32)


def _commit_over_newest(self, k, v, chunk):
    """The ring keeps writing one slot after it is full (the newest is lost)."""
    i = min(self.next, self.slots - 1)
    self.k[i], self.v[i], self.chunk[i] = k, v, chunk
    self.next += 1


# ---------------------------------------------------------------- cases

MUTATIONS = {
    "mrope rotates by -theta": (
        lambda mp: mp.setattr(rope, "apply", _rope_with(_rotate_negative_angle)),
        [P.test_text_mrope_equals_1d_rope_for_every_split]),
    "mrope pairs interleaved": (
        lambda mp: mp.setattr(rope, "apply", _rope_with(_rotate_interleaved)),
        [P.test_text_mrope_equals_1d_rope_for_every_split, P.test_mrope_preserves_pair_norms]),
    "mrope frequency exponent without the factor 2": (
        lambda mp: mp.setattr(rope, "inv_freq", _inv_freq_without_the_two),
        [P.test_text_mrope_equals_1d_rope_for_every_split]),
    "mrope t and h sections swapped": (
        lambda mp: mp.setattr(rope, "pair_axis", _pair_axis_t_h_swapped),
        [P.test_mrope_sections_select_axes]),
    "block-causal mask hides the query's own chunk": (
        lambda mp: _patch_allow(mp, _allow_with(strict_chunks=True)),
        [P.test_mask_semantics] + [lambda s=s: P.test_mask_vectorised_equals_equation_construction(
            mask.BLOCK_CAUSAL, s) for s in range(4)]),
    "AR attention not causal": (
        lambda mp: _patch_allow(mp, _allow_with(ar_not_causal=True)),
        [P.test_mask_semantics, lambda: P.test_mask_vectorised_equals_equation_construction(mask.FULL, 0)]),
    "AR rows read every key": (
        lambda mp: _patch_allow(mp, _allow_with(ar_sees_all=True)),
        [P.test_mask_semantics, lambda: P.test_ar_outputs_independent_of_dm_tokens_and_generator_weights("full")]),
    "attention without the 1/sqrt(hd) scale": (
        lambda mp: mp.setattr(layer, "attention", _attention_without_scale(layer.attention)),
        [P.test_attention_matches_brute_force_loops]),
    "grouped queries read the wrong kv head": (
        lambda mp: mp.setattr(layer, "attention", _attention_heads_modulo),
        [P.test_attention_matches_brute_force_loops]),
    "RMSNorm by the mean absolute value": (
        lambda mp: mp.setattr(layer, "rms_norm", _rms_norm_mean_abs),
        [P.test_rmsnorm_and_silu_closed_forms, P.test_gated_ffn_and_velocity_head_closed_form]),
    "RMSNorm eps outside the root": (
        lambda mp: mp.setattr(layer, "rms_norm", _rms_norm_eps_outside),
        [P.test_rmsnorm_and_silu_closed_forms]),
    "SiLU replaced by the sigmoid": (
        lambda mp: mp.setattr(layer, "silu", lambda z: 1.0 / (1.0 + np.exp(-z))),
        [P.test_rmsnorm_and_silu_closed_forms, P.test_gated_ffn_and_velocity_head_closed_form]),
    "Euler step with the sign of dsigma flipped": (
        lambda mp: mp.setattr(layer, "euler_step", lambda x, v, s, sn: np.asarray(x, float) + (s - sn) * np.asarray(v)),
        [P.test_euler_is_exact_on_the_linear_flow_path]),
    "Reasoner and Generator sets swapped": (
        lambda mp: mp.setattr(layer, "routed", _routed_sets_swapped(layer.routed)),
        [lambda: P.test_ar_outputs_independent_of_dm_tokens_and_generator_weights("full"),
         P.test_dm_outputs_use_reasoner_kv_but_not_reasoner_o_or_mlp]),
    "AR-to-DM time offset dropped": (
        lambda mp: mp.setattr(layout, "AR_DM_TIME_OFFSET", 0),
        [lambda: P.test_time_steps_golden(GOLDEN)]),
    "video time step from FPS * 4 tokens per second": (
        lambda mp: mp.setattr(layout, "video_time_step", lambda fps: 6.0 / (4.0 * fps)),
        [P.test_video_dt_real_time_scaling, lambda: P.test_time_steps_golden(GOLDEN)]),
    "flow shift applied as 1/s": (
        lambda mp: mp.setattr(layer, "shift_sigmas", lambda n, s: (1.0 - np.arange(n + 1) / n) /
                              (s + (1.0 - s) * (1.0 - np.arange(n + 1) / n))),
        [P.test_shift_schedule_properties]),
    "action velocity without the final norm": (
        lambda mp: mp.setattr(layer, "action_velocity",
                              lambda dims, h_last, g_fin, w_out: np.asarray(h_last) @ np.asarray(w_out).T),
        [P.test_policy_step_with_residual_only_layers_is_the_closed_form]),
    "camera views not tiled along w": (
        lambda mp: mp.setattr(layout, "_video_group", _video_group_views_stacked),
        [P.test_views_tile_along_w]),
    "stream ring overwrites its newest block": (
        lambda mp: mp.setattr(layer.StreamState, "commit", _commit_over_newest),
        [P.test_stream_ring_evicts_oldest]),
    "guidance extrapolates from the conditioned velocity": (
        lambda mp: mp.setattr(layer, "cfg_combine", lambda vc, vb, w: np.asarray(vc) + float(w) * (np.asarray(vc) -
                                                                                                   np.asarray(vb))),
        [P.test_cfg_limits_reduce_to_single_passes]),
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_mistake_fails_a_pin(name, monkeypatch):
    plant, pins = MUTATIONS[name]
    plant(monkeypatch)
    failed = 0
    for pin in pins:
        try:
            pin()
        except Exception:  # an assertion, or the wrong oracle breaking outright
            failed += 1
    assert failed, f"every pin still passes with the planted mistake: {name}"
