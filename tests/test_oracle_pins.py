"""Pins of the fp64 oracle against what the pages and the mathematics fix.

Each test checks the oracle against something other than itself: a value the
pages print (tests/golden), a closed form, a textbook routine written another
way, an invariant the pages state, or brute force on tiny inputs.
"""

import json
import os

import numpy as np
import pytest

import synth
from synth import LayoutSpec, ModelDims, VideoSpec
from oracle import layer, layout, mask, rope

TINY = ModelDims(d_model=64, n_heads=4, n_kv_heads=2, head_dim=16, ffn=96, rope_sections=(2, 3, 3))


def _weights(dims, seed=7):
    return layer.weights_from_bits(dims, synth.make_weights(dims, seed))


def _h(n, d, seed=11):
    return synth.bf16_to_f64(synth.make_activations(n, d, seed))


def _small_layout(**kw):
    spec = LayoutSpec(n_text=kw.pop("n_text", 5), video=kw.pop("video", VideoSpec(1, 2, 3, 24, 1, 2)), **kw)
    return layout.build_layout(spec)


# ---------------------------------------------------------------- golden values

def test_latent_sizes_golden(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "latent_sizes.json")))
    v = g["video_480p"]
    assert v["width"] // v["spatial_stride"] == v["grid_w"]
    assert v["height"] // v["spatial_stride"] == v["grid_h"]
    assert 1 + (g["frames"] - 1) // g["temporal_compression"] == g["latent_steps"]
    # The 480p text-to-video workload reproduces the printed token count.
    lay = layout.build_layout(synth.preset("t2v480").layout)
    assert lay.n_noisy == g["latent_tokens"] == g["latent_steps"] * v["grid_w"] * v["grid_h"]
    assert lay.n_clean == 0 and lay.n_ar == 256 + 2
    # I2V: one clean latent step, 47 noisy ones.
    i2v = synth.preset("i2v720").layout.video
    assert (i2v.clean_steps, i2v.noisy_steps) == (g["i2v"]["clean_latent_steps"], g["i2v"]["noisy_latent_steps"])
    lay5 = layout.build_layout(synth.preset("i2v720").layout)
    assert (lay5.n_ar, lay5.n_clean, lay5.n_noisy) == (514, 880, 41360)
    lay3 = layout.build_layout(synth.preset("droid").layout)
    assert (lay3.n_ar, lay3.n_clean, lay3.n_noisy) == (130, 181, 392)


def test_resolution_table_golden(golden_dir):
    """The published resolutions against the stride-32 latent grid read from
    §4.1 (832x480 -> 26x15).  In the 480p and 720p classes the five aspect
    buckets have the same pixel area to within 3 %, and so the same number of
    tokens per latent step (the 256p class on the page is not equal-area);
    transposed aspects swap the grid; every 256p and 480p side divides by 32;
    1280x720 floors to 40x22 (the 720p workload's grid)."""
    g = json.load(open(os.path.join(golden_dir, "resolutions.json")))
    for cls in ("256p", "480p", "720p"):
        grids = [(w // 32, h // 32) for w, h in g[cls]]
        assert grids[0] == grids[4][::-1] and grids[1] == grids[3][::-1], cls
        if cls in ("256p", "480p"):
            assert all(w % 32 == 0 and h % 32 == 0 for w, h in g[cls]), cls
        if cls in ("480p", "720p"):
            areas = [w * h for w, h in g[cls]]
            tokens = [gw * gh for gw, gh in grids]
            assert max(areas) <= 1.03 * min(areas), (cls, areas)
            assert max(tokens) <= 1.03 * min(tokens), (cls, tokens)
    v = synth.preset("t2v480").layout.video
    assert (g["480p"][0][0] // 32, g["480p"][0][1] // 32) == (v.grid_w, v.grid_h) == (26, 15)
    v = synth.preset("i2v720").layout.video
    assert (g["720p"][0][0] // 32, g["720p"][0][1] // 32) == (v.grid_w, v.grid_h) == (40, 22)


def test_time_steps_golden(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "time_steps.json")))
    assert layout.video_time_step(g["video_fps"]) == g["video_dt"]
    assert abs(layout.rate_time_step(g["audio_tokens_per_second"]) - g["audio_dt"]) < 1e-15
    assert abs(layout.rate_time_step(g["action_hz"]) - g["action_dt"]) < 1e-15
    assert layout.AR_DM_TIME_OFFSET == g["ar_dm_time_offset"]
    # The steps appear in the coordinates themselves.
    lay = _small_layout(audio_clean=3, audio_noisy=4, action_noisy=5, action_hz=15)
    t = lay.pos64[:, 0]
    aud = np.where(lay.modality == layout.MOD_AUDIO)[0]
    act = np.where(lay.modality == layout.MOD_ACTION)[0]
    vid = np.where(lay.modality == layout.MOD_VIDEO)[0]
    np.testing.assert_allclose(np.diff(t[aud]), g["audio_dt"], atol=1e-9)
    np.testing.assert_allclose(np.diff(t[act]), g["action_dt"], atol=1e-9)
    steps = np.unique(t[vid])
    np.testing.assert_allclose(np.diff(steps), g["video_dt"], atol=1e-12)
    # DM time starts g["ar_dm_time_offset"] after the AR index range.
    assert steps[0] == lay.n_ar + g["ar_dm_time_offset"]


def test_video_dt_real_time_scaling():
    # §5: dt = 6/TPS with TPS = FPS/4; 15 FPS video (DROID) -> 1.6, 30 FPS -> 0.8.
    assert abs(layout.video_time_step(15) - 1.6) < 1e-15
    assert abs(layout.video_time_step(30) - 0.8) < 1e-15
    # One second of video, audio and action spans the same t range.
    assert abs(6 * layout.video_time_step(24) - 25 * layout.rate_time_step(25)) < 1e-12
    assert abs(6 * layout.video_time_step(24) - 15 * layout.rate_time_step(15)) < 1e-12


# ---------------------------------------------------------------- layout order

def test_packed_order_and_regions():
    lay = _small_layout(audio_clean=2, audio_noisy=3, action_clean=1, action_noisy=4, proprio=1)
    r, m = lay.region, lay.modality
    assert np.all(np.diff(r) >= 0), "AR, then clean DM, then noisy DM"
    assert lay.n_ar == 5 + 2
    clean_m = m[r == layout.REGION_CLEAN]
    noisy_m = m[r == layout.REGION_NOISY]
    order = {layout.MOD_VIDEO: 0, layout.MOD_AUDIO: 1, layout.MOD_ACTION: 2, layout.MOD_PROPRIO: 2}
    assert np.all(np.diff([order[x] for x in clean_m]) >= 0)
    assert np.all(np.diff([order[x] for x in noisy_m]) >= 0)
    # AR tokens carry t = h = w = index (text reduces to 1D RoPE).
    k = np.arange(lay.n_ar)
    np.testing.assert_array_equal(lay.pos64[:lay.n_ar], np.stack([k, k, k], 1))
    # Audio and action use t only.
    nv = m != layout.MOD_VIDEO
    dm = r != layout.REGION_AR
    assert np.all(lay.pos64[nv & dm][:, 1:] == 0)


def test_clean_prefix_and_noisy_future_share_time_axis():
    lay = _small_layout(video=VideoSpec(1, 2, 2, 24, 2, 3))
    vid = lay.modality == layout.MOD_VIDEO
    t_clean = np.unique(lay.pos64[vid & (lay.region == layout.REGION_CLEAN), 0])
    t_noisy = np.unique(lay.pos64[vid & (lay.region == layout.REGION_NOISY), 0])
    allt = np.concatenate([t_clean, t_noisy])
    np.testing.assert_allclose(np.diff(allt), 1.0)
    np.testing.assert_array_equal(np.unique(lay.chunk[vid]), np.arange(5))


def test_views_tile_along_w():
    lay = layout.build_layout(synth.preset("droid").layout)
    vid = lay.modality == layout.MOD_VIDEO
    w = lay.pos64[vid, 2]
    assert w.max() == 3 * 10 - 1 and lay.pos64[vid, 1].max() == 6 - 1


def test_positions_float32_is_rounded_float64():
    lay = layout.build_layout(synth.preset("droid").layout)
    np.testing.assert_array_equal(lay.pos, lay.pos64.astype(np.float32))
    assert lay.pos.dtype == np.float32


# ---------------------------------------------------------------- mRoPE

def test_text_mrope_equals_1d_rope_for_every_split():
    hd = 16
    rng = np.random.default_rng(0)
    x = rng.standard_normal((9, 3, hd))
    k = np.arange(9, dtype=np.float64)
    pos = np.stack([k, k, k], 1)
    # Textbook RoPE as complex rotation: z_i = x_i + i x_{i+hd/2}, z_i * exp(i k theta_i).
    theta = 10000.0 ** (-np.arange(hd // 2) * 2.0 / hd)
    z = x[..., : hd // 2] + 1j * x[..., hd // 2:]
    z = z * np.exp(1j * k[:, None, None] * theta[None, None, :])
    want = np.concatenate([z.real, z.imag], axis=-1)
    for sections in [(8, 0, 0), (2, 3, 3), (4, 2, 2), (0, 4, 4), (1, 1, 6)]:
        got = rope.apply(x, pos, hd, sections, 10000.0)
        np.testing.assert_allclose(got, want, rtol=0, atol=1e-12)


def test_mrope_uniform_shift_leaves_scores_unchanged():
    hd = 16
    rng = np.random.default_rng(1)
    q = rng.standard_normal((7, 1, hd))
    k = rng.standard_normal((7, 1, hd))
    pos = rng.uniform(0, 50, size=(7, 3))
    s0 = np.einsum("ihd,jhd->ij", rope.apply(q, pos, hd, (2, 3, 3), 1e4), rope.apply(k, pos, hd, (2, 3, 3), 1e4))
    pos2 = pos + 13.25
    s1 = np.einsum("ihd,jhd->ij", rope.apply(q, pos2, hd, (2, 3, 3), 1e4), rope.apply(k, pos2, hd, (2, 3, 3), 1e4))
    np.testing.assert_allclose(s1, s0, rtol=1e-12, atol=1e-12)
    # Shifting only one axis changes scores (the axes are really distinct).
    pos3 = pos.copy()
    pos3[:5, 1] += 3.0
    s2 = np.einsum("ihd,jhd->ij", rope.apply(q, pos3, hd, (2, 3, 3), 1e4), rope.apply(k, pos3, hd, (2, 3, 3), 1e4))
    assert np.abs(s2 - s0).max() > 1e-3


def test_mrope_preserves_pair_norms():
    hd = 16
    rng = np.random.default_rng(2)
    x = rng.standard_normal((5, 2, hd))
    pos = rng.uniform(0, 15000, size=(5, 3))
    y = rope.apply(x, pos, hd, (2, 3, 3), 1e4)
    n0 = x[..., :8] ** 2 + x[..., 8:] ** 2
    n1 = y[..., :8] ** 2 + y[..., 8:] ** 2
    np.testing.assert_allclose(n1, n0, rtol=1e-12)


def test_mrope_sections_select_axes():
    hd = 16
    sections = (2, 3, 3)
    x = np.random.default_rng(3).standard_normal((1, 1, hd))
    base = rope.apply(x, np.array([[5.0, 6.0, 7.0]]), hd, sections, 1e4)
    for axis, sl in ((0, slice(0, 2)), (1, slice(2, 5)), (2, slice(5, 8))):
        p = np.array([[5.0, 6.0, 7.0]])
        p[0, axis] += 1.0
        y = rope.apply(x, p, hd, sections, 1e4)
        changed = np.abs(y - base)[0, 0]
        pair_changed = (changed[:8] + changed[8:]) > 1e-12
        want = np.zeros(8, bool)
        want[sl] = True
        np.testing.assert_array_equal(pair_changed, want)


# ---------------------------------------------------------------- mask

@pytest.mark.parametrize("mode", [mask.FULL, mask.BLOCK_CAUSAL])
@pytest.mark.parametrize("seed", range(4))
def test_mask_vectorised_equals_equation_construction(mode, seed):
    rng = np.random.default_rng(seed)
    spec = LayoutSpec(n_text=int(rng.integers(0, 6)),
                      video=VideoSpec(int(rng.integers(1, 3)), 2, 2, 24, int(rng.integers(0, 3)), int(rng.integers(1, 3))),
                      audio_noisy=int(rng.integers(0, 4)), action_noisy=int(rng.integers(0, 4)))
    lay = layout.build_layout(spec)
    a = mask.allow_matrix(np.arange(lay.n_tokens), lay.region, lay.chunk, mode)
    b = mask.allow_matrix_from_equations(lay.region, lay.chunk, mode)
    np.testing.assert_array_equal(a, b)


def test_mask_semantics():
    lay = _small_layout(video=VideoSpec(1, 1, 2, 24, 1, 2))
    n_ar = lay.n_ar
    full = mask.allow_matrix(np.arange(lay.n_tokens), lay.region, lay.chunk, mask.FULL)
    bc = mask.allow_matrix(np.arange(lay.n_tokens), lay.region, lay.chunk, mask.BLOCK_CAUSAL)
    assert not full[:n_ar, n_ar:].any(), "AR never reads DM"
    np.testing.assert_array_equal(full[:n_ar, :n_ar], np.tril(np.ones((n_ar, n_ar), bool)))
    assert full[n_ar:, :].all(), "DM reads AR and all DM in full mode"
    assert bc[n_ar:, :n_ar].all()
    c = lay.chunk[n_ar:]
    np.testing.assert_array_equal(bc[n_ar:, n_ar:], c[None, :] <= c[:, None])
    assert bc.any(axis=1).all(), "no row is empty"


# ---------------------------------------------------------------- attention

def test_attention_matches_brute_force_loops():
    rng = np.random.default_rng(4)
    nq, nk, H, Hkv, hd = 6, 9, 4, 2, 5
    q = rng.standard_normal((nq, H, hd))
    k = rng.standard_normal((nk, Hkv, hd))
    v = rng.standard_normal((nk, Hkv, hd))
    allow = rng.random((nq, nk)) < 0.6
    allow[:, 0] = True
    allow[3] = False  # an empty row outputs zeros
    got = layer.attention(q, k, v, allow, 0.37)
    for i in range(nq):
        for h in range(H):
            g = h // (H // Hkv)
            keys = [j for j in range(nk) if allow[i, j]]
            if not keys:
                np.testing.assert_array_equal(got[i, h], 0.0)
                continue
            sc = [0.37 * sum(q[i, h, c] * k[j, g, c] for c in range(hd)) for j in keys]
            mx = max(sc)
            w = [np.exp(s - mx) for s in sc]
            tot = sum(w)
            want = [sum(w[t] / tot * v[keys[t], g, c] for t in range(len(keys))) for c in range(hd)]
            np.testing.assert_allclose(got[i, h], want, rtol=1e-12, atol=1e-13)


def test_attention_of_constant_values_is_constant():
    rng = np.random.default_rng(5)
    lay = _small_layout()
    n = lay.n_tokens
    q = rng.standard_normal((n, 2, 8)) * 3
    k = rng.standard_normal((n, 2, 8)) * 3
    v = np.ones((n, 2, 8))
    for mode in (mask.FULL, mask.BLOCK_CAUSAL):
        allow = mask.allow_matrix(np.arange(n), lay.region, lay.chunk, mode)
        np.testing.assert_allclose(layer.attention(q, k, v, allow, 0.5), 1.0, rtol=1e-14)


# ---------------------------------------------------------------- routing and passthrough

def _run(dims, W, h, lay, mode="full", s0=0.8, s1=0.7, **kw):
    return layer.layer_forward(dims, W, h, lay.region, lay.pos, lay.chunk, s0, s1, mode, **kw)


@pytest.mark.parametrize("mode", ["full", "block_causal"])
def test_ar_outputs_independent_of_dm_tokens_and_generator_weights(mode):
    lay = _small_layout()
    W = _weights(TINY)
    h = _h(lay.n_tokens, TINY.d_model)
    base = _run(TINY, W, h, lay, mode)
    h2 = h.copy()
    h2[lay.n_ar:] += np.random.default_rng(0).standard_normal(h2[lay.n_ar:].shape)
    W2 = _weights(TINY)
    for f in ("wq", "wk", "wv", "wo", "wg", "wu", "wd", "g1", "g2"):
        setattr(W2.G, f, getattr(W2.G, f) * 1.5 + 0.01)
    pert = _run(TINY, W2, h2, lay, mode)
    np.testing.assert_array_equal(pert["h2"][:lay.n_ar], base["h2"][:lay.n_ar])
    assert np.abs(pert["h2"][lay.n_ar:] - base["h2"][lay.n_ar:]).max() > 1e-3


def test_dm_outputs_use_reasoner_kv_but_not_reasoner_o_or_mlp():
    lay = _small_layout()
    W = _weights(TINY)
    h = _h(lay.n_tokens, TINY.d_model)
    base = _run(TINY, W, h, lay)
    W2 = _weights(TINY)
    for f in ("wo", "wg", "wu", "wd", "g2"):
        setattr(W2.R, f, getattr(W2.R, f) * -2.0)
    p = _run(TINY, W2, h, lay)
    np.testing.assert_array_equal(p["h2"][lay.n_ar:], base["h2"][lay.n_ar:])
    W3 = _weights(TINY)
    W3.R.wk = W3.R.wk * 3.0  # DM queries read AR keys
    p3 = _run(TINY, W3, h, lay)
    assert np.abs(p3["h2"][lay.n_ar:] - base["h2"][lay.n_ar:]).max() > 1e-6


# ---------------------------------------------------------------- layer stacks

def _stack(dims, n, seed=21):
    return [layer.weights_from_bits(dims, w) for w in synth.make_stack_weights(dims, seed, n)]


def test_stack_of_one_layer_is_the_layer():
    lay = _small_layout()
    Ws = _stack(TINY, 1)
    h = _h(lay.n_tokens, TINY.d_model)
    one = _run(TINY, Ws[0], h, lay)
    st = layer.stack_forward(TINY, Ws, h, lay.region, lay.pos, lay.chunk, 0.8, 0.7)
    np.testing.assert_array_equal(st["h_out"], one["h2"])
    np.testing.assert_array_equal(st["x_new"], one["x_new"])
    np.testing.assert_array_equal(st["vel"], one["vel"])


def test_stack_of_residual_only_layers_is_the_identity():
    """With W_o = W_down = 0 in every layer each layer returns its input, so the
    stack output is h and the step is the velocity head applied to h itself
    (closed form)."""
    lay = _small_layout()
    Ws = _stack(TINY, 3)
    for W in Ws:
        for s_ in (W.R, W.G):
            s_.wo = np.zeros_like(s_.wo)
            s_.wd = np.zeros_like(s_.wd)
    h = _h(lay.n_tokens, TINY.d_model)
    st = layer.stack_forward(TINY, Ws, h, lay.region, lay.pos, lay.chunk, 0.8, 0.7)
    np.testing.assert_array_equal(st["h_out"], h)
    noisy = lay.region == layout.REGION_NOISY
    g, wv = Ws[-1].gfin, Ws[-1].wvel
    x = h[noisy]
    v = (x / np.sqrt(np.mean(x * x, axis=1, keepdims=True) + TINY.eps) * g) @ wv.T
    np.testing.assert_allclose(st["x_new"][noisy], x - 0.1 * v, rtol=0, atol=1e-12)


@pytest.mark.parametrize("mode", ["full", "block_causal"])
def test_stack_ar_rows_independent_of_dm_rows_and_generator_weights(mode):
    """AR rows stay Reasoner-only through any depth: their outputs after every
    layer ignore DM inputs and every Generator weight (so AR K/V can be cached
    across sampler steps for a whole stack)."""
    lay = _small_layout()
    Ws = _stack(TINY, 3)
    h = _h(lay.n_tokens, TINY.d_model)
    base = layer.stack_forward(TINY, Ws, h, lay.region, lay.pos, lay.chunk, 0.8, 0.7, mode)
    h2 = h.copy()
    h2[lay.n_ar:] += 0.5
    Ws2 = _stack(TINY, 3)
    for W in Ws2:
        W.G.wv = W.G.wv * -1.0
        W.G.wd = W.G.wd * 2.0
    pert = layer.stack_forward(TINY, Ws2, h2, lay.region, lay.pos, lay.chunk, 0.8, 0.7, mode)
    for a, b in zip(base["hidden"], pert["hidden"]):
        np.testing.assert_array_equal(a[:lay.n_ar], b[:lay.n_ar])
    assert np.abs(pert["h_out"][lay.n_ar:] - base["h_out"][lay.n_ar:]).max() > 1e-3


def test_stack_clean_rows_read_noisy_rows_from_the_second_layer():
    """Full mask: clean DM rows attend to noisy rows, so after the first layer
    their hidden state (and the next layer's clean K/V) changes with the noisy
    state; block-causal: clean chunks before every noisy chunk do not."""
    lay = _small_layout(video=VideoSpec(1, 2, 3, 24, 1, 2))
    Ws = _stack(TINY, 2)
    h = _h(lay.n_tokens, TINY.d_model)
    clean = lay.region == layout.REGION_CLEAN
    noisy = lay.region == layout.REGION_NOISY
    h2 = h.copy()
    h2[noisy] += 0.5
    for mode, changes in (("full", True), ("block_causal", False)):
        a = layer.stack_forward(TINY, Ws, h, lay.region, lay.pos, lay.chunk, 0.8, 0.7, mode)
        b = layer.stack_forward(TINY, Ws, h2, lay.region, lay.pos, lay.chunk, 0.8, 0.7, mode)
        d = np.abs(a["hidden"][0][clean] - b["hidden"][0][clean]).max()
        assert (d > 1e-6) == changes, (mode, d)


# ---------------------------------------------------------------- schedules and action heads

def test_shift_schedule_properties():
    """sigma = s t_bar / (1 + (s - 1) t_bar): identity at s = 1, endpoints 1
    and 0, strictly decreasing, and t_bar = sigma / (s - (s - 1) sigma) maps it
    back onto the uniform grid (the closed-form inverse)."""
    np.testing.assert_array_equal(layer.shift_sigmas(10, 1.0), 1.0 - np.arange(11) / 10)
    for s_ in (0.5, 3.0, 5.0, 10.0):
        sig = layer.shift_sigmas(7, s_)
        assert sig[0] == 1.0 and sig[-1] == 0.0
        assert np.all(np.diff(sig) < 0)
        t_bar = sig / (s_ - (s_ - 1.0) * sig)
        np.testing.assert_allclose(t_bar, 1.0 - np.arange(8) / 7, rtol=0, atol=1e-15)
    # a shift above 1 spends more of the steps at high noise
    assert np.all(layer.shift_sigmas(4, 5.0)[1:-1] > layer.shift_sigmas(4, 1.0)[1:-1])
    from fractions import Fraction as Fr
    want = [Fr(1), Fr(15, 16), Fr(5, 6), Fr(5, 8), Fr(0)]  # 4 steps, shift 5, by hand
    np.testing.assert_allclose(layer.shift_sigmas(4, 5.0), [float(v) for v in want], rtol=0, atol=1e-15)


def _policy_case(n_layers=2, residual_only=False):
    spec = LayoutSpec(n_text=5, video=VideoSpec(1, 2, 3, 24, 1, 1), action_clean=3, action_noisy=4, action_hz=15)
    lay = layout.build_layout(spec)
    Ws = _stack(TINY, n_layers)
    if residual_only:
        for W in Ws:
            for s_ in (W.R, W.G):
                s_.wo = np.zeros_like(s_.wo)
                s_.wd = np.zeros_like(s_.wd)
    ca = 6
    w_in = synth.bf16_to_f64(synth.normal_bf16((TINY.d_model, ca), 40, 1, std=0.3))
    w_out = synth.bf16_to_f64(synth.normal_bf16((ca, TINY.d_model), 41, 1, std=0.1))
    x_a = synth.bf16_to_f64(synth.normal_bf16((7, ca), 42, 1))
    h = _h(lay.n_tokens, TINY.d_model)
    return lay, Ws, w_in, w_out, x_a, h


def test_policy_step_with_residual_only_layers_is_the_closed_form():
    """Residual-only layers pass the embedded actions through, so the action
    velocity is RMSNorm(x_a W_in^T; g_fin) W_out^T exactly (closed form); clean
    actions stay put; the action rows of h carry the embedding."""
    lay, Ws, w_in, w_out, x_a, h = _policy_case(residual_only=True)
    h_new, xa_new = layer.policy_step(TINY, Ws, h, x_a, w_in, w_out, lay, 0.9, 0.7, 0.6, 0.5)
    e = x_a[3:] @ w_in.T
    v = (e / np.sqrt(np.mean(e * e, axis=1, keepdims=True) + TINY.eps) * Ws[-1].gfin) @ w_out.T
    np.testing.assert_allclose(xa_new[3:], x_a[3:] - 0.1 * v, rtol=0, atol=1e-12)
    np.testing.assert_array_equal(xa_new[:3], x_a[:3])
    act = lay.modality == layout.MOD_ACTION
    np.testing.assert_allclose(h_new[act], x_a @ w_in.T, rtol=0, atol=1e-12)


def test_policy_step_modalities_have_their_own_noise_levels():
    lay, Ws, w_in, w_out, x_a, h = _policy_case()
    vid = (lay.region == layout.REGION_NOISY) & (lay.modality != layout.MOD_ACTION)
    h1, xa1 = layer.policy_step(TINY, Ws, h, x_a, w_in, w_out, lay, 0.9, 0.7, 0.6, 0.6)
    np.testing.assert_array_equal(xa1, x_a)  # action noise level held: actions do not move
    assert np.abs(h1[vid] - h[vid]).max() > 1e-4
    h2, xa2 = layer.policy_step(TINY, Ws, h, x_a, w_in, w_out, lay, 0.9, 0.9, 0.6, 0.4)
    np.testing.assert_array_equal(h2[vid], h[vid])  # video held
    assert np.abs(xa2[3:] - x_a[3:]).max() > 1e-4
    # the same forward pass: the action step is linear in its sigma step
    _, xa3 = layer.policy_step(TINY, Ws, h, x_a, w_in, w_out, lay, 0.9, 0.9, 0.6, 0.2)
    np.testing.assert_allclose(xa3[3:] - x_a[3:], 2.0 * (xa2[3:] - x_a[3:]), rtol=1e-12, atol=1e-15)


def test_policy_step_guidance_limits():
    """Guidance 1 is the conditioned pass alone; guidance 0 the baseline alone."""
    lay, Ws, w_in, w_out, x_a, h = _policy_case()
    hb = h.copy()
    hb[:lay.n_ar] = _h(lay.n_ar, TINY.d_model, seed=99)
    c = layer.policy_step(TINY, Ws, h, x_a, w_in, w_out, lay, 0.9, 0.7, 0.6, 0.5)
    b = layer.policy_step(TINY, Ws, hb, x_a, w_in, w_out, lay, 0.9, 0.7, 0.6, 0.5)
    g1 = layer.policy_step(TINY, Ws, h, x_a, w_in, w_out, lay, 0.9, 0.7, 0.6, 0.5, guidance=1.0, h_base=hb,
                           x_a_base=x_a)
    g0 = layer.policy_step(TINY, Ws, h, x_a, w_in, w_out, lay, 0.9, 0.7, 0.6, 0.5, guidance=0.0, h_base=hb,
                           x_a_base=x_a)
    noisy = lay.region == layout.REGION_NOISY
    np.testing.assert_allclose(g1[1], c[1], rtol=0, atol=1e-13)
    np.testing.assert_allclose(g0[1], b[1], rtol=0, atol=1e-13)
    np.testing.assert_allclose(g1[0][noisy], c[0][noisy], rtol=0, atol=1e-13)
    np.testing.assert_allclose(g0[0][noisy], b[0][noisy], rtol=0, atol=1e-13)


def test_clean_rows_pass_through_unchanged():
    lay = _small_layout(video=VideoSpec(1, 2, 2, 24, 2, 2), proprio=1)
    W = _weights(TINY)
    h = _h(lay.n_tokens, TINY.d_model)
    out = _run(TINY, W, h, lay)
    clean = lay.region == layout.REGION_CLEAN
    np.testing.assert_array_equal(out["x_new"][clean], h[clean])
    assert np.isnan(out["vel"][clean]).all()
    noisy = lay.region == layout.REGION_NOISY
    assert np.abs(out["x_new"][noisy] - h[noisy]).max() > 1e-4


def test_dm_permutation_equivariance_without_rope():
    lay = _small_layout(video=VideoSpec(1, 2, 2, 24, 1, 2))
    W = _weights(TINY)
    h = _h(lay.n_tokens, TINY.d_model)
    pos0 = np.zeros_like(lay.pos)  # RoPE off: every rotation is the identity
    perm = np.arange(lay.n_tokens)
    rng = np.random.default_rng(6)
    perm[lay.n_ar:] = lay.n_ar + rng.permutation(lay.n_dm)
    a = layer.layer_forward(TINY, W, h, lay.region, pos0, lay.chunk, 0.8, 0.7)
    b = layer.layer_forward(TINY, W, h[perm], lay.region[perm], pos0, lay.chunk[perm], 0.8, 0.7)
    np.testing.assert_allclose(b["h2"], a["h2"][perm], rtol=0, atol=1e-12)
    np.testing.assert_allclose(np.nan_to_num(b["x_new"]), np.nan_to_num(a["x_new"][perm]), atol=1e-12)


# ---------------------------------------------------------------- composition with special weights

def _zero_set(dims):
    d, f, qc, kc = dims.d_model, dims.ffn, dims.q_cols, dims.kv_cols
    z = np.zeros
    return layer.SetWeights(g1=np.ones(d), wq=z((qc, d)), wk=z((kc, d)), wv=z((kc, d)), wo=z((d, qc)),
                            g2=np.ones(d), wg=z((f, d)), wu=z((f, d)), wd=z((d, f)))


def test_residual_mask_and_value_path_closed_form():
    """Wq = Wk = 0 makes attention a plain mean over visible keys.  With Wv a
    permutation P and Wo = I, h2_i = h_i + mean_{j visible to i} P a_j."""
    dims = ModelDims(d_model=16, n_heads=2, n_kv_heads=2, head_dim=8, ffn=8, rope_sections=(1, 1, 2))
    lay = _small_layout(n_text=3, video=VideoSpec(1, 1, 2, 24, 1, 2))
    rng = np.random.default_rng(7)
    P = np.eye(16)[rng.permutation(16)]
    sets = {}
    for s in "RG":
        ws = _zero_set(dims)
        ws.g1 = 1.0 + 0.1 * rng.standard_normal(16)
        ws.wv = P.copy()
        ws.wo = np.eye(16)
        sets[s] = ws
    W = layer.LayerWeights(R=sets["R"], G=sets["G"], gfin=np.ones(16), wvel=np.eye(16))
    h = rng.standard_normal((lay.n_tokens, 16))
    for mode in ("full", "block_causal"):
        out = layer.layer_forward(dims, W, h, lay.region, lay.pos, lay.chunk, 0.5, 0.25, mode)
        for i in range(lay.n_tokens):
            vis = []
            for j in range(lay.n_tokens):
                if lay.region[i] == layout.REGION_AR:
                    ok = lay.region[j] == layout.REGION_AR and j <= i
                else:
                    ok = lay.region[j] == layout.REGION_AR or mode == "full" or lay.chunk[j] <= lay.chunk[i]
                if ok:
                    vis.append(j)
            vals = []
            for j in vis:
                g = sets["R" if lay.region[j] == layout.REGION_AR else "G"].g1
                a = h[j] * g / np.sqrt(np.mean(h[j] ** 2) + 1e-6)
                vals.append(P @ a)
            np.testing.assert_allclose(out["h2"][i], h[i] + np.mean(vals, axis=0), rtol=0, atol=1e-12)


def test_gated_ffn_and_velocity_head_closed_form():
    """Attention branch off (Wo = 0); Wg = [I;0], Wu = [cI;0], Wd = [I,0]:
    h2 = h + silu(b) * c b with b = RMSNorm(h; g2).  Wvel = P gives
    x' = x + (s1 - s0) P RMSNorm(h2; gfin) on noisy rows."""
    d, f = 8, 24
    dims = ModelDims(d_model=d, n_heads=1, n_kv_heads=1, head_dim=8, ffn=f, rope_sections=(1, 1, 2))
    lay = _small_layout(n_text=2, video=VideoSpec(1, 1, 2, 24, 1, 1))
    rng = np.random.default_rng(8)
    c = 0.75
    sets = {}
    for s, cs in (("R", c), ("G", -c)):
        ws = _zero_set(dims)
        ws.g2 = 1.0 + 0.1 * rng.standard_normal(d)
        ws.wg = np.zeros((f, d)); ws.wg[:d] = np.eye(d)
        ws.wu = np.zeros((f, d)); ws.wu[:d] = cs * np.eye(d)
        ws.wd = np.zeros((d, f)); ws.wd[:, :d] = np.eye(d)
        sets[s] = ws
    P = np.eye(d)[rng.permutation(d)]
    gfin = 1.0 + 0.1 * rng.standard_normal(d)
    W = layer.LayerWeights(R=sets["R"], G=sets["G"], gfin=gfin, wvel=P)
    h = rng.standard_normal((lay.n_tokens, d)) * 2
    s0, s1 = 0.9, 0.6
    out = layer.layer_forward(dims, W, h, lay.region, lay.pos, lay.chunk, s0, s1)
    for i in range(lay.n_tokens):
        s = "R" if lay.region[i] == layout.REGION_AR else "G"
        b = h[i] * sets[s].g2 / np.sqrt(np.mean(h[i] ** 2) + 1e-6)
        cs = c if s == "R" else -c
        h2 = h[i] + b / (1 + np.exp(-b)) * (cs * b)
        np.testing.assert_allclose(out["h2"][i], h2, rtol=0, atol=1e-12)
        if lay.region[i] == layout.REGION_NOISY:
            n = h2 * gfin / np.sqrt(np.mean(h2 ** 2) + 1e-6)
            np.testing.assert_allclose(out["x_new"][i], h[i] + (s1 - s0) * (P @ n), rtol=0, atol=1e-12)


def test_rmsnorm_and_silu_closed_forms():
    g = np.array([1.0, 2.0, -0.5, 3.0])
    for c in (-3.0, 0.25, 7.0):
        np.testing.assert_allclose(layer.rms_norm(np.full(4, c), g, 1e-6), g * c / np.sqrt(c * c + 1e-6), rtol=1e-15)
    x = np.random.default_rng(9).standard_normal(32)
    np.testing.assert_allclose(layer.rms_norm(5 * x, g[0], 0.0), layer.rms_norm(x, g[0], 0.0), rtol=1e-14)
    z = np.linspace(-30, 30, 121)
    np.testing.assert_allclose(layer.silu(z) - layer.silu(-z), z, atol=1e-12)
    assert layer.silu(0.0) == 0.0
    np.testing.assert_allclose(layer.silu(np.array([40.0])), 40.0, rtol=1e-15)


# ---------------------------------------------------------------- sampler

def test_euler_is_exact_on_the_linear_flow_path():
    """§6.3 path x_s = s eps + (1 - s) x0 has constant velocity v* = eps - x0;
    §7.2 Euler steps from s = 1 to 0 therefore land on x0."""
    rng = np.random.default_rng(10)
    x0 = rng.standard_normal(1000)
    eps = rng.standard_normal(1000)
    sig = synth.preset("droid").sigmas
    assert sig[0] == 1.0 and sig[-1] == 0.0 and all(a > b for a, b in zip(sig, sig[1:]))
    x = eps.copy()
    for s0, s1 in zip(sig[:-1], sig[1:]):
        np.testing.assert_allclose(x, s0 * eps + (1 - s0) * x0, atol=1e-12)
        x = layer.euler_step(x, eps - x0, s0, s1)
    np.testing.assert_allclose(x, x0, atol=1e-12)
    # sigma_next == sigma leaves x unchanged.
    np.testing.assert_array_equal(layer.euler_step(x0, eps, 0.3, 0.3), x0)


def test_sampler_loop_equals_repeated_steps():
    lay = _small_layout()
    W = _weights(TINY)
    h = _h(lay.n_tokens, TINY.d_model)
    sig = (1.0, 0.6, 0.0)
    hf, outs = layer.sample(TINY, W, h, lay, sig)
    h1 = h.copy()
    noisy = lay.region == layout.REGION_NOISY
    for s0, s1 in zip(sig[:-1], sig[1:]):
        o = _run(TINY, W, h1, lay, s0=s0, s1=s1)
        h1[noisy] = o["x_new"][noisy]
    np.testing.assert_array_equal(hf, h1)
    np.testing.assert_array_equal(hf[~noisy], h[~noisy])


# ---------------------------------------------------------------- guidance

def _cfg_case():
    lay = _small_layout(video=VideoSpec(1, 2, 2, 24, 1, 2))
    W = _weights(TINY)
    hc = _h(lay.n_tokens, TINY.d_model, seed=21)
    hb = hc.copy()
    hb[:lay.n_ar] = _h(lay.n_ar, TINY.d_model, seed=22)  # a different prompt, same DM rows
    return lay, W, hc, hb


def test_cfg_limits_reduce_to_single_passes():
    """w = 1 is the conditioned step, w = 0 the baseline step (§7.2)."""
    lay, W, hc, hb = _cfg_case()
    noisy = lay.region == layout.REGION_NOISY
    x1, oc, ob = layer.cfg_step(TINY, W, hc, hb, lay, 0.8, 0.7, 1.0)
    np.testing.assert_allclose(x1, oc["x_new"][noisy], rtol=0, atol=1e-13)
    x0, _, _ = layer.cfg_step(TINY, W, hc, hb, lay, 0.8, 0.7, 0.0)
    np.testing.assert_allclose(x0, ob["x_new"][noisy], rtol=0, atol=1e-13)
    assert np.abs(x1 - x0).max() > 1e-4, "the prompt must matter"


def test_cfg_is_affine_in_guidance_and_inert_for_equal_prompts():
    lay, W, hc, hb = _cfg_case()
    xs = [layer.cfg_step(TINY, W, hc, hb, lay, 0.8, 0.7, g)[0] for g in (0.0, 3.0, 6.0)]
    np.testing.assert_allclose(xs[2] - xs[1], xs[1] - xs[0], rtol=0, atol=1e-12)
    # guidance weight w extrapolates past the conditioned velocity: x(6) - x(0) = 6 (x(1) - x(0))
    x1 = layer.cfg_step(TINY, W, hc, hb, lay, 0.8, 0.7, 1.0)[0]
    np.testing.assert_allclose(xs[2] - xs[0], 6.0 * (x1 - xs[0]), rtol=0, atol=1e-12)
    same = [layer.cfg_step(TINY, W, hc, hc, lay, 0.8, 0.7, g)[0] for g in (0.0, 7.5)]
    np.testing.assert_allclose(same[0], same[1], rtol=0, atol=1e-13)
    with pytest.raises(ValueError):
        hb2 = hb.copy()
        hb2[-1] += 1.0
        layer.cfg_step(TINY, W, hc, hb2, lay, 0.8, 0.7, 2.0)


# ---------------------------------------------------------------- streaming

def test_stream_cache_equals_block_causal_sequence():
    """A block denoised against committed history K/V equals the same block as
    the last chunk of one packed block-causal sequence holding the history."""
    dims = TINY
    W = _weights(dims)
    vid = VideoSpec(1, 2, 2, 24, 0, 1)
    spec_blk = LayoutSpec(n_text=3, video=vid)
    hist = 3
    rng_h = _h(spec_blk.n_ar + (hist + 1) * vid.tokens_per_step, dims.d_model, seed=12)
    h_ar = rng_h[:spec_blk.n_ar]
    blocks = [rng_h[spec_blk.n_ar + b * 4: spec_blk.n_ar + (b + 1) * 4] for b in range(hist + 1)]
    st = layer.StreamState(slots=hist)
    for b in range(hist):
        lb = layout.build_layout(spec_blk, tau_offset=b)
        layer.stream_commit(dims, W, st, blocks[b], lb)
    lcur = layout.build_layout(spec_blk, tau_offset=hist)
    x, out = layer.stream_block(dims, W, st, h_ar, blocks[hist], lcur, (0.8, 0.7))
    # Same thing as one sequence: history blocks as clean DM rows, then the block.
    big = layout.build_layout(LayoutSpec(n_text=3, video=VideoSpec(1, 2, 2, 24, hist, 1)))
    hb = np.concatenate([h_ar] + blocks)
    ref = layer.layer_forward(dims, W, hb, big.region, big.pos, big.chunk, 0.8, 0.7, mode="block_causal")
    np.testing.assert_allclose(out["h2"], ref["h2"][-4:], rtol=0, atol=1e-12)
    np.testing.assert_allclose(x, ref["x_new"][-4:], rtol=0, atol=1e-12)
    np.testing.assert_array_equal(lcur.pos, big.pos[np.r_[0:big.n_ar, big.n_tokens - 4:big.n_tokens]])


def test_stream_ring_evicts_oldest():
    st = layer.StreamState(slots=2)
    for b in range(3):
        st.commit(np.full((1, 1, 1), b), np.full((1, 1, 1), b), np.array([b]))
    k, v, c = st.cache()
    assert sorted(c.tolist()) == [1, 2]
