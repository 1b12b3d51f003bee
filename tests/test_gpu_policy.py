"""Action heads and the policy step on the GPU against the fp64 oracle (needs a
B200).  "Cosmos 3 方法原理全解" §4.2 (domain W_in / W_out, the sampler in the
normalised action space), §6.3 (per-modality noise levels), §7.2-7.3 (guided
step)."""

import numpy as np
import pytest

import synth
from oracle import layer as olayer
from oracle import layout as olayout
from synth import LayoutSpec, ModelDims, VideoSpec
from tolerance import SIGMA_VEL, assert_close, rms

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():  # pragma: no cover
    pytest.skip("no CUDA device", allow_module_level=True)

from flow_matching_dit_cosmot_b200 import api as A  # noqa: E402
from flow_matching_dit_cosmot_b200 import _lib as L  # noqa: E402
from gpu_helpers import assert_device_ok, bits, device_weights, dims as cdims, layout_spec, to_dev, to_f64  # noqa

GQA = ModelDims(d_model=512, n_heads=4, n_kv_heads=2, head_dim=128, ffn=1536, rope_sections=(16, 24, 24))


@pytest.mark.parametrize("ca", [8, 10])
def test_action_embed_kernel(ca):
    d = 512
    w_in, _ = synth.make_action_weights(d, ca, 51)
    x = synth.make_actions(50, ca, 52)
    segs = [(0, 7, 3, 0, 0), (7, 20, 40, 0, 0), (20, 50, 100, 0, 0)]
    h = torch.zeros((140, d), dtype=torch.bfloat16, device="cuda")
    xd, wd = to_dev(x), to_dev(w_in)
    L.cosmot_action_embed(A.ptr(xd), ca, segs, A.ptr(wd), ca, d, A.ptr(h), d, A.stream_handle())
    torch.cuda.synchronize()
    assert_device_ok()
    ref = olayer.action_embed(synth.bf16_to_f64(x), synth.bf16_to_f64(w_in))
    got = to_f64(h)
    for r0, r1, o, _, _ in segs:
        assert_close(got[o:o + r1 - r0], ref[r0:r1], f"embed rows {r0}-{r1}")
    untouched = np.ones(140, bool)
    for r0, r1, o, _, _ in segs:
        untouched[o:o + r1 - r0] = False
    assert not bits(h)[untouched].any()


@pytest.mark.parametrize("guidance", [None, 3.0])
def test_action_head_kernel(guidance):
    d, ca = 512, 8
    _, w_out = synth.make_action_weights(d, ca, 53)
    g = synth.normal_bf16((d,), 54, 1, std=0.02, mean=1.0)
    hl = synth.make_activations(64, d, 55)
    x0 = synth.make_actions(32, ca, 56)
    # two groups of 16 rows each: h rows 0-15 -> x rows 0-15, h rows 40-55 -> x rows 16-31
    segs = [(0, 16, 0, 0, 0), (40, 56, 16, 0, 0)]
    x = x0.copy()
    if guidance is not None:
        x[16:] = x[:16]  # a (conditioned, baseline) pair shares its state
    xd, hd_, gd, wd = to_dev(x), to_dev(hl), to_dev(g), to_dev(w_out)
    L.cosmot_action_head(A.ptr(hd_), d, segs, A.ptr(gd), 1e-6, A.ptr(wd), ca, d, A.ptr(xd), ca, 0.8, 0.55,
                         guidance, A.stream_handle())
    torch.cuda.synchronize()
    assert_device_ok()
    dims = ModelDims(d_model=d, n_heads=4, n_kv_heads=4, head_dim=128, ffn=1024, rope_sections=(16, 24, 24))
    h64, g64, w64, x64 = (synth.bf16_to_f64(a) for a in (hl, g, w_out, x))
    v0 = olayer.action_velocity(dims, h64[0:16], g64, w64)
    v1 = olayer.action_velocity(dims, h64[40:56], g64, w64)
    if guidance is None:
        want = np.concatenate([olayer.euler_step(x64[:16], v0, 0.8, 0.55), olayer.euler_step(x64[16:], v1, 0.8, 0.55)])
        v = np.concatenate([v0, v1])
    else:
        v = olayer.cfg_combine(v0, v1, guidance)
        one = olayer.euler_step(x64[:16], v, 0.8, 0.55)
        want = np.concatenate([one, one])
        np.testing.assert_array_equal(bits(xd)[:16], bits(xd)[16:])
    # bf16 inputs, fp32 norm, dot products and combine: no intermediate bf16 storage
    assert_close(to_f64(xd), want, "action head x'")


def _policy_setup(batch, guided):
    spec = LayoutSpec(n_text=40, video=VideoSpec(1, 4, 6, 24, 1, 2), action_clean=8, action_noisy=16, action_hz=15)
    lay = olayout.build_layout(spec)
    n, d, ca = lay.n_tokens, GQA.d_model, 8
    w = synth.make_stack_weights(GQA, 3300, 2)
    W = [olayer.weights_from_bits(GQA, x) for x in w]
    w_in, w_out = synth.make_action_weights(d, ca, 3400)
    na = 24
    h = np.stack([synth.make_activations(n, d, 3500 + 100 * b) for b in range(batch)])
    xa = np.concatenate([synth.make_actions(na, ca, 3600 + b) for b in range(batch)])
    if guided:  # each pair shares its DM rows and action state; the prompts differ
        for p in range(batch // 2):
            h[2 * p + 1, lay.n_ar:] = h[2 * p, lay.n_ar:]
            xa[(2 * p + 1) * na:(2 * p + 2) * na] = xa[2 * p * na:(2 * p + 1) * na]
    return spec, lay, w, W, w_in, w_out, h, xa, ca, na


@pytest.mark.parametrize("guided", [False, True])
def test_policy_step(guided):
    batch = 2
    spec, lay, w, W, w_in, w_out, h, xa, ca, na = _policy_setup(batch, guided)
    dlay = A.build_layout(layout_spec(A, spec))
    cs = A.mrope_table(dlay.pos, GQA.head_dim, GQA.rope_sections)
    stack = A.MoTStack(cdims(A, GQA), [device_weights(x) for x in w])
    seq = stack.seq_desc(lay.n_ar, lay.n_clean, lay.n_noisy, batch, cs, dlay.chunk)
    hd_, xd = to_dev(h), to_dev(xa)
    h_out = torch.empty_like(hd_)
    wi, wo = to_dev(w_in), to_dev(w_out)
    act_rows = np.nonzero(lay.modality == olayout.MOD_ACTION)[0]
    clean_row = int(act_rows[0])
    act = L.ActionDesc(ca, 8, 16, clean_row, A.ptr(wi), A.ptr(wo), A.ptr(xd), ca, 0.8, 0.5)
    ws = stack.workspace(seq)
    gw = 3.0 if guided else None
    L.cosmot_policy_step(stack.dims, stack.cw, seq, act, A.ptr(hd_), A.ptr(h_out), 0.9, 0.7, gw, A.ptr(ws),
                         ws.numel(), A.stream_handle())
    torch.cuda.synchronize()
    assert_device_ok()
    noisy = lay.region == olayout.REGION_NOISY
    act_m = lay.modality == olayout.MOD_ACTION
    vid = noisy & ~act_m
    w_in64, w_out64 = synth.bf16_to_f64(w_in), synth.bf16_to_f64(w_out)
    for p in range(batch // 2 if guided else batch):
        b = 2 * p if guided else p
        kw = {}
        if guided:
            kw = dict(guidance=gw, h_base=synth.bf16_to_f64(h[b + 1]),
                      x_a_base=synth.bf16_to_f64(xa[(b + 1) * na:(b + 2) * na]))
        h_ref, xa_ref = olayer.policy_step(GQA, W, synth.bf16_to_f64(h[b]), synth.bf16_to_f64(xa[b * na:(b + 1) * na]),
                                           w_in64, w_out64, lay, 0.9, 0.7, 0.8, 0.5, **kw)
        got_h = to_f64(hd_[b])
        # the step's own size |dsigma| rms(v) scales the rounding terms; a guided
        # velocity v_base + w (v_cond - v_base) carries the two passes' errors
        # with weights (1 - w) and w, and the hidden-space velocities are stored
        # in bf16 before the combine (one more rounding unit)
        h64, xa64 = synth.bf16_to_f64(h[b]), synth.bf16_to_f64(xa[b * na:(b + 1) * na])
        mix = float(np.hypot(1.0 - gw, gw)) if guided else 1.0
        sig_v = float(np.hypot(SIGMA_VEL, 1.0)) if guided else SIGMA_VEL
        br_v = mix * rms(h_ref[vid] - h64[vid])
        br_a = mix * rms(xa_ref[8:] - xa64[8:])
        assert_close(got_h[vid], h_ref[vid], f"policy video x' [{b}]", sigma=sig_v, branch_rms=br_v, depth=2)
        assert_close(got_h[act_m], h_ref[act_m], f"policy action embedding [{b}]")
        got_x = to_f64(xd)[b * na:(b + 1) * na]
        assert_close(got_x[8:], xa_ref[8:], f"policy action x' [{b}]", sigma=SIGMA_VEL, branch_rms=br_a, depth=2)
        np.testing.assert_array_equal(bits(xd)[b * na:b * na + 8], xa[b * na:b * na + 8])  # clean actions stay
        keep = ~noisy & ~act_m
        np.testing.assert_array_equal(bits(hd_[b])[keep], h[b][keep])
        if guided:  # both states of the pair receive the same step
            np.testing.assert_array_equal(bits(hd_[b])[noisy], bits(hd_[b + 1])[noisy])
            np.testing.assert_array_equal(bits(xd)[b * na:(b + 1) * na], bits(xd)[(b + 1) * na:(b + 2) * na])
