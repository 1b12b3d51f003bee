"""Parity at the workloads' full sizes, in the launch configuration bench.py
times, on sampled output rows the oracle computes one by one (needs a B200).

The oracle forms K and V of every row in float64 and the full layer only for
the sampled rows (every segment's first and last row plus a seeded random
subset), so each case takes seconds to a minute of host time.
"""

import numpy as np
import pytest

import synth
from oracle import layer as olayer
from oracle import layout as olayout
from tolerance import assert_close

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():  # pragma: no cover
    pytest.skip("no CUDA device", allow_module_level=True)

from flow_matching_dit_cosmot_b200 import api as A  # noqa: E402
from flow_matching_dit_cosmot_b200 import _lib as L  # noqa: E402
from gpu_helpers import assert_device_ok, bits, device_weights, dims as cdims, layout_spec, sample_rows, to_dev, to_f64  # noqa

_W = {}


def _weights(wl):
    if wl.name not in _W:
        _W.clear()  # keep one workload's weights at a time
        w = synth.make_weights(wl.dims, wl.weight_seed)
        _W[wl.name] = (w, device_weights(w), olayer.weights_from_bits(wl.dims, w))
    return _W[wl.name]


@pytest.mark.parametrize("name", ["t2v480", "i2v720", "t2v480_nano", "i2v720_super"])
def test_full_size_layer_on_sampled_rows(name):
    wl = synth.preset(name)
    w, dw, W = _weights(wl)
    lay = olayout.build_layout(wl.layout)
    n = lay.n_tokens
    h = synth.make_activations(n, wl.dims.d_model, wl.act_seed())
    dlay = A.build_layout(layout_spec(A, wl.layout))
    cs = A.mrope_table(dlay.pos, wl.dims.head_dim, wl.dims.rope_sections, wl.dims.rope_base)
    layer = A.MoTLayer(cdims(A, wl.dims), dw)
    seq = layer.seq_desc(dlay.n_ar, dlay.n_clean, dlay.n_noisy, 1, cs, dlay.chunk)
    hd_ = to_dev(h)
    h_out = torch.empty_like(hd_)
    s0, s1 = wl.sigmas[0], wl.sigmas[1]
    layer.forward(hd_, h_out, s0, s1, seq)
    torch.cuda.synchronize()
    assert_device_ok()
    np.testing.assert_array_equal(dlay.pos.cpu().numpy().view(np.uint32), lay.pos.view(np.uint32))

    z0 = lay.n_ar + lay.n_clean
    rows = sample_rows(n, [(0, lay.n_ar), (lay.n_ar, z0), (z0, n)], 96, seed=7)
    ref = olayer.layer_forward(wl.dims, W, synth.bf16_to_f64(h), lay.region, lay.pos, lay.chunk, s0, s1,
                               wl.mask_mode, rows=rows)
    assert_close(to_f64(h_out)[rows], ref["h2"], f"{name} h_out (sampled rows)", rounded_inputs=3)
    noisy = lay.region[rows] == olayout.REGION_NOISY
    vel = ref["vel"][noisy]
    assert_close(to_f64(hd_)[rows][noisy], ref["x_new"][noisy], f"{name} x' (sampled noisy rows)", rounded_inputs=2,
                 branch_rms=abs(s1 - s0) * float(np.sqrt(np.mean(vel ** 2))))
    # clean and AR rows of h are untouched
    keep = lay.region != olayout.REGION_NOISY
    np.testing.assert_array_equal(bits(hd_)[keep], h[keep])


def test_full_width_droid_sampler():
    """DROID policy step at d_model 4096: the 10-step sampler with AR K/V kept
    in the workspace after step 1, against the oracle's full recomputation."""
    wl = synth.preset("droid")
    w, dw, W = _weights(wl)
    lay = olayout.build_layout(wl.layout)
    n = lay.n_tokens
    h0 = synth.make_activations(n, wl.dims.d_model, wl.act_seed())
    dlay = A.build_layout(layout_spec(A, wl.layout))
    cs = A.mrope_table(dlay.pos, wl.dims.head_dim, wl.dims.rope_sections, wl.dims.rope_base)
    layer = A.MoTLayer(cdims(A, wl.dims), dw)
    h = to_dev(h0)
    h_out = torch.empty_like(h)
    ws = None
    states = []
    sig = wl.sigmas
    for k, (s0, s1) in enumerate(zip(sig[:-1], sig[1:])):
        seq = layer.seq_desc(dlay.n_ar, dlay.n_clean, dlay.n_noisy, 1, cs, dlay.chunk, n_cached=dlay.n_ar if k else 0)
        if ws is None:
            ws = torch.empty(layer.workspace_bytes(seq), dtype=torch.uint8, device="cuda")
        layer.forward(h, h_out, s0, s1, seq, workspace=ws)
        states.append(h.clone())
    torch.cuda.synchronize()
    assert_device_ok()
    _, outs = olayer.sample(wl.dims, W, synth.bf16_to_f64(h0), lay, sig)
    noisy = lay.region == olayout.REGION_NOISY
    vel_rms = float(np.sqrt(np.mean(np.concatenate([o["vel"][noisy] for o in outs]) ** 2)))
    for k, o in enumerate(outs):
        assert_close(to_f64(states[k])[noisy], o["x_new"][noisy], f"droid x after step {k + 1}", rounded_inputs=2,
                     branch_rms=vel_rms, n_steps=k + 1)


def test_full_width_streaming_step():
    """One denoising step of a 1,560-token block against the 8-block cache and
    the 66 AR rows, at d_model 4096, on sampled block rows."""
    wl = synth.preset("stream")
    w, dw, W = _weights(wl)
    v = wl.layout.video
    hist = wl.stream.cached_blocks
    spec_blk = synth.LayoutSpec(n_text=wl.layout.n_text, video=v)
    lay_blk = olayout.build_layout(spec_blk, tau_offset=hist)
    n_ar, T = lay_blk.n_ar, lay_blk.n_noisy
    h_ar = synth.make_activations(n_ar, wl.dims.d_model, wl.act_seed())
    hist_x = [synth.make_activations(T, wl.dims.d_model, 4000 + k) for k in range(hist)]
    x0 = synth.make_activations(T, wl.dims.d_model, 5000)
    layer = A.MoTLayer(cdims(A, wl.dims), dw)
    dl = A.build_layout(A.layout_spec(wl.layout.n_text, (v.views, v.grid_h, v.grid_w, v.fps, hist, 1)))
    cs = A.mrope_table(dl.pos, wl.dims.head_dim, wl.dims.rope_sections, wl.dims.rope_base)
    seq0 = layer.seq_desc(dl.n_ar, dl.n_clean, dl.n_noisy, 1, cs, dl.chunk, L.COSMOT_MASK_BLOCK_CAUSAL)
    h = to_dev(np.concatenate([h_ar] + hist_x + [x0]))
    ws = torch.empty(layer.workspace_bytes(seq0), dtype=torch.uint8, device="cuda")
    layer.commit_kv(h, seq0, 0, workspace=ws)  # AR + history K/V
    seq = layer.seq_desc(dl.n_ar, dl.n_clean, dl.n_noisy, 1, cs, dl.chunk, L.COSMOT_MASK_BLOCK_CAUSAL,
                         n_cached=dl.n_ar + dl.n_clean)
    h_out = torch.empty_like(h)
    s0, s1 = wl.sigmas[0], wl.sigmas[1]
    layer.forward(h, h_out, s0, s1, seq, workspace=ws)
    torch.cuda.synchronize()
    assert_device_ok()

    st = olayer.StreamState(slots=hist)
    for k, x in enumerate(hist_x):
        olayer.stream_commit(wl.dims, W, st, synth.bf16_to_f64(x), olayout.build_layout(spec_blk, tau_offset=k))
    rows = sample_rows(T, [(0, T)], 64, seed=8)
    _, out = olayer.stream_block(wl.dims, W, st, synth.bf16_to_f64(h_ar), synth.bf16_to_f64(x0), lay_blk, (s0, s1),
                                 rows=rows)
    z0 = dl.n_ar + dl.n_clean
    assert_close(to_f64(h_out)[z0 + rows], out["h2"], "stream h_out (sampled rows)", rounded_inputs=3)
    vel = out["vel"]
    assert_close(to_f64(h)[z0 + rows], out["x_new"], "stream x' (sampled rows)", rounded_inputs=2,
                 branch_rms=abs(s1 - s0) * float(np.sqrt(np.mean(vel ** 2))))
