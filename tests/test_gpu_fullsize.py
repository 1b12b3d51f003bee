"""Parity at the workloads' full sizes, in the launch configuration bench.py
times, on output rows the oracle computes one by one (needs a B200).

The oracle forms K and V of every row in float64 and the full layer only for
the sampled rows: at least 2,048 of them, every segment's first and last row
included, drawn with a fixed seed.  Besides h_out and the state x', every
case checks the velocity v itself (the stricter output: x' = x + dsigma v
with |dsigma| = 0.03 hides most of v's error).  Samplers keep their state in
float32 between steps (cosmot_layer_forward_io) and are checked at the
one-step bounds after every step.
"""

import numpy as np
import pytest

import synth
from oracle import layer as olayer
from oracle import layout as olayout

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():  # pragma: no cover
    pytest.skip("no CUDA device", allow_module_level=True)

from flow_matching_dit_cosmot_b200 import api as A  # noqa: E402
from flow_matching_dit_cosmot_b200 import _lib as L  # noqa: E402
from gpu_helpers import (assert_device_ok, bits, device_weights, dims as cdims, layer_parity, layout_spec,  # noqa
                         sample_rows, to_dev, to_f64)

N_SAMPLED = 2048
_W = {}


def _weights(wl):
    if wl.name not in _W:
        _W.clear()  # keep one workload's weights at a time
        w = synth.make_weights(wl.dims, wl.weight_seed)
        _W[wl.name] = (w, device_weights(w), olayer.weights_from_bits(wl.dims, w))
    return _W[wl.name]


def _f32(t):
    return t.double().cpu().numpy()


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
    s0, s1 = wl.sigmas[0], wl.sigmas[1]
    # the plain entry point (what the bench times) ...
    hd_ = to_dev(h)
    h_out = torch.empty_like(hd_)
    layer.forward(hd_, h_out, s0, s1, seq)
    # ... and the io entry point on the same inputs: float32 state and velocity
    h_io = to_dev(h)
    out_io = torch.empty_like(h_io)
    x32 = torch.empty((1, lay.n_noisy, wl.dims.d_model), dtype=torch.float32, device="cuda")
    vel = torch.empty((1, lay.n_noisy, wl.dims.d_model), dtype=torch.bfloat16, device="cuda")
    layer.forward(h_io, out_io, s0, s1, seq, x_state=x32, state_from_h=True, vel=vel)
    torch.cuda.synchronize()
    assert_device_ok()
    np.testing.assert_array_equal(dlay.pos.cpu().numpy().view(np.uint32), lay.pos.view(np.uint32))
    np.testing.assert_array_equal(bits(out_io), bits(h_out))
    np.testing.assert_array_equal(bits(h_io), bits(hd_))

    z0 = lay.n_ar + lay.n_clean
    rows = sample_rows(n, [(0, lay.n_ar), (lay.n_ar, z0), (z0, n)], N_SAMPLED, seed=7)
    assert len(rows) >= N_SAMPLED
    ref = olayer.layer_forward(wl.dims, W, synth.bf16_to_f64(h), lay.region, lay.pos, lay.chunk, s0, s1,
                               wl.mask_mode, rows=rows)
    noisy = lay.region[rows] == olayout.REGION_NOISY
    zr = rows[noisy] - z0  # sampled noisy rows in the packed noisy order
    layer_parity(name, ref, noisy, s1 - s0, h_out=to_f64(h_out)[rows], x_new=to_f64(hd_)[rows][noisy])
    layer_parity(f"{name} io", ref, noisy, s1 - s0, x_new=_f32(x32[0])[zr], vel=to_f64(vel[0])[zr], x_f32=True)
    # clean and AR rows of h are untouched
    keep = lay.region != olayout.REGION_NOISY
    np.testing.assert_array_equal(bits(hd_)[keep], h[keep])


def _droid_sampler(layer, dlay, cs, h0_bits, sig, batch):
    """The 10-step DROID sampler: AR K/V kept in the workspace after step 1,
    float32 state.  Returns the state after every step."""
    h = to_dev(h0_bits)
    h_out = torch.empty_like(h)
    x32 = torch.empty((batch, dlay.n_noisy, layer.dims.d_model), dtype=torch.float32, device="cuda")
    ws, states = None, []
    for k, (s0, s1) in enumerate(zip(sig[:-1], sig[1:])):
        seq = layer.seq_desc(dlay.n_ar, dlay.n_clean, dlay.n_noisy, batch, cs, dlay.chunk,
                             n_cached=dlay.n_ar if k else 0)
        if ws is None:
            ws = torch.empty(layer.workspace_bytes(seq), dtype=torch.uint8, device="cuda")
        layer.forward(h, h_out, s0, s1, seq, workspace=ws, x_state=x32, state_from_h=(k == 0))
        states.append(x32.clone())
    torch.cuda.synchronize()
    assert_device_ok()
    # the layer's next input is the float32 state rounded to nearest even
    np.testing.assert_array_equal(bits(h)[:, dlay.n_ar + dlay.n_clean:], bits(x32.to(torch.bfloat16)))
    return states


def test_full_width_droid_sampler():
    """DROID policy step at d_model 4096: the 10-step sampler against the
    oracle's full recomputation, after every step, at the one-step bounds."""
    wl = synth.preset("droid")
    w, dw, W = _weights(wl)
    lay = olayout.build_layout(wl.layout)
    h0 = synth.make_activations(lay.n_tokens, wl.dims.d_model, wl.act_seed())
    dlay = A.build_layout(layout_spec(A, wl.layout))
    cs = A.mrope_table(dlay.pos, wl.dims.head_dim, wl.dims.rope_sections, wl.dims.rope_base)
    layer = A.MoTLayer(cdims(A, wl.dims), dw)
    states = _droid_sampler(layer, dlay, cs, h0[None], wl.sigmas, 1)
    _, outs = olayer.sample(wl.dims, W, synth.bf16_to_f64(h0), lay, wl.sigmas)
    noisy = lay.region == olayout.REGION_NOISY
    sig = wl.sigmas
    for k, o in enumerate(outs):
        layer_parity(f"droid step {k + 1}", o, noisy, sig[k + 1] - sig[k], x_new=_f32(states[k][0]), x_f32=True)


def test_full_width_droid_batch16():
    """DROID at batch 16 (16 sequences, shared weights, seeded activations per
    sequence), 10 steps.  Every sequence's state after every step is bit-
    identical to a batch-1 run of that sequence (no tile or work item mixes
    sequences); step 1 of every sequence matches the oracle on sampled rows
    (h_out, v, x'); the last sequence matches the oracle's 10-step sampler."""
    wl = synth.preset("droid_b16")
    w, dw, W = _weights(wl)
    lay = olayout.build_layout(wl.layout)
    n, B, sig = lay.n_tokens, wl.batch, wl.sigmas
    h0 = np.stack([synth.make_activations(n, wl.dims.d_model, wl.act_seed(b)) for b in range(B)])
    dlay = A.build_layout(layout_spec(A, wl.layout))
    cs = A.mrope_table(dlay.pos, wl.dims.head_dim, wl.dims.rope_sections, wl.dims.rope_base)
    layer = A.MoTLayer(cdims(A, wl.dims), dw)
    states = _droid_sampler(layer, dlay, cs, h0, sig, B)
    for b in range(B):
        one = _droid_sampler(layer, dlay, cs, h0[b:b + 1], sig, 1)
        for k in range(len(one)):
            np.testing.assert_array_equal(states[k][b].cpu().numpy(), one[k][0].cpu().numpy())

    # step 1 of every sequence, with h_out and v: one more batch-16 call with outputs
    h = to_dev(h0)
    h_out = torch.empty_like(h)
    x32 = torch.empty((B, lay.n_noisy, wl.dims.d_model), dtype=torch.float32, device="cuda")
    vel = torch.empty((B, lay.n_noisy, wl.dims.d_model), dtype=torch.bfloat16, device="cuda")
    seq = layer.seq_desc(dlay.n_ar, dlay.n_clean, dlay.n_noisy, B, cs, dlay.chunk)
    layer.forward(h, h_out, sig[0], sig[1], seq, x_state=x32, state_from_h=True, vel=vel)
    torch.cuda.synchronize()
    assert_device_ok()
    np.testing.assert_array_equal(x32.cpu().numpy(), states[0].cpu().numpy())
    z0 = lay.n_ar + lay.n_clean
    per_seq = -(-N_SAMPLED // B)
    for b in range(B):
        rows = sample_rows(n, [(0, lay.n_ar), (lay.n_ar, z0), (z0, n)], per_seq, seed=100 + b)
        ref = olayer.layer_forward(wl.dims, W, synth.bf16_to_f64(h0[b]), lay.region, lay.pos, lay.chunk, sig[0],
                                   sig[1], rows=rows)
        noisy = lay.region[rows] == olayout.REGION_NOISY
        zr = rows[noisy] - z0
        layer_parity(f"droid b16 [{b}] step 1", ref, noisy, sig[1] - sig[0], h_out=to_f64(h_out[b])[rows],
                     x_new=_f32(x32[b])[zr], vel=to_f64(vel[b])[zr], x_f32=True)
    b = B - 1
    _, outs = olayer.sample(wl.dims, W, synth.bf16_to_f64(h0[b]), lay, sig)
    noisy = lay.region == olayout.REGION_NOISY
    for k, o in enumerate(outs):
        layer_parity(f"droid b16 [{b}] step {k + 1}", o, noisy, sig[k + 1] - sig[k], x_new=_f32(states[k][b]),
                     x_f32=True)


def test_full_width_streaming_rollout():
    """Two 1,560-token blocks of the streaming rollout at d_model 4096
    ("NVIDIA 发布 Cosmos 3 系列四个开放权重世界模型", "流式生成如何工作"): 66 AR rows
    and 8 cached history blocks, 4 denoising steps per block, then the block's
    K/V committed over the oldest ring slot, so the second block sees history
    blocks 1-7 and the first block (history block 0 evicted).  Checked on every
    row: the first step (h_out, v, x', from identical inputs) and each block's
    final float32 state against the oracle's rollout with its own cache."""
    wl = synth.preset("stream")
    w, dw, W = _weights(wl)
    v = wl.layout.video
    hist = wl.stream.cached_blocks
    sig = wl.sigmas
    spec_blk = synth.LayoutSpec(n_text=wl.layout.n_text, video=v)
    d = wl.dims.d_model
    n_ar = spec_blk.n_ar
    T = v.tokens_per_step
    h_ar = synth.make_activations(n_ar, d, wl.act_seed())
    hist_x = [synth.make_activations(T, d, 4000 + k) for k in range(hist)]
    noise = [synth.make_activations(T, d, 5000 + k) for k in range(2)]
    layer = A.MoTLayer(cdims(A, wl.dims), dw)

    def seq_for(block, n_cached):
        dl = A.build_layout(A.layout_spec(wl.layout.n_text, (v.views, v.grid_h, v.grid_w, v.fps, hist, 1),
                                          tau_offset=block))
        c = A.mrope_table(dl.pos, wl.dims.head_dim, wl.dims.rope_sections, wl.dims.rope_base)
        return layer.seq_desc(dl.n_ar, dl.n_clean, dl.n_noisy, 1, c, dl.chunk, L.COSMOT_MASK_BLOCK_CAUSAL,
                              n_cached=n_cached), (dl, c)

    h = to_dev(np.concatenate([h_ar] + hist_x + [noise[0]]))
    seq0, keep0 = seq_for(0, 0)
    ws = torch.empty(layer.workspace_bytes(seq0), dtype=torch.uint8, device="cuda")
    layer.commit_kv(h, seq0, 0, workspace=ws)  # AR + history K/V in place
    h_out = torch.empty_like(h)
    x32 = torch.empty((1, T, d), dtype=torch.float32, device="cuda")
    vel = torch.empty((1, T, d), dtype=torch.bfloat16, device="cuda")
    z0 = n_ar + hist * T
    finals, first = [], None
    for blk in range(2):
        h[z0:] = to_dev(noise[blk])
        seq, keep = seq_for(blk, z0)
        for k, (s0, s1) in enumerate(zip(sig[:-1], sig[1:])):
            layer.forward(h, h_out, s0, s1, seq, workspace=ws, x_state=x32, state_from_h=(k == 0),
                          vel=vel if (blk, k) == (0, 0) else None)
            if (blk, k) == (0, 0):
                first = (h_out[z0:].clone(), x32[0].clone(), vel[0].clone())
        finals.append(x32[0].clone())
        layer.commit_kv(h, seq, n_ar + (blk % hist) * T, workspace=ws)  # over the oldest slot
    torch.cuda.synchronize()
    assert_device_ok()

    # the oracle's rollout, step by step over every block row
    st = olayer.StreamState(slots=hist)
    for k, x in enumerate(hist_x):
        olayer.stream_commit(wl.dims, W, st, synth.bf16_to_f64(x), olayout.build_layout(spec_blk, tau_offset=k))
    har = synth.bf16_to_f64(h_ar)
    for blk in range(2):
        lb = olayout.build_layout(spec_blk, tau_offset=hist + blk)
        x = synth.bf16_to_f64(noise[blk])
        rows = np.arange(n_ar, n_ar + T)
        for k, (s0, s1) in enumerate(zip(sig[:-1], sig[1:])):
            out = olayer.layer_forward(wl.dims, W, np.concatenate([har, x]), lb.region, lb.pos, lb.chunk, s0, s1,
                                       mode="block_causal", rows=rows, cache=st.cache())
            if (blk, k) == (0, 0):
                noisy = np.ones(T, dtype=bool)
                layer_parity("stream block 0 step 1", out, noisy, s1 - s0, h_out=to_f64(first[0]),
                             x_new=_f32(first[1]), vel=to_f64(first[2]), x_f32=True)
            x = out["x_new"]
        layer_parity(f"stream block {blk} after {len(sig) - 1} steps", out, np.ones(T, dtype=bool),
                     sig[-1] - sig[-2], x_new=_f32(finals[blk]), x_f32=True)
        olayer.stream_commit(wl.dims, W, st, x, lb)
