"""Sampler loop with cached AR K/V and the streaming rollout with a key/value
ring, against the fp64 oracle (needs a B200)."""

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
from gpu_helpers import assert_device_ok, bits, device_weights, dims as cdims, layer_parity, layout_spec, to_dev, to_f64  # noqa

MEDIUM = ModelDims(d_model=512, n_heads=4, n_kv_heads=4, head_dim=128, ffn=1536, rope_sections=(16, 24, 24))


def _run_sampler(layer, dlay, cs, h0_bits, sigmas, batch, cached: bool, f32_state: bool = False):
    """The sampler loop; with f32_state the state of the noisy rows is kept in
    float32 across steps (cosmot_layer_forward_io), taken from h at step 1.
    Returns the final h and h_out, the state after every step, and h as the
    last step read it."""
    h = to_dev(h0_bits)
    h_out = torch.empty_like(h)
    x32 = torch.empty((batch, dlay.n_noisy, layer.dims.d_model), dtype=torch.float32, device="cuda")
    ws = None
    states = []
    h_last_in = None
    for k, (s0, s1) in enumerate(zip(sigmas[:-1], sigmas[1:])):
        seq = layer.seq_desc(dlay.n_ar, dlay.n_clean, dlay.n_noisy, batch, cs, dlay.chunk,
                             n_cached=dlay.n_ar if (cached and k > 0) else 0)
        if ws is None:
            ws = torch.empty(layer.workspace_bytes(seq), dtype=torch.uint8, device="cuda")
        if k == len(sigmas) - 2:
            h_last_in = h.clone()
        if f32_state:
            layer.forward(h, h_out, s0, s1, seq, workspace=ws, x_state=x32, state_from_h=(k == 0))
            states.append(x32.clone())
        else:
            layer.forward(h, h_out, s0, s1, seq, workspace=ws)
            states.append(h.clone())
    torch.cuda.synchronize()
    assert_device_ok()
    return h, h_out, states, h_last_in


def test_sampler_loop_with_cached_ar_kv():
    """DROID-style 10-step Euler sampler: step 1 computes every row, steps 2-10
    reuse the AR K/V left in the workspace and compute DM rows only."""
    wl = synth.preset("droid")
    spec, sig, batch = wl.layout, wl.sigmas, 2
    w = synth.make_weights(MEDIUM, 1003)
    lay = olayout.build_layout(spec)
    n = lay.n_tokens
    h0 = np.stack([synth.make_activations(n, MEDIUM.d_model, 2003 + 100 * b) for b in range(batch)])
    dlay = A.build_layout(layout_spec(A, spec))
    cs = A.mrope_table(dlay.pos, MEDIUM.head_dim, MEDIUM.rope_sections)
    layer = A.MoTLayer(cdims(A, MEDIUM), device_weights(w))
    h_c, out_c, states, h_in_last = _run_sampler(layer, dlay, cs, h0, sig, batch, cached=True, f32_state=True)
    h_f, out_f, states_f, _ = _run_sampler(layer, dlay, cs, h0, sig, batch, cached=False, f32_state=True)
    # Caching the AR K/V is exact on the GPU too: same bits as recomputing them,
    # with the float32 state and with the plain bf16 state alike.
    np.testing.assert_array_equal(bits(h_c), bits(h_f))
    np.testing.assert_array_equal(bits(out_c), bits(out_f))
    for a, b_ in zip(states, states_f):
        np.testing.assert_array_equal(a.cpu().numpy(), b_.cpu().numpy())
    hb_c, outb_c, _, _ = _run_sampler(layer, dlay, cs, h0, sig, batch, cached=True)
    hb_f, outb_f, _, _ = _run_sampler(layer, dlay, cs, h0, sig, batch, cached=False)
    np.testing.assert_array_equal(bits(hb_c), bits(hb_f))
    np.testing.assert_array_equal(bits(outb_c), bits(outb_f))
    W = olayer.weights_from_bits(MEDIUM, w)
    noisy = lay.region == olayout.REGION_NOISY
    for b in range(batch):
        hf, outs = olayer.sample(MEDIUM, W, synth.bf16_to_f64(h0[b]), lay, sig)
        # The float32 state meets the one-step bounds after every step.
        for k, o in enumerate(outs):
            layer_parity(f"step {k + 1} [{b}]", o, noisy, sig[k + 1] - sig[k],
                         x_new=states[k][b].double().cpu().numpy(), x_f32=True)
        np.testing.assert_array_equal(bits(h_c[b])[~noisy], h0[b][~noisy])
        np.testing.assert_array_equal(bits(h_c[b])[noisy], bits(states[-1][b].to(torch.bfloat16)))
        # h_out of the last step (AR rows kept from step 1), against the oracle's
        # layer on the same bf16 input the GPU's last step read
        ref = olayer.layer_forward(MEDIUM, W, to_f64(h_in_last[b]), lay.region, lay.pos, lay.chunk, sig[-2], sig[-1])
        layer_parity(f"last step [{b}]", ref, noisy, sig[-1] - sig[-2], h_out=to_f64(out_c[b]))


def _virtual_spec(n_text, video, hist, tau_offset):
    """[AR; history blocks as clean steps; the current block as the noisy step]."""
    v = video
    return A.layout_spec(n_text, (v.views, v.grid_h, v.grid_w, v.fps, hist, 1), tau_offset=tau_offset)


@pytest.mark.parametrize("mode", [L.COSMOT_MASK_BLOCK_CAUSAL, L.COSMOT_MASK_FULL])
def test_streaming_rollout_with_kv_ring(mode):
    dims = ModelDims(d_model=256, n_heads=4, n_kv_heads=2, head_dim=64, ffn=512, rope_sections=(8, 12, 12))
    video = VideoSpec(2, 3, 5, 24, 0, 1)  # 30 tokens per block
    n_text, hist, blocks, sig = 6, 3, 5, (1.0, 0.75, 0.5, 0.25, 0.0)
    T = video.tokens_per_step
    n_ar = n_text + 2
    w = synth.make_weights(dims, 1004)
    layer = A.MoTLayer(cdims(A, dims), device_weights(w))
    # seeded inputs: AR rows, the prefilled history blocks, the noise of each new block
    h_ar = synth.make_activations(n_ar, dims.d_model, 2004)
    hist_x = [synth.make_activations(T, dims.d_model, 2104 + i) for i in range(hist)]
    noise = [synth.make_activations(T, dims.d_model, 2204 + b) for b in range(blocks)]
    N = n_ar + hist * T + T

    def seq_for(b, n_cached):
        dl = A.build_layout(_virtual_spec(n_text, video, hist, b))
        cs = A.mrope_table(dl.pos, dims.head_dim, dims.rope_sections)
        s = layer.seq_desc(dl.n_ar, dl.n_clean, dl.n_noisy, 1, cs, dl.chunk, mask_mode=mode, n_cached=n_cached)
        return s, (dl, cs)

    # prefill: AR + history K/V computed in place
    h = to_dev(np.concatenate([h_ar] + hist_x + [noise[0]]))
    seq0, keep0 = seq_for(0, 0)
    ws = torch.empty(layer.workspace_bytes(seq0), dtype=torch.uint8, device="cuda")
    layer.commit_kv(h, seq0, 0, workspace=ws)
    h_out = torch.empty_like(h)
    x32 = torch.empty((1, T, dims.d_model), dtype=torch.float32, device="cuda")
    outs = []
    for b in range(blocks):
        h[n_ar + hist * T:] = to_dev(noise[b])
        seq, keep = seq_for(b, n_ar + hist * T)
        for k, (s0, s1) in enumerate(zip(sig[:-1], sig[1:])):
            layer.forward(h, h_out, s0, s1, seq, workspace=ws, x_state=x32, state_from_h=(k == 0))
        outs.append(x32[0].clone())
        layer.commit_kv(h, seq, n_ar + (b % hist) * T, workspace=ws)
    torch.cuda.synchronize()
    assert_device_ok()

    # oracle: the same rollout with its own cache
    W = olayer.weights_from_bits(dims, w)
    spec_blk = LayoutSpec(n_text=n_text, video=video)
    st = olayer.StreamState(slots=hist)
    for i in range(hist):
        olayer.stream_commit(dims, W, st, synth.bf16_to_f64(hist_x[i]), olayout.build_layout(spec_blk, tau_offset=i))
    for b in range(blocks):
        lb = olayout.build_layout(spec_blk, tau_offset=hist + b)
        x, last = olayer.stream_block(dims, W, st, synth.bf16_to_f64(h_ar), synth.bf16_to_f64(noise[b]), lb, sig)
        got = outs[b].double().cpu().numpy()
        # the float32 state after the block's last step, at the one-step bound
        vel = last["vel"]  # the block's rows only
        assert_close(got, x, f"block {b}", sigma=SIGMA_VEL, branch_rms=abs(sig[-1] - sig[-2]) * rms(vel),
                     out_bf16=False)
        # each side commits the K/V of its own final x
        olayer.stream_commit(dims, W, st, x, lb)


def test_streaming_block_with_key_split():
    """A streaming block whose attention the layer splits by keys (few query
    tiles against a long cache: 8 heads x 4 query-tile pairs = 32 work items
    on the SMs, 33 key tiles): four denoising steps against the oracle."""
    dims = ModelDims(d_model=1024, n_heads=8, n_kv_heads=8, head_dim=128, ffn=2048, rope_sections=(16, 24, 24))
    video = VideoSpec(4, 16, 16, 24, 0, 1)  # 1,024 tokens per block
    n_text, hist, sig = 8, 3, (1.0, 0.75, 0.5, 0.25, 0.0)
    T = video.tokens_per_step
    n_ar = n_text + 2
    w = synth.make_weights(dims, 1005)
    layer = A.MoTLayer(cdims(A, dims), device_weights(w))
    h_ar = synth.make_activations(n_ar, dims.d_model, 2005)
    hist_x = [synth.make_activations(T, dims.d_model, 2105 + i) for i in range(hist)]
    noise = synth.make_activations(T, dims.d_model, 2205)
    dl = A.build_layout(_virtual_spec(n_text, video, hist, 0))
    cs = A.mrope_table(dl.pos, dims.head_dim, dims.rope_sections)
    mode = L.COSMOT_MASK_BLOCK_CAUSAL
    seq0 = layer.seq_desc(dl.n_ar, dl.n_clean, dl.n_noisy, 1, cs, dl.chunk, mask_mode=mode)
    seq = layer.seq_desc(dl.n_ar, dl.n_clean, dl.n_noisy, 1, cs, dl.chunk, mask_mode=mode, n_cached=n_ar + hist * T)
    N = n_ar + hist * T + T
    ad = L.AttnDesc(n_q=T, q_key_offset=N - T, n_keys=N, n_ar=n_ar, n_heads=8, n_kv_heads=8, head_dim=128,
                    mask_mode=mode, chunk=A.ptr(dl.chunk), batch=1, flags=L.COSMOT_ATTN_NO_TILE_SKIP)
    assert L.cosmot_attention_kv_split(ad) > 1  # the layer takes the split path here
    h = to_dev(np.concatenate([h_ar] + hist_x + [noise]))
    ws = torch.empty(layer.workspace_bytes(seq0), dtype=torch.uint8, device="cuda")
    layer.commit_kv(h, seq0, 0, workspace=ws)
    h_out = torch.empty_like(h)
    x32 = torch.empty((1, T, dims.d_model), dtype=torch.float32, device="cuda")
    for k, (s0, s1) in enumerate(zip(sig[:-1], sig[1:])):
        layer.forward(h, h_out, s0, s1, seq, workspace=ws, x_state=x32, state_from_h=(k == 0))
    torch.cuda.synchronize()
    assert_device_ok()
    W = olayer.weights_from_bits(dims, w)
    spec_blk = LayoutSpec(n_text=n_text, video=video)
    st = olayer.StreamState(slots=hist)
    for i in range(hist):
        olayer.stream_commit(dims, W, st, synth.bf16_to_f64(hist_x[i]), olayout.build_layout(spec_blk, tau_offset=i))
    lb = olayout.build_layout(spec_blk, tau_offset=hist)
    x, last = olayer.stream_block(dims, W, st, synth.bf16_to_f64(h_ar), synth.bf16_to_f64(noise), lb, sig)
    assert_close(x32[0].double().cpu().numpy(), x, "split-key block", sigma=SIGMA_VEL,
                 branch_rms=abs(sig[-1] - sig[-2]) * rms(last["vel"]), out_bf16=False)


def test_sampler_without_clean_rows_stays_bit_identical():
    """A text-to-video-like layout (no clean rows) whose noisy-only attention
    would be worth a key split (8 heads x 8 query-tile pairs against 17 key
    tiles): the sampler's later steps reuse only the AR rows, never split, and
    stay bit-identical to a full recompute."""
    dims = ModelDims(d_model=1024, n_heads=8, n_kv_heads=8, head_dim=128, ffn=2048, rope_sections=(16, 24, 24))
    spec = LayoutSpec(n_text=30, video=VideoSpec(1, 16, 16, 24, 0, 8))  # 32 AR + 2,048 noisy
    lay = olayout.build_layout(spec)
    w = synth.make_weights(dims, 1006)
    h0 = synth.make_activations(lay.n_tokens, dims.d_model, 2006)[None]
    dlay = A.build_layout(layout_spec(A, spec))
    cs = A.mrope_table(dlay.pos, dims.head_dim, dims.rope_sections)
    layer = A.MoTLayer(cdims(A, dims), device_weights(w))
    sig = (1.0, 0.8, 0.6)
    h_c, out_c, st_c, _ = _run_sampler(layer, dlay, cs, h0, sig, 1, cached=True, f32_state=True)
    h_f, out_f, st_f, _ = _run_sampler(layer, dlay, cs, h0, sig, 1, cached=False, f32_state=True)
    np.testing.assert_array_equal(bits(h_c), bits(h_f))
    np.testing.assert_array_equal(bits(out_c)[0, lay.n_ar:], bits(out_f)[0, lay.n_ar:])
    for a, b_ in zip(st_c, st_f):
        np.testing.assert_array_equal(a.cpu().numpy(), b_.cpu().numpy())
