"""Classifier-free guidance on the GPU against the fp64 oracle (needs a B200)."""

import numpy as np
import pytest

import synth
from oracle import layer as olayer
from oracle import layout as olayout
from synth import ModelDims
from tolerance import SIGMA_VEL, assert_close, rms

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():  # pragma: no cover
    pytest.skip("no CUDA device", allow_module_level=True)

from flow_matching_dit_cosmot_b200 import api as A  # noqa: E402
from flow_matching_dit_cosmot_b200 import _lib as L  # noqa: E402
from gpu_helpers import assert_device_ok, bits, device_weights, dims as cdims, layer_parity, layout_spec, to_dev, to_f64  # noqa

MEDIUM = ModelDims(d_model=512, n_heads=4, n_kv_heads=4, head_dim=128, ffn=1536, rope_sections=(16, 24, 24))


def test_guided_euler_step_kernel():
    n, c = 777, 264
    x = synth.normal_bf16((n, c), 90, 1)
    vc = synth.normal_bf16((n, c), 91, 1)
    vb = synth.normal_bf16((n, c), 92, 1)
    xc, xb, dvc, dvb = to_dev(x), to_dev(x), to_dev(vc), to_dev(vb)
    L.cosmot_flow_cfg_euler_step(A.ptr(xc), A.ptr(xb), c, A.ptr(dvc), A.ptr(dvb), c, n, c, 0.9, 0.6, 4.5,
                                 A.stream_handle())
    torch.cuda.synchronize()
    v = olayer.cfg_combine(synth.bf16_to_f64(vc), synth.bf16_to_f64(vb), 4.5)
    ref = olayer.euler_step(synth.bf16_to_f64(x), v, 0.9, 0.6)
    assert_close(to_f64(xc), ref, "guided step")
    np.testing.assert_array_equal(bits(xc), bits(xb))


@pytest.mark.parametrize("guidance", [1.0, 6.0])
def test_guided_layer_two_pairs(guidance):
    spec = synth.preset("droid").layout
    lay = olayout.build_layout(spec)
    n, d = lay.n_tokens, MEDIUM.d_model
    w = synth.make_weights(MEDIUM, 1006)
    pairs = 2
    h = np.empty((2 * pairs, n, d), dtype=np.uint16)
    for p in range(pairs):
        x = synth.make_activations(n, d, 2600 + p)  # DM rows shared by the pair
        h[2 * p] = x
        h[2 * p + 1] = x
        h[2 * p + 1, :lay.n_ar] = synth.make_activations(lay.n_ar, d, 2700 + p)  # baseline prompt
    dlay = A.build_layout(layout_spec(A, spec))
    cs = A.mrope_table(dlay.pos, MEDIUM.head_dim, MEDIUM.rope_sections)
    layer = A.MoTLayer(cdims(A, MEDIUM), device_weights(w))
    seq = layer.seq_desc(dlay.n_ar, dlay.n_clean, dlay.n_noisy, 2 * pairs, cs, dlay.chunk)
    hd_ = to_dev(h)
    h_out = torch.empty_like(hd_)
    layer.forward_cfg(hd_, h_out, 1.0, 0.9, guidance, seq)
    torch.cuda.synchronize()
    assert_device_ok()
    W = olayer.weights_from_bits(MEDIUM, w)
    noisy = lay.region == olayout.REGION_NOISY
    for p in range(pairs):
        x_ref, oc, ob = olayer.cfg_step(MEDIUM, W, synth.bf16_to_f64(h[2 * p]), synth.bf16_to_f64(h[2 * p + 1]),
                                        lay, 1.0, 0.9, guidance)
        got = to_f64(hd_[2 * p])[noisy]
        # v_base + w (v_cond - v_base): the two velocities' errors enter with
        # weights (1 - w) and w; each velocity is also stored in bf16 before the
        # combine (one more rounding unit)
        mix = float(np.hypot(1.0 - guidance, guidance))
        assert_close(got, x_ref, f"guided x' pair {p}", sigma=float(np.hypot(SIGMA_VEL, 1.0)),
                     branch_rms=0.1 * mix * rms(ob["vel"][noisy]))
        np.testing.assert_array_equal(bits(hd_[2 * p])[noisy], bits(hd_[2 * p + 1])[noisy])
        layer_parity(f"cond {p}", oc, noisy, -0.1, h_out=to_f64(h_out[2 * p]))
        layer_parity(f"base {p}", ob, noisy, -0.1, h_out=to_f64(h_out[2 * p + 1]))
        # AR and clean rows of both states untouched
        np.testing.assert_array_equal(bits(hd_[2 * p])[~noisy], h[2 * p][~noisy])
        np.testing.assert_array_equal(bits(hd_[2 * p + 1])[~noisy], h[2 * p + 1][~noisy])


def test_guided_layer_rejects_odd_batch():
    dims = A.make_dims(512, 4, 4, 128, 1536, (16, 24, 24))
    cs = torch.zeros((16, 2), dtype=torch.float32, device="cuda")
    seq = L.SeqDesc(130, 181, 392, 3, 0, 0, cs.data_ptr(), 0)
    code = L.cosmot_layer_forward_cfg(dims, L.LayerWeights(), seq, 256, 256, 1.0, 0.9, 3.0, 256, 1 << 30,
                                      torch.cuda.current_stream().cuda_stream, check=False)
    assert code == L.COSMOT_ERR_INVALID_ARG


def test_guided_timed_entry_matches():
    """The stage-timed entry point with a guidance weight computes exactly the
    guided step."""
    spec = synth.preset("droid").layout
    lay = olayout.build_layout(spec)
    n, d = lay.n_tokens, MEDIUM.d_model
    w = synth.make_weights(MEDIUM, 1007)
    x = synth.make_activations(n, d, 2800)
    h = np.stack([x, x])
    h[1, :lay.n_ar] = synth.make_activations(lay.n_ar, d, 2801)
    dlay = A.build_layout(layout_spec(A, spec))
    cs = A.mrope_table(dlay.pos, MEDIUM.head_dim, MEDIUM.rope_sections)
    layer = A.MoTLayer(cdims(A, MEDIUM), device_weights(w))
    seq = layer.seq_desc(dlay.n_ar, dlay.n_clean, dlay.n_noisy, 2, cs, dlay.chunk)
    ha, hb = to_dev(h), to_dev(h)
    oa, ob = torch.empty_like(ha), torch.empty_like(hb)
    layer.forward_cfg(ha, oa, 1.0, 0.9, 3.0, seq)
    ws = layer.workspace(seq, ha.device)
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(L.COSMOT_LAYER_STAGES + 1)]
    for e in evs:
        e.record()
    L.cosmot_layer_forward_timed(layer.dims, layer.cw, seq, hb.data_ptr(), ob.data_ptr(), 1.0, 0.9, ws.data_ptr(),
                                 ws.numel(), A.stream_handle(), [e.cuda_event for e in evs], 3.0)
    torch.cuda.synchronize()
    assert_device_ok()
    np.testing.assert_array_equal(bits(ha), bits(hb))
    np.testing.assert_array_equal(bits(oa), bits(ob))


def test_timed_entry_with_sparse_events_matches():
    """The stage-timed entry given only the two events around the attention
    stage (the other boundaries NULL and unmarked) computes exactly the plain
    layer step, and the given pair times the stage."""
    spec = synth.preset("droid").layout
    lay = olayout.build_layout(spec)
    n, d = lay.n_tokens, MEDIUM.d_model
    w = synth.make_weights(MEDIUM, 1011)
    h = synth.make_activations(n, d, 2810)[None]
    dlay = A.build_layout(layout_spec(A, spec))
    cs = A.mrope_table(dlay.pos, MEDIUM.head_dim, MEDIUM.rope_sections)
    layer = A.MoTLayer(cdims(A, MEDIUM), device_weights(w))
    seq = layer.seq_desc(dlay.n_ar, dlay.n_clean, dlay.n_noisy, 1, cs, dlay.chunk)
    ha, hb = to_dev(h), to_dev(h)
    oa, ob = torch.empty_like(ha), torch.empty_like(hb)
    layer.forward(ha, oa, 1.0, 0.9, seq)
    ws = layer.workspace(seq, ha.device)
    attention = 2  # stage index of the attention
    evs = [torch.cuda.Event(enable_timing=True) if k in (attention, attention + 1) else None
           for k in range(L.COSMOT_LAYER_STAGES + 1)]
    for e in evs:
        if e is not None:
            e.record()
    L.cosmot_layer_forward_timed(layer.dims, layer.cw, seq, hb.data_ptr(), ob.data_ptr(), 1.0, 0.9, ws.data_ptr(),
                                 ws.numel(), A.stream_handle(), [e.cuda_event if e is not None else None for e in evs])
    torch.cuda.synchronize()
    assert_device_ok()
    np.testing.assert_array_equal(bits(ha), bits(hb))
    np.testing.assert_array_equal(bits(oa), bits(ob))
    assert evs[attention].elapsed_time(evs[attention + 1]) > 0
