"""Degenerate and empty inputs on the GPU (needs a B200): a layer with no noisy
rows, a layout with no text (only EOS/BOG in the AR prefix), a single noisy
row, zero-query attention, an empty Euler range and an empty segment in a
routed GEMM.  Each either matches the oracle or is a no-op that writes nothing.
"""

import numpy as np
import pytest

import synth
from oracle import layer as olayer
from oracle import layout as olayout
from synth import LayoutSpec, ModelDims, VideoSpec
from tolerance import assert_close

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():  # pragma: no cover
    pytest.skip("no CUDA device", allow_module_level=True)

from flow_matching_dit_cosmot_b200 import api as A  # noqa: E402
from flow_matching_dit_cosmot_b200 import _lib as L  # noqa: E402
from gpu_helpers import assert_device_ok, bits, device_weights, dims as cdims, layer_parity, layout_spec, to_dev, to_f64  # noqa

DIMS = ModelDims(d_model=256, n_heads=4, n_kv_heads=2, head_dim=64, ffn=512, rope_sections=(8, 12, 12))


def _layer_case(spec, seed=4100):
    lay = olayout.build_layout(spec)
    w = synth.make_weights(DIMS, seed)
    h = synth.make_activations(lay.n_tokens, DIMS.d_model, seed + 1)
    dlay = A.build_layout(layout_spec(A, spec))
    cs = A.mrope_table(dlay.pos, DIMS.head_dim, DIMS.rope_sections)
    layer = A.MoTLayer(cdims(A, DIMS), device_weights(w))
    seq = layer.seq_desc(lay.n_ar, lay.n_clean, lay.n_noisy, 1, cs, dlay.chunk)
    hd_ = to_dev(h[None])
    h_out = torch.empty_like(hd_)
    layer.forward(hd_, h_out, 0.8, 0.6, seq)
    torch.cuda.synchronize()
    assert_device_ok()
    ref = olayer.layer_forward(DIMS, olayer.weights_from_bits(DIMS, w), synth.bf16_to_f64(h), lay.region, lay.pos,
                               lay.chunk, 0.8, 0.6)
    noisy = lay.region == olayout.REGION_NOISY
    layer_parity("edge", ref, noisy, -0.2, h_out=to_f64(h_out[0]), x_new=to_f64(hd_[0])[noisy])
    np.testing.assert_array_equal(bits(hd_[0])[~noisy], h[~noisy])
    return lay


def test_layer_without_noisy_rows():
    """Conditioning only: the head and the Euler step have nothing to do and
    the state is left exactly as it was."""
    lay = _layer_case(LayoutSpec(n_text=10, video=VideoSpec(1, 3, 5, 24, 2, 0)))
    assert lay.n_noisy == 0


def test_layer_without_text():
    """No prompt tokens: the AR prefix is EOS and BOG alone."""
    lay = _layer_case(LayoutSpec(n_text=0, video=VideoSpec(1, 3, 5, 24, 1, 2)))
    assert lay.n_ar == 2


def test_layer_with_a_single_noisy_row():
    lay = _layer_case(LayoutSpec(n_text=3, video=None, action_noisy=1, action_hz=15))
    assert lay.n_noisy == 1


def test_zero_query_attention_and_empty_euler_range_write_nothing():
    n, H, hd = 300, 2, 64
    qkv = to_dev(synth.normal_bf16((n, 3 * H * hd), 4200, 1))
    o = torch.full((n, H * hd), 3.0, dtype=torch.bfloat16, device="cuda")
    d = L.AttnDesc(n_q=0, q_key_offset=n, n_keys=n, n_ar=10, n_heads=H, n_kv_heads=H, head_dim=hd,
                   mask_mode=L.COSMOT_MASK_FULL, batch=1)
    base = qkv.data_ptr()
    L.cosmot_mot_attention(d, base, 3 * H * hd, base + H * hd * 2, base + 2 * H * hd * 2, 3 * H * hd, o.data_ptr(),
                           H * hd, A.stream_handle())
    x = to_dev(synth.normal_bf16((40, 64), 4201, 1))
    x0 = bits(x).copy()
    v = to_dev(synth.normal_bf16((40, 64), 4202, 1))
    L.cosmot_flow_euler_step(x.data_ptr(), 64, v.data_ptr(), 64, 17, 17, 64, 0.9, 0.5, A.stream_handle())
    torch.cuda.synchronize()
    assert_device_ok()
    assert (o.float() == 3.0).all()
    np.testing.assert_array_equal(bits(x), x0)


def test_routed_linear_with_an_empty_segment():
    """An empty segment between two others contributes no tile; the rows
    around it are computed with their own weight sets."""
    k, n_out = 128, 136
    a = synth.normal_bf16((300, k), 4300, 1)
    w0 = synth.normal_bf16((n_out, k), 4301, 1, std=1.0 / np.sqrt(k))
    w1 = synth.normal_bf16((n_out, k), 4302, 1, std=1.0 / np.sqrt(k))
    segs = [(0, 90, 0, 0), (90, 90, 90, 1), (90, 300, 90, 1)]
    out = torch.empty((300, n_out), dtype=torch.bfloat16, device="cuda")
    ad, w0d, w1d = to_dev(a), to_dev(w0), to_dev(w1)
    L.cosmot_routed_linear(A.ptr(ad), k, k, segs, A.ptr(w0d), A.ptr(w1d), n_out, A.ptr(out), n_out,
                           stream=A.stream_handle())
    torch.cuda.synchronize()
    assert_device_ok()
    a64, w064, w164 = (synth.bf16_to_f64(x) for x in (a, w0, w1))
    ref = np.concatenate([a64[:90] @ w064.T, a64[90:] @ w164.T])
    assert_close(to_f64(out), ref, "gemm with an empty segment")


def test_layer_at_the_largest_batch():
    """32 sequences, the largest batch one call takes (64 row segments in
    every routed launch): every sequence's outputs equal those of the same
    sequence run alone, bit for bit, and the first and last match the oracle."""
    spec = LayoutSpec(n_text=5, video=VideoSpec(1, 3, 4, 24, 1, 1))
    lay = olayout.build_layout(spec)
    B = 32
    w = synth.make_weights(DIMS, 4700)
    h = np.stack([synth.make_activations(lay.n_tokens, DIMS.d_model, 4701 + b) for b in range(B)])
    dlay = A.build_layout(layout_spec(A, spec))
    cs = A.mrope_table(dlay.pos, DIMS.head_dim, DIMS.rope_sections)
    layer = A.MoTLayer(cdims(A, DIMS), device_weights(w))
    hd_, h_out = to_dev(h), torch.empty((B, lay.n_tokens, DIMS.d_model), dtype=torch.bfloat16, device="cuda")
    layer.forward(hd_, h_out, 0.8, 0.6, layer.seq_desc(lay.n_ar, lay.n_clean, lay.n_noisy, B, cs, dlay.chunk))
    torch.cuda.synchronize()
    assert_device_ok()
    W = olayer.weights_from_bits(DIMS, w)
    noisy = lay.region == olayout.REGION_NOISY
    for b in range(B):
        one, one_out = to_dev(h[b:b + 1]), torch.empty((1, lay.n_tokens, DIMS.d_model), dtype=torch.bfloat16,
                                                       device="cuda")
        layer.forward(one, one_out, 0.8, 0.6, layer.seq_desc(lay.n_ar, lay.n_clean, lay.n_noisy, 1, cs, dlay.chunk))
        torch.cuda.synchronize()
        np.testing.assert_array_equal(bits(h_out[b]), bits(one_out[0]))
        np.testing.assert_array_equal(bits(hd_[b]), bits(one[0]))
        if b in (0, B - 1):
            ref = olayer.layer_forward(DIMS, W, synth.bf16_to_f64(h[b]), lay.region, lay.pos, lay.chunk, 0.8, 0.6)
            layer_parity(f"batch {B} [{b}]", ref, noisy, -0.2, h_out=to_f64(h_out[b]), x_new=to_f64(hd_[b])[noisy])
    bad = layer.seq_desc(lay.n_ar, lay.n_clean, lay.n_noisy, B + 1, cs, dlay.chunk)
    ws = torch.empty((1 << 20,), dtype=torch.uint8, device="cuda")
    code = L.cosmot_layer_forward(layer.dims, layer.cw, bad, hd_.data_ptr(), h_out.data_ptr(), 0.8, 0.6,
                                  ws.data_ptr(), ws.numel(), A.stream_handle(), check=False)
    assert code == L.COSMOT_ERR_UNSUPPORTED
