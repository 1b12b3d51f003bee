"""Whole-layer parity of cosmot_layer_forward against the fp64 oracle (needs a B200)."""

import numpy as np
import pytest

import synth
from oracle import layer as olayer
from oracle import layout as olayout
from synth import LayoutSpec, ModelDims, VideoSpec

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():  # pragma: no cover
    pytest.skip("no CUDA device", allow_module_level=True)

from flow_matching_dit_cosmot_b200 import api as A  # noqa: E402
from flow_matching_dit_cosmot_b200 import _lib as L  # noqa: E402
from gpu_helpers import (Guarded, assert_device_ok, bits, device_weights, dims as cdims, layer_parity,  # noqa: E402
                         layout_spec, to_dev, to_f64)


class LayerRun:
    """Seeded weights and inputs on the device, one layer forward, the oracle beside it."""

    def __init__(self, dims: ModelDims, spec: LayoutSpec, batch=1, mode="full", weight_seed=1001, act_seed=2001):
        self.dims, self.spec, self.batch, self.mode = dims, spec, batch, mode
        self.w = synth.make_weights(dims, weight_seed)
        self.lay = olayout.build_layout(spec)
        n = self.lay.n_tokens
        self.h = np.stack([synth.make_activations(n, dims.d_model, act_seed + 100 * b) for b in range(batch)])
        self.dw = device_weights(self.w)
        self.dlay = A.build_layout(layout_spec(A, spec))
        self.cs = A.mrope_table(self.dlay.pos, dims.head_dim, dims.rope_sections, dims.rope_base)
        self.layer = A.MoTLayer(cdims(A, dims), self.dw)
        self.seq = self.layer.seq_desc(self.lay.n_ar, self.lay.n_clean, self.lay.n_noisy, batch, self.cs,
                                       self.dlay.chunk, L.COSMOT_MASK_FULL if mode == "full" else L.COSMOT_MASK_BLOCK_CAUSAL)

    def gpu(self, h_bits=None, sigma=0.8, sigma_next=0.7):
        # both buffers sit between canary guard bands: nothing outside them may change
        h = Guarded(to_dev(self.h if h_bits is None else h_bits))
        h_out = Guarded(torch.empty_like(h.t))
        self.layer.forward(h.t, h_out.t, sigma, sigma_next, self.seq)
        torch.cuda.synchronize()
        assert_device_ok()
        h.assert_canaries("h")
        h_out.assert_canaries("h_out")
        return h.t, h_out.t

    def gpu_io(self, sigma=0.8, sigma_next=0.7):
        """cosmot_layer_forward_io: the float32 state (taken from h on this first
        step) and the velocity of the noisy rows as extra outputs."""
        h = to_dev(self.h)
        h_out = torch.empty_like(h)
        nz = self.lay.n_noisy
        x32 = torch.full((self.batch, nz, self.dims.d_model), float("nan"), dtype=torch.float32, device="cuda")
        vel = torch.full((self.batch, nz, self.dims.d_model), float("nan"), dtype=torch.bfloat16, device="cuda")
        self.layer.forward(h, h_out, sigma, sigma_next, self.seq, x_state=x32, state_from_h=True, vel=vel)
        torch.cuda.synchronize()
        assert_device_ok()
        return h, h_out, x32, vel

    def oracle(self, b=0, sigma=0.8, sigma_next=0.7, h_bits=None):
        W = olayer.weights_from_bits(self.dims, self.w)
        h = synth.bf16_to_f64((self.h if h_bits is None else h_bits)[b])
        return olayer.layer_forward(self.dims, W, h, self.lay.region, self.lay.pos, self.lay.chunk, sigma, sigma_next,
                                    self.mode)


def _check(run, h_dev, hout_dev, sigma=0.8, sigma_next=0.7):
    """Plain entry point: h_out and the bf16 state in h against the oracle.
    The io entry point on the same inputs: identical h_out and h bits, and its
    float32 state and velocity against the oracle."""
    lay = run.lay
    noisy = lay.region == olayout.REGION_NOISY
    h_io, hout_io, x32, vel = run.gpu_io(sigma, sigma_next)
    np.testing.assert_array_equal(bits(hout_io), bits(hout_dev))
    np.testing.assert_array_equal(bits(h_io), bits(h_dev))
    for b in range(run.batch):
        ref = run.oracle(b, sigma, sigma_next)
        ds = sigma_next - sigma
        layer_parity(f"[{b}]", ref, noisy, ds, h_out=to_f64(hout_dev[b]), x_new=to_f64(h_dev[b])[noisy])
        if noisy.any():
            layer_parity(f"io [{b}]", ref, noisy, ds, x_new=x32[b].double().cpu().numpy(), vel=to_f64(vel[b]),
                         x_f32=True)
            # the bf16 copy in h is the float32 state rounded to nearest even
            np.testing.assert_array_equal(bits(h_io[b])[noisy], bits(x32[b].to(torch.bfloat16)))
        # AR and clean rows of h are never written (clean DM tokens pass through bit-exact)
        np.testing.assert_array_equal(bits(h_dev[b])[~noisy], run.h[b][~noisy])


def test_layer_tiny_workload():
    wl = synth.preset("tiny")
    run = LayerRun(wl.dims, wl.layout, weight_seed=wl.weight_seed, act_seed=wl.act_seed())
    h, h_out = run.gpu(sigma=wl.sigmas[0], sigma_next=wl.sigmas[1])
    _check(run, h, h_out, wl.sigmas[0], wl.sigmas[1])


MEDIUM = ModelDims(d_model=512, n_heads=4, n_kv_heads=4, head_dim=128, ffn=1536, rope_sections=(16, 24, 24))


def test_layer_medium_droid_layout_batch2():
    run = LayerRun(MEDIUM, synth.preset("droid").layout, batch=2)
    h, h_out = run.gpu(sigma=1.0, sigma_next=0.9)
    _check(run, h, h_out, 1.0, 0.9)


def test_layer_gqa_and_block_causal():
    dims = ModelDims(d_model=512, n_heads=4, n_kv_heads=2, head_dim=128, ffn=1024, rope_sections=(16, 24, 24))
    spec = LayoutSpec(n_text=20, video=VideoSpec(2, 5, 13, 24, 2, 3))
    run = LayerRun(dims, spec, mode="block_causal")
    h, h_out = run.gpu()
    _check(run, h, h_out)


def test_layer_hd64_gqa():
    dims = ModelDims(d_model=256, n_heads=4, n_kv_heads=2, head_dim=64, ffn=1024, rope_sections=(8, 12, 12))
    run = LayerRun(dims, synth.preset("tiny").layout)
    h, h_out = run.gpu()
    _check(run, h, h_out)


def test_ar_rows_bit_identical_under_dm_perturbation():
    """AR never reads DM: on the GPU the AR rows of h_out do not change by a
    single bit when every DM input row changes (no tile mixes AR and DM rows,
    no atomics, no split-K)."""
    run = LayerRun(MEDIUM, synth.preset("droid").layout)
    _, out_a = run.gpu()
    h2 = run.h.copy()
    n_ar = run.lay.n_ar
    h2[:, n_ar:] = synth.make_activations(h2.shape[1] - n_ar, MEDIUM.d_model, 999)[None]
    _, out_b = run.gpu(h_bits=h2)
    np.testing.assert_array_equal(bits(out_a[0])[:n_ar], bits(out_b[0])[:n_ar])
    assert (bits(out_a[0])[n_ar:] != bits(out_b[0])[n_ar:]).any()


def test_ar_rows_bit_identical_under_generator_weight_change():
    """AR rows use only Reasoner weights: replacing every Generator weight
    (norm gains, QKV, O, FFN) leaves the AR rows of h_out unchanged to the bit
    and changes the DM rows."""
    run = LayerRun(MEDIUM, synth.preset("droid").layout)
    _, out_a = run.gpu()
    other = synth.make_weights(MEDIUM, 1099)
    w2 = {k: (other[k] if k.startswith("G.") else v) for k, v in run.w.items()}
    layer2 = A.MoTLayer(cdims(A, MEDIUM), device_weights(w2))
    h = to_dev(run.h)
    out_b = torch.empty_like(h)
    layer2.forward(h, out_b, 0.8, 0.7, run.seq)
    torch.cuda.synchronize()
    assert_device_ok()
    n_ar = run.lay.n_ar
    np.testing.assert_array_equal(bits(out_a[0])[:n_ar], bits(out_b[0])[:n_ar])
    assert (bits(out_a[0])[n_ar:] != bits(out_b[0])[n_ar:]).any()


def test_layer_is_deterministic():
    run = LayerRun(MEDIUM, synth.preset("droid").layout)
    a = run.gpu()
    b = run.gpu()
    np.testing.assert_array_equal(bits(a[0]), bits(b[0]))
    np.testing.assert_array_equal(bits(a[1]), bits(b[1]))
