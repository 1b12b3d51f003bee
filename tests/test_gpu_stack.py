"""Layer stacks on the GPU against the fp64 oracle (needs a B200).

"Cosmos 3 方法原理全解" §12.4: the released models stack 28/36/64 MoT layers;
the velocity head and the Euler step follow the last one (§7.2).  Every layer
stores its output in bf16 and adds its own independent rounding error, so the
Gaussian rounding term and rel-L2 grow with the square root of the layer count
(`depth` in tests/tolerance.py).  The sampler over a stack keeps its state in
float32 (cosmot_stack_forward_io): its steps add nothing further.
"""

import numpy as np
import pytest

import synth
from oracle import layer as olayer
from oracle import layout as olayout
from synth import ModelDims
from tolerance import SIGMA_H_OUT, SIGMA_VEL, assert_close, rms

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():  # pragma: no cover
    pytest.skip("no CUDA device", allow_module_level=True)

from flow_matching_dit_cosmot_b200 import api as A  # noqa: E402
from flow_matching_dit_cosmot_b200 import _lib as L  # noqa: E402
from gpu_helpers import assert_device_ok, bits, device_weights, dims as cdims, layout_spec, to_dev, to_f64  # noqa

GQA = ModelDims(d_model=512, n_heads=4, n_kv_heads=2, head_dim=128, ffn=1536, rope_sections=(16, 24, 24))


class StackRun:
    def __init__(self, dims, spec, n_layers, batch=1, seed=3100, act_seed=3200, mode="full"):
        self.dims, self.n_layers, self.batch, self.mode = dims, n_layers, batch, mode
        self.lay = olayout.build_layout(spec)
        self.w = synth.make_stack_weights(dims, seed, n_layers)
        self.W = [olayer.weights_from_bits(dims, w) for w in self.w]
        n = self.lay.n_tokens
        self.h = np.stack([synth.make_activations(n, dims.d_model, act_seed + 100 * b) for b in range(batch)])
        self.dlay = A.build_layout(layout_spec(A, spec))
        self.cs = A.mrope_table(self.dlay.pos, dims.head_dim, dims.rope_sections, dims.rope_base)
        self.stack = A.MoTStack(cdims(A, dims), [device_weights(w) for w in self.w])
        mm = L.COSMOT_MASK_FULL if mode == "full" else L.COSMOT_MASK_BLOCK_CAUSAL
        self.seq = lambda n_cached=0: self.stack.seq_desc(self.lay.n_ar, self.lay.n_clean, self.lay.n_noisy, batch,
                                                          self.cs, self.dlay.chunk, mm, n_cached=n_cached)


@pytest.mark.parametrize("mode", ["full", "block_causal"])
def test_stack_of_three_layers(mode):
    run = StackRun(GQA, synth.preset("droid").layout, 3, batch=2, mode=mode)
    hd_ = to_dev(run.h)
    h_out = torch.empty_like(hd_)
    run.stack.forward(hd_, h_out, 1.0, 0.9, run.seq())
    torch.cuda.synchronize()
    assert_device_ok()
    lay = run.lay
    noisy = lay.region == olayout.REGION_NOISY
    for b in range(run.batch):
        ref = olayer.stack_forward(GQA, run.W, synth.bf16_to_f64(run.h[b]), lay.region, lay.pos, lay.chunk, 1.0,
                                   0.9, mode)
        # the FFN branch of the last layer: its attention half from the oracle's
        # layer on the stack's hidden state before it
        last_in = ref["hidden"][-2] if run.n_layers > 1 else synth.bf16_to_f64(run.h[b])
        last = olayer.layer_forward(GQA, run.W[-1], last_in, lay.region, lay.pos, lay.chunk, 1.0, 0.9, mode,
                                    head=False)
        assert_close(to_f64(h_out[b]), ref["h_out"], f"stack h_out[{b}]", sigma=SIGMA_H_OUT,
                     branch_rms=rms(last["h2"] - last["h1"]), depth=run.n_layers)
        vel = ref["vel"][noisy]
        assert_close(to_f64(hd_[b])[noisy], ref["x_new"][noisy], f"stack x'[{b}]", sigma=SIGMA_VEL,
                     branch_rms=0.1 * rms(vel), depth=run.n_layers)
        np.testing.assert_array_equal(bits(hd_[b])[~noisy], run.h[b][~noisy])


def test_stack_sampler_reuses_every_layers_ar_kv():
    """Steps after the first skip the AR rows in every layer; the result is
    bit-identical to recomputing them (deterministic kernels, AR rows never
    read DM rows), and the three steps follow the oracle's stack sampler."""
    run = StackRun(GQA, synth.preset("droid").layout, 4)
    sig = (1.0, 0.8, 0.6, 0.4)
    hd_ = to_dev(run.h)
    h_out = torch.empty_like(hd_)
    ws = run.stack.workspace(run.seq())
    lay = run.lay
    noisy = lay.region == olayout.REGION_NOISY
    ref_h, outs = olayer.stack_sample(GQA, run.W, synth.bf16_to_f64(run.h[0]), lay, sig)
    x32 = torch.empty((1, lay.n_noisy, GQA.d_model), dtype=torch.float32, device="cuda")
    for k, (s0, s1) in enumerate(zip(sig[:-1], sig[1:])):
        if k == 0:
            run.stack.forward(hd_, h_out, s0, s1, run.seq(0), ws, x_state=x32, state_from_h=True)
        else:
            # the same step recomputed from scratch in a separate workspace
            h_full, out_full, x_full = hd_.clone(), torch.empty_like(h_out), x32.clone()
            ws2 = torch.empty_like(ws)
            run.stack.forward(h_full, out_full, s0, s1, run.seq(0), ws2, x_state=x_full)
            run.stack.forward(hd_, h_out, s0, s1, run.seq(lay.n_ar), ws, x_state=x32)
            torch.cuda.synchronize()
            np.testing.assert_array_equal(bits(hd_), bits(h_full))
            np.testing.assert_array_equal(x32.cpu().numpy(), x_full.cpu().numpy())
            np.testing.assert_array_equal(bits(h_out)[0, lay.n_ar:], bits(out_full)[0, lay.n_ar:])
        torch.cuda.synchronize()
        assert_device_ok()
        vel = outs[k]["vel"][noisy]
        assert_close(x32[0].double().cpu().numpy(), outs[k]["x_new"][noisy], f"stack sampler x' step {k + 1}",
                     sigma=SIGMA_VEL, branch_rms=abs(s1 - s0) * rms(vel), depth=run.n_layers, out_bf16=False)
        np.testing.assert_array_equal(bits(hd_[0])[noisy], bits(x32[0].to(torch.bfloat16)))
    np.testing.assert_allclose(to_f64(hd_[0])[~noisy], ref_h[~noisy], rtol=0, atol=0)


def test_stack_argument_errors():
    run = StackRun(GQA, synth.preset("tiny").layout, 2)
    hd_ = to_dev(run.h)
    h_out = torch.empty_like(hd_)
    ws = run.stack.workspace(run.seq())
    sh = A.stream_handle()
    f = L.cosmot_stack_forward
    assert f(run.stack.dims, run.stack.cw, run.seq(), hd_.data_ptr(), hd_.data_ptr(), 1.0, 0.9, ws.data_ptr(),
             ws.numel(), sh, check=False) == L.COSMOT_ERR_INVALID_ARG
    assert f(run.stack.dims, run.stack.cw, run.seq(run.lay.n_ar + 1), hd_.data_ptr(), h_out.data_ptr(), 1.0, 0.9,
             ws.data_ptr(), ws.numel(), sh, check=False) == L.COSMOT_ERR_UNSUPPORTED
    assert f(run.stack.dims, run.stack.cw, run.seq(), hd_.data_ptr(), h_out.data_ptr(), 1.0, 0.9, ws.data_ptr(),
             ws.numel() - 256, sh, check=False) == L.COSMOT_ERR_WORKSPACE
    torch.cuda.synchronize()
    assert_device_ok()


def test_stack_timed_entry_matches():
    """The stage-timed stack entry computes exactly what the plain one does."""
    run = StackRun(GQA, synth.preset("droid").layout, 2)
    ha, hb = to_dev(run.h), to_dev(run.h)
    oa, ob = torch.empty_like(ha), torch.empty_like(hb)
    run.stack.forward(ha, oa, 1.0, 0.9, run.seq())
    ws = torch.empty_like(run.stack.workspace(run.seq()))
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(8 * 2 + 2)]
    for e in evs:
        e.record()
    L.cosmot_stack_forward_timed(run.stack.dims, run.stack.cw, run.seq(), hb.data_ptr(), ob.data_ptr(), 1.0, 0.9,
                                 ws.data_ptr(), ws.numel(), A.stream_handle(), [e.cuda_event for e in evs])
    torch.cuda.synchronize()
    assert_device_ok()
    np.testing.assert_array_equal(bits(ha), bits(hb))
    np.testing.assert_array_equal(bits(oa), bits(ob))
    assert all(evs[i].elapsed_time(evs[i + 1]) >= 0 for i in range(len(evs) - 1))


def test_stack_timed_entry_with_sparse_events_matches():
    """Given only the two events around one stage of every layer (the others
    NULL, which leaves those boundaries unmarked), the stage-timed stack entry
    still computes exactly what the plain one does, and each given pair times
    its stage."""
    run = StackRun(GQA, synth.preset("droid").layout, 2)
    ha, hb = to_dev(run.h), to_dev(run.h)
    oa, ob = torch.empty_like(ha), torch.empty_like(hb)
    run.stack.forward(ha, oa, 1.0, 0.9, run.seq())
    ws = torch.empty_like(run.stack.workspace(run.seq()))
    gate_up = 5  # stage index of the gate/up projection inside a layer
    keep = {8 * lyr + gate_up + e for lyr in range(2) for e in (0, 1)}
    evs = [torch.cuda.Event(enable_timing=True) if k in keep else None for k in range(8 * 2 + 2)]
    for e in evs:
        if e is not None:
            e.record()
    L.cosmot_stack_forward_timed(run.stack.dims, run.stack.cw, run.seq(), hb.data_ptr(), ob.data_ptr(), 1.0, 0.9,
                                 ws.data_ptr(), ws.numel(), A.stream_handle(),
                                 [e.cuda_event if e is not None else None for e in evs])
    torch.cuda.synchronize()
    assert_device_ok()
    np.testing.assert_array_equal(bits(ha), bits(hb))
    np.testing.assert_array_equal(bits(oa), bits(ob))
    for lyr in range(2):
        assert evs[8 * lyr + gate_up].elapsed_time(evs[8 * lyr + gate_up + 1]) > 0
