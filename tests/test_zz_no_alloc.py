"""The layer entry point for callers that may not allocate device memory.

Some callers cannot call cudaMalloc once they run: a robot or simulator
control loop with a hard per-step deadline (an allocation can synchronise the
device and stall), or a host framework whose own pool owns all device memory.
cosmot_layer_forward_noalloc runs the same layer as cosmot_layer_forward but
takes its workspace from a fixed array inside the library.

Checked through the C ABI against the regular entry point (caller-allocated
workspace) on two calls in a row after a first call on a different layout,
so the calls under test start from whatever earlier calls left in the shared
array.  The regular entry point's workspace is filled with 0xFF (bf16 NaN)
before each of its calls, so a read of scratch that the call did not write
would show up as a difference.  After the warm-up call the device's free
memory must not change across a call.  Kept in a file that pytest collects
last.
"""

import numpy as np
import pytest

import synth
from oracle import layout as olayout
from synth import ModelDims
from tolerance import assert_close

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():  # pragma: no cover
    pytest.skip("no CUDA device", allow_module_level=True)

from flow_matching_dit_cosmot_b200 import api as A  # noqa: E402
from flow_matching_dit_cosmot_b200 import _lib as L  # noqa: E402
from gpu_helpers import assert_device_ok, bits, device_weights, dims as cdims, layout_spec, to_dev, to_f64  # noqa


def _setup(dims, spec, weight_seed, act_seeds):
    w = synth.make_weights(dims, weight_seed)
    lay = olayout.build_layout(spec)
    dlay = A.build_layout(layout_spec(A, spec))
    cs = A.mrope_table(dlay.pos, dims.head_dim, dims.rope_sections, dims.rope_base)
    layer = A.MoTLayer(cdims(A, dims), device_weights(w))
    seq = layer.seq_desc(dlay.n_ar, dlay.n_clean, dlay.n_noisy, 1, cs, dlay.chunk)
    hs = [synth.make_activations(lay.n_tokens, dims.d_model, s) for s in act_seeds]
    return layer, seq, hs, (dlay, cs)


def _noalloc(layer, seq, h_bits):
    sh = torch.cuda.current_stream().cuda_stream
    h = to_dev(h_bits)
    out = torch.empty_like(h)
    torch.cuda.synchronize()
    free_before = torch.cuda.mem_get_info()[0]
    L.cosmot_layer_forward_noalloc(layer.dims, layer.cw, seq, h.data_ptr(), out.data_ptr(), 0.8, 0.7, sh)
    torch.cuda.synchronize()
    free_after = torch.cuda.mem_get_info()[0]
    assert_device_ok()
    return h, out, free_before, free_after


@pytest.mark.parametrize("case", ["tiny", "droid_medium"])
def test_noalloc_matches_regular_entry_point_twice(case):
    tiny = synth.preset("tiny")
    if case == "tiny":
        dims, spec, seeds = tiny.dims, tiny.layout, (tiny.act_seed(), tiny.act_seed() + 1)
        other = (ModelDims(d_model=512, n_heads=4, n_kv_heads=4, head_dim=128, ffn=1536, rope_sections=(16, 24, 24)),
                 synth.preset("droid").layout)
    else:
        dims = ModelDims(d_model=512, n_heads=4, n_kv_heads=4, head_dim=128, ffn=1536, rope_sections=(16, 24, 24))
        spec, seeds = synth.preset("droid").layout, (2003, 2004)
        other = (tiny.dims, tiny.layout)
    # a call on another layout first: the array then holds that call's leftovers
    o_layer, o_seq, o_hs, _o_keep = _setup(other[0], other[1], 1002, (2005,))
    _noalloc(o_layer, o_seq, o_hs[0])

    layer, seq, hs, _keep = _setup(dims, spec, 1001, seeds)
    assert layer.workspace_bytes(seq) <= L.COSMOT_NOALLOC_SCRATCH_BYTES
    for h_bits in hs:  # two calls in a row with different inputs
        h_ref = to_dev(h_bits)
        out_ref = torch.empty_like(h_ref)
        ws = torch.empty(layer.workspace_bytes(seq), dtype=torch.uint8, device="cuda")
        ws.fill_(255)  # every unwritten byte reads as a bf16 NaN
        layer.forward(h_ref, out_ref, 0.8, 0.7, seq, workspace=ws)  # regular entry point
        h_na, out_na, free_before, free_after = _noalloc(layer, seq, h_bits)
        assert free_after == free_before, "the no-alloc call changed the device's free memory"
        assert_close(to_f64(out_na), to_f64(out_ref), "h_out (no-alloc vs regular)")
        assert_close(to_f64(h_na), to_f64(h_ref), "x' (no-alloc vs regular)")
        # same kernels, deterministic: identical bits as well
        np.testing.assert_array_equal(bits(out_na), bits(out_ref))
        np.testing.assert_array_equal(bits(h_na), bits(h_ref))
        assert np.isfinite(to_f64(out_na)).all()


def test_noalloc_rejects_sizes_beyond_its_array():
    wl = synth.preset("t2v480")  # about 1.7 GB of workspace
    dm = wl.dims
    dims = A.make_dims(dm.d_model, dm.n_heads, dm.n_kv_heads, dm.head_dim, dm.ffn, dm.rope_sections)
    cs = torch.zeros((16, 2), dtype=torch.float32, device="cuda")
    seq = L.SeqDesc(258, 0, 18720, 1, 0, 0, cs.data_ptr(), 0)
    assert L.cosmot_layer_workspace_size(dims, seq) > L.COSMOT_NOALLOC_SCRATCH_BYTES
    h = torch.zeros((16, 8), dtype=torch.bfloat16, device="cuda")
    code = L.cosmot_layer_forward_noalloc(dims, L.LayerWeights(), seq, h.data_ptr(), h.data_ptr(), 1.0, 0.97,
                                          torch.cuda.current_stream().cuda_stream, check=False)
    assert code == L.COSMOT_ERR_WORKSPACE
    seq_cached = L.SeqDesc(2, 0, 4, 1, 0, 2, cs.data_ptr(), 0)
    code = L.cosmot_layer_forward_noalloc(dims, L.LayerWeights(), seq_cached, h.data_ptr(), h.data_ptr(), 1.0, 0.97,
                                          torch.cuda.current_stream().cuda_stream, check=False)
    assert code == L.COSMOT_ERR_UNSUPPORTED
