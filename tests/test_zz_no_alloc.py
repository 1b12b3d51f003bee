"""The layer entry point for callers that may not allocate device memory.

It runs the same layer as cosmot_layer_forward but takes its workspace from
the fixed array inside the library.  Checked through the C ABI against the
regular entry point (with a caller-allocated workspace) on two calls in a row,
so the second call starts from whatever the first left in the shared array.
Kept in a file that pytest collects last.
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


@pytest.mark.parametrize("case", ["tiny", "droid_medium"])
def test_noalloc_matches_regular_entry_point_twice(case):
    if case == "tiny":
        wl = synth.preset("tiny")
        dims, spec, seeds = wl.dims, wl.layout, (wl.act_seed(), wl.act_seed() + 1)
    else:
        dims = ModelDims(d_model=512, n_heads=4, n_kv_heads=4, head_dim=128, ffn=1536, rope_sections=(16, 24, 24))
        spec, seeds = synth.preset("droid").layout, (2003, 2004)
    layer, seq, hs, _keep = _setup(dims, spec, 1001, seeds)
    assert layer.workspace_bytes(seq) <= L.COSMOT_NOALLOC_SCRATCH_BYTES
    sh = torch.cuda.current_stream().cuda_stream
    for h_bits in hs:  # two calls in a row with different inputs
        h_ref, out_ref = to_dev(h_bits), None
        out_ref = torch.empty_like(h_ref)
        layer.forward(h_ref, out_ref, 0.8, 0.7, seq)  # regular entry point, torch-allocated workspace
        h_na = to_dev(h_bits)
        out_na = torch.empty_like(h_na)
        L.cosmot_layer_forward_noalloc(layer.dims, layer.cw, seq, h_na.data_ptr(), out_na.data_ptr(), 0.8, 0.7, sh)
        torch.cuda.synchronize()
        assert_device_ok()
        assert_close(to_f64(out_na), to_f64(out_ref), "h_out (no-alloc vs regular)")
        assert_close(to_f64(h_na), to_f64(h_ref), "x' (no-alloc vs regular)")
        # same kernels, deterministic: identical bits as well
        np.testing.assert_array_equal(bits(out_na), bits(out_ref))
        np.testing.assert_array_equal(bits(h_na), bits(h_ref))


def test_noalloc_rejects_sizes_beyond_its_array():
    wl = synth.preset("t2v480")  # about 1.55 GB of workspace
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
