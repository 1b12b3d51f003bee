"""The debug build (libcosmot_debug.so) on the GPU (needs a B200).

Its kernels check the index of every global store against the extent the
host derived for the output and latch COSMOT_ERR_BOUNDS instead of writing out
of place.  On odd sizes (an AR prefix of EOS and BOG only, no clean rows, a
noisy count that is not a multiple of 128, chunks that cut key tiles) every
check passes and every output is bit-identical to the release build's.  The
test-only self-check makes one check fail on purpose (its store would still
have been in bounds): the status word reports it and the context keeps
working.  Nothing here faults or traps.
"""

import ctypes

import numpy as np
import pytest

import synth
from oracle import layout as olayout
from synth import LayoutSpec, ModelDims, VideoSpec

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():  # pragma: no cover
    pytest.skip("no CUDA device", allow_module_level=True)

from flow_matching_dit_cosmot_b200 import api as A  # noqa: E402
from flow_matching_dit_cosmot_b200 import _lib as L  # noqa: E402
from gpu_helpers import Guarded, bits, device_weights, dims as cdims, layout_spec, to_dev  # noqa: E402

DIMS = ModelDims(d_model=512, n_heads=4, n_kv_heads=2, head_dim=128, ffn=1536, rope_sections=(16, 24, 24))


def _status(lib):
    st, where = ctypes.c_int32(0), ctypes.c_int32(0)
    assert lib.cosmot_get_device_status(A.stream_handle(), ctypes.byref(st), ctypes.byref(where)) == L.COSMOT_OK
    return st.value, where.value


def _layer(lib, layer, seq, h_bits):
    h = Guarded(to_dev(h_bits))
    out = Guarded(torch.empty_like(h.t))
    ws = torch.full((layer.workspace_bytes(seq),), 255, dtype=torch.uint8, device="cuda")
    code = lib.cosmot_layer_forward(ctypes.byref(layer.dims), ctypes.byref(layer.cw), ctypes.byref(seq),
                                    h.t.data_ptr(), out.t.data_ptr(), 1.0, 0.9, ws.data_ptr(), ws.numel(),
                                    A.stream_handle())
    assert code == L.COSMOT_OK, L.status_string(code)
    torch.cuda.synchronize()
    h.assert_canaries("h")
    out.assert_canaries("h_out")
    return h.t, out.t


@pytest.mark.parametrize("mode", ["full", "block_causal"])
def test_debug_build_passes_its_checks_and_matches_release(mode):
    D = L.lib_debug()
    assert D.cosmot_debug_checks() == 1 and L.lib().cosmot_debug_checks() == 0
    spec = LayoutSpec(n_text=0, video=VideoSpec(1, 5, 7, 24, 0, 3), action_noisy=2)  # 2 AR + 0 clean + 107 noisy
    lay = olayout.build_layout(spec)
    assert lay.n_ar == 2 and lay.n_clean == 0 and lay.n_noisy % 128
    w = synth.make_weights(DIMS, 4500)
    dlay = A.build_layout(layout_spec(A, spec))
    cs = A.mrope_table(dlay.pos, DIMS.head_dim, DIMS.rope_sections)
    layer = A.MoTLayer(cdims(A, DIMS), device_weights(w))
    mm = L.COSMOT_MASK_FULL if mode == "full" else L.COSMOT_MASK_BLOCK_CAUSAL
    seq = layer.seq_desc(lay.n_ar, lay.n_clean, lay.n_noisy, 2, cs, dlay.chunk, mm)
    h = np.stack([synth.make_activations(lay.n_tokens, DIMS.d_model, 4501 + b) for b in range(2)])
    assert _status(D) == (0, 0)
    hd, od = _layer(D, layer, seq, h)
    assert _status(D) == (0, 0), "a store index check of the debug build failed"
    hr, orel = _layer(L.lib(), layer, seq, h)
    np.testing.assert_array_equal(bits(hd), bits(hr))
    np.testing.assert_array_equal(bits(od), bits(orel))


def test_debug_self_check_latches_bounds_and_the_context_keeps_working():
    D = L.lib_debug()
    sh = A.stream_handle()
    assert _status(D) == (0, 0)
    assert D.cosmot_selftest_bounds_check(sh) == L.COSMOT_OK
    torch.cuda.synchronize()
    assert _status(D) == (L.COSMOT_ERR_BOUNDS, L.COSMOT_SITE_SELFTEST_BOUNDS)
    assert _status(D) == (0, 0)  # reading clears it
    # the release build has no such check
    assert L.lib().cosmot_selftest_bounds_check(sh) == L.COSMOT_ERR_UNSUPPORTED
    # later launches of the debug build run normally
    x = to_dev(synth.normal_bf16((64, 64), 4600, 1))
    v = to_dev(synth.normal_bf16((64, 64), 4601, 1))
    x0 = synth.bf16_to_f64(bits(x))
    assert D.cosmot_flow_euler_step(x.data_ptr(), 64, v.data_ptr(), 64, 0, 64, 64, 1.0, 0.5, sh) == L.COSMOT_OK
    torch.cuda.synchronize()
    assert _status(D) == (0, 0)
    want = x0 + (0.5 - 1.0) * synth.bf16_to_f64(bits(v))
    assert np.abs(synth.bf16_to_f64(bits(x)) - want).max() < 2e-2
