"""Sequence-parallel layer phases on one GPU (needs a B200).

P ranks are emulated in one process: each shard runs its phases through the
library and the two exchanges are done by copying between the shards'
buffers (the ranks never wait on one another).  The reassembled result is
checked against the fp64 oracle's layer (h_out and x' of every row), and,
since every output element is computed with the same arithmetic as the
single-GPU layer, it must also be bit-identical to cosmot_layer_forward.
"""

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
from flow_matching_dit_cosmot_b200.ulysses import UlyssesShard, emulate  # noqa: E402
from gpu_helpers import (assert_device_ok, bits, device_weights, dims as cdims, layer_parity, layout_spec,  # noqa: E402
                         to_dev, to_f64)

DIMS = ModelDims(d_model=512, n_heads=8, n_kv_heads=4, head_dim=64, ffn=1024, rope_sections=(8, 12, 12))


@pytest.mark.parametrize("p,name,mode", [(2, "droid", "full"), (4, "droid", "full"),
                                         (2, "unaligned", "block_causal"), (4, "unaligned", "block_causal")])
def test_emulated_ranks_equal_the_single_gpu_layer(p, name, mode):
    spec = {"droid": synth.preset("droid").layout,
            "unaligned": LayoutSpec(n_text=20, video=VideoSpec(2, 5, 13, 24, 2, 3))}[name]
    lay = olayout.build_layout(spec)
    n = lay.n_tokens
    w = synth.make_weights(DIMS, 4400)
    h = synth.make_activations(n, DIMS.d_model, 4401)
    dlay = A.build_layout(layout_spec(A, spec))
    cs = A.mrope_table(dlay.pos, DIMS.head_dim, DIMS.rope_sections)
    layer = A.MoTLayer(cdims(A, DIMS), device_weights(w))
    mm = L.COSMOT_MASK_FULL if mode == "full" else L.COSMOT_MASK_BLOCK_CAUSAL
    seq = layer.seq_desc(lay.n_ar, lay.n_clean, lay.n_noisy, 1, cs, dlay.chunk, mm)
    h_ref = to_dev(h[None])
    out_ref = torch.empty_like(h_ref)
    layer.forward(h_ref, out_ref, 0.8, 0.6, seq)

    shards = [UlyssesShard(layer, seq, p, r) for r in range(p)]
    h_loc = [to_dev(h[sh.row0:sh.row1]) for sh in shards]
    out_loc = [torch.empty_like(x) for x in h_loc]
    emulate(shards, h_loc, out_loc, 0.8, 0.6)
    torch.cuda.synchronize()
    assert_device_ok()
    # the shards' rows put back together, against the oracle ("Cosmos 3 方法原理全解" §3, §7.2)
    got_h = np.concatenate([to_f64(x) for x in h_loc])
    got_out = np.concatenate([to_f64(o) for o in out_loc])
    ref = olayer.layer_forward(DIMS, olayer.weights_from_bits(DIMS, w), synth.bf16_to_f64(h), lay.region, lay.pos,
                               lay.chunk, 0.8, 0.6, mode)
    noisy = lay.region == olayout.REGION_NOISY
    layer_parity(f"ulysses P={p} {name}", ref, noisy, 0.6 - 0.8, h_out=got_out, x_new=got_h[noisy])
    np.testing.assert_array_equal(bits(torch.cat(h_loc))[~noisy], h[~noisy])
    for sh, x, o in zip(shards, h_loc, out_loc):
        np.testing.assert_array_equal(bits(x), bits(h_ref[0, sh.row0:sh.row1]))
        np.testing.assert_array_equal(bits(o), bits(out_ref[0, sh.row0:sh.row1]))


def test_shard_entries_reject_batches_and_cached_prefixes():
    layer_dims = cdims(A, DIMS)
    cs = torch.zeros((16, 2), dtype=torch.float32, device="cuda")
    ws = torch.empty((1 << 20,), dtype=torch.uint8, device="cuda")
    for batch, cached in ((2, 0), (1, 10)):
        seq = L.SeqDesc(20, 0, 100, batch, 0, cached, cs.data_ptr(), 0)
        code = L.cosmot_layer_shard_pre(layer_dims, L.LayerWeights(), seq, 0, 60, 256, 256, ws.data_ptr(), ws.numel(),
                                        A.stream_handle(), check=False)
        assert code == L.COSMOT_ERR_UNSUPPORTED
    seq = L.SeqDesc(20, 0, 100, 1, 0, 0, cs.data_ptr(), 0)
    code = L.cosmot_layer_shard_pre(layer_dims, L.LayerWeights(), seq, 60, 200, 256, 256, ws.data_ptr(), ws.numel(),
                                    A.stream_handle(), check=False)
    assert code == L.COSMOT_ERR_INVALID_ARG
