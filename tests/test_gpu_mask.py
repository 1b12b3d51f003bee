"""The attention kernel's masking, exported by cosmot_mot_mask_export, against
the oracle's visibility matrix ("Cosmos 3 方法原理全解" §3 equations; the
block-causal variant of "流式生成如何工作").  Needs a B200.

The element visibility must equal the oracle's bit for bit.  The tile codes
are the kernel's own choice; the test checks what the definition fixes about
them: a skipped tile holds no key the row sees, an unmasked tile holds only
keys the row sees, a masked tile holds at least one it does not, and every
CTA (AR or DM, full or block-causal mask) visits exactly the key tiles that
one of its rows needs: fully masked tiles are skipped.
"""

import numpy as np
import pytest

from oracle import layout as olayout
from oracle import mask as omask
import synth
from synth import LayoutSpec, VideoSpec

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():  # pragma: no cover
    pytest.skip("no CUDA device", allow_module_level=True)

from flow_matching_dit_cosmot_b200 import api as A  # noqa: E402
from flow_matching_dit_cosmot_b200 import _lib as L  # noqa: E402
from gpu_helpers import assert_device_ok  # noqa: E402

BKV = 128
CTA_ROWS = 256  # two 128-row query tiles per CTA


def _export(region, chunk, mode, q_off, n_q):
    n_keys = len(region)
    n_ar = int((region == olayout.REGION_AR).sum())
    n_kt = (n_keys + BKV - 1) // BKV
    tiles = torch.full((n_q, n_kt), 255, dtype=torch.uint8, device="cuda")
    vis = torch.full((n_q, n_keys), 255, dtype=torch.uint8, device="cuda")
    chd = torch.from_numpy(np.ascontiguousarray(chunk, dtype=np.int32)).cuda()
    d = L.AttnDesc(n_q=n_q, q_key_offset=q_off, n_keys=n_keys, n_ar=n_ar, n_heads=4, n_kv_heads=2, head_dim=128,
                   mask_mode=L.COSMOT_MASK_FULL if mode == omask.FULL else L.COSMOT_MASK_BLOCK_CAUSAL,
                   chunk=A.ptr(chd), batch=1)
    L.cosmot_mot_mask_export(d, A.ptr(tiles), A.ptr(vis), A.stream_handle())
    torch.cuda.synchronize()
    assert_device_ok()
    return tiles.cpu().numpy(), vis.cpu().numpy(), n_ar


def _check(region, chunk, mode, q_off=0, n_q=None):
    n_keys = len(region)
    n_q = n_keys - q_off if n_q is None else n_q
    codes, vis, n_ar = _export(region, chunk, mode, q_off, n_q)
    rows = q_off + np.arange(n_q)
    allow = omask.allow_matrix(rows, region, chunk, mode)
    np.testing.assert_array_equal(vis.astype(bool), allow)
    assert set(np.unique(codes)) <= {0, 1, 2}

    n_kt = codes.shape[1]
    pad = n_kt * BKV - n_keys
    allow_t = np.concatenate([allow, np.zeros((n_q, pad), bool)], axis=1).reshape(n_q, n_kt, BKV)
    in_range = np.concatenate([np.ones(n_keys, bool), np.zeros(pad, bool)]).reshape(n_kt, BKV)
    any_vis = allow_t.any(axis=2)
    all_vis = allow_t.all(axis=2) & in_range.all(axis=1)[None, :]
    assert not (any_vis & (codes == 0)).any(), "a skipped tile holds a visible key"
    assert (all_vis[codes == 1]).all(), "an unmasked tile holds a hidden key"
    assert not (all_vis[codes == 2]).any(), "a fully visible tile was masked"

    is_ar_q = region[rows] == olayout.REGION_AR
    # AR query rows and DM query rows are each grouped into CTAs of 256
    # consecutive rows from their first row; a CTA visits exactly the key tiles
    # that one of its rows needs.
    for idx in (np.nonzero(is_ar_q)[0], np.nonzero(~is_ar_q)[0]):
        for g0 in range(0, len(idx), CTA_ROWS):
            grp = idx[g0:g0 + CTA_ROWS]
            needed = any_vis[grp].any(axis=0)
            visited = (codes[grp] != 0)
            assert (visited == needed[None, :]).all(), "a CTA's visited tiles differ from what its rows need"
    return codes


def _layout(spec):
    lay = olayout.build_layout(spec)
    return lay, np.asarray(lay.region), np.asarray(lay.chunk, dtype=np.int32)


@pytest.mark.parametrize("mode", [omask.FULL, omask.BLOCK_CAUSAL])
@pytest.mark.parametrize("name", ["tiny", "droid", "unaligned_chunks", "long_ar", "long_block_causal"])
def test_mask_export_matches_oracle(name, mode):
    spec = {
        "tiny": LayoutSpec(n_text=32, video=VideoSpec(1, 4, 4, 24, 2, 4)),
        "droid": LayoutSpec(n_text=128, video=VideoSpec(3, 6, 10, 15, 1, 2), action_noisy=32, action_hz=15,
                            proprio=1),
        "unaligned_chunks": LayoutSpec(n_text=20, video=VideoSpec(2, 5, 13, 24, 2, 3)),
        "long_ar": LayoutSpec(n_text=600, video=VideoSpec(1, 4, 4, 24, 0, 2)),
        "long_block_causal": LayoutSpec(n_text=30, video=VideoSpec(1, 8, 16, 24, 2, 6)),
    }[name]
    _, region, chunk = _layout(spec)
    codes = _check(region, chunk, mode)
    if mode == omask.BLOCK_CAUSAL and name != "tiny":
        assert (codes == 2).any()
    if mode == omask.BLOCK_CAUSAL and name == "long_block_causal":
        dm = region != olayout.REGION_AR
        assert (codes[dm] == 0).any()  # early DM rows skip the tiles of later chunks


def test_mask_export_query_suffixes():
    """Streaming step (queries = the last block) and a query range that starts
    inside the AR prefix."""
    _, region, chunk = _layout(LayoutSpec(n_text=30, video=VideoSpec(1, 6, 10, 24, 3, 1)))
    n_noisy = int((region == olayout.REGION_NOISY).sum())
    _check(region, chunk, omask.BLOCK_CAUSAL, q_off=len(region) - n_noisy)
    _, region, chunk = _layout(LayoutSpec(n_text=600, video=VideoSpec(1, 4, 4, 24, 0, 2)))
    _check(region, chunk, omask.FULL, q_off=100)
    _check(region, chunk, omask.BLOCK_CAUSAL, q_off=300, n_q=len(region) - 300)


def test_mask_export_rejects_bad_descriptor():
    d = L.AttnDesc(n_q=10, q_key_offset=0, n_keys=10, n_ar=2, n_heads=3, n_kv_heads=2, head_dim=128, batch=1)
    assert L.cosmot_mot_mask_export(d, 256, 0, A.stream_handle(), check=False) == L.COSMOT_ERR_INVALID_ARG
    d = L.AttnDesc(n_q=10, q_key_offset=0, n_keys=10, n_ar=2, n_heads=2, n_kv_heads=2, head_dim=128, batch=1,
                   mask_mode=L.COSMOT_MASK_BLOCK_CAUSAL)
    assert L.cosmot_mot_mask_export(d, 256, 0, A.stream_handle(), check=False) == L.COSMOT_ERR_INVALID_ARG


def test_no_tile_skip_hint_changes_visits_not_results():
    """COSMOT_ATTN_NO_TILE_SKIP only stops the search for skippable tiles:
    every DM tile is visited, the element visibility is unchanged, and the
    attention output is bit-identical (a visited fully hidden tile adds exact
    zeros)."""
    from gpu_helpers import to_dev
    _, region, chunk = _layout(LayoutSpec(n_text=30, video=VideoSpec(1, 8, 16, 24, 2, 6)))
    n = len(region)
    n_ar = int((region == olayout.REGION_AR).sum())
    chd = torch.from_numpy(np.ascontiguousarray(chunk, dtype=np.int32)).cuda()
    n_kt = (n + BKV - 1) // BKV
    H, hd = 4, 128
    q = to_dev(synth.normal_bf16((n, H * hd), 61, 1))
    k = to_dev(synth.normal_bf16((n, H * hd), 62, 1))
    v = to_dev(synth.normal_bf16((n, H * hd), 63, 1))
    outs, codes, viss = [], [], []
    for flags in (0, L.COSMOT_ATTN_NO_TILE_SKIP):
        d = L.AttnDesc(n_q=n, q_key_offset=0, n_keys=n, n_ar=n_ar, n_heads=H, n_kv_heads=H, head_dim=hd,
                       mask_mode=L.COSMOT_MASK_BLOCK_CAUSAL, chunk=A.ptr(chd), batch=1, flags=flags)
        tiles = torch.full((n, n_kt), 255, dtype=torch.uint8, device="cuda")
        vis = torch.full((n, n), 255, dtype=torch.uint8, device="cuda")
        L.cosmot_mot_mask_export(d, A.ptr(tiles), A.ptr(vis), A.stream_handle())
        o = torch.empty((n, H * hd), dtype=torch.bfloat16, device="cuda")
        L.cosmot_mot_attention(d, A.ptr(q), H * hd, A.ptr(k), A.ptr(v), H * hd, A.ptr(o), H * hd, A.stream_handle())
        torch.cuda.synchronize()
        assert_device_ok()
        outs.append(o.cpu().view(torch.int16).numpy())
        codes.append(tiles.cpu().numpy())
        viss.append(vis.cpu().numpy())
    dm = region != olayout.REGION_AR
    assert (codes[0][dm] == 0).any() and not (codes[1][dm] == 0).any()
    np.testing.assert_array_equal(viss[0], viss[1])
    np.testing.assert_array_equal(outs[0], outs[1])
