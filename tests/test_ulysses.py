"""Sequence-parallel (Ulysses) host logic on CPU.

The index plan (row shards, the head columns each rank owns, the blocks each
pair of ranks trades) and the exchange over torch.distributed are the parts of
flow_matching_dit_cosmot_b200.ulysses that run on the host.  Here gloo ranks
follow that plan with the fp64 oracle doing the arithmetic of each phase, and
the reassembled result must equal the oracle's single-process layer.  The GPU
phases are tested by emulating the ranks on one GPU (test_gpu_ulysses.py).
"""

import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def test_row_shards_and_head_blocks_partition_the_work():
    sys.path.insert(0, ROOT)
    from flow_matching_dit_cosmot_b200.ulysses import head_split, shard_rows
    for n, p in ((703, 2), (703, 4), (18978, 8), (5, 5)):
        rows = shard_rows(n, p)
        assert rows[0][0] == 0 and rows[-1][1] == n
        assert all(a[1] == b[0] for a, b in zip(rows, rows[1:]))
        sizes = [r1 - r0 for r0, r1 in rows]
        assert max(sizes) - min(sizes) <= 1
    with pytest.raises(ValueError):
        shard_rows(3, 4)
    with pytest.raises(ValueError):
        head_split(32, 8, 128, 3)
    for H, Hkv, p in ((32, 8, 4), (32, 8, 8), (64, 8, 8), (40, 40, 8), (4, 2, 2)):
        hs = head_split(H, Hkv, 128, p)
        covered = np.zeros((H + 2 * Hkv) * 128, int)
        for s in range(p):
            packed = np.zeros(hs.packed_cols, int)
            for src, width, dst in hs.blocks(s):
                covered[src:src + width] += 1
                packed[dst:dst + width] += 1
            # a rank's query heads read its own key/value heads (GQA groups stay whole)
            q0 = hs.blocks(s)[0][0] // 128
            k0 = (hs.blocks(s)[1][0] - H * 128) // 128
            assert q0 // (H // Hkv) == k0
            assert (packed == 1).all()  # each rank's packed row is filled exactly once
        assert (covered == 1).all()      # every column of a q/k/v row goes to exactly one rank


def _worker(rank, world, port, q, mode):
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import synth
        from oracle import layer as ol
        from oracle import layout as olayout
        from oracle import rope as orope
        from oracle.mask import allow_matrix
        from flow_matching_dit_cosmot_b200.ulysses import exchange, head_split, shard_rows

        dims = synth.ModelDims(d_model=64, n_heads=8, n_kv_heads=4, head_dim=8, ffn=96, rope_sections=(1, 1, 2))
        spec = synth.LayoutSpec(n_text=7, video=synth.VideoSpec(1, 3, 4, 24, 1, 2))
        lay = olayout.build_layout(spec)
        W = ol.weights_from_bits(dims, synth.make_weights(dims, 77))
        h = synth.bf16_to_f64(synth.make_activations(lay.n_tokens, dims.d_model, 78))
        n, H, Hk, hd = lay.n_tokens, dims.n_heads, dims.n_kv_heads, dims.head_dim
        rows = shard_rows(n, world)
        r0, r1 = rows[rank]
        hs = head_split(H, Hk, hd, world)
        hl = h[r0:r1]
        ar = lay.region[r0:r1] == olayout.REGION_AR

        def proj(name, x, heads):
            out = ol.routed(x, ar, lambda xx, s, sel: ol.rms_norm(xx, getattr(W, s).g1, dims.eps)
                            @ getattr(getattr(W, s), name).T)
            return out.reshape(len(x), heads, hd)

        # phase 1: q, k, v of this rank's rows (rotated), as one full q/k/v row
        pos = lay.pos[r0:r1]
        qr = orope.apply(proj("wq", hl, H), pos, hd, dims.rope_sections, dims.rope_base)
        kr = orope.apply(proj("wk", hl, Hk), pos, hd, dims.rope_sections, dims.rope_base)
        vr = proj("wv", hl, Hk)
        full = np.concatenate([qr.reshape(len(hl), -1), kr.reshape(len(hl), -1), vr.reshape(len(hl), -1)], axis=1)
        send1 = []
        for s in range(world):
            packed = np.zeros((len(hl), hs.packed_cols))
            for src, width, dst in hs.blocks(s):
                packed[:, dst:dst + width] = full[:, src:src + width]
            send1.append(torch.from_numpy(packed))
        recv1 = [torch.empty((b - a, hs.packed_cols), dtype=torch.float64) for a, b in rows]
        exchange(send1, recv1)
        qkv = torch.cat(recv1).numpy()
        # phase 2: this rank's heads over every row
        qh = qkv[:, :hs.hq * hd].reshape(n, hs.hq, hd)
        kh = qkv[:, hs.hq * hd:(hs.hq + hs.hk) * hd].reshape(n, hs.hk, hd)
        vh = qkv[:, (hs.hq + hs.hk) * hd:].reshape(n, hs.hk, hd)
        allow = allow_matrix(np.arange(n), lay.region, lay.chunk, mode)
        oh = ol.attention(qh, kh, vh, allow, 1.0 / np.sqrt(hd)).reshape(n, hs.hq * hd)
        send2 = [torch.from_numpy(np.ascontiguousarray(oh[a:b])) for a, b in rows]
        recv2 = [torch.empty((r1 - r0, hs.hq * hd), dtype=torch.float64) for _ in range(world)]
        exchange(send2, recv2)
        o_local = torch.cat(recv2, dim=1).numpy()
        # phase 3: the rest of the layer on this rank's rows
        h1 = hl + ol.routed(o_local, ar, lambda x, s, sel: x @ getattr(W, s).wo.T)

        def ffn(x, s, sel):
            ws = getattr(W, s)
            b = ol.rms_norm(x, ws.g2, dims.eps)
            return (ol.silu(b @ ws.wg.T) * (b @ ws.wu.T)) @ ws.wd.T

        h2 = h1 + ol.routed(h1, ar, ffn)
        noisy = lay.region[r0:r1] == olayout.REGION_NOISY
        x_new = hl.copy()
        if noisy.any():
            vel = ol.rms_norm(h2[noisy], W.gfin, dims.eps) @ W.wvel.T
            x_new[noisy] = ol.euler_step(hl[noisy], vel, 0.8, 0.6)
        q.put((rank, r0, r1, h2, x_new))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,mode", [(2, "full"), (4, "full"), (2, "block_causal")])
def test_sequence_parallel_plan_reproduces_the_layer(world, mode):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q, mode)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=300) for _ in range(world)]
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    sys.path.insert(0, ROOT)
    import synth
    from oracle import layer as ol
    from oracle import layout as olayout
    dims = synth.ModelDims(d_model=64, n_heads=8, n_kv_heads=4, head_dim=8, ffn=96, rope_sections=(1, 1, 2))
    lay = olayout.build_layout(synth.LayoutSpec(n_text=7, video=synth.VideoSpec(1, 3, 4, 24, 1, 2)))
    W = ol.weights_from_bits(dims, synth.make_weights(dims, 77))
    h = synth.bf16_to_f64(synth.make_activations(lay.n_tokens, dims.d_model, 78))
    ref = ol.layer_forward(dims, W, h, lay.region, lay.pos, lay.chunk, 0.8, 0.6, mode)
    noisy = lay.region == olayout.REGION_NOISY
    want_x = h.copy()
    want_x[noisy] = ref["x_new"][noisy]
    for rank, r0, r1, h2, x_new in res:
        np.testing.assert_allclose(h2, ref["h2"][r0:r1], rtol=0, atol=1e-12)
        np.testing.assert_allclose(x_new, want_x[r0:r1], rtol=0, atol=1e-12)
