"""Sequence-parallel (Ulysses) execution of one MoT layer over P ranks.

One long sequence is split into P contiguous row shards.  Each rank runs the
routed norm and the QKV projection (with mRoPE) on its rows, trades rows for
heads in one all-to-all (every rank then holds all rows of H/P query heads and
Hkv/P key/value heads), runs the MoT attention for its heads over the whole
sequence, trades back in a second all-to-all, and finishes the O projection,
the FFN and the velocity head on its own rows.  The routed projections need no
communication; the two exchanges move each rank's q/k/v and o once.

The arithmetic of every output element is that of the single-GPU layer
(cosmot_layer_forward): a projection row does not depend on the other rows of
its tile, and a head's attention does not depend on the other heads.

This module is host logic: the index plan (row shards, head columns, the
blocks each pair of ranks trades), the exchange over torch.distributed, and
the per-rank phases that call the library.  Device memory comes from torch.
"""

from __future__ import annotations

from dataclasses import dataclass
from typing import List, Tuple

import torch

from . import _lib as L
from .api import MoTLayer, ptr, stream_handle


def shard_rows(n: int, p: int) -> List[Tuple[int, int]]:
    """Contiguous row ranges of p ranks over n rows (sizes differ by at most one)."""
    if p < 1 or n < p:
        raise ValueError(f"cannot split {n} rows over {p} ranks")
    return [(r * n // p, (r + 1) * n // p) for r in range(p)]


@dataclass(frozen=True)
class HeadSplit:
    """The heads rank s owns and where they sit in a full q/k/v row."""
    hq: int      # query heads per rank
    hk: int      # key/value heads per rank
    head_dim: int
    q_cols: int  # H * head_dim: K starts here in a full q/k/v row
    kv_cols: int  # Hkv * head_dim

    def blocks(self, s: int) -> List[Tuple[int, int, int]]:
        """(source column, width, destination column) of rank s's q, k and v
        blocks: full q/k/v row -> the rank's packed [q | k | v] row."""
        hd = self.head_dim
        return [(s * self.hq * hd, self.hq * hd, 0),
                (self.q_cols + s * self.hk * hd, self.hk * hd, self.hq * hd),
                (self.q_cols + self.kv_cols + s * self.hk * hd, self.hk * hd, (self.hq + self.hk) * hd)]

    @property
    def packed_cols(self) -> int:
        return (self.hq + 2 * self.hk) * self.head_dim


def head_split(n_heads: int, n_kv_heads: int, head_dim: int, p: int) -> HeadSplit:
    if n_heads % p or n_kv_heads % p:
        raise ValueError(f"{n_heads} query and {n_kv_heads} key/value heads do not split over {p} ranks")
    return HeadSplit(n_heads // p, n_kv_heads // p, head_dim, n_heads * head_dim, n_kv_heads * head_dim)


def exchange(send: List[torch.Tensor], recv: List[torch.Tensor], group=None):
    """recv[r] on this rank <- send[me] on rank r, for every r (tensors of
    matching shapes; recv[me] receives this rank's own send[me]).  One NCCL
    all-to-all where the backend has it; point-to-point sends and receives
    otherwise (gloo)."""
    import torch.distributed as dist
    if dist.get_backend(group) == "nccl":
        dist.all_to_all(recv, send, group=group)
        return
    me = dist.get_rank(group)
    ops = []
    for r in range(len(send)):
        if r == me:
            recv[r].copy_(send[r])
            continue
        ops.append(dist.P2POp(dist.isend, send[r].contiguous(), r, group))
        ops.append(dist.P2POp(dist.irecv, recv[r], r, group))
    for req in dist.batch_isend_irecv(ops) if ops else []:
        req.wait()


class UlyssesShard:
    """One rank's part of a sequence-parallel layer step.

    Phases: pre() -> exchange(send1, recv1) -> attend() -> exchange(send2,
    recv2) -> post().  The exchange buffers are attributes, so a caller can
    run them over torch.distributed or, to emulate P ranks in one process,
    by copying between shards.
    """

    def __init__(self, layer: MoTLayer, seq: L.SeqDesc, p: int, rank: int, device="cuda"):
        if seq.batch != 1 or seq.n_cached != 0:
            raise ValueError("sequence parallelism takes one sequence without a cached prefix")
        self.layer, self.seq, self.p, self.rank = layer, seq, p, rank
        d = layer.dims
        self.n = seq.n_ar + seq.n_clean + seq.n_noisy
        self.rows = shard_rows(self.n, p)
        self.row0, self.row1 = self.rows[rank]
        self.split = head_split(d.n_heads, d.n_kv_heads, d.head_dim, p)
        self.qkv_cols = (d.n_heads + 2 * d.n_kv_heads) * d.head_dim
        nl = self.row1 - self.row0
        hs = self.split
        bf = dict(dtype=torch.bfloat16, device=device)
        self.qkv_local = torch.empty((nl, self.qkv_cols), **bf)
        self.send1 = [torch.empty((nl, hs.packed_cols), **bf) for _ in range(p)]
        self.qkv_heads = torch.empty((self.n, hs.packed_cols), **bf)  # all rows, this rank's heads
        self.recv1 = [self.qkv_heads[r0:r1] for r0, r1 in self.rows]
        self.o_heads = torch.empty((self.n, hs.hq * hs.head_dim), **bf)
        self.send2 = [self.o_heads[r0:r1] for r0, r1 in self.rows]
        self.recv2 = [torch.empty((nl, hs.hq * hs.head_dim), **bf) for _ in range(p)]
        self.o_local = torch.empty((nl, d.n_heads * d.head_dim), **bf)
        self.ws = torch.empty((L.cosmot_shard_workspace_size(d, nl),), dtype=torch.uint8, device=device)

    def pre(self, h_local: torch.Tensor, stream=None):
        """Norm and QKV of the rank's rows, packed per destination rank."""
        sh = stream_handle(stream)
        L.cosmot_layer_shard_pre(self.layer.dims, self.layer.cw, self.seq, self.row0, self.row1, ptr(h_local),
                                 ptr(self.qkv_local), ptr(self.ws), self.ws.numel(), sh)
        nl = self.row1 - self.row0
        es = self.qkv_local.element_size()
        for s in range(self.p):
            for src_col, width, dst_col in self.split.blocks(s):
                L.cosmot_copy_columns(ptr(self.qkv_local) + src_col * es, self.qkv_cols,
                                      ptr(self.send1[s]) + dst_col * es, self.split.packed_cols, nl, width, sh)

    def attend(self, stream=None):
        """The rank's heads over all rows (after the first exchange)."""
        hs, seq = self.split, self.seq
        es = self.qkv_heads.element_size()
        d = L.AttnDesc(n_q=self.n, q_key_offset=0, n_keys=self.n, n_ar=seq.n_ar, n_heads=hs.hq, n_kv_heads=hs.hk,
                       head_dim=hs.head_dim, mask_mode=seq.mask_mode, chunk=seq.chunk, batch=1)
        base = ptr(self.qkv_heads)
        L.cosmot_mot_attention(d, base, hs.packed_cols, base + hs.hq * hs.head_dim * es,
                               base + (hs.hq + hs.hk) * hs.head_dim * es, hs.packed_cols, ptr(self.o_heads),
                               hs.hq * hs.head_dim, stream_handle(stream))

    def post(self, h_local: torch.Tensor, h_out_local: torch.Tensor, sigma: float, sigma_next: float, stream=None):
        """Reassemble o (heads in order) and finish the layer on the rank's rows."""
        sh = stream_handle(stream)
        nl = self.row1 - self.row0
        w = self.split.hq * self.split.head_dim
        es = self.o_local.element_size()
        for s in range(self.p):
            L.cosmot_copy_columns(ptr(self.recv2[s]), w, ptr(self.o_local) + s * w * es, self.o_local.shape[1], nl, w,
                                  sh)
        L.cosmot_layer_shard_post(self.layer.dims, self.layer.cw, self.seq, self.row0, self.row1, ptr(h_local),
                                  ptr(self.o_local), ptr(h_out_local), sigma, sigma_next, ptr(self.ws),
                                  self.ws.numel(), sh)

    def forward(self, h_local, h_out_local, sigma, sigma_next, group=None):
        """All phases on this rank, the exchanges over torch.distributed."""
        self.pre(h_local)
        exchange(self.send1, self.recv1, group)
        self.attend()
        exchange(self.send2, self.recv2, group)
        self.post(h_local, h_out_local, sigma, sigma_next)


def emulate(shards: List[UlyssesShard], h_locals, h_out_locals, sigma: float, sigma_next: float):
    """All P ranks of one layer step in one process on one GPU: the same phases,
    the exchanges done by copying between the shards' buffers."""
    for sh, h in zip(shards, h_locals):
        sh.pre(h)
    for s, dst in enumerate(shards):
        for r, src in enumerate(shards):
            dst.recv1[r].copy_(src.send1[s])
    for sh in shards:
        sh.attend()
    for r, dst in enumerate(shards):
        for s, src in enumerate(shards):
            dst.recv2[s].copy_(src.send2[r])
    for sh, h, ho in zip(shards, h_locals, h_out_locals):
        sh.post(h, ho, sigma, sigma_next)
