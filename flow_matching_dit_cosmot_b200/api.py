"""PyTorch-facing helpers around the C ABI.

PyTorch provides device memory and streams; every step of the layer runs in
libcosmot's kernels.  These helpers only allocate outputs/workspace with torch
and translate tensors into the pointers and structs the C entry points take.
"""

from __future__ import annotations

from dataclasses import dataclass
from typing import Optional

import torch

from . import _lib as L

L.lib()  # the CUDA library must be present; no fallback


def ptr(t: Optional[torch.Tensor]) -> int:
    return 0 if t is None else t.data_ptr()


def stream_handle(stream: Optional[torch.cuda.Stream] = None) -> int:
    return (stream if stream is not None else torch.cuda.current_stream()).cuda_stream


def _need_cuda(*ts):
    for t in ts:
        if t is not None and not t.is_cuda:
            raise ValueError("libcosmot takes CUDA tensors only (no CPU fallback)")


WEIGHT_TENSORS = ("g1", "wqkv", "wo", "g2", "wg", "wu", "wd")


def weight_shapes(dims: L.Dims) -> dict:
    """Shape of every tensor of a layer's weight dict (row-major [out, in])."""
    d, f, hd = dims.d_model, dims.ffn, dims.head_dim
    per_set = {"g1": (d,), "wqkv": ((dims.n_heads + 2 * dims.n_kv_heads) * hd, d), "wo": (d, dims.n_heads * hd),
               "g2": (d,), "wg": (f, d), "wu": (f, d), "wd": (d, f)}
    shapes = {f"{s}.{t}": shp for s in ("R", "G") for t, shp in per_set.items()}
    shapes["gfin"] = (d,)
    shapes["wvel"] = (d, d)
    return shapes


def _check_bf16(t: torch.Tensor, name: str):
    if t.dtype != torch.bfloat16 or not t.is_contiguous():
        raise ValueError(f"{name}: libcosmot takes contiguous bf16 tensors (got {t.dtype}, "
                         f"{'contiguous' if t.is_contiguous() else 'strided'})")


def check_weights(dims: L.Dims, weights: dict):
    """The kernels read every weight through a bare pointer, so a tensor of the
    wrong shape, dtype or layout would be read out of bounds: refuse it here."""
    for name, shp in weight_shapes(dims).items():
        if name not in weights:
            raise ValueError(f"weight {name!r} missing")
        t = weights[name]
        if tuple(t.shape) != shp:
            raise ValueError(f"weight {name!r} has shape {tuple(t.shape)}, expected {shp}")
        _check_bf16(t, f"weight {name!r}")
    _need_cuda(*weights.values())


def _check_state(seq: L.SeqDesc, d: int, **ts):
    """h / h_out hold [batch][N][d] bf16 (N = n_ar + n_clean + n_noisy)."""
    rows = seq.batch * (seq.n_ar + seq.n_clean + seq.n_noisy)
    for name, t in ts.items():
        _check_bf16(t, name)
        if t.numel() < rows * d:
            raise ValueError(f"{name} holds {t.numel()} elements, fewer than batch x N x d = {rows * d}")
    _need_cuda(*ts.values())


def layout_spec(n_text: int, video=None, audio_clean=0, audio_noisy=0, audio_rate=25, action_clean=0,
                action_noisy=0, action_hz=15, proprio=0, tau_offset=0) -> L.LayoutSpec:
    """`video` = (views, grid_h, grid_w, fps, clean_steps, noisy_steps) or None."""
    v = video if video is not None else (0, 0, 0, 0, 0, 0)
    return L.LayoutSpec(n_text, *[int(x) for x in v], audio_clean, audio_noisy, audio_rate, action_clean,
                        action_noisy, action_hz, proprio, tau_offset)


@dataclass
class DeviceLayout:
    pos: torch.Tensor     # float32 [N, 3]
    chunk: torch.Tensor   # int32 [N]
    region: torch.Tensor  # int8 [N]
    n_ar: int
    n_clean: int
    n_noisy: int

    @property
    def n_tokens(self) -> int:
        return self.n_ar + self.n_clean + self.n_noisy


def build_layout(spec: L.LayoutSpec, device="cuda", stream=None) -> DeviceLayout:
    n, a, c, z = L.cosmot_layout_counts(spec)
    pos = torch.empty((n, 3), dtype=torch.float32, device=device)
    chunk = torch.empty((n,), dtype=torch.int32, device=device)
    region = torch.empty((n,), dtype=torch.int8, device=device)
    L.cosmot_build_layout(spec, ptr(pos), ptr(chunk), ptr(region), stream_handle(stream))
    return DeviceLayout(pos, chunk, region, a, c, z)


def mrope_table(pos: torch.Tensor, head_dim: int, sections, rope_base: float = 10000.0, stream=None) -> torch.Tensor:
    _need_cuda(pos)
    cs = torch.empty((pos.shape[0], head_dim // 2, 2), dtype=torch.float32, device=pos.device)
    L.cosmot_mrope_table(ptr(pos), pos.shape[0], head_dim, sections, rope_base, ptr(cs), stream_handle(stream))
    return cs


def make_dims(d_model, n_heads, n_kv_heads, head_dim, ffn, rope_sections, rope_base=10000.0, eps=1e-6) -> L.Dims:
    return L.Dims(d_model, n_heads, n_kv_heads, head_dim, ffn, (L.c_i32 * 3)(*rope_sections), rope_base, eps, 0)


class MoTLayer:
    """One MoT layer: both weight sets resident on the device.

    `weights` maps names to bf16 CUDA tensors: "R.*"/"G.*" for the Reasoner and
    Generator sets (g1, wqkv, wo, g2, wg, wu, wd), plus "gfin" and "wvel".
    """

    def __init__(self, dims: L.Dims, weights: dict):
        self.dims = dims
        self.weights = weights
        check_weights(dims, weights)
        sets = []
        for s in ("R", "G"):
            sets.append(L.SetWeights(*[ptr(weights[f"{s}.{t}"]) for t in ("g1", "wqkv", "wo", "g2", "wg", "wu", "wd")]))
        self.cw = L.LayerWeights((L.SetWeights * 2)(*sets), ptr(weights["gfin"]), ptr(weights["wvel"]))
        self._ws = None

    def seq_desc(self, n_ar, n_clean, n_noisy, batch, rope_cs, chunk=None, mask_mode=L.COSMOT_MASK_FULL,
                 n_cached=0) -> L.SeqDesc:
        """The descriptor holds raw pointers: rope_cs and chunk must stay alive while it is used."""
        return L.SeqDesc(n_ar, n_clean, n_noisy, batch, mask_mode, n_cached, ptr(rope_cs), ptr(chunk))

    def workspace_bytes(self, seq: L.SeqDesc) -> int:
        return L.cosmot_layer_workspace_size(self.dims, seq)

    def workspace(self, seq: L.SeqDesc, device="cuda") -> torch.Tensor:
        n = self.workspace_bytes(seq)
        if self._ws is None or self._ws.numel() < n:
            self._ws = torch.empty((n,), dtype=torch.uint8, device=device)
        return self._ws

    def commit_kv(self, h: torch.Tensor, seq: L.SeqDesc, dst_row: int, workspace: Optional[torch.Tensor] = None,
                  stream=None):
        """K/V of rows [seq.n_cached, N) of h into cache rows [dst_row, ...) of the workspace."""
        _check_state(seq, self.dims.d_model, h=h)
        ws = workspace if workspace is not None else self.workspace(seq, h.device)
        L.cosmot_layer_commit_kv(self.dims, self.cw, seq, ptr(h), dst_row, ptr(ws), ws.numel(), stream_handle(stream))

    def forward_cfg(self, h: torch.Tensor, h_out: torch.Tensor, sigma: float, sigma_next: float, guidance: float,
                    seq: L.SeqDesc, workspace: Optional[torch.Tensor] = None, stream=None):
        """Guided step: h [2P, N, d] holds (conditioned, baseline) pairs sharing their DM rows."""
        _check_state(seq, self.dims.d_model, h=h, h_out=h_out)
        ws = workspace if workspace is not None else self.workspace(seq, h.device)
        L.cosmot_layer_forward_cfg(self.dims, self.cw, seq, ptr(h), ptr(h_out), float(sigma), float(sigma_next),
                                   float(guidance), ptr(ws), ws.numel(), stream_handle(stream))

    def forward(self, h: torch.Tensor, h_out: torch.Tensor, sigma: float, sigma_next: float, seq: L.SeqDesc,
                workspace: Optional[torch.Tensor] = None, stream=None, x_state: Optional[torch.Tensor] = None,
                state_from_h: bool = False, vel: Optional[torch.Tensor] = None):
        """h [batch, N, d] bf16 (noisy DM rows updated in place to x'); h_out [batch, N, d] bf16.

        x_state: optional float32 [batch, n_noisy, d] sampler state of the noisy
        rows, read (unless state_from_h) and written in float32; h's noisy rows
        then receive its bf16 copy.  vel: optional bf16 [batch, n_noisy, d]
        receiving the velocity (see cosmot_layer_forward_io)."""
        _check_state(seq, self.dims.d_model, h=h, h_out=h_out)
        ws = workspace if workspace is not None else self.workspace(seq, h.device)
        io = self.step_io(seq, x_state, state_from_h, vel)
        if io is None:
            L.cosmot_layer_forward(self.dims, self.cw, seq, ptr(h), ptr(h_out), float(sigma), float(sigma_next),
                                   ptr(ws), ws.numel(), stream_handle(stream))
        else:
            L.cosmot_layer_forward_io(self.dims, self.cw, seq, ptr(h), ptr(h_out), float(sigma), float(sigma_next),
                                      io, ptr(ws), ws.numel(), stream_handle(stream))

    def step_io(self, seq: L.SeqDesc, x_state: Optional[torch.Tensor] = None, state_from_h: bool = False,
                vel: Optional[torch.Tensor] = None) -> Optional[L.StepIO]:
        """The StepIO struct for an optional float32 state and velocity output,
        both [batch, n_noisy, d] contiguous (checked here: the kernels read and
        write them through bare pointers)."""
        if x_state is None and vel is None:
            return None
        d, rows = self.dims.d_model, seq.batch * seq.n_noisy
        for name, t, dt in (("x_state", x_state, torch.float32), ("vel", vel, torch.bfloat16)):
            if t is None:
                continue
            _need_cuda(t)
            if t.dtype != dt or not t.is_contiguous() or t.numel() < rows * d:
                raise ValueError(f"{name}: expected a contiguous {dt} tensor of batch x n_noisy x d = {rows * d} "
                                 f"elements (got {t.dtype}, {t.numel()})")
        return L.step_io(ptr(x_state), d, ptr(vel), d, state_from_h)


class MoTStack:
    """A stack of MoT layers with one velocity head (that of the last layer).

    `layers` is a list of weight dicts as MoTLayer takes (bf16 CUDA tensors);
    the same dict may appear more than once.
    """

    def __init__(self, dims: L.Dims, layers: list):
        self.dims = dims
        self.layers = [MoTLayer(dims, w) for w in layers]
        self.cw = (L.LayerWeights * len(self.layers))(*[m.cw for m in self.layers])
        self._ws = None

    def seq_desc(self, *args, **kw) -> L.SeqDesc:
        return self.layers[0].seq_desc(*args, **kw)

    def workspace_bytes(self, seq: L.SeqDesc) -> int:
        return L.cosmot_stack_workspace_size(self.dims, len(self.layers), seq)

    def workspace(self, seq: L.SeqDesc, device="cuda") -> torch.Tensor:
        n = self.workspace_bytes(seq)
        if self._ws is None or self._ws.numel() < n:
            self._ws = torch.empty((n,), dtype=torch.uint8, device=device)
        return self._ws

    def forward(self, h: torch.Tensor, h_out: torch.Tensor, sigma: float, sigma_next: float, seq: L.SeqDesc,
                workspace: Optional[torch.Tensor] = None, stream=None, x_state: Optional[torch.Tensor] = None,
                state_from_h: bool = False, vel: Optional[torch.Tensor] = None):
        """h^L into h_out; x' into the noisy rows of h (see cosmot_stack_forward);
        x_state / vel as for MoTLayer.forward."""
        _check_state(seq, self.dims.d_model, h=h, h_out=h_out)
        ws = workspace if workspace is not None else self.workspace(seq, h.device)
        io = self.layers[0].step_io(seq, x_state, state_from_h, vel)
        if io is None:
            L.cosmot_stack_forward(self.dims, self.cw, seq, ptr(h), ptr(h_out), sigma, sigma_next, ptr(ws),
                                   ws.numel(), stream_handle(stream))
        else:
            L.cosmot_stack_forward_io(self.dims, self.cw, seq, ptr(h), ptr(h_out), sigma, sigma_next, io, ptr(ws),
                                      ws.numel(), stream_handle(stream))
