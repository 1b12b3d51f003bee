"""Shared helpers for the GPU parity tests: moving seeded bf16 inputs to the
device and results back, and translating synth workloads into C-ABI structs."""

from __future__ import annotations

import numpy as np
import torch

import synth


def to_dev(u16: np.ndarray) -> torch.Tensor:
    """bf16 bit pattern (uint16) -> CUDA bf16 tensor with identical bits."""
    t = torch.from_numpy(np.ascontiguousarray(u16).view(np.int16)).view(torch.bfloat16)
    return t.cuda()


def to_f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().view(torch.int16).numpy().view(np.uint16)


def layout_spec(A, spec, tau_offset: int = 0):
    v = spec.video
    video = None if v is None else (v.views, v.grid_h, v.grid_w, v.fps, v.clean_steps, v.noisy_steps)
    return A.layout_spec(spec.n_text, video, spec.audio_clean, spec.audio_noisy, spec.audio_rate,
                         spec.action_clean, spec.action_noisy, spec.action_hz, spec.proprio, tau_offset)


def dims(A, d: synth.ModelDims):
    return A.make_dims(d.d_model, d.n_heads, d.n_kv_heads, d.head_dim, d.ffn, d.rope_sections, d.rope_base, d.eps)


def device_weights(w: dict) -> dict:
    return {k: to_dev(v) for k, v in w.items()}


def assert_device_ok():
    from flow_matching_dit_cosmot_b200 import _lib as L
    st, where = L.cosmot_get_device_status(torch.cuda.current_stream().cuda_stream)
    assert st == 0, f"device status {L.status_string(st)} at site {where}"


def sample_rows(n: int, seg_bounds, k: int, seed: int = 0) -> np.ndarray:
    """A seeded row subset that holds the first and last row of every segment."""
    rng = np.random.default_rng(seed)
    rows = set(rng.choice(n, size=min(k, n), replace=False).tolist())
    for b, e in seg_bounds:
        if e > b:
            rows.update([b, e - 1])
    return np.array(sorted(rows), dtype=np.int64)


def layer_parity(what, ref, noisy, dsigma, h_out=None, x_new=None, vel=None, x_f32=False, depth=1):
    """The parity checks of one layer call against the oracle's outputs `ref`
    (layer_forward's dict, rows already selected to match the arrays given):
    h_out against h2 (its rounding term propagates through the FFN branch
    h2 - h1), and on the `noisy` rows the velocity against v and the state
    against x' = x + dsigma v.  `x_new` and `vel` hold the noisy rows only;
    `x_f32`: the state is the float32 sampler state (no bf16 half-ulp)."""
    from tolerance import SIGMA_H_OUT, SIGMA_VEL, assert_close, rms
    if h_out is not None:
        assert_close(h_out, ref["h2"], f"{what} h_out", sigma=SIGMA_H_OUT, branch_rms=rms(ref["h2"] - ref["h1"]),
                     depth=depth)
    if not np.asarray(noisy).any():
        return
    v = ref["vel"][noisy]
    if vel is not None:
        assert_close(vel, v, f"{what} velocity", sigma=SIGMA_VEL, branch_rms=rms(v), depth=depth)
    if x_new is not None:
        assert_close(x_new, ref["x_new"][noisy], f"{what} x'", sigma=SIGMA_VEL, branch_rms=abs(dsigma) * rms(v),
                     depth=depth, out_bf16=not x_f32)


CANARY = 0x7BAD  # a bf16 NaN pattern no kernel writes


class Guarded:
    """A contiguous bf16 buffer with `guard` canary elements before and after
    it, so a test can check that a call wrote nothing outside its output."""

    def __init__(self, data: torch.Tensor, guard: int = 4096):
        n = data.numel()
        self.raw = torch.full((n + 2 * guard,), CANARY, dtype=torch.int16, device=data.device)
        self.guard = guard
        self.t = self.raw[guard:guard + n].view(torch.bfloat16).view(data.shape)
        self.t.copy_(data)

    def assert_canaries(self, what: str = ""):
        g = self.guard
        raw = self.raw.cpu().numpy()
        bad = int((raw[:g] != CANARY).sum() + (raw[-g:] != CANARY).sum())
        assert bad == 0, f"{what}: {bad} guard elements around the buffer were overwritten"
