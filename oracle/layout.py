"""Packed sequence layout and unified 3D mRoPE coordinates (fp64 oracle).

TEST INFRASTRUCTURE (see the package docstring): imported only by tests, the
smoke check and the benchmark's CPU-baseline leg.

Follows "Cosmos 3 方法原理全解":
  §2   one sequence [AR ..., EOS, BOG, DM clean ..., DM noisy ...]; inside each
       DM group the order is vision, audio, action; absent modalities are
       left out.
  §5   every token gets (t, h, w): text t = h = w (1D RoPE); video t = time,
       (h, w) = latent grid; audio and action use t only, h = w = 0.  Video
       latent rate TPS = FPS / 4 and the time step is 6 / TPS, so 24 FPS video
       steps by 1, 25 tok/s audio by 0.24 and 15 Hz actions by 0.4.  The DM
       time axis is offset by 15000 from the AR coordinates (no tokens are
       inserted), and a clean prefix and the noisy future share one time axis.
  §8.2 several camera views are tiled into one canvas; here views sit side by
       side along w.

Readings where the pages leave the formula open:
  * EOS and BOG are AR tokens (Reasoner weights, causal, visible to DM).
  * AR token k has (k, k, k); the DM time origin is T0 = n_ar + 15000.
  * video token (step tau, view v, row y, col x) -> (T0 + tau*dt_v, y, x + v*W).
  * audio token k (counted over the clip, clean first) -> (T0 + k*dt_a, 0, 0).
  * action token k -> (T0 + tau_a0*dt_v + k*dt_act, 0, 0), tau_a0 = first
    noisy video step; proprioception -> (T0 + tau_last_clean*dt_v, 0, 0).
  * chunk id (the block-causal unit) = latent time step: tau for video; the
    step a non-video token's time falls in for the others, in exact integers.
  * coordinates are computed in float64 in the order written above and then
    rounded once to float32; that float32 array is the exact contract.
"""

from __future__ import annotations

from dataclasses import dataclass

import numpy as np

REGION_AR, REGION_CLEAN, REGION_NOISY = 0, 1, 2
MOD_TEXT, MOD_VIDEO, MOD_AUDIO, MOD_ACTION, MOD_PROPRIO = 0, 1, 2, 3, 4

AR_DM_TIME_OFFSET = 15000


def video_time_step(fps: float) -> float:
    """dt for one video latent step: TPS = FPS/4, dt = 6/TPS (§5)."""
    tps = fps / 4.0
    return 6.0 / tps


def rate_time_step(tokens_per_second: float) -> float:
    """dt for a stream sampled at `tokens_per_second` (audio, actions): 6/TPS (§5)."""
    return 6.0 / tokens_per_second


@dataclass
class Layout:
    region: np.ndarray    # int8  [N]   0 AR, 1 clean DM, 2 noisy DM
    modality: np.ndarray  # int8  [N]
    pos64: np.ndarray     # float64 [N, 3]  (t, h, w) before rounding
    pos: np.ndarray       # float32 [N, 3]  the exact contract
    chunk: np.ndarray     # int32 [N]   -1 for AR rows, latent step for DM rows
    n_ar: int
    n_clean: int
    n_noisy: int

    @property
    def n_tokens(self) -> int:
        return self.n_ar + self.n_clean + self.n_noisy

    @property
    def n_dm(self) -> int:
        return self.n_clean + self.n_noisy


def _video_group(video, taus, t0, dt_v):
    """Video tokens ordered by latent step, then view, then grid row, then column."""
    tau, view, y, x = np.meshgrid(np.asarray(taus, dtype=np.int64), np.arange(video.views),
                                  np.arange(video.grid_h), np.arange(video.grid_w), indexing="ij")
    tau, view, y, x = (a.reshape(-1) for a in (tau, view, y, x))
    t = t0 + tau.astype(np.float64) * dt_v
    h = y.astype(np.float64)
    w = (x + view * video.grid_w).astype(np.float64)
    return np.stack([t, h, w], axis=1), tau.astype(np.int32)


def build_layout(spec, tau_offset: int = 0) -> Layout:
    """Layout of one packed sequence described by a ``synth.LayoutSpec``.

    `tau_offset` shifts every video latent step (used for streaming blocks,
    whose single step sits after the cached history).
    """
    n_ar = spec.n_ar
    t0 = float(n_ar + AR_DM_TIME_OFFSET)
    video = spec.video
    fps = video.fps if video is not None else 24
    dt_v = video_time_step(fps)
    dt_a = rate_time_step(spec.audio_rate)
    dt_act = rate_time_step(spec.action_hz)
    cs = video.clean_steps if video is not None else 0
    ns = video.noisy_steps if video is not None else 0
    tau_a0 = tau_offset + cs            # first noisy video step
    tau_p = tau_offset + max(cs - 1, 0)  # last clean video step

    regions, mods, poss, chunks = [], [], [], []

    # AR: text, EOS, BOG with t = h = w = index (§5: text reduces to 1D RoPE).
    k = np.arange(n_ar, dtype=np.float64)
    regions.append(np.full(n_ar, REGION_AR, np.int8))
    mods.append(np.full(n_ar, MOD_TEXT, np.int8))
    poss.append(np.stack([k, k, k], axis=1))
    chunks.append(np.full(n_ar, -1, np.int32))

    def add(region, mod, pos, chunk):
        regions.append(np.full(len(pos), region, np.int8))
        mods.append(np.full(len(pos), mod, np.int8))
        poss.append(pos.reshape(-1, 3))
        chunks.append(np.asarray(chunk, np.int32).reshape(-1))

    def audio(k_lo, k_hi):
        kk = np.arange(k_lo, k_hi, dtype=np.int64)
        t = t0 + kk.astype(np.float64) * dt_a
        z = np.zeros_like(t)
        ch = tau_offset + (kk * fps) // (4 * spec.audio_rate)
        return np.stack([t, z, z], axis=1), ch

    def action(k_lo, k_hi):
        kk = np.arange(k_lo, k_hi, dtype=np.int64)
        a0 = t0 + float(tau_a0) * dt_v
        t = a0 + kk.astype(np.float64) * dt_act
        z = np.zeros_like(t)
        ch = tau_a0 + (kk * fps) // (4 * spec.action_hz)
        return np.stack([t, z, z], axis=1), ch

    # Clean group: vision, audio, action (proprioception counted with actions).
    if video is not None and cs > 0:
        p, ch = _video_group(video, range(tau_offset, tau_offset + cs), t0, dt_v)
        add(REGION_CLEAN, MOD_VIDEO, p, ch)
    if spec.audio_clean:
        p, ch = audio(0, spec.audio_clean)
        add(REGION_CLEAN, MOD_AUDIO, p, ch)
    if spec.action_clean:
        p, ch = action(0, spec.action_clean)
        add(REGION_CLEAN, MOD_ACTION, p, ch)
    if spec.proprio:
        tp = t0 + float(tau_p) * dt_v
        p = np.tile(np.array([[tp, 0.0, 0.0]]), (spec.proprio, 1))
        add(REGION_CLEAN, MOD_PROPRIO, p, np.full(spec.proprio, tau_p))

    # Noisy group: vision, audio, action.
    if video is not None and ns > 0:
        p, ch = _video_group(video, range(tau_offset + cs, tau_offset + cs + ns), t0, dt_v)
        add(REGION_NOISY, MOD_VIDEO, p, ch)
    if spec.audio_noisy:
        p, ch = audio(spec.audio_clean, spec.audio_clean + spec.audio_noisy)
        add(REGION_NOISY, MOD_AUDIO, p, ch)
    if spec.action_noisy:
        p, ch = action(spec.action_clean, spec.action_clean + spec.action_noisy)
        add(REGION_NOISY, MOD_ACTION, p, ch)

    region = np.concatenate(regions)
    pos64 = np.concatenate(poss).astype(np.float64)
    lay = Layout(region=region, modality=np.concatenate(mods), pos64=pos64,
                 pos=pos64.astype(np.float32), chunk=np.concatenate(chunks),
                 n_ar=n_ar, n_clean=int((region == REGION_CLEAN).sum()),
                 n_noisy=int((region == REGION_NOISY).sum()))
    return lay
