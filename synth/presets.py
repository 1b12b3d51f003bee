"""Workload shapes of the Cosmos 3 Mixture-of-Transformers layer.

Five named workloads.  Each one fixes the model widths, the packed-sequence
contents (how many AR text tokens, which DM modalities, how many clean and
noisy latent steps) and the sampler schedule.  Only sizes and counts live
here; the coordinates and masks derived from them are computed separately by
the oracle and by the CUDA layout kernel.

Sources for the numbers (page titles as published):
  * "Cosmos 3 方法原理全解" §4.1: 832x480 video -> 26x15 latent grid, 189
    frames -> 48 latent steps; §8.1: I2V = 1 clean + 47 noisy latent steps;
    §8.2: DROID policy, three camera views, 15 Hz actions, 32 action steps.
  * "NVIDIA 发布 Cosmos 3 系列四个开放权重世界模型", "流式生成如何工作":
    block-causal streaming with a key/value cache, one latent step (four RGB
    frames) per block.
  * NVIDIA/cosmos README, generation settings: 24 FPS default, 480p =
    832x480, 720p = 1280x720, 256p = 320x192.
"""

from __future__ import annotations

from dataclasses import dataclass, field
from typing import Optional, Tuple


@dataclass(frozen=True)
class ModelDims:
    """Widths of one MoT layer (both weight sets share them)."""

    d_model: int
    n_heads: int
    n_kv_heads: int
    head_dim: int
    ffn: int
    rope_sections: Tuple[int, int, int]  # frequency pairs given to t, h, w
    rope_base: float = 10000.0
    eps: float = 1e-6

    @property
    def q_cols(self) -> int:
        return self.n_heads * self.head_dim

    @property
    def kv_cols(self) -> int:
        return self.n_kv_heads * self.head_dim

    @property
    def qkv_cols(self) -> int:
        return self.q_cols + 2 * self.kv_cols


@dataclass(frozen=True)
class VideoSpec:
    """Video latents: `views` camera views tiled along w, each grid_h x grid_w
    tokens per latent step; `clean_steps` conditioning steps first, then
    `noisy_steps` steps to be generated, on one continuous time axis."""

    views: int
    grid_h: int
    grid_w: int
    fps: int
    clean_steps: int
    noisy_steps: int

    @property
    def tokens_per_step(self) -> int:
        return self.views * self.grid_h * self.grid_w


@dataclass(frozen=True)
class StreamSpec:
    """Streaming rollout: a ring of `cached_blocks` history blocks, `blocks`
    new blocks generated, `steps_per_block` denoising steps each."""

    cached_blocks: int
    blocks: int
    steps_per_block: int


@dataclass(frozen=True)
class LayoutSpec:
    """Contents of one packed sequence [AR text, EOS, BOG, clean DM, noisy DM]."""

    n_text: int
    video: Optional[VideoSpec]
    audio_clean: int = 0
    audio_noisy: int = 0
    audio_rate: int = 25  # tokens per second (48 kHz, hop 1920)
    action_clean: int = 0
    action_noisy: int = 0
    action_hz: int = 15
    proprio: int = 0  # clean proprioception tokens

    @property
    def n_ar(self) -> int:
        return self.n_text + 2  # + EOS + BOG

    @property
    def n_clean(self) -> int:
        v = self.video.clean_steps * self.video.tokens_per_step if self.video else 0
        return v + self.audio_clean + self.action_clean + self.proprio

    @property
    def n_noisy(self) -> int:
        v = self.video.noisy_steps * self.video.tokens_per_step if self.video else 0
        return v + self.audio_noisy + self.action_noisy

    @property
    def n_dm(self) -> int:
        return self.n_clean + self.n_noisy

    @property
    def n_tokens(self) -> int:
        return self.n_ar + self.n_dm


@dataclass(frozen=True)
class Workload:
    name: str
    config_id: int
    dims: ModelDims
    layout: LayoutSpec
    sigmas: Tuple[float, ...]  # sampler schedule, sigma_0 > sigma_1 > ...
    batch: int = 1
    mask_mode: str = "full"  # "full" | "block_causal"
    stream: Optional[StreamSpec] = None
    guidance: Optional[float] = None  # classifier-free guidance weight; batch = (cond, base) pairs
    n_layers: int = 1  # > 1: a layer stack with one velocity head
    weight_draws: int = 0  # > 0: that many distinct layer weight draws, cycled over the stack
    shift: float = 0.0  # > 0: sigmas come from the flow-shift schedule over n_sampler_steps (sigmas left empty)
    n_sampler_steps: int = 0
    action_dim: int = 0  # > 0: the action rows go through W_in / W_out heads of this width
    description: str = ""
    extra: dict = field(default_factory=dict)

    @property
    def weight_seed(self) -> int:
        return 1000 + self.config_id

    def act_seed(self, batch_idx: int = 0) -> int:
        return 2000 + self.config_id + 100 * batch_idx


_NANO_LIKE = ModelDims(d_model=4096, n_heads=32, n_kv_heads=32, head_dim=128,
                       ffn=14336, rope_sections=(16, 24, 24))
_SUPER_LIKE = ModelDims(d_model=5120, n_heads=40, n_kv_heads=40, head_dim=128,
                        ffn=20480, rope_sections=(16, 24, 24))
# Page-exact widths ("Cosmos 3 方法原理全解" §12.4 model table): Nano 36 layers,
# hidden 4096, 32 query / 8 key-value heads, FFN 12288; Super 64 layers, hidden
# 5120, 64 / 8 heads, FFN 25600.  Head size 128 in both (not printed; the
# Qwen3-VL-initialised Reasoner uses 128, so Super's query width is 8192).
NANO = ModelDims(d_model=4096, n_heads=32, n_kv_heads=8, head_dim=128, ffn=12288, rope_sections=(16, 24, 24))
SUPER = ModelDims(d_model=5120, n_heads=64, n_kv_heads=8, head_dim=128, ffn=25600, rope_sections=(16, 24, 24))
_TINY = ModelDims(d_model=256, n_heads=4, n_kv_heads=4, head_dim=64, ffn=1024,
                  rope_sections=(8, 12, 12))


def _linear_sigmas(steps: int) -> Tuple[float, ...]:
    return tuple(1.0 - k / steps for k in range(steps)) + (0.0,)


PRESETS = {
    "tiny": Workload(
        name="tiny", config_id=1, dims=_TINY,
        layout=LayoutSpec(n_text=32, video=VideoSpec(1, 4, 4, 24, 2, 4)),
        sigmas=(0.8, 0.7),
        description="tiny MoT layer: d 256, 4x64 heads, FFN 1024; 34 AR + 32 clean + 64 noisy"),
    "t2v480": Workload(
        name="t2v480", config_id=2, dims=_NANO_LIKE,
        layout=LayoutSpec(n_text=256, video=VideoSpec(1, 15, 26, 24, 0, 48)),
        sigmas=(1.0, 0.97),
        description="480p text-to-video layer: d 4096, 32x128 heads, FFN 14336; 258 AR + 18720 noisy"),
    "t2v480_cfg": Workload(
        name="t2v480_cfg", config_id=2, dims=_NANO_LIKE,
        layout=LayoutSpec(n_text=256, video=VideoSpec(1, 15, 26, 24, 0, 48)),
        sigmas=(1.0, 0.97), batch=2, guidance=6.0,
        description="480p text-to-video guided step: one (cond, base) prompt pair sharing the 18720 noisy "
                    "rows, guidance 6"),
    "droid": Workload(
        name="droid", config_id=3, dims=_NANO_LIKE,
        layout=LayoutSpec(n_text=128, video=VideoSpec(3, 6, 10, 15, 1, 2),
                          action_noisy=32, action_hz=15, proprio=1),
        sigmas=_linear_sigmas(10),
        description="DROID policy step: 130 AR + 181 clean + 392 noisy, 10 Euler steps"),
    "droid_b16": Workload(
        name="droid_b16", config_id=3, dims=_NANO_LIKE,
        layout=LayoutSpec(n_text=128, video=VideoSpec(3, 6, 10, 15, 1, 2),
                          action_noisy=32, action_hz=15, proprio=1),
        sigmas=_linear_sigmas(10), batch=16,
        description="DROID policy step, batch 16"),
    "stream": Workload(
        name="stream", config_id=4, dims=_NANO_LIKE,
        layout=LayoutSpec(n_text=64, video=VideoSpec(4, 15, 26, 24, 0, 1)),
        sigmas=(1.0, 0.75, 0.5, 0.25, 0.0), mask_mode="block_causal",
        stream=StreamSpec(cached_blocks=8, blocks=16, steps_per_block=4),
        description="streaming block-causal rollout: 1560-token blocks, 8 cached blocks, 66 AR"),
    "t2v480_nano": Workload(
        name="t2v480_nano", config_id=2, dims=NANO,
        layout=LayoutSpec(n_text=256, video=VideoSpec(1, 15, 26, 24, 0, 48)),
        sigmas=(1.0, 0.97),
        description="480p text-to-video layer at Nano's widths: d 4096, 32 query / 8 key-value heads of 128, "
                    "FFN 12288; 258 AR + 18720 noisy"),
    "i2v720_super": Workload(
        name="i2v720_super", config_id=5, dims=SUPER,
        layout=LayoutSpec(n_text=512, video=VideoSpec(1, 22, 40, 24, 1, 47)),
        sigmas=(1.0, 0.97),
        description="720p image-to-video layer at Super's widths: d 5120, 64 query / 8 key-value heads of 128, "
                    "FFN 25600; 514 AR + 880 clean + 41360 noisy"),
    "droid_nano36": Workload(
        name="droid_nano36", config_id=3, dims=NANO,
        layout=LayoutSpec(n_text=128, video=VideoSpec(3, 6, 10, 15, 1, 2),
                          action_noisy=32, action_hz=15, proprio=1),
        sigmas=_linear_sigmas(10), n_layers=36, weight_draws=4,
        description="DROID policy step through Nano's 36-layer stack (page widths), 10 Euler steps; 4 distinct "
                    "layer weight draws of 0.77 GB cycled over the 36 layers"),
    "droid_policy": Workload(
        name="droid_policy", config_id=3, dims=NANO,
        layout=LayoutSpec(n_text=128, video=VideoSpec(3, 6, 10, 15, 1, 2),
                          action_noisy=32, action_hz=15, proprio=1),
        sigmas=(), n_layers=36, weight_draws=4, shift=5.0, n_sampler_steps=4, guidance=3.0, batch=2,
        action_dim=8,
        description="DROID policy inference: Nano's 36-layer stack, a (cond, base) prompt pair with guidance 3, "
                    "4 steps of the shift-5 schedule, 32 x 8-D joint-position actions through W_in / W_out; 4 "
                    "distinct layer weight draws cycled over the 36 layers"),
    "i2v720": Workload(
        name="i2v720", config_id=5, dims=_SUPER_LIKE,
        layout=LayoutSpec(n_text=512, video=VideoSpec(1, 22, 40, 24, 1, 47)),
        sigmas=(1.0, 0.97),
        description="720p image-to-video layer: d 5120, 40x128 heads, FFN 20480; 514 AR + 880 clean + 41360 noisy"),
}


def preset(name: str) -> Workload:
    if name not in PRESETS:
        raise KeyError(f"unknown workload {name!r}; known: {sorted(PRESETS)}")
    return PRESETS[name]
