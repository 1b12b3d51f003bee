"""The bench's algorithmic work accounting, checked on CPU against the oracle.

The roofline fractions divide algorithmic FLOPs by measured time; the
attention FLOPs count only visible (query, key) pairs.  These tests hold the
bench's closed-form pair count to the oracle's visibility matrix, and its
stage FLOP formulas to the GEMM shapes of the layer definition.
"""

import numpy as np
import pytest

import synth
from oracle import layout as olayout
from oracle import mask as omask
from synth import LayoutSpec, VideoSpec

SPECS = {
    "tiny": synth.preset("tiny").layout,
    "droid": synth.preset("droid").layout,
    "unaligned_chunks": LayoutSpec(n_text=20, video=VideoSpec(2, 5, 13, 24, 2, 3)),
    "audio_action": LayoutSpec(n_text=5, video=VideoSpec(2, 3, 4, 15, 1, 2), audio_clean=3, audio_noisy=7,
                               action_clean=2, action_noisy=9, action_hz=15, proprio=1),
    "no_text": LayoutSpec(n_text=0, video=VideoSpec(1, 2, 2, 30, 0, 3), audio_noisy=11),
}


@pytest.mark.parametrize("mode", [omask.FULL, omask.BLOCK_CAUSAL])
@pytest.mark.parametrize("name", sorted(SPECS))
def test_attention_pair_count_matches_oracle_mask(name, mode):
    import bench
    lay = olayout.build_layout(SPECS[name])
    counts = bench.Counts(lay.n_ar, lay.n_clean, lay.n_noisy, np.asarray(lay.chunk))
    allow = omask.allow_matrix(np.arange(lay.n_tokens), lay.region, lay.chunk, mode)
    assert bench.attention_pairs(counts, mode) == int(allow.sum())


def test_stage_flops_follow_the_layer_shapes():
    """Per stage, 2 x rows x K x N for each projection of the layer (QKV,
    O, gate and up, down, velocity) and 4 x heads x head_dim per visible pair."""
    import bench
    d = synth.presets.NANO
    R, nz, pairs = 1000, 300, 123456
    w = bench.stage_work(d, R, nz, pairs)
    qc = d.n_heads * d.head_dim
    kvc = d.n_kv_heads * d.head_dim
    assert w["qkv_mrope"][0] == 2 * R * d.d_model * (qc + 2 * kvc)
    assert w["attention"][0] == 4 * pairs * d.n_heads * d.head_dim
    assert w["oproj_residual"][0] == 2 * R * qc * d.d_model
    assert w["gateup_silu"][0] == 2 * R * d.d_model * 2 * d.ffn
    assert w["down_residual"][0] == 2 * R * d.ffn * d.d_model
    assert w["velocity_euler"][0] == 2 * nz * d.d_model * d.d_model
    assert all(w[k][0] == 0 for k in ("norm1", "norm2", "norm_final"))


def test_traffic_counters_follow_the_kernel_code_not_its_comments():
    """The ncu traffic a bench line reports is keyed on the kernel's code: a
    comment edit keeps it, any code edit drops it."""
    import bench
    code = "int f(int a) {  // add one\n  return a + 1;\n}\n"
    assert bench.code_sha(code) == bench.code_sha("// header\nint f(int a) {\n\n  return a + 1;  // note\n}\n")
    assert bench.code_sha(code) != bench.code_sha(code.replace("a + 1", "a + 2"))
    for rec in bench.NCU_TRAFFIC.values():
        assert len(rec["src_sha"]) == 16 and rec["bytes_per_launch"] > 0


class _Ev:
    """A stand-in for a CUDA event: a timestamp in ms."""

    def __init__(self, t):
        self.t = t

    def elapsed_time(self, other):
        return other.t - self.t


@pytest.mark.parametrize("n_layers", [1, 2, 36])
def test_stage_spans_follow_the_timed_entry_event_layout(n_layers):
    """Every stage of a layer call maps to one pair of consecutive events, in the
    order the stage-timed entry points record them (one layer: before each stage
    and after the last; a stack: 8 l + i before stage i of layer l, 8 l + 7
    after its last, then the velocity stage between 8 n and 8 n + 1)."""
    import bench
    n_stage = 9
    n_ev = 8 * n_layers + 2 if n_layers > 1 else n_stage + 1
    spans = bench.stage_spans(n_layers, n_stage)
    per_stage = {j: [k for jj, k in spans if jj == j] for j in range(n_stage)}
    for j in range(n_stage):
        assert len(per_stage[j]) == (n_layers if (n_layers > 1 and j < 7) else 1)
    # the spans start at every event but the last, except that in a stack the
    # event after layer l's last stage (8 l + 7, l < n - 1) starts no stage: the
    # time up to the next layer's first event lies between two layers
    starts = sorted(k for _, k in spans)
    between = {8 * lyr + 7 for lyr in range(n_layers - 1)} if n_layers > 1 else set()
    assert starts == [k for k in range(n_ev - 1) if k not in between]


@pytest.mark.parametrize("n_layers,dom", [(1, 2), (1, 8), (2, 5), (36, 5), (36, 7), (36, 8)])
def test_dominant_marks_time_only_the_dominant_stage(n_layers, dom):
    """A timed step given only the dominant stage's events reads back that stage's
    time exactly as a fully marked step does, and no other stage."""
    import bench
    n_stage = 9
    n_ev = 8 * n_layers + 2 if n_layers > 1 else n_stage + 1
    rng = np.random.default_rng(n_layers * 10 + dom)
    t = np.concatenate([[0.0], np.cumsum(rng.uniform(0.1, 2.0, n_ev - 1))])
    full = [[_Ev(x) for x in t]]
    keep = bench.dominant_marks(n_layers, n_stage, dom)
    assert len(keep) == 2 * (n_layers if (n_layers > 1 and dom < 7) else 1)
    sparse = [[_Ev(x) if k in keep else None for k, x in enumerate(t)]]
    all_ms = bench.stage_times([full], n_layers, n_stage, 1)
    dom_ms = bench.stage_times([sparse], n_layers, n_stage, 1)
    assert dom_ms[dom] == pytest.approx(all_ms[dom])
    for j in range(n_stage):
        if j != dom:
            assert dom_ms[j] == 0.0
    # the fully marked stages add up to the whole call less the time between layers
    between = sum(t[8 * lyr + 8] - t[8 * lyr + 7] for lyr in range(n_layers - 1)) if n_layers > 1 else 0.0
    assert all_ms.sum() == pytest.approx(t[-1] - t[0] - between)
