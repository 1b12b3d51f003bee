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
