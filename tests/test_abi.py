"""The C-ABI library builds, loads and exports every declared entry point;
host-side argument checks and layout counts work without a GPU."""

import ctypes
import os
import re
import subprocess
import sys

import numpy as np
import pytest

import synth
from oracle import layout as olayout

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "cosmot.h")


def _declared():
    src = open(HEADER).read()
    return sorted(set(re.findall(r"COSMOT_API\s+[\w\s\*]+?\b(cosmot_\w+)\s*\(", src)))


def test_header_declares_the_hot_path_entry_points():
    names = _declared()
    for n in ("cosmot_routed_linear", "cosmot_mrope_apply", "cosmot_mot_attention", "cosmot_flow_euler_step",
              "cosmot_layer_forward", "cosmot_build_layout", "cosmot_get_device_status"):
        assert n in names


@pytest.mark.parametrize("debug", [False, True])
def test_library_exports_every_declared_symbol(debug):
    """Both builds (release, and the debug build with device-side store
    checks) export every entry the header declares."""
    from flow_matching_dit_cosmot_b200 import _lib as L
    lib = L.lib_debug() if debug else L.lib()
    path = L.LIB_DEBUG_PATH if debug else L.LIB_PATH
    out = subprocess.run(["nm", "-D", "--defined-only", path], capture_output=True, text=True, check=True).stdout
    exported = set(re.findall(r"\sT\s(cosmot_\w+)", out))
    missing = [n for n in _declared() if n not in exported]
    assert not missing, missing
    assert set(_declared()) == set(L.SIGNATURES), "binding and header disagree"
    assert lib.cosmot_debug_checks() == (1 if debug else 0)
    if not debug:  # host-only: the release build has no store checks to exercise
        assert lib.cosmot_selftest_bounds_check(None) == L.COSMOT_ERR_UNSUPPORTED


def test_status_strings_and_version():
    from flow_matching_dit_cosmot_b200 import _lib as L
    assert L.status_string(0) == "COSMOT_OK"
    assert L.status_string(4) == "COSMOT_ERR_TIMEOUT"
    assert L.status_string(6) == "COSMOT_ERR_BOUNDS"
    assert L.status_string(99) == "COSMOT_ERR_UNKNOWN"
    assert L.cosmot_version() >= 100


@pytest.mark.parametrize("name", sorted(synth.PRESETS))
def test_layout_counts_match_oracle(name):
    from flow_matching_dit_cosmot_b200 import api as A
    from gpu_helpers import layout_spec
    wl = synth.preset(name)
    lay = olayout.build_layout(wl.layout)
    n, a, c, z = A.L.cosmot_layout_counts(layout_spec(A, wl.layout))
    assert (n, a, c, z) == (lay.n_tokens, lay.n_ar, lay.n_clean, lay.n_noisy)


def test_invalid_arguments_are_rejected_before_any_launch():
    from flow_matching_dit_cosmot_b200 import _lib as L
    lib = L.lib()
    seg = (L.Segment * 1)(L.Segment(0, 10, 0, 0, 0))
    epi = L.Epilogue(kind=0)
    # null input
    assert lib.cosmot_routed_linear(None, 64, 64, seg, 1, 16, 16, None, None, 64, 16, 64, ctypes.byref(epi),
                                    None) == L.COSMOT_ERR_INVALID_ARG
    # k not a multiple of 8
    assert lib.cosmot_routed_linear(16, 64, 60, seg, 1, 16, 16, None, None, 64, 16, 64, ctypes.byref(epi),
                                    None) == L.COSMOT_ERR_INVALID_ARG
    # misaligned pointer
    assert lib.cosmot_routed_linear(18, 64, 64, seg, 1, 16, 16, None, None, 64, 16, 64, ctypes.byref(epi),
                                    None) == L.COSMOT_ERR_INVALID_ARG
    # bad weight set id
    bad = (L.Segment * 1)(L.Segment(0, 10, 0, 2, 0))
    assert lib.cosmot_routed_linear(16, 64, 64, bad, 1, 16, 16, None, None, 64, 16, 64, ctypes.byref(epi),
                                    None) == L.COSMOT_ERR_INVALID_ARG
    # attention: heads not divisible by kv heads; unsupported head_dim
    d = L.AttnDesc(n_q=4, q_key_offset=0, n_keys=4, n_ar=1, n_heads=3, n_kv_heads=2, head_dim=128, batch=1)
    assert lib.cosmot_mot_attention(ctypes.byref(d), 16, 384, 16, 16, 256, 16, 384, None) == L.COSMOT_ERR_INVALID_ARG
    d = L.AttnDesc(n_q=4, q_key_offset=0, n_keys=4, n_ar=1, n_heads=2, n_kv_heads=2, head_dim=96, batch=1)
    assert lib.cosmot_mot_attention(ctypes.byref(d), 16, 192, 16, 16, 192, 16, 192, None) == L.COSMOT_ERR_UNSUPPORTED
    # queries past the keys
    d = L.AttnDesc(n_q=5, q_key_offset=0, n_keys=4, n_ar=1, n_heads=2, n_kv_heads=2, head_dim=128, batch=1)
    assert lib.cosmot_mot_attention(ctypes.byref(d), 16, 256, 16, 16, 256, 16, 256, None) == L.COSMOT_ERR_INVALID_ARG
    # block-causal without chunk ids
    d = L.AttnDesc(n_q=4, q_key_offset=0, n_keys=4, n_ar=1, n_heads=2, n_kv_heads=2, head_dim=128, batch=1,
                   mask_mode=L.COSMOT_MASK_BLOCK_CAUSAL)
    assert lib.cosmot_mot_attention(ctypes.byref(d), 16, 256, 16, 16, 256, 16, 256, None) == L.COSMOT_ERR_INVALID_ARG
    # euler: odd column count
    assert lib.cosmot_flow_euler_step(16, 8, 16, 8, 0, 4, 7, 1.0, 0.9, None) == L.COSMOT_ERR_INVALID_ARG
    # mrope table: sections do not cover head_dim/2
    sec = (L.c_i32 * 3)(16, 24, 23)
    assert lib.cosmot_mrope_table(16, 4, 128, sec, 1e4, 16, None) == L.COSMOT_ERR_INVALID_ARG


def test_layer_workspace_and_validation():
    from flow_matching_dit_cosmot_b200 import api as A
    wl = synth.preset("t2v480")
    dm = wl.dims
    dims = A.make_dims(dm.d_model, dm.n_heads, dm.n_kv_heads, dm.head_dim, dm.ffn, dm.rope_sections)
    seq = A.L.SeqDesc(258, 0, 18720, 1, 0, 0, 16, 0)
    n = A.L.cosmot_layer_workspace_size(dims, seq)
    rows = 18978
    want = rows * (4096 + 12288 + 4096 + 2 * 4096 + 14336) * 2  # h1 is float32
    assert want <= n <= want + 5 * 256
    # the layer rejects a short workspace and bad dims without launching
    lib = A.L.lib()
    assert lib.cosmot_layer_forward(ctypes.byref(dims), ctypes.byref(A.L.LayerWeights()), ctypes.byref(seq), 256, 256,
                                    1.0, 0.97, 256, 1024, None) == A.L.COSMOT_ERR_WORKSPACE
    bad = A.make_dims(4096, 32, 5, 128, 14336, (16, 24, 24))
    assert lib.cosmot_layer_forward(ctypes.byref(bad), ctypes.byref(A.L.LayerWeights()), ctypes.byref(seq), 256, 256,
                                    1.0, 0.97, 256, n, None) == A.L.COSMOT_ERR_INVALID_ARG


def test_stack_workspace_and_validation():
    """Stack workspace = one layer's working set + a hidden buffer + the AR
    q/k/v rows of every layer; argument errors return before any launch."""
    from flow_matching_dit_cosmot_b200 import api as A
    dm = synth.preset("droid_nano36").dims
    dims = A.make_dims(dm.d_model, dm.n_heads, dm.n_kv_heads, dm.head_dim, dm.ffn, dm.rope_sections)
    seq = A.L.SeqDesc(130, 181, 392, 1, 0, 0, 16, 0)
    one = A.L.cosmot_layer_workspace_size(dims, seq)
    n36 = A.L.cosmot_stack_workspace_size(dims, 36, seq)
    qkv_cols = (32 + 2 * 8) * 128
    per_layer_cache = 130 * qkv_cols * 2
    hidden = 703 * 4096 * 2
    assert one + hidden + 36 * per_layer_cache <= n36 <= one + hidden + 36 * (per_layer_cache + 256) + 256
    lib = A.L.lib()
    arr = (A.L.LayerWeights * 2)()
    args = lambda layers, n, s, h, ho, ws, wsb: (ctypes.byref(dims), layers, n, ctypes.byref(s), h, ho, 1.0, 0.9, ws,
                                                 wsb, None)
    n2 = A.L.cosmot_stack_workspace_size(dims, 2, seq)
    assert lib.cosmot_stack_forward(*args(arr, 2, seq, 256, 256, 256, n2)) == A.L.COSMOT_ERR_INVALID_ARG  # h == h_out
    assert lib.cosmot_stack_forward(*args(arr, 0, seq, 256, 512, 256, n2)) == A.L.COSMOT_ERR_INVALID_ARG
    assert lib.cosmot_stack_forward(*args(arr, 2, seq, 256, 512, 256, n2 - 256)) == A.L.COSMOT_ERR_WORKSPACE
    cached = A.L.SeqDesc(130, 181, 392, 1, 0, 311, 16, 0)  # clean prefix: not step-invariant in a stack
    assert lib.cosmot_stack_forward(*args(arr, 2, cached, 256, 512, 256, n2)) == A.L.COSMOT_ERR_UNSUPPORTED
    with pytest.raises(Exception):
        A.L.cosmot_stack_workspace_size(dims, 0, seq)


def test_shift_schedule_host_function_matches_oracle():
    """cosmot_flow_shift_sigmas is host arithmetic: bit-identical to the
    oracle's schedule; bad arguments rejected."""
    from flow_matching_dit_cosmot_b200 import api as A
    from oracle import layer as olayer
    for n, s in ((1, 1.0), (4, 5.0), (10, 1.0), (30, 5.0), (35, 10.0), (7, 0.5)):
        got = np.array(A.L.cosmot_flow_shift_sigmas(n, s))
        np.testing.assert_array_equal(got, olayer.shift_sigmas(n, s))
    lib = A.L.lib()
    buf = (ctypes.c_double * 8)()
    assert lib.cosmot_flow_shift_sigmas(0, 5.0, buf) == A.L.COSMOT_ERR_INVALID_ARG
    assert lib.cosmot_flow_shift_sigmas(4, 0.0, buf) == A.L.COSMOT_ERR_INVALID_ARG
    assert lib.cosmot_flow_shift_sigmas(4, float("inf"), buf) == A.L.COSMOT_ERR_INVALID_ARG
    assert lib.cosmot_flow_shift_sigmas(4, 5.0, None) == A.L.COSMOT_ERR_INVALID_ARG


def _random_specs():
    from hypothesis import strategies as st
    video = st.one_of(st.none(), st.tuples(st.integers(1, 4), st.integers(1, 8), st.integers(1, 8),
                                            st.sampled_from([10, 15, 24, 30]), st.integers(0, 3), st.integers(0, 3)))
    return st.builds(lambda nt, v, ac, an, rate, xc, xn, hz, pr: synth.LayoutSpec(
        n_text=nt, video=None if v is None else synth.VideoSpec(*v), audio_clean=ac, audio_noisy=an, audio_rate=rate,
        action_clean=xc, action_noisy=xn, action_hz=hz, proprio=pr),
        st.integers(0, 40), video, st.integers(0, 9), st.integers(0, 9), st.sampled_from([25, 50]),
        st.integers(0, 9), st.integers(0, 9), st.sampled_from([10, 15, 20]), st.integers(0, 2))


def test_layout_counts_match_oracle_on_random_layouts():
    """cosmot_layout_counts (host arithmetic) agrees with the oracle's layout
    builder on random layouts: any mix of text, views, clean/noisy steps,
    audio, actions and proprioception."""
    from hypothesis import given, settings
    from flow_matching_dit_cosmot_b200 import api as A
    from gpu_helpers import layout_spec

    @settings(max_examples=150, deadline=None)
    @given(_random_specs())
    def check(spec):
        lay = olayout.build_layout(spec)
        n, a, c, z = A.L.cosmot_layout_counts(layout_spec(A, spec))
        assert (n, a, c, z) == (lay.n_tokens, lay.n_ar, lay.n_clean, lay.n_noisy)

    check()


def _all_model_widths():
    from synth import ModelDims
    from synth import presets
    widths = {p.dims for p in (synth.preset(n) for n in presets.PRESETS)}
    widths |= {presets.NANO, presets.SUPER,
               ModelDims(d_model=512, n_heads=4, n_kv_heads=4, head_dim=128, ffn=1536, rope_sections=(16, 24, 24)),
               ModelDims(d_model=512, n_heads=4, n_kv_heads=2, head_dim=128, ffn=1024, rope_sections=(16, 24, 24)),
               ModelDims(d_model=256, n_heads=4, n_kv_heads=2, head_dim=64, ffn=512, rope_sections=(8, 12, 12)),
               ModelDims(d_model=512, n_heads=8, n_kv_heads=4, head_dim=64, ffn=1024, rope_sections=(8, 12, 12))}
    return widths


def test_api_weight_shapes_match_the_weights_synth_draws():
    """MoTLayer refuses weights whose shapes differ from api.weight_shapes;
    every width the tests, the bench and smoke() use draws exactly those."""
    from flow_matching_dit_cosmot_b200 import api as A
    for d in _all_model_widths():
        cd = A.make_dims(d.d_model, d.n_heads, d.n_kv_heads, d.head_dim, d.ffn, d.rope_sections, d.rope_base, d.eps)
        assert A.weight_shapes(cd) == synth.rng.weight_shapes(d), d


def test_api_refuses_weights_and_states_it_cannot_read_safely():
    import torch
    from flow_matching_dit_cosmot_b200 import api as A
    d = synth.ModelDims(d_model=64, n_heads=4, n_kv_heads=2, head_dim=16, ffn=96, rope_sections=(2, 3, 3))
    cd = A.make_dims(d.d_model, d.n_heads, d.n_kv_heads, d.head_dim, d.ffn, d.rope_sections)

    def weights():
        return {k: torch.from_numpy(v.view(np.int16)).view(torch.bfloat16) for k, v in synth.make_weights(d, 7).items()}

    with pytest.raises(ValueError, match="CUDA tensors only"):  # shapes, dtype and layout pass; the device does not
        A.check_weights(cd, weights())
    w = weights()
    w["G.wo"] = w["G.wo"][:, :-16].contiguous()
    with pytest.raises(ValueError, match="'G.wo' has shape"):
        A.check_weights(cd, w)
    w = weights()
    w["R.wqkv"] = w["R.wqkv"].float()
    with pytest.raises(ValueError, match="contiguous bf16"):
        A.check_weights(cd, w)
    w = weights()
    w["wvel"] = w["wvel"].t()
    with pytest.raises(ValueError, match="strided"):
        A.check_weights(cd, w)
    w = weights()
    del w["gfin"]
    with pytest.raises(ValueError, match="'gfin' missing"):
        A.check_weights(cd, w)
    seq = A.L.SeqDesc(3, 4, 5, 2, 0, 0, 0, 0)  # batch 2 x N 12 rows
    ok = torch.zeros((2, 12, 64), dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="CUDA tensors only"):
        A._check_state(seq, 64, h=ok, h_out=ok.clone())
    with pytest.raises(ValueError, match="fewer than"):
        A._check_state(seq, 64, h=ok[:1].clone())


def test_ctypes_structs_and_constants_match_the_header(tmp_path):
    """gcc compiles the header and prints every struct's size and field
    offsets and every constant; the ctypes binding must agree on all of them."""
    import shutil
    from flow_matching_dit_cosmot_b200 import _lib as L
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    structs = {"cosmot_layout_spec": L.LayoutSpec, "cosmot_segment": L.Segment, "cosmot_epilogue": L.Epilogue,
               "cosmot_attn_desc": L.AttnDesc, "cosmot_dims": L.Dims, "cosmot_set_weights": L.SetWeights,
               "cosmot_layer_weights": L.LayerWeights, "cosmot_seq_desc": L.SeqDesc,
               "cosmot_action_desc": L.ActionDesc, "cosmot_step_io": L.StepIO}
    consts = [n for n in dir(L) if re.fullmatch(r"COSMOT_[A-Z_]+", n)]
    lines = ["#include <stdio.h>", "#include <stddef.h>", '#include "cosmot.h"', "int main(void) {"]
    for cname, cls in structs.items():
        lines.append(f'  printf("{cname} %zu\\n", sizeof({cname}));')
        for f, _ in cls._fields_:
            lines.append(f'  printf("{cname}.{f} %zu\\n", offsetof({cname}, {f}));')
    for n in consts:
        lines.append(f'  printf("{n} %lld\\n", (long long)({n}));')
    lines += ["  return 0;", "}"]
    src = tmp_path / "layout.c"
    src.write_text("\n".join(lines) + "\n")
    exe = tmp_path / "layout"
    include = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include")
    subprocess.run([cc, "-std=c11", "-I", include, str(src), "-o", str(exe)], check=True, capture_output=True)
    got = dict(line.rsplit(" ", 1) for line in subprocess.run([str(exe)], capture_output=True, text=True,
                                                               check=True).stdout.splitlines())
    for cname, cls in structs.items():
        assert int(got[cname]) == ctypes.sizeof(cls), cname
        for f, _ in cls._fields_:
            assert int(got[f"{cname}.{f}"]) == getattr(cls, f).offset, f"{cname}.{f}"
    for n in consts:
        assert int(got[n]) == getattr(L, n), n


def _c_kind(param: str) -> str:
    """Kind of one C parameter declaration: ptr, i32, i64, size, f32 or f64."""
    p = param.strip()
    if "*" in p or "[" in p or p.startswith("cosmot_stream_t"):
        return "ptr"
    for ctype, kind in (("int32_t", "i32"), ("int64_t", "i64"), ("size_t", "size"), ("double", "f64"),
                        ("float", "f32"), ("cosmot_status", "i32")):
        if p.startswith(ctype) or p.startswith("const " + ctype):
            return kind
    raise AssertionError(f"unclassified parameter {p!r}")


def _py_kind(t) -> str:
    if t in (ctypes.c_void_p, ctypes.c_char_p) or (isinstance(t, type) and issubclass(t, ctypes._Pointer)):
        return "ptr"
    return {ctypes.c_int32: "i32", ctypes.c_int64: "i64", ctypes.c_size_t: "size", ctypes.c_double: "f64",
            ctypes.c_float: "f32"}[t]


def test_binding_signatures_match_the_header_prototypes():
    """Every entry the binding declares has the header's argument count and,
    argument by argument, the same kind (pointer, 32/64-bit integer, size_t,
    float, double), so ctypes marshals each value the way the C side reads it."""
    from flow_matching_dit_cosmot_b200 import _lib as L
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    header = open(os.path.join(root, "include", "cosmot.h")).read()
    header = re.sub(r"/\*.*?\*/", "", header, flags=re.S)
    protos = {m.group(2): m.group(3) for m in
              re.finditer(r"COSMOT_API\s+([\w\s\*]+?)\s*\b(cosmot_\w+)\s*\(([^)]*)\)\s*;", header)}
    assert set(L.SIGNATURES) == set(protos), set(L.SIGNATURES) ^ set(protos)  # one binding per entry
    for name, (_, argtypes) in L.SIGNATURES.items():
        params = [x for x in protos[name].split(",") if x.strip() and x.strip() != "void"]
        assert len(params) == len(argtypes), name
        for i, (cp, pt) in enumerate(zip(params, argtypes)):
            assert _c_kind(cp) == _py_kind(pt), f"{name} argument {i}: {cp.strip()!r} vs {pt}"


def test_product_never_reaches_the_oracle_and_has_no_fallback():
    """The package and the CUDA sources neither import nor name the oracle, and
    the binding raises when libcosmot.so is absent instead of computing on the
    CPU."""
    import ast
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    pkg = os.path.join(root, "flow_matching_dit_cosmot_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            path = os.path.join(dirpath, f)
            if f.endswith(".py"):
                tree = ast.parse(open(path).read())
                for node in ast.walk(tree):
                    names = []
                    if isinstance(node, ast.Import):
                        names = [a.name for a in node.names]
                    elif isinstance(node, ast.ImportFrom):
                        names = [node.module or ""]
                    assert not any(n == "oracle" or n.startswith("oracle.") for n in names), (path, names)
            elif f.endswith((".cu", ".cuh", ".h")):
                assert "oracle" not in open(path).read(), path
    code = ("import sys; sys.path.insert(0, %r); from flow_matching_dit_cosmot_b200 import _lib as L; "
            "L.LIB_PATH = L.LIB_PATH + '.absent'; L._lib = None\n"
            "try:\n    L.lib()\nexcept ImportError:\n    print('refused')\n" % root)
    out = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True)
    assert out.stdout.strip() == "refused", out.stdout + out.stderr


def test_readme_c_example_compiles_against_the_header(tmp_path):
    """The C usage example in README.md stays in step with include/cosmot.h."""
    import shutil
    cc = shutil.which("gcc") or shutil.which("cc")
    cuda_inc = "/usr/local/cuda/include"
    if cc is None or not os.path.exists(os.path.join(cuda_inc, "cuda_runtime.h")):
        pytest.skip("no C compiler or CUDA headers")
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    text = open(os.path.join(root, "README.md"), encoding="utf-8").read()
    blocks = re.findall(r"```c\n(.*?)```", text, flags=re.S)
    assert blocks, "README has no C example"
    src = tmp_path / "example.c"
    src.write_text(blocks[0])
    r = subprocess.run([cc, "-std=c11", "-fsyntax-only", "-Wall", "-Werror", "-I", os.path.join(root, "include"),
                        "-I", cuda_inc, str(src)], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr


def test_attention_key_split_choice_and_workspace():
    """Host-only: the key split the layer takes for a call shape (148 SMs
    assumed without a device) and the workspace it needs.  A streaming step
    (1,560 query rows, 32 heads, 14,106 keys: 224 work items, 1.5 waves)
    splits 3 ways; the 480p layer (2,368 items, exactly 16 waves) does not;
    block-causal calls that may skip key tiles never split."""
    from flow_matching_dit_cosmot_b200 import _lib as L

    def desc(n_q, n_keys, n_ar, heads=32, batch=1, mode=0, flags=L.COSMOT_ATTN_NO_TILE_SKIP):
        return L.AttnDesc(n_q=n_q, q_key_offset=n_keys - n_q, n_keys=n_keys, n_ar=n_ar, n_heads=heads,
                          n_kv_heads=heads, head_dim=128, mask_mode=mode, batch=batch, flags=flags)

    stream = desc(1560, 66 + 9 * 1560, 66)
    assert L.cosmot_attention_kv_split(stream) == 3
    assert L.cosmot_attention_kv_split(desc(18720, 18978, 258)) == 1
    assert L.cosmot_attention_kv_split(desc(1560, 66 + 9 * 1560, 66, mode=L.COSMOT_MASK_BLOCK_CAUSAL, flags=0)) == 1
    assert L.cosmot_attention_kv_split(desc(392, 703, 130)) == 1  # 6 key tiles: too few to split
    n = L.cosmot_attention_split_workspace(stream, 3)
    assert n >= 3 * 1560 * 32 * 128 * 4 + 3 * 1560 * 32 * 8
    assert L.cosmot_attention_split_workspace(stream, 1) == 0


def test_streaming_workspace_holds_the_key_split_partials():
    """The layer workspace of a streaming layout reserves the key split's
    float32 partials (the split runs when a step's queries are the block's
    noisy rows); the 480p layout reserves none."""
    from flow_matching_dit_cosmot_b200 import api as A
    dm = synth.preset("stream").dims
    dims = A.make_dims(dm.d_model, dm.n_heads, dm.n_kv_heads, dm.head_dim, dm.ffn, dm.rope_sections)
    n_ar, hist, T = 66, 8 * 1560, 1560
    base = A.L.SeqDesc(n_ar, hist, T, 1, 1, 0, 16, 16)
    rows = n_ar + hist + T
    layer_only = rows * (4096 + 12288 + 4096 + 2 * 4096 + 14336) * 2
    got = A.L.cosmot_layer_workspace_size(dims, base)
    assert got >= layer_only + 3 * T * 4096 * 4
    t2v = A.L.SeqDesc(258, 0, 18720, 1, 0, 0, 16, 0)
    assert A.L.cosmot_layer_workspace_size(dims, t2v) <= 18978 * (4096 + 12288 + 4096 + 2 * 4096 + 14336) * 2 + 6 * 256
