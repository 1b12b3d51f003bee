"""Per-kernel parity of the CUDA path against the fp64 oracle (needs a B200).

Inputs come from the seeded generators in ``synth``; expected values from
``oracle``.  Sizes span several tiles with ragged tails; index and layout work
is compared bit for bit.
"""

import numpy as np
import pytest

import synth
from oracle import layer as olayer
from oracle import layout as olayout
from oracle import mask as omask
from oracle import rope as orope
from tolerance import SIGMA_ATTN, assert_close, rms

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():  # pragma: no cover
    pytest.skip("no CUDA device", allow_module_level=True)

from flow_matching_dit_cosmot_b200 import api as A  # noqa: E402
from flow_matching_dit_cosmot_b200 import _lib as L  # noqa: E402
from gpu_helpers import Guarded, assert_device_ok, bits, layout_spec, to_dev, to_f64  # noqa: E402
from synth import LayoutSpec, VideoSpec  # noqa: E402


def _bf16(shape, seed, std=1.0):
    return synth.normal_bf16(shape, seed, 1, std=std)


# ---------------------------------------------------------------- layout (bit-exact)

_EXTRA_SPECS = [
    LayoutSpec(n_text=5, video=VideoSpec(2, 3, 4, 15, 1, 2), audio_clean=3, audio_noisy=7, action_clean=2,
               action_noisy=9, action_hz=15, proprio=1),
    LayoutSpec(n_text=0, video=VideoSpec(1, 2, 2, 30, 0, 3), audio_noisy=11),
    LayoutSpec(n_text=7, video=None, audio_noisy=4, action_noisy=3),
    LayoutSpec(n_text=3, video=VideoSpec(3, 5, 7, 10, 2, 1), action_noisy=6, action_hz=20, proprio=2),
]


@pytest.mark.parametrize("case", sorted(synth.PRESETS) + [f"extra{i}" for i in range(len(_EXTRA_SPECS))])
@pytest.mark.parametrize("tau_offset", [0, 9])
def test_build_layout_bit_exact(case, tau_offset):
    spec = synth.preset(case).layout if case in synth.PRESETS else _EXTRA_SPECS[int(case[5:])]
    ref = olayout.build_layout(spec, tau_offset=tau_offset)
    dev = A.build_layout(layout_spec(A, spec, tau_offset))
    torch.cuda.synchronize()
    assert (dev.n_ar, dev.n_clean, dev.n_noisy) == (ref.n_ar, ref.n_clean, ref.n_noisy)
    np.testing.assert_array_equal(dev.pos.cpu().numpy().view(np.uint32), ref.pos.view(np.uint32))
    np.testing.assert_array_equal(dev.chunk.cpu().numpy(), ref.chunk)
    np.testing.assert_array_equal(dev.region.cpu().numpy(), ref.region)
    assert_device_ok()


def test_build_layout_bit_exact_on_random_layouts():
    """Positions, chunk ids and regions from the GPU equal the oracle's bit for
    bit on random layouts (text, views, clean/noisy steps, audio, actions,
    proprioception, time offsets)."""
    from hypothesis import given, settings
    from hypothesis import strategies as st
    from test_abi import _random_specs

    @settings(max_examples=60, deadline=None)
    @given(_random_specs(), st.integers(0, 12))
    def check(spec, tau):
        ref = olayout.build_layout(spec, tau_offset=tau)
        dev = A.build_layout(layout_spec(A, spec, tau))
        torch.cuda.synchronize()
        assert (dev.n_ar, dev.n_clean, dev.n_noisy) == (ref.n_ar, ref.n_clean, ref.n_noisy)
        np.testing.assert_array_equal(dev.pos.cpu().numpy().view(np.uint32), ref.pos.view(np.uint32))
        np.testing.assert_array_equal(dev.chunk.cpu().numpy(), ref.chunk)
        np.testing.assert_array_equal(dev.region.cpu().numpy(), ref.region)

    check()
    assert_device_ok()


@pytest.mark.parametrize("hd,sections", [(128, (16, 24, 24)), (64, (8, 12, 12))])
def test_mrope_table(hd, sections):
    ref = olayout.build_layout(synth.preset("i2v720").layout)
    pos = torch.from_numpy(ref.pos).cuda()
    cs = A.mrope_table(pos, hd, sections).cpu().numpy().astype(np.float64)
    th = orope.angles(ref.pos, hd, sections, 10000.0)
    np.testing.assert_allclose(cs[..., 0], np.cos(th), atol=2e-7, rtol=0)
    np.testing.assert_allclose(cs[..., 1], np.sin(th), atol=2e-7, rtol=0)


# ---------------------------------------------------------------- RMSNorm

@pytest.mark.parametrize("d", [256, 4096, 5120])
def test_rmsnorm_routed(d):
    rows = 300
    h = _bf16((rows, d), 3)
    g0 = synth.normal_bf16((d,), 4, 1, std=0.02, mean=1.0)
    g1 = synth.normal_bf16((d,), 5, 1, std=0.02, mean=1.0)
    hd_, g0d, g1d = to_dev(h), to_dev(g0), to_dev(g1)
    og = Guarded(torch.zeros((rows + 7, d), dtype=torch.bfloat16, device="cuda"))
    out = og.t
    segs = [(0, 37, 7, 0), (37, 300, 44, 1)]  # output rows shifted by 7
    L.cosmot_rmsnorm_routed(A.ptr(hd_), d, segs, A.ptr(g0d), A.ptr(g1d), d, 1e-6, A.ptr(out), d,
                            A.stream_handle())
    got = to_f64(out)[7:]
    h64 = synth.bf16_to_f64(h)
    ref = np.concatenate([olayer.rms_norm(h64[:37], synth.bf16_to_f64(g0), 1e-6),
                          olayer.rms_norm(h64[37:], synth.bf16_to_f64(g1), 1e-6)])
    assert_close(got, ref, "rmsnorm")
    assert np.all(bits(out)[:7] == 0)
    og.assert_canaries("rmsnorm output")


# ---------------------------------------------------------------- routed GEMM

def _gemm_case(m_split, m_total, k, n_out, seed=0):
    a = _bf16((m_total, k), 10 + seed)
    w0 = _bf16((n_out, k), 11 + seed, std=1.0 / np.sqrt(k))
    w1 = _bf16((n_out, k), 12 + seed, std=1.0 / np.sqrt(k))
    segs = [(0, m_split, 0, 0), (m_split, m_total, m_split, 1)]
    a64, w064, w164 = (synth.bf16_to_f64(x) for x in (a, w0, w1))
    acc = np.concatenate([a64[:m_split] @ w064.T, a64[m_split:] @ w164.T])
    return a, w0, w1, segs, acc


@pytest.mark.parametrize("m_split,m_total,k,n_out", [(200, 533, 320, 384), (130, 703, 200, 264), (1, 129, 64, 8),
                                                     (258, 1000, 4096, 512)])
def test_routed_linear_plain(m_split, m_total, k, n_out):
    a, w0, w1, segs, acc = _gemm_case(m_split, m_total, k, n_out)
    og = Guarded(torch.empty((m_total, n_out), dtype=torch.bfloat16, device="cuda"))
    out = og.t
    ad, w0d, w1d = to_dev(a), to_dev(w0), to_dev(w1)
    L.cosmot_routed_linear(A.ptr(ad), k, k, segs, A.ptr(w0d), A.ptr(w1d), n_out, A.ptr(out), n_out,
                           stream=A.stream_handle())
    assert_close(to_f64(out), acc, "gemm")
    assert_device_ok()
    og.assert_canaries("gemm output")


def test_routed_linear_pair_and_single_tiles_agree_bit_for_bit():
    """Most calls run 256-row tiles on a pair of CTAs (tcgen05.mma.cta_group::2);
    a call whose pairs would need clearly more rounds over the SMs runs
    128-row tiles on single CTAs.  On 148 SMs, 4736 rows x 1024 columns are
    148 single tiles (one round) but 76 pair tiles (two rounds over 74
    pairs): single CTAs; the same rows x 256 columns fit in one round either
    way: pairs.  Every element is the same K-ordered fp32 sum in both, so the
    shared columns agree to the bit, and both meet the reference."""
    m_total, k = 4736, 256
    a, w0, w1, segs, acc = _gemm_case(300, m_total, k, 1024, seed=7)
    ad, w0d, w1d = to_dev(a), to_dev(w0), to_dev(w1)
    wide = torch.empty((m_total, 1024), dtype=torch.bfloat16, device="cuda")
    narrow = torch.empty((m_total, 256), dtype=torch.bfloat16, device="cuda")
    L.cosmot_routed_linear(A.ptr(ad), k, k, segs, A.ptr(w0d), A.ptr(w1d), 1024, A.ptr(wide), 1024,
                           stream=A.stream_handle())
    L.cosmot_routed_linear(A.ptr(ad), k, k, segs, A.ptr(w0d), A.ptr(w1d), 256, A.ptr(narrow), 256,
                           stream=A.stream_handle())
    torch.cuda.synchronize()
    assert_device_ok()
    assert_close(to_f64(wide), acc, "gemm, single-CTA tiles")
    assert_close(to_f64(narrow), acc[:, :256], "gemm, pair tiles")
    np.testing.assert_array_equal(bits(narrow), bits(wide[:, :256]))


def test_routed_linear_224_wide_pair_tiles():
    """A few thousand rows against a 4096-wide output (a streaming step's O,
    down and velocity projections) run 256 x 224 pair tiles: 1,560 rows are
    7 pair row tiles, and 19 column tiles of 224 fill the second of two
    rounds over 74 pairs better than 16 of 256.  Residual epilogue with a
    float32 output, two segments, against the reference."""
    m_total, k, n_out = 1560, 256, 4096
    a, w0, w1, segs, acc = _gemm_case(60, m_total, k, n_out, seed=8)
    rng = np.random.default_rng(23)
    res = rng.standard_normal((m_total, n_out)).astype(np.float32)
    out = torch.full((m_total, n_out), float("nan"), dtype=torch.float32, device="cuda")
    ad, w0d, w1d, rd = to_dev(a), to_dev(w0), to_dev(w1), torch.from_numpy(res).cuda()
    e = L.Epilogue(kind=L.COSMOT_EPI_RESIDUAL, res=A.ptr(rd), ld_res=n_out,
                   flags=L.COSMOT_EPI_OUT_F32 | L.COSMOT_EPI_RES_F32)
    L.cosmot_routed_linear(A.ptr(ad), k, k, segs, A.ptr(w0d), A.ptr(w1d), n_out, A.ptr(out), n_out, e,
                           stream=A.stream_handle())
    torch.cuda.synchronize()
    assert_device_ok()
    got = out.double().cpu().numpy()
    # fp32 accumulation and one fp32 add: far inside the bf16 bounds
    assert np.abs(got - (acc + res.astype(np.float64))).max() < 1e-4


def test_routed_linear_equal_sets_equal_single_segment():
    """With both weight sets holding the same matrix (in separate buffers) the
    routed projection is bit-identical to one segment over all rows: routing
    changes which weights a row meets, never how a row is computed."""
    a, w0, _, segs, _ = _gemm_case(203, 700, 512, 264, seed=5)
    ad, w0d, w1d = to_dev(a), to_dev(w0), to_dev(w0.copy())
    routed = torch.empty((700, 264), dtype=torch.bfloat16, device="cuda")
    single = torch.empty_like(routed)
    L.cosmot_routed_linear(A.ptr(ad), 512, 512, segs, A.ptr(w0d), A.ptr(w1d), 264, A.ptr(routed), 264,
                           stream=A.stream_handle())
    L.cosmot_routed_linear(A.ptr(ad), 512, 512, [(0, 700, 0, 0)], A.ptr(w0d), A.ptr(w1d), 264, A.ptr(single), 264,
                           stream=A.stream_handle())
    torch.cuda.synchronize()
    assert_device_ok()
    np.testing.assert_array_equal(bits(routed), bits(single))


def test_routed_linear_residual():
    m_split, m_total, k, n_out = 77, 400, 512, 264
    a, w0, w1, segs, acc = _gemm_case(m_split, m_total, k, n_out, seed=1)
    res = _bf16((m_total, n_out), 20)
    out = torch.empty((m_total, n_out), dtype=torch.bfloat16, device="cuda")
    ad, w0d, w1d, rd = to_dev(a), to_dev(w0), to_dev(w1), to_dev(res)
    e = L.Epilogue(kind=L.COSMOT_EPI_RESIDUAL, res=A.ptr(rd), ld_res=n_out)
    L.cosmot_routed_linear(A.ptr(ad), k, k, segs, A.ptr(w0d), A.ptr(w1d), n_out, A.ptr(out), n_out, e,
                           stream=A.stream_handle())
    assert_close(to_f64(out), acc + synth.bf16_to_f64(res), "gemm+residual")


@pytest.mark.parametrize("flags", ["out_f32", "res_f32", "both"])
def test_routed_linear_residual_float32(flags):
    """The residual epilogue with a float32 output (the layer's h1) and/or a
    float32 residual (h1 read back by the down projection): fp32 values are
    stored and read without rounding."""
    m_split, m_total, k, n_out = 77, 400, 512, 264
    a, w0, w1, segs, acc = _gemm_case(m_split, m_total, k, n_out, seed=2)
    fl = {"out_f32": L.COSMOT_EPI_OUT_F32, "res_f32": L.COSMOT_EPI_RES_F32,
          "both": L.COSMOT_EPI_OUT_F32 | L.COSMOT_EPI_RES_F32}[flags]
    rng = np.random.default_rng(21)
    res32 = rng.standard_normal((m_total, n_out)).astype(np.float32)  # values a bf16 cannot hold
    res16 = _bf16((m_total, n_out), 22)
    use_f32_res = bool(fl & L.COSMOT_EPI_RES_F32)
    rd = torch.from_numpy(res32).cuda() if use_f32_res else to_dev(res16)
    out = torch.empty((m_total, n_out), dtype=torch.float32 if fl & L.COSMOT_EPI_OUT_F32 else torch.bfloat16,
                      device="cuda")
    ad, w0d, w1d = to_dev(a), to_dev(w0), to_dev(w1)
    e = L.Epilogue(kind=L.COSMOT_EPI_RESIDUAL, res=A.ptr(rd), ld_res=n_out, flags=fl)
    L.cosmot_routed_linear(A.ptr(ad), k, k, segs, A.ptr(w0d), A.ptr(w1d), n_out, A.ptr(out), n_out, e,
                           stream=A.stream_handle())
    torch.cuda.synchronize()
    assert_device_ok()
    ref = acc + (res32.astype(np.float64) if use_f32_res else synth.bf16_to_f64(res16))
    got = out.double().cpu().numpy()
    if fl & L.COSMOT_EPI_OUT_F32:  # fp32 accumulation and one fp32 add: far inside the bf16 bounds
        assert np.abs(got - ref).max() < 1e-4, np.abs(got - ref).max()
    else:
        assert_close(got, ref, "gemm+float32 residual")


def test_routed_linear_rejects_float32_flags_off_the_residual_epilogue():
    a = torch.zeros((16, 64), dtype=torch.bfloat16, device="cuda")
    e = L.Epilogue(kind=L.COSMOT_EPI_NONE, flags=L.COSMOT_EPI_OUT_F32)
    code = L.cosmot_routed_linear(A.ptr(a), 64, 64, [(0, 16, 0, 0)], A.ptr(a), A.ptr(a), 16, A.ptr(a), 64, e,
                                  stream=A.stream_handle(), check=False)
    assert code == L.COSMOT_ERR_INVALID_ARG
    e = L.Epilogue(kind=L.COSMOT_EPI_RESIDUAL, res=A.ptr(a), ld_res=64, flags=4)
    code = L.cosmot_routed_linear(A.ptr(a), 64, 64, [(0, 16, 0, 0)], A.ptr(a), A.ptr(a), 16, A.ptr(a), 64, e,
                                  stream=A.stream_handle(), check=False)
    assert code == L.COSMOT_ERR_INVALID_ARG


def test_routed_linear_silu_mul():
    m_split, m_total, k, f = 150, 450, 256, 384
    a = _bf16((m_total, k), 30)
    wg = [_bf16((f, k), 31 + s, std=0.1) for s in range(2)]
    wu = [_bf16((f, k), 33 + s, std=0.1) for s in range(2)]
    segs = [(0, m_split, 0, 0), (m_split, m_total, m_split, 1)]
    out = torch.empty((m_total, f), dtype=torch.bfloat16, device="cuda")
    dv = [to_dev(x) for x in (a, wg[0], wg[1], wu[0], wu[1])]
    e = L.Epilogue(kind=L.COSMOT_EPI_SILU_MUL)
    L.cosmot_routed_linear(A.ptr(dv[0]), k, k, segs, A.ptr(dv[1]), A.ptr(dv[2]), f, A.ptr(out), f, e,
                           w0_up=A.ptr(dv[3]), w1_up=A.ptr(dv[4]), stream=A.stream_handle())
    a64 = synth.bf16_to_f64(a)
    ref = []
    for s, (b, e_) in enumerate([(0, m_split), (m_split, m_total)]):
        x = a64[b:e_]
        ref.append(olayer.silu(x @ synth.bf16_to_f64(wg[s]).T) * (x @ synth.bf16_to_f64(wu[s]).T))
    assert_close(to_f64(out), np.concatenate(ref), "gemm+silu")


@pytest.mark.parametrize("hd,n_heads,n_kv", [(128, 4, 2), (64, 4, 4)])
def test_routed_linear_mrope(hd, n_heads, n_kv):
    spec = LayoutSpec(n_text=60, video=VideoSpec(2, 5, 7, 24, 1, 3))
    lay = olayout.build_layout(spec)
    n = lay.n_tokens
    sections = (hd // 8, 3 * hd // 16, 3 * hd // 16)
    k = 256
    n_out = (n_heads + 2 * n_kv) * hd
    a = _bf16((2 * n, k), 40)  # two sequences back to back; the table wraps every n rows
    w = [_bf16((n_out, k), 41 + s, std=0.06) for s in range(2)]
    segs = [(0, lay.n_ar, 0, 0), (lay.n_ar, n, lay.n_ar, 1), (n, n + lay.n_ar, n, 0), (n + lay.n_ar, 2 * n, n + lay.n_ar, 1)]
    pos = torch.from_numpy(lay.pos).cuda()
    cs = A.mrope_table(pos, hd, sections)
    out = torch.empty((2 * n, n_out), dtype=torch.bfloat16, device="cuda")
    dv = [to_dev(x) for x in (a, w[0], w[1])]
    rope_cols = (n_heads + n_kv) * hd
    e = L.Epilogue(kind=L.COSMOT_EPI_MROPE, head_dim=hd, rope_cols=rope_cols, rope_cs=A.ptr(cs), rope_period=n)
    L.cosmot_routed_linear(A.ptr(dv[0]), k, k, segs, A.ptr(dv[1]), A.ptr(dv[2]), n_out, A.ptr(out), n_out, e,
                           stream=A.stream_handle())
    a64 = synth.bf16_to_f64(a)
    ref = np.empty((2 * n, n_out))
    for (b, e_, _, s) in segs:
        ref[b:e_] = a64[b:e_] @ synth.bf16_to_f64(w[s]).T
    pos2 = np.concatenate([lay.pos, lay.pos])
    heads = ref[:, :rope_cols].reshape(2 * n, n_heads + n_kv, hd)
    ref[:, :rope_cols] = orope.apply(heads, pos2, hd, sections, 10000.0).reshape(2 * n, rope_cols)
    assert_close(to_f64(out), ref, "gemm+mrope")


def test_routed_linear_euler_in_place():
    n_rows, k, c = 300, 256, 256
    xrows = 500
    a = _bf16((n_rows, k), 50)
    w = _bf16((c, k), 51, std=0.06)
    x = _bf16((xrows, c), 52)
    xd = to_dev(x)
    ad, wd = to_dev(a), to_dev(w)
    # velocity rows 0..299 update x rows 150..449 in place; everything else untouched
    segs = [(0, n_rows, 150, 1)]
    ds = np.float32(0.7 - 0.8)
    e = L.Epilogue(kind=L.COSMOT_EPI_EULER, x=A.ptr(xd), ld_x=c, dsigma=float(ds))
    L.cosmot_routed_linear(A.ptr(ad), k, k, segs, A.ptr(wd), A.ptr(wd), c, A.ptr(xd), c, e, stream=A.stream_handle())
    got = to_f64(xd)
    v = synth.bf16_to_f64(a) @ synth.bf16_to_f64(w).T
    ref = olayer.euler_step(synth.bf16_to_f64(x)[150:450], v, 0.8, 0.7)
    assert_close(got[150:450], ref, "gemm+euler")
    np.testing.assert_array_equal(bits(xd)[:150], x[:150])
    np.testing.assert_array_equal(bits(xd)[450:], x[450:])


def test_routed_linear_euler_float32_state_and_velocity():
    """The Euler epilogue with a float32 state (indexed by input row) and the
    velocity written out: the first call reads x from the bf16 rows
    (state_from_x), the second from the float32 state it left; both write the
    bf16 copy into the output rows."""
    n_rows, k, c, xrows = 300, 256, 256, 500
    a = _bf16((n_rows, k), 53)
    w = _bf16((c, k), 54, std=0.06)
    x = _bf16((xrows, c), 55)
    xd, ad, wd = to_dev(x), to_dev(a), to_dev(w)
    x32 = torch.full((n_rows, c), float("nan"), dtype=torch.float32, device="cuda")
    vel = torch.full((n_rows, c), float("nan"), dtype=torch.bfloat16, device="cuda")
    segs = [(0, n_rows, 150, 1)]
    v = synth.bf16_to_f64(a) @ synth.bf16_to_f64(w).T
    ref = synth.bf16_to_f64(x)[150:450]
    for step, (s0, s1) in enumerate(((0.8, 0.7), (0.7, 0.55))):
        e = L.Epilogue(kind=L.COSMOT_EPI_EULER, x=A.ptr(xd), ld_x=c, dsigma=float(np.float32(s1 - s0)),
                       x_state=A.ptr(x32), ld_state=c, vel=A.ptr(vel), ld_vel=c, state_from_x=1 if step == 0 else 0)
        L.cosmot_routed_linear(A.ptr(ad), k, k, segs, A.ptr(wd), A.ptr(wd), c, A.ptr(xd), c, e,
                               stream=A.stream_handle())
        torch.cuda.synchronize()
        assert_device_ok()
        ref = olayer.euler_step(ref, v, s0, s1)
        got32 = x32.double().cpu().numpy()
        assert np.abs(got32 - ref).max() < 1e-4, np.abs(got32 - ref).max()  # no bf16 rounding of the state
        np.testing.assert_array_equal(bits(xd)[150:450], bits(x32.to(torch.bfloat16)))
        assert_close(to_f64(vel), v, "velocity output")
    np.testing.assert_array_equal(bits(xd)[:150], x[:150])
    np.testing.assert_array_equal(bits(xd)[450:], x[450:])


# ---------------------------------------------------------------- mRoPE, Euler (standalone)

def test_mrope_apply():
    lay = olayout.build_layout(synth.preset("droid").layout)
    n, hd, nq, nk = lay.n_tokens, 128, 4, 2
    q = _bf16((n, nq * hd + 64), 60)  # padded leading dimension
    k = _bf16((n, nk * hd), 61)
    qd, kd = to_dev(q), to_dev(k)
    cs = A.mrope_table(torch.from_numpy(lay.pos).cuda(), hd, (16, 24, 24))
    L.cosmot_mrope_apply(A.ptr(qd), nq * hd + 64, nq, A.ptr(kd), nk * hd, nk, n, hd, A.ptr(cs), A.stream_handle())
    qr = orope.apply(synth.bf16_to_f64(q)[:, :nq * hd].reshape(n, nq, hd), lay.pos, hd, (16, 24, 24), 1e4)
    kr = orope.apply(synth.bf16_to_f64(k).reshape(n, nk, hd), lay.pos, hd, (16, 24, 24), 1e4)
    assert_close(to_f64(qd)[:, :nq * hd], qr.reshape(n, -1), "mrope q")
    assert_close(to_f64(kd), kr.reshape(n, -1), "mrope k")
    np.testing.assert_array_equal(bits(qd)[:, nq * hd:], q[:, nq * hd:])


def test_flow_euler_step():
    x = _bf16((1000, 264), 70)
    v = _bf16((1000, 264), 71)
    xd, vd = to_dev(x), to_dev(v)
    L.cosmot_flow_euler_step(A.ptr(xd), 264, A.ptr(vd), 264, 100, 731, 264, 0.97, 0.5, A.stream_handle())
    got = to_f64(xd)
    ref = olayer.euler_step(synth.bf16_to_f64(x)[100:731], synth.bf16_to_f64(v)[100:731], 0.97, 0.5)
    assert_close(got[100:731], ref, "euler")
    np.testing.assert_array_equal(bits(xd)[:100], x[:100])
    np.testing.assert_array_equal(bits(xd)[731:], x[731:])


def test_euler_sampler_lands_on_x0():
    """Linear flow path with its analytic velocity: 10 Euler steps land on x0
    within bf16 rounding of the running state."""
    x0 = synth.bf16_to_f64(_bf16((64, 256), 72))
    eps = synth.bf16_to_f64(_bf16((64, 256), 73))
    v = synth.bf16_round((eps - x0).astype(np.float32))
    xd, vd = to_dev(synth.bf16_round(eps.astype(np.float32))), to_dev(v)
    sig = synth.preset("droid").sigmas
    for s0, s1 in zip(sig[:-1], sig[1:]):
        L.cosmot_flow_euler_step(A.ptr(xd), 256, A.ptr(vd), 256, 0, 64, 256, s0, s1, A.stream_handle())
    err = np.abs(to_f64(xd) - x0)
    assert err.max() < 0.1 and np.sqrt(np.mean(err ** 2)) < 0.02


# ---------------------------------------------------------------- attention

def _attn_case(n_keys, n_ar, n_q, q_off, H, Hkv, hd, mode, chunk=None, batch=1, seed=0, kv_split=1):
    rng_seed = 80 + seed
    q = _bf16((batch * n_q, H * hd), rng_seed)
    k = _bf16((batch * n_keys, Hkv * hd), rng_seed + 1)
    v = _bf16((batch * n_keys, Hkv * hd), rng_seed + 2)
    region = np.where(np.arange(n_keys) < n_ar, olayout.REGION_AR, olayout.REGION_NOISY).astype(np.int8)
    ch = chunk if chunk is not None else np.where(np.arange(n_keys) < n_ar, -1, 0).astype(np.int32)
    allow = omask.allow_matrix(q_off + np.arange(n_q), region, ch, mode)
    ref = []
    for b in range(batch):
        qq = synth.bf16_to_f64(q[b * n_q:(b + 1) * n_q]).reshape(n_q, H, hd)
        kk = synth.bf16_to_f64(k[b * n_keys:(b + 1) * n_keys]).reshape(n_keys, Hkv, hd)
        vv = synth.bf16_to_f64(v[b * n_keys:(b + 1) * n_keys]).reshape(n_keys, Hkv, hd)
        ref.append(olayer.attention(qq, kk, vv, allow, 1.0 / np.sqrt(hd)).reshape(n_q, H * hd))
    qd, kd, vd = to_dev(q), to_dev(k), to_dev(v)
    og = Guarded(torch.full((batch * n_q, H * hd), float("nan"), dtype=torch.bfloat16, device="cuda"))
    o = og.t
    chd = torch.from_numpy(ch).cuda()
    d = L.AttnDesc(n_q=n_q, q_key_offset=q_off, n_keys=n_keys, n_ar=n_ar, n_heads=H, n_kv_heads=Hkv, head_dim=hd,
                   mask_mode=L.COSMOT_MASK_FULL if mode == "full" else L.COSMOT_MASK_BLOCK_CAUSAL,
                   chunk=A.ptr(chd), batch=batch, q_batch_stride=n_q, kv_batch_stride=n_keys, o_batch_stride=n_q,
                   flags=L.COSMOT_ATTN_NO_TILE_SKIP if kv_split > 1 else 0)
    if kv_split > 1:
        ws = torch.full((L.cosmot_attention_split_workspace(d, kv_split),), 255, dtype=torch.uint8, device="cuda")
        L.cosmot_mot_attention_split(d, A.ptr(qd), H * hd, A.ptr(kd), A.ptr(vd), Hkv * hd, A.ptr(o), H * hd, kv_split,
                                     A.ptr(ws), ws.numel(), A.stream_handle())
    else:
        L.cosmot_mot_attention(d, A.ptr(qd), H * hd, A.ptr(kd), A.ptr(vd), Hkv * hd, A.ptr(o), H * hd,
                               A.stream_handle())
    got = to_f64(o)
    assert_device_ok()
    og.assert_canaries("attention output")
    return got, np.concatenate(ref)


def test_attention_of_constant_values_is_one():
    """With V = 1 every visible set of softmax weights sums to one, so every
    output is 1 ("Cosmos 3 方法原理全解" §3: attention is a convex combination of
    values).  P is stored in bf16 for the PV product while the row sum is kept
    in fp32, so the output may differ from 1 by the bf16 rounding of P: at most
    2^-9 relative, plus the output's own rounding."""
    n_keys, n_ar, H, hd = 700, 130, 2, 128
    ch = np.full(n_keys, -1, np.int32)
    ch[n_ar:] = np.arange(n_keys - n_ar) // 97
    for mode in ("full", "block_causal"):
        q = _bf16((n_keys, H * hd), 95)
        k = _bf16((n_keys, H * hd), 96)
        ones = torch.ones((n_keys, H * hd), dtype=torch.bfloat16, device="cuda")
        o = torch.full((n_keys, H * hd), float("nan"), dtype=torch.bfloat16, device="cuda")
        qd, kd, chd = to_dev(q), to_dev(k), torch.from_numpy(ch).cuda()
        d = L.AttnDesc(n_q=n_keys, q_key_offset=0, n_keys=n_keys, n_ar=n_ar, n_heads=H, n_kv_heads=H, head_dim=hd,
                       mask_mode=L.COSMOT_MASK_FULL if mode == "full" else L.COSMOT_MASK_BLOCK_CAUSAL,
                       chunk=A.ptr(chd), batch=1)
        L.cosmot_mot_attention(d, A.ptr(qd), H * hd, A.ptr(kd), A.ptr(ones), H * hd, A.ptr(o), H * hd,
                               A.stream_handle())
        torch.cuda.synchronize()
        assert_device_ok()
        assert np.abs(to_f64(o) - 1.0).max() <= 2.0 ** -8, mode


@pytest.mark.parametrize("hd", [128, 64])
def test_attention_full_mask(hd):
    got, ref = _attn_case(n_keys=700, n_ar=130, n_q=700, q_off=0, H=4, Hkv=2, hd=hd, mode="full")
    assert_close(got, ref, f"attention hd{hd}", sigma=SIGMA_ATTN, branch_rms=rms(ref))


def test_attention_causal_ar_only_and_tiny():
    got, ref = _attn_case(n_keys=300, n_ar=300, n_q=300, q_off=0, H=2, Hkv=2, hd=128, mode="full", seed=1)
    assert_close(got, ref, "causal", sigma=SIGMA_ATTN, branch_rms=rms(ref))
    got, ref = _attn_case(n_keys=3, n_ar=2, n_q=3, q_off=0, H=1, Hkv=1, hd=128, mode="full", seed=2)
    assert_close(got, ref, "tiny", sigma=SIGMA_ATTN, branch_rms=rms(ref))


def test_attention_block_causal_and_batch():
    n_keys, n_ar = 600, 66
    ch = np.full(n_keys, -1, np.int32)
    ch[n_ar:] = (np.arange(n_keys - n_ar) // 89)  # chunks not aligned to 128-key tiles
    got, ref = _attn_case(n_keys, n_ar, n_keys, 0, H=4, Hkv=4, hd=128, mode="block_causal", chunk=ch, batch=2, seed=3)
    assert_close(got, ref, "block causal", sigma=SIGMA_ATTN, branch_rms=rms(ref))


def test_attention_block_causal_hd64_gqa():
    """The tile-skipping instance at head_dim 64 with grouped key/value heads:
    chunks of 200 keys, so early DM query tiles skip the later key tiles."""
    n_keys, n_ar = 1100, 50
    ch = np.full(n_keys, -1, np.int32)
    ch[n_ar:] = np.arange(n_keys - n_ar) // 200
    got, ref = _attn_case(n_keys, n_ar, n_keys, 0, H=4, Hkv=2, hd=64, mode="block_causal", chunk=ch, batch=2, seed=5)
    assert_close(got, ref, "block causal hd64", sigma=SIGMA_ATTN, branch_rms=rms(ref))


def test_attention_query_suffix_streaming():
    """Queries are the last block of the key sequence (a streaming step)."""
    n_keys, n_ar = 66 + 3 * 250 + 250, 66
    ch = np.full(n_keys, -1, np.int32)
    ch[n_ar:] = np.arange(n_keys - n_ar) // 250
    got, ref = _attn_case(n_keys, n_ar, 250, n_keys - 250, H=2, Hkv=1, hd=128, mode="block_causal", chunk=ch, seed=4)
    assert_close(got, ref, "stream", sigma=SIGMA_ATTN, branch_rms=rms(ref))


@pytest.mark.parametrize("kv_split", [2, 3])
@pytest.mark.parametrize("case", ["full_with_ar", "suffix_block_causal", "hd64_gqa_batch2"])
def test_attention_key_split(kv_split, case):
    """The keys of every DM query item split across CTAs, the float32 partials
    combined by the merge kernel: against the oracle, and close to the unsplit
    kernel (only the order of the softmax sums differs).  AR query rows are
    never split."""
    if case == "full_with_ar":
        args = dict(n_keys=1100, n_ar=130, n_q=1100, q_off=0, H=4, Hkv=2, hd=128, mode="full")
    elif case == "suffix_block_causal":
        n_keys, n_ar = 66 + 3 * 250 + 250, 66
        ch = np.full(n_keys, -1, np.int32)
        ch[n_ar:] = np.arange(n_keys - n_ar) // 250
        args = dict(n_keys=n_keys, n_ar=n_ar, n_q=250, q_off=n_keys - 250, H=2, Hkv=1, hd=128, mode="block_causal",
                    chunk=ch)
    else:
        args = dict(n_keys=900, n_ar=40, n_q=900, q_off=0, H=4, Hkv=2, hd=64, mode="full", batch=2)
    got, ref = _attn_case(**args, seed=7, kv_split=kv_split)
    assert_close(got, ref, f"attention split {kv_split} {case}", sigma=SIGMA_ATTN, branch_rms=rms(ref))
    plain, _ = _attn_case(**args, seed=7)
    assert np.abs(got - plain).max() <= 2.0 ** -7 * np.abs(plain).max() + 1e-3
    n_ar_q = max(0, min(args["n_q"], args["n_ar"] - args["q_off"]))
    if n_ar_q:  # AR rows take the unsplit path: identical bits
        rows = np.concatenate([np.arange(b * args["n_q"], b * args["n_q"] + n_ar_q) for b in range(args.get("batch", 1))])
        np.testing.assert_array_equal(got[rows], plain[rows])


def test_attention_key_split_argument_errors():
    n, H, hd = 600, 2, 128
    qkv = torch.zeros((n, 3 * H * hd), dtype=torch.bfloat16, device="cuda")
    o = torch.zeros((n, H * hd), dtype=torch.bfloat16, device="cuda")
    ch = torch.zeros((n,), dtype=torch.int32, device="cuda")
    base = qkv.data_ptr()
    ws = torch.zeros((1 << 24,), dtype=torch.uint8, device="cuda")
    f = L.cosmot_mot_attention_split

    def call(d, split, nbytes=ws.numel()):
        return f(d, base, 3 * H * hd, base + 2 * H * hd, base + 4 * H * hd, 3 * H * hd, o.data_ptr(), H * hd, split,
                 ws.data_ptr(), nbytes, A.stream_handle(), check=False)
    full = L.AttnDesc(n_q=n, q_key_offset=0, n_keys=n, n_ar=10, n_heads=H, n_kv_heads=H, head_dim=hd, batch=1)
    assert call(full, 6) == L.COSMOT_ERR_INVALID_ARG  # 5 key tiles cannot be split 6 ways
    assert call(full, 9) == L.COSMOT_ERR_INVALID_ARG
    assert call(full, 2, nbytes=1024) == L.COSMOT_ERR_WORKSPACE
    skip = L.AttnDesc(n_q=n, q_key_offset=0, n_keys=n, n_ar=10, n_heads=H, n_kv_heads=H, head_dim=hd, batch=1,
                      mask_mode=L.COSMOT_MASK_BLOCK_CAUSAL, chunk=ch.data_ptr())
    assert call(skip, 2) == L.COSMOT_ERR_UNSUPPORTED  # tile skipping and key splits do not mix
    torch.cuda.synchronize()
    assert_device_ok()


def test_routed_linear_narrow_tiles_on_few_rows():
    """573 rows against a 4,096-wide output (a DROID denoising step at Nano
    widths) give 80 tiles 256 wide for 148 SMs, so the projection takes
    160-wide tiles (130 of them, the last one 96 columns wide).  Against the
    oracle, and bit-identical to the same rows computed inside a larger call
    that keeps 256-wide tiles: the tile width changes how many columns a CTA
    computes, never how one output element is accumulated."""
    k, n_out, m_small, m_big = 512, 4096, 573, 5000
    a = _bf16((m_big, k), 60)
    w0 = _bf16((n_out, k), 61, std=1.0 / np.sqrt(k))
    w1 = _bf16((n_out, k), 62, std=1.0 / np.sqrt(k))
    res = _bf16((m_big, n_out), 63)
    ad, w0d, w1d, rd = to_dev(a), to_dev(w0), to_dev(w1), to_dev(res)
    outs = {}
    split = 128  # one AR row tile, then the DM rows: 5 row tiles for 573 rows
    for m in (m_small, m_big):
        segs = [(0, split, 0, 0), (split, m, split, 1)]
        og = Guarded(torch.empty((m, n_out), dtype=torch.bfloat16, device="cuda"))
        e = L.Epilogue(kind=L.COSMOT_EPI_RESIDUAL, res=A.ptr(rd), ld_res=n_out)
        L.cosmot_routed_linear(A.ptr(ad), k, k, segs, A.ptr(w0d), A.ptr(w1d), n_out, A.ptr(og.t), n_out, e,
                               stream=A.stream_handle())
        torch.cuda.synchronize()
        assert_device_ok()
        og.assert_canaries(f"gemm {m} rows")
        outs[m] = og.t
    a64, r64 = synth.bf16_to_f64(a[:m_small]), synth.bf16_to_f64(res[:m_small])
    ref = np.concatenate([a64[:split] @ synth.bf16_to_f64(w0).T, a64[split:] @ synth.bf16_to_f64(w1).T]) + r64
    assert_close(to_f64(outs[m_small]), ref, "gemm 160-wide tiles")
    np.testing.assert_array_equal(bits(outs[m_small]), bits(outs[m_big][:m_small]))
