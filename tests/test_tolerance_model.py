"""Where the parity tolerance's rounding constants come from (CPU, no GPU).

The CUDA path keeps fp32 accumulators but stores intermediates in bf16 (round
to nearest even) where a kernel hands them to the next one; the fp64 oracle
stores nothing.  `emulate_layer` below runs the oracle's arithmetic in float64
and rounds to bf16 exactly where the kernels store a value:

    a   = RMSNorm(h; g1)              (operand of the QKV GEMM)
    q,k = mRoPE(a Wq^T), mRoPE(a Wk^T); v = a Wv^T   (attention operands)
    P   = exp(s - m)                  (softmax weights, bf16 in tensor memory;
                                       the row sum stays unrounded)
    o   = (P V) / l                   (operand of the O GEMM)
    h1  = h + o Wo^T                  (float32: not rounded)
    b   = RMSNorm(h1; g2)             (operand of gate and up)
    u   = silu(b Wg^T) * (b Wu^T)     (operand of the down GEMM)
    h2  = h1 + u Wd^T                 (the layer output)
    af  = RMSNorm(h2; g_fin)          (operand of the velocity GEMM)
    v   = af Wvel^T (fp32 accumulator); x' = x + (sigma_next - sigma) v

so it models the CUDA path with exact accumulation (fp32 accumulation adds
~1e-6 relative, far below these terms).  The widths are small enough to run
in seconds; the weights are scaled by sqrt(fan_in at full width / fan_in
here) so that every pre-activation has the variance it has at d_model 4096,
FFN 14336 with N(0, 0.02) weights (the workloads' distribution).

Checked: the propagated error of h2, v and x' (before the output's own
rounding) has a standard deviation within the tolerance's SIGMA_* units of
2^-9/sqrt(3) * rms(branch), at two widths (so the constant does not grow with
the width), and stays under the tolerance's max-abs bound; rel-L2 stays under
5e-3 with a margin.  A 10-step sampler that keeps its state in float32 (as
cosmot_layer_forward_io does) meets the one-step bounds after every step (its
error is the sum of the steps' velocity errors times dsigma: rel-L2 1.6e-3
after 10 steps), while the same sampler storing its state in bf16 after every
step passes rel-L2 5e-3 by the last step (5.4e-3: one rounding of x per step).
"""

import numpy as np
import pytest

import synth
from oracle import layer as olayer
from oracle import layout as olayout
from oracle import mask as omask
from oracle import rope as orope
from tolerance import (MAX_ABS, REL_L2, SIGMA_ATTN, SIGMA_H_OUT, SIGMA_VEL, TAIL, UNIT, compare, half_ulp_bf16,
                       rms)


def bf(x):
    """float64 -> float32 -> bf16 (RN-even) -> float64: a kernel's fp32 value stored as bf16."""
    return synth.bf16_to_f64(synth.bf16_round(np.asarray(x, dtype=np.float32)))


def scaled_weights(dims, seed):
    """bf16 weights whose products have the full-width (d 4096, FFN 14336,
    N(0, 0.02)) pre-activation variance at this width; gains 1 + N(0, 0.02)."""
    rng = np.random.default_rng(seed)
    d, f = dims.d_model, dims.ffn

    def w(shape, full_fan):
        return bf(rng.standard_normal(shape) * 0.02 * np.sqrt(full_fan / shape[1]))

    def gain():
        return bf(1.0 + 0.02 * rng.standard_normal(d))

    def one():
        return olayer.SetWeights(g1=gain(), wq=w((dims.q_cols, d), 4096), wk=w((dims.kv_cols, d), 4096),
                                 wv=w((dims.kv_cols, d), 4096), wo=w((d, dims.q_cols), 4096), g2=gain(),
                                 wg=w((f, d), 4096), wu=w((f, d), 4096), wd=w((d, f), 14336))

    return olayer.LayerWeights(R=one(), G=one(), gfin=gain(), wvel=w((d, d), 4096))


def emulate_layer(dims, W, h, lay, sigma, sigma_next, x=None, mode="full"):
    """The CUDA path's storage roundings on the oracle's arithmetic (see the
    module docstring).  h: the bf16 layer input; x: the sampler state of the
    noisy rows (float64; defaults to h's noisy rows).  Returns h2 before and
    after its rounding, v and x' (unrounded)."""
    n, hd, H, Hkv = len(h), dims.head_dim, dims.n_heads, dims.n_kv_heads
    is_ar = lay.region == olayout.REGION_AR
    noisy = lay.region == olayout.REGION_NOISY

    def routed(xx, fn):
        out = None
        for sel, s in ((is_ar, W.R), (~is_ar, W.G)):
            if not sel.any():
                continue
            y = fn(xx[sel], s)
            if out is None:
                out = np.zeros((len(xx),) + y.shape[1:])
            out[sel] = y
        return out

    a = bf(routed(h, lambda r, s: olayer.rms_norm(r, s.g1, dims.eps)))
    q = routed(a, lambda r, s: r @ s.wq.T).reshape(n, H, hd)
    k = routed(a, lambda r, s: r @ s.wk.T).reshape(n, Hkv, hd)
    v = bf(routed(a, lambda r, s: r @ s.wv.T)).reshape(n, Hkv, hd)
    q = bf(orope.apply(q, lay.pos, hd, dims.rope_sections, dims.rope_base))
    k = bf(orope.apply(k, lay.pos, hd, dims.rope_sections, dims.rope_base))
    o = bf(attention_p_bf16(q, k, v, omask.allow_matrix(np.arange(n), lay.region, lay.chunk, mode))
           .reshape(n, H * hd))
    h1 = h + routed(o, lambda r, s: r @ s.wo.T)
    b = bf(routed(h1, lambda r, s: olayer.rms_norm(r, s.g2, dims.eps)))
    u = bf(routed(b, lambda r, s: olayer.silu(r @ s.wg.T) * (r @ s.wu.T)))
    h2_pre = h1 + routed(u, lambda r, s: r @ s.wd.T)
    h2 = bf(h2_pre)
    af = bf(olayer.rms_norm(h2[noisy], W.gfin, dims.eps))
    vel = af @ W.wvel.T
    x0 = h[noisy] if x is None else x
    return {"h2_pre": h2_pre, "h2": h2, "vel": vel, "x_new": x0 + (float(sigma_next) - float(sigma)) * vel}


def attention_p_bf16(q, k, v, allow):
    """Softmax attention with the weights P rounded to bf16 before the PV
    product and the row sum l taken over the unrounded weights."""
    nq, H, hd = q.shape
    g = H // k.shape[1]
    out = np.zeros((nq, H, hd))
    for hh in range(H):
        s = np.where(allow, q[:, hh] @ k[:, hh // g].T / np.sqrt(hd), -np.inf)
        p = np.exp(s - s.max(axis=1, keepdims=True))
        out[:, hh] = (bf(p) @ v[:, hh // g]) / p.sum(axis=1, keepdims=True)
    return out


def _setup(d, seed=11):
    dims = synth.ModelDims(d_model=d, n_heads=d // 128, n_kv_heads=d // 128, head_dim=128, ffn=int(3.5 * d),
                           rope_sections=(16, 24, 24))
    W = scaled_weights(dims, seed)
    lay = olayout.build_layout(synth.preset("droid").layout)  # 130 AR + 181 clean + 392 noisy
    h = bf(np.random.default_rng(seed + 1).standard_normal((lay.n_tokens, d)))
    return dims, W, lay, h


def _units(err, branch):
    return float(np.std(err)) / (UNIT * branch)


@pytest.mark.parametrize("d", [512, 1024])
def test_rounding_constants_bound_the_emulated_error(d):
    dims, W, lay, h = _setup(d)
    s0, s1 = 1.0, 0.9
    ref = olayer.layer_forward(dims, W, h, lay.region, lay.pos, lay.chunk, s0, s1)
    emu = emulate_layer(dims, W, h, lay, s0, s1)
    noisy = lay.region == olayout.REGION_NOISY
    br_h = rms(ref["h2"] - ref["h1"])
    vref = ref["vel"][noisy]
    br_v = rms(vref)
    u_h = _units(emu["h2_pre"] - ref["h2"], br_h)
    u_v = _units(emu["vel"] - vref, br_v)
    # the propagated errors are as the tolerance's constants say, with margin
    assert 2.5 < u_h <= 0.95 * SIGMA_H_OUT, u_h
    assert 2.5 < u_v <= 0.95 * SIGMA_VEL, u_v
    # the full bounds hold on the emulated outputs (h2 and v stored in bf16)
    r_h = compare(emu["h2"], ref["h2"], SIGMA_H_OUT, br_h)
    r_v = compare(bf(emu["vel"]), vref, SIGMA_VEL, br_v)
    r_x = compare(emu["x_new"], ref["x_new"][noisy], SIGMA_VEL, abs(s1 - s0) * br_v, out_bf16=False)
    for r in (r_h, r_v, r_x):
        assert r["over"] == 0 and r["rel_l2"] <= 0.9 * REL_L2, r
    # the Gaussian term is what carries h2's bound, not the stated 2e-2
    assert TAIL * SIGMA_H_OUT * UNIT * br_h > MAX_ABS


def test_rounding_constant_of_the_attention_kernel():
    """The attention kernel alone (bf16 q, k, v in, P rounded to bf16, output
    rounded): the deviation before the output's rounding, in units of
    2^-9/sqrt(3) * rms(o), on the kernel tests' input distribution."""
    rng = np.random.default_rng(3)
    n, n_ar, H, hd = 700, 130, 4, 128
    q, k, v = (bf(rng.standard_normal((n, H, hd))) for _ in range(3))
    region = np.where(np.arange(n) < n_ar, olayout.REGION_AR, olayout.REGION_NOISY).astype(np.int8)
    allow = omask.allow_matrix(np.arange(n), region, np.where(np.arange(n) < n_ar, -1, 0), "full")
    ref = olayer.attention(q, k, v, allow, 1.0 / np.sqrt(hd))
    emu = attention_p_bf16(q, k, v, allow)
    u = _units(emu - ref, rms(ref))
    assert 0.3 < u <= 0.9 * SIGMA_ATTN, u
    r = compare(bf(emu), ref, SIGMA_ATTN, rms(ref))
    assert r["over"] == 0 and r["rel_l2"] <= 0.9 * REL_L2, r


def test_float32_sampler_state_meets_the_per_step_bound_after_every_step():
    """Ten Euler steps of the DROID schedule ("Cosmos 3 方法原理全解" §7.2):
    with the state in float32 (the layer reads its bf16 copy) every step's x'
    meets the one-step bound; re-rounding the state to bf16 after every step
    instead adds a rounding of x per step and ends above the stated rel-L2."""
    dims, W, lay, h0 = _setup(512)
    sig = synth.preset("droid").sigmas
    noisy = lay.region == olayout.REGION_NOISY
    _, outs = olayer.sample(dims, W, h0, lay, sig)
    h32, x32 = h0.copy(), h0[noisy].copy()
    h16 = h0.copy()
    rel32, rel16 = [], []
    for k, (s0, s1) in enumerate(zip(sig[:-1], sig[1:])):
        e32 = emulate_layer(dims, W, h32, lay, s0, s1, x=x32)
        e16 = emulate_layer(dims, W, h16, lay, s0, s1)
        x32 = e32["x_new"]
        h32[noisy] = bf(x32)
        h16[noisy] = bf(e16["x_new"])
        want = outs[k]["x_new"][noisy]
        r = compare(x32, want, SIGMA_VEL, abs(s1 - s0) * rms(outs[k]["vel"][noisy]), out_bf16=False)
        assert r["over"] == 0 and r["rel_l2"] <= REL_L2, (k, r)
        rel32.append(r["rel_l2"])
        rel16.append(float(np.linalg.norm(h16[noisy] - want) / np.linalg.norm(want)))
    print("rel-L2 per step, float32 state:", np.round(rel32, 5), "bf16 state:", np.round(rel16, 5))
    assert max(rel32) < 0.5 * REL_L2, rel32
    assert rel16[-1] > REL_L2 > 3 * rel32[-1], (rel16, rel32)


def test_half_ulp_term_is_needed_above_eight():
    """A bf16 value at |x| in [8, 16) carries up to 2^-5 of rounding alone,
    more than the stated 2e-2: the tolerance's half-ulp term."""
    assert half_ulp_bf16(np.array([9.0]))[0] == 2.0 ** -5
    x = np.float32(8.0 + 2.0 ** -5 * 0.999)
    assert abs(bf(x) - float(x)) > MAX_ABS
