"""One Mixture-of-Transformers layer forward plus the Euler sampler step (fp64 oracle).

TEST INFRASTRUCTURE (see the package docstring).

Per "Cosmos 3 方法原理全解" §3 a MoT layer holds two rooms with their own
norms, QKV, O and MLP weights: the Reasoner set acts on AR tokens, the
Generator set on DM tokens; there is no router.  One attention is shared under
the §3 mask (see ``oracle.mask``).  §7.2: each Generator forward outputs a
velocity v and the sampler moves x_next = x + (sigma_next - sigma) * v, with
sigma_next < sigma; §2.2 / §4.2: clean tokens are fixed conditions and are not
updated.

Readings where the pages are silent:
  * norms are pre-norm RMSNorm with a gain and eps = 1e-6, no biases anywhere;
  * the FFN is SiLU-gated: (silu(b Wg^T) * (b Wu^T)) Wd^T, silu(z) = z/(1+e^-z);
  * the DM state x lives in the hidden space: the DM rows of the layer input
    are x, and the velocity is v = RMSNorm(h2; g_fin) Wvel^T on noisy rows;
  * sigma enters only through the Euler step (no timestep embedding);
  * n_kv_heads may divide n_heads (grouped queries): head q reads kv head
    q // (n_heads / n_kv_heads).

For one sequence with rows r and set s(r) = Reasoner if r is AR else Generator:
    a_r  = RMSNorm(h_r; g1_s)
    q, k, v = a_r Wq_s^T, a_r Wk_s^T, a_r Wv_s^T;  q, k <- mRoPE(pos_r)
    o_r  = sum_{j visible} softmax_j(q_r . k_j / sqrt(head_dim)) v_j   (per head)
    h1_r = h_r + o_r Wo_s^T
    b_r  = RMSNorm(h1_r; g2_s)
    h2_r = h1_r + (silu(b_r Wg_s^T) * (b_r Wu_s^T)) Wd_s^T
    noisy DM rows: x'_r = x_r + (sigma_next - sigma) * (RMSNorm(h2_r; g_fin) Wvel^T)
    clean DM rows: x'_r = x_r
"""

from __future__ import annotations

from dataclasses import dataclass

import numpy as np

from . import rope as _rope
from .layout import MOD_ACTION, REGION_AR, REGION_CLEAN, REGION_NOISY
from .mask import allow_matrix


def _f64(bits):
    b = np.ascontiguousarray(bits, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


@dataclass
class SetWeights:
    g1: np.ndarray
    wq: np.ndarray
    wk: np.ndarray
    wv: np.ndarray
    wo: np.ndarray
    g2: np.ndarray
    wg: np.ndarray
    wu: np.ndarray
    wd: np.ndarray


@dataclass
class LayerWeights:
    R: SetWeights     # Reasoner: AR tokens
    G: SetWeights     # Generator: DM tokens
    gfin: np.ndarray  # final DM norm gain
    wvel: np.ndarray  # velocity head [d, d]


def weights_from_bits(dims, w: dict) -> LayerWeights:
    """Promote the bf16 weight bits of ``synth.make_weights`` exactly to float64."""
    qc, kc = dims.q_cols, dims.kv_cols

    def one(s):
        wqkv = _f64(w[f"{s}.wqkv"])
        return SetWeights(g1=_f64(w[f"{s}.g1"]), wq=wqkv[:qc], wk=wqkv[qc:qc + kc],
                          wv=wqkv[qc + kc:qc + 2 * kc], wo=_f64(w[f"{s}.wo"]),
                          g2=_f64(w[f"{s}.g2"]), wg=_f64(w[f"{s}.wg"]),
                          wu=_f64(w[f"{s}.wu"]), wd=_f64(w[f"{s}.wd"]))

    return LayerWeights(R=one("R"), G=one("G"), gfin=_f64(w["gfin"]), wvel=_f64(w["wvel"]))


def rms_norm(h, g, eps):
    """h * g / sqrt(mean(h^2) + eps) over the last axis."""
    h = np.asarray(h, dtype=np.float64)
    return h * g / np.sqrt(np.mean(h * h, axis=-1, keepdims=True) + eps)


def silu(z):
    return z / (1.0 + np.exp(-z))


def routed(x, is_ar, fn):
    """Apply fn(rows, set) to AR rows with the Reasoner set and to the rest with
    the Generator set; `fn` gets the row block and "R" or "G"."""
    is_ar = np.asarray(is_ar, dtype=bool)
    out = None
    for sel, s in ((is_ar, "R"), (~is_ar, "G")):
        if not sel.any():
            continue
        y = fn(x[sel], s, sel)
        if out is None:
            out = np.zeros((len(x),) + y.shape[1:], dtype=np.float64)
        out[sel] = y
    return out


def attention(q, k, v, allow, scale, q_block: int = 2048):
    """Masked softmax attention per head in float64.

    q [nq, H, hd], k and v [nk, Hkv, hd], allow [nq, nk] bool.  Query head h
    reads kv head h // (H / Hkv).  A row with no visible key outputs zeros.
    Query rows are taken in blocks of `q_block` only to bound memory.
    """
    nq, n_heads, hd = q.shape
    n_kv = k.shape[1]
    group = n_heads // n_kv
    out = np.zeros((nq, n_heads, v.shape[2]), dtype=np.float64)
    for r0 in range(0, nq, q_block):
        r1 = min(nq, r0 + q_block)
        al = allow[r0:r1]
        any_key = al.any(axis=1)
        for hh in range(n_heads):
            g = hh // group
            s = (q[r0:r1, hh, :] @ k[:, g, :].T) * scale
            s = np.where(al, s, -np.inf)
            m = np.max(s, axis=1, keepdims=True)
            m = np.where(np.isfinite(m), m, 0.0)
            p = np.exp(s - m)
            l = p.sum(axis=1, keepdims=True)
            l = np.where(l > 0, l, 1.0)
            out[r0:r1, hh, :] = np.where(any_key[:, None], (p / l) @ v[:, g, :], 0.0)
    return out


def project_kv(dims, W: LayerWeights, h, region, pos):
    """Rotated K and V [n, Hkv, hd] of rows h (pre-attention norm, routed)."""
    hd, nkv = dims.head_dim, dims.n_kv_heads
    is_ar = np.asarray(region) == REGION_AR

    def fn(x, s, sel):
        ws = getattr(W, s)
        a = rms_norm(x, ws.g1, dims.eps)
        return np.concatenate([a @ ws.wk.T, a @ ws.wv.T], axis=1)

    kv = routed(np.asarray(h, np.float64), is_ar, fn)
    k = kv[:, :dims.kv_cols].reshape(-1, nkv, hd)
    v = kv[:, dims.kv_cols:].reshape(-1, nkv, hd)
    k = _rope.apply(k, pos, hd, dims.rope_sections, dims.rope_base)
    return k, v


def layer_forward(dims, W: LayerWeights, h, region, pos, chunk, sigma, sigma_next,
                  mode="full", rows=None, cache=None, head=True):
    """One MoT layer forward over one packed sequence, plus the Euler step.

    h [N, d] float64 (DM rows are the sampler state x), region/pos/chunk from
    ``oracle.layout``.  `rows` selects the output rows (all by default); K and V
    are always formed for every row.  `cache` = (k, v, chunk) of extra DM keys
    (already rotated) that sit between the AR keys and this sequence's DM keys
    in key order, as a streaming key/value cache does.

    Returns a dict with h2 [len(rows), d], the attention half h1 [len(rows), d],
    x_new [len(rows), d] (NaN on AR rows), vel [len(rows), d] (NaN except on
    noisy rows) and the row indices.
    With head=False the velocity head and the Euler step are left out (x_new
    and vel all NaN): a layer inside a stack.
    """
    h = np.asarray(h, dtype=np.float64)
    region = np.asarray(region)
    chunk = np.asarray(chunk)
    n = len(h)
    rows = np.arange(n) if rows is None else np.asarray(rows, dtype=np.int64)
    hd, nh = dims.head_dim, dims.n_heads
    is_ar = region == REGION_AR

    # Keys and values of every row of the sequence.
    k_seq, v_seq = project_kv(dims, W, h, region, pos)

    # Key order: AR rows, cached rows, DM rows of this sequence.
    n_ar = int(is_ar.sum())
    if not np.all(is_ar[:n_ar]) or is_ar[n_ar:].any():
        raise ValueError("AR rows must form the prefix of the packed sequence")
    if cache is not None:
        kc, vc, cc = cache
        nc = len(kc)
        k_all = np.concatenate([k_seq[:n_ar], kc, k_seq[n_ar:]])
        v_all = np.concatenate([v_seq[:n_ar], vc, v_seq[n_ar:]])
        key_region = np.concatenate([region[:n_ar], np.full(nc, REGION_CLEAN, region.dtype), region[n_ar:]])
        key_chunk = np.concatenate([chunk[:n_ar], np.asarray(cc, chunk.dtype), chunk[n_ar:]])
    else:
        nc = 0
        k_all, v_all, key_region, key_chunk = k_seq, v_seq, region, chunk
    key_of_row = np.where(np.arange(n) < n_ar, np.arange(n), np.arange(n) + nc)

    # Queries of the selected rows.
    hr = h[rows]
    ar_r = is_ar[rows]

    def qfn(x, s, sel):
        ws = getattr(W, s)
        return rms_norm(x, ws.g1, dims.eps) @ ws.wq.T

    q = routed(hr, ar_r, qfn).reshape(-1, nh, hd)
    q = _rope.apply(q, np.asarray(pos)[rows], hd, dims.rope_sections, dims.rope_base)

    allow = allow_matrix(key_of_row[rows], key_region, key_chunk, mode)
    o = attention(q, k_all, v_all, allow, 1.0 / np.sqrt(hd)).reshape(len(rows), nh * hd)

    h1 = hr + routed(o, ar_r, lambda x, s, sel: x @ getattr(W, s).wo.T)

    def ffn(x, s, sel):
        ws = getattr(W, s)
        b = rms_norm(x, ws.g2, dims.eps)
        return (silu(b @ ws.wg.T) * (b @ ws.wu.T)) @ ws.wd.T

    h2 = h1 + routed(h1, ar_r, ffn)

    x_new = np.full_like(h2, np.nan)
    vel = np.full_like(h2, np.nan)
    if not head:
        return {"rows": rows, "h1": h1, "h2": h2, "x_new": x_new, "vel": vel}
    reg_r = region[rows]
    clean = reg_r == REGION_CLEAN
    noisy = reg_r == REGION_NOISY
    x_new[clean] = hr[clean]
    if noisy.any():
        vel[noisy] = rms_norm(h2[noisy], W.gfin, dims.eps) @ W.wvel.T
        x_new[noisy] = euler_step(hr[noisy], vel[noisy], sigma, sigma_next)
    return {"rows": rows, "h1": h1, "h2": h2, "x_new": x_new, "vel": vel}


def euler_step(x, v, sigma, sigma_next):
    """x_next = x + (sigma_next - sigma) * v ("Cosmos 3 方法原理全解" §7.2)."""
    return np.asarray(x, np.float64) + (float(sigma_next) - float(sigma)) * np.asarray(v, np.float64)


def cfg_combine(v_cond, v_base, guidance):
    """Classifier-free guidance ("Cosmos 3 方法原理全解" §7.2):
    v = v_base + w * (v_cond - v_base)."""
    v_cond = np.asarray(v_cond, np.float64)
    v_base = np.asarray(v_base, np.float64)
    return v_base + float(guidance) * (v_cond - v_base)


def cfg_step(dims, W, h_cond, h_base, lay, sigma, sigma_next, guidance, mode="full"):
    """One guided sampler step ("Cosmos 3 方法原理全解" §7.2-7.3): two Generator
    forwards that share the DM rows (the state x) and differ in their AR rows
    (the prompt and the baseline prompt), the guided velocity, one Euler step.

    Reading: both AR sequences have the same length (the baseline prompt is
    padded to the prompt's length), so the two passes share one layout.
    Returns x' of the noisy rows and both passes' outputs.
    """
    noisy = lay.region == REGION_NOISY
    if not np.array_equal(np.asarray(h_cond)[lay.n_ar:], np.asarray(h_base)[lay.n_ar:]):
        raise ValueError("the two guidance passes must share their DM rows")
    oc = layer_forward(dims, W, h_cond, lay.region, lay.pos, lay.chunk, sigma, sigma_next, mode)
    ob = layer_forward(dims, W, h_base, lay.region, lay.pos, lay.chunk, sigma, sigma_next, mode)
    v = cfg_combine(oc["vel"][noisy], ob["vel"][noisy], guidance)
    x = np.asarray(h_cond, np.float64)[noisy]
    return euler_step(x, v, sigma, sigma_next), oc, ob


def stack_forward(dims, layers, h, region, pos, chunk, sigma, sigma_next, mode="full"):
    """A stack of MoT layers, then the flow-matching step ("Cosmos 3 方法原理全解"
    §3 for the layer, §12.4 for the stacked models, §7.2 for the step).

    h^0 = h; h^l = layer_l(h^{l-1}) for each entry of `layers` (LayerWeights,
    applied in order); on the noisy rows v = RMSNorm(h^L; g_fin) W_vel^T with
    the final norm and velocity head of the last entry, and x' = x + (sigma_next
    - sigma) v where x is the noisy rows of h (the state is the stack's input).
    Returns h_out = h^L, the hidden states after every layer, vel and x_new as
    layer_forward does.
    """
    h = np.asarray(h, dtype=np.float64)
    region = np.asarray(region)
    x = h
    hidden = []
    for W in layers:
        x = layer_forward(dims, W, x, region, pos, chunk, sigma, sigma_next, mode, head=False)["h2"]
        hidden.append(x)
    vel = np.full_like(x, np.nan)
    x_new = np.full_like(x, np.nan)
    clean = region == REGION_CLEAN
    noisy = region == REGION_NOISY
    x_new[clean] = h[clean]
    if noisy.any():
        last = layers[-1]
        vel[noisy] = rms_norm(x[noisy], last.gfin, dims.eps) @ last.wvel.T
        x_new[noisy] = euler_step(h[noisy], vel[noisy], sigma, sigma_next)
    return {"h_out": x, "hidden": hidden, "vel": vel, "x_new": x_new}


def stack_sample(dims, layers, h, lay, sigmas, mode="full"):
    """Sampler loop over a layer stack: one stack forward and one Euler step per
    (sigma, sigma_next); the noisy rows of h carry the state."""
    h = np.array(h, dtype=np.float64)
    noisy = lay.region == REGION_NOISY
    outs = []
    for s0, s1 in zip(sigmas[:-1], sigmas[1:]):
        out = stack_forward(dims, layers, h, lay.region, lay.pos, lay.chunk, s0, s1, mode)
        h[noisy] = out["x_new"][noisy]
        outs.append(out)
    return h, outs


def shift_sigmas(n_steps: int, shift: float) -> np.ndarray:
    """Sampler noise levels with the flow shift ("Cosmos 3 方法原理全解" §6.3:
    t_bar = 1 - t, sigma = s t_bar / (1 + (s - 1) t_bar)), evaluated on the
    uniform grid t_k = k / n_steps, k = 0 .. n_steps: sigma_0 = 1, sigma_n = 0.

    Reading: the pages define the shift for the training-time noise draw and
    quote an inference "shift" beside the step count; applying the same map to
    the uniform inference grid is the plainest reading.
    """
    if n_steps < 1 or not shift > 0:
        raise ValueError("n_steps >= 1 and shift > 0 required")
    t_bar = 1.0 - np.arange(n_steps + 1, dtype=np.float64) / n_steps
    return shift * t_bar / (1.0 + (shift - 1.0) * t_bar)


def action_embed(x_a, w_in):
    """Domain-specific action input projection ("Cosmos 3 方法原理全解" §4.2:
    normalised actions, clean or noisy, enter the Generator through W_in):
    rows x_a [n, C_a] -> x_a W_in^T [n, d]."""
    return np.asarray(x_a, np.float64) @ np.asarray(w_in, np.float64).T


def action_velocity(dims, h_last, g_fin, w_out):
    """Action velocity from the last hidden states of the noisy action rows
    (§4.2: W_out returns the velocity at the current sigma, in the normalised
    action space): RMSNorm with the final DM gain, then W_out [C_a, d]."""
    return rms_norm(np.asarray(h_last, np.float64), g_fin, dims.eps) @ np.asarray(w_out, np.float64).T


def policy_step(dims, layers, h, x_a, w_in, w_out, lay, sigma, sigma_next, sigma_a, sigma_a_next, mode="full",
                guidance=None, h_base=None, x_a_base=None):
    """One sampler step of a policy with an action head (§4.2, §7.2, §7.3).

    The action rows of the layer input (clean and noisy, in packed order) are
    x_a W_in^T; the stack runs; the other noisy rows take the hidden-space
    velocity head and the Euler step with (sigma, sigma_next); the noisy action
    rows take v_a = RMSNorm(h^L; g_fin) W_out^T and x_a' = x_a + (sigma_a_next
    - sigma_a) v_a (each modality has its own noise level, §6.3).  With a
    guidance weight the baseline pass (h_base, x_a_base: same DM rows, other
    AR rows) runs too and both velocities are combined before the steps.

    Returns (h_new, x_a_new): h_new is the stack input (action rows = x_a
    W_in^T) with its noisy non-action rows stepped; x_a_new has its noisy rows
    stepped.
    """
    act = lay.modality == MOD_ACTION
    noisy = lay.region == REGION_NOISY
    act_noisy = act & noisy
    vid_noisy = noisy & ~act

    def forward(h_in, xa):
        hh = np.array(h_in, dtype=np.float64)
        hh[act] = action_embed(xa, w_in)
        x = hh
        for W in layers:
            x = layer_forward(dims, W, x, lay.region, lay.pos, lay.chunk, sigma, sigma_next, mode, head=False)["h2"]
        last = layers[-1]
        v = rms_norm(x[vid_noisy], last.gfin, dims.eps) @ last.wvel.T
        va = action_velocity(dims, x[act_noisy], last.gfin, w_out)
        return hh, v, va

    hh, v, va = forward(h, x_a)
    if guidance is not None:
        _, vb, vab = forward(h_base, x_a_base)
        v = cfg_combine(v, vb, guidance)
        va = cfg_combine(va, vab, guidance)
    h_new = hh  # the action rows hold the embedding of x_a (the state is x_a)
    h_new[vid_noisy] = euler_step(h_new[vid_noisy], v, sigma, sigma_next)
    x_new = np.array(x_a, dtype=np.float64)
    n_act_clean = int((act & (lay.region == REGION_CLEAN)).sum())
    x_new[n_act_clean:] = euler_step(x_new[n_act_clean:], va, sigma_a, sigma_a_next)
    return h_new, x_new


def sample(dims, W, h, lay, sigmas, mode="full"):
    """Sampler loop: one layer forward and one Euler step per (sigma, sigma_next).

    The noisy DM rows of h are replaced by x' after each step; AR and clean rows
    stay fixed.  AR outputs never depend on DM rows, so recomputing them every
    step equals caching them after the first.
    """
    h = np.array(h, dtype=np.float64)
    noisy = lay.region == REGION_NOISY
    outs = []
    for s0, s1 in zip(sigmas[:-1], sigmas[1:]):
        out = layer_forward(dims, W, h, lay.region, lay.pos, lay.chunk, s0, s1, mode)
        h[noisy] = out["x_new"][noisy]
        outs.append(out)
    return h, outs


class StreamState:
    """Key/value cache of a streaming rollout.

    AR keys are formed once.  A ring of `slots` history blocks holds the
    rotated K and V of past blocks; committing a block writes its K and V
    (projected from the block's final x) over the oldest slot.
    """

    def __init__(self, slots: int):
        self.slots = slots
        self.k = [None] * slots
        self.v = [None] * slots
        self.chunk = [None] * slots
        self.next = 0

    def commit(self, k, v, chunk):
        self.k[self.next], self.v[self.next], self.chunk[self.next] = k, v, chunk
        self.next = (self.next + 1) % self.slots

    def cache(self):
        ks = [x for x in self.k if x is not None]
        if not ks:
            return None
        vs = [x for x in self.v if x is not None]
        cs = [x for x in self.chunk if x is not None]
        return np.concatenate(ks), np.concatenate(vs), np.concatenate(cs)


def stream_commit(dims, W, state: StreamState, x_block, lay_block):
    """Commit a finished block: K/V of its rows (Generator QKV + mRoPE on K)."""
    dm = lay_block.region != REGION_AR
    k, v = project_kv(dims, W, x_block, lay_block.region[dm], lay_block.pos[dm])
    state.commit(k, v, lay_block.chunk[dm])


def stream_block(dims, W, state: StreamState, h_ar, x_block, lay_block, sigmas, rows=None):
    """Denoise one streaming block with `len(sigmas) - 1` Euler steps.

    The sequence is [AR rows; block rows]; keys are AR, the cached history and
    the block itself (block-causal: history chunks precede the block's).
    Returns the final x of the block and the last step's outputs.
    """
    x = np.array(x_block, dtype=np.float64)
    n_ar = len(h_ar)
    out = None
    for s0, s1 in zip(sigmas[:-1], sigmas[1:]):
        h = np.concatenate([np.asarray(h_ar, np.float64), x])
        r = None if rows is None else n_ar + np.asarray(rows)
        out = layer_forward(dims, W, h, lay_block.region, lay_block.pos, lay_block.chunk, s0, s1,
                            mode="block_causal", rows=r if r is not None else np.arange(n_ar, len(h)),
                            cache=state.cache())
        if rows is None:
            x = out["x_new"]
        else:
            x = None  # a row subset cannot feed the next step
            break
    return x, out
