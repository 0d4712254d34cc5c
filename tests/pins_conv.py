"""Pins of the oracle's short convolution (the depthwise convolution + SiLU in
front of the scan) against facts that do not come from its own loops:

* numpy's ``correlate`` on each channel: the causal convolution of a channel
  over [conv state; inputs] is their valid-mode correlation with the taps; the
  anti-causal, block-local one is the same operation on the block read right
  to left from zeros;
* impulse responses: a single 1 at token t0 of one channel comes out as the
  taps in a fixed order (the newest input meets the last tap), which pins the
  tap orientation, the shift and the block boundary of the reverse direction;
* closed forms of the activation: zero inputs give silu(bias) = bias / (1 +
  exp(-bias)) (scipy's expit), and silu off gives the plain affine map;
* the conv state: its rows are the last width-1 rows of [state; inputs], so
  with L < width-1 the old rows shift up;
* the all-block pass: every noisy block's forward convolution equals a
  one-block convolution whose conv state is the clean stream's rows before the
  block (taken by slicing the inputs).

The definition pinned: a Mamba layer's depthwise convolution over x, B, C with
the conv state in the cache ("Training Hybrid Block Diffusion Language Models
with Partial Bidirectionality", the paragraph after eq. (14)), anti-causal for
the reverse direction ("Breaking the Bottleneck with DiffuApriel", section
3.2, after eq. (5)) and confined to the block like the reverse scan (first
page, eq. (12)).
"""
from __future__ import annotations

import numpy as np
from scipy.special import expit


def _shape(**kw):
    s = dict(batch=2, seqlen=12, nheads=2, headdim=3, dstate=2, ngroups=1, block_len=4)
    s.update(kw)
    return s


def _channels(s):
    return s["nheads"] * s["headdim"] + 2 * s["ngroups"] * s["dstate"]


def _direction(s, width, rng, bias=True):
    B, L, H, P, N, G = (s[k] for k in ("batch", "seqlen", "nheads", "headdim", "dstate", "ngroups"))
    cx = _channels(s)
    d = {"x": rng.normal(0, 1, (B, L, H, P)), "B": rng.normal(0, 1, (B, L, G, N)),
         "C": rng.normal(0, 1, (B, L, G, N)), "weight": rng.normal(0, 0.7, (cx, width))}
    if bias:
        d["bias"] = rng.normal(0, 0.5, (cx,))
    return d


def _rows(s, d):
    """[B][L][Cx] rows, channel order x | B | C (the documented packing)."""
    B, L = s["batch"], s["seqlen"]
    parts = [np.asarray(d[k], dtype=np.float64) for k in ("x", "B", "C")]
    return np.concatenate([a.reshape(B, L, int(np.prod(a.shape[2:]))) for a in parts], axis=2)


def _act(v, silu):
    return v * expit(v) if silu else v


def _correlate_causal(u, w, state, silu, bias):
    """Reference by numpy: per batch row and channel, correlate [state; u] with w."""
    B, L, cx = u.shape
    W = w.shape[1]
    out = np.zeros_like(u)
    for b in range(B):
        for c in range(cx):
            pre = state[b, :, c] if state is not None else np.zeros(W - 1)
            seq = np.concatenate([pre, u[b, :, c]])
            out[b, :, c] = np.correlate(seq, w[c], mode="valid") + (bias[c] if bias is not None else 0.0)
    return _act(out, silu)


def _correlate_anticausal(u, w, T, silu, bias):
    """Reference by numpy: each block reversed, correlated from zeros, reversed back."""
    B, L, cx = u.shape
    W = w.shape[1]
    out = np.zeros_like(u)
    for b in range(B):
        for k in range(L // T):
            for c in range(cx):
                seq = np.concatenate([np.zeros(W - 1), u[b, k * T:(k + 1) * T, c][::-1]])
                out[b, k * T:(k + 1) * T, c] = (np.correlate(seq, w[c], mode="valid")[::-1]
                                                + (bias[c] if bias is not None else 0.0))
    return _act(out, silu)


def _close(a, b, what):
    a, b = np.asarray(a), np.asarray(b)
    assert a.shape == b.shape, (what, a.shape, b.shape)
    err = np.max(np.abs(a - b)) if a.size else 0.0
    assert err <= 1e-12 * max(1.0, np.max(np.abs(b)) if b.size else 1.0), f"{what}: max err {err}"


def pin_correlate_prefix(o):
    """Both directions of a sequence against numpy's correlate, several widths,
    with and without a conv state and SiLU."""
    for width, silu, with_state, T in ((4, True, True, 4), (3, False, True, 2), (2, True, False, 6),
                                       (1, True, True, 3), (4, True, True, 1)):
        s = _shape(block_len=T)
        rng = np.random.default_rng(10 + width + 7 * T)
        fwd, rev = _direction(s, width, rng), _direction(s, width, rng, bias=(width != 2))
        st = rng.normal(0, 1, (s["batch"], width - 1, _channels(s))) if with_state else None
        vf, vr, _ = o.conv_prefix(s, width, silu, fwd, rev, st)
        _close(_rows(s, vf), _correlate_causal(_rows(s, fwd), fwd["weight"], st, silu, fwd.get("bias")),
               f"forward w={width}")
        _close(_rows(s, vr), _correlate_anticausal(_rows(s, rev), rev["weight"], T, silu, rev.get("bias")),
               f"reverse w={width} T={T}")


def pin_impulse_response(o):
    """A single 1 at token t0 of one channel, no bias, no SiLU: the forward output
    at t0 + i is tap W-1-i, the reverse output at t0 - i is tap W-1-i while
    t0 - i stays in t0's block, and every other output is zero."""
    s = _shape(batch=1, seqlen=12, block_len=4)
    W = 4
    cx = _channels(s)
    rng = np.random.default_rng(3)
    w = rng.normal(0, 1, (cx, W))
    for c, t0 in ((0, 5), (cx - 1, 4), (s["nheads"] * s["headdim"] + 1, 11), (2, 0)):
        u = np.zeros((1, s["seqlen"], cx))
        u[0, t0, c] = 1.0
        d = _unrows(s, u)
        d["weight"] = w
        vf, vr, _ = o.conv_prefix(s, W, False, d, d, None)
        f, r = _rows(s, vf), _rows(s, vr)
        ef, er = np.zeros_like(u), np.zeros_like(u)
        for i in range(W):
            if t0 + i < s["seqlen"]:
                ef[0, t0 + i, c] = w[c, W - 1 - i]
            if t0 - i >= (t0 // s["block_len"]) * s["block_len"]:
                er[0, t0 - i, c] = w[c, W - 1 - i]
        _close(f, ef, f"forward impulse c={c} t0={t0}")
        _close(r, er, f"reverse impulse c={c} t0={t0}")


def _unrows(s, u):
    B, L, H, P, N, G = (s[k] for k in ("batch", "seqlen", "nheads", "headdim", "dstate", "ngroups"))
    hp, gn = H * P, G * N
    return {"x": u[:, :, :hp].reshape(B, L, H, P).copy(), "B": u[:, :, hp:hp + gn].reshape(B, L, G, N).copy(),
            "C": u[:, :, hp + gn:].reshape(B, L, G, N).copy()}


def pin_activation_closed_form(o):
    """Zero inputs and zero state: the output is silu(bias) (bias / (1 + exp(-bias))
    through scipy's expit) with SiLU, the bias itself without."""
    s = _shape(batch=1, seqlen=4, block_len=4)
    cx = _channels(s)
    rng = np.random.default_rng(5)
    bias = rng.normal(0, 3, (cx,))
    d = _unrows(s, np.zeros((1, 4, cx)))
    d["weight"], d["bias"] = rng.normal(0, 1, (cx, 4)), bias
    for silu in (True, False):
        vf, vr, _ = o.conv_prefix(s, 4, silu, d, d, None)
        want = np.broadcast_to(bias * expit(bias) if silu else bias, (1, 4, cx))
        _close(_rows(s, vf), want, "forward bias only")
        _close(_rows(s, vr), want, "reverse bias only")


def pin_state_out(o):
    """The new conv state holds the last W-1 rows of [state; inputs]: taken
    by slicing, including L < W-1 where old rows shift up."""
    for L, T in ((12, 4), (2, 2), (1, 1)):
        s = _shape(seqlen=L, block_len=T)
        W = 4
        rng = np.random.default_rng(20 + L)
        d = _direction(s, W, rng)
        st = rng.normal(0, 1, (s["batch"], W - 1, _channels(s)))
        _, _, so = o.conv_prefix(s, W, True, d, None, st, want_state_out=True)
        want = np.concatenate([st, _rows(s, d)], axis=1)[:, -(W - 1):, :]
        _close(so, want, f"state_out L={L}")
    s = _shape(seqlen=0, block_len=4)
    st = np.random.default_rng(1).normal(0, 1, (2, 3, _channels(s)))
    _, _, so = o.conv_prefix(s, 4, True, _direction(s, 4, np.random.default_rng(2)), None, st,
                             want_state_out=True)
    _close(so, st, "state_out L=0")


def pin_allblock_noisy_from_clean_rows(o):
    """All-block pass: the clean stream equals the one-sequence convolution, and
    noisy block k's forward output equals a one-block convolution whose conv
    state is the clean rows before the block (the given state for rows before
    token 0)."""
    for W, T in ((4, 4), (4, 2), (3, 1)):
        s = _shape(seqlen=8, block_len=T)
        rng = np.random.default_rng(30 + W + T)
        cf, cr, nf, nr = (_direction(s, W, rng) for _ in range(4))
        st = rng.normal(0, 1, (s["batch"], W - 1, _channels(s)))
        outs = o.conv_allblock(s, W, True, cf, cr, nf, nr, st)
        vf, vr, _ = o.conv_prefix(s, W, True, cf, cr, st)
        _close(_rows(s, outs[0]), _rows(s, vf), "clean fwd")
        _close(_rows(s, outs[1]), _rows(s, vr), "clean rev")
        clean = np.concatenate([st, _rows(s, cf)], axis=1)   # row i is token i - (W-1)
        noisy = _rows(s, nf)
        for k in range(s["seqlen"] // T):
            bs = dict(s, seqlen=T)
            prev = clean[:, k * T:k * T + W - 1, :]
            blk = _unrows(bs, noisy[:, k * T:(k + 1) * T, :])
            blk["weight"], blk["bias"] = nf["weight"], nf["bias"]
            one, _, _ = o.conv_prefix(bs, W, True, blk, None, prev)
            _close(_rows(s, outs[2])[:, k * T:(k + 1) * T, :], _rows(bs, one), f"noisy fwd block {k}")
        _close(_rows(s, outs[3]), _correlate_anticausal(_rows(s, nr), nr["weight"], T, True, nr["bias"]),
               "noisy rev")


ALL_CONV_PINS = [pin_correlate_prefix, pin_impulse_response, pin_activation_closed_form, pin_state_out,
                 pin_allblock_noisy_from_clean_rows]
