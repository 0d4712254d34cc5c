"""Pins of the fp64 oracle against facts that do not come from the oracle itself.

Each ``pin_*`` function takes an oracle handle (the ``oracle`` package or an
``oracle.Variant`` built from an edited copy of its source) and raises
AssertionError when the handle disagrees with an independent statement of the
scan:

* closed forms (zero decay -> cumulative sums; linear time-invariant special
  case -> a direct convolution via ``numpy.convolve``; a single token),
* exact rational arithmetic on a small worked example (decay exactly 1/2),
* brute force on tiny inputs (the unrolled recurrence with explicit products)
  and the chunked/quadratic form that the device kernels compute,
* invariants the pages state: continuation of a cached state equals one scan,
  the reverse scan is the forward scan of the flipped block, the cached
  boundary state depends on the clean prefix only, superposition in h0, and
  the all-block noisy stream with noisy == clean reproduces the clean stream.

The equations are those of "Training Hybrid Block Diffusion Language Models
with Partial Bidirectionality", eqs. (1) and (10)-(14), and "Breaking the
Bottleneck with DiffuApriel", section 3.2 eqs. (4)-(6).
"""
from __future__ import annotations

import json
import os
from fractions import Fraction

import numpy as np
import torch

from bidirectional_mamba_state_b200 import workload as W

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _np(d):
    return {k: v.double().numpy() for k, v in d.items()}


def _close(a, b, rtol=1e-11, atol=1e-12, what=""):
    a = np.asarray(a)
    b = np.asarray(b)
    assert a.shape == b.shape, (what, a.shape, b.shape)
    err = np.max(np.abs(a - b)) if a.size else 0.0
    lim = atol + rtol * (np.max(np.abs(b)) if b.size else 0.0)
    assert err <= lim, f"{what}: max abs err {err:.3e} > {lim:.3e}"


def _shape(**kw):
    base = dict(batch=2, seqlen=64, nheads=4, headdim=8, dstate=16, ngroups=2, block_len=16,
                chunk_len=16, in_dtype="fp32")
    base.update(kw)
    return W.Shape(**base)


def _gidx(h, H, G):
    return h // (H // G)


# --------------------------------------------------------------------------- closed forms
def pin_zero_decay_cumsum(orc):
    """A = 0: h_t = sum_{s<=t} dt_s x_s B_s^T (a cumulative sum); the reverse
    direction gives suffix sums inside each block; y = y_fwd + y_rev."""
    s = _shape()
    f = W.make_dir(s, 11, 0, W.CLEAN_FWD, ssm_zero_decay=True)
    r = W.make_dir(s, 11, 0, W.CLEAN_REV, ssm_zero_decay=True)
    h0 = W.make_state(s, 11, scale=0.5)
    y, st, fin = orc.prefix(s.as_dict(), f, r, h0=h0)
    F, R = _np(f), _np(r)
    B, L, H, P, N, G, T = s.batch, s.seqlen, s.nheads, s.headdim, s.dstate, s.ngroups, s.block_len
    ref = np.zeros((B, L, H, P))
    ref_states = np.zeros((B, L // T, H, P, N))
    for b in range(B):
        for h in range(H):
            g = _gidx(h, H, G)
            # forward: cumulative sum of the rank-1 inputs, plus the constant h0
            inc = F["dt"][b, :, h, None, None] * F["x"][b, :, h, :, None] * F["B"][b, :, g, None, :]
            hs = np.cumsum(inc, axis=0) + h0[b, h].double().numpy()[None]
            ref[b, :, h] = np.einsum("tpn,tn->tp", hs, F["C"][b, :, g]) + F["D"][h] * F["x"][b, :, h]
            ref_states[b, :, h] = hs[T - 1::T]
            # reverse: suffix sums inside each block
            incr = R["dt"][b, :, h, None, None] * R["x"][b, :, h, :, None] * R["B"][b, :, g, None, :]
            for k in range(L // T):
                blk = incr[k * T:(k + 1) * T]
                suff = np.cumsum(blk[::-1], axis=0)[::-1]
                ref[b, k * T:(k + 1) * T, h] += (np.einsum("tpn,tn->tp", suff, R["C"][b, k * T:(k + 1) * T, g])
                                                 + R["D"][h] * R["x"][b, k * T:(k + 1) * T, h])
    _close(y, ref, what="A=0 outputs")
    _close(st, ref_states, what="A=0 states")
    _close(fin, ref_states[:, -1], what="A=0 final state")


def _lti_dir(s, seed, stream):
    """Constant dt, B, C along the sequence -> a linear time-invariant system."""
    d = W.make_dir(s, seed, 0, stream)
    for key in ("dt", "B", "C"):
        v = d[key]
        d[key] = v[:, :1].expand_as(v).contiguous()
    return d


def pin_lti_convolution(orc):
    """Constant dt, B, C: the forward output is a causal convolution of x with the
    kernel k_j = dt (C.B) a^j, a = exp(dt A); the reverse output is the
    anti-causal convolution restricted to each block.  Checked with numpy.convolve."""
    s = _shape(batch=1, seqlen=48, nheads=2, headdim=3, dstate=5, ngroups=1, block_len=16)
    f, r = _lti_dir(s, 5, W.CLEAN_FWD), _lti_dir(s, 5, W.CLEAN_REV)
    y, _, _ = orc.prefix(s.as_dict(), f, r)
    F, R = _np(f), _np(r)
    L, T = s.seqlen, s.block_len
    ref = np.zeros_like(y)
    for h in range(s.nheads):
        dt, a = F["dt"][0, 0, h], np.exp(F["dt"][0, 0, h] * F["A"][h])
        cb = float(np.dot(F["C"][0, 0, 0], F["B"][0, 0, 0]))
        kern = dt * cb * a ** np.arange(L)
        dtr, ar = R["dt"][0, 0, h], np.exp(R["dt"][0, 0, h] * R["A"][h])
        cbr = float(np.dot(R["C"][0, 0, 0], R["B"][0, 0, 0]))
        kernr = dtr * cbr * ar ** np.arange(T)
        for p in range(s.headdim):
            xf = F["x"][0, :, h, p]
            ref[0, :, h, p] = np.convolve(xf, kern)[:L] + F["D"][h] * xf
            xr = R["x"][0, :, h, p]
            for k in range(L // T):
                blk = xr[k * T:(k + 1) * T][::-1]
                ref[0, k * T:(k + 1) * T, h, p] += (np.convolve(blk, kernr)[:T][::-1]
                                                   + R["D"][h] * xr[k * T:(k + 1) * T])
    _close(y, ref, what="LTI convolution")


def pin_single_token(orc):
    """L = T = 1: y = dt (C.B) x + D x for each direction, summed; the boundary
    state is dt x B^T (+ a h0)."""
    s = _shape(batch=3, seqlen=1, nheads=4, headdim=5, dstate=7, ngroups=2, block_len=1)
    f, r = W.make_dir(s, 3, 0, W.CLEAN_FWD), W.make_dir(s, 3, 0, W.CLEAN_REV)
    h0 = W.make_state(s, 3)
    y, st, _ = orc.prefix(s.as_dict(), f, r, h0=h0)
    F, R, H0 = _np(f), _np(r), h0.double().numpy()
    ref = np.zeros_like(y)
    ref_st = np.zeros_like(st)
    for b in range(s.batch):
        for h in range(s.nheads):
            g = _gidx(h, s.nheads, s.ngroups)
            for d, init in ((F, H0[b, h]), (R, 0.0 * H0[b, h])):
                dt, x = d["dt"][b, 0, h], d["x"][b, 0, h]
                a = np.exp(dt * d["A"][h])
                hs = a * init + dt * np.outer(x, d["B"][b, 0, g])
                ref[b, 0, h] += hs @ d["C"][b, 0, g] + d["D"][h] * x
                if d is F:
                    ref_st[b, 0, h] = hs
    _close(y, ref, what="single token")
    _close(st, ref_st, what="single-token state")


# --------------------------------------------------------------------------- exact worked example
def _worked_inputs():
    with open(os.path.join(GOLDEN, "worked_example.json")) as fh:
        return json.load(fh)


def _frac_scan(ex, direction, h0):
    """Exact rational evaluation of eq. (1) for one head (P = N = 2), decay 1/2."""
    d = ex[direction]
    L, P, N = len(d["x"]), 2, 2
    a = Fraction(1, 2)
    ys = []
    hs = [[Fraction(v) for v in row] for row in h0]
    order = range(L) if direction == "fwd" else range(L - 1, -1, -1)
    out = [None] * L
    for t in order:
        dt = Fraction(d["dt"][t])
        x = [Fraction(v) for v in d["x"][t]]
        Bt = [Fraction(v) for v in d["B"][t]]
        Ct = [Fraction(v) for v in d["C"][t]]
        hs = [[a * hs[p][n] + dt * x[p] * Bt[n] for n in range(N)] for p in range(P)]
        out[t] = [sum(Ct[n] * hs[p][n] for n in range(N)) + Fraction(d["D"]) * x[p] for p in range(P)]
    return out, hs


def pin_worked_example(orc):
    """A 4-token, two-block example with P = N = 2 whose per-token decay is exactly
    1/2 (dt = 1/2, A = -2 ln 2), evaluated in exact rational arithmetic and
    compared with the oracle and with the stored oracle output."""
    ex = _worked_inputs()
    T = ex["block_len"]
    L = len(ex["fwd"]["x"])
    shape = dict(batch=1, seqlen=L, nheads=1, headdim=2, dstate=2, ngroups=1, block_len=T)

    def as_dir(d):
        return {"x": np.array(d["x"], float).reshape(1, L, 1, 2),
                "dt": np.array(d["dt"], float).reshape(1, L, 1),
                "B": np.array(d["B"], float).reshape(1, L, 1, 2),
                "C": np.array(d["C"], float).reshape(1, L, 1, 2),
                "A": np.array([d["A"]], float), "D": np.array([d["D"]], float)}

    h0 = np.array(ex["h0"], float).reshape(1, 1, 2, 2)
    y, st, fin = orc.prefix(shape, as_dir(ex["fwd"]), as_dir(ex["rev"]), h0=h0)
    yf, hf = _frac_scan(ex, "fwd", ex["h0"])
    exact = [[float(v) for v in row] for row in yf]
    states_exact = []
    hs = [[Fraction(v) for v in row] for row in ex["h0"]]
    # boundary states: forward state after each block
    for k in range(L // T):
        sub = dict(ex)
        sub_f = {key: (val[:(k + 1) * T] if isinstance(val, list) else val)
                 for key, val in ex["fwd"].items()}
        _, hk = _frac_scan({"fwd": sub_f}, "fwd", ex["h0"])
        states_exact.append([[float(v) for v in row] for row in hk])
    for k in range(L // T):
        sub_r = {key: (val[k * T:(k + 1) * T] if isinstance(val, list) else val)
                 for key, val in ex["rev"].items()}
        yr, _ = _frac_scan({"rev": sub_r}, "rev", [[0, 0], [0, 0]])
        for j in range(T):
            exact[k * T + j] = [exact[k * T + j][p] + float(yr[j][p]) for p in range(2)]
    _close(y.reshape(L, 2), np.array(exact), rtol=1e-13, what="worked example y")
    _close(st.reshape(L // T, 2, 2), np.array(states_exact), rtol=1e-13, what="worked example states")
    _close(fin.reshape(2, 2), np.array(states_exact[-1]), rtol=1e-13, what="worked example final")
    stored = ex["oracle_output"]
    _close(np.array(stored["y"]), y.reshape(L, 2), rtol=1e-14, what="stored oracle output")


# --------------------------------------------------------------------------- brute force
def _bruteforce_prefix(s, F, R, H0):
    """Unrolled recurrence: y_t = sum_{s<=t} (C_t.B_s) dt_s prod_{u=s+1..t} a_u x_s
    + prod_{u=0..t} a_u C_t.h0 + D x_t, with every product formed explicitly."""
    B, L, H, P, N, G, T = s.batch, s.seqlen, s.nheads, s.headdim, s.dstate, s.ngroups, s.block_len
    y = np.zeros((B, L, H, P))
    for b in range(B):
        for h in range(H):
            g = _gidx(h, H, G)
            a = np.exp(F["dt"][b, :, h] * F["A"][h])
            ar = np.exp(R["dt"][b, :, h] * R["A"][h])
            for t in range(L):
                acc = F["D"][h] * F["x"][b, t, h].copy()
                decay0 = np.prod(a[:t + 1])
                acc += decay0 * (H0[b, h] @ F["C"][b, t, g])
                for u in range(t + 1):
                    w = np.prod(a[u + 1:t + 1]) * F["dt"][b, u, h] * np.dot(F["C"][b, t, g], F["B"][b, u, g])
                    acc += w * F["x"][b, u, h]
                k0 = (t // T) * T
                acc += R["D"][h] * R["x"][b, t, h]
                for u in range(t, k0 + T):
                    w = np.prod(ar[t:u]) * R["dt"][b, u, h] * np.dot(R["C"][b, t, g], R["B"][b, u, g])
                    acc += w * R["x"][b, u, h]
                y[b, t, h] = acc
    return y


def pin_bruteforce(orc):
    """Tiny shapes with H = 4, G = 2 (head-to-group mapping), P != N (orientation)."""
    s = _shape(batch=2, seqlen=12, nheads=4, headdim=3, dstate=5, ngroups=2, block_len=4)
    f, r = W.make_dir(s, 7, 0, W.CLEAN_FWD), W.make_dir(s, 7, 0, W.CLEAN_REV)
    h0 = W.make_state(s, 7)
    y, _, _ = orc.prefix(s.as_dict(), f, r, h0=h0)
    ref = _bruteforce_prefix(s, _np(f), _np(r), h0.double().numpy())
    _close(y, ref, what="brute force")


def _chunked_prefix(s, F, R, H0, Q):
    """The chunked (state-space-duality) form the device kernels compute:
    within a chunk of Q tokens, cum_t = sum_{u in chunk, u<=t} dt_u A,
      y_t = exp(cum_t) C_t.h_start + sum_{s<=t in chunk} (C_t.B_s) exp(cum_t-cum_s) dt_s x_s
      h_end = exp(cum_end) h_start + sum_s exp(cum_end - cum_s) dt_s x_s B_s^T,
    and the block-local reverse as the same quadratic form on the reversed block."""
    B, L, H, P, N, G, T = s.batch, s.seqlen, s.nheads, s.headdim, s.dstate, s.ngroups, s.block_len
    y = np.zeros((B, L, H, P))
    states = np.zeros((B, L // T, H, P, N))
    for b in range(B):
        for h in range(H):
            g = _gidx(h, H, G)
            hs = H0[b, h].copy()
            for c0 in range(0, L, Q):
                sl = slice(c0, c0 + Q)
                dA = F["dt"][b, sl, h] * F["A"][h]
                cum = np.cumsum(dA)
                Cc, Bc, Xc, dtc = F["C"][b, sl, g], F["B"][b, sl, g], F["x"][b, sl, h], F["dt"][b, sl, h]
                mask = np.tril(np.ones((Q, Q)))
                Lmat = np.exp((cum[:, None] - cum[None, :]) * mask) * mask
                M = (Cc @ Bc.T) * Lmat * dtc[None, :]
                y[b, sl, h] = M @ Xc + np.exp(cum)[:, None] * (Cc @ hs.T) + F["D"][h] * Xc
                for j in range(T - 1, Q, T):  # boundary states inside the chunk
                    w = np.exp(cum[j] - cum[:j + 1]) * dtc[:j + 1]
                    states[b, (c0 + j) // T, h] = np.exp(cum[j]) * hs + (Xc[:j + 1] * w[:, None]).T @ Bc[:j + 1]
                hs = states[b, (c0 + Q - 1) // T, h].copy()
            for k0 in range(0, L, T):
                sl = slice(k0, k0 + T)
                dA = (R["dt"][b, sl, h] * R["A"][h])[::-1]
                cum = np.cumsum(dA)
                Cc, Bc = R["C"][b, sl, g][::-1], R["B"][b, sl, g][::-1]
                Xc, dtc = R["x"][b, sl, h][::-1], R["dt"][b, sl, h][::-1]
                mask = np.tril(np.ones((T, T)))
                M = (Cc @ Bc.T) * np.exp((cum[:, None] - cum[None, :]) * mask) * mask * dtc[None, :]
                y[b, sl, h] += (M @ Xc + R["D"][h] * Xc)[::-1]
    return y, states


def pin_chunked_form(orc):
    """The chunked form with chunk Q = T and Q = 2T equals the sequential oracle."""
    s = _shape(batch=2, seqlen=32, nheads=4, headdim=4, dstate=6, ngroups=2, block_len=8)
    f, r = W.make_dir(s, 9, 0, W.CLEAN_FWD), W.make_dir(s, 9, 0, W.CLEAN_REV)
    h0 = W.make_state(s, 9)
    y, st, _ = orc.prefix(s.as_dict(), f, r, h0=h0)
    for Q in (8, 16):
        yc, sc = _chunked_prefix(s, _np(f), _np(r), h0.double().numpy(), Q)
        _close(y, yc, what=f"chunked y Q={Q}")
        _close(st, sc, what=f"chunked states Q={Q}")


# --------------------------------------------------------------------------- invariants
def pin_superposition(orc):
    """y(h0) - y(0) = exp(cum_t) C_t.h0 and states[k](h0) - states[k](0) =
    exp(cum_end(k)) h0, with cum_t = sum_{u<=t} dt_u A (linearity in the state)."""
    s = _shape(batch=2, seqlen=48, nheads=4, headdim=6, dstate=8, ngroups=2, block_len=16)
    f, r = W.make_dir(s, 13, 0, W.CLEAN_FWD), W.make_dir(s, 13, 0, W.CLEAN_REV)
    h0 = W.make_state(s, 13)
    y1, s1, _ = orc.prefix(s.as_dict(), f, r, h0=h0)
    y0, s0, _ = orc.prefix(s.as_dict(), f, r, h0=None)
    F, H0 = _np(f), h0.double().numpy()
    T = s.block_len
    for b in range(s.batch):
        for h in range(s.nheads):
            g = _gidx(h, s.nheads, s.ngroups)
            cum = np.cumsum(F["dt"][b, :, h] * F["A"][h])
            dy = np.exp(cum)[:, None] * (F["C"][b, :, g] @ H0[b, h].T)
            _close(y1[b, :, h] - y0[b, :, h], dy, rtol=1e-9, atol=1e-11, what="superposition y")
            ds = np.exp(cum[T - 1::T])[:, None, None] * H0[b, h][None]
            _close(s1[b, :, h] - s0[b, :, h], ds, rtol=1e-9, atol=1e-11, what="superposition states")


def pin_continuation(orc):
    """Scanning the prefix, then the last block from the cached final state
    (block_step, with its own block-local reverse), equals one prefix scan over
    the whole sequence on that block; the committed state equals the final
    boundary state."""
    s = _shape(batch=2, seqlen=64, nheads=4, headdim=8, dstate=16, ngroups=2, block_len=16)
    f, r = W.make_dir(s, 17, 0, W.CLEAN_FWD), W.make_dir(s, 17, 0, W.CLEAN_REV)
    h0 = W.make_state(s, 17)
    y, st, fin = orc.prefix(s.as_dict(), f, r, h0=h0)
    T, L = s.block_len, s.seqlen
    sp = s.with_(seqlen=L - T)
    _, _, fin_p = orc.prefix(sp.as_dict(), W.sub_batch_block(f, 0, L - T),
                             W.sub_batch_block(r, 0, L - T), h0=h0)
    _close(fin_p, st[:, -2], what="prefix final == boundary state")
    sb = s.with_(seqlen=T)
    yb, so = orc.block_step(sb.as_dict(), W.sub_batch_block(f, L - T, L),
                            W.sub_batch_block(r, L - T, L), fin_p, want_state_out=True)
    _close(yb, y[:, L - T:], what="continuation y")
    _close(so, fin, what="committed state")


def pin_reverse_is_flipped_forward(orc):
    """Reverse part of a block == flip(forward scan of the flipped block from 0)."""
    s = _shape(batch=2, seqlen=32, nheads=4, headdim=5, dstate=6, ngroups=2, block_len=8)
    f, r = W.make_dir(s, 19, 0, W.CLEAN_FWD), W.make_dir(s, 19, 0, W.CLEAN_REV)
    y_both, _, _ = orc.prefix(s.as_dict(), f, r)
    y_fwd, _, _ = orc.prefix(s.as_dict(), f, None)
    y_rev = y_both - y_fwd
    T = s.block_len
    for k in range(s.seqlen // T):
        blk = W.sub_batch_block(r, k * T, (k + 1) * T)
        flipped = {key: (v.flip(1).contiguous() if key not in ("A", "D") else v) for key, v in blk.items()}
        yf, _, _ = orc.prefix(s.with_(seqlen=T).as_dict(), flipped, None)
        _close(y_rev[:, k * T:(k + 1) * T], yf[:, ::-1], rtol=1e-10, what=f"reverse block {k}")


def pin_cache_independence(orc):
    """Boundary states depend on the clean prefix only: a perturbation of clean x
    at token j changes exactly states[k] for k >= j // T (bitwise equal before);
    changing the noisy stream or the reverse direction changes no state bit."""
    s = _shape(batch=1, seqlen=64, nheads=4, headdim=4, dstate=8, ngroups=2, block_len=16)
    cf, cr, nf, nr = W.make_streams(s, 23)
    _, _, st = orc.allblock(s.as_dict(), cf, cr, nf, nr, want_clean=False)
    T = s.block_len
    for j in (0, 17, 40, 63):
        cf2 = {k: v.clone() for k, v in cf.items()}
        cf2["x"][0, j] += 1.0
        _, _, st2 = orc.allblock(s.as_dict(), cf2, cr, nf, nr, want_clean=False)
        kb = j // T
        assert np.array_equal(st2[:, :kb], st[:, :kb]), f"states before block {kb} changed (j={j})"
        for k in range(kb, s.seqlen // T):
            assert not np.array_equal(st2[:, k], st[:, k]), f"state {k} did not change (j={j})"
    nf2 = W.make_dir(s, 99, 0, W.NOISY_FWD)
    nr2 = W.make_dir(s, 99, 0, W.NOISY_REV)
    cr2 = W.make_dir(s, 99, 0, W.CLEAN_REV)
    _, _, st3 = orc.allblock(s.as_dict(), cf, cr2, nf2, nr2, want_clean=False)
    assert np.array_equal(st3, st), "states depend on the noisy stream or reverse direction"


def pin_allblock_noisy_equals_clean(orc):
    """With the noisy stream equal to the clean stream, every noisy block resumes
    from the state the clean scan had there, so y_noisy == y_clean; and each
    noisy block equals a block_step from states[k-1]."""
    s = _shape(batch=2, seqlen=48, nheads=4, headdim=4, dstate=8, ngroups=2, block_len=16)
    cf, cr, nf, nr = W.make_streams(s, 29)
    h0 = W.make_state(s, 29)
    yc, yn, st = orc.allblock(s.as_dict(), cf, cr, cf, cr, h0=h0)
    _close(yn, yc, rtol=1e-13, what="noisy == clean")
    yc2, yn2, _ = orc.allblock(s.as_dict(), cf, cr, nf, nr, h0=h0)
    T = s.block_len
    sb = s.with_(seqlen=T)
    for k in range(s.seqlen // T):
        init = h0 if k == 0 else st[:, k - 1]
        yb, _ = orc.block_step(sb.as_dict(), W.sub_batch_block(nf, k * T, (k + 1) * T),
                               W.sub_batch_block(nr, k * T, (k + 1) * T), init)
        _close(yn2[:, k * T:(k + 1) * T], yb, rtol=1e-13, what=f"noisy block {k}")
    _close(yc2, yc, rtol=0, atol=0, what="clean output independent of the noisy stream")


def pin_gate(orc):
    """Gate: each direction's output is multiplied by silu(z_dir) before the sum;
    checked against the ungated oracle on the forward-only path with z constant
    per (b,t,h,p)."""
    s = _shape(batch=1, seqlen=16, nheads=2, headdim=3, dstate=4, ngroups=1, block_len=8)
    f = W.make_dir(s, 31, 0, W.CLEAN_FWD, gated=True)
    r = W.make_dir(s, 31, 0, W.CLEAN_REV, gated=True)
    y, _, _ = orc.prefix(s.as_dict(), f, r)
    fu = {k: v for k, v in f.items() if k != "z"}
    ru = {k: v for k, v in r.items() if k != "z"}
    yf, _, _ = orc.prefix(s.as_dict(), fu, None)
    yb, _, _ = orc.prefix(s.as_dict(), fu, ru)
    yr = yb - yf
    zf, zr = f["z"].double().numpy(), r["z"].double().numpy()
    silu = lambda v: v / (1.0 + np.exp(-v))
    _close(y, yf * silu(zf) + yr * silu(zr), rtol=1e-12, what="gate")


ALL_PINS = [pin_zero_decay_cumsum, pin_lti_convolution, pin_single_token, pin_worked_example,
            pin_bruteforce, pin_chunked_form, pin_superposition, pin_continuation,
            pin_reverse_is_flipped_forward, pin_cache_independence,
            pin_allblock_noisy_equals_clean, pin_gate]
