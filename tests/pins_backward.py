"""Pins of the oracle's backward pass (the reverse-mode derivative of the
all-block pass) against facts that do not come from its own arithmetic:

* central finite differences of the oracle's FORWARD pass (itself pinned by
  ``pins.py``), element by element, in double precision;
* linearity: the gradient is linear in the output gradients (dy_clean,
  dy_noisy, dstates), so the gradient of a sum of losses is the sum;
* the clean-only special case: with no output gradient on the noisy stream or
  the states, the noisy directions get zero gradients.

The loss is L = <wc, y_clean> + <wn, y_noisy> + <ws, states> for fixed random
weights, so dL/dy_clean = wc, dL/dy_noisy = wn and dL/dstates = ws.  The
forward it differentiates is "Training Hybrid Block Diffusion Language Models
with Partial Bidirectionality", eq. (1) with eqs. (10)-(14).
"""
from __future__ import annotations

import numpy as np

KEYS = ("x", "dt", "B", "C", "A", "D")


def _shape(**kw):
    s = dict(batch=2, seqlen=8, nheads=4, headdim=3, dstate=2, ngroups=2, block_len=4)
    s.update(kw)
    return s


def _inputs(s, seed, with_rev=True, with_h0=True):
    rng = np.random.default_rng(seed)
    B, L, H, P, N, G = (s[k] for k in ("batch", "seqlen", "nheads", "headdim", "dstate", "ngroups"))

    def direction():
        return {"x": rng.normal(0, 1, (B, L, H, P)),
                "dt": np.log1p(np.exp(rng.normal(-1.0, 0.5, (B, L, H)))),
                "B": rng.normal(0, 0.5, (B, L, G, N)), "C": rng.normal(0, 0.5, (B, L, G, N)),
                "A": -np.exp(rng.uniform(0, np.log(4.0), (H,))), "D": rng.normal(0, 1, (H,))}

    dirs = [direction(), direction() if with_rev else None, direction(), direction() if with_rev else None]
    h0 = rng.normal(0, 1, (B, H, P, N)) if with_h0 else None
    K = L // s["block_len"]
    w = (rng.normal(0, 1, (B, L, H, P)), rng.normal(0, 1, (B, L, H, P)), rng.normal(0, 1, (B, K, H, P, N)))
    return dirs, h0, w


def _loss(orc, s, dirs, h0, w, terms=(True, True, True)):
    yc, yn, st = orc.allblock(s, dirs[0], dirs[1], dirs[2], dirs[3], h0=h0)
    out = 0.0
    if terms[0]:
        out += float(np.sum(w[0] * yc))
    if terms[1]:
        out += float(np.sum(w[1] * yn))
    if terms[2]:
        out += float(np.sum(w[2] * st))
    return out


def _fd_check(orc, s, dirs, h0, w, grads, dh0, per_tensor, seed, eps=1e-5, tol=2e-7):
    rng = np.random.default_rng(seed + 1000)
    checked = 0
    for di, d in enumerate(dirs):
        if d is None:
            continue
        for key in KEYS:
            arr = d[key]
            flat = arr.reshape(-1)
            idx = range(flat.size) if flat.size <= per_tensor else rng.choice(flat.size, per_tensor, replace=False)
            for i in idx:
                old = flat[i]
                flat[i] = old + eps
                fp = _loss(orc, s, dirs, h0, w)
                flat[i] = old - eps
                fm = _loss(orc, s, dirs, h0, w)
                flat[i] = old
                num = (fp - fm) / (2 * eps)
                ana = grads[di][key].reshape(-1)[i]
                assert abs(num - ana) <= tol * (1.0 + abs(num)), \
                    f"direction {di} d{key}[{i}]: analytic {ana:.10e} vs finite difference {num:.10e}"
                checked += 1
    if h0 is not None:
        flat = h0.reshape(-1)
        for i in range(flat.size):
            old = flat[i]
            flat[i] = old + eps
            fp = _loss(orc, s, dirs, h0, w)
            flat[i] = old - eps
            fm = _loss(orc, s, dirs, h0, w)
            flat[i] = old
            num = (fp - fm) / (2 * eps)
            ana = dh0.reshape(-1)[i]
            assert abs(num - ana) <= tol * (1.0 + abs(num)), f"dh0[{i}]: {ana:.10e} vs {num:.10e}"
            checked += 1
    assert checked > 0


def pin_backward_finite_differences(orc):
    s = _shape()
    dirs, h0, w = _inputs(s, 11)
    grads, dh0 = orc.allblock_backward(s, dirs[0], dirs[1], dirs[2], dirs[3], h0=h0,
                                       dy_clean=w[0], dy_noisy=w[1], dstates=w[2])
    _fd_check(orc, s, dirs, h0, w, grads, dh0, per_tensor=12, seed=11)


def pin_backward_finite_differences_forward_only(orc):
    # no reverse directions, no h0, three blocks, one head per group
    s = _shape(seqlen=12, nheads=2, ngroups=2, headdim=2, dstate=3)
    dirs, h0, w = _inputs(s, 12, with_rev=False, with_h0=False)
    grads, dh0 = orc.allblock_backward(s, dirs[0], None, dirs[2], None, h0=None,
                                       dy_clean=w[0], dy_noisy=w[1], dstates=w[2])
    assert grads[1] is None and grads[3] is None
    _fd_check(orc, s, dirs, None, w, grads, dh0, per_tensor=10, seed=12)


def pin_backward_linearity(orc):
    s = _shape()
    dirs, h0, w = _inputs(s, 13)
    full, dh_full = orc.allblock_backward(s, *dirs, h0=h0, dy_clean=w[0], dy_noisy=w[1], dstates=w[2])
    parts = [orc.allblock_backward(s, *dirs, h0=h0, dy_clean=w[0], dy_noisy=np.zeros_like(w[1])),
             orc.allblock_backward(s, *dirs, h0=h0, dy_clean=None, dy_noisy=w[1]),
             orc.allblock_backward(s, *dirs, h0=h0, dy_clean=None, dy_noisy=np.zeros_like(w[1]), dstates=w[2])]
    for di in range(4):
        for key in KEYS:
            tot = sum(p[0][di][key] for p in parts)
            assert np.allclose(tot, full[di][key], rtol=1e-12, atol=1e-12), (di, key)
    assert np.allclose(sum(p[1] for p in parts), dh_full, rtol=1e-12, atol=1e-12)


def pin_backward_clean_only(orc):
    s = _shape()
    dirs, h0, w = _inputs(s, 14)
    grads, _ = orc.allblock_backward(s, *dirs, h0=h0, dy_clean=w[0], dy_noisy=np.zeros_like(w[1]))
    for di in (2, 3):
        for key in KEYS:
            assert np.all(grads[di][key] == 0.0), (di, key)


ALL_BACKWARD_PINS = [pin_backward_finite_differences, pin_backward_finite_differences_forward_only,
                     pin_backward_linearity, pin_backward_clean_only]
