"""Pins of the oracle's gated RMSNorm (the normalisation of the summed output
before the layer's projection: "Breaking the Bottleneck with DiffuApriel",
section 3.2 after eq. (6), read as the Mamba-2 layer's gated RMSNorm with the
gate applied before the norm) against facts that do not come from its loops:

* the invariant that defines an RMS normalisation: with unit weights and
  eps = 0, every group of every row comes out with root-mean-square exactly 1;
* scale invariance (eps = 0): multiplying a group by a positive constant
  leaves its output unchanged, a negative one flips the sign;
* a closed form for constant groups: y = a everywhere gives a * w / sqrt(a^2 + eps);
* group independence: changing one group of a row leaves the others' outputs
  bit for bit unchanged, and a group's output depends only on its own values;
* gate placement: a constant gate z scales v uniformly by silu(z), so with
  eps = 0 it leaves the output unchanged up to the sign of z (a gate applied
  after the norm would scale it by silu(z)); z = 0 zeroes the output;
* per-channel weights: the output is linear in w, channel by channel.
"""
from __future__ import annotations

import numpy as np
from scipy.special import expit


def _close(a, b, what, tol=1e-12):
    a, b = np.asarray(a), np.asarray(b)
    assert a.shape == b.shape, (what, a.shape, b.shape)
    err = float(np.max(np.abs(a - b))) if a.size else 0.0
    assert err <= tol * max(1.0, float(np.max(np.abs(b))) if b.size else 1.0), f"{what}: max err {err}"


def pin_unit_rms(o):
    rng = np.random.default_rng(1)
    for C, groups in ((32, 1), (48, 3), (64, 16)):
        y = rng.normal(0, 3, (5, C))
        out = o.gated_rmsnorm(y, None, np.ones(C), groups, 0.0)
        gs = C // groups
        rms = np.sqrt((out.reshape(5, groups, gs) ** 2).mean(axis=2))
        _close(rms, np.ones_like(rms), f"unit rms C={C} groups={groups}")


def pin_scale_invariance(o):
    rng = np.random.default_rng(2)
    C, groups = 48, 4
    gs = C // groups
    y = rng.normal(0, 1, (3, C))
    w = rng.normal(0, 1, C)
    base = o.gated_rmsnorm(y, None, w, groups, 0.0)
    scale = np.repeat(rng.choice([-7.0, -0.25, 0.5, 3.0], size=(3, groups)), gs, axis=1)
    out = o.gated_rmsnorm(y * scale, None, w, groups, 0.0)
    _close(out, base * np.sign(scale), "scale invariance")


def pin_constant_closed_form(o):
    C = 16
    w = np.linspace(-2, 2, C)
    for a, eps in ((0.5, 1e-2), (-3.0, 1e-5), (2.0, 0.0), (1e-3, 1e-6)):
        y = np.full((2, C), a)
        out = o.gated_rmsnorm(y, None, w, 2, eps)
        _close(out, np.broadcast_to(a * w / np.sqrt(a * a + eps), (2, C)), f"constant a={a} eps={eps}")


def pin_group_independence(o):
    rng = np.random.default_rng(4)
    C, groups = 60, 5
    gs = C // groups
    y = rng.normal(0, 1, (2, C))
    w = rng.normal(0, 1, C)
    base = o.gated_rmsnorm(y, None, w, groups, 1e-5)
    for g in range(groups):
        y2 = y.copy()
        y2[:, g * gs:(g + 1) * gs] *= rng.normal(0, 2, (2, gs))
        out = o.gated_rmsnorm(y2, None, w, groups, 1e-5)
        keep = np.ones(C, bool)
        keep[g * gs:(g + 1) * gs] = False
        assert np.array_equal(out[:, keep], base[:, keep]), f"group {g} leaked into others"
        # the group alone, normalised as a one-group row, gives the same values
        alone = o.gated_rmsnorm(y2[:, g * gs:(g + 1) * gs], None, w[g * gs:(g + 1) * gs], 1, 1e-5)
        _close(out[:, ~keep], alone, f"group {g} alone")


def pin_gate_before_norm(o):
    rng = np.random.default_rng(5)
    C = 32
    y = rng.normal(0, 1, (4, C))
    w = rng.normal(0, 1, C)
    base = o.gated_rmsnorm(y, None, w, 2, 0.0)
    for zc in (-1.5, 0.3, 4.0):
        # silu(z) = z * sigmoid(z) has the sign of z: a negative gate flips the output
        out = o.gated_rmsnorm(y, np.full((4, C), zc), w, 2, 0.0)
        _close(out, base * np.sign(zc), f"constant gate z={zc}")
    out = o.gated_rmsnorm(y, np.zeros((4, C)), w, 2, 1e-5)
    assert np.all(out == 0.0), "z = 0 must zero the output"
    # a varying gate: v = y * z * expit(z) (scipy), normalised
    z = rng.normal(0, 1, (4, C))
    v = y * z * expit(z)
    out = o.gated_rmsnorm(y, z, np.ones(C), 1, 0.0)
    _close(out, o.gated_rmsnorm(v, None, np.ones(C), 1, 0.0), "gate = scaling by z * sigmoid(z)")


def pin_weight_linearity(o):
    rng = np.random.default_rng(6)
    C = 24
    y = rng.normal(0, 1, (3, C))
    w1, w2 = rng.normal(0, 1, C), rng.normal(0, 1, C)
    a = o.gated_rmsnorm(y, None, w1, 3, 1e-4)
    b = o.gated_rmsnorm(y, None, w2, 3, 1e-4)
    c = o.gated_rmsnorm(y, None, 2 * w1 - w2, 3, 1e-4)
    _close(c, 2 * a - b, "weight linearity")
    one = o.gated_rmsnorm(y, None, np.ones(C), 3, 1e-4)
    _close(a, one * w1, "per-channel weight")


ALL_NORM_PINS = [pin_unit_rms, pin_scale_invariance, pin_constant_closed_form, pin_group_independence,
                 pin_gate_before_norm, pin_weight_linearity]
