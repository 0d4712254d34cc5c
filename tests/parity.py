"""Shared helpers of the GPU-vs-oracle parity tests.

Tolerances (fixed by the workloads' statement): outputs max abs error <= 2e-2
and relative L2 error <= 5e-3; fp32 states relative L2 <= 1e-3 over the whole
tensor and over every block; when y is stored in bf16 the max-abs bound adds
half a bf16 ulp of |ref| (the rounding of the stored value itself).
"""
import numpy as np
import torch

Y_MAX_ABS = 2e-2
Y_REL_L2 = 5e-3
S_REL_L2 = 1e-3


def _np(t):
    return t.detach().to("cpu").to(torch.float64).numpy() if hasattr(t, "detach") else np.asarray(t)


def check_y(got, ref, bf16_out=False, what="y"):
    g, r = _np(got), np.asarray(ref)
    assert g.shape == r.shape, (what, g.shape, r.shape)
    assert np.all(np.isfinite(g)), f"{what}: non-finite values"
    err = np.abs(g - r)
    bound = Y_MAX_ABS + (np.abs(r) * 2.0 ** -9 if bf16_out else 0.0)
    worst = np.max(err - bound) if err.size else -1
    assert worst <= 0, f"{what}: max abs err {np.max(err):.3e} exceeds bound"
    nr = np.linalg.norm(r)
    rel = np.linalg.norm(g - r) / nr if nr > 0 else np.linalg.norm(g - r)
    assert rel <= Y_REL_L2, f"{what}: rel L2 {rel:.3e} > {Y_REL_L2}"
    return float(np.max(err)) if err.size else 0.0, float(rel)


def check_states(got, ref, what="states"):
    g, r = _np(got), np.asarray(ref)
    assert g.shape == r.shape, (what, g.shape, r.shape)
    assert np.all(np.isfinite(g)), f"{what}: non-finite values"
    nr = np.linalg.norm(r)
    rel = np.linalg.norm(g - r) / nr if nr > 0 else np.linalg.norm(g - r)
    assert rel <= S_REL_L2, f"{what}: rel L2 {rel:.3e} > {S_REL_L2}"
    if g.ndim == 5:  # [B, K, H, P, N]: every block
        for k in range(g.shape[1]):
            nk = np.linalg.norm(r[:, k])
            relk = np.linalg.norm(g[:, k] - r[:, k]) / nk if nk > 0 else np.linalg.norm(g[:, k] - r[:, k])
            assert relk <= S_REL_L2, f"{what}: block {k} rel L2 {relk:.3e} > {S_REL_L2}"
    return float(rel)


def heads(d: dict, hs) -> dict:
    """The inputs of a subset of heads (G == 1: B and C are shared)."""
    out = {}
    for k, v in d.items():
        if k in ("A", "D"):
            out[k] = v[hs]
        elif k in ("B", "C"):
            out[k] = v
        else:
            out[k] = v[:, :, hs]
    return out
