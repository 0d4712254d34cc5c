"""Device backward of the all-block pass (bdscan_allblock_backward) against the
fp64 oracle's reverse-mode derivative, on the same seeded inputs."""
import numpy as np
import pytest
import torch

import oracle
from bidirectional_mamba_state_b200 import bdscan as bd
from bidirectional_mamba_state_b200 import workload as W

pytestmark = pytest.mark.gpu
DEV = "cuda:0"
KEYS = ("x", "dt", "B", "C", "A", "D")


def _shape(**kw):
    d = dict(batch=2, seqlen=96, nheads=4, headdim=64, dstate=128, ngroups=2, block_len=32,
             chunk_len=32, in_dtype="bf16", out_dtype="fp32")
    d.update(kw)
    return W.Shape(**d)


def _rel_l2(a, r):
    n = np.linalg.norm(r)
    return float(np.linalg.norm(a - r) / n) if n > 0 else float(np.linalg.norm(a))


def _check(dev_t, ref, what, rtol=1e-4):
    a = dev_t.detach().double().cpu().numpy()
    assert a.shape == ref.shape, (what, a.shape, ref.shape)
    scale = float(np.max(np.abs(ref))) if ref.size else 0.0
    err = float(np.max(np.abs(a - ref))) if ref.size else 0.0
    assert err <= 1e-3 * scale + 1e-6, f"{what}: max abs err {err:.3e} (scale {scale:.3e})"
    assert _rel_l2(a, ref) <= rtol, f"{what}: rel L2 {_rel_l2(a, ref):.3e}"


def _run(s, with_rev=True, with_h0=True, with_dyc=True, with_dst=True, seed=5):
    cf, cr, nf, nr = W.make_streams(s, seed, device=DEV)
    if not with_rev:
        cr = nr = None
    h0 = W.make_state(s, seed, device=DEV) if with_h0 else None
    yc, yn, st = bd.allblock(s, cf, cr, nf, nr, h0=h0)
    g = torch.Generator(device=DEV).manual_seed(seed + 17)
    tout = yn.dtype
    dyn = torch.randn(yn.shape, generator=g, device=DEV).to(tout)
    dyc = torch.randn(yn.shape, generator=g, device=DEV).to(tout) if with_dyc else None
    dst = torch.randn(st.shape, generator=g, device=DEV) * 0.1 if with_dst else None
    grads, dh0 = bd.allblock_backward(s, cf, cr, nf, nr, st, dyn, dy_clean=dyc, dstates=dst, h0=h0)
    torch.cuda.synchronize()
    ref, ref_dh0 = oracle.allblock_backward(s.as_dict(), cf, cr, nf, nr, h0=h0, dy_clean=dyc,
                                            dy_noisy=dyn, dstates=dst)
    names = ["clean fwd", "clean rev", "noisy fwd", "noisy rev"]
    for i in range(4):
        if ref[i] is None:
            assert grads[i] is None
            continue
        for k in KEYS:
            _check(grads[i][k], ref[i][k], f"{names[i]} d{k}")
    _check(dh0, ref_dh0, "dh0")


SHAPES = {
    "bf16_g2": _shape(),
    "fp32_in_bf16_out": _shape(in_dtype="fp32", out_dtype="bf16", seqlen=64),
    "bf16_in_bf16_out": _shape(out_dtype="bf16", seqlen=64),  # bf16 dy through the 16-byte loads
    "p16_n48_t16": _shape(headdim=16, dstate=48, block_len=16, chunk_len=16, seqlen=80, nheads=6, ngroups=3),
    "one_block": _shape(seqlen=32, batch=3),
}


@pytest.mark.parametrize("name", sorted(SHAPES))
def test_backward_parity(name):
    _run(SHAPES[name])


def test_backward_forward_only_no_h0_no_dy_clean():
    _run(_shape(), with_rev=False, with_h0=False, with_dyc=False, with_dst=False)


def test_backward_deterministic_bitwise():
    s = _shape()
    cf, cr, nf, nr = W.make_streams(s, 9, device=DEV)
    _, yn, st = bd.allblock(s, cf, cr, nf, nr)
    dyn = torch.randn(yn.shape, device=DEV)
    a, da = bd.allblock_backward(s, cf, cr, nf, nr, st, dyn)
    b, db = bd.allblock_backward(s, cf, cr, nf, nr, st, dyn)
    torch.cuda.synchronize()
    for i in range(4):
        for k in KEYS:
            assert torch.equal(a[i][k], b[i][k]), (i, k)
    assert torch.equal(da, db)


def test_backward_87m_shape_two_rows():
    # the 87M all-block layer's per-sequence shape (1024 tokens, 24 heads x 64,
    # d_state 128, one group), two batch rows
    s = W.WORKLOADS["87m_allblock"].with_(batch=2)
    _run(s, seed=1)


def test_backward_rejects_gated():
    s = _shape()
    cf, cr, nf, nr = W.make_streams(s, 3, device=DEV, gated=True)
    _, yn, st = bd.allblock(s, cf, cr, nf, nr)
    with pytest.raises(bd.BdscanError):
        bd.allblock_backward(s, cf, cr, nf, nr, st, torch.zeros_like(yn))
