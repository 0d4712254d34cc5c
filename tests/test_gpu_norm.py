"""Device gated RMSNorm (bdscan_gated_rmsnorm) against the fp64 oracle, element
by element, on the same seeded inputs.

Tolerance, from the arithmetic: v = y * silu(z) in fp32 (a few ulp per
element), per-vector sums of squares and a group sum of gs terms in fp32
(relative error at most about gs * 2^-24 <= 3.1e-4 for 5120 channels, far
less in practice), one square root and division (1 ulp each), then one
rounding to bf16 (half an ulp: at most 2^-8 relative).  So
|device - oracle| <= (2^-8 + 4e-4) * |oracle| + 1e-6 * max |oracle|."""
import numpy as np
import pytest
import torch

import oracle
from bidirectional_mamba_state_b200 import bdscan as bd
from bidirectional_mamba_state_b200 import workload as W

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def _shape(**kw):
    d = dict(batch=2, seqlen=64, nheads=24, headdim=64, dstate=128, ngroups=1, block_len=32,
             chunk_len=32, in_dtype="bf16", out_dtype="fp32")
    d.update(kw)
    return W.Shape(**d)


def _inputs(s, seed, gated):
    g = torch.Generator(device=DEV).manual_seed(seed)
    tout = torch.bfloat16 if s.out_dtype == "bf16" else torch.float32
    tin = torch.bfloat16 if s.in_dtype == "bf16" else torch.float32
    y = (torch.randn((s.batch, s.seqlen, s.nheads, s.headdim), generator=g, device=DEV) * 3).to(tout)
    z = torch.randn((s.batch, s.seqlen, s.nheads, s.headdim), generator=g, device=DEV).to(tin) if gated else None
    w = 1.0 + 0.2 * torch.randn((s.nheads * s.headdim,), generator=g, device=DEV)
    return y, z, w


def _check(out, ref, what):
    a = out.double().cpu().numpy()
    scale = float(np.max(np.abs(ref))) if ref.size else 0.0
    tol = (2.0 ** -8 + 4e-4) * np.abs(ref) + 1e-6 * scale
    bad = np.abs(a - ref) > tol
    assert not bad.any(), f"{what}: {int(bad.sum())} of {bad.size} outside tolerance, max err {np.max(np.abs(a - ref)):.3e}"


@pytest.mark.parametrize("kw,groups,gated,eps", [
    (dict(), 1, True, 1e-5),                                   # 87M widths, one group, gated
    (dict(), 1, False, 1e-5),
    (dict(), 4, True, 1e-6),                                   # four groups of 384 channels
    (dict(), 24, True, 1e-5),                                  # one group per head
    (dict(), 48, True, 1e-5),                                  # 48 groups of 32: the shared-memory path
    (dict(nheads=48), 1, True, 1e-5),                          # 700M widths
    (dict(nheads=80, batch=1, seqlen=32), 2, True, 1e-5),      # 3B widths, one block
    (dict(out_dtype="bf16"), 1, True, 1e-5),                   # bf16 scan output
    (dict(in_dtype="fp32"), 3, True, 0.0),                     # fp32 gate, eps 0
    (dict(nheads=4, headdim=16, seqlen=8, batch=3, block_len=8, chunk_len=8), 16, False, 1e-3),  # groups of 4
])
def test_gated_rmsnorm_parity(kw, groups, gated, eps):
    s = _shape(**kw)
    y, z, w = _inputs(s, 3, gated)
    out = bd.gated_rmsnorm(s, y, z, w, groups, eps)
    torch.cuda.synchronize()
    ref = oracle.gated_rmsnorm(y, z, w, groups, eps)
    _check(out, ref, f"groups={groups} gated={gated}")


def test_gated_rmsnorm_in_place_and_deterministic():
    s = _shape(out_dtype="bf16")
    y, z, w = _inputs(s, 5, True)
    ref = oracle.gated_rmsnorm(y, z, w, 2, 1e-5)
    first = bd.gated_rmsnorm(s, y, z, w, 2, 1e-5)
    again = bd.gated_rmsnorm(s, y, z, w, 2, 1e-5)
    torch.cuda.synchronize()
    assert torch.equal(first, again), "not deterministic"
    yy = y.clone()
    out = bd.gated_rmsnorm(s, yy, z, w, 2, 1e-5, out=yy)
    torch.cuda.synchronize()
    assert out.data_ptr() == yy.data_ptr()
    assert torch.equal(yy, first), "in place differs"
    _check(first, ref, "in place")


def test_gated_rmsnorm_empty_and_zero_rows():
    s = _shape(seqlen=0)
    y, z, w = _inputs(s, 1, True)
    bd.gated_rmsnorm(s, y, z, w, 1, 1e-5)
    s = _shape(batch=1, seqlen=32)
    y = torch.zeros((1, 32, 24, 64), device=DEV)
    w = torch.ones(24 * 64, device=DEV)
    out = bd.gated_rmsnorm(s, y, None, w, 1, 1e-5)
    torch.cuda.synchronize()
    assert not out.any(), "a zero row with eps > 0 must stay zero"


def test_scan_then_norm_87m_full_size_sampled_rows():
    """The 87M all-block layer's noisy output through the norm, at full size, in
    the launch configuration the benchmark times; compared on two batch rows."""
    s = W.WORKLOADS["87m_allblock"]
    cf, cr, nf, nr = W.make_streams(s, W.SEEDS["87m_allblock"], device=DEV)
    _, yn, _ = bd.allblock(s, cf, cr, nf, nr, want_clean=False)
    g = torch.Generator(device=DEV).manual_seed(9)
    z = torch.randn(yn.shape, generator=g, device=DEV).to(torch.bfloat16)
    w = 1.0 + 0.2 * torch.randn((s.nheads * s.headdim,), generator=g, device=DEV)
    out = bd.gated_rmsnorm(s, yn, z, w, 1, 1e-5)
    torch.cuda.synchronize()
    rows = [0, s.batch - 1]
    ref = oracle.gated_rmsnorm(yn[rows], z[rows], w, 1, 1e-5)
    _check(out[rows], ref, "87M noisy output")
