"""Device checks that stand in for a memory-race / out-of-bounds sanitizer
(which is not available here) and for fault isolation:

* guard regions: every output buffer is a view into a larger allocation whose
  head and tail are filled with a sentinel; after the call the sentinels must
  be intact, bit for bit (no kernel writes outside its outputs);
* NaN confinement: a NaN planted in one (batch row, head) of x stays in that
  sequence's outputs and states; every other sequence is bit-identical to a
  clean run.
"""
import numpy as np
import pytest
import torch

from bidirectional_mamba_state_b200 import bdscan as bd
from bidirectional_mamba_state_b200 import workload as W

pytestmark = pytest.mark.gpu
DEV = "cuda:0"
GUARD_BYTES = 4096
SENTINEL = 0x5A


class Guarded:
    """A tensor of `shape` placed between two sentinel-filled guard regions."""

    def __init__(self, shape, dtype):
        esz = torch.tensor([], dtype=dtype).element_size()
        n = int(np.prod(shape)) if len(shape) else 1
        self.g = GUARD_BYTES
        self.raw = torch.full((2 * self.g + n * esz,), SENTINEL, dtype=torch.uint8, device=DEV)
        self.t = self.raw[self.g:self.g + n * esz].view(dtype).view(shape)

    def intact(self):
        head = self.raw[:self.g]
        tail = self.raw[self.raw.numel() - self.g:]
        return bool((head == SENTINEL).all()) and bool((tail == SENTINEL).all())


def _shape(**kw):
    d = dict(batch=3, seqlen=96, nheads=4, headdim=64, dstate=128, ngroups=2, block_len=32,
             chunk_len=32, in_dtype="bf16", out_dtype="fp32")
    d.update(kw)
    return W.Shape(**d)


@pytest.mark.parametrize("kw", [dict(), dict(in_dtype="fp32", block_len=16, seqlen=80, chunk_len=16),
                                dict(out_dtype="bf16", ngroups=1, batch=2)])
def test_scan_outputs_stay_inside_their_buffers(kw):
    s = _shape(**kw)
    tout = torch.bfloat16 if s.out_dtype == "bf16" else torch.float32
    cf, cr, nf, nr = W.make_streams(s, 2, device=DEV)
    yshape = (s.batch, s.seqlen, s.nheads, s.headdim)
    sshape = (s.batch, s.nblocks, s.nheads, s.headdim, s.dstate)
    yc, yn, st = Guarded(yshape, tout), Guarded(yshape, tout), Guarded(sshape, torch.float32)
    bd.allblock(s, cf, cr, nf, nr, y_clean=yc.t, y_noisy=yn.t, states=st.t)
    yp, stp, fin = Guarded(yshape, tout), Guarded(sshape, torch.float32), \
        Guarded((s.batch, s.nheads, s.headdim, s.dstate), torch.float32)
    bd.prefix(s, cf, cr, y=yp.t, states=stp.t, final=fin.t)
    one = s.with_(seqlen=s.block_len)
    af, ar = (W.sub_batch_block(d, 0, s.block_len) for d in (cf, cr))
    ys = Guarded((s.batch, s.block_len, s.nheads, s.headdim), tout)
    so = Guarded((s.batch, s.nheads, s.headdim, s.dstate), torch.float32)
    bd.block_step(one, af, ar, fin.t, state_out=so.t, y=ys.t)
    torch.cuda.synchronize()
    for name, g in (("y_clean", yc), ("y_noisy", yn), ("states", st), ("prefix y", yp),
                    ("prefix states", stp), ("final", fin), ("step y", ys), ("state_out", so)):
        assert g.intact(), f"{name}: a guard region was overwritten"
    assert torch.isfinite(yn.t.float()).all() and torch.isfinite(so.t).all()


def test_conv_and_norm_outputs_stay_inside_their_buffers():
    s = _shape(seqlen=64, ngroups=1)
    dirs = [W.make_conv_dir(s, 4, 1, stream=i, device=DEV) for i in range(4)]
    tin = torch.bfloat16
    outs = [{"x": Guarded((s.batch, s.seqlen, s.nheads, s.headdim), tin),
             "B": Guarded((s.batch, s.seqlen, s.ngroups, s.dstate), tin),
             "C": Guarded((s.batch, s.seqlen, s.ngroups, s.dstate), tin)} for _ in range(4)]
    bd.conv_allblock(s, 4, True, *dirs, outs=[{k: g.t for k, g in o.items()} for o in outs])
    cx = bd.conv_channels(s)
    st_in = W.make_conv_state(s, 4, 1, device=DEV)
    st_out = Guarded((s.batch, 3, cx), tin)
    pf = {k: Guarded(v.t.shape, tin) for k, v in outs[0].items()}
    bd.conv_prefix(s, 4, True, dirs[0], None, st_in, st_out.t, out_fwd={k: g.t for k, g in pf.items()})
    y = torch.randn((s.batch, s.seqlen, s.nheads, s.headdim), device=DEV)
    z = torch.randn(y.shape, device=DEV).to(torch.bfloat16)
    nout = Guarded(y.shape, torch.bfloat16)
    bd.gated_rmsnorm(s, y, z, torch.ones(s.nheads * s.headdim, device=DEV), 2, 1e-5, out=nout.t)
    torch.cuda.synchronize()
    for i, o in enumerate(outs):
        for k, g in o.items():
            assert g.intact(), f"conv direction {i} {k}: a guard region was overwritten"
    for k, g in pf.items():
        assert g.intact(), f"conv prefix {k}"
    assert st_out.intact() and nout.intact()


def test_backward_gradients_stay_inside_their_buffers():
    s = _shape(batch=2, seqlen=64)
    cf, cr, nf, nr = W.make_streams(s, 3, device=DEV)
    _, yn, st = bd.allblock(s, cf, cr, nf, nr)
    dyn = torch.randn(yn.shape, device=DEV)
    B, L, H, P, N, G = s.batch, s.seqlen, s.nheads, s.headdim, s.dstate, s.ngroups
    shapes = {"x": (B, L, H, P), "dt": (B, L, H), "B": (B, L, G, N), "C": (B, L, G, N), "A": (H,), "D": (H,)}
    gs = [{k: Guarded(v, torch.float32) for k, v in shapes.items()} for _ in range(4)]
    grads, dh0 = bd.allblock_backward(s, cf, cr, nf, nr, st, dyn, grads=[{k: g.t for k, g in d.items()} for d in gs])
    torch.cuda.synchronize()
    for i, d in enumerate(gs):
        for k, g in d.items():
            assert g.intact(), f"gradient {i} d{k}: a guard region was overwritten"


@pytest.mark.parametrize("kw", [dict(), dict(in_dtype="fp32", ngroups=1)])
def test_nan_stays_in_its_sequence(kw):
    """A NaN in x of one (b, h) reaches only that sequence's outputs and states;
    all other sequences are bit-identical to the clean run."""
    s = _shape(**kw)
    cf, cr, nf, nr = W.make_streams(s, 5, device=DEV)
    yc0, yn0, st0 = bd.allblock(s, cf, cr, nf, nr)
    b, h = 1, 2
    bad = dict(cf)
    bad["x"] = cf["x"].clone()
    bad["x"][b, 40, h, 5] = float("nan")
    yc1, yn1, st1 = bd.allblock(s, bad, cr, nf, nr)
    torch.cuda.synchronize()
    mask_y = torch.ones(yc0.shape, dtype=torch.bool, device=DEV)
    mask_y[b, :, h] = False
    mask_s = torch.ones(st0.shape, dtype=torch.bool, device=DEV)
    mask_s[b, :, h] = False
    for name, a0, a1, m in (("y_clean", yc0, yc1, mask_y), ("y_noisy", yn0, yn1, mask_y),
                            ("states", st0, st1, mask_s)):
        assert torch.equal(a0[m], a1[m]), f"{name}: the NaN leaked into another sequence"
    assert torch.isnan(yc1[b, :, h]).any() and torch.isnan(st1[b, :, h]).any()


@pytest.mark.parametrize("gated", [False, True])
def test_one_launch_step_guards_and_nan(gated):
    """The one-launch small-batch step (C B^T computed in the scan kernel): its
    output stays inside its buffer, the state is not written, and a NaN in one
    (b, h)'s x reaches only that sequence (a NaN in B or C of a group reaches
    exactly the heads of that group)."""
    s = _shape(seqlen=32, chunk_len=32, nheads=6, ngroups=2, batch=2)
    f = W.make_dir(s, 6, 0, W.CLEAN_FWD, DEV, gated=gated)
    r = W.make_dir(s, 6, 0, W.CLEAN_REV, DEV, gated=gated)
    state = W.make_state(s, 6, device=DEV)
    keep = state.clone()
    tout = torch.float32
    y = Guarded((s.batch, s.seqlen, s.nheads, s.headdim), tout)
    bd.block_step(s, f, r, state, y=y.t)
    torch.cuda.synchronize()
    assert y.intact(), "step y: a guard region was overwritten"
    assert torch.equal(state, keep), "the cached state was written by a non-committing step"
    y0 = y.t.clone()
    b, h = 1, 4
    bad = dict(f)
    bad["x"] = f["x"].clone()
    bad["x"][b, 7, h, 3] = float("nan")
    y1, _ = bd.block_step(s, bad, r, state)
    torch.cuda.synchronize()
    m = torch.ones(y0.shape, dtype=torch.bool, device=DEV)
    m[b, :, h] = False
    assert torch.equal(y0[m], y1[m]), "the NaN leaked into another sequence"
    assert torch.isnan(y1[b, :, h]).any()
    # a NaN in B of group 0 of row b reaches the heads of that group only
    badb = dict(f)
    badb["B"] = f["B"].clone()
    badb["B"][b, 5, 0, 11] = float("nan")
    y2, _ = bd.block_step(s, badb, r, state)
    torch.cuda.synchronize()
    hpg = s.nheads // s.ngroups
    m2 = torch.ones(y0.shape, dtype=torch.bool, device=DEV)
    m2[b, :, :hpg] = False
    assert torch.equal(y0[m2], y2[m2]), "a NaN in B leaked beyond its group"
    assert torch.isnan(y2[b, :, :hpg]).any()
