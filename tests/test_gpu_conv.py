"""Device short convolution (bdscan_conv_prefix / bdscan_conv_allblock) against
the fp64 oracle, element by element, on the same seeded inputs.

Tolerance, from the arithmetic: the kernel forms the pre-activation
a = bias + sum_j w_j u_j as a chain of W fp32 fused multiply-adds (error at
most W * 2^-24 * S, S = |bias| + sum_j |w_j u_j|), then silu(a) = a / (1 +
exp(-a)) in fp32 (a few ulp of |silu(a)|; silu's slope is below 1.1).  So
|device - oracle| <= 1e-6 * S + 1e-6 * |v| for fp32 outputs (about 4x the
bound), plus half a bf16 ulp of |v| (2^-9 |v|, taken as 2^-8 |v| for values on a
rounding boundary) for bf16 outputs.  The conv state holds copies of inputs:
compared bit for bit."""
import numpy as np
import pytest
import torch

import oracle
from bidirectional_mamba_state_b200 import bdscan as bd
from bidirectional_mamba_state_b200 import workload as W

pytestmark = pytest.mark.gpu
DEV = "cuda:0"
KEYS = ("x", "B", "C")


def _shape(**kw):
    d = dict(batch=2, seqlen=128, nheads=4, headdim=64, dstate=128, ngroups=1, block_len=32,
             chunk_len=32, in_dtype="bf16", out_dtype="fp32")
    d.update(kw)
    return W.Shape(**d)


def _abs_dir(d):
    return {k: (v.abs() if hasattr(v, "abs") else v) for k, v in d.items() if v is not None}


def _check_dir(s, got, want, scale, v_ref, what):
    bf16 = s.in_dtype == "bf16"
    for k in KEYS:
        a = got[k].detach().double().cpu().numpy()
        r = want[k]
        S = scale[k]
        assert a.shape == r.shape, (what, k, a.shape, r.shape)
        tol = 1e-6 * S + 1e-6 * np.abs(r) + (2.0 ** -8 * np.abs(r) if bf16 else 0.0)
        bad = np.abs(a - r) > tol
        assert not bad.any(), (f"{what} {k}: {int(bad.sum())} of {bad.size} outside tolerance, "
                               f"max err {float(np.max(np.abs(a - r))):.3e}")


def _scales_prefix(s, width, fwd, rev, st):
    """S = |bias| + sum |w u| per output: the oracle run on absolute values, no SiLU."""
    af = _abs_dir(fwd)
    ar = _abs_dir(rev) if rev is not None else None
    ast = st.abs() if st is not None else None
    sf, sr, _ = oracle.conv_prefix(s.as_dict(), width, False, af, ar, ast)
    return sf, sr


def _run_prefix(s, width=4, silu=True, with_rev=True, with_state=True, state_out=None, seed=3,
                bias=True):
    fwd = W.make_conv_dir(s, width, seed, stream=W.CLEAN_FWD, device=DEV, bias=bias)
    rev = W.make_conv_dir(s, width, seed, stream=W.CLEAN_REV, device=DEV, bias=bias) if with_rev else None
    st = W.make_conv_state(s, width, seed, device=DEV) if with_state else None
    st_host = st.clone() if st is not None else None
    if state_out == "inplace":
        so = st
    elif state_out:
        so = True
    else:
        so = None
    of, orv, so = bd.conv_prefix(s, width, silu, fwd, rev, st, so)
    torch.cuda.synchronize()
    rf, rr, rso = oracle.conv_prefix(s.as_dict(), width, silu, fwd, rev, st_host,
                                     want_state_out=so is not None)
    sf, sr = _scales_prefix(s, width, fwd, rev, st_host)
    _check_dir(s, of, rf, sf, rf, "fwd")
    if with_rev:
        _check_dir(s, orv, rr, sr, rr, "rev")
    if so is not None:
        got = so.detach().double().cpu().numpy()
        assert np.array_equal(got, rso), "conv state_out differs"
    return of, orv, so


@pytest.mark.parametrize("kw", [
    dict(),                                                       # several blocks, bf16
    dict(in_dtype="fp32"),
    dict(batch=1, seqlen=256, nheads=4, headdim=16, dstate=16, in_dtype="fp32"),  # tiny workload shape
    dict(block_len=8, seqlen=64),                                 # short blocks: 8-token tiles
    dict(block_len=64, seqlen=192, chunk_len=64),                 # long blocks: 32-token tiles in a block
    dict(block_len=4, seqlen=12, chunk_len=4),                    # ragged last forward tile
    dict(block_len=1, seqlen=5, chunk_len=1),                     # one-token blocks
    dict(ngroups=2, dstate=16, nheads=4, headdim=32),             # two groups, G*N = 32
    dict(batch=3, seqlen=96, nheads=48, headdim=64),              # 700M widths
])
def test_conv_prefix_parity(kw):
    s = _shape(**kw)
    _run_prefix(s, state_out=True)


@pytest.mark.parametrize("width", [1, 2, 3])
@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
def test_conv_widths(width, dtype):
    s = _shape(in_dtype=dtype, seqlen=96)
    _run_prefix(s, width=width, silu=(width != 2), state_out=True)


def test_conv_no_bias_no_rev_no_state():
    s = _shape()
    _run_prefix(s, with_rev=False, with_state=False, bias=False, state_out=True)


@pytest.mark.parametrize("batch,nheads", [(1, 48), (3, 80)])
def test_conv_block_step_inplace_commit(batch, nheads):
    """A denoising step of the active block (seqlen == block_len) from the cached
    conv state, committing into the same buffer."""
    s = _shape(batch=batch, nheads=nheads, seqlen=32, block_len=32, chunk_len=32)
    _run_prefix(s, state_out="inplace")


def test_conv_state_shift_short_sequence():
    """seqlen < width-1: the new state keeps the old rows that are still among the last W-1."""
    s = _shape(seqlen=2, block_len=2, chunk_len=2)
    _run_prefix(s, state_out="inplace")
    _run_prefix(s, state_out=True)


def test_conv_empty():
    s = _shape(seqlen=0)
    st = W.make_conv_state(s, 4, 1, device=DEV)
    fwd = W.make_conv_dir(s, 4, 1, device=DEV)
    _, _, so = bd.conv_prefix(s, 4, True, fwd, None, st, True)
    torch.cuda.synchronize()
    assert torch.equal(so, st)
    _, _, so = bd.conv_prefix(s, 4, True, fwd, None, None, True)
    torch.cuda.synchronize()
    assert not so.any()
    s0 = _shape(batch=0)
    bd.conv_prefix(s0, 4, True, W.make_conv_dir(s0, 4, 1, device=DEV))
    torch.cuda.synchronize()


def _run_allblock(s, width=4, silu=True, with_rev=True, with_state=True, seed=7):
    dirs = [W.make_conv_dir(s, width, seed, stream=i, device=DEV) for i in range(4)]
    if not with_rev:
        dirs[1] = dirs[3] = None
    st = W.make_conv_state(s, width, seed, device=DEV) if with_state else None
    outs = bd.conv_allblock(s, width, silu, *dirs, st)
    torch.cuda.synchronize()
    ref = oracle.conv_allblock(s.as_dict(), width, silu, *dirs, st)
    absd = [None if d is None else _abs_dir(d) for d in dirs]
    sc = oracle.conv_allblock(s.as_dict(), width, False, *absd, st.abs() if st is not None else None)
    names = ["clean fwd", "clean rev", "noisy fwd", "noisy rev"]
    for i in range(4):
        if ref[i] is None:
            assert outs[i] is None
            continue
        _check_dir(s, outs[i], ref[i], sc[i], ref[i], names[i])


@pytest.mark.parametrize("kw", [dict(), dict(block_len=8, seqlen=64), dict(block_len=2, seqlen=16, chunk_len=2),
                                dict(in_dtype="fp32", block_len=64, seqlen=128, chunk_len=64)])
def test_conv_allblock_parity(kw):
    _run_allblock(_shape(**kw))


def test_conv_allblock_no_rev_no_state():
    _run_allblock(_shape(), with_rev=False, with_state=False, width=3)


def test_conv_allblock_87m_full_size_sampled_rows():
    """The 87M all-block layer at full size, in the launch configuration the
    benchmark times; compared in full on two batch rows (rows are independent,
    so the oracle on those rows gives their exact expected values)."""
    s = W.WORKLOADS["87m_allblock"]
    width = 4
    dirs = [W.make_conv_dir(s, width, W.SEEDS["87m_allblock"], stream=i, device=DEV) for i in range(4)]
    outs = bd.conv_allblock(s, width, True, *dirs, None)
    torch.cuda.synchronize()
    rows = [0, s.batch - 1]
    sub = s.with_(batch=len(rows))
    pick = [None if d is None else {k: (v[rows] if k in KEYS else v) for k, v in d.items()} for d in dirs]
    ref = oracle.conv_allblock(sub.as_dict(), width, True, *pick, None)
    absd = [{k: v.abs() for k, v in d.items()} for d in pick]
    sc = oracle.conv_allblock(sub.as_dict(), width, False, *absd, None)
    for i in range(4):
        got = {k: outs[i][k][rows] for k in KEYS}
        _check_dir(sub, got, ref[i], sc[i], ref[i], f"direction {i}")

