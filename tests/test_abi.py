"""CPU tests of the C-ABI library: it loads without a GPU, exports every symbol
the header declares, sizes workspaces, and rejects bad arguments with the
documented status codes before any launch (validation is host-side)."""
import ctypes

import pytest

from bidirectional_mamba_state_b200 import bdscan as bd
from bidirectional_mamba_state_b200.workload import Shape, WORKLOADS


def test_exports_every_header_symbol():
    names = bd.header_symbols()
    assert {"bdscan_prefix", "bdscan_block_step", "bdscan_allblock", "bdscan_workspace_size",
            "bdscan_check_status", "bdscan_status_string"} <= set(names)
    L = bd.lib()
    missing = [n for n in names if not hasattr(L, n)]
    assert not missing, f"libbdscan.so lacks {missing}"


def test_status_strings_and_version():
    for code in bd.STATUS:
        assert bd.bdscan_status_string(code)
    assert bd.bdscan_status_string(12345) == "unknown status"
    assert bd.bdscan_version() >= 100


@pytest.mark.parametrize("name", sorted(WORKLOADS))
def test_workspace_size_valid(name):
    s = bd.c_shape(WORKLOADS[name])
    for op in (bd.BDSCAN_OP_PREFIX, bd.BDSCAN_OP_ALLBLOCK):
        assert bd.bdscan_workspace_size(ctypes.byref(s), op) >= 256
    if WORKLOADS[name].seqlen == WORKLOADS[name].block_len:
        assert bd.bdscan_workspace_size(ctypes.byref(s), bd.BDSCAN_OP_BLOCK_STEP) >= 256


def _plan_segments(shape, op) -> int:
    """The segment count the library planned for a tensor-core call, read back
    from the workspace it asks for: header, C B^T tiles, then (when cut into
    segments) two [B][H][nseg][P][N] fp32 state arrays and [B][H][nseg] decays,
    each rounded up to 256 bytes."""
    al = lambda x: (x + 255) // 256 * 256
    K = shape.seqlen // shape.block_len
    sets = 4 if op == bd.BDSCAN_OP_ALLBLOCK else 2
    base = 1024 + al(sets * shape.batch * K * shape.ngroups * 2048)
    ws = bd.bdscan_workspace_size(ctypes.byref(bd.c_shape(shape)), op)
    if ws == base:
        return 1
    for nseg in range(2, K + 1):
        bh = shape.batch * shape.nheads
        if ws == base + 2 * al(bh * nseg * shape.headdim * shape.dstate * 4) + al(bh * nseg * 4):
            return nseg
    raise AssertionError(f"workspace {ws} matches no plan")


@pytest.mark.parametrize("name,op,nseg,launches", [
    # 48 sequences of 256 blocks: 3 segments (144 items, one wave on 148 SMs)
    ("700m_prefill_8k", "prefix", 3, 4),
    ("700m_prefill_64k", "prefix", 3, 4),
    # 80 sequences of 8192 blocks: segments enough for 13 waves of 148 items
    ("3b_prefill_256k", "prefix", 24, 4),
    # 128 sequences (one wave) and 384 sequences: not cut
    ("350m_allblock", "allblock", 1, 2),
    ("87m_allblock", "allblock", 1, 2),
    ("3b_step_b64", "prefix", 1, 2),
])
def test_segment_plan(name, op, nseg, launches):
    """The planner's choices for the stated workloads (host logic: a cost model
    of the waves of work items on 148 SMs), seen through the workspace size and
    the launch count."""
    s = WORKLOADS[name]
    o = bd.BDSCAN_OP_PREFIX if op == "prefix" else bd.BDSCAN_OP_ALLBLOCK
    assert _plan_segments(s, o) == nseg
    assert bd.bdscan_kernel_launches(ctypes.byref(bd.c_shape(s)), o) == launches


BAD_SHAPES = [
    (dict(seqlen=100), -2),        # not a multiple of block_len
    (dict(chunk_len=40), -2),      # chunk not a multiple of block
    (dict(nheads=5), -2),          # H % G != 0 (G = 2 below)
    (dict(headdim=48), -2),
    (dict(dstate=512), -2),
    (dict(block_len=48, seqlen=96, chunk_len=96), -2),
    (dict(batch=-1), -1),
    (dict(nheads=0), -1),
    (dict(in_dtype="fp16"), None),  # not representable: checked below via raw enum
]


def _base(**kw):
    d = dict(batch=2, seqlen=64, nheads=4, headdim=16, dstate=32, ngroups=2, block_len=16,
             chunk_len=32, in_dtype="bf16", out_dtype="fp32")
    d.update(kw)
    return d


@pytest.mark.parametrize("kw,code", BAD_SHAPES[:-1])
def test_bad_shape_rejected(kw, code):
    s = bd.c_shape(Shape(**_base(**kw)))
    assert bd.bdscan_workspace_size(ctypes.byref(s), bd.BDSCAN_OP_PREFIX) == 0
    fwd = _fake_dir(0x10000)
    rc = bd.bdscan_prefix(ctypes.byref(s), ctypes.byref(fwd), None, None, 0x900000, None, None,
                          0xA00000, 1 << 20, None)
    assert rc == code


def test_bad_dtype_enum():
    s = bd.c_shape(Shape(**_base()))
    s.in_dtype = 7
    fwd = _fake_dir(0x10000)
    rc = bd.bdscan_prefix(ctypes.byref(s), ctypes.byref(fwd), None, None, 0x900000, None, None,
                          0xA00000, 1 << 20, None)
    assert rc == -1


def _fake_dir(base, step=0x100000):
    # Distinct, 16-byte aligned, non-overlapping fake device addresses.  They are
    # never dereferenced: every call below fails validation before any launch.
    p = [base + i * step for i in range(7)]
    return bd.bdscan_dir_t(p[0], p[1], p[2], p[3], None, p[4], p[5])


def _prefix(shape_kw=None, fwd=None, rev=None, h0=None, y=0x90000000, states=None, final=None,
            ws=0xA0000000, ws_bytes=1 << 20):
    s = bd.c_shape(Shape(**_base(**(shape_kw or {}))))
    fwd = _fake_dir(0x10000000) if fwd is None else fwd
    return bd.bdscan_prefix(ctypes.byref(s), ctypes.byref(fwd) if fwd != "null" else None,
                            ctypes.byref(rev) if rev is not None else None, h0, y, states, final,
                            ws, ws_bytes, None)


def test_null_pointers_rejected():
    assert _prefix(fwd="null") == -1
    assert _prefix(y=None) == -1
    d = _fake_dir(0x10000000)
    d.x = None
    assert _prefix(fwd=d) == -1
    d = _fake_dir(0x10000000)
    d.A = None
    assert _prefix(fwd=d) == -1


def test_misaligned_rejected():
    d = _fake_dir(0x10000000)
    d.B = d.B + 4
    assert _prefix(fwd=d) == -3
    assert _prefix(y=0x90000008) == -3
    assert _prefix(ws=0xA0000004) == -3


def test_workspace_checked():
    assert _prefix(ws=None) == -4
    assert _prefix(ws_bytes=16) == -4


def test_output_aliasing_rejected():
    d = _fake_dir(0x10000000)
    assert _prefix(fwd=d, y=d.x) == -1           # y over x
    assert _prefix(fwd=d, y=d.x + 0x100) == -1   # partial overlap
    assert _prefix(states=0x90000000) == -1      # states over y


def test_block_step_requires_single_block():
    s = bd.c_shape(Shape(**_base()))  # seqlen 64 != block_len 16
    fwd = _fake_dir(0x10000000)
    rc = bd.bdscan_block_step(ctypes.byref(s), ctypes.byref(fwd), None, 0x80000000, 0x90000000, None,
                              0xA0000000, 1 << 20, None)
    assert rc == -2


def test_block_step_state_aliasing():
    s = bd.c_shape(Shape(**_base(seqlen=16)))
    fwd = _fake_dir(0x10000000)
    # partial overlap of state_out with state_in is rejected
    rc = bd.bdscan_block_step(ctypes.byref(s), ctypes.byref(fwd), None, 0x80000000, 0x90000000,
                              0x80000100, 0xA0000000, 1 << 20, None)
    assert rc == -1
    # y over state_in is rejected
    rc = bd.bdscan_block_step(ctypes.byref(s), ctypes.byref(fwd), None, 0x80000000, 0x80000000,
                              None, 0xA0000000, 1 << 20, None)
    assert rc == -1
    # null state_in is rejected
    rc = bd.bdscan_block_step(ctypes.byref(s), ctypes.byref(fwd), None, None, 0x90000000, None,
                              0xA0000000, 1 << 20, None)
    assert rc == -1


def test_allblock_requires_outputs():
    s = bd.c_shape(Shape(**_base()))
    cf, nf = _fake_dir(0x10000000), _fake_dir(0x20000000)
    rc = bd.bdscan_allblock(ctypes.byref(s), ctypes.byref(cf), None, ctypes.byref(nf), None, None,
                            None, None, 0x90000000, 0xA0000000, 1 << 20, None)
    assert rc == -1   # y_noisy missing
    rc = bd.bdscan_allblock(ctypes.byref(s), ctypes.byref(cf), None, None, None, None,
                            None, 0x90000000, 0x98000000, 0xA0000000, 1 << 20, None)
    assert rc == -1   # noisy_fwd missing


def _fake_grad(base, step=0x100000):
    p = [base + i * step for i in range(6)]
    return bd.bdscan_grad_t(*p)


def _backward(s_kw=None, gated=False, states=0x70000000, dyn=0x71000000, g_cf=None, g_nf=None,
              ws=0xA0000000, ws_bytes=None):
    s = bd.c_shape(Shape(**_base(**(s_kw or {}))))
    cf, nf = _fake_dir(0x10000000), _fake_dir(0x20000000)
    if gated:
        cf.z = 0x30000000
    g_cf = _fake_grad(0x40000000) if g_cf is None else g_cf
    g_nf = _fake_grad(0x50000000) if g_nf is None else g_nf
    if ws_bytes is None:
        ws_bytes = bd.bdscan_workspace_size(ctypes.byref(s), bd.BDSCAN_OP_ALLBLOCK_BACKWARD)
    return bd.bdscan_allblock_backward(ctypes.byref(s), ctypes.byref(cf), None, ctypes.byref(nf), None, None,
                                       states, None, dyn, None, ctypes.byref(g_cf), None,
                                       ctypes.byref(g_nf) if g_nf != "null" else None, None, None, ws,
                                       ws_bytes, None)


def test_backward_validation():
    s = bd.c_shape(Shape(**_base()))
    assert bd.bdscan_workspace_size(ctypes.byref(s), bd.BDSCAN_OP_ALLBLOCK_BACKWARD) > 1024
    assert _backward(gated=True) == -2            # the backward is ungated only
    assert _backward(states=None) == -1           # forward states required
    assert _backward(dyn=None) == -1              # dy_noisy required
    assert _backward(g_nf="null") == -1           # gradients of a present direction required
    g = _fake_grad(0x40000000)
    g.dx = g.dx + 4
    assert _backward(g_cf=g) == -3                # misaligned gradient
    g = _fake_grad(0x40000000)
    g.dx = 0x10000000                             # gradient over an input
    assert _backward(g_cf=g) == -1
    assert _backward(ws_bytes=64) == -4           # workspace too small
    # a block whose shared-memory plan does not fit one CTA
    assert _backward(s_kw=dict(headdim=128, dstate=256, block_len=64, chunk_len=64, seqlen=128)) == -2


def _fake_conv(base, step=0x100000):
    p = [base + i * step for i in range(8)]
    return bd.bdscan_conv_t(*p)


def _conv(s_kw=None, width=4, fwd=None, rev=None, st_in=None, st_out=None):
    s = bd.c_shape(Shape(**_base(**(s_kw or {}))))
    fwd = _fake_conv(0x10000000) if fwd is None else fwd
    return bd.bdscan_conv_prefix(ctypes.byref(s), width, 1, ctypes.byref(fwd) if fwd != "null" else None,
                                 ctypes.byref(rev) if rev is not None else None, st_in, st_out, None)


def test_conv_validation():
    s = bd.c_shape(Shape(**_base()))
    for op in (bd.BDSCAN_OP_CONV_PREFIX, bd.BDSCAN_OP_CONV_ALLBLOCK):
        assert bd.bdscan_workspace_size(ctypes.byref(s), op) == 0      # no workspace
        assert bd.bdscan_kernel_launches(ctypes.byref(s), op) == 1
    assert _conv(width=0) == -2 and _conv(width=5) == -2                # 1 <= width <= 4
    assert _conv(s_kw=dict(dstate=2, ngroups=1, nheads=4)) == -2        # G*N not a multiple of 4
    assert _conv(fwd="null") == -1
    d = _fake_conv(0x10000000)
    d.weight = None
    assert _conv(fwd=d) == -1                                           # taps required
    d = _fake_conv(0x10000000)
    d.C_out = d.C_out + 8
    assert _conv(fwd=d) == -3                                           # misaligned output
    d = _fake_conv(0x10000000)
    d.x_out = d.x                                                       # output over an input
    assert _conv(fwd=d) == -1
    assert _conv(st_in=0x80000000, st_out=0x80000100) == -1            # partial state overlap
    assert _conv(st_in=0x80000000, st_out=0x80000000) == -1            # in place needs seqlen <= 32
    assert _conv(st_in=0x80000004) == -3                                # misaligned state
    r = _fake_conv(0x20000000)
    r.x_out = _fake_conv(0x10000000).x_out                              # two directions write one buffer
    assert _conv(rev=r) == -1
    cf, nf = _fake_conv(0x10000000), _fake_conv(0x20000000)
    rc = bd.bdscan_conv_allblock(ctypes.byref(s), 4, 1, ctypes.byref(cf), None, None, None, None, None)
    assert rc == -1                                                     # noisy_fwd required


def test_gated_rmsnorm_validation():
    s = bd.c_shape(Shape(**_base()))   # H*P = 64 channels, fp32 y (out_dtype), bf16 z
    assert bd.bdscan_workspace_size(ctypes.byref(s), bd.BDSCAN_OP_GATED_RMSNORM) == 0
    assert bd.bdscan_kernel_launches(ctypes.byref(s), bd.BDSCAN_OP_GATED_RMSNORM) == 1
    y, z, w, out = 0x10000000, 0x20000000, 0x30000000, 0x40000000

    def call(y=y, z=z, w=w, groups=1, eps=1e-5, out=out, shape=s):
        return bd.bdscan_gated_rmsnorm(ctypes.byref(shape), y, z, w, groups, eps, out, None)

    assert call(groups=0) == -1
    assert call(eps=-1.0) == -1 and call(eps=float("nan")) == -1
    assert call(groups=3) == -2            # 64 % 3 != 0
    assert call(groups=32) == -2           # groups of 2 channels: not whole 4-channel vectors
    assert call(w=None) == -1 and call(out=None) == -1 and call(y=None) == -1
    assert call(out=out + 8) == -3         # misaligned
    assert call(out=y) == -1               # in place needs a bf16 y
    assert call(out=y + 0x40) == -1       # partial overlap with y
    assert call(out=z) == -1 and call(out=w) == -1


def test_binding_checks_caller_outputs():
    """The torch-facing helpers reject caller-provided outputs and workspaces of
    the wrong shape, dtype or device before anything reaches the C ABI (the C
    side trusts the sizes its pointers imply)."""
    import torch
    from bidirectional_mamba_state_b200 import workload as W
    s = W.Shape(1, 64, 2, 64, 128, 1, 32, 32, "bf16")
    f, r = W.make_streams(s, 0, streams=(W.CLEAN_FWD, W.CLEAN_REV))
    good_y = torch.empty((1, 64, 2, 64))
    bad = {
        "y short": dict(y=torch.empty((1, 32, 2, 64))),
        "y dtype": dict(y=torch.empty((1, 64, 2, 64), dtype=torch.bfloat16)),
        "states shape": dict(y=good_y, states=torch.empty((1, 1, 2, 64, 128))),
        "final dtype": dict(y=good_y, final=torch.empty((1, 2, 64, 128), dtype=torch.float64)),
        "ws dtype": dict(y=good_y, ws=torch.empty(1 << 20, dtype=torch.float32)),
        "ws small": dict(y=good_y, ws=torch.empty(16, dtype=torch.uint8)),
        "y strided": dict(y=torch.empty((1, 64, 2, 128))[..., ::2]),
    }
    for what, kw in bad.items():
        with pytest.raises(ValueError):
            bd.prefix(s, f, r, **kw)
    st = s.with_(seqlen=32)
    sf, sr = W.make_streams(st, 0, streams=(W.CLEAN_FWD, W.CLEAN_REV))
    state = torch.zeros((1, 2, 64, 128))
    for kw in (dict(state_out=torch.empty((1, 2, 64, 64))), dict(y=torch.empty((1, 64, 2, 64))),
               dict(ws=torch.empty(8, dtype=torch.uint8))):
        with pytest.raises(ValueError):
            bd.block_step(st, sf, sr, state, **kw)
    cf, cr, nf, nr = W.make_streams(s, 0)
    for kw in (dict(y_noisy=torch.empty((1, 64, 2, 32))), dict(y_clean=torch.empty((2, 64, 2, 64))),
               dict(states=torch.empty((1, 2, 2, 64, 128), dtype=torch.bfloat16))):
        with pytest.raises(ValueError):
            bd.allblock(s, cf, cr, nf, nr, **kw)
    yn = torch.empty((1, 64, 2, 64))
    sts = torch.empty((1, 2, 2, 64, 128))
    grads = [{"x": torch.empty((1, 64, 2, 64)), "dt": torch.empty((1, 64, 2)), "B": torch.empty((1, 64, 1, 128)),
              "C": torch.empty((1, 64, 1, 128)), "A": torch.empty(2), "D": torch.empty(2)} for _ in range(4)]
    grads[2]["B"] = torch.empty((1, 64, 1, 64))
    with pytest.raises(ValueError):
        bd.allblock_backward(s, cf, cr, nf, nr, sts, yn, grads=grads)


def test_options_set_get_restore():
    """Process-wide options: set returns the previous value, get the current
    one, out-of-range values and unknown options are rejected, the context
    manager restores the old value (host-side only: no GPU needed)."""
    for opt in (bd.BDSCAN_OPT_FORCE_GENERIC, bd.BDSCAN_OPT_VERBOSE, bd.BDSCAN_OPT_CB_PREPASS):
        old = bd.bdscan_get_option(opt)
        assert old in (0, 1)
        assert bd.bdscan_set_option(opt, 1) == old
        assert bd.bdscan_get_option(opt) == 1
        assert bd.bdscan_set_option(opt, 2) == -1  # BDSCAN_ERR_INVALID_ARG, value unchanged
        assert bd.bdscan_get_option(opt) == 1
        assert bd.bdscan_set_option(opt, old) == 1
        with bd.option(opt, 1 - old):
            assert bd.bdscan_get_option(opt) == 1 - old
        assert bd.bdscan_get_option(opt) == old
    t0 = bd.bdscan_get_option(bd.BDSCAN_OPT_WAIT_TIMEOUT_NS)
    assert t0 > 0
    with bd.option(bd.BDSCAN_OPT_WAIT_TIMEOUT_NS, 12345):
        assert bd.bdscan_get_option(bd.BDSCAN_OPT_WAIT_TIMEOUT_NS) == 12345
    assert bd.bdscan_get_option(bd.BDSCAN_OPT_WAIT_TIMEOUT_NS) == t0
    assert bd.bdscan_get_option(99) == -1
    assert bd.bdscan_set_option(99, 0) == -1


def _conv_step(s_kw=None, width=4, cf=None, cr=None, f=None, r=None, st=0x70000000, y=0x71000000,
               cst=None, ws=0xA0000000, ws_bytes=1 << 24):
    s = bd.c_shape(Shape(**_base(**dict(dict(seqlen=16, chunk_len=16), **(s_kw or {})))))
    cf = _fake_conv(0x10000000) if cf is None else cf
    cr = _fake_conv(0x20000000) if cr is None else cr
    f = _fake_dir(0x30000000) if f is None else f
    r = _fake_dir(0x40000000) if r is None else r
    ref = lambda v: None if v == "null" else ctypes.byref(v)
    return bd.bdscan_conv_block_step(ctypes.byref(s), width, 1, ref(cf), ref(cr), cst, ref(f), ref(r), st, y,
                                     ws, ws_bytes, None)


def test_conv_block_step_validation():
    """Every call fails validation before any launch (fake addresses)."""
    s = bd.c_shape(Shape(**_base(seqlen=16, chunk_len=16)))
    need = bd.bdscan_workspace_size(ctypes.byref(s), bd.BDSCAN_OP_CONV_BLOCK_STEP)
    assert need > bd.bdscan_workspace_size(ctypes.byref(s), bd.BDSCAN_OP_BLOCK_STEP)
    s64 = bd.c_shape(Shape(**_base()))
    assert bd.bdscan_workspace_size(ctypes.byref(s64), bd.BDSCAN_OP_CONV_BLOCK_STEP) == 0  # seqlen != block_len
    assert _conv_step(s_kw=dict(seqlen=32, chunk_len=32)) == -2
    assert _conv_step(width=5) == -2
    assert _conv_step(cr="null") == -1 and _conv_step(r="null") == -1  # both directions required
    d = _fake_conv(0x10000000)
    d.weight = None
    assert _conv_step(cf=d) == -1
    d = _fake_dir(0x30000000)
    d.dt = None
    assert _conv_step(f=d) == -1
    assert _conv_step(y=0x71000004) == -3                              # misaligned output
    assert _conv_step(y=0x10000000) == -1                              # output over the conv input
    assert _conv_step(cst=0x80000008) == -3                            # misaligned conv state
    assert _conv_step(st=None) == -1                                   # scan state required
    assert _conv_step(ws_bytes=need - 16) == -4                        # workspace too small
    assert _conv_step(ws=None) == -4
