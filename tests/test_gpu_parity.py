"""GPU parity: the CUDA path through the C ABI against the fp64 oracle on the
same seeded inputs, plus the invariants that must hold bit-exactly on the
device (boundary-state independence, state_in untouched, determinism)."""

import pytest
import torch

import oracle
from bidirectional_mamba_state_b200 import bdscan as bd
from bidirectional_mamba_state_b200 import workload as W
from parity import check_states, check_y, heads

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _shape(**kw):
    d = dict(batch=2, seqlen=160, nheads=6, headdim=64, dstate=128, ngroups=2, block_len=32,
             chunk_len=64, in_dtype="bf16", out_dtype="fp32")
    d.update(kw)
    return W.Shape(**d)


# shapes spanning several tiles, ragged tails and the degenerate cases
SMALL = {
    "tiny_fp32": W.WORKLOADS["tiny"],
    "bf16_multi": _shape(),
    "bf16_p16_n48_t16": _shape(headdim=16, dstate=48, block_len=16, chunk_len=16, seqlen=80),
    "fp32_p32_n16_t8": _shape(headdim=32, dstate=16, block_len=8, chunk_len=8, seqlen=40,
                              in_dtype="fp32", nheads=4),
    "bf16_t64_p128_n256": _shape(headdim=128, dstate=256, block_len=64, chunk_len=64, seqlen=128,
                                 nheads=2, ngroups=1, batch=1),
    "bf16_out_bf16": _shape(out_dtype="bf16"),
    "g1_h8": _shape(ngroups=1, nheads=8, batch=1, seqlen=96),
    # few sequences, many blocks: the tensor-core path cuts each sequence into
    # segments (aggregate pass + segment combine + main pass)
    "bf16_segmented": _shape(batch=1, nheads=2, ngroups=1, seqlen=1280),
    # more work items than SMs: each persistent CTA walks several (b, h)
    # sequences, resp. several segments, with the pipeline running across them
    # (80 sequences of 64 blocks: 5 segments each, 400 items in three waves)
    "bf16_many_items": _shape(batch=5, nheads=64, ngroups=4, seqlen=96),
    "bf16_segmented_many_items": _shape(batch=1, nheads=80, ngroups=2, seqlen=2048),
}


@pytest.mark.parametrize("name", sorted(SMALL))
@pytest.mark.parametrize("with_h0", [False, True])
def test_prefix_parity(name, with_h0):
    s = SMALL[name]
    f, r = W.make_streams(s, 1, streams=(W.CLEAN_FWD, W.CLEAN_REV), device=DEV)
    h0 = W.make_state(s, 1, device=DEV) if with_h0 else None
    y, st, fin = bd.prefix(s, f, r, h0=h0)
    ry, rst, rfin = oracle.prefix(s.as_dict(), f, r, h0=h0)
    check_y(y, ry, bf16_out=s.out_dtype == "bf16")
    check_states(st, rst)
    check_states(fin, rfin, "final")


@pytest.mark.parametrize("name", sorted(SMALL))
def test_allblock_parity(name):
    s = SMALL[name]
    cf, cr, nf, nr = W.make_streams(s, 2, device=DEV)
    h0 = W.make_state(s, 2, device=DEV)
    yc, yn, st = bd.allblock(s, cf, cr, nf, nr, h0=h0)
    ryc, ryn, rst = oracle.allblock(s.as_dict(), cf, cr, nf, nr, h0=h0)
    check_y(yc, ryc, bf16_out=s.out_dtype == "bf16", what="y_clean")
    check_y(yn, ryn, bf16_out=s.out_dtype == "bf16", what="y_noisy")
    check_states(st, rst)


@pytest.mark.parametrize("name", sorted(SMALL))
@pytest.mark.parametrize("commit", ["none", "new", "inplace"])
def test_block_step_parity(name, commit):
    s = SMALL[name].with_(seqlen=SMALL[name].block_len, chunk_len=SMALL[name].block_len)
    f, r = W.make_streams(s, 3, streams=(W.CLEAN_FWD, W.CLEAN_REV), device=DEV)
    state = W.make_state(s, 3, device=DEV, scale=2.0)
    keep = state.clone()
    ry, rso = oracle.block_step(s.as_dict(), f, r, keep, want_state_out=True)
    out = {"none": None, "new": True, "inplace": state}[commit]
    y, so = bd.block_step(s, f, r, state, state_out=out)
    torch.cuda.synchronize()
    check_y(y, ry, bf16_out=s.out_dtype == "bf16")
    if commit == "none":
        assert torch.equal(state, keep), "state_in modified by a non-committing step"
    else:
        check_states(so, rso, "state_out")


@pytest.mark.parametrize("name", ["bf16_multi", "bf16_out_bf16", "g1_h8"])
def test_block_step_cb_in_kernel_and_prepass(name):
    """Small-batch steps without a state out compute C B^T inside the scan
    kernel (one launch); with BDSCAN_OPT_CB_PREPASS they take the pre-pass.
    Both against the oracle, and against each other within the bf16 rounding
    of the pre-pass's C B^T tiles."""
    s = SMALL[name].with_(seqlen=32, chunk_len=32)
    f, r = W.make_streams(s, 15, streams=(W.CLEAN_FWD, W.CLEAN_REV), device=DEV)
    state = W.make_state(s, 15, device=DEV, scale=2.0)
    ry, _ = oracle.block_step(s.as_dict(), f, r, state)
    y, _ = bd.block_step(s, f, r, state)
    with bd.option(bd.BDSCAN_OPT_CB_PREPASS, 1):
        y2, _ = bd.block_step(s, f, r, state)
    torch.cuda.synchronize()
    bf = s.out_dtype == "bf16"
    check_y(y, ry, bf16_out=bf, what="C B^T in the scan kernel")
    check_y(y2, ry, bf16_out=bf, what="C B^T pre-pass")
    if not bf:  # two bf16-rounded results may sit a whole bf16 ulp apart
        check_y(y, y2.double().cpu().numpy(), what="in-kernel vs pre-pass")


def test_block_step_cb_in_kernel_timeout_reports_status():
    """The one-launch step (no pre-pass clears the status word there) reports
    a run-out wait through the status word too, and the next call is clean."""
    s = _shape(batch=1, seqlen=32, chunk_len=32)
    f, r = W.make_streams(s, 16, streams=(W.CLEAN_FWD, W.CLEAN_REV), device=DEV)
    state = W.make_state(s, 16, device=DEV)
    ws = bd.workspace(s, bd.BDSCAN_OP_BLOCK_STEP, DEV)
    stream = torch.cuda.current_stream().cuda_stream
    with bd.option(bd.BDSCAN_OPT_WAIT_TIMEOUT_NS, 0):
        bd.block_step(s, f, r, state, ws=ws)
    assert bd.bdscan_check_status(ws.data_ptr(), stream) == -6
    y, _ = bd.block_step(s, f, r, state, ws=ws)
    assert bd.bdscan_check_status(ws.data_ptr(), stream) == 0
    ry, _ = oracle.block_step(s.as_dict(), f, r, state)
    check_y(y, ry)


def test_no_reverse_and_gated():
    s = _shape()
    f = W.make_dir(s, 4, 0, W.CLEAN_FWD, DEV, gated=True)
    r = W.make_dir(s, 4, 0, W.CLEAN_REV, DEV, gated=True)
    for rev in (None, r):
        y, st, fin = bd.prefix(s, f, rev)
        ry, rst, rfin = oracle.prefix(s.as_dict(), f, rev)
        check_y(y, ry)
        check_states(st, rst)


@pytest.mark.parametrize("which", ["all", "fwd_only", "rev_only"])
def test_gated_allblock(which):
    """Gate per direction, y_dir * silu(z_dir) before the sum, on the
    tensor-core path (bf16, P = 64, N = 128, T = 32): every direction gated,
    or only the forward / only the reverse directions."""
    s = _shape(batch=2, seqlen=192)
    gate = {"all": (True, True), "fwd_only": (True, False), "rev_only": (False, True)}[which]
    dirs = [W.make_dir(s, 12, 0, k, DEV, gated=gate[k in (W.CLEAN_REV, W.NOISY_REV)])
            for k in (W.CLEAN_FWD, W.CLEAN_REV, W.NOISY_FWD, W.NOISY_REV)]
    h0 = W.make_state(s, 12, device=DEV)
    yc, yn, st = bd.allblock(s, *dirs, h0=h0)
    ryc, ryn, rst = oracle.allblock(s.as_dict(), *dirs, h0=h0)
    check_y(yc, ryc, what="y_clean")
    check_y(yn, ryn, what="y_noisy")
    check_states(st, rst)


@pytest.mark.parametrize("commit", [False, True])
def test_gated_block_step_and_prefix(commit):
    s = _shape(batch=3, seqlen=32, chunk_len=32)
    f = W.make_dir(s, 13, 0, W.CLEAN_FWD, DEV, gated=True)
    r = W.make_dir(s, 13, 0, W.CLEAN_REV, DEV, gated=True)
    state = W.make_state(s, 13, device=DEV)
    y, so = bd.block_step(s, f, r, state, state_out=True if commit else None)
    ry, rso = oracle.block_step(s.as_dict(), f, r, state, want_state_out=commit)
    check_y(y, ry)
    if commit:
        check_states(so, rso, "state_out")
    sp = _shape(batch=1, nheads=4, ngroups=1, seqlen=1280)  # segmented plan
    f = W.make_dir(sp, 14, 0, W.CLEAN_FWD, DEV, gated=True)
    r = W.make_dir(sp, 14, 0, W.CLEAN_REV, DEV, gated=True)
    y, st, fin = bd.prefix(sp, f, r)
    ry, rst, rfin = oracle.prefix(sp.as_dict(), f, r)
    check_y(y, ry)
    check_states(st, rst)
    check_states(fin, rfin, "final")


def test_gated_87m_allblock_full():
    """The 87M all-block layer with every direction gated, at full size."""
    s = W.WORKLOADS["87m_allblock"]
    cf, cr, nf, nr = W.make_streams(s, W.SEEDS["87m_allblock"], device=DEV, gated=True)
    yc, yn, st = bd.allblock(s, cf, cr, nf, nr)
    ryc, ryn, rst = oracle.allblock(s.as_dict(), cf, cr, nf, nr)
    check_y(yc, ryc, what="y_clean")
    check_y(yn, ryn, what="y_noisy")
    check_states(st, rst)


def test_cache_independent_of_active_block_bitwise():
    """Boundary states do not depend on the noisy stream or the reverse
    direction (bit-exact), and a perturbation of clean x at token j leaves
    states[k] for k < j // T bit-identical."""
    s = _shape(batch=1)
    cf, cr, nf, nr = W.make_streams(s, 5, device=DEV)
    _, _, st = bd.allblock(s, cf, cr, nf, nr)
    nf2, nr2, cr2 = (W.make_dir(s, 77, 0, k, DEV) for k in (W.NOISY_FWD, W.NOISY_REV, W.CLEAN_REV))
    _, _, st2 = bd.allblock(s, cf, cr2, nf2, nr2)
    assert torch.equal(st, st2)
    j = 70
    cf3 = {k: v.clone() for k, v in cf.items()}
    cf3["x"][0, j] += 1.0
    _, _, st3 = bd.allblock(s, cf3, cr, nf, nr)
    kb = j // s.block_len
    assert torch.equal(st3[:, :kb], st[:, :kb])
    assert not torch.equal(st3[:, kb], st[:, kb])


def test_deterministic_bitwise():
    s = _shape()
    cf, cr, nf, nr = W.make_streams(s, 6, device=DEV)
    a = bd.allblock(s, cf, cr, nf, nr)
    b = bd.allblock(s, cf, cr, nf, nr)
    for u, v in zip(a, b):
        assert torch.equal(u, v)


def test_empty_inputs():
    for kw in (dict(batch=0), dict(seqlen=0)):
        s = _shape(**kw)
        f = W.make_dir(s, 7, 0, W.CLEAN_FWD, DEV)
        h0 = torch.randn((s.batch, s.nheads, s.headdim, s.dstate), device=DEV)
        y, st, fin = bd.prefix(s, f, None, h0=h0)
        torch.cuda.synchronize()
        assert y.numel() == 0 or s.batch == 0
        if s.seqlen == 0:
            assert torch.equal(fin, h0)


def test_noisy_equals_clean_on_device():
    s = _shape(batch=1)
    cf, cr, _, _ = W.make_streams(s, 8, device=DEV)
    yc, yn, _ = bd.allblock(s, cf, cr, cf, cr)
    torch.testing.assert_close(yn, yc, rtol=1e-5, atol=1e-5)


def test_status_word_clear_after_call():
    s = _shape(batch=1)
    cf, cr, nf, nr = W.make_streams(s, 9, device=DEV)
    ws = bd.workspace(s, bd.BDSCAN_OP_ALLBLOCK, DEV)
    bd.allblock(s, cf, cr, nf, nr, ws=ws)
    assert bd.bdscan_check_status(ws.data_ptr(), torch.cuda.current_stream().cuda_stream) == 0


# ---------------------------------------------------------------- the five workloads
def test_workload_tiny():
    s = W.WORKLOADS["tiny"]
    cf, cr, nf, nr = W.make_streams(s, W.SEEDS["tiny"], device=DEV)
    yc, yn, st = bd.allblock(s, cf, cr, nf, nr)
    ryc, ryn, rst = oracle.allblock(s.as_dict(), cf, cr, nf, nr)
    check_y(yc, ryc)
    check_y(yn, ryn)
    check_states(st, rst)


def test_workload_87m_allblock_full():
    """87M all-block layer at full size (B16 x 1024, 24 heads), every output."""
    s = W.WORKLOADS["87m_allblock"]
    cf, cr, nf, nr = W.make_streams(s, W.SEEDS["87m_allblock"], device=DEV)
    yc, yn, st = bd.allblock(s, cf, cr, nf, nr)
    ryc, ryn, rst = oracle.allblock(s.as_dict(), cf, cr, nf, nr)
    check_y(yc, ryc, what="y_clean")
    check_y(yn, ryn, what="y_noisy")
    check_states(st, rst)


# ---------------------------------------------------------------- both device paths
def test_tensor_core_path_matches_generic_path():
    """The tcgen05 kernel and the CUDA-core kernel agree on the same inputs
    (both are also checked against the oracle above)."""
    s = _shape(batch=3, seqlen=256, nheads=4, ngroups=2)
    cf, cr, nf, nr = W.make_streams(s, 10, device=DEV)
    h0 = W.make_state(s, 10, device=DEV)
    tc = bd.allblock(s, cf, cr, nf, nr, h0=h0)
    with bd.option(bd.BDSCAN_OPT_FORCE_GENERIC, 1):
        gen = bd.allblock(s, cf, cr, nf, nr, h0=h0)
    # same bounds as against the oracle (the generic path is within 1e-6 of it)
    check_y(tc[0], gen[0].double().cpu().numpy(), what="y_clean tc vs generic")
    check_y(tc[1], gen[1].double().cpu().numpy(), what="y_noisy tc vs generic")
    check_states(tc[2], gen[2].double().cpu().numpy(), "states tc vs generic")


def test_bounded_wait_timeout_reports_status():
    """With the wait limit forced to zero every bounded wait gives up at once:
    the kernel reports BDSCAN_ERR_TIMEOUT through the workspace status word and
    returns; the context stays usable and the next call is correct."""
    s = _shape(batch=1, seqlen=128)
    cf, cr, nf, nr = W.make_streams(s, 11, device=DEV)
    ws = bd.workspace(s, bd.BDSCAN_OP_ALLBLOCK, DEV)
    stream = torch.cuda.current_stream().cuda_stream
    with bd.option(bd.BDSCAN_OPT_WAIT_TIMEOUT_NS, 0):
        bd.allblock(s, cf, cr, nf, nr, ws=ws)
    assert bd.bdscan_check_status(ws.data_ptr(), stream) == -6
    yc, yn, st = bd.allblock(s, cf, cr, nf, nr, ws=ws)
    assert bd.bdscan_check_status(ws.data_ptr(), stream) == 0
    ryc, ryn, rst = oracle.allblock(s.as_dict(), cf, cr, nf, nr)
    check_y(yn, ryn)
    check_states(st, rst)


def test_bounded_wait_timeout_segmented_prefix():
    """The same for a segmented prefix (the aggregate pass, the segment combine
    and the main pass): a zero wait limit gives BDSCAN_ERR_TIMEOUT, the next
    call is clean and matches the oracle."""
    s = _shape(batch=1, nheads=2, ngroups=1, seqlen=1280)
    assert bd.kernel_launches(s, bd.BDSCAN_OP_PREFIX) == 4  # segmented plan
    f, r = W.make_streams(s, 12, streams=(W.CLEAN_FWD, W.CLEAN_REV), device=DEV)
    ws = bd.workspace(s, bd.BDSCAN_OP_PREFIX, DEV)
    stream = torch.cuda.current_stream().cuda_stream
    with bd.option(bd.BDSCAN_OPT_WAIT_TIMEOUT_NS, 0):
        bd.prefix(s, f, r, want_states=False, ws=ws)
    assert bd.bdscan_check_status(ws.data_ptr(), stream) == -6
    y, _, fin = bd.prefix(s, f, r, want_states=False, ws=ws)
    assert bd.bdscan_check_status(ws.data_ptr(), stream) == 0
    ry, _, rfin = oracle.prefix(s.as_dict(), f, r)
    check_y(y, ry)
    check_states(fin, rfin)


@pytest.mark.parametrize("case", ["pairs_eq_sms", "pairs_over_sms", "fwd_only", "gated_g2", "bf16_out_g2"])
def test_block_step_one_launch_edges(case):
    """Edges of the one-launch small-batch step (C B^T in the scan kernel):
    exactly as many (sequence, head) pairs as SMs, one sequence more (pre-pass path),
    a forward-only step (pre-pass path), gated directions with two groups, bf16
    output; each against the oracle, and the pair-count edges also against the
    pre-pass path."""
    nsm = torch.cuda.get_device_properties(0).multi_processor_count
    kw = dict(batch=2, seqlen=32, chunk_len=32, nheads=6, ngroups=2)
    if case in ("pairs_eq_sms", "pairs_over_sms"):
        assert nsm % 4 == 0
        kw.update(batch=nsm // 4, nheads=4, ngroups=1)
    elif case == "bf16_out_g2":
        kw.update(out_dtype="bf16")
    s = _shape(**kw)
    if case == "pairs_over_sms":  # one more sequence than fills the SMs
        s = s.with_(batch=s.batch + 1)
    gated = case == "gated_g2"
    f = W.make_dir(s, 17, 0, W.CLEAN_FWD, DEV, gated=gated)
    r = None if case == "fwd_only" else W.make_dir(s, 17, 0, W.CLEAN_REV, DEV, gated=gated)
    state = W.make_state(s, 17, device=DEV, scale=2.0)
    y, _ = bd.block_step(s, f, r, state)
    with bd.option(bd.BDSCAN_OPT_CB_PREPASS, 1):
        y2, _ = bd.block_step(s, f, r, state)
    torch.cuda.synchronize()
    ry, _ = oracle.block_step(s.as_dict(), f, r, state)
    bf = s.out_dtype == "bf16"
    check_y(y, ry, bf16_out=bf, what=case)
    check_y(y2, ry, bf16_out=bf, what=case + " (pre-pass)")
    if r is not None:  # the launch count assumes both directions
        assert bd.kernel_launches(s, bd.BDSCAN_OP_BLOCK_STEP) == (1 if s.batch * s.nheads <= nsm else 2)
