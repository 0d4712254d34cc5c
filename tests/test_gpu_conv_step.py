"""GPU parity of bdscan_conv_block_step (the short convolution and the scan
step of a denoising step in one call).

- Against the device's two-call path (bdscan_conv_prefix into buffers, then
  bdscan_block_step on them): bit-identical, for every width, with and without
  SiLU, bias, conv state and gate, one and two B/C groups (the call runs the
  same kernels on workspace buffers, so nothing may differ).
- Against the fp64 oracle composed the same way (oracle convolution, rounded
  to bf16 like the device's convolved inputs, then the oracle step), within
  the scan's output tolerance; at the 700M and 3B batch-1 step sizes over all
  heads.
- Shapes outside the one-launch step kernel (fp32 inputs, a batch with more
  (sequence, head) pairs than SMs, the C B^T pre-pass option) give the same
  result as calling the two entry points directly.
"""
import numpy as np
import pytest
import torch

import oracle
from bidirectional_mamba_state_b200 import bdscan as bd
from bidirectional_mamba_state_b200 import workload as W
from parity import check_y

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def _shape(**kw):
    d = dict(batch=1, seqlen=32, nheads=6, headdim=64, dstate=128, ngroups=2, block_len=32, chunk_len=32,
             in_dtype="bf16", out_dtype="fp32")
    d.update(kw)
    return W.Shape(**d)


def _inputs(s, width, seed, gated=False, bias=True, with_state=True):
    conv = [W.make_conv_dir(s, width, seed, 0, k, device=DEV, bias=bias) for k in (W.CLEAN_FWD, W.CLEAN_REV)]
    scan = [W.make_dir(s, seed, 0, k, DEV, gated=gated) for k in (W.CLEAN_FWD, W.CLEAN_REV)]
    cstate = W.make_conv_state(s, width, seed, device=DEV) if with_state and width > 1 else None
    state = W.make_state(s, seed, device=DEV)
    return conv, scan, cstate, state


def _two_calls(s, width, silu, conv, scan, cstate, state):
    of, orv, _ = bd.conv_prefix(s, width, silu, conv[0], conv[1], state_in=cstate)
    f = dict(scan[0], **of)
    r = dict(scan[1], **orv)
    y, _ = bd.block_step(s, f, r, state)
    return y


def _oracle(s, width, silu, conv, scan, cstate, state):
    of, orv, _ = oracle.conv_prefix(s.as_dict(), width, silu, conv[0], conv[1], state_in=cstate)
    tin = torch.bfloat16 if s.in_dtype == "bf16" else torch.float32
    rnd = lambda d: {k: torch.from_numpy(np.asarray(v)).to(tin) for k, v in d.items()}
    f = dict(scan[0], **rnd(of))
    r = dict(scan[1], **rnd(orv))
    ry, _ = oracle.block_step(s.as_dict(), f, r, state)
    return ry


CASES = [
    # width, silu, gated, bias, conv state, shape overrides
    (4, True, False, True, True, {}),
    (4, True, True, True, True, {}),
    (4, False, False, False, True, {}),
    (3, True, False, True, True, dict(batch=2)),
    (2, True, False, True, False, dict(ngroups=1, nheads=8)),
    (1, True, False, True, False, {}),
    (4, True, False, True, True, dict(out_dtype="bf16")),
]


@pytest.mark.parametrize("case", range(len(CASES)))
def test_conv_step_matches_two_calls_and_oracle(case):
    width, silu, gated, bias, with_state, kw = CASES[case]
    s = _shape(**kw)
    conv, scan, cstate, state = _inputs(s, width, 20 + case, gated, bias, with_state)
    keep = state.clone()
    y = bd.conv_block_step(s, width, silu, conv[0], conv[1], cstate, scan[0], scan[1], state)
    y2 = _two_calls(s, width, silu, conv, scan, cstate, state)
    torch.cuda.synchronize()
    assert torch.equal(y, y2), "one call vs the two entry points"
    assert torch.equal(state, keep), "scan state modified"
    ry = _oracle(s, width, silu, conv, scan, cstate, state)
    check_y(y, ry, bf16_out=s.out_dtype == "bf16")


def test_conv_step_launch_count():
    s = _shape()
    assert bd.kernel_launches(s, bd.BDSCAN_OP_CONV_BLOCK_STEP) == 2
    assert bd.kernel_launches(s, bd.BDSCAN_OP_BLOCK_STEP) == 1
    with bd.option(bd.BDSCAN_OPT_CB_PREPASS, 1):
        assert bd.kernel_launches(s, bd.BDSCAN_OP_CONV_BLOCK_STEP) == 3
        assert bd.kernel_launches(s, bd.BDSCAN_OP_BLOCK_STEP) == 2


@pytest.mark.parametrize("which", ["fp32", "many_pairs", "prepass_option"])
def test_conv_step_two_call_fallback(which):
    if which == "fp32":
        s = _shape(in_dtype="fp32", headdim=32, dstate=16, nheads=4)
    elif which == "many_pairs":
        s = _shape(batch=3, nheads=64, ngroups=4)  # 192 (sequence, head) pairs > SMs
    else:
        s = _shape()
    conv, scan, cstate, state = _inputs(s, 4, 31, gated=which == "prepass_option")
    if which == "prepass_option":
        with bd.option(bd.BDSCAN_OPT_CB_PREPASS, 1):
            y = bd.conv_block_step(s, 4, True, conv[0], conv[1], cstate, scan[0], scan[1], state)
            y2 = _two_calls(s, 4, True, conv, scan, cstate, state)
    else:
        y = bd.conv_block_step(s, 4, True, conv[0], conv[1], cstate, scan[0], scan[1], state)
        y2 = _two_calls(s, 4, True, conv, scan, cstate, state)
    torch.cuda.synchronize()
    assert torch.equal(y, y2)
    ry = _oracle(s, 4, True, conv, scan, cstate, state)
    check_y(y, ry)


def test_conv_step_timeout_reports_status():
    """A run-out wait in the step's kernel is reported through the status word;
    the next call is clean and correct."""
    s = _shape()
    conv, scan, cstate, state = _inputs(s, 4, 33)
    ws = bd.workspace(s, bd.BDSCAN_OP_CONV_BLOCK_STEP, DEV)
    stream = torch.cuda.current_stream().cuda_stream
    with bd.option(bd.BDSCAN_OPT_WAIT_TIMEOUT_NS, 0):
        bd.conv_block_step(s, 4, True, conv[0], conv[1], cstate, scan[0], scan[1], state, ws=ws)
    assert bd.bdscan_check_status(ws.data_ptr(), stream) == -6
    y = bd.conv_block_step(s, 4, True, conv[0], conv[1], cstate, scan[0], scan[1], state, ws=ws)
    assert bd.bdscan_check_status(ws.data_ptr(), stream) == 0
    check_y(y, _oracle(s, 4, True, conv, scan, cstate, state))


@pytest.mark.parametrize("name", ["700m_step", "3b_step_b1"])
def test_conv_step_full_size(name):
    """The 700M (48 heads) and 3B (80 heads) batch-1 steps, width 4 with SiLU,
    from a random conv state: every head against the oracle, and the two-call
    path bit for bit."""
    s = W.WORKLOADS[name]
    conv, scan, cstate, state = _inputs(s, 4, W.SEEDS[name])
    y = bd.conv_block_step(s, 4, True, conv[0], conv[1], cstate, scan[0], scan[1], state)
    y2 = _two_calls(s, 4, True, conv, scan, cstate, state)
    torch.cuda.synchronize()
    assert torch.equal(y, y2)
    check_y(y, _oracle(s, 4, True, conv, scan, cstate, state))
