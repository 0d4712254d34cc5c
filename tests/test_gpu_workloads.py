"""GPU parity at the stated workloads' full sizes, against the fp64 oracle.

- 350M all-block layer (B4 x 8192, 32 heads): every output and every boundary
  state.
- 700M inference layer (48 heads), prefill of 8K / 32K / 64K tokens with the
  final state only: layer 0 over all heads (final state and the last two
  blocks' outputs; every output at 8K and 32K), the whole output of 8 sampled
  heads, then two denoising steps and a commit from the device's cached state
  over all heads; layers 1 and 2 (their own weights) on 8 sampled heads.
- 3B layer (80 heads), prefill of 262,144 tokens: layer 0 over all heads (final
  state, last two blocks), the whole output of 8 sampled heads, a batch-1
  denoising step with commit from the device's cached state over all heads;
  layers 1 and 2 on 8 sampled heads; a batch-64 step with commit over all 64 x
  80 sequences.

The device always runs every head.  The oracle runs the heads in groups (with
one B/C group the heads are independent problems that share B and C), which
covers all heads without holding every head's fp64 copy at once.
"""
import numpy as np
import pytest
import torch

import oracle
from bidirectional_mamba_state_b200 import bdscan as bd
from bidirectional_mamba_state_b200 import workload as W
from parity import check_states, check_y, heads

pytestmark = pytest.mark.gpu
DEV = "cuda:0"
HEAD_CHUNK = 16
SAMPLED = 8


def _sampled_heads(H: int, layer: int) -> list:
    """8 heads spread evenly over [0, H) (first and last included for layer 0),
    shifted by 3 per further layer."""
    base = [round(i * (H - 1) / (SAMPLED - 1)) for i in range(SAMPLED)]
    return sorted((h + 3 * layer) % H for h in base)


def _oracle_prefix_by_heads(s: W.Shape, f: dict, r: dict, hs: list, last_tokens=None, want_y=True):
    """The oracle's prefix (final state only) over the heads `hs`, in groups of
    HEAD_CHUNK heads.  Returns (y of those heads -- all tokens, or the last
    `last_tokens` -- or None, final state of those heads)."""
    assert s.ngroups == 1
    ys, fins = [], []
    for i in range(0, len(hs), HEAD_CHUNK):
        ch = hs[i:i + HEAD_CHUNK]
        sub = s.with_(nheads=len(ch))
        ry, _, rfin = oracle.prefix(sub.as_dict(), heads(f, ch), heads(r, ch), want_states=False)
        if want_y:
            ys.append(ry[:, -last_tokens:] if last_tokens else ry)
        fins.append(rfin)
        del ry
    y = np.concatenate(ys, axis=2) if want_y else None
    return y, np.concatenate(fins, axis=1)


def test_350m_allblock_full():
    """350M all-block layer at full size: y_clean, y_noisy and all 256 boundary
    states of every sequence, compared in full."""
    s = W.WORKLOADS["350m_allblock"]
    cf, cr, nf, nr = W.make_streams(s, W.SEEDS["350m_allblock"], device=DEV)
    yc, yn, st = bd.allblock(s, cf, cr, nf, nr)
    torch.cuda.synchronize()
    ryc, ryn, rst = oracle.allblock(s.as_dict(), cf, cr, nf, nr)
    check_y(yc, ryc, what="y_clean")
    check_y(yn, ryn, what="y_noisy")
    del ryc, ryn
    assert st.shape[1] == 256
    check_states(st, rst)


def _prefill(name: str, layer: int):
    s = W.WORKLOADS[name]
    f, r = W.make_streams(s, W.SEEDS[name], layer, streams=(W.CLEAN_FWD, W.CLEAN_REV), device=DEV)
    y, _, fin = bd.prefix(s, f, r, want_states=False)
    torch.cuda.synchronize()
    return s, f, r, y, fin


@pytest.mark.parametrize("name", ["700m_prefill_8k", "700m_prefill_32k", "700m_prefill_64k"])
def test_700m_prefill_all_heads_then_steps(name):
    s, f, r, y, fin = _prefill(name, 0)
    H, T = s.nheads, s.block_len
    all_h = list(range(H))
    full = s.seqlen <= 32768
    ry, rfin = _oracle_prefix_by_heads(s, f, r, all_h, last_tokens=None if full else 2 * T)
    check_states(fin, rfin, "final state, all heads")
    if full:
        check_y(y, ry, what="y, all heads")
        ry = ry[:, -2 * T:]
    check_y(y[:, -2 * T:], ry, what="last two blocks, all heads")
    del ry
    hs = _sampled_heads(H, 0)
    if not full:
        ryh, _ = _oracle_prefix_by_heads(s, f, r, hs)
        check_y(y[:, :, hs], ryh, what="y, sampled heads")
        del ryh
    del f, r, y
    # denoising steps from the cached state, all heads, then a commit
    st = W.WORKLOADS["700m_step"]
    for step in range(2):
        af, ar = W.make_streams(st, 100 + step, streams=(W.CLEAN_FWD, W.CLEAN_REV), device=DEV)
        yb, _ = bd.block_step(st, af, ar, fin)
        ryb, _ = oracle.block_step(st.as_dict(), af, ar, rfin)
        check_y(yb, ryb, what=f"step {step}")
    yb, so = bd.block_step(st, af, ar, fin, state_out=True)
    _, rso = oracle.block_step(st.as_dict(), af, ar, rfin, want_state_out=True)
    check_states(so, rso, "commit")


@pytest.mark.parametrize("layer", [1, 2])
def test_700m_prefill_further_layers(layer):
    s, f, r, y, fin = _prefill("700m_prefill_8k", layer)
    hs = _sampled_heads(s.nheads, layer)
    ry, rfin = _oracle_prefix_by_heads(s, f, r, hs)
    check_y(y[:, :, hs], ry, what=f"layer {layer} y, sampled heads")
    check_states(fin[:, hs], rfin, f"layer {layer} final, sampled heads")


def test_3b_256k_prefill_all_heads_then_step():
    s, f, r, y, fin = _prefill("3b_prefill_256k", 0)
    H, T = s.nheads, s.block_len
    ry, rfin = _oracle_prefix_by_heads(s, f, r, list(range(H)), last_tokens=2 * T)
    check_states(fin, rfin, "final state, all heads")
    check_y(y[:, -2 * T:], ry, what="last two blocks, all heads")
    hs = _sampled_heads(H, 0)
    ryh, _ = _oracle_prefix_by_heads(s, f, r, hs)
    check_y(y[:, :, hs], ryh, what="y, sampled heads")
    del f, r, y, ry, ryh
    # a batch-1 denoising step (scan only) from the cached 256K state, all heads
    st = W.WORKLOADS["3b_step_b1"]
    af, ar = W.make_streams(st, 104, streams=(W.CLEAN_FWD, W.CLEAN_REV), device=DEV)
    yb, so = bd.block_step(st, af, ar, fin, state_out=True)
    ryb, rso = oracle.block_step(st.as_dict(), af, ar, rfin, want_state_out=True)
    check_y(yb, ryb, what="batch-1 step")
    check_states(so, rso, "batch-1 commit")


@pytest.mark.parametrize("layer", [1, 2])
def test_3b_256k_prefill_further_layers(layer):
    s, f, r, y, fin = _prefill("3b_prefill_256k", layer)
    hs = _sampled_heads(s.nheads, layer)
    ry, rfin = _oracle_prefix_by_heads(s, f, r, hs)
    check_y(y[:, :, hs], ry, what=f"layer {layer} y, sampled heads")
    check_states(fin[:, hs], rfin, f"layer {layer} final, sampled heads")


def test_3b_batch64_step_all_sequences():
    """Batch-64 denoising step with commit: all 64 x 80 (sequence, head) pairs."""
    st = W.WORKLOADS["3b_step_b64"]
    af, ar = W.make_streams(st, W.SEEDS["3b_step_b64"], streams=(W.CLEAN_FWD, W.CLEAN_REV), device=DEV)
    state = W.make_state(st, W.SEEDS["3b_step_b64"], device=DEV, scale=1.0)
    keep = state.clone()
    yb, so = bd.block_step(st, af, ar, state, state_out=True)
    ryb, rso = oracle.block_step(st.as_dict(), af, ar, keep, want_state_out=True)
    check_y(yb, ryb, what="batch-64 step")
    check_states(so, rso, "batch-64 commit")
    assert torch.equal(state, keep)
