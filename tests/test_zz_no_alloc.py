"""The allocation-free denoising step, bdscan_block_step_noalloc.

It serves callers that cannot allocate device memory (a static memory arena
that already holds all device memory, or code running during stream capture):
its scratch is a fixed buffer inside the library instead of a caller
workspace.  These tests call it through the C ABI and check it against the
ordinary bdscan_block_step on the same inputs, on two calls in a row (the
calls share the buffer), for a tensor-core shape and a generic-path shape.
This file is collected last on purpose.
"""
import ctypes

import pytest
import torch

from bidirectional_mamba_state_b200 import bdscan as bd
from bidirectional_mamba_state_b200 import workload as W
from parity import check_states, check_y

DEV = "cuda:0"

SHAPES = {
    # tensor-core path: bf16, P = 64, N = 128, T = 32
    "tensor_core": W.Shape(batch=4, seqlen=32, nheads=8, headdim=64, dstate=128, ngroups=2,
                           block_len=32, chunk_len=32, in_dtype="bf16"),
    # generic path: fp32 inputs, small P and N
    "generic": W.Shape(batch=2, seqlen=16, nheads=4, headdim=16, dstate=32, ngroups=1,
                       block_len=16, chunk_len=16, in_dtype="fp32"),
}


def _noalloc(s, f, r, state_in, y, state_out):
    dev = torch.device(DEV)
    cs, cf, cr = bd.c_shape(s), bd.c_dir(s, f, dev), bd.c_dir(s, r, dev)
    return bd.bdscan_block_step_noalloc(ctypes.byref(cs), ctypes.byref(cf), ctypes.byref(cr),
                                        state_in.data_ptr(), y.data_ptr(), state_out.data_ptr(),
                                        torch.cuda.current_stream().cuda_stream)


@pytest.mark.gpu
@pytest.mark.parametrize("name", sorted(SHAPES))
def test_noalloc_step_matches_block_step(name):
    s = SHAPES[name]
    for call in range(2):  # two calls in a row share the library's scratch buffer
        f, r = W.make_streams(s, 40 + call, streams=(W.CLEAN_FWD, W.CLEAN_REV), device=DEV)
        state = W.make_state(s, 40 + call, device=DEV)
        y_ref, so_ref = bd.block_step(s, f, r, state, state_out=True)
        y = torch.full_like(y_ref, float("nan"))
        so = torch.full_like(so_ref, float("nan"))
        rc = _noalloc(s, f, r, state, y, so)
        assert rc == 0, bd.bdscan_status_string(rc)
        torch.cuda.synchronize()
        check_y(y, y_ref.double().cpu().numpy(), what=f"{name} y, call {call}")
        check_states(so, so_ref.double().cpu().numpy(), f"{name} state_out, call {call}")
        scratch = bd.bdscan_noalloc_scratch()
        assert scratch
        assert bd.bdscan_check_status(scratch, torch.cuda.current_stream().cuda_stream) == 0


@pytest.mark.gpu
def test_noalloc_step_rejects_shapes_beyond_its_scratch():
    # batch * ngroups = 1040 > 1024 tensor-core tiles' worth of scratch; rejected
    # on the host before anything is launched
    s = W.Shape(batch=1040, seqlen=32, nheads=1, headdim=64, dstate=128, ngroups=1, block_len=32,
                chunk_len=32, in_dtype="bf16")
    f, r = W.make_streams(s, 50, streams=(W.CLEAN_FWD, W.CLEAN_REV), device=DEV)
    state = W.make_state(s, 50, device=DEV)
    y = torch.empty((s.batch, s.seqlen, s.nheads, s.headdim), device=DEV)
    so = torch.empty_like(state)
    assert _noalloc(s, f, r, state, y, so) == -7
