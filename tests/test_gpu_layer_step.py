"""The selective-scan core of one Mamba layer's denoising step, composed through
the public API the way a decoder calls it: the short convolution of both
directions from the cached conv state writes the scan's x, B, C in place, the
scan continues from the cached state (forward) with the block-local reverse,
the committed conv and scan states replace the cache, and the gated RMSNorm
turns the summed output into bf16.  Each stage is checked against the oracle
on that stage's actual device inputs, so the hand-offs (layouts, in-place
outputs, state updates) are what is tested."""
import numpy as np
import pytest
import torch

import oracle
from bidirectional_mamba_state_b200 import bdscan as bd
from bidirectional_mamba_state_b200 import workload as W
from parity import check_states, check_y

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


@pytest.mark.parametrize("name", ["700m_step", "3b_step_b1"])
def test_layer_step_composed(name):
    st = W.WORKLOADS[name]
    conv = [W.make_conv_dir(st, 4, 3, stream=i, device=DEV) for i in (0, 1)]
    scan = W.make_streams(st, 3, device=DEV, streams=(W.CLEAN_FWD, W.CLEAN_REV))
    conv_state = W.make_conv_state(st, 4, 3, device=DEV)
    ssm_state = W.make_state(st, 3, device=DEV)
    conv_state0, ssm_state0 = conv_state.clone(), ssm_state.clone()
    # conv + SiLU into the scan's inputs, committing the conv state in place
    bd.conv_prefix(st, 4, True, conv[0], conv[1], conv_state, conv_state,
                   out_fwd={k: scan[0][k] for k in "xBC"}, out_rev={k: scan[1][k] for k in "xBC"})
    # scan step from the cache, committing the scan state in place
    y, _ = bd.block_step(st, scan[0], scan[1], ssm_state, state_out=ssm_state)
    z = torch.randn(y.shape, device=DEV, generator=torch.Generator(device=DEV).manual_seed(4)).to(torch.bfloat16)
    w = 1.0 + 0.1 * torch.randn(st.nheads * st.headdim, device=DEV, generator=torch.Generator(device=DEV).manual_seed(5))
    out = bd.gated_rmsnorm(st, y, z, w)
    torch.cuda.synchronize()
    # stage 1: the convolution and the committed conv state
    rf, rr, rso = oracle.conv_prefix(st.as_dict(), 4, True, conv[0], conv[1], conv_state0, want_state_out=True)
    for got, ref in ((scan[0], rf), (scan[1], rr)):
        for k in "xBC":
            a = got[k].double().cpu().numpy()
            assert np.max(np.abs(a - ref[k])) <= 2.0 ** -8 * np.max(np.abs(ref[k])) + 1e-6, f"conv {k}"
    assert np.array_equal(conv_state.double().cpu().numpy(), rso), "committed conv state"
    # stage 2: the scan on the device's convolution outputs, and the committed state
    ry, rs = oracle.block_step(st.as_dict(), scan[0], scan[1], ssm_state0, want_state_out=True)
    check_y(y, ry, what="layer step y")
    check_states(ssm_state, rs, "committed scan state")
    # stage 3: the norm of the device's summed output
    rn = oracle.gated_rmsnorm(y, z, w, 1, 1e-5)
    a = out.double().cpu().numpy()
    assert np.all(np.abs(a - rn) <= (2.0 ** -8 + 4e-4) * np.abs(rn) + 1e-6 * np.max(np.abs(rn))), "norm"
