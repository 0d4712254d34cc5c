"""CPU checks of the seeded input generators that the device path and the
oracle share: reproducible per (seed, layer, stream, tensor), independent
across streams, with the documented shapes, dtypes and distributions."""
import math

import torch

from bidirectional_mamba_state_b200 import workload as W


def test_streams_are_reproducible_and_independent():
    s = W.WORKLOADS["tiny"]
    a = W.make_streams(s, seed=3)
    b = W.make_streams(s, seed=3)
    for da, db in zip(a, b):
        for k in da:
            assert torch.equal(da[k], db[k]), k
    assert not torch.equal(a[0]["x"], a[2]["x"])      # clean and noisy streams differ
    assert not torch.equal(a[0]["x"], W.make_dir(s, seed=4)["x"])


def test_shapes_dtypes_and_ranges():
    s = W.WORKLOADS["87m_allblock"].with_(batch=2, seqlen=128)
    d = W.make_dir(s, seed=1)
    assert d["x"].shape == (2, 128, 24, 64) and d["x"].dtype == torch.bfloat16
    assert d["B"].shape == (2, 128, 1, 128) and d["C"].shape == (2, 128, 1, 128)
    assert d["dt"].shape == (2, 128, 24) and (d["dt"].float() > 0).all()
    assert d["A"].dtype == torch.float32 and (d["A"] <= -1.0).all() and (d["A"] >= -16.0).all()
    assert abs(float(d["x"].float().std()) - 1.0) < 0.05
    assert abs(float(d["B"].float().std()) - 0.25) < 0.02
    c = W.make_conv_dir(s, 4, seed=1)
    cx = 24 * 64 + 2 * 128
    assert c["weight"].shape == (cx, 4) and c["bias"].shape == (cx,)
    bound = 1.0 / math.sqrt(4)
    assert float(c["weight"].abs().max()) <= bound and float(c["bias"].abs().max()) <= bound
    st = W.make_conv_state(s, 4, seed=1)
    assert st.shape == (2, 3, cx) and st.dtype == torch.bfloat16
