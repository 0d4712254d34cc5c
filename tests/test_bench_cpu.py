"""Host-side helpers of bench.py on CPU: the oracle rates that the secondary
lines carry (backward, short convolution, gated RMSNorm) run on one batch row
of host copies of the line's inputs, and a failing one is reported in its line."""
import torch

import bench
from bidirectional_mamba_state_b200 import workload as W

S = W.Shape(batch=2, seqlen=64, nheads=2, headdim=16, dstate=16, ngroups=1, block_len=16,
            chunk_len=16, in_dtype="bf16")


def _check(r, sample_word):
    assert r["kind"] == "oracle" and "error" not in r, r
    assert r["unit"] == "tokens/s" and r["value"] > 0 and r["cores"] >= 1
    assert sample_word in r["sample"] and f"1 of {S.batch} batch rows" in r["sample"]


def test_backward_oracle_rate():
    dirs = W.make_streams(S, 3, device="cpu")
    g = torch.Generator().manual_seed(1)
    dyn = torch.randn((S.batch, S.seqlen, S.nheads, S.headdim), generator=g)
    dyc = torch.randn(dyn.shape, generator=g)
    _check(bench._backward_oracle_rate(S, dirs, dyn, dyc), "allblock_backward")


def test_conv_oracle_rate():
    dirs = [W.make_conv_dir(S, 4, 3, stream=i, device="cpu") for i in range(4)]
    _check(bench._conv_oracle_rate(S, 4, dirs), "conv_allblock")


def test_norm_oracle_rate():
    g = torch.Generator().manual_seed(2)
    yn = torch.randn((S.batch, S.seqlen, S.nheads, S.headdim), generator=g)
    z = torch.randn(yn.shape, generator=g).to(torch.bfloat16)
    _check(bench._norm_oracle_rate(S, yn, z, torch.ones(S.nheads * S.headdim)), "gated_rmsnorm")


def test_guarded_reports_failure():
    r = bench._guarded(lambda: 1 // 0)
    assert r["kind"] == "oracle" and "ZeroDivisionError" in r["error"]
