"""Seeded synthetic inputs for the block-diffusion scan.

This module only draws random tensors; it holds none of the scan's arithmetic,
so both the device path's tests/benchmark and the CPU oracle can consume its
output.  Every tensor is drawn in fp32 from its own stream
``(seed, layer, stream, tensor)`` and rounded once to the input dtype.

Value distributions (the workloads' stated recipe):
  x ~ N(0, 1);  B, C ~ N(0, 0.25) (std 1/sqrt(16));  dt = softplus(u),
  u ~ N(-3, 0.5);  A_h = -exp(U(0, ln 16)) (fp32);  D_h ~ N(0, 1) (fp32);
  z ~ N(0, 1) (gated runs only).  The reverse direction and the noisy stream
  are independent draws.
Short convolution in front of the scan: pre-convolution x, B, C ~ N(0, 1)
  (the input projection's unit-scale outputs); taps and bias ~ U(-1/sqrt(W),
  1/sqrt(W)) (the usual initialisation bound of a depthwise filter of W taps,
  fan-in W); conv state ~ N(0, 1) rounded to the input dtype.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, asdict, replace

import torch

# stream ids
CLEAN_FWD, CLEAN_REV, NOISY_FWD, NOISY_REV = 0, 1, 2, 3
_TENSOR_IDS = {"x": 0, "dt": 1, "B": 2, "C": 3, "z": 4, "A": 5, "D": 6, "h0": 7,
               "conv_x": 8, "conv_B": 9, "conv_C": 10, "conv_w": 11, "conv_b": 12, "conv_state": 13}


@dataclass(frozen=True)
class Shape:
    batch: int
    seqlen: int
    nheads: int
    headdim: int
    dstate: int
    ngroups: int = 1
    block_len: int = 32
    chunk_len: int = 32
    in_dtype: str = "bf16"   # "bf16" | "fp32"
    out_dtype: str = "fp32"  # "fp32" | "bf16"

    def as_dict(self) -> dict:
        return asdict(self)

    def with_(self, **kw) -> "Shape":
        return replace(self, **kw)

    @property
    def nblocks(self) -> int:
        return self.seqlen // self.block_len


# The five workloads, by what they are.  Configs 4 and 5 leave G and Q unstated;
# G = 1 and Q = 128 are taken, as in the 350M workload.
WORKLOADS = {
    "tiny": Shape(1, 256, 4, 16, 16, 1, 32, 32, "fp32"),
    "87m_allblock": Shape(16, 1024, 24, 64, 128, 1, 32, 64, "bf16"),
    "350m_allblock": Shape(4, 8192, 32, 64, 128, 1, 32, 128, "bf16"),
    "700m_prefill_8k": Shape(1, 8192, 48, 64, 128, 1, 32, 128, "bf16"),
    "700m_prefill_32k": Shape(1, 32768, 48, 64, 128, 1, 32, 128, "bf16"),
    "700m_prefill_64k": Shape(1, 65536, 48, 64, 128, 1, 32, 128, "bf16"),
    "700m_step": Shape(1, 32, 48, 64, 128, 1, 32, 32, "bf16"),
    "3b_prefill_256k": Shape(1, 262144, 80, 64, 128, 1, 32, 128, "bf16"),
    "3b_step_b1": Shape(1, 32, 80, 64, 128, 1, 32, 32, "bf16"),
    "3b_step_b64": Shape(64, 32, 80, 64, 128, 1, 32, 32, "bf16"),
}
# seed = workload index - 1 (the tiny workload is seed 0)
SEEDS = {"tiny": 0, "87m_allblock": 1, "350m_allblock": 2, "700m_prefill_8k": 3,
         "700m_prefill_32k": 3, "700m_prefill_64k": 3, "700m_step": 3,
         "3b_prefill_256k": 4, "3b_step_b1": 4, "3b_step_b64": 4}
LAYERS = {"700m": 24, "3b": 40}


def _dtype(name: str) -> torch.dtype:
    return {"bf16": torch.bfloat16, "fp32": torch.float32}[name]


def _gen(seed: int, layer: int, stream: int, tensor: str, device) -> torch.Generator:
    g = torch.Generator(device=device)
    # distinct, reproducible 63-bit stream per (seed, layer, stream, tensor)
    key = (((seed * 1009 + layer) * 31 + stream) * 17 + _TENSOR_IDS[tensor]) * 2654435761
    g.manual_seed(key % (2 ** 63 - 1))
    return g


def _normal(shape, mean, std, g, device):
    return torch.randn(shape, generator=g, device=device, dtype=torch.float32) * std + mean


def make_dir(shape: Shape, seed: int = 0, layer: int = 0, stream: int = CLEAN_FWD,
             device="cpu", gated: bool = False, ssm_zero_decay: bool = False) -> dict:
    """Draw one direction's inputs (x, dt, B, C, [z], A, D) for ``shape``."""
    Bsz, L, H, P, N, G = (shape.batch, shape.seqlen, shape.nheads, shape.headdim,
                          shape.dstate, shape.ngroups)
    dev = torch.device(device)
    dt_in = _dtype(shape.in_dtype)
    d = {}
    d["x"] = _normal((Bsz, L, H, P), 0.0, 1.0, _gen(seed, layer, stream, "x", dev), dev).to(dt_in)
    u = _normal((Bsz, L, H), -3.0, 0.5, _gen(seed, layer, stream, "dt", dev), dev)
    d["dt"] = torch.nn.functional.softplus(u).to(dt_in)
    d["B"] = _normal((Bsz, L, G, N), 0.0, 0.25, _gen(seed, layer, stream, "B", dev), dev).to(dt_in)
    d["C"] = _normal((Bsz, L, G, N), 0.0, 0.25, _gen(seed, layer, stream, "C", dev), dev).to(dt_in)
    if gated:
        d["z"] = _normal((Bsz, L, H, P), 0.0, 1.0, _gen(seed, layer, stream, "z", dev), dev).to(dt_in)
    gA = _gen(seed, layer, stream, "A", dev)
    uA = torch.rand((H,), generator=gA, device=dev, dtype=torch.float32) * math.log(16.0)
    d["A"] = -torch.exp(uA)
    if ssm_zero_decay:
        d["A"] = torch.zeros_like(d["A"])
    d["D"] = _normal((H,), 0.0, 1.0, _gen(seed, layer, stream, "D", dev), dev)
    return d


def make_state(shape: Shape, seed: int = 0, layer: int = 0, scale: float = 1.0,
               device="cpu") -> torch.Tensor:
    """A random fp32 cached state [B, H, P, N] (used for h0 / state_in in tests)."""
    dev = torch.device(device)
    g = _gen(seed, layer, 9, "h0", dev)
    return _normal((shape.batch, shape.nheads, shape.headdim, shape.dstate), 0.0, scale, g, dev)


def make_streams(shape: Shape, seed: int = 0, layer: int = 0, device="cpu", gated: bool = False,
                 streams=(CLEAN_FWD, CLEAN_REV, NOISY_FWD, NOISY_REV)) -> list:
    return [make_dir(shape, seed, layer, s, device, gated) for s in streams]


def sub_batch_block(d: dict, t0: int, t1: int) -> dict:
    """Slice tokens [t0, t1) out of a direction (a view-free contiguous copy)."""
    out = {}
    for k, v in d.items():
        if k in ("A", "D"):
            out[k] = v
        else:
            out[k] = v[:, t0:t1].contiguous()
    return out


def make_conv_dir(shape: Shape, width: int = 4, seed: int = 0, layer: int = 0, stream: int = CLEAN_FWD,
                  device="cpu", bias: bool = True) -> dict:
    """Draw one direction's short-convolution inputs: pre-convolution x, B, C
    (input dtype), weight [H*P + 2*G*N][width] and bias (fp32)."""
    Bsz, L, H, P, N, G = (shape.batch, shape.seqlen, shape.nheads, shape.headdim,
                          shape.dstate, shape.ngroups)
    dev = torch.device(device)
    dt_in = _dtype(shape.in_dtype)
    cx = H * P + 2 * G * N
    d = {"x": _normal((Bsz, L, H, P), 0.0, 1.0, _gen(seed, layer, stream, "conv_x", dev), dev).to(dt_in),
         "B": _normal((Bsz, L, G, N), 0.0, 1.0, _gen(seed, layer, stream, "conv_B", dev), dev).to(dt_in),
         "C": _normal((Bsz, L, G, N), 0.0, 1.0, _gen(seed, layer, stream, "conv_C", dev), dev).to(dt_in)}
    bound = 1.0 / math.sqrt(width)
    gw = _gen(seed, layer, stream, "conv_w", dev)
    d["weight"] = (torch.rand((cx, width), generator=gw, device=dev, dtype=torch.float32) * 2 - 1) * bound
    if bias:
        gb = _gen(seed, layer, stream, "conv_b", dev)
        d["bias"] = (torch.rand((cx,), generator=gb, device=dev, dtype=torch.float32) * 2 - 1) * bound
    return d


def make_conv_state(shape: Shape, width: int = 4, seed: int = 0, layer: int = 0, device="cpu") -> torch.Tensor:
    """A random conv state [B, width-1, H*P + 2*G*N] in the input dtype."""
    dev = torch.device(device)
    cx = shape.nheads * shape.headdim + 2 * shape.ngroups * shape.dstate
    g = _gen(seed, layer, 9, "conv_state", dev)
    return _normal((shape.batch, width - 1, cx), 0.0, 1.0, g, dev).to(_dtype(shape.in_dtype))
