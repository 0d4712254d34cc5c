"""Algorithmic byte and flop counts of the three operations (the roofline model).

Bytes count every input read once, every output written once and every
boundary state written once; a re-read of anything is not counted (it is the
kernel's cost, not the algorithm's).  Flops are those of the chunked form
with block-sized chunks (the form the tensor-core kernel computes):
  per (b, h, block) of T tokens:  S = (w o X)^T B  -> 2 T P N    (clean forward)
                                  Y_off = C h^T      -> 2 T N P    (per forward stream)
                                  Y_diag = M X       -> 2 T T P    (per direction)
  per (b, g, block):              C B^T              -> 2 T T N    (per direction)
This is the memory-bound throughput model of "Breaking the Bottleneck with
DiffuApriel", section 4.2 (T_max ~ M_p / bytes per token), applied per call.
"""
from __future__ import annotations

from .workload import Shape


def _elt(dtype: str) -> int:
    return 2 if dtype == "bf16" else 4


def dir_bytes(s: Shape) -> int:
    e = _elt(s.in_dtype)
    return e * s.batch * s.seqlen * (s.nheads * s.headdim + s.nheads + 2 * s.ngroups * s.dstate) \
        + 8 * s.nheads


def y_bytes(s: Shape) -> int:
    return _elt(s.out_dtype) * s.batch * s.seqlen * s.nheads * s.headdim


def state_bytes(s: Shape) -> int:
    return 4 * s.batch * s.nheads * s.headdim * s.dstate


def allblock_bytes(s: Shape, with_clean_y: bool = True, with_rev: bool = True, gated: bool = False) -> int:
    """gated: every direction also reads its gate z (the input dtype, like x)."""
    ndir = 4 if with_rev else 2
    z = ndir * _elt(s.in_dtype) * s.batch * s.seqlen * s.nheads * s.headdim if gated else 0
    return ndir * dir_bytes(s) + z + (2 if with_clean_y else 1) * y_bytes(s) + \
        s.nblocks * state_bytes(s)


def prefix_bytes(s: Shape, with_rev: bool = True, block_states: bool = True,
                 final_state: bool = True, with_h0: bool = False) -> int:
    return (2 if with_rev else 1) * dir_bytes(s) + y_bytes(s) + \
        (s.nblocks * state_bytes(s) if block_states else 0) + \
        (state_bytes(s) if final_state else 0) + (state_bytes(s) if with_h0 else 0)


def block_step_bytes(s: Shape, with_rev: bool = True, commit: bool = False) -> int:
    return (2 if with_rev else 1) * dir_bytes(s) + y_bytes(s) + state_bytes(s) * (2 if commit else 1)


def allblock_flops(s: Shape) -> int:
    B, H, P, N, G, T, K = s.batch, s.nheads, s.headdim, s.dstate, s.ngroups, s.block_len, s.nblocks
    per_bhk = 2 * T * P * N + 2 * (2 * T * N * P) + 4 * (2 * T * T * P)
    per_bgk = 4 * (2 * T * T * N)
    return B * K * (H * per_bhk + G * per_bgk)


def prefix_flops(s: Shape, with_rev: bool = True) -> int:
    B, H, P, N, G, T, K = s.batch, s.nheads, s.headdim, s.dstate, s.ngroups, s.block_len, s.nblocks
    nd = 2 if with_rev else 1
    per_bhk = 2 * T * P * N + 2 * T * N * P + nd * 2 * T * T * P
    return B * K * (H * per_bhk + G * nd * 2 * T * T * N)


def allblock_backward_bytes(s: Shape, with_dy_clean: bool = True, with_dstates: bool = False) -> int:
    """Inputs of the four directions, dy (output dtype), the forward's boundary
    states, (dstates), and fp32 gradients of every input plus dh0."""
    B, L, H, P, N, G = s.batch, s.seqlen, s.nheads, s.headdim, s.dstate, s.ngroups
    grads = 4 * (4 * B * L * H * P + 4 * B * L * H + 2 * 4 * B * L * G * N + 8 * H)
    return 4 * dir_bytes(s) + (2 if with_dy_clean else 1) * y_bytes(s) + \
        s.nblocks * state_bytes(s) * (2 if with_dstates else 1) + grads + state_bytes(s)


def allblock_backward_flops(s: Shape) -> int:
    """Flops of the per-block closed-form derivative (per (b, h, block)):
    Gram matrices C B^T and dy x^T of every direction, the products with the
    start state (forward directions) and with the end-state gradient (clean
    forward), the intra-block sums for dx, dB, dC and the start-state gradient."""
    B, H, P, N, T, K = s.batch, s.nheads, s.headdim, s.dstate, s.block_len, s.nblocks
    gram = 2 * T * T * (N + P)              # C B^T and dy x^T
    intra = 2 * T * T * (P + 2 * N) // 2    # dx, dC, dB sums over the causal triangle
    tpn = 2 * T * P * N
    per = (gram + intra + 5 * tpn) + (gram + intra + 3 * tpn) + 2 * (gram + intra)
    return B * H * K * per


def conv_channels(s: Shape) -> int:
    return s.nheads * s.headdim + 2 * s.ngroups * s.dstate


def conv_dir_bytes(s: Shape, width: int) -> int:
    """One direction of the short convolution: pre-convolution rows read once,
    outputs written once (input dtype), taps and bias (fp32)."""
    cx = conv_channels(s)
    return 2 * _elt(s.in_dtype) * s.batch * s.seqlen * cx + 4 * cx * (width + 1)


def conv_state_bytes(s: Shape, width: int) -> int:
    return _elt(s.in_dtype) * s.batch * (width - 1) * conv_channels(s)


def conv_bytes(s: Shape, width: int, ndir: int, state_in: bool = False, state_out: bool = False) -> int:
    """A convolution call over ``ndir`` directions (halo rows a tile shares
    with its neighbour, or a noisy block with the clean stream, are re-reads
    and not counted)."""
    return ndir * conv_dir_bytes(s, width) + conv_state_bytes(s, width) * (int(state_in) + int(state_out))


def conv_flops(s: Shape, width: int, ndir: int) -> int:
    """2 flops per tap per output (SiLU not counted)."""
    return ndir * 2 * width * s.batch * s.seqlen * conv_channels(s)


def norm_bytes(s: Shape, gated: bool = True) -> int:
    """Gated RMSNorm of one scan output: y (out dtype) and z (input dtype) read
    once, the bf16 result written once, the fp32 weights."""
    n = s.batch * s.seqlen * s.nheads * s.headdim
    return n * (_elt(s.out_dtype) + (_elt(s.in_dtype) if gated else 0) + 2) + 4 * s.nheads * s.headdim
