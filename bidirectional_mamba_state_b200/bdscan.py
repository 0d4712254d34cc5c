"""Python binding of libbdscan (ctypes; argument marshalling only).

The functions named ``bdscan_*`` mirror the C ABI in ``include/bdscan.h`` one to
one and take raw pointers / ctypes structs.  ``prefix``, ``block_step`` and
``allblock`` are the torch-facing conveniences: they check devices, dtypes and
contiguity, allocate the outputs and the workspace with torch, and call the C
ABI on the current torch CUDA stream.  Every step of the scan runs in the
library's CUDA kernels; there is no CPU or PyTorch fallback, and a missing
library is an error.
"""
from __future__ import annotations

import ctypes
import functools
import os
import re
import threading

import torch

from .workload import Shape

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libbdscan.so")
HEADER = os.path.join(os.path.dirname(_PKG), "include", "bdscan.h")

BDSCAN_BF16, BDSCAN_FP32 = 0, 1
BDSCAN_OP_PREFIX, BDSCAN_OP_BLOCK_STEP, BDSCAN_OP_ALLBLOCK, BDSCAN_OP_ALLBLOCK_BACKWARD = 0, 1, 2, 3
BDSCAN_OP_CONV_PREFIX, BDSCAN_OP_CONV_ALLBLOCK, BDSCAN_OP_GATED_RMSNORM = 4, 5, 6
BDSCAN_OP_CONV_BLOCK_STEP = 7
STATUS = {0: "BDSCAN_OK", -1: "BDSCAN_ERR_INVALID_ARG", -2: "BDSCAN_ERR_UNSUPPORTED_SHAPE",
          -3: "BDSCAN_ERR_MISALIGNED", -4: "BDSCAN_ERR_WORKSPACE", -5: "BDSCAN_ERR_CUDA",
          -6: "BDSCAN_ERR_TIMEOUT", -7: "BDSCAN_ERR_SCRATCH_LIMIT"}


class bdscan_shape_t(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int64) for n in ("batch", "seqlen", "nheads", "headdim", "dstate",
                                               "ngroups", "block_len", "chunk_len")] + \
               [("in_dtype", ctypes.c_int32), ("out_dtype", ctypes.c_int32)]


class bdscan_dir_t(ctypes.Structure):
    _fields_ = [("x", ctypes.c_void_p), ("dt", ctypes.c_void_p), ("B", ctypes.c_void_p),
                ("C", ctypes.c_void_p), ("z", ctypes.c_void_p), ("A", ctypes.c_void_p),
                ("D", ctypes.c_void_p)]


class bdscan_grad_t(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in ("dx", "ddt", "dB", "dC", "dA", "dD")]


class bdscan_conv_t(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in ("x", "B", "C", "weight", "bias", "x_out", "B_out", "C_out")]


class BdscanError(RuntimeError):
    def __init__(self, fn: str, status: int, msg: str):
        super().__init__(f"{fn} failed: {STATUS.get(status, status)} ({msg})")
        self.status = status


_lock = threading.Lock()
_lib = None


def lib() -> ctypes.CDLL:
    """Load libbdscan.so (built in-tree by ``bidirectional_mamba_state_b200.build``)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError(f"libbdscan.so is not built ({LIB_PATH}); run "
                                   "`python -m bidirectional_mamba_state_b200.build` or "
                                   "`__graft_entry__.build()`")
            L = ctypes.CDLL(LIB_PATH)
            vp, sz = ctypes.c_void_p, ctypes.c_size_t
            sp, dp = ctypes.POINTER(bdscan_shape_t), ctypes.POINTER(bdscan_dir_t)
            L.bdscan_prefix.argtypes = [sp, dp, dp, vp, vp, vp, vp, vp, sz, vp]
            L.bdscan_block_step.argtypes = [sp, dp, dp, vp, vp, vp, vp, sz, vp]
            L.bdscan_allblock.argtypes = [sp, dp, dp, dp, dp, vp, vp, vp, vp, vp, sz, vp]
            gp = ctypes.POINTER(bdscan_grad_t)
            L.bdscan_allblock_backward.argtypes = [sp, dp, dp, dp, dp, vp, vp, vp, vp, vp, gp, gp, gp, gp,
                                                   vp, vp, sz, vp]
            cp, ci = ctypes.POINTER(bdscan_conv_t), ctypes.c_int
            L.bdscan_conv_prefix.argtypes = [sp, ci, ci, cp, cp, vp, vp, vp]
            L.bdscan_conv_allblock.argtypes = [sp, ci, ci, cp, cp, cp, cp, vp, vp]
            L.bdscan_conv_block_step.argtypes = [sp, ci, ci, cp, cp, vp, dp, dp, vp, vp, vp, sz, vp]
            L.bdscan_gated_rmsnorm.argtypes = [sp, vp, vp, vp, ctypes.c_int64, ctypes.c_float, vp, vp]
            for fn in ("bdscan_prefix", "bdscan_block_step", "bdscan_allblock", "bdscan_allblock_backward",
                       "bdscan_conv_prefix", "bdscan_conv_allblock", "bdscan_conv_block_step",
                       "bdscan_gated_rmsnorm",
                       "bdscan_check_status", "bdscan_version"):
                getattr(L, fn).restype = ctypes.c_int
            L.bdscan_workspace_size.argtypes = [sp, ctypes.c_int]
            L.bdscan_workspace_size.restype = ctypes.c_size_t
            L.bdscan_kernel_launches.argtypes = [sp, ctypes.c_int]
            L.bdscan_kernel_launches.restype = ctypes.c_int
            L.bdscan_block_step_noalloc.argtypes = [sp, dp, dp, vp, vp, vp, vp]
            L.bdscan_block_step_noalloc.restype = ctypes.c_int
            L.bdscan_noalloc_scratch.argtypes = []
            L.bdscan_noalloc_scratch.restype = ctypes.c_void_p
            L.bdscan_set_option.argtypes = [ctypes.c_int, ctypes.c_longlong]
            L.bdscan_set_option.restype = ctypes.c_longlong
            L.bdscan_get_option.argtypes = [ctypes.c_int]
            L.bdscan_get_option.restype = ctypes.c_longlong
            L.bdscan_check_status.argtypes = [vp, vp]
            L.bdscan_status_string.argtypes = [ctypes.c_int]
            L.bdscan_status_string.restype = ctypes.c_char_p
            _lib = L
    return _lib


def header_symbols() -> list[str]:
    """Names of the functions declared in include/bdscan.h."""
    with open(HEADER) as f:
        text = re.sub(r"/\*.*?\*/", "", f.read(), flags=re.S)
    return sorted(set(re.findall(r"\b(bdscan_\w+)\s*\(", text)))


# ----------------------------------------------------------------------------- raw C ABI
def bdscan_prefix(shape, fwd, rev, h0, y, block_states, final_state, ws, ws_bytes, stream) -> int:
    return lib().bdscan_prefix(shape, fwd, rev, h0, y, block_states, final_state, ws, ws_bytes, stream)


def bdscan_block_step(shape, fwd, rev, state_in, y, state_out, ws, ws_bytes, stream) -> int:
    return lib().bdscan_block_step(shape, fwd, rev, state_in, y, state_out, ws, ws_bytes, stream)


def bdscan_allblock(shape, cf, cr, nf, nr, h0, y_clean, y_noisy, block_states, ws, ws_bytes,
                    stream) -> int:
    return lib().bdscan_allblock(shape, cf, cr, nf, nr, h0, y_clean, y_noisy, block_states, ws,
                                 ws_bytes, stream)


def bdscan_allblock_backward(shape, cf, cr, nf, nr, h0, block_states, dy_clean, dy_noisy, dstates,
                             g_cf, g_cr, g_nf, g_nr, dh0, ws, ws_bytes, stream) -> int:
    return lib().bdscan_allblock_backward(shape, cf, cr, nf, nr, h0, block_states, dy_clean, dy_noisy,
                                          dstates, g_cf, g_cr, g_nf, g_nr, dh0, ws, ws_bytes, stream)


def bdscan_conv_block_step(shape, width, silu, conv_fwd, conv_rev, conv_state_in, fwd, rev, state_in, y, ws,
                           ws_bytes, stream) -> int:
    return lib().bdscan_conv_block_step(shape, width, silu, conv_fwd, conv_rev, conv_state_in, fwd, rev, state_in,
                                        y, ws, ws_bytes, stream)


def bdscan_conv_prefix(shape, width, silu, fwd, rev, conv_state_in, conv_state_out, stream) -> int:
    return lib().bdscan_conv_prefix(shape, width, silu, fwd, rev, conv_state_in, conv_state_out, stream)


def bdscan_conv_allblock(shape, width, silu, cf, cr, nf, nr, conv_state_in, stream) -> int:
    return lib().bdscan_conv_allblock(shape, width, silu, cf, cr, nf, nr, conv_state_in, stream)


def bdscan_gated_rmsnorm(shape, y, z, weight, groups, eps, out, stream) -> int:
    return lib().bdscan_gated_rmsnorm(shape, y, z, weight, groups, eps, out, stream)


def bdscan_block_step_noalloc(shape, fwd, rev, state_in, y, state_out, stream) -> int:
    return lib().bdscan_block_step_noalloc(shape, fwd, rev, state_in, y, state_out, stream)


def bdscan_noalloc_scratch() -> int | None:
    return lib().bdscan_noalloc_scratch()


def bdscan_workspace_size(shape, op: int) -> int:
    return int(lib().bdscan_workspace_size(shape, op))


def bdscan_kernel_launches(shape, op: int) -> int:
    return int(lib().bdscan_kernel_launches(shape, op))


def bdscan_check_status(ws, stream) -> int:
    return int(lib().bdscan_check_status(ws, stream))


def bdscan_status_string(status: int) -> str:
    return lib().bdscan_status_string(int(status)).decode()


def bdscan_version() -> int:
    return int(lib().bdscan_version())


BDSCAN_OPT_WAIT_TIMEOUT_NS, BDSCAN_OPT_FORCE_GENERIC, BDSCAN_OPT_VERBOSE, BDSCAN_OPT_CB_PREPASS = 0, 1, 2, 3


def bdscan_set_option(option: int, value: int) -> int:
    return int(lib().bdscan_set_option(int(option), int(value)))


def bdscan_get_option(option: int) -> int:
    return int(lib().bdscan_get_option(int(option)))


class option:
    """Context manager that sets a process-wide option and restores it."""

    def __init__(self, opt: int, value: int):
        self.opt, self.value = opt, value

    def __enter__(self):
        old = bdscan_set_option(self.opt, self.value)
        if old < 0 and self.opt != BDSCAN_OPT_WAIT_TIMEOUT_NS:
            raise BdscanError("bdscan_set_option", old, "bad option or value")
        self.old = old
        return self

    def __exit__(self, *exc):
        bdscan_set_option(self.opt, self.old)


# ----------------------------------------------------------------------------- torch-facing
_DT = {"bf16": (torch.bfloat16, BDSCAN_BF16), "fp32": (torch.float32, BDSCAN_FP32)}


def c_shape(s: Shape) -> bdscan_shape_t:
    return bdscan_shape_t(s.batch, s.seqlen, s.nheads, s.headdim, s.dstate, s.ngroups, s.block_len,
                          s.chunk_len, _DT[s.in_dtype][1], _DT[s.out_dtype][1])


def _ptr(t) -> int | None:
    return None if t is None else t.data_ptr()


def _check_tensor(name, t, shape, dtype, device):
    if t is None:
        raise ValueError(f"{name} is required")
    if t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    if t.dtype != dtype:
        raise ValueError(f"{name} has dtype {t.dtype}, expected {dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def c_dir(s: Shape, d: dict | None, device) -> bdscan_dir_t | None:
    if d is None:
        return None
    tin = _DT[s.in_dtype][0]
    B, L, H, P, N, G = s.batch, s.seqlen, s.nheads, s.headdim, s.dstate, s.ngroups
    _check_tensor("x", d["x"], (B, L, H, P), tin, device)
    _check_tensor("dt", d["dt"], (B, L, H), tin, device)
    _check_tensor("B", d["B"], (B, L, G, N), tin, device)
    _check_tensor("C", d["C"], (B, L, G, N), tin, device)
    if d.get("z") is not None:
        _check_tensor("z", d["z"], (B, L, H, P), tin, device)
    _check_tensor("A", d["A"], (H,), torch.float32, device)
    _check_tensor("D", d["D"], (H,), torch.float32, device)
    return bdscan_dir_t(_ptr(d["x"]), _ptr(d["dt"]), _ptr(d["B"]), _ptr(d["C"]), _ptr(d.get("z")),
                        _ptr(d["A"]), _ptr(d["D"]))


def _ref(x):
    return ctypes.byref(x) if x is not None else None


def _stream(device, stream=None) -> int:
    s = stream if stream is not None else torch.cuda.current_stream(device)
    return s.cuda_stream


@functools.lru_cache(maxsize=256)
def _ws_bytes(s: Shape, op: int) -> int:
    return bdscan_workspace_size(ctypes.byref(c_shape(s)), op)


def _check_ws(ws, s: Shape, op: int, device):
    """A caller-provided workspace: a contiguous uint8 tensor on ``device``
    with at least bdscan_workspace_size(shape, op) bytes."""
    if ws.device != device:
        raise ValueError(f"ws is on {ws.device}, expected {device}")
    if ws.dtype != torch.uint8 or ws.dim() != 1 or not ws.is_contiguous():
        raise ValueError("ws must be a contiguous 1-D uint8 tensor")
    need = _ws_bytes(s, op)
    if ws.numel() < need:
        raise ValueError(f"ws holds {ws.numel()} bytes, the call needs {need}")


def workspace(s: Shape, op: int, device) -> torch.Tensor:
    n = bdscan_workspace_size(ctypes.byref(c_shape(s)), op)
    if n == 0:
        raise BdscanError("bdscan_workspace_size", -2, "invalid shape or op")
    return torch.empty(((n + 255) // 256) * 256, dtype=torch.uint8, device=device)


def kernel_launches(s: Shape, op: int) -> int:
    """Kernels one call of ``op`` launches for shape ``s``."""
    return bdscan_kernel_launches(ctypes.byref(c_shape(s)), op)


def _raise(fn, rc):
    if rc != 0:
        raise BdscanError(fn, rc, bdscan_status_string(rc))


def _out(s: Shape, device):
    return torch.empty((s.batch, s.seqlen, s.nheads, s.headdim), device=device,
                       dtype=_DT[s.out_dtype][0])


def _state(s: Shape, device, K=None):
    if K is None:
        return torch.empty((s.batch, s.nheads, s.headdim, s.dstate), device=device, dtype=torch.float32)
    return torch.empty((s.batch, K, s.nheads, s.headdim, s.dstate), device=device, dtype=torch.float32)


def prefix(s: Shape, fwd: dict, rev: dict | None = None, h0=None, want_states: bool = True,
           want_final: bool = True, y=None, states=None, final=None, ws=None, stream=None):
    """Clean-prefix scan (prefill / commit).  Returns (y, block_states or None,
    final_state or None)."""
    dev = fwd["x"].device
    cs, cf, cr = c_shape(s), c_dir(s, fwd, dev), c_dir(s, rev, dev)
    if h0 is not None:
        _check_tensor("h0", h0, (s.batch, s.nheads, s.headdim, s.dstate), torch.float32, dev)
    B, L, H, P, N = s.batch, s.seqlen, s.nheads, s.headdim, s.dstate
    if y is None:
        y = _out(s, dev)
    _check_tensor("y", y, (B, L, H, P), _DT[s.out_dtype][0], dev)
    if states is None:
        states = _state(s, dev, s.nblocks) if want_states else None
    else:
        _check_tensor("states", states, (B, s.nblocks, H, P, N), torch.float32, dev)
    if final is None:
        final = _state(s, dev) if want_final else None
    else:
        _check_tensor("final", final, (B, H, P, N), torch.float32, dev)
    if ws is None:
        ws = workspace(s, BDSCAN_OP_PREFIX, dev)
    _check_ws(ws, s, BDSCAN_OP_PREFIX, dev)
    rc = bdscan_prefix(ctypes.byref(cs), ctypes.byref(cf), _ref(cr), _ptr(h0), _ptr(y), _ptr(states),
                       _ptr(final), _ptr(ws), ws.numel(), _stream(dev, stream))
    _raise("bdscan_prefix", rc)
    return y, states, final


def block_step(s: Shape, fwd: dict, rev: dict | None, state_in, state_out=None, y=None, ws=None,
               stream=None):
    """One denoising step of the active block from the cached state.  ``state_out``:
    None (no commit), a tensor (commit into it; may be ``state_in``) or True
    (allocate).  Returns (y, state_out or None)."""
    dev = fwd["x"].device
    cs, cf, cr = c_shape(s), c_dir(s, fwd, dev), c_dir(s, rev, dev)
    _check_tensor("state_in", state_in, (s.batch, s.nheads, s.headdim, s.dstate), torch.float32, dev)
    if state_out is True:
        state_out = _state(s, dev)
    elif state_out is not None:
        _check_tensor("state_out", state_out, (s.batch, s.nheads, s.headdim, s.dstate), torch.float32, dev)
    if y is None:
        y = _out(s, dev)
    _check_tensor("y", y, (s.batch, s.seqlen, s.nheads, s.headdim), _DT[s.out_dtype][0], dev)
    if ws is None:
        ws = workspace(s, BDSCAN_OP_BLOCK_STEP, dev)
    _check_ws(ws, s, BDSCAN_OP_BLOCK_STEP, dev)
    rc = bdscan_block_step(ctypes.byref(cs), ctypes.byref(cf), _ref(cr), _ptr(state_in), _ptr(y),
                           _ptr(state_out), _ptr(ws), ws.numel(), _stream(dev, stream))
    _raise("bdscan_block_step", rc)
    return y, state_out


def allblock(s: Shape, clean_fwd: dict, clean_rev: dict | None, noisy_fwd: dict,
             noisy_rev: dict | None, h0=None, want_clean: bool = True, y_clean=None, y_noisy=None,
             states=None, ws=None, stream=None):
    """All-block training pass.  Returns (y_clean or None, y_noisy, block_states)."""
    dev = clean_fwd["x"].device
    cs = c_shape(s)
    cf, cr = c_dir(s, clean_fwd, dev), c_dir(s, clean_rev, dev)
    nf, nr = c_dir(s, noisy_fwd, dev), c_dir(s, noisy_rev, dev)
    if h0 is not None:
        _check_tensor("h0", h0, (s.batch, s.nheads, s.headdim, s.dstate), torch.float32, dev)
    yshape, tout = (s.batch, s.seqlen, s.nheads, s.headdim), _DT[s.out_dtype][0]
    if y_clean is None:
        y_clean = _out(s, dev) if want_clean else None
    else:
        _check_tensor("y_clean", y_clean, yshape, tout, dev)
    if y_noisy is None:
        y_noisy = _out(s, dev)
    _check_tensor("y_noisy", y_noisy, yshape, tout, dev)
    if states is None:
        states = _state(s, dev, s.nblocks)
    _check_tensor("states", states, (s.batch, s.nblocks, s.nheads, s.headdim, s.dstate), torch.float32, dev)
    if ws is None:
        ws = workspace(s, BDSCAN_OP_ALLBLOCK, dev)
    _check_ws(ws, s, BDSCAN_OP_ALLBLOCK, dev)
    rc = bdscan_allblock(ctypes.byref(cs), ctypes.byref(cf), _ref(cr), ctypes.byref(nf), _ref(nr),
                         _ptr(h0), _ptr(y_clean), _ptr(y_noisy), _ptr(states), _ptr(ws), ws.numel(),
                         _stream(dev, stream))
    _raise("bdscan_allblock", rc)
    return y_clean, y_noisy, states


GRAD_KEYS = ("x", "dt", "B", "C", "A", "D")


def allblock_backward(s: Shape, clean_fwd: dict, clean_rev: dict | None, noisy_fwd: dict,
                      noisy_rev: dict | None, states, dy_noisy, dy_clean=None, dstates=None, h0=None,
                      want_dh0: bool = True, grads=None, ws=None, stream=None):
    """Backward of the all-block pass.  ``states`` is the forward call's block
    states; ``dy_*`` have the output dtype.  Returns (grads, dh0): grads[i]
    (i = clean fwd, clean rev, noisy fwd, noisy rev; None if absent) is a dict
    of fp32 tensors keyed like the inputs (x, dt, B, C, A, D)."""
    dev = clean_fwd["x"].device
    cs = c_shape(s)
    dirs = [clean_fwd, clean_rev, noisy_fwd, noisy_rev]
    cd = [c_dir(s, d, dev) for d in dirs]
    B, L, H, P, N, G, K = s.batch, s.seqlen, s.nheads, s.headdim, s.dstate, s.ngroups, s.nblocks
    tout = _DT[s.out_dtype][0]
    _check_tensor("states", states, (B, K, H, P, N), torch.float32, dev)
    _check_tensor("dy_noisy", dy_noisy, (B, L, H, P), tout, dev)
    if dy_clean is not None:
        _check_tensor("dy_clean", dy_clean, (B, L, H, P), tout, dev)
    if dstates is not None:
        _check_tensor("dstates", dstates, (B, K, H, P, N), torch.float32, dev)
    if h0 is not None:
        _check_tensor("h0", h0, (B, H, P, N), torch.float32, dev)
    if grads is None:
        f = dict(device=dev, dtype=torch.float32)
        grads = [None if d is None else
                 {"x": torch.empty((B, L, H, P), **f), "dt": torch.empty((B, L, H), **f),
                  "B": torch.empty((B, L, G, N), **f), "C": torch.empty((B, L, G, N), **f),
                  "A": torch.empty((H,), **f), "D": torch.empty((H,), **f)} for d in dirs]
    gshapes = {"x": (B, L, H, P), "dt": (B, L, H), "B": (B, L, G, N), "C": (B, L, G, N), "A": (H,), "D": (H,)}
    for i, (d, g) in enumerate(zip(dirs, grads)):
        if d is None:
            continue
        if g is None:
            raise ValueError(f"grads[{i}] is required for a present direction")
        for k in GRAD_KEYS:
            _check_tensor(f"grads[{i}][{k}]", g[k], gshapes[k], torch.float32, dev)
    cg = [None if g is None or d is None else bdscan_grad_t(*(_ptr(g[k]) for k in GRAD_KEYS))
          for d, g in zip(dirs, grads)]
    dh0 = _state(s, dev) if want_dh0 else None
    if ws is None:
        ws = workspace(s, BDSCAN_OP_ALLBLOCK_BACKWARD, dev)
    _check_ws(ws, s, BDSCAN_OP_ALLBLOCK_BACKWARD, dev)
    rc = bdscan_allblock_backward(ctypes.byref(cs), _ref(cd[0]), _ref(cd[1]), _ref(cd[2]), _ref(cd[3]),
                                  _ptr(h0), _ptr(states), _ptr(dy_clean), _ptr(dy_noisy), _ptr(dstates),
                                  _ref(cg[0]), _ref(cg[1]), _ref(cg[2]), _ref(cg[3]), _ptr(dh0), _ptr(ws),
                                  ws.numel(), _stream(dev, stream))
    _raise("bdscan_allblock_backward", rc)
    return grads, dh0


# ----------------------------------------------------------------------------- short convolution
CONV_KEYS = ("x", "B", "C")


def conv_channels(s: Shape) -> int:
    """Channels of the convolution: x's H*P, then B's and C's G*N each."""
    return s.nheads * s.headdim + 2 * s.ngroups * s.dstate


def c_conv(s: Shape, d: dict | None, width: int, device, out: dict | None = None):
    """ctypes struct of one convolution direction.  ``d`` holds the pre-convolution
    x, B, C (in_dtype), weight [Cx][width] and optionally bias [Cx] (fp32);
    ``out`` the output tensors (allocated when None).  Returns (struct, out)."""
    if d is None:
        return None, None
    tin = _DT[s.in_dtype][0]
    B, L, H, P, N, G = s.batch, s.seqlen, s.nheads, s.headdim, s.dstate, s.ngroups
    shapes = {"x": (B, L, H, P), "B": (B, L, G, N), "C": (B, L, G, N)}
    for k in CONV_KEYS:
        _check_tensor(k, d[k], shapes[k], tin, device)
    cx = conv_channels(s)
    _check_tensor("weight", d["weight"], (cx, width), torch.float32, device)
    if d.get("bias") is not None:
        _check_tensor("bias", d["bias"], (cx,), torch.float32, device)
    if out is None:
        out = {k: torch.empty(shapes[k], dtype=tin, device=device) for k in CONV_KEYS}
    st = bdscan_conv_t(_ptr(d["x"]), _ptr(d["B"]), _ptr(d["C"]), _ptr(d["weight"]), _ptr(d.get("bias")),
                       _ptr(out["x"]), _ptr(out["B"]), _ptr(out["C"]))
    return st, out


def c_dir_scan(s: Shape, d: dict, device) -> bdscan_dir_t:
    """ctypes struct of a scan direction whose x, B, C come from elsewhere (the
    convolution of bdscan_conv_block_step): dt, A, D and the optional z only."""
    tin = _DT[s.in_dtype][0]
    B, L, H, P = s.batch, s.seqlen, s.nheads, s.headdim
    _check_tensor("dt", d["dt"], (B, L, H), tin, device)
    if d.get("z") is not None:
        _check_tensor("z", d["z"], (B, L, H, P), tin, device)
    _check_tensor("A", d["A"], (H,), torch.float32, device)
    _check_tensor("D", d["D"], (H,), torch.float32, device)
    return bdscan_dir_t(None, _ptr(d["dt"]), None, None, _ptr(d.get("z")), _ptr(d["A"]), _ptr(d["D"]))


def _check_conv_state(name, t, s: Shape, width: int, device):
    if t is not None:
        _check_tensor(name, t, (s.batch, width - 1, conv_channels(s)), _DT[s.in_dtype][0], device)


def conv_prefix(s: Shape, width: int, silu: bool, fwd: dict, rev: dict | None = None, state_in=None,
                state_out=None, out_fwd=None, out_rev=None, stream=None):
    """Short convolution (+SiLU) of one sequence: causal for ``fwd`` from
    ``state_in`` ([B][width-1][Cx], None = zeros), anti-causal inside each
    block for ``rev``.  ``state_out``: None, a tensor (may be ``state_in`` when
    seqlen <= 32) or True (allocate).  Returns (fwd outputs, rev outputs or
    None, state_out or None); outputs are dicts keyed x, B, C."""
    dev = fwd["x"].device
    cs = c_shape(s)
    cf, out_fwd = c_conv(s, fwd, width, dev, out_fwd)
    cr, out_rev = c_conv(s, rev, width, dev, out_rev)
    _check_conv_state("state_in", state_in, s, width, dev)
    if state_out is True:
        state_out = torch.empty((s.batch, width - 1, conv_channels(s)), dtype=_DT[s.in_dtype][0], device=dev)
    _check_conv_state("state_out", state_out, s, width, dev)
    rc = bdscan_conv_prefix(ctypes.byref(cs), int(width), 1 if silu else 0, ctypes.byref(cf), _ref(cr),
                            _ptr(state_in), _ptr(state_out), _stream(dev, stream))
    _raise("bdscan_conv_prefix", rc)
    return out_fwd, out_rev, state_out


def conv_allblock(s: Shape, width: int, silu: bool, clean_fwd: dict, clean_rev: dict | None,
                  noisy_fwd: dict, noisy_rev: dict | None, state_in=None, outs=None, stream=None):
    """Short convolution of the all-block pass: the clean stream as in
    ``conv_prefix``; every noisy block's forward convolution reads the clean
    rows before it.  Returns four output dicts (None for absent directions)."""
    dev = clean_fwd["x"].device
    cs = c_shape(s)
    dirs = [clean_fwd, clean_rev, noisy_fwd, noisy_rev]
    outs = outs or [None] * 4
    built = [c_conv(s, d, width, dev, o) for d, o in zip(dirs, outs)]
    _check_conv_state("state_in", state_in, s, width, dev)
    cd = [b[0] for b in built]
    rc = bdscan_conv_allblock(ctypes.byref(cs), int(width), 1 if silu else 0, _ref(cd[0]), _ref(cd[1]),
                              _ref(cd[2]), _ref(cd[3]), _ptr(state_in), _stream(dev, stream))
    _raise("bdscan_conv_allblock", rc)
    return [b[1] for b in built]


def conv_block_step(s: Shape, width: int, silu: bool, conv_fwd: dict, conv_rev: dict, conv_state_in, fwd: dict,
                    rev: dict, state_in, y=None, ws=None, stream=None):
    """One denoising step of a layer's selective-scan core without commit: the
    short convolution of both directions' x, B, C (``conv_fwd``/``conv_rev``:
    pre-convolution inputs, weight, bias) from ``conv_state_in``, then the scan
    step from ``state_in`` with ``fwd``/``rev``'s dt, A, D and z.  One launch
    when the tensor-core step takes the shape.  Returns y."""
    dev = conv_fwd["x"].device
    cs = c_shape(s)
    cf, _ = c_conv(s, conv_fwd, width, dev, {k: None for k in CONV_KEYS})
    cr, _ = c_conv(s, conv_rev, width, dev, {k: None for k in CONV_KEYS})
    _check_conv_state("conv_state_in", conv_state_in, s, width, dev)
    sf, sr = c_dir_scan(s, fwd, dev), c_dir_scan(s, rev, dev)
    _check_tensor("state_in", state_in, (s.batch, s.nheads, s.headdim, s.dstate), torch.float32, dev)
    if y is None:
        y = _out(s, dev)
    _check_tensor("y", y, (s.batch, s.seqlen, s.nheads, s.headdim), _DT[s.out_dtype][0], dev)
    if ws is None:
        ws = workspace(s, BDSCAN_OP_CONV_BLOCK_STEP, dev)
    _check_ws(ws, s, BDSCAN_OP_CONV_BLOCK_STEP, dev)
    rc = bdscan_conv_block_step(ctypes.byref(cs), int(width), 1 if silu else 0, ctypes.byref(cf), ctypes.byref(cr),
                                _ptr(conv_state_in), ctypes.byref(sf), ctypes.byref(sr), _ptr(state_in), _ptr(y),
                                _ptr(ws), ws.numel(), _stream(dev, stream))
    _raise("bdscan_conv_block_step", rc)
    return y


# ----------------------------------------------------------------------------- gated RMSNorm
def gated_rmsnorm(s: Shape, y, z=None, weight=None, groups: int = 1, eps: float = 1e-5, out=None,
                  stream=None):
    """Gated RMSNorm of a scan output ``y`` [B, L, H, P] (out_dtype): per token row
    and group of H*P/groups channels, v * weight / sqrt(mean(v^2) + eps) with
    v = y * silu(z) (z in_dtype, optional); bf16 result (``out`` may be ``y``
    when y is bf16)."""
    dev = y.device
    B, L, H, P = s.batch, s.seqlen, s.nheads, s.headdim
    _check_tensor("y", y, (B, L, H, P), _DT[s.out_dtype][0], dev)
    if z is not None:
        _check_tensor("z", z, (B, L, H, P), _DT[s.in_dtype][0], dev)
    _check_tensor("weight", weight, (H * P,), torch.float32, dev)
    if out is None:
        out = torch.empty((B, L, H, P), dtype=torch.bfloat16, device=dev)
    _check_tensor("out", out, (B, L, H, P), torch.bfloat16, dev)
    rc = bdscan_gated_rmsnorm(ctypes.byref(c_shape(s)), _ptr(y), _ptr(z), _ptr(weight), int(groups),
                              float(eps), _ptr(out), _stream(dev, stream))
    _raise("bdscan_gated_rmsnorm", rc)
    return out
