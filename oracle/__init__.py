"""fp64 CPU oracle for the block-diffusion bidirectional Mamba-2 scan.

TEST INFRASTRUCTURE ONLY.  Only the test suite, ``__graft_entry__.smoke()`` and
the CPU-baseline leg of ``bench.py`` may import this package; the product path
(``bidirectional_mamba_state_b200``) never does, and this package never imports
the product.  The arithmetic lives in ``bdscan_oracle.c`` (plain sequential
recurrence in double precision, see that file's header for the equations it
follows); this module only marshals arrays through ctypes.

Inputs are dictionaries with keys ``x, dt, B, C, A, D`` and optionally ``z``
(torch tensors or numpy arrays, any dtype, any device).  They are widened
exactly to float64 on the host before the call, so the oracle sees the same
rounded values the device consumed.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "bdscan_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libbdscan_oracle.so")
_lock = threading.Lock()
_lib = None


class _Shape(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int64) for n in
                ("batch", "seqlen", "nheads", "headdim", "dstate", "ngroups", "block_len")]


_dp = ctypes.POINTER(ctypes.c_double)


class _Dir(ctypes.Structure):
    _fields_ = [("x", _dp), ("dt", _dp), ("Bm", _dp), ("Cm", _dp), ("z", _dp),
                ("A", _dp), ("D", _dp)]


class _Grad(ctypes.Structure):
    _fields_ = [("dx", _dp), ("ddt", _dp), ("dB", _dp), ("dC", _dp), ("dA", _dp), ("dD", _dp)]


class _ConvShape(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int64) for n in
                ("batch", "seqlen", "channels", "width", "block_len", "silu")]


class _ConvDir(ctypes.Structure):
    _fields_ = [("u", _dp), ("w", _dp), ("bias", _dp), ("v", _dp)]


def build(force: bool = False) -> str:
    """Compile the oracle shared library with gcc (-O2, OpenMP).  Returns its path."""
    if force or not os.path.exists(_LIB_PATH) or (
            os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC)):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp",
               "-fno-fast-math", "-ffp-contract=off", _SRC, "-o", tmp, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _open(path: str):
    lib = ctypes.CDLL(path)
    for name in ("oracle_prefix", "oracle_block_step", "oracle_allblock", "oracle_allblock_backward",
                 "oracle_conv_prefix", "oracle_conv_allblock", "oracle_gated_rmsnorm"):
        getattr(lib, name).restype = ctypes.c_int
    lib.oracle_max_threads.restype = ctypes.c_int
    lib.oracle_set_threads.argtypes = [ctypes.c_int]
    return lib


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            _lib = _open(_LIB_PATH)
    return _lib


def max_threads() -> int:
    return int(_load().oracle_max_threads())


def set_threads(n: int) -> None:
    _load().oracle_set_threads(int(n))


def _f64(t) -> np.ndarray:
    """Exact widening of a torch tensor / numpy array to a C-contiguous float64 array."""
    if t is None:
        return None
    if hasattr(t, "detach"):  # torch tensor
        t = t.detach().to("cpu")
        import torch
        t = t.to(torch.float64).contiguous().numpy()
    return np.ascontiguousarray(np.asarray(t, dtype=np.float64))


def _ptr(a):
    return a.ctypes.data_as(_dp) if a is not None else None


class _Marshal:
    """Keeps the float64 copies alive for the duration of one oracle call."""

    def __init__(self):
        self.keep = []

    def arr(self, t):
        a = _f64(t)
        if a is not None:
            self.keep.append(a)
        return a

    def dir(self, d):
        if d is None:
            return None
        fields = {}
        for key, cname in (("x", "x"), ("dt", "dt"), ("B", "Bm"), ("C", "Cm"), ("z", "z"),
                           ("A", "A"), ("D", "D")):
            fields[cname] = _ptr(self.arr(d.get(key)))
        return ctypes.pointer(_Dir(**fields))


def _shape(s: dict) -> _Shape:
    return _Shape(*(int(s[k]) for k in
                    ("batch", "seqlen", "nheads", "headdim", "dstate", "ngroups", "block_len")))


def _check(rc: int, name: str):
    if rc != 0:
        raise ValueError(f"{name}: oracle returned {rc}")


def prefix(shape: dict, fwd: dict, rev: dict | None = None, h0=None,
           want_states: bool = True, want_final: bool = True, lib=None):
    """Forward scan of the clean stream from h0 (eq. (10) boundary states), plus a
    block-local reverse scan of every block when ``rev`` is given (eq. (12)),
    summed (eq. (13)).  Returns (y, states or None, final or None) as float64."""
    lib = lib or _load()
    B, L, H, P, N, T = (int(shape[k]) for k in
                        ("batch", "seqlen", "nheads", "headdim", "dstate", "block_len"))
    K = L // T
    m = _Marshal()
    y = np.zeros((B, L, H, P))
    st = np.zeros((B, K, H, P, N)) if want_states else None
    fin = np.zeros((B, H, P, N)) if want_final else None
    rc = lib.oracle_prefix(ctypes.byref(_shape(shape)), m.dir(fwd), m.dir(rev),
                           _ptr(m.arr(h0)), _ptr(y), _ptr(st), _ptr(fin))
    _check(rc, "oracle_prefix")
    return y, st, fin


def block_step(shape: dict, fwd: dict, rev: dict | None, state_in, want_state_out: bool = False,
               lib=None):
    """One denoising step on a single block from the cached state (eq. (11)-(13)).
    ``shape['seqlen']`` must equal ``shape['block_len']``.  Returns (y, state_out or None)."""
    lib = lib or _load()
    B, L, H, P, N = (int(shape[k]) for k in ("batch", "seqlen", "nheads", "headdim", "dstate"))
    m = _Marshal()
    y = np.zeros((B, L, H, P))
    so = np.zeros((B, H, P, N)) if want_state_out else None
    rc = lib.oracle_block_step(ctypes.byref(_shape(shape)), m.dir(fwd), m.dir(rev),
                               _ptr(m.arr(state_in)), _ptr(y), _ptr(so))
    _check(rc, "oracle_block_step")
    return y, so


def allblock(shape: dict, clean_fwd: dict, clean_rev: dict | None, noisy_fwd: dict,
             noisy_rev: dict | None, h0=None, want_clean: bool = True, lib=None):
    """All-block pass (eq. (14)): clean stream as in ``prefix``; every noisy block k
    continues from the clean boundary state before it.  Returns
    (y_clean or None, y_noisy, states)."""
    lib = lib or _load()
    B, L, H, P, N, T = (int(shape[k]) for k in
                        ("batch", "seqlen", "nheads", "headdim", "dstate", "block_len"))
    K = L // T
    m = _Marshal()
    yc = np.zeros((B, L, H, P)) if want_clean else None
    yn = np.zeros((B, L, H, P))
    st = np.zeros((B, K, H, P, N))
    rc = lib.oracle_allblock(ctypes.byref(_shape(shape)), m.dir(clean_fwd), m.dir(clean_rev),
                             m.dir(noisy_fwd), m.dir(noisy_rev), _ptr(m.arr(h0)),
                             _ptr(yc), _ptr(yn), _ptr(st))
    _check(rc, "oracle_allblock")
    return yc, yn, st


GRAD_KEYS = ("x", "dt", "B", "C", "A", "D")


def allblock_backward(shape: dict, clean_fwd: dict, clean_rev: dict | None, noisy_fwd: dict,
                      noisy_rev: dict | None, h0=None, dy_clean=None, dy_noisy=None, dstates=None,
                      lib=None):
    """Gradients of a loss L(y_clean, y_noisy, states) through the all-block pass
    (ungated), given dL/dy_clean (or None), dL/dy_noisy and dL/dstates (or None).
    Returns (grads, dh0): grads[i] (i = 0 clean fwd, 1 clean rev, 2 noisy fwd,
    3 noisy rev; None for an absent direction) is a dict with keys
    x, dt, B, C, A, D holding float64 arrays shaped like the inputs."""
    lib = lib or _load()
    B, L, H, P, N, G = (int(shape[k]) for k in
                        ("batch", "seqlen", "nheads", "headdim", "dstate", "ngroups"))
    m = _Marshal()
    dirs = [clean_fwd, clean_rev, noisy_fwd, noisy_rev]
    grads, structs = [], []
    for d in dirs:
        if d is None:
            grads.append(None)
            structs.append(None)
            continue
        g = {"x": np.zeros((B, L, H, P)), "dt": np.zeros((B, L, H)), "B": np.zeros((B, L, G, N)),
             "C": np.zeros((B, L, G, N)), "A": np.zeros((H,)), "D": np.zeros((H,))}
        grads.append(g)
        structs.append(ctypes.pointer(_Grad(dx=_ptr(g["x"]), ddt=_ptr(g["dt"]), dB=_ptr(g["B"]),
                                            dC=_ptr(g["C"]), dA=_ptr(g["A"]), dD=_ptr(g["D"]))))
    dh0 = np.zeros((B, H, P, N))
    rc = lib.oracle_allblock_backward(ctypes.byref(_shape(shape)), m.dir(clean_fwd), m.dir(clean_rev),
                                      m.dir(noisy_fwd), m.dir(noisy_rev), _ptr(m.arr(h0)),
                                      _ptr(m.arr(dy_clean)), _ptr(m.arr(dy_noisy)), _ptr(m.arr(dstates)),
                                      structs[0], structs[1], structs[2], structs[3], _ptr(dh0))
    _check(rc, "oracle_allblock_backward")
    return grads, dh0


# ---- short convolution in front of the scan --------------------------------
#
# A direction's convolution inputs are a dict with keys x [B][L][H][P],
# B and C [B][L][G][N] (pre-convolution), weight [H*P + 2*G*N][width] and
# optionally bias [H*P + 2*G*N].  The channels are packed x | B | C into flat
# rows for the C code and unpacked again; outputs are dicts with keys x, B, C.


def _pack_rows(shape: dict, d: dict) -> np.ndarray:
    B, L = int(shape["batch"]), int(shape["seqlen"])
    parts = []
    for k in ("x", "B", "C"):
        a = _f64(d[k])
        parts.append(a.reshape(B, L, int(np.prod(a.shape[2:]))))
    return np.ascontiguousarray(np.concatenate(parts, axis=2))


def _unpack_rows(shape: dict, v: np.ndarray) -> dict:
    B, L, H, P, N, G = (int(shape[k]) for k in
                        ("batch", "seqlen", "nheads", "headdim", "dstate", "ngroups"))
    hp, gn = H * P, G * N
    return {"x": v[:, :, :hp].reshape(B, L, H, P), "B": v[:, :, hp:hp + gn].reshape(B, L, G, N),
            "C": v[:, :, hp + gn:].reshape(B, L, G, N)}


def _conv_shape(shape: dict, width: int, silu: bool) -> _ConvShape:
    H, P, N, G = (int(shape[k]) for k in ("nheads", "headdim", "dstate", "ngroups"))
    return _ConvShape(int(shape["batch"]), int(shape["seqlen"]), H * P + 2 * G * N, int(width),
                      int(shape["block_len"]), 1 if silu else 0)


class _ConvMarshal(_Marshal):
    def __init__(self, shape: dict):
        super().__init__()
        self.shape = shape
        self.outs = []

    def conv(self, d):
        if d is None:
            self.outs.append(None)
            return None
        u = _pack_rows(self.shape, d)
        v = np.zeros_like(u)
        self.keep += [u, v]
        self.outs.append(v)
        w = self.arr(d["weight"])
        bias = self.arr(d.get("bias"))
        return ctypes.pointer(_ConvDir(u=_ptr(u), w=_ptr(w), bias=_ptr(bias), v=_ptr(v)))


def conv_prefix(shape: dict, width: int, silu: bool, fwd: dict, rev: dict | None = None,
                state_in=None, want_state_out: bool = False, lib=None):
    """Short convolution of one sequence: causal for ``fwd`` from ``state_in``
    ([B][width-1][H*P + 2*G*N], None = zeros), anti-causal inside each block for
    ``rev``.  Returns (fwd outputs, rev outputs or None, state_out or None)."""
    lib = lib or _load()
    m = _ConvMarshal(shape)
    cs = _conv_shape(shape, width, silu)
    pf, pr = m.conv(fwd), m.conv(rev)
    so = np.zeros((int(shape["batch"]), int(width) - 1, cs.channels)) if want_state_out else None
    rc = lib.oracle_conv_prefix(ctypes.byref(cs), pf, pr, _ptr(m.arr(state_in)), _ptr(so))
    _check(rc, "oracle_conv_prefix")
    vf, vr = m.outs
    return (_unpack_rows(shape, vf), None if vr is None else _unpack_rows(shape, vr), so)


def conv_allblock(shape: dict, width: int, silu: bool, clean_fwd: dict, clean_rev: dict | None,
                  noisy_fwd: dict, noisy_rev: dict | None, state_in=None, lib=None):
    """Short convolution of the all-block pass: the clean stream as in
    ``conv_prefix``; every noisy block's forward convolution reads the clean rows
    before it.  Returns a list of four output dicts (None for absent directions)."""
    lib = lib or _load()
    m = _ConvMarshal(shape)
    cs = _conv_shape(shape, width, silu)
    ptrs = [m.conv(d) for d in (clean_fwd, clean_rev, noisy_fwd, noisy_rev)]
    rc = lib.oracle_conv_allblock(ctypes.byref(cs), *ptrs, _ptr(m.arr(state_in)))
    _check(rc, "oracle_conv_allblock")
    return [None if v is None else _unpack_rows(shape, v) for v in m.outs]


def gated_rmsnorm(y, z=None, weight=None, groups: int = 1, eps: float = 1e-5, lib=None):
    """Gated RMSNorm of token rows: y (and z) [..., H, P] or [..., C]; the last
    two dimensions (or the last) are the channels.  Returns float64 of y's shape:
    per row and group of C / groups channels, v * w / sqrt(mean(v^2) + eps) with
    v = y * silu(z) (v = y without z)."""
    lib = lib or _load()
    ya = _f64(y)
    shape = ya.shape
    C = int(np.asarray(_f64(weight)).size)
    rows = int(ya.size // C) if C else 0
    m = _Marshal()
    yk = m.arr(ya.reshape(rows, C))
    zk = m.arr(None if z is None else _f64(z).reshape(rows, C))
    wk = m.arr(weight)
    out = np.zeros((rows, C))
    rc = lib.oracle_gated_rmsnorm(ctypes.c_int64(rows), ctypes.c_int64(C), ctypes.c_int64(int(groups)),
                                  ctypes.c_double(float(eps)), _ptr(yk), _ptr(zk), _ptr(wk), _ptr(out))
    _check(rc, "oracle_gated_rmsnorm")
    return out.reshape(shape)


class Variant:
    """The same API bound to another build of the oracle source (used by the
    tests that plant a mistake in a copy of the oracle and check that the pins
    catch it)."""

    def __init__(self, lib_path: str):
        self.lib = _open(lib_path)

    def prefix(self, *a, **k):
        return prefix(*a, lib=self.lib, **k)

    def block_step(self, *a, **k):
        return block_step(*a, lib=self.lib, **k)

    def allblock(self, *a, **k):
        return allblock(*a, lib=self.lib, **k)

    def allblock_backward(self, *a, **k):
        return allblock_backward(*a, lib=self.lib, **k)

    def conv_prefix(self, *a, **k):
        return conv_prefix(*a, lib=self.lib, **k)

    def conv_allblock(self, *a, **k):
        return conv_allblock(*a, lib=self.lib, **k)

    def gated_rmsnorm(self, *a, **k):
        return gated_rmsnorm(*a, lib=self.lib, **k)


def compile_variant(src_text: str, out_path: str) -> str:
    """Compile an edited copy of the oracle source to ``out_path``."""
    src = out_path + ".c"
    with open(src, "w") as f:
        f.write(src_text)
    subprocess.run(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-fno-fast-math",
                    "-ffp-contract=off", src, "-o", out_path, "-lm"], check=True)
    return out_path


def source_text() -> str:
    with open(_SRC) as f:
        return f.read()
