"""fp64 CPU oracle for the Mamba-2 selective state-space layer.

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, by ``__graft_entry__.smoke()``
and by the CPU-baseline leg of ``bench.py``.  The product library never loads
it, and it shares no code with the CUDA path.

The arithmetic lives in ``ssd_oracle.c`` (plain C, double precision); this
module only compiles it with gcc on first use and marshals numpy arrays.
See the header of ``ssd_oracle.c`` for the definitions and their sources:
the recurrence of "Hybrid Architectures for Language Models" (summary page,
section 2 Background) and the conv-cache shape of its appendix C.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "ssd_oracle.c")
_LIB = os.path.join(_HERE, "libssd_oracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile ssd_oracle.c into libssd_oracle.so (gcc, -O2, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fno-fast-math",
             "-ffp-contract=off", "-pthread", _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def open_library(path: str):
    """Load a compiled oracle library (the default build, or another build of
    the same source, e.g. a deliberately broken copy in a mutation test)."""
    lib = ctypes.CDLL(path)
    d = ctypes.POINTER(ctypes.c_double)
    i64 = ctypes.c_int64
    lib.oracle_conv1d_silu.argtypes = [d, d, d, d, d, i64, i64, i64, i64]
    lib.oracle_conv1d_silu.restype = None
    lib.oracle_selective_scan.argtypes = [d] * 10 + [i64] * 6 + [ctypes.c_int]
    lib.oracle_selective_scan.restype = ctypes.c_int
    lib.oracle_state_update.argtypes = [d] * 9 + [i64] * 5 + [ctypes.c_int]
    lib.oracle_state_update.restype = ctypes.c_int
    lib.oracle_selective_scan_bwd.argtypes = [d] * 18 + [i64] * 6 + [ctypes.c_int]
    lib.oracle_selective_scan_bwd.restype = ctypes.c_int
    return lib


_override = threading.local()


def _load():
    lib = getattr(_override, "lib", None)
    if lib is not None:
        return lib
    global _lib
    with _lock:
        if _lib is None:
            _lib = open_library(build())
    return _lib


class using_library:
    """Context manager: route this thread's oracle calls to another build."""

    def __init__(self, lib):
        self.lib = lib

    def __enter__(self):
        self.prev = getattr(_override, "lib", None)
        _override.lib = self.lib
        return self

    def __exit__(self, *exc):
        _override.lib = self.prev
        return False


def _f64(a, shape=None):
    if a is None:
        return None
    a = np.ascontiguousarray(np.asarray(a, dtype=np.float64))
    if shape is not None and a.shape != tuple(shape):
        a = a.reshape(shape)
    return a


def _ptr(a):
    if a is None:
        return None
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def default_threads() -> int:
    return max(1, os.cpu_count() or 1)


def conv1d_silu(xBC, w, bias=None, conv_state=None):
    """Causal depthwise conv (cross-correlation, taps [conv_dim, k]) + SiLU.

    xBC [b, L, conv_dim]; conv_state [b, conv_dim, k] or None.
    Returns (u [b, L, conv_dim], new_conv_state or None), all float64.
    """
    xBC = _f64(xBC)
    b, L, cd = xBC.shape
    w = _f64(w)
    k = w.shape[1]
    assert w.shape == (cd, k)
    bias = _f64(bias)
    st = None if conv_state is None else _f64(conv_state).copy()
    out = np.empty_like(xBC)
    _load().oracle_conv1d_silu(_ptr(xBC), _ptr(out), _ptr(w), _ptr(bias), _ptr(st), b, L, cd, k)
    return out, st


def selective_scan(x, B, C, dt_raw, A, dt_bias=None, D=None, init_state=None,
                   nthreads: int | None = None):
    """Token-by-token recurrence.

    x [b, L, H, P]; B, C [b, L, G, N]; dt_raw [b, L, H]; A, dt_bias, D [H];
    init_state [b, H, P, N] or None.  Returns (y [b, L, H, P], final_state).
    """
    x = _f64(x)
    b, L, H, P = x.shape
    B = _f64(B)
    G, N = B.shape[2], B.shape[3]
    C = _f64(C)
    assert B.shape == (b, L, G, N) and C.shape == B.shape
    dt_raw = _f64(dt_raw, (b, L, H))
    A = _f64(A, (H,))
    dt_bias = _f64(dt_bias, (H,))
    D = _f64(D, (H,))
    init_state = _f64(init_state, (b, H, P, N))
    y = np.empty_like(x)
    fs = np.empty((b, H, P, N), dtype=np.float64)
    rc = _load().oracle_selective_scan(
        _ptr(x), _ptr(B), _ptr(C), _ptr(dt_raw), _ptr(dt_bias), _ptr(A), _ptr(D),
        _ptr(init_state), _ptr(y), _ptr(fs), b, L, H, P, N, G,
        nthreads or default_threads())
    if rc != 0:
        raise ValueError("oracle_selective_scan: bad sizes")
    return y, fs


def selective_scan_varlen(x, B, C, dt_raw, A, cu_seqlens, dt_bias=None, D=None, init_state=None,
                          nthreads: int | None = None):
    """The recurrence on a ragged batch packed along the token dimension:
    sequence s is tokens cu_seqlens[s] .. cu_seqlens[s+1]-1, run from its own
    initial state (the chunked-prefill reading of "Hybrid Architectures for
    Language Models", section 2: each sequence is an independent recurrence).

    x [T, H, P]; B, C [T, G, N]; dt_raw [T, H]; init_state [nseq, H, P, N]
    or None.  Returns (y [T, H, P], final_state [nseq, H, P, N]); an empty
    sequence's final state is its initial state (or zero).
    """
    x = _f64(x)
    T, H, P = x.shape
    B = _f64(B)
    G, N = B.shape[1], B.shape[2]
    C = _f64(C)
    dt_raw = _f64(dt_raw, (T, H))
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    nseq = cu.size - 1
    if nseq < 0 or cu[0] != 0 or cu[-1] != T or np.any(np.diff(cu) < 0):
        raise ValueError("cu_seqlens must start at 0, not decrease and end at T")
    init_state = _f64(init_state, (nseq, H, P, N))
    y = np.zeros_like(x)
    fs = np.zeros((nseq, H, P, N), dtype=np.float64)
    for s in range(nseq):
        a, b = int(cu[s]), int(cu[s + 1])
        init = None if init_state is None else init_state[s:s + 1]
        if a == b:
            if init is not None:
                fs[s] = init[0]
            continue
        ys, fss = selective_scan(x[None, a:b], B[None, a:b], C[None, a:b], dt_raw[None, a:b], A,
                                 dt_bias, D, init, nthreads)
        y[a:b] = ys[0]
        fs[s] = fss[0]
    return y, fs


def state_update(state, x, B, C, dt_raw, A, dt_bias=None, D=None, nthreads: int | None = None):
    """One decode token.  state [b, H, P, N]; x [b, H, P]; B, C [b, G, N];
    dt_raw [b, H].  Returns (y [b, H, P], new_state); inputs are not modified."""
    st = _f64(state).copy()
    b, H, P, N = st.shape
    x = _f64(x, (b, H, P))
    B = _f64(B)
    G = B.shape[1]
    C = _f64(C, B.shape)
    dt_raw = _f64(dt_raw, (b, H))
    y = np.empty((b, H, P), dtype=np.float64)
    rc = _load().oracle_state_update(
        _ptr(st), _ptr(x), _ptr(B), _ptr(C), _ptr(dt_raw), _ptr(_f64(dt_bias, (H,))),
        _ptr(_f64(A, (H,))), _ptr(_f64(D, (H,))), _ptr(y), b, H, P, N, G,
        nthreads or default_threads())
    if rc != 0:
        raise ValueError("oracle_state_update: bad sizes")
    return y, st


def selective_scan_bwd(x, B, C, dt_raw, A, dy, dt_bias=None, D=None, init_state=None, dfinal=None,
                       nthreads: int | None = None):
    """Gradient of sum(dy * y) + sum(dfinal * final_state) through
    selective_scan, by the reverse-mode token loop of ssd_oracle.c.

    Shapes as for selective_scan; dy [b, L, H, P], dfinal [b, H, P, N] or None.
    Returns a dict of float64 arrays: dx, dB, dC, ddt_raw, dA, dD, ddt_bias,
    dinit (the gradient with respect to the initial state, also when none
    was given: the state is then zero)."""
    x = _f64(x)
    b, L, H, P = x.shape
    B = _f64(B)
    G, N = B.shape[2], B.shape[3]
    C = _f64(C, B.shape)
    dt_raw = _f64(dt_raw, (b, L, H))
    dy = _f64(dy, (b, L, H, P))
    out = dict(dx=np.empty((b, L, H, P)), dB=np.empty((b, L, G, N)), dC=np.empty((b, L, G, N)),
               ddt_raw=np.empty((b, L, H)), dA=np.empty(H), dD=np.empty(H), ddt_bias=np.empty(H),
               dinit=np.empty((b, H, P, N)))
    rc = _load().oracle_selective_scan_bwd(
        _ptr(x), _ptr(B), _ptr(C), _ptr(dt_raw), _ptr(_f64(dt_bias, (H,))), _ptr(_f64(A, (H,))),
        _ptr(_f64(D, (H,))), _ptr(_f64(init_state, (b, H, P, N))), _ptr(dy),
        _ptr(_f64(dfinal, (b, H, P, N))), _ptr(out["dx"]), _ptr(out["dB"]), _ptr(out["dC"]),
        _ptr(out["ddt_raw"]), _ptr(out["dA"]), _ptr(out["dD"]), _ptr(out["ddt_bias"]), _ptr(out["dinit"]),
        b, L, H, P, N, G, nthreads or default_threads())
    if rc != 0:
        raise ValueError("oracle_selective_scan_bwd: bad sizes")
    return out


def split_xBC(u, H, P, G, N):
    """Split conv-output channels [x (H*P) | B (G*N) | C (G*N)] into views."""
    b, L, cd = u.shape
    assert cd == H * P + 2 * G * N
    x = u[..., : H * P].reshape(b, L, H, P)
    B = u[..., H * P: H * P + G * N].reshape(b, L, G, N)
    C = u[..., H * P + G * N:].reshape(b, L, G, N)
    return x, B, C


def layer_prefill(xBC, w, bias, conv_state, dt_raw, A, dt_bias, D, init_state, H, P, G, N,
                  nthreads: int | None = None):
    """conv1d+SiLU then the selective scan, all in fp64.
    Returns (y, final_state, new_conv_state)."""
    u, cs = conv1d_silu(xBC, w, bias, conv_state)
    x, B, C = split_xBC(u, H, P, G, N)
    y, fs = selective_scan(x, B, C, dt_raw, A, dt_bias, D, init_state, nthreads)
    return y, fs, cs


# ---------------------------------------------------------------------------
# The Mamba-2 mixer around the path: in_proj, conv1d+SiLU, the scan, the
# gated RMSNorm and out_proj (Nemotron feasibility report, section 3.2: the
# block is x + Mamba2(RMSNorm(x)); section 3.3: in_proj / out_proj are
# linear layers, the scan stays bf16/fp32).  The pages fix neither the order
# of the in_proj outputs nor the gate; the readings taken are: output rows
# z (H*P) | xBC (H*P + 2*G*N) | dt_raw (H); the gate y * SiLU(z); then an
# RMSNorm over each of `groups` equal slices of every token's H*P vector
# (one slice by default), times a weight.
# ---------------------------------------------------------------------------

def silu(v):
    """SiLU(v) = v / (1 + e^-v) in float64 (v -> -inf gives -0)."""
    v = np.asarray(v, dtype=np.float64)
    with np.errstate(over="ignore"):
        return v / (1.0 + np.exp(-v))


def rmsnorm_gated(y, z, weight, groups: int = 1, eps: float = 1e-5):
    """g = y * SiLU(z); every token's vector (last axis) is cut into `groups`
    equal contiguous slices, each divided by sqrt(mean of its squares + eps),
    then the whole vector is multiplied elementwise by weight."""
    g = np.asarray(y, dtype=np.float64) * silu(z)
    shp = g.shape
    d = shp[-1]
    if d % groups:
        raise ValueError("rmsnorm_gated: groups must divide the vector length")
    gs = g.reshape(*shp[:-1], groups, d // groups)
    ms = np.mean(gs * gs, axis=-1, keepdims=True)
    return (gs / np.sqrt(ms + eps)).reshape(shp) * np.asarray(weight, dtype=np.float64)


def mixer_forward(hidden, W_in, conv_w, conv_bias, dt_bias, A, D, norm_w, W_out, H, P, G, N, *,
                  norm_groups: int = 1, eps: float = 1e-5, conv_state=None, init_state=None,
                  nthreads: int | None = None):
    """The Mamba-2 mixer in float64.

    hidden [b, L, d_model]; W_in [2 H P + 2 G N + H, d_model] (rows: z, xBC,
    dt_raw); conv_w [conv_dim, k], conv_bias [conv_dim] or None; dt_bias, A,
    D [H]; norm_w [H P]; W_out [d_model, H P].  Returns (out [b, L, d_model],
    final_state [b, H, P, N], conv_state_out [b, conv_dim, k])."""
    hidden = _f64(hidden)
    b, L, _ = hidden.shape
    d_inner = H * P
    conv_dim = d_inner + 2 * G * N
    W_in = _f64(W_in)
    if W_in.shape[0] != d_inner + conv_dim + H:
        raise ValueError("mixer_forward: W_in must have 2 H P + 2 G N + H rows")
    zxbcdt = hidden @ W_in.T
    z = zxbcdt[..., :d_inner]
    xBC = np.ascontiguousarray(zxbcdt[..., d_inner:d_inner + conv_dim])
    dt_raw = np.ascontiguousarray(zxbcdt[..., d_inner + conv_dim:])
    y, fs, cs = layer_prefill(xBC, conv_w, conv_bias, conv_state, dt_raw, A, dt_bias, D, init_state,
                              H, P, G, N, nthreads)
    n = rmsnorm_gated(y.reshape(b, L, d_inner), z, norm_w, norm_groups, eps)
    out = n @ _f64(W_out).T
    return out, fs, cs
