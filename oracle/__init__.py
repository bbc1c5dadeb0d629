"""fp64 CPU oracle of the BlockFFN layer forward -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product path (the CUDA library and its
Python binding) never imports it, links it or falls back to it.

The arithmetic lives in ``blockffn_oracle.c`` (plain C, fp64, loops in the order
the method is written); this module compiles it with gcc on first use and
marshals numpy arrays.  See that file's header for the definitions and the
passages they follow:

* ``route``               -- g = RMSNorm(ReLU(W_r x + b_r)) over the expert axis
* ``chunk_union``         -- per-chunk union of active experts, token bitmasks
* ``forward_dense``       -- y = sum over ALL experts of gate * expert(x)
                             (expert biases optional)
* ``forward_chunk_union`` -- union experts over whole chunks, masked after compute
* ``sparsity``            -- token-level and L-token chunk-level sparsity
* ``residual_layernorm``  -- LayerNorm(y + x) over the hidden dimension

Every function is pinned by ``tests/test_oracle_pins.py`` against facts that do
not come from this code (closed forms, a library MLP, brute force, invariants).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "blockffn_oracle.c")
_BUILD_DIR = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD_DIR, "liboracle.so")

_lib = None

_D = ctypes.POINTER(ctypes.c_double)
_I32 = ctypes.POINTER(ctypes.c_int32)
_U32 = ctypes.POINTER(ctypes.c_uint32)


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (fp64, -O2, OpenMP, no fast-math)."""
    os.makedirs(_BUILD_DIR, exist_ok=True)
    stale = (not os.path.exists(_LIB_PATH)) or (
        os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC))
    if force or stale:
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-fno-fast-math", "-ffp-contract=off", "-fopenmp",
               "-shared", "-fPIC", "-std=c11", _SRC, "-o", tmp, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        lib.oracle_num_threads.restype = ctypes.c_int
        lib.oracle_route.argtypes = [_D, _D, _D, _D, ctypes.c_double, ctypes.c_int,
                                     ctypes.c_int, ctypes.c_int, _D, _D]
        lib.oracle_chunk_union.argtypes = [_D, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                           _I32, _I32, _U32]
        lib.oracle_forward_dense.argtypes = [_D, _D, _D, _D, _D, _D, ctypes.c_int, ctypes.c_int,
                                             ctypes.c_int, ctypes.c_int, _D]
        lib.oracle_forward_chunk_union.argtypes = [_D, _D, _D, _D, _D, _D, ctypes.c_int,
                                                   ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                                   ctypes.c_int, _D]
        lib.oracle_sparsity.argtypes = [_D, ctypes.c_int, ctypes.c_int, ctypes.c_int, _D]
        lib.oracle_residual_layernorm.argtypes = [_D, _D, _D, _D, ctypes.c_double, ctypes.c_int,
                                                  ctypes.c_int, _D]
        _lib = lib
    return _lib


def _f64(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _p(a: np.ndarray, t):
    return a.ctypes.data_as(t)


def num_threads() -> int:
    """Threads the oracle's OpenMP loops use."""
    return int(_load().oracle_num_threads())


def route(x, W_r, gamma, eps: float, b_r=None):
    """Router: returns (logits [T,E], gates [T,E]) in fp64."""
    lib = _load()
    x, W_r, gamma = _f64(x), _f64(W_r), _f64(gamma)
    T, d_h = x.shape
    E = W_r.shape[0]
    assert W_r.shape == (E, d_h) and gamma.shape == (E,)
    br = None if b_r is None else _f64(b_r)
    logits = np.empty((T, E), np.float64)
    gates = np.empty((T, E), np.float64)
    lib.oracle_route(_p(x, _D), _p(W_r, _D), None if br is None else _p(br, _D),
                     _p(gamma, _D), float(eps), T, d_h, E, _p(logits, _D), _p(gates, _D))
    return logits, gates


def chunk_union(gates, n: int):
    """Chunk union: returns (counts [C] int32, idx [C,E] int32, tmask [C,E] uint32)."""
    lib = _load()
    g = _f64(gates)
    T, E = g.shape
    assert 1 <= n <= 32
    C = (T + n - 1) // n
    counts = np.empty(C, np.int32)
    idx = np.empty((C, E), np.int32)
    tmask = np.empty((C, E), np.uint32)
    lib.oracle_chunk_union(_p(g, _D), T, E, n, _p(counts, _I32), _p(idx, _I32),
                           _p(tmask, _U32))
    return counts, idx, tmask


def _biases(b_in, b_out, E, d_e, d_h):
    bi = None if b_in is None else _f64(b_in)
    bo = None if b_out is None else _f64(b_out)
    assert bi is None or bi.shape == (E, d_e)
    assert bo is None or bo.shape == (E, d_h)
    return bi, bo


def forward_dense(x, gates, W_in, W_out, b_in=None, b_out=None) -> np.ndarray:
    """y = sum over all experts of gate * (W_out_e Swish(W_in_e x + b_in_e) + b_out_e),
    fp64; b_in [E, d_e] and b_out [E, d_h] are optional (absent = no bias)."""
    lib = _load()
    x, g, W_in, W_out = _f64(x), _f64(gates), _f64(W_in), _f64(W_out)
    T, d_h = x.shape
    E, d_e, _ = W_in.shape
    assert W_in.shape == (E, d_e, d_h) and W_out.shape == (E, d_h, d_e) and g.shape == (T, E)
    bi, bo = _biases(b_in, b_out, E, d_e, d_h)
    y = np.empty((T, d_h), np.float64)
    lib.oracle_forward_dense(_p(x, _D), _p(g, _D), _p(W_in, _D), _p(W_out, _D),
                             None if bi is None else _p(bi, _D), None if bo is None else _p(bo, _D),
                             T, d_h, E, d_e, _p(y, _D))
    return y


def forward_chunk_union(x, gates, W_in, W_out, n: int, b_in=None, b_out=None) -> np.ndarray:
    """Union experts over whole n-token chunks, masked after computing, fp64
    (expert biases optional, as in ``forward_dense``)."""
    lib = _load()
    x, g, W_in, W_out = _f64(x), _f64(gates), _f64(W_in), _f64(W_out)
    T, d_h = x.shape
    E, d_e, _ = W_in.shape
    assert W_in.shape == (E, d_e, d_h) and W_out.shape == (E, d_h, d_e) and g.shape == (T, E)
    assert 1 <= n <= 32
    bi, bo = _biases(b_in, b_out, E, d_e, d_h)
    y = np.empty((T, d_h), np.float64)
    lib.oracle_forward_chunk_union(_p(x, _D), _p(g, _D), _p(W_in, _D), _p(W_out, _D),
                                   None if bi is None else _p(bi, _D),
                                   None if bo is None else _p(bo, _D),
                                   T, d_h, E, d_e, n, _p(y, _D))
    return y


def sparsity(gates, L: int):
    """(TLS, CLS_L) of a gate matrix."""
    lib = _load()
    g = _f64(gates)
    T, E = g.shape
    out = np.empty(2, np.float64)
    lib.oracle_sparsity(_p(g, _D), T, E, int(L), _p(out, _D))
    return float(out[0]), float(out[1])


def residual_layernorm(y, x, ln_gamma, ln_beta, eps: float) -> np.ndarray:
    """out = LayerNorm(y + x) over the hidden dimension (scale ln_gamma, shift ln_beta), fp64."""
    lib = _load()
    y, x, g, b = _f64(y), _f64(x), _f64(ln_gamma), _f64(ln_beta)
    T, d_h = x.shape
    assert y.shape == (T, d_h) and g.shape == (d_h,) and b.shape == (d_h,)
    out = np.empty((T, d_h), np.float64)
    lib.oracle_residual_layernorm(_p(y, _D), _p(x, _D), _p(g, _D), _p(b, _D), float(eps), T, d_h,
                                  _p(out, _D))
    return out
