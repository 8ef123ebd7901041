"""fp64 CPU oracle of the ButterflyMoE expert-layer forward (ctypes wrapper).

TEST INFRASTRUCTURE, NOT THE PRODUCT.  Only ``tests/``, the package smoke
check and the benchmark's CPU-baseline leg may import this module.  The C
source next to it (``bfmoe_oracle.c``) is the oracle; this file only builds
it with the host compiler and marshals numpy arrays.  It shares no code with
the CUDA library.

Parity pins for every function live in ``tests/test_oracle_pins.py``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "bfmoe_oracle.c")
_BUILD = os.path.join(_HERE, "_build")
_LIB = os.path.join(_BUILD, "liboracle.so")

OK = 0
ERR_INVALID_ARG = 1
ERR_NONFINITE = 4


def build(force: bool = False, extra_flags: tuple = (), out: str | None = None) -> str:
    """Compile the oracle with gcc (-O2, OpenMP, no fast-math)."""
    out = out or _LIB
    os.makedirs(os.path.dirname(out), exist_ok=True)
    if not force and os.path.exists(out) and os.path.getmtime(out) >= os.path.getmtime(_SRC) and not extra_flags:
        return out
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-Wall", "-Wextra",
           *extra_flags, _SRC, "-o", out, "-lm"]
    subprocess.run(cmd, check=True)
    return out


_lib = None


def _declare(lib):
    P = ctypes.c_void_p
    I = ctypes.c_int
    lib.oracle_butterfly_vec.argtypes = [I, P, I, P, P]
    lib.oracle_butterfly_rows.argtypes = [I, I, I, P, P, I, P, P]
    lib.oracle_route.argtypes = [P, I, I, I, P, P, P, P]
    lib.oracle_pack_base.argtypes = [P, I, ctypes.c_float, P]
    lib.oracle_unpack_base.argtypes = [P, I, P, P, P]
    lib.oracle_packed_base_bytes.argtypes = [I]
    lib.oracle_packed_base_bytes.restype = ctypes.c_size_t
    lib.oracle_expert_apply.argtypes = [I, P, ctypes.c_float, P, P, P, P]
    lib.oracle_forward.argtypes = [P, I, I, P, I, I, P, ctypes.c_float, P, P, P, I]
    lib.oracle_max_threads.argtypes = []
    lib.oracle_angles_per_butterfly.argtypes = [I]
    lib.oracle_angles_per_butterfly.restype = ctypes.c_longlong
    lib.oracle_layer_bytes.argtypes = [I, I]
    lib.oracle_layer_bytes.restype = ctypes.c_longlong
    return lib


def load(path: str | None = None):
    """Load (building first if needed) the oracle library."""
    global _lib
    if path is not None:
        return _declare(ctypes.CDLL(path))
    if _lib is None:
        # ORACLE_LIB points the tests at a deliberately broken copy of the
        # oracle (tests/test_oracle_mutants.py); it is never set otherwise.
        alt = os.environ.get("ORACLE_LIB")
        _lib = _declare(ctypes.CDLL(alt if alt else build()))
    return _lib


def _p(a: np.ndarray | None):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _f32(a):
    return np.ascontiguousarray(a, dtype=np.float32)


class OracleError(RuntimeError):
    def __init__(self, code):
        super().__init__(f"oracle status {code}")
        self.code = code


def _check(code):
    if code != OK:
        raise OracleError(code)


def butterfly(x: np.ndarray, angles: np.ndarray, transpose: bool = False,
              expert_of_row: np.ndarray | None = None, lib=None) -> np.ndarray:
    """y[r] = B(angles[e_r]) x[r]  (or B^T).  angles: [L][d/2] or [N][L][d/2]."""
    lib = lib or load()
    x = np.ascontiguousarray(x, dtype=np.float64)
    squeeze = x.ndim == 1
    x2 = x.reshape(-1, x.shape[-1])
    rows, d = x2.shape
    ang = _f32(angles)
    if ang.ndim == 2:
        ang = ang[None]
    N = ang.shape[0]
    eor = None if expert_of_row is None else np.ascontiguousarray(expert_of_row, dtype=np.int32)
    y = np.empty_like(x2)
    _check(lib.oracle_butterfly_rows(rows, d, N, _p(ang), _p(eor), int(bool(transpose)), _p(x2), _p(y)))
    return y.reshape(x.shape) if not squeeze else y[0]


def route(logits: np.ndarray, k: int, lib=None):
    """Returns (topk_idx [T][k] int32, gates [T][k] fp64, perm [T*k] int32, offsets [N+1] int32)."""
    lib = lib or load()
    lg = _f32(logits)
    T, N = lg.shape
    idx = np.zeros((T, k), np.int32)
    gates = np.zeros((T, k), np.float64)
    perm = np.zeros(T * k, np.int32)
    offsets = np.zeros(N + 1, np.int32)
    _check(lib.oracle_route(_p(lg), T, N, k, _p(idx), _p(gates), _p(perm), _p(offsets)))
    return idx, gates, perm, offsets


def pack_base(w: np.ndarray, alpha: float, lib=None) -> np.ndarray:
    lib = lib or load()
    w = np.ascontiguousarray(w, dtype=np.int8)
    d = w.shape[0]
    out = np.zeros(int(lib.oracle_packed_base_bytes(d)), np.uint8)
    _check(lib.oracle_pack_base(_p(w), d, float(alpha), _p(out)))
    return out


def unpack_base(packed: np.ndarray, lib=None):
    lib = lib or load()
    packed = np.ascontiguousarray(packed, dtype=np.uint8)
    d = ctypes.c_int(0)
    a = ctypes.c_float(0)
    _check(lib.oracle_unpack_base(_p(packed), 0, None, ctypes.byref(d), ctypes.byref(a)))
    w = np.zeros((d.value, d.value), np.int8)
    _check(lib.oracle_unpack_base(_p(packed), d.value, _p(w), None, None))
    return w, float(a.value)


def expert_apply(x: np.ndarray, w: np.ndarray, alpha: float, theta_e: np.ndarray, phi_e: np.ndarray,
                 lib=None) -> np.ndarray:
    lib = lib or load()
    x = np.ascontiguousarray(x, dtype=np.float64)
    w = np.ascontiguousarray(w, dtype=np.int8)
    u = np.empty_like(x)
    _check(lib.oracle_expert_apply(x.shape[0], _p(w), float(alpha), _p(_f32(theta_e)), _p(_f32(phi_e)),
                                   _p(x), _p(u)))
    return u


def forward(x: np.ndarray, logits: np.ndarray, k: int, w: np.ndarray, alpha: float, theta: np.ndarray,
            phi: np.ndarray, nthreads: int = 0, lib=None) -> np.ndarray:
    """y [T][d] fp64 of the layer; x holds the (bf16-representable) input values."""
    lib = lib or load()
    x = _f32(x)
    lg = _f32(logits)
    T, d = x.shape
    N = lg.shape[1]
    y = np.zeros((T, d), np.float64)
    _check(lib.oracle_forward(_p(x), T, d, _p(lg), N, k, _p(np.ascontiguousarray(w, dtype=np.int8)),
                              float(alpha), _p(_f32(theta)), _p(_f32(phi)), _p(y), int(nthreads)))
    return y


def max_threads(lib=None) -> int:
    lib = lib or load()
    return int(lib.oracle_max_threads())


def angles_per_butterfly(d: int, lib=None) -> int:
    lib = lib or load()
    return int(lib.oracle_angles_per_butterfly(d))


def layer_bytes(d: int, N: int, lib=None) -> int:
    lib = lib or load()
    return int(lib.oracle_layer_bytes(d, N))


def packed_base_bytes(d: int, lib=None) -> int:
    lib = lib or load()
    return int(lib.oracle_packed_base_bytes(d))
