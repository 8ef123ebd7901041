"""ButterflyMoE expert-layer forward on NVIDIA B200 (sm_100a).

Thin ctypes binding of the C ABI in ``include/bfmoe.h`` (``libbfmoe.so``,
built in-tree by ``python -m ternary_moe_butterfly_b200.build``).  The
``bfmoe_*`` functions take raw pointers and sizes exactly like the C calls;
the lower-case helpers take torch tensors and only marshal them (device
pointers, the current CUDA stream, workspace sizing).  Every step of the
layer runs in the library's CUDA kernels; there is no CPU or library
fallback, and loading fails loudly if the shared library is missing.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libbfmoe.so")

OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_WORKSPACE, ERR_NONFINITE, ERR_TIMEOUT, ERR_CUDA = range(7)
F32, BF16 = 0, 1


class BfmoeError(RuntimeError):
    def __init__(self, code: int, what: str):
        super().__init__(f"{what}: {status_string(code)} ({code})")
        self.code = code


class WsLayout(ctypes.Structure):
    _fields_ = [(n, ctypes.c_size_t) for n in ("status", "topk_idx", "gates", "perm", "offsets", "total")]


_lib = None


def lib():
    """The loaded CUDA library (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with `python -m ternary_moe_butterfly_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        P, I, Z = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
        sigs = {
            "bfmoe_status_string": (ctypes.c_char_p, [I]),
            "bfmoe_version": (I, []),
            "bfmoe_packed_base_bytes": (Z, [I]),
            "bfmoe_pack_base": (I, [P, I, ctypes.c_float, P, P]),
            "bfmoe_route_workspace_bytes": (Z, [I, I, I]),
            "bfmoe_route": (I, [P, I, I, I, P, P, P, P, P, Z, P]),
            "bfmoe_butterfly_workspace_bytes": (Z, [I, I]),
            "bfmoe_butterfly_apply": (I, [P, I, I, I, I, P, P, I, P, P, Z, P]),
            "bfmoe_forward_workspace_bytes": (Z, [I, I, I, I]),
            "bfmoe_forward_ws_layout": (I, [I, I, I, I, ctypes.POINTER(WsLayout)]),
            "bfmoe_forward": (I, [P, I, I, I, P, I, I, P, P, P, P, P, Z, P]),
            "bfmoe_sync_status": (I, [P, P]),
            "bfmoe_forward_profile": (I, [P, I, I, I, P, I, I, P, P, P, P, P, Z, P, P, P]),
            "bfmoe_stage_name": (ctypes.c_char_p, [I]),
            "bfmoe_debug_set": (None, [I, I]),
            "bfmoe_route_static": (I, [P, I, I, I, P, P, P, P, P]),
        }
        for name, (res, args) in sigs.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


# ------------------------------------------------------------------ raw ABI
# Same names and arguments as the C entry points (pointers as ints).

def bfmoe_status_string(code):
    return lib().bfmoe_status_string(int(code)).decode()


status_string = bfmoe_status_string


def bfmoe_version():
    return lib().bfmoe_version()


def bfmoe_packed_base_bytes(d):
    return lib().bfmoe_packed_base_bytes(d)


def bfmoe_pack_base(w, d, alpha, packed, stream):
    return lib().bfmoe_pack_base(w, d, alpha, packed, stream)


def bfmoe_route_workspace_bytes(T, N, k):
    return lib().bfmoe_route_workspace_bytes(T, N, k)


def bfmoe_route(logits, T, N, k, topk_idx, gates, perm, offsets, ws, ws_bytes, stream):
    return lib().bfmoe_route(logits, T, N, k, topk_idx, gates, perm, offsets, ws, ws_bytes, stream)


def bfmoe_route_static(logits, T, N, k, topk_idx, gates, perm, offsets, stream):
    """bfmoe_route without a workspace (library-held scratch); see include/bfmoe.h."""
    return lib().bfmoe_route_static(logits, T, N, k, topk_idx, gates, perm, offsets, stream)


def bfmoe_butterfly_workspace_bytes(d, N):
    return lib().bfmoe_butterfly_workspace_bytes(d, N)


def bfmoe_butterfly_apply(x, dt, rows, d, N, angles, expert_of_row, transpose, y, ws, ws_bytes, stream):
    return lib().bfmoe_butterfly_apply(x, dt, rows, d, N, angles, expert_of_row, transpose, y, ws, ws_bytes,
                                       stream)


def bfmoe_forward_workspace_bytes(T, d, N, k):
    return lib().bfmoe_forward_workspace_bytes(T, d, N, k)


def bfmoe_forward_ws_layout(T, d, N, k):
    out = WsLayout()
    code = lib().bfmoe_forward_ws_layout(T, d, N, k, ctypes.byref(out))
    return code, out


def bfmoe_forward(x, dt, T, d, logits, N, k, packed_base, theta, phi, y, ws, ws_bytes, stream):
    return lib().bfmoe_forward(x, dt, T, d, logits, N, k, packed_base, theta, phi, y, ws, ws_bytes, stream)


def bfmoe_sync_status(ws, stream):
    return lib().bfmoe_sync_status(ws, stream)


MAX_STAGES = 16


def bfmoe_forward_profile(x, dt, T, d, logits, N, k, packed_base, theta, phi, y, ws, ws_bytes, stream, stage_ms,
                          n_stages):
    return lib().bfmoe_forward_profile(x, dt, T, d, logits, N, k, packed_base, theta, phi, y, ws, ws_bytes, stream,
                                       stage_ms, n_stages)


DEBUG_SKIP_ARRIVE_BLOCK = 1


def bfmoe_debug_set(key, value):
    """Test hook; see include/bfmoe.h."""
    lib().bfmoe_debug_set(int(key), int(value))


def bfmoe_stage_name(i):
    r = lib().bfmoe_stage_name(int(i))
    return None if r is None else r.decode()


# ------------------------------------------------------- tensor marshalling

def _torch():
    import torch
    return torch


def _stream(stream=None):
    if stream is not None:
        return int(getattr(stream, "cuda_stream", stream))
    return int(_torch().cuda.current_stream().cuda_stream)


def _dt(t):
    torch = _torch()
    if t.dtype == torch.float32:
        return F32
    if t.dtype == torch.bfloat16:
        return BF16
    raise TypeError(f"x must be float32 or bfloat16, got {t.dtype}")


def _ptr(t):
    return None if t is None else int(t.data_ptr())


def _need(t, name, dtype=None, dims=None, numel=None, min_numel=None):
    """t must be passable to the C ABI as a plain pointer: a contiguous
    tensor of the given dtype, rank and size (the device is checked by
    _on_device once every argument has passed)."""
    torch = _torch()
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor, got {type(t).__name__}")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if dims is not None and t.dim() != dims:
        raise ValueError(f"{name} must have {dims} dimensions, got shape {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if numel is not None and t.numel() != numel:
        raise ValueError(f"{name} has {t.numel()} elements, expected {numel}")
    if min_numel is not None and t.numel() < min_numel:
        raise ValueError(f"{name} has {t.numel()} elements, needs at least {min_numel}")
    return t


def _on_device(first, **others):
    """Every tensor argument on one CUDA device (the kernels dereference
    the pointers there); returns that device."""
    dev = first.device
    if dev.type != "cuda":
        raise ValueError(f"the arguments must be CUDA tensors, got one on {dev}")
    for name, t in others.items():
        if t is not None and t.device != dev:
            raise ValueError(f"{name} is on {t.device}, the other arguments on {dev}")
    return dev


def _angle_count(N, d):
    """Elements of an angle table [N][log2 d][d/2] (None when d is not a
    power of two: the C call rejects that width)."""
    if d < 2 or d & (d - 1):
        return None
    return N * (d.bit_length() - 1) * (d // 2)


def _check(code, what):
    if code != OK:
        raise BfmoeError(code, what)


def _ws(nbytes, device):
    torch = _torch()
    return torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)


def pack_base(w, alpha: float, stream=None):
    """int8 [d][d] ternary (device) -> packed uint8 tensor (synchronises)."""
    torch = _torch()
    if not isinstance(w, torch.Tensor) or w.dim() != 2 or w.shape[0] != w.shape[1]:
        raise ValueError("w must be a square [d][d] tensor")
    w = _need(w.contiguous(), "w", torch.int8)
    dev = _on_device(w)
    d = int(w.shape[0])
    out = torch.empty(max(int(bfmoe_packed_base_bytes(d)), 16), dtype=torch.uint8, device=dev)
    _check(bfmoe_pack_base(_ptr(w), d, float(alpha), _ptr(out), _stream(stream)), "bfmoe_pack_base")
    return out


def route(logits, k: int, ws=None, stream=None):
    """Top-k routing and bucketing; returns (topk_idx, gates, perm, offsets, ws)."""
    torch = _torch()
    _need(logits, "logits", torch.float32, dims=2)
    T, N = map(int, logits.shape)
    if ws is not None:
        _need(ws, "ws", torch.uint8)
    dev = _on_device(logits, ws=ws)
    idx = torch.empty((T, k), dtype=torch.int32, device=dev)
    gates = torch.empty((T, k), dtype=torch.float32, device=dev)
    perm = torch.empty(T * k, dtype=torch.int32, device=dev)
    offsets = torch.empty(N + 1, dtype=torch.int32, device=dev)
    need = bfmoe_route_workspace_bytes(T, N, k)
    if ws is None:
        ws = _ws(need, dev)
    _check(bfmoe_route(_ptr(logits), T, N, k, _ptr(idx), _ptr(gates), _ptr(perm), _ptr(offsets), _ptr(ws),
                       ws.numel(), _stream(stream)), "bfmoe_route")
    return idx, gates, perm, offsets, ws


def butterfly_apply(x, angles, expert_of_row=None, transpose: bool = False, ws=None, out=None, stream=None):
    """y[r] = B(angles[e_r]) x[r] (or B^T); x [rows][d] fp32/bf16 on the device."""
    torch = _torch()
    _need(x, "x", dims=2)
    _dt(x)
    rows, d = map(int, x.shape)
    if not isinstance(angles, torch.Tensor) or angles.dim() < 1:
        raise ValueError("angles must be a tensor [N][log2 d][d/2]")
    N = int(angles.shape[0])
    _need(angles, "angles", torch.float32, numel=_angle_count(N, d))
    if expert_of_row is not None:
        _need(expert_of_row, "expert_of_row", torch.int32, numel=rows)
    if out is not None:
        _need(out, "out", x.dtype, numel=rows * d)
    if ws is not None:
        _need(ws, "ws", torch.uint8)
    dev = _on_device(x, angles=angles, expert_of_row=expert_of_row, out=out, ws=ws)
    y = torch.empty_like(x) if out is None else out
    if ws is None:
        ws = _ws(bfmoe_butterfly_workspace_bytes(d, N), dev)
    _check(bfmoe_butterfly_apply(_ptr(x), _dt(x), rows, d, N, _ptr(angles), _ptr(expert_of_row),
                                 int(bool(transpose)), _ptr(y), _ptr(ws), ws.numel(), _stream(stream)),
           "bfmoe_butterfly_apply")
    return y, ws


def forward_workspace(T: int, d: int, N: int, k: int, device):
    return _ws(bfmoe_forward_workspace_bytes(T, d, N, k), device)


def _check_layer_args(x, logits, packed, theta, phi, ws, out):
    """Checks of forward's tensor arguments; returns (T, d, N, device)."""
    torch = _torch()
    _need(x, "x", dims=2)
    _dt(x)
    T, d = map(int, x.shape)
    _need(logits, "logits", torch.float32, dims=2)
    if int(logits.shape[0]) != T:
        raise ValueError(f"logits has {int(logits.shape[0])} rows, x has {T}")
    N = int(logits.shape[1])
    _need(packed, "packed", torch.uint8, min_numel=int(bfmoe_packed_base_bytes(d)))
    _need(theta, "theta", torch.float32, numel=_angle_count(N, d))
    _need(phi, "phi", torch.float32, numel=_angle_count(N, d))
    if out is not None:
        _need(out, "out", x.dtype, numel=T * d)
    if ws is not None:
        _need(ws, "ws", torch.uint8)
    dev = _on_device(x, logits=logits, packed=packed, theta=theta, phi=phi, out=out, ws=ws)
    return T, d, N, dev


def forward(x, logits, k: int, packed, theta, phi, ws=None, out=None, stream=None):
    """The expert layer: y = sum_j g_j alpha B(phi_e) W_base B(theta_e)^T x."""
    torch = _torch()
    T, d, N, dev = _check_layer_args(x, logits, packed, theta, phi, ws, out)
    y = torch.empty_like(x) if out is None else out
    if ws is None:
        ws = forward_workspace(T, d, N, k, dev)
    _check(bfmoe_forward(_ptr(x), _dt(x), T, d, _ptr(logits), N, k, _ptr(packed), _ptr(theta), _ptr(phi), _ptr(y),
                         _ptr(ws), ws.numel(), _stream(stream)), "bfmoe_forward")
    return y, ws


def forward_routing(ws, T: int, d: int, N: int, k: int):
    """Views of the routing results bfmoe_forward left in its workspace:
    (topk_idx [T][k], gates [T][k], perm [T*k], offsets [N+1])."""
    torch = _torch()
    code, lay = bfmoe_forward_ws_layout(T, d, N, k)
    _check(code, "bfmoe_forward_ws_layout")

    def view(off, n, dtype):
        return ws[off:off + 4 * n].view(dtype)

    idx = view(lay.topk_idx, T * k, torch.int32).view(T, k)
    gates = view(lay.gates, T * k, torch.float32).view(T, k)
    perm = view(lay.perm, T * k, torch.int32)
    offsets = view(lay.offsets, N + 1, torch.int32)
    return idx, gates, perm, offsets


def forward_profile(x, logits, k: int, packed, theta, phi, ws, out, stream=None):
    """bfmoe_forward with a CUDA event after each kernel (synchronises);
    returns {stage name: milliseconds}."""
    T, d, N, _ = _check_layer_args(x, logits, packed, theta, phi, ws, out)
    ms = (ctypes.c_float * MAX_STAGES)()
    n = ctypes.c_int(0)
    _check(bfmoe_forward_profile(_ptr(x), _dt(x), T, d, _ptr(logits), N, k, _ptr(packed), _ptr(theta), _ptr(phi),
                                 _ptr(out), _ptr(ws), ws.numel(), _stream(stream),
                                 ctypes.cast(ms, ctypes.c_void_p), ctypes.cast(ctypes.pointer(n), ctypes.c_void_p)),
           "bfmoe_forward_profile")
    return {bfmoe_stage_name(i): float(ms[i]) for i in range(n.value)}


def sync_status(ws, stream=None) -> int:
    """Synchronise and return (and clear) the device status word of ws."""
    return int(bfmoe_sync_status(_ptr(ws), _stream(stream)))
