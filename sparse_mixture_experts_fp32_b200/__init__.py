"""Switch Transformer sparse FFN layer forward pass on NVIDIA B200 (sm_100a).

Python binding of the C ABI in ``include/switch_moe.h``.  It only marshals
arguments: every step of the layer runs in the CUDA kernels of
``libswitchmoe.so``, which this module loads from the package directory.
There is no other implementation behind these functions; if the library is
missing or cannot be loaded, every call raises.

PyTorch supplies device memory and the CUDA stream (the current stream of the
tensors' device unless one is given).

Low level (same names and argument order as the C functions, tensors in
place of pointers):
    switch_capacity, switch_workspace_size, switch_route, switch_dispatch,
    switch_expert_ffn, switch_combine, switch_layer_fwd, switch_check
High level (allocate outputs and workspace with torch):
    capacity, layer_fwd, route, dispatch, expert_ffn, combine
"""
from __future__ import annotations

import ctypes
from pathlib import Path

_PKG = Path(__file__).resolve().parent
LIB_PATH = _PKG / "libswitchmoe.so"

SWITCH_F32 = 0
SWITCH_BF16 = 1
SWITCH_FLAG_SIMT_FFN = 1
SWITCH_FLAG_SIMT_ROUTER = 2
SWITCH_FLAG_GEMM_1CTA = 4
SWITCH_FLAG_FFN_TWO_LAUNCHES = 8
SWITCH_FLAG_SEPARATE_SCAN = 16
SWITCH_FLAG_TRAINING = 32
SWITCH_FLAG_ROUTER_STATS = 64
SWITCH_FLAG_MULTI_KERNEL = 128
SWITCH_FLAG_STAGED_MOVES = 256

STATUS = {
    0: "SWITCH_OK", 1: "SWITCH_ERR_NULL", 2: "SWITCH_ERR_SHAPE", 3: "SWITCH_ERR_DTYPE", 4: "SWITCH_ERR_ALIGN",
    5: "SWITCH_ERR_WORKSPACE", 6: "SWITCH_ERR_UNSUPPORTED", 7: "SWITCH_ERR_CUDA", 8: "SWITCH_ERR_DEVICE_TIMEOUT",
    9: "SWITCH_ERR_TOO_LARGE",
}

EXPORTED = ("switch_capacity", "switch_workspace_size", "switch_route", "switch_route_noalloc", "switch_dispatch",
            "switch_expert_ffn",
            "switch_combine", "switch_layer_fwd", "switch_route_top2", "switch_combine_top2", "switch_layer_fwd_top2",
            "switch_layer_bwd", "switch_router_stats",
            "switch_check", "switch_selftest_wait_timeout", "switch_check_noalloc",
            "switch_selftest_wait_timeout_noalloc", "switch_status_string",
            "switch_launch_count",
            "switch_trace_start", "switch_trace_read", "switch_trace_stop", "switch_kernel_name")


class SwitchError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {STATUS.get(status, status)} ({_status_text(status)})")


class SwitchDims(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int64), ("d_model", ctypes.c_int32), ("d_ff", ctypes.c_int32),
                ("num_experts", ctypes.c_int32), ("capacity", ctypes.c_int32), ("dtype", ctypes.c_int32),
                ("flags", ctypes.c_int32)]

    def __repr__(self):
        return (f"SwitchDims(T={self.T}, d_model={self.d_model}, d_ff={self.d_ff}, num_experts={self.num_experts}, "
                f"capacity={self.capacity}, dtype={self.dtype}, flags={self.flags})")


_lib = None


def lib() -> ctypes.CDLL:
    """The loaded CUDA library; raises if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    if not LIB_PATH.exists():
        raise RuntimeError(f"{LIB_PATH.name} is not built; run `python -m sparse_mixture_experts_fp32_b200.build`")
    L = ctypes.CDLL(str(LIB_PATH))
    P, S = ctypes.c_void_p, ctypes.c_size_t
    D = ctypes.POINTER(SwitchDims)
    I = ctypes.c_int
    sig = {
        "switch_capacity": (ctypes.c_int64, [ctypes.c_int64, ctypes.c_int32, ctypes.c_double]),
        "switch_workspace_size": (I, [D, ctypes.POINTER(ctypes.c_size_t)]),
        "switch_route": (I, [D, P, P, P, P, P, P, P, P, P, P, S, P]),
        "switch_route_noalloc": (I, [D, P, P, P, P, P, P, P, P, P, P]),
        "switch_dispatch": (I, [D, P, P, P, P, P]),
        "switch_expert_ffn": (I, [D, P, P, P, P, P, P, S, P]),
        "switch_combine": (I, [D, P, P, P, P, P, P]),
        "switch_layer_fwd": (I, [D, P, P, P, P, P, P, P, P, P, P, P, P, S, P]),
        "switch_route_top2": (I, [D, P, P, P, P, P, P, P, P, P, P, S, P]),
        "switch_combine_top2": (I, [D, P, P, P, P, P, P]),
        "switch_layer_fwd_top2": (I, [D, P, P, P, P, P, P, P, P, P, P, P, P, S, P]),
        "switch_layer_bwd": (I, [D, P, P, P, P, P, P, P, P, P, ctypes.c_float, P, P, P, P, P, P, S, P]),
        "switch_router_stats": (I, [D, P, P, S, P, P]),
        "switch_check": (I, [P, S, P]),
        "switch_selftest_wait_timeout": (I, [P, S, P]),
        "switch_check_noalloc": (I, [P]),
        "switch_selftest_wait_timeout_noalloc": (I, [P]),
        "switch_status_string": (ctypes.c_char_p, [I]),
        "switch_launch_count": (ctypes.c_int64, []),
        "switch_trace_start": (I, [ctypes.c_int32]),
        "switch_trace_read": (ctypes.c_int32, [P, P, ctypes.c_int32]),
        "switch_trace_stop": (None, []),
        "switch_kernel_name": (ctypes.c_char_p, [ctypes.c_int32]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(L, name)
        fn.restype = res
        fn.argtypes = args
    _lib = L
    return L


def _status_text(status: int) -> str:
    try:
        return lib().switch_status_string(status).decode()
    except Exception:
        return "?"


def _ok(status: int, where: str) -> None:
    if status != 0:
        raise SwitchError(status, where)


# ---------------------------------------------------------------------------
# marshalling helpers
# ---------------------------------------------------------------------------
def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    if not t.is_cuda:
        raise TypeError("switch_moe tensors must be CUDA tensors")
    if not t.is_contiguous():
        raise TypeError("switch_moe tensors must be contiguous")
    return t.data_ptr()


def _stream(stream, like=None):
    import torch
    if stream is None:
        dev = like.device if like is not None and hasattr(like, "device") else None
        return torch.cuda.current_stream(dev).cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def dtype_code(dtype) -> int:
    import torch
    if dtype == torch.float32:
        return SWITCH_F32
    if dtype == torch.bfloat16:
        return SWITCH_BF16
    raise TypeError(f"activations and expert weights must be float32 or bfloat16, got {dtype}")


def dims(T: int, d_model: int, d_ff: int, num_experts: int, capacity: int, dtype, flags: int = 0) -> SwitchDims:
    code = dtype if isinstance(dtype, int) else dtype_code(dtype)
    return SwitchDims(int(T), int(d_model), int(d_ff), int(num_experts), int(capacity), code, int(flags))


# ---------------------------------------------------------------------------
# low level: the C functions
# ---------------------------------------------------------------------------
def switch_capacity(T: int, num_experts: int, capacity_factor: float) -> int:
    return int(lib().switch_capacity(int(T), int(num_experts), float(capacity_factor)))


def switch_workspace_size(d: SwitchDims) -> int:
    out = ctypes.c_size_t(0)
    _ok(lib().switch_workspace_size(ctypes.byref(d), ctypes.byref(out)), "switch_workspace_size")
    return int(out.value)


def switch_route(d, x, w_r, logit_bias, expert, gate, slot, counts, slot_token, aux, workspace, stream=None):
    _ok(lib().switch_route(ctypes.byref(d), _ptr(x), _ptr(w_r), _ptr(logit_bias), _ptr(expert), _ptr(gate),
                           _ptr(slot), _ptr(counts), _ptr(slot_token), _ptr(aux), _ptr(workspace),
                           workspace.numel() * workspace.element_size(), _stream(stream, workspace)),
        "switch_route")


def switch_route_noalloc(d, x, w_r, logit_bias, expert, gate, slot, counts, slot_token, aux, stream=None):
    """switch_route without a workspace: for callers that cannot allocate
    device memory where they route (the scratch is a static array inside the
    library; calls that overlap on the GPU race)."""
    _ok(lib().switch_route_noalloc(ctypes.byref(d), _ptr(x), _ptr(w_r), _ptr(logit_bias), _ptr(expert), _ptr(gate),
                                   _ptr(slot), _ptr(counts), _ptr(slot_token), _ptr(aux), _stream(stream, counts)),
        "switch_route_noalloc")


def switch_dispatch(d, x, slot_token, counts, xbuf, stream=None):
    _ok(lib().switch_dispatch(ctypes.byref(d), _ptr(x), _ptr(slot_token), _ptr(counts), _ptr(xbuf),
                              _stream(stream, xbuf)), "switch_dispatch")


def switch_expert_ffn(d, xbuf, w_in, w_out, counts, ybuf, workspace, stream=None):
    _ok(lib().switch_expert_ffn(ctypes.byref(d), _ptr(xbuf), _ptr(w_in), _ptr(w_out), _ptr(counts), _ptr(ybuf),
                                _ptr(workspace), workspace.numel() * workspace.element_size(),
                                _stream(stream, workspace)), "switch_expert_ffn")


def switch_combine(d, ybuf, expert, slot, gate, y, stream=None):
    _ok(lib().switch_combine(ctypes.byref(d), _ptr(ybuf), _ptr(expert), _ptr(slot), _ptr(gate), _ptr(y),
                             _stream(stream, ybuf)), "switch_combine")


def switch_layer_fwd(d, x, w_r, logit_bias, w_in, w_out, y, expert, gate, slot, counts, aux, workspace, stream=None):
    _ok(lib().switch_layer_fwd(ctypes.byref(d), _ptr(x), _ptr(w_r), _ptr(logit_bias), _ptr(w_in), _ptr(w_out),
                               _ptr(y), _ptr(expert), _ptr(gate), _ptr(slot), _ptr(counts), _ptr(aux),
                               _ptr(workspace), workspace.numel() * workspace.element_size(),
                               _stream(stream, workspace)), "switch_layer_fwd")


def switch_route_top2(d, x, w_r, logit_bias, expert, gate, slot, counts, slot_token, aux, workspace, stream=None):
    _ok(lib().switch_route_top2(ctypes.byref(d), _ptr(x), _ptr(w_r), _ptr(logit_bias), _ptr(expert), _ptr(gate),
                                _ptr(slot), _ptr(counts), _ptr(slot_token), _ptr(aux), _ptr(workspace),
                                workspace.numel() * workspace.element_size(), _stream(stream, workspace)),
        "switch_route_top2")


def switch_combine_top2(d, ybuf, expert, slot, gate, y, stream=None):
    _ok(lib().switch_combine_top2(ctypes.byref(d), _ptr(ybuf), _ptr(expert), _ptr(slot), _ptr(gate), _ptr(y),
                                  _stream(stream, ybuf)), "switch_combine_top2")


def switch_layer_fwd_top2(d, x, w_r, logit_bias, w_in, w_out, y, expert, gate, slot, counts, aux, workspace,
                          stream=None):
    _ok(lib().switch_layer_fwd_top2(ctypes.byref(d), _ptr(x), _ptr(w_r), _ptr(logit_bias), _ptr(w_in), _ptr(w_out),
                                    _ptr(y), _ptr(expert), _ptr(gate), _ptr(slot), _ptr(counts), _ptr(aux),
                                    _ptr(workspace), workspace.numel() * workspace.element_size(),
                                    _stream(stream, workspace)), "switch_layer_fwd_top2")


def switch_layer_bwd(d, x, w_r, w_in, w_out, expert, gate, slot, counts, dy, g_aux, dx, dw_r, dbias, dw_in, dw_out,
                     workspace, stream=None):
    _ok(lib().switch_layer_bwd(ctypes.byref(d), _ptr(x), _ptr(w_r), _ptr(w_in), _ptr(w_out), _ptr(expert),
                               _ptr(gate), _ptr(slot), _ptr(counts), _ptr(dy), float(g_aux), _ptr(dx), _ptr(dw_r),
                               _ptr(dbias), _ptr(dw_in), _ptr(dw_out), _ptr(workspace),
                               workspace.numel() * workspace.element_size(), _stream(stream, workspace)),
        "switch_layer_bwd")


def switch_router_stats(d, counts, workspace, stats, stream=None):
    _ok(lib().switch_router_stats(ctypes.byref(d), _ptr(counts), _ptr(workspace),
                                  workspace.numel() * workspace.element_size(), _ptr(stats),
                                  _stream(stream, workspace)), "switch_router_stats")


def switch_check(workspace, stream=None) -> int:
    """Synchronise and return the device status code (0 = ok); does not raise."""
    return int(lib().switch_check(_ptr(workspace), workspace.numel() * workspace.element_size(),
                                  _stream(stream, workspace)))


def selftest_wait_timeout(workspace, stream=None) -> None:
    """Launch the bounded-wait self-test; switch_check(workspace) afterwards
    reports SWITCH_ERR_DEVICE_TIMEOUT (8)."""
    _ok(lib().switch_selftest_wait_timeout(_ptr(workspace), workspace.numel() * workspace.element_size(),
                                           _stream(stream, workspace)), "switch_selftest_wait_timeout")


def switch_check_noalloc(stream=None) -> int:
    """switch_check for the static array switch_route_noalloc uses (0 = ok); does not raise."""
    return int(lib().switch_check_noalloc(_stream(stream)))


def selftest_wait_timeout_noalloc(stream=None) -> None:
    """The bounded-wait self-test on the static routing array's status word."""
    _ok(lib().switch_selftest_wait_timeout_noalloc(_stream(stream)), "switch_selftest_wait_timeout_noalloc")


def launch_count() -> int:
    return int(lib().switch_launch_count())


def trace_start(max_launches: int) -> None:
    _ok(lib().switch_trace_start(int(max_launches)), "switch_trace_start")


def trace_read(capacity: int = 4096) -> list[tuple[str, float]]:
    ids = (ctypes.c_int32 * capacity)()
    ms = (ctypes.c_float * capacity)()
    n = lib().switch_trace_read(ids, ms, capacity)
    return [(lib().switch_kernel_name(ids[k]).decode(), float(ms[k])) for k in range(n)]


def trace_stop() -> None:
    lib().switch_trace_stop()


# ---------------------------------------------------------------------------
# high level: torch-allocating wrappers
# ---------------------------------------------------------------------------
def capacity(T: int, num_experts: int, capacity_factor: float) -> int:
    c = switch_capacity(T, num_experts, capacity_factor)
    if c < 1:
        raise ValueError("capacity needs T >= 0, num_experts >= 1 and a positive capacity factor")
    return c


def _resolve_capacity(T, N, cap, capacity_factor):
    if cap is not None:
        return int(cap)
    if capacity_factor is None:
        raise ValueError("give capacity or capacity_factor")
    c = switch_capacity(T, N, capacity_factor)
    if c < 1:
        raise ValueError("capacity needs T >= 0, num_experts >= 1 and a positive capacity factor")
    return c


def workspace(d: SwitchDims, device):
    import torch
    return torch.empty(switch_workspace_size(d), dtype=torch.uint8, device=device)


def layer_dims(x, w_in, capacity=None, capacity_factor=None, flags: int = 0) -> SwitchDims:
    T, dm = x.shape
    N, F, dm2 = w_in.shape
    if dm2 != dm:
        raise ValueError("w_in must be [N, d_ff, d_model]")
    if w_in.dtype != x.dtype:
        raise TypeError("x and the expert weights must share a dtype")
    C = _resolve_capacity(T, N, capacity, capacity_factor)
    return dims(T, dm, F, N, C, x.dtype, flags)


def layer_fwd(x, w_r, w_in, w_out, capacity=None, capacity_factor=None, logit_bias=None, flags: int = 0,
              ws=None, out=None, stream=None):
    """The Switch layer forward pass.  Returns a dict with y [T, d] float32
    (no residual), aux (1-element float32), expert, gate, slot, counts."""
    import torch
    d = layer_dims(x, w_in, capacity, capacity_factor, flags)
    T, dev = x.shape[0], x.device
    if out is None:
        out = dict(y=torch.empty(x.shape, dtype=torch.float32, device=dev), expert=torch.empty(T, dtype=torch.int32, device=dev),
                   gate=torch.empty(T, dtype=torch.float32, device=dev),
                   slot=torch.empty(T, dtype=torch.int32, device=dev),
                   counts=torch.empty(d.num_experts, dtype=torch.int32, device=dev),
                   aux=torch.empty(1, dtype=torch.float32, device=dev))
    if ws is None:
        ws = workspace(d, dev)
    switch_layer_fwd(d, x, w_r, logit_bias, w_in, w_out, out["y"], out["expert"], out["gate"], out["slot"],
                     out["counts"], out["aux"], ws, stream)
    out["capacity"] = d.capacity
    out["flags"] = d.flags
    out["workspace"] = ws
    return out


def route(x, w_r, num_experts=None, capacity=None, capacity_factor=None, logit_bias=None, d_ff: int = 64,
          ws=None, stream=None, flags: int = 0):
    """Router, top-1, capacity assignment, counts and aux (switch_route)."""
    import torch
    T, dm = x.shape
    N = w_r.shape[0] if num_experts is None else num_experts
    C = _resolve_capacity(T, N, capacity, capacity_factor)
    d = dims(T, dm, d_ff, N, C, x.dtype, flags)
    dev = x.device
    out = dict(expert=torch.empty(T, dtype=torch.int32, device=dev),
               gate=torch.empty(T, dtype=torch.float32, device=dev),
               slot=torch.empty(T, dtype=torch.int32, device=dev),
               counts=torch.empty(N, dtype=torch.int32, device=dev),
               slot_token=torch.empty(N * C, dtype=torch.int32, device=dev),
               aux=torch.empty(1, dtype=torch.float32, device=dev))
    if ws is None:
        ws = workspace(d, dev)
    switch_route(d, x, w_r, logit_bias, out["expert"], out["gate"], out["slot"], out["counts"], out["slot_token"],
                 out["aux"], ws, stream)
    out["capacity"] = C
    out["flags"] = d.flags
    out["workspace"] = ws
    return out


def layer_fwd_top2(x, w_r, w_in, w_out, capacity=None, capacity_factor=None, logit_bias=None, flags: int = 0,
                   ws=None, out=None, stream=None):
    """The top-2 mixture-of-experts layer forward pass.  Returns a dict with
    y [T, d] float32, aux, expert / gate / slot [T, 2], counts [N]."""
    import torch
    d = layer_dims(x, w_in, capacity, capacity_factor, flags)
    T, dev = x.shape[0], x.device
    if out is None:
        out = dict(y=torch.empty(x.shape, dtype=torch.float32, device=dev),
                   expert=torch.empty(T, 2, dtype=torch.int32, device=dev),
                   gate=torch.empty(T, 2, dtype=torch.float32, device=dev),
                   slot=torch.empty(T, 2, dtype=torch.int32, device=dev),
                   counts=torch.empty(d.num_experts, dtype=torch.int32, device=dev),
                   aux=torch.empty(1, dtype=torch.float32, device=dev))
    if ws is None:
        ws = workspace(d, dev)
    switch_layer_fwd_top2(d, x, w_r, logit_bias, w_in, w_out, out["y"], out["expert"], out["gate"], out["slot"],
                          out["counts"], out["aux"], ws, stream)
    out["capacity"] = d.capacity
    out["workspace"] = ws
    return out


def route_top2(x, w_r, capacity=None, capacity_factor=None, logit_bias=None, d_ff: int = 64, ws=None, stream=None,
               flags: int = 0):
    """Router, top-2, capacity assignment, counts and aux (switch_route_top2)."""
    import torch
    T, dm = x.shape
    N = w_r.shape[0]
    C = _resolve_capacity(T, N, capacity, capacity_factor)
    d = dims(T, dm, d_ff, N, C, x.dtype, flags)
    dev = x.device
    out = dict(expert=torch.empty(T, 2, dtype=torch.int32, device=dev),
               gate=torch.empty(T, 2, dtype=torch.float32, device=dev),
               slot=torch.empty(T, 2, dtype=torch.int32, device=dev),
               counts=torch.empty(N, dtype=torch.int32, device=dev),
               slot_token=torch.empty(N * C, dtype=torch.int32, device=dev),
               aux=torch.empty(1, dtype=torch.float32, device=dev))
    if ws is None:
        ws = workspace(d, dev)
    switch_route_top2(d, x, w_r, logit_bias, out["expert"], out["gate"], out["slot"], out["counts"],
                      out["slot_token"], out["aux"], ws, stream)
    out["capacity"] = C
    out["flags"] = d.flags
    out["workspace"] = ws
    return out


def layer_bwd(fwd: dict, x, w_r, w_in, w_out, dy, g_aux: float = 0.0, logit_bias=None, stream=None):
    """Gradients of sum(y * dy) + g_aux * aux after ``layer_fwd(..., flags=SWITCH_FLAG_TRAINING)``
    (whose result dict, with its workspace, is ``fwd``).  Returns dx, dw_r, dbias
    (None without a logit bias), dw_in, dw_out, all float32."""
    import torch
    T, dm = x.shape
    N, F, _ = w_in.shape
    dev = x.device
    d = layer_dims(x, w_in, capacity=fwd["capacity"], flags=fwd.get("flags", SWITCH_FLAG_TRAINING))
    out = dict(dx=torch.empty(T, dm, dtype=torch.float32, device=dev),
               dw_r=torch.empty(N, dm, dtype=torch.float32, device=dev),
               dbias=torch.empty(N, dtype=torch.float32, device=dev) if logit_bias is not None else None,
               dw_in=torch.empty(N, F, dm, dtype=torch.float32, device=dev),
               dw_out=torch.empty(N, dm, F, dtype=torch.float32, device=dev))
    switch_layer_bwd(d, x, w_r, w_in, w_out, fwd["expert"], fwd["gate"], fwd["slot"], fwd["counts"], dy, g_aux,
                     out["dx"], out["dw_r"], out["dbias"], out["dw_in"], out["dw_out"], fwd["workspace"], stream)
    return out


def router_stats(result: dict, T: int, d_model: int, d_ff: int, dtype, stream=None):
    """Router statistics of a route / layer_fwd result made with SWITCH_FLAG_ROUTER_STATS:
    a 4-element float32 tensor (mean entropy, dropped fraction, capacity utilisation, busiest load)."""
    import torch
    counts = result["counts"]
    d = dims(T, d_model, d_ff, counts.numel(), result["capacity"], dtype, result.get("flags", SWITCH_FLAG_ROUTER_STATS))
    stats = torch.empty(4, dtype=torch.float32, device=counts.device)
    switch_router_stats(d, counts, result["workspace"], stats, stream)
    return stats
