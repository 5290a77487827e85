"""Thin Python binding of the C ABI in include/moe.h (libmoe_b200.so).

Argument marshalling only: torch tensors are passed as raw device pointers
with the current CUDA stream; every step of the layer runs in the library's
kernels.  There is no fallback: if the library is missing or fails to load,
every call raises.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Tuple

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoe_b200.so")

MOE_OK = 0
MOE_ERR_INVALID_ARG = -1
MOE_ERR_UNSUPPORTED = -2
MOE_ERR_CUDA = -3
MOE_ERR_WORKSPACE = -4
MOE_ERR_TIMEOUT = -5
MOE_ERR_DEVICE = -6
MOE_F32, MOE_BF16 = 0, 1

# workspace regions (indices into moe_workspace_layout)
WS_REGIONS = ["status", "counts", "offsets", "block_counts", "topk_idx", "topk_w", "row_src",
              "x_perm", "h", "h_shared", "slots", "y_shared"]
WS_TOTAL = len(WS_REGIONS)
ROW_ALIGN = 128

# every entry point declared in include/moe.h
SYMBOLS = ["moe_workspace_bytes", "moe_workspace_layout", "moe_route", "moe_forward",
           "moe_get_device_status", "moe_clear_device_status", "moe_selftest_timeout",
           "moe_set_stage_events", "moe_status_string", "moe_version",
           "moe_expert_counts_noalloc", "moe_route_ex", "moe_forward_ex", "moe_saved_bytes",
           "moe_forward_train", "moe_backward_workspace_bytes", "moe_backward",
           "moe_set_backward_stage_events", "moe_dispatch_workspace_bytes", "moe_dispatch",
           "moe_experts_workspace_bytes", "moe_experts_forward", "moe_shared_workspace_bytes",
           "moe_shared_forward", "moe_combine"]
GATES = {"sigmoid": 0, "softmax": 1}  # MOE_GATE_SIGMOID, MOE_GATE_SOFTMAX_TOPK
N_STAGE_EVENTS = 6
STAGES = ["route", "permute", "gate_up", "down", "combine"]

_lib = None


class MoeError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {status_string(status)} ({status})")


def lib() -> ctypes.CDLL:
    """Load libmoe_b200.so (raises if it is missing: there is no other path)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"CUDA library not built: {LIB_PATH} "
                               "(python -m sparse_mixture_experts_03_b200.build)")
        L = ctypes.CDLL(LIB_PATH)
        i, vp, sz = ctypes.c_int, ctypes.c_void_p, ctypes.c_size_t
        L.moe_workspace_bytes.argtypes = [i] * 7
        L.moe_workspace_bytes.restype = sz
        L.moe_workspace_layout.argtypes = [i] * 7 + [ctypes.POINTER(sz), i]
        L.moe_workspace_layout.restype = i
        L.moe_route.argtypes = [vp, vp] + [i] * 7 + [vp, vp, vp]
        L.moe_route.restype = i
        L.moe_forward.argtypes = [vp] * 5 + [i] * 10 + [vp, vp, vp, vp, sz, vp]
        L.moe_forward.restype = i
        L.moe_get_device_status.argtypes = [vp, ctypes.POINTER(i), ctypes.POINTER(i), vp]
        L.moe_get_device_status.restype = i
        L.moe_clear_device_status.argtypes = [vp, vp]
        L.moe_clear_device_status.restype = i
        L.moe_selftest_timeout.argtypes = [vp, i, vp]
        L.moe_selftest_timeout.restype = i
        L.moe_set_stage_events.argtypes = [ctypes.POINTER(vp), i]
        L.moe_set_stage_events.restype = i
        L.moe_status_string.argtypes = [i]
        L.moe_status_string.restype = ctypes.c_char_p
        L.moe_version.restype = i
        L.moe_expert_counts_noalloc.argtypes = [vp, i, i, i, vp, vp, vp]
        L.moe_expert_counts_noalloc.restype = i
        L.moe_route_ex.argtypes = [vp, vp] + [i] * 8 + [vp, vp, vp, vp]
        L.moe_route_ex.restype = i
        L.moe_forward_ex.argtypes = [vp] * 5 + [i] * 11 + [vp, vp, vp, vp, vp, vp, sz, vp]
        L.moe_forward_ex.restype = i
        L.moe_saved_bytes.argtypes = [i] * 4
        L.moe_saved_bytes.restype = sz
        L.moe_forward_train.argtypes = ([vp] * 5 + [i] * 11 + [vp, vp, vp, vp, vp, vp, sz, vp, sz,
                                                               vp])
        L.moe_forward_train.restype = i
        L.moe_backward_workspace_bytes.argtypes = [i] * 6
        L.moe_backward_workspace_bytes.restype = sz
        L.moe_backward.argtypes = [vp] * 9 + [i] * 8 + [vp] * 6 + [sz, vp]
        L.moe_backward.restype = i
        L.moe_set_backward_stage_events.argtypes = [ctypes.POINTER(vp), i]
        L.moe_set_backward_stage_events.restype = i
        L.moe_dispatch_workspace_bytes.argtypes = [i] * 3
        L.moe_dispatch_workspace_bytes.restype = sz
        L.moe_dispatch.argtypes = [vp, vp] + [i] * 8 + [vp] * 8 + [sz, vp]
        L.moe_dispatch.restype = i
        L.moe_experts_workspace_bytes.argtypes = [i] * 4
        L.moe_experts_workspace_bytes.restype = sz
        L.moe_experts_forward.argtypes = [vp, vp, vp, i, i, vp, vp, i, i, i, i, vp, vp, sz, vp]
        L.moe_experts_forward.restype = i
        L.moe_shared_workspace_bytes.argtypes = [i] * 4
        L.moe_shared_workspace_bytes.restype = sz
        L.moe_shared_forward.argtypes = [vp, vp, i, i, i, i, i, vp, vp, sz, vp]
        L.moe_shared_forward.restype = i
        L.moe_combine.argtypes = [vp, i, vp, vp, i, i, i, i, vp, vp, vp]
        L.moe_combine.restype = i
        _lib = L
    return _lib


def status_string(status: int) -> str:
    return lib().moe_status_string(status).decode()


def _dt(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return MOE_BF16
    if t.dtype == torch.float32:
        return MOE_F32
    raise TypeError(f"unsupported dtype {t.dtype}")


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_contiguous():
        raise ValueError("tensors must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream: Optional[torch.cuda.Stream]):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _check(status: int, what: str) -> None:
    if status != MOE_OK:
        raise MoeError(status, what)


def workspace_bytes(T, d, E, k, inter, n_shared, dtype: torch.dtype) -> int:
    n = lib().moe_workspace_bytes(T, d, E, k, inter, n_shared,
                                  MOE_BF16 if dtype == torch.bfloat16 else MOE_F32)
    if n == 0:
        raise MoeError(MOE_ERR_INVALID_ARG, "moe_workspace_bytes")
    return int(n)


def workspace_layout(T, d, E, k, inter, n_shared, dtype: torch.dtype) -> dict:
    arr = (ctypes.c_size_t * (WS_TOTAL + 1))()
    _check(lib().moe_workspace_layout(T, d, E, k, inter, n_shared,
                                      MOE_BF16 if dtype == torch.bfloat16 else MOE_F32,
                                      arr, WS_TOTAL + 1), "moe_workspace_layout")
    out = {name: int(arr[i]) for i, name in enumerate(WS_REGIONS)}
    out["total"] = int(arr[WS_TOTAL])
    return out


def alloc_workspace(T, d, E, k, inter, n_shared, dtype, device="cuda") -> torch.Tensor:
    return torch.empty(workspace_bytes(T, d, E, k, inter, n_shared, dtype), dtype=torch.uint8,
                       device=device)


def route(x: torch.Tensor, W_router: torch.Tensor, k: int, n_group: int, topk_group: int,
          topk_idx: Optional[torch.Tensor] = None, topk_w: Optional[torch.Tensor] = None,
          stream=None, gate: str = "sigmoid",
          expert_bias: Optional[torch.Tensor] = None) -> Tuple[torch.Tensor, torch.Tensor]:
    """moe_route_ex: (topk_idx int32 [T,k], topk_w fp32 [T,k]); gate "sigmoid"
    or "softmax", expert_bias a device float32 [E] selection-only bias."""
    T, d = x.shape
    E = W_router.shape[0]
    if topk_idx is None:
        topk_idx = torch.empty(T, k, dtype=torch.int32, device=x.device)
    if topk_w is None:
        topk_w = torch.empty(T, k, dtype=torch.float32, device=x.device)
    _check(lib().moe_route_ex(_ptr(x), _ptr(W_router), T, d, E, k, n_group, topk_group, _dt(x),
                              GATES[gate], _ptr(expert_bias), _ptr(topk_idx), _ptr(topk_w),
                              _stream(stream)), "moe_route_ex")
    return topk_idx, topk_w


def expert_counts_noalloc(topk_idx: torch.Tensor, E: int, counts: torch.Tensor,
                          offsets: torch.Tensor, stream=None) -> None:
    """moe_expert_counts_noalloc: counts int32 [E] and offsets int32 [E+1] of a
    routing result, into the caller's tensors; the library allocates nothing."""
    T, k = topk_idx.shape
    _check(lib().moe_expert_counts_noalloc(_ptr(topk_idx), T, k, E, _ptr(counts), _ptr(offsets),
                                           _stream(stream)), "moe_expert_counts_noalloc")


def forward(x: torch.Tensor, W_router: torch.Tensor, W_gate_up: torch.Tensor,
            W_down: torch.Tensor, W_shared: Optional[torch.Tensor], k: int, n_group: int,
            topk_group: int, inter: int, n_shared: int, out_dtype: torch.dtype = torch.float32,
            y: Optional[torch.Tensor] = None, topk_idx: Optional[torch.Tensor] = None,
            topk_w: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
            stream=None, gate: str = "sigmoid", expert_bias: Optional[torch.Tensor] = None,
            expert_load: Optional[torch.Tensor] = None) -> torch.Tensor:
    """moe_forward_ex: y [T, d] in out_dtype (float32 or bfloat16).  gate
    "sigmoid" (the FusionLLM gate) or "softmax" (over the chosen k);
    expert_bias: device float32 [E] selection-only bias; expert_load: device
    int32 [E] filled with the tokens routed to each expert."""
    T, d = x.shape
    E = W_router.shape[0]
    if y is None:
        y = torch.empty(T, d, dtype=out_dtype, device=x.device)
    if workspace is None:
        workspace = alloc_workspace(T, d, E, k, inter, n_shared, x.dtype, x.device)
    st = lib().moe_forward_ex(_ptr(x), _ptr(W_router), _ptr(W_gate_up), _ptr(W_down),
                              _ptr(W_shared), T, d, E, k, n_group, topk_group, inter, n_shared,
                              _dt(x), _dt(y), GATES[gate], _ptr(expert_bias), _ptr(y),
                              _ptr(topk_idx), _ptr(topk_w), _ptr(expert_load),
                              _ptr(workspace), workspace.numel(), _stream(stream))
    _check(st, "moe_forward_ex")
    return y


def saved_bytes(T, k, inter, n_shared) -> int:
    """Bytes of the pre-activations moe_forward_train saves for the backward."""
    return int(lib().moe_saved_bytes(T, k, inter, n_shared))


def forward_train(x: torch.Tensor, W_router: torch.Tensor, W_gate_up: torch.Tensor,
                  W_down: torch.Tensor, W_shared: Optional[torch.Tensor], k: int, n_group: int,
                  topk_group: int, inter: int, n_shared: int,
                  out_dtype: torch.dtype = torch.float32, y: Optional[torch.Tensor] = None,
                  topk_idx: Optional[torch.Tensor] = None, topk_w: Optional[torch.Tensor] = None,
                  saved: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
                  stream=None, gate: str = "sigmoid", expert_bias: Optional[torch.Tensor] = None,
                  expert_load: Optional[torch.Tensor] = None):
    """moe_forward_train: (y, topk_idx, topk_w, saved) -- the forward plus the
    routing and pre-activations that backward() takes."""
    T, d = x.shape
    E = W_router.shape[0]
    dev = x.device
    if y is None:
        y = torch.empty(T, d, dtype=out_dtype, device=dev)
    if topk_idx is None:
        topk_idx = torch.empty(T, k, dtype=torch.int32, device=dev)
    if topk_w is None:
        topk_w = torch.empty(T, k, dtype=torch.float32, device=dev)
    if saved is None:
        saved = torch.empty(max(saved_bytes(T, k, inter, n_shared), 16), dtype=torch.uint8,
                            device=dev)
    if workspace is None:
        workspace = alloc_workspace(T, d, E, k, inter, n_shared, x.dtype, dev)
    st = lib().moe_forward_train(_ptr(x), _ptr(W_router), _ptr(W_gate_up), _ptr(W_down),
                                 _ptr(W_shared), T, d, E, k, n_group, topk_group, inter, n_shared,
                                 _dt(x), _dt(y), GATES[gate], _ptr(expert_bias), _ptr(y),
                                 _ptr(topk_idx), _ptr(topk_w), _ptr(expert_load), _ptr(saved),
                                 saved.numel(), _ptr(workspace), workspace.numel(),
                                 _stream(stream))
    _check(st, "moe_forward_train")
    return y, topk_idx, topk_w, saved


def backward_workspace_bytes(T, d, E, k, inter, n_shared) -> int:
    n = lib().moe_backward_workspace_bytes(T, d, E, k, inter, n_shared)
    if n == 0:
        raise MoeError(MOE_ERR_UNSUPPORTED, "moe_backward_workspace_bytes")
    return int(n)


class Grads:
    """fp32 gradients of the layer: dx [T,d], dW_router [E,d], dW_gate_up
    [E,2I,d], dW_down [E,d,I], dW_shared [3*SI*d] or None."""

    def __init__(self, dx, dW_router, dW_gate_up, dW_down, dW_shared):
        self.dx, self.dW_router, self.dW_gate_up = dx, dW_router, dW_gate_up
        self.dW_down, self.dW_shared = dW_down, dW_shared


def alloc_grads(T, d, E, inter, n_shared, device="cuda") -> Grads:
    f = dict(dtype=torch.float32, device=device)
    SI = n_shared * inter
    return Grads(torch.empty(T, d, **f), torch.empty(E, d, **f), torch.empty(E, 2 * inter, d, **f),
                 torch.empty(E, d, inter, **f), torch.empty(3 * SI * d, **f) if n_shared else None)


def backward(x: torch.Tensor, W_router: torch.Tensor, W_gate_up: torch.Tensor,
             W_down: torch.Tensor, W_shared: Optional[torch.Tensor], dy: torch.Tensor,
             topk_idx: torch.Tensor, topk_w: torch.Tensor, saved: torch.Tensor, k: int,
             inter: int, n_shared: int, gate: str = "sigmoid", grads: Optional[Grads] = None,
             workspace: Optional[torch.Tensor] = None, stream=None) -> Grads:
    """moe_backward: gradients of the layer for the forward_train call that
    returned topk_idx, topk_w and saved; dy = dL/dy in the dtype of x."""
    T, d = x.shape
    E = W_router.shape[0]
    if grads is None:
        grads = alloc_grads(T, d, E, inter, n_shared, x.device)
    if workspace is None:
        workspace = torch.empty(backward_workspace_bytes(T, d, E, k, inter, n_shared),
                                dtype=torch.uint8, device=x.device)
    st = lib().moe_backward(_ptr(x), _ptr(W_router), _ptr(W_gate_up), _ptr(W_down),
                            _ptr(W_shared), _ptr(dy), _ptr(topk_idx), _ptr(topk_w), _ptr(saved),
                            T, d, E, k, inter, n_shared, _dt(x), GATES[gate], _ptr(grads.dx),
                            _ptr(grads.dW_router), _ptr(grads.dW_gate_up), _ptr(grads.dW_down),
                            _ptr(grads.dW_shared), _ptr(workspace), workspace.numel(),
                            _stream(stream))
    _check(st, "moe_backward")
    return grads


def device_status(workspace: torch.Tensor, stream=None) -> Tuple[int, int]:
    """(status, site) of the last moe_forward using `workspace` (synchronises)."""
    s, w = ctypes.c_int(0), ctypes.c_int(0)
    _check(lib().moe_get_device_status(_ptr(workspace), ctypes.byref(s), ctypes.byref(w),
                                       _stream(stream)), "moe_get_device_status")
    return s.value, w.value


def clear_device_status(workspace: torch.Tensor, stream=None) -> None:
    _check(lib().moe_clear_device_status(_ptr(workspace), _stream(stream)),
           "moe_clear_device_status")


def selftest_timeout(workspace: torch.Tensor, limit_us: int, stream=None) -> None:
    _check(lib().moe_selftest_timeout(_ptr(workspace), limit_us, _stream(stream)),
           "moe_selftest_timeout")


def set_stage_events(events) -> None:
    """Record torch.cuda.Event objects at stage boundaries of every following
    forward (None turns it off).  The events must have been recorded once so
    that their CUDA handles exist."""
    if events is None:
        _check(lib().moe_set_stage_events(None, 0), "moe_set_stage_events")
        return
    arr = (ctypes.c_void_p * len(events))(
        *[ctypes.c_void_p(e.cuda_event if e is not None else None) for e in events])
    _check(lib().moe_set_stage_events(arr, len(events)), "moe_set_stage_events")


BWD_STAGES = ["gather", "dgrad_down", "dlogit", "dgrad_gate_up", "dx_sum", "wgrad_down",
              "wgrad_gate_up", "dweight_router"]
N_BWD_STAGE_EVENTS = len(BWD_STAGES) + 1


def set_backward_stage_events(events) -> None:
    """Record torch.cuda.Event objects at the stage boundaries of every
    following backward (None turns it off); see set_stage_events."""
    if events is None:
        _check(lib().moe_set_backward_stage_events(None, 0), "moe_set_backward_stage_events")
        return
    arr = (ctypes.c_void_p * len(events))(
        *[ctypes.c_void_p(e.cuda_event if e is not None else None) for e in events])
    _check(lib().moe_set_backward_stage_events(arr, len(events)),
           "moe_set_backward_stage_events")


# ---- expert parallelism (the compute on either side of the all-to-all exchanges)

class Dispatched:
    """One rank's moe_dispatch result: topk_idx / topk_w [T,k], counts int32
    [E] (rows per expert), x_perm bf16 [T*k,d] (rows by expert, then token),
    w_perm f32 [T*k] (each row's gate weight), slot_row int32 [T*k] (slot
    t*k+j -> its row)."""

    def __init__(self, topk_idx, topk_w, counts, x_perm, w_perm, slot_row):
        self.topk_idx, self.topk_w, self.counts = topk_idx, topk_w, counts
        self.x_perm, self.w_perm, self.slot_row = x_perm, w_perm, slot_row


def _scratch(n: int, device) -> torch.Tensor:
    if n == 0:
        raise MoeError(MOE_ERR_INVALID_ARG, "workspace size")
    return torch.empty(n, dtype=torch.uint8, device=device)


def dispatch(x: torch.Tensor, W_router: torch.Tensor, k: int, n_group: int, topk_group: int,
             gate: str = "sigmoid", expert_bias: Optional[torch.Tensor] = None,
             workspace: Optional[torch.Tensor] = None, stream=None) -> Dispatched:
    """moe_dispatch: routing and expert-contiguous rows of this rank's tokens."""
    T, d = x.shape
    E = W_router.shape[0]
    dev = x.device
    out = Dispatched(torch.empty(T, k, dtype=torch.int32, device=dev),
                     torch.empty(T, k, dtype=torch.float32, device=dev),
                     torch.empty(E, dtype=torch.int32, device=dev),
                     torch.empty(T * k, d, dtype=x.dtype, device=dev),
                     torch.empty(T * k, dtype=torch.float32, device=dev),
                     torch.empty(T * k, dtype=torch.int32, device=dev))
    if workspace is None:
        workspace = _scratch(lib().moe_dispatch_workspace_bytes(T, E, k), dev)
    _check(lib().moe_dispatch(_ptr(x), _ptr(W_router), T, d, E, k, n_group, topk_group, _dt(x),
                              GATES[gate], _ptr(expert_bias), _ptr(out.topk_idx),
                              _ptr(out.topk_w), _ptr(out.counts), _ptr(out.x_perm),
                              _ptr(out.w_perm), _ptr(out.slot_row), _ptr(workspace),
                              workspace.numel(), _stream(stream)), "moe_dispatch")
    return out


def experts_forward(x_rows: torch.Tensor, w_rows: torch.Tensor, recv_counts: torch.Tensor,
                    W_gate_up: torch.Tensor, W_down: torch.Tensor, inter: int,
                    y_rows: Optional[torch.Tensor] = None,
                    workspace: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """moe_experts_forward: y_rows bf16 [R,d] = w * local expert(row), in the
    receive order; recv_counts int32 [n_src, E_local] on the device."""
    R, d = x_rows.shape
    n_src, E_l = recv_counts.shape
    if y_rows is None:
        y_rows = torch.empty(R, d, dtype=x_rows.dtype, device=x_rows.device)
    if workspace is None:
        workspace = _scratch(lib().moe_experts_workspace_bytes(R, d, E_l, inter), x_rows.device)
    _check(lib().moe_experts_forward(_ptr(x_rows), _ptr(w_rows), _ptr(recv_counts), n_src, R,
                                     _ptr(W_gate_up), _ptr(W_down), d, E_l, inter, _dt(x_rows),
                                     _ptr(y_rows), _ptr(workspace), workspace.numel(),
                                     _stream(stream)), "moe_experts_forward")
    return y_rows


def shared_forward(x: torch.Tensor, W_shared: torch.Tensor, inter: int, n_shared: int,
                   y_shared: Optional[torch.Tensor] = None,
                   workspace: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """moe_shared_forward: fp32 [T,d] sum of the shared experts."""
    T, d = x.shape
    if y_shared is None:
        y_shared = torch.empty(T, d, dtype=torch.float32, device=x.device)
    if workspace is None:
        workspace = _scratch(lib().moe_shared_workspace_bytes(T, d, inter, n_shared), x.device)
    _check(lib().moe_shared_forward(_ptr(x), _ptr(W_shared), T, d, inter, n_shared, _dt(x),
                                    _ptr(y_shared), _ptr(workspace), workspace.numel(),
                                    _stream(stream)), "moe_shared_forward")
    return y_shared


def combine(rows: torch.Tensor, slot_row: torch.Tensor, shared: Optional[torch.Tensor], T: int,
            k: int, out_dtype: torch.dtype = torch.float32, y: Optional[torch.Tensor] = None,
            status_ws: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """moe_combine: y [T,d] = shared + the k rows of each token, in order."""
    n_rows, d = rows.shape
    if y is None:
        y = torch.empty(T, d, dtype=out_dtype, device=rows.device)
    _check(lib().moe_combine(_ptr(rows), n_rows, _ptr(slot_row), _ptr(shared), T, d, k, _dt(y),
                             _ptr(y), _ptr(status_ws), _stream(stream)), "moe_combine")
    return y


class MoELayer:
    """Device-resident weights plus a reusable workspace for one layer shape."""

    def __init__(self, x_example_T: int, W_router, W_gate_up, W_down, W_shared, k, n_group,
                 topk_group, inter, n_shared, out_dtype=torch.float32):
        self.W_router, self.W_gate_up, self.W_down, self.W_shared = (
            W_router, W_gate_up, W_down, W_shared)
        self.k, self.n_group, self.topk_group = k, n_group, topk_group
        self.inter, self.n_shared, self.out_dtype = inter, n_shared, out_dtype
        self.E, self.d = W_router.shape
        self.T_cap = x_example_T
        self.workspace = alloc_workspace(x_example_T, self.d, self.E, k, inter, n_shared,
                                         W_router.dtype, W_router.device)

    def __call__(self, x: torch.Tensor, y: Optional[torch.Tensor] = None, topk_idx=None,
                 topk_w=None, stream=None) -> torch.Tensor:
        if x.shape[0] > self.T_cap:
            raise ValueError("more tokens than the workspace was sized for")
        return forward(x, self.W_router, self.W_gate_up, self.W_down, self.W_shared, self.k,
                       self.n_group, self.topk_group, self.inter, self.n_shared,
                       self.out_dtype, y=y, topk_idx=topk_idx, topk_w=topk_w,
                       workspace=self.workspace, stream=stream)
