"""Host-side checks of the C-ABI library (no GPU needed): it loads, exports
every entry point include/moe.h declares, computes workspace sizes, and
rejects invalid arguments before touching the device."""
import ctypes
import os
import re

import pytest
import torch

from sparse_mixture_experts_03_b200 import moe

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_symbols():
    with open(os.path.join(ROOT, "include", "moe.h")) as f:
        text = f.read()
    return sorted(set(re.findall(r"MOE_API\s+[\w\s\*]+?\b(moe_\w+)\s*\(", text)))


def test_header_symbols_match_binding_list():
    assert declared_symbols() == sorted(moe.SYMBOLS)


def test_library_exports_every_declared_symbol():
    L = moe.lib()
    for name in declared_symbols():
        assert hasattr(L, name), name
    assert L.moe_version() == 1


def test_status_strings():
    for code in range(-6, 1):
        assert moe.status_string(code) != "unknown status"
    assert moe.status_string(-99) == "unknown status"


def test_workspace_layout_regions():
    T, d, E, k, I, S = 4096, 2048, 64, 6, 1536, 4
    lay = moe.workspace_layout(T, d, E, k, I, S, torch.bfloat16)
    offs = [lay[n] for n in moe.WS_REGIONS] + [lay["total"]]
    assert offs == sorted(offs) and offs[0] == 0
    assert all(o % 1024 == 0 for o in offs)
    rows_cap = T * k + moe.ROW_ALIGN * E
    assert lay["h"] - lay["x_perm"] >= rows_cap * d * 2
    assert lay["slots"] - lay["h_shared"] >= T * S * I * 2
    assert lay["total"] - lay["slots"] >= T * k * d * 2  # bf16 slots
    assert moe.workspace_bytes(T, d, E, k, I, S, torch.bfloat16) == lay["total"]


@pytest.mark.parametrize("args", [
    (64, 100, 8, 2, 256, 0),      # d % 64
    (64, 128, 8, 2, 200, 0),      # inter % 128
    (64, 128, 300, 2, 256, 0),    # E > 256
    (64, 128, 8, 9, 256, 0),      # k > 8
    (-1, 128, 8, 2, 256, 0),      # T < 0
])
def test_workspace_bytes_rejects_bad_sizes(args):
    assert moe.lib().moe_workspace_bytes(*args, moe.MOE_BF16) == 0


def _route(T=8, d=128, E=8, k=2, G=1, TG=1, dt=moe.MOE_F32):
    return moe.lib().moe_route(None, None, T, d, E, k, G, TG, dt, None, None, None)


def test_route_rejects_invalid_arguments_on_host():
    assert _route(E=8, G=3) == moe.MOE_ERR_INVALID_ARG          # E % n_group
    assert _route(G=2, TG=3) == moe.MOE_ERR_INVALID_ARG         # topk_group > n_group
    assert _route(E=8, k=5, G=2, TG=1) == moe.MOE_ERR_INVALID_ARG  # k > TG * E/G
    assert _route(d=96) == moe.MOE_ERR_UNSUPPORTED              # d % 64
    assert _route(dt=7) == moe.MOE_ERR_INVALID_ARG
    assert _route(T=0) == moe.MOE_OK                            # empty batch queues nothing


def test_forward_rejects_bad_workspace_and_shared_mismatch():
    L = moe.lib()
    f = lambda W_sh, S, ws, wsb: L.moe_forward(None, None, None, None, W_sh, 8, 256, 8, 2, 1, 1,
                                               128, S, moe.MOE_BF16, moe.MOE_F32, None, None,
                                               None, ws, wsb, None)
    assert f(None, 1, None, 0) == moe.MOE_ERR_INVALID_ARG           # shared count without weights
    assert f(None, 0, None, 0) == moe.MOE_ERR_WORKSPACE             # no workspace
    assert f(None, 0, ctypes.c_void_p(256), 10) == moe.MOE_ERR_WORKSPACE  # too small
    # bf16 path needs d % 256
    assert L.moe_forward(None, None, None, None, None, 8, 192, 8, 2, 1, 1, 128, 0, moe.MOE_BF16,
                         moe.MOE_F32, None, None, None, None, 0, None) == moe.MOE_ERR_UNSUPPORTED


def _backward(T=8, d=256, E=8, k=2, I=256, S=0, dt=moe.MOE_BF16, gate=0, W_sh=None, dW_sh=None,
              ws=None, wsb=0):
    return moe.lib().moe_backward(None, None, None, None, W_sh, None, None, None, None, T, d, E,
                                  k, I, S, dt, gate, None, None, None, None, dW_sh, ws, wsb, None)


def test_training_entry_points_reject_invalid_arguments_on_host():
    assert _backward(dt=moe.MOE_F32) == moe.MOE_ERR_UNSUPPORTED      # bf16 layers only
    assert _backward(I=128) == moe.MOE_ERR_UNSUPPORTED               # inter % 256
    assert _backward(d=100) == moe.MOE_ERR_UNSUPPORTED               # d % 64 (size check)
    assert _backward(d=320) == moe.MOE_ERR_UNSUPPORTED               # d % 256 (bf16 GEMMs)
    assert _backward(gate=5) == moe.MOE_ERR_INVALID_ARG              # unknown gate
    assert _backward(S=1) == moe.MOE_ERR_INVALID_ARG                 # shared count without weights
    assert _backward(S=0, W_sh=ctypes.c_void_p(256)) == moe.MOE_ERR_INVALID_ARG
    assert _backward() == moe.MOE_ERR_WORKSPACE                      # no workspace
    assert _backward(ws=ctypes.c_void_p(256), wsb=16) == moe.MOE_ERR_WORKSPACE
    assert _backward(k=9) == moe.MOE_ERR_INVALID_ARG                 # k > 8
    # forward_train: bf16 only; T > 0 needs routing outputs and a saved buffer
    L = moe.lib()
    ft = lambda dt, saved, sb, idx=None, w=None: L.moe_forward_train(
        None, None, None, None, None, 8, 256, 8, 2, 1, 1, 256, 0, dt, moe.MOE_F32, 0, None, None,
        idx, w, None, saved, sb, None, 0, None)
    assert ft(moe.MOE_F32, None, 0) == moe.MOE_ERR_UNSUPPORTED
    assert ft(moe.MOE_BF16, None, 0) == moe.MOE_ERR_INVALID_ARG       # no topk outputs
    assert ft(moe.MOE_BF16, None, 0, ctypes.c_void_p(256), ctypes.c_void_p(512)) == \
        moe.MOE_ERR_INVALID_ARG                                       # no saved buffer


def test_training_buffer_sizes():
    T, d, E, k, I, S = 4096, 2048, 64, 6, 1536, 4
    # saved: routed [T*k, 2I] then shared [T, 2*S*I], bf16
    assert moe.saved_bytes(T, k, I, S) == 2 * (T * k * 2 * I + T * 2 * S * I)
    assert moe.saved_bytes(T, k, I, 0) == 2 * T * k * 2 * I
    n = moe.backward_workspace_bytes(T, d, E, k, I, S)
    rows_cap = T * k + moe.ROW_ALIGN * E
    # at least: x and dy rows, dg|du and w*h per padded row, dx slots, shared rows
    assert n >= 2 * rows_cap * (2 * d + 3 * I) + 2 * T * k * d + 2 * T * 3 * S * I
    assert n % 1024 == 0
    assert moe.lib().moe_backward_workspace_bytes(T, d, E, k, 1664, S) == 0  # inter % 256
    assert moe.lib().moe_backward_workspace_bytes(T, 2112, E, k, I, S) == 0  # d % 256
