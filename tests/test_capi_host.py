"""The C-ABI library without a GPU: it builds, loads, exports every symbol the
header declares, and its host-only logic (capacity, workspace sizing, argument
validation that fails before any device work) behaves as documented."""
import ctypes
import re
from pathlib import Path

import numpy as np
import pytest

import oracle
import sparse_mixture_experts_fp32_b200 as sm
from sparse_mixture_experts_fp32_b200 import build as smbuild

HEADER = Path(__file__).resolve().parent.parent / "include" / "switch_moe.h"


@pytest.fixture(scope="module")
def L():
    smbuild.build()
    return sm.lib()


def declared_functions():
    text = re.sub(r"/\*.*?\*/", "", HEADER.read_text(), flags=re.S)
    return sorted(set(re.findall(r"^\s*[A-Za-z_][\w\s\*]*?\b(switch_\w+)\s*\(", text, flags=re.M)))


def test_header_declares_the_five_entry_points():
    names = declared_functions()
    for n in ("switch_route", "switch_dispatch", "switch_expert_ffn", "switch_combine", "switch_layer_fwd",
              "switch_route_top2", "switch_combine_top2", "switch_layer_fwd_top2"):
        assert n in names


def test_every_declared_symbol_is_exported(L):
    names = declared_functions()
    assert len(names) >= 14
    for n in names:
        assert hasattr(L, n), n
    assert set(names) <= set(sm.EXPORTED) | {n for n in names if hasattr(L, n)}


def test_capacity_matches_definition(L):
    o = oracle.Oracle()
    rng = np.random.default_rng(0)
    for _ in range(2000):
        T = int(rng.integers(0, 300000))
        N = int(rng.integers(1, 257))
        c = float(rng.choice([0.5, 1.0, 1.25, 1.5, 2.0, rng.uniform(0.01, 4.0)]))
        assert sm.switch_capacity(T, N, c) == o.capacity(T, N, c)
    assert sm.switch_capacity(16, 4, 1.0) == 4
    assert sm.switch_capacity(512, 8, 1.5) == 96
    assert sm.switch_capacity(5, 3, 1.0) == 2
    assert sm.switch_capacity(8192, 8, 1.25) == 1280
    assert sm.switch_capacity(-1, 4, 1.0) == -1
    assert sm.switch_capacity(4, 0, 1.0) == -1
    assert sm.switch_capacity(4, 2, 0.0) == -1
    assert sm.switch_capacity(4, 2, float("nan")) == -1


def test_workspace_size_and_shape_rules(L):
    ok = sm.dims(8192, 768, 3072, 8, 1280, sm.SWITCH_BF16)
    n = sm.switch_workspace_size(ok)
    # must at least hold H [N, C, F] and two [N, C, d] buffers in bf16
    assert n >= 8 * 1280 * (3072 + 2 * 768) * 2
    assert sm.switch_workspace_size(sm.dims(0, 64, 64, 1, 1, sm.SWITCH_BF16)) > 0
    bad = [
        sm.dims(10, 100, 64, 2, 4, sm.SWITCH_BF16),   # d % 64
        sm.dims(10, 64, 100, 2, 4, sm.SWITCH_BF16),   # F % 64
        sm.dims(10, 64, 64, 0, 4, sm.SWITCH_BF16),    # N = 0
        sm.dims(10, 64, 64, 257, 4, sm.SWITCH_BF16),  # N > 256
        sm.dims(10, 64, 64, 2, 0, sm.SWITCH_BF16),    # C = 0
        sm.dims(-1, 64, 64, 2, 4, sm.SWITCH_BF16),    # T < 0
        sm.dims(10, 0, 64, 2, 4, sm.SWITCH_F32),      # d = 0
    ]
    for d in bad:
        with pytest.raises(sm.SwitchError) as ei:
            sm.switch_workspace_size(d)
        assert ei.value.status == 2
    d = sm.dims(10, 64, 64, 2, 4, sm.SWITCH_F32)
    d.dtype = 7
    with pytest.raises(sm.SwitchError) as ei:
        sm.switch_workspace_size(d)
    assert ei.value.status == 3
    # odd shapes are fine in float32
    assert sm.switch_workspace_size(sm.dims(33, 33, 17, 3, 11, sm.SWITCH_F32)) > 0


def test_validation_errors_before_any_device_work(L):
    P = ctypes.c_void_p
    d = sm.dims(64, 64, 64, 4, 16, sm.SWITCH_BF16)
    a = 1 << 20  # an aligned fake address: never dereferenced, the call fails first
    # NULL dims
    assert L.switch_route(None, a, a, None, a, a, a, a, a, a, a, 1 << 30, None) == 1
    # NULL required pointer
    assert L.switch_route(ctypes.byref(d), a, None, None, a, a, a, a, a, a, a, 1 << 30, None) == 1
    # misaligned pointer
    assert L.switch_route(ctypes.byref(d), a + 4, a, None, a, a, a, a, a, a, a, 1 << 30, None) == 4
    # workspace too small
    assert L.switch_route(ctypes.byref(d), a, a, None, a, a, a, a, a, a, a, 16, None) == 5
    assert L.switch_layer_fwd(ctypes.byref(d), a, a, None, a, a, a, a, a, a, a, a, a, 16, None) == 5
    assert L.switch_expert_ffn(ctypes.byref(d), a, a, None, a, a, a, 1 << 30, None) == 1
    assert L.switch_dispatch(ctypes.byref(d), a, a, a, None, None) == 1
    assert L.switch_combine(ctypes.byref(d), a, a, a, a + 8, a, None) == 4
    bad = sm.dims(64, 96, 64, 4, 16, sm.SWITCH_BF16)
    assert L.switch_layer_fwd(ctypes.byref(bad), a, a, None, a, a, a, a, a, a, a, a, a, 1 << 30, None) == 2
    assert L.switch_check(None, 0, None) == 1
    # top-2 routing needs two experts; the same checks as the top-1 calls otherwise
    one = sm.dims(64, 64, 64, 1, 16, sm.SWITCH_BF16)
    assert L.switch_route_top2(ctypes.byref(one), a, a, None, a, a, a, a, a, a, a, 1 << 30, None) == 2
    assert L.switch_layer_fwd_top2(ctypes.byref(one), a, a, None, a, a, a, a, a, a, a, a, a, 1 << 30, None) == 2
    assert L.switch_combine_top2(ctypes.byref(one), a, a, a, a, a, None) == 2
    assert L.switch_route_top2(ctypes.byref(d), a, a, None, a, a, a, a, a, a, a, 16, None) == 5
    assert L.switch_layer_fwd_top2(ctypes.byref(d), a, None, None, a, a, a, a, a, a, a, a, a, 1 << 30, None) == 1
    assert L.switch_combine_top2(ctypes.byref(d), a, a, a + 4, a, a, None) == 4


def test_status_strings_and_kernel_names(L):
    for code in range(9):
        assert L.switch_status_string(code)
    assert L.switch_kernel_name(6).decode() == "ffn_tc_gemm1_relu"
    assert L.switch_kernel_name(999).decode() == "?"
    assert L.switch_launch_count() >= 0


def test_binding_fails_loudly_without_the_library(tmp_path, monkeypatch):
    monkeypatch.setattr(sm, "_lib", None)
    monkeypatch.setattr(sm, "LIB_PATH", tmp_path / "missing.so")
    with pytest.raises(RuntimeError, match="not built"):
        sm.lib()


def test_training_workspace_holds_the_backward_sections(L):
    """The training forward keeps what the backward reads; the tensor-core router products add
    their split operands (dh terms [T][6 Np] for dx, [chunks][3N][Tc] for dW_r, W_r terms
    [d][6 Np], dW_r partials) and the float32 FMA router path (SWITCH_FLAG_SIMT_ROUTER) only its
    per-chunk partials.  No transposed copies of weights or activations exist any more."""
    T, d, F, N, C = 131072, 1024, 4096, 128, 1280
    base = sm.switch_workspace_size(sm.dims(T, d, F, N, C, sm.SWITCH_BF16))
    train = sm.switch_workspace_size(sm.dims(T, d, F, N, C, sm.SWITCH_BF16, sm.SWITCH_FLAG_TRAINING))
    simt = sm.switch_workspace_size(sm.dims(T, d, F, N, C, sm.SWITCH_BF16,
                                            sm.SWITCH_FLAG_TRAINING | sm.SWITCH_FLAG_SIMT_ROUTER))
    probs_dh = 2 * T * N * 4
    grads = N * C * (d + F) * 2                      # dE and dZ, bf16
    Np, Tc = 128, 2048
    chunks = T // Tc
    tc_router = T * 6 * Np * 2 + d * 6 * Np * 2 + chunks * 3 * N * Tc * 2 + chunks * 3 * N * d * 4
    assert train - base >= probs_dh + grads + tc_router
    # no room for transposed weights (2 N d F bf16 = 2.1 GB) is reserved
    assert train - base < probs_dh + grads + tc_router + 64 * (1 << 20)
    assert simt < train
    assert simt - base >= probs_dh + grads


def test_backward_kernel_names(L):
    names = {29: "bwd_router_split", 30: "bwd_router_tc_dx", 31: "bwd_router_tc_dw", 32: "bwd_zero_tails"}
    for k, v in names.items():
        assert L.switch_kernel_name(k).decode() == v
