"""fp64 CPU oracle for the Switch Transformer sparse FFN layer forward pass.

TEST INFRASTRUCTURE ONLY: the test-suite, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg are the only callers.  The product library never
imports, links or executes anything in this folder, and this folder imports
nothing from the product package.

The arithmetic lives in ``switch_oracle.c`` (plain C, double precision,
OpenMP over independent tokens).  This module compiles it with gcc on first
use and wraps it with ctypes; the numpy code here only marshals arguments.
"""
from __future__ import annotations

import ctypes
import hashlib
import os
import subprocess
from pathlib import Path

import numpy as np

_HERE = Path(__file__).resolve().parent
_SRC = _HERE / "switch_oracle.c"
_BUILD = _HERE / "_build"

F32 = 0
BF16 = 1

_lib = None


def _source_tag() -> str:
    return hashlib.sha1(_SRC.read_bytes()).hexdigest()[:12]


def library_path() -> Path:
    return _BUILD / f"liboracle_{_source_tag()}.so"


def build(force: bool = False, source: Path | None = None, out: Path | None = None) -> Path:
    """Compile the oracle (or another copy of its source) into a shared object."""
    src = Path(source) if source is not None else _SRC
    dst = Path(out) if out is not None else library_path()
    if dst.exists() and not force:
        return dst
    dst.parent.mkdir(parents=True, exist_ok=True)
    tmp = dst.with_suffix(f".{os.getpid()}.tmp")
    cmd = ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-o", str(tmp), str(src), "-lm"]
    subprocess.run(cmd, check=True, capture_output=True)
    os.replace(tmp, dst)
    return dst


def _bind(lib: ctypes.CDLL) -> ctypes.CDLL:
    P = ctypes.c_void_p
    I64, I32, D = ctypes.c_int64, ctypes.c_int32, ctypes.c_double
    lib.oracle_capacity.argtypes = [I64, I32, D]
    lib.oracle_capacity.restype = I64
    lib.oracle_router_logits.argtypes = [I64, I32, I32, P, ctypes.c_int, P, P, P]
    lib.oracle_router_logits.restype = None
    lib.oracle_softmax_top1.argtypes = [I64, I32, P, P, P, P, P, P]
    lib.oracle_softmax_top1.restype = None
    lib.oracle_assign.argtypes = [I64, I32, I64, P, P, P, P]
    lib.oracle_assign.restype = None
    lib.oracle_aux.argtypes = [I64, I32, P, P]
    lib.oracle_aux.restype = D
    lib.oracle_expert_row.argtypes = [I32, I32, P, ctypes.c_int, P, P, ctypes.c_int, D, P]
    lib.oracle_expert_row.restype = None
    lib.oracle_output_rows.argtypes = [I32, I32, I64, P, P, ctypes.c_int, P, P, ctypes.c_int, P, P, P, P]
    lib.oracle_output_rows.restype = None
    lib.oracle_threads.argtypes = []
    lib.oracle_threads.restype = ctypes.c_int
    lib.oracle_softmax_top2.argtypes = [I64, I32, P, P, P, P, P, P]
    lib.oracle_softmax_top2.restype = None
    lib.oracle_assign_top2.argtypes = [I64, I32, I64, P, P, P, P, P]
    lib.oracle_assign_top2.restype = None
    lib.oracle_output_rows_top2.argtypes = [I32, I32, I64, P, P, ctypes.c_int, P, P, ctypes.c_int, P, P, P, P]
    lib.oracle_output_rows_top2.restype = None
    lib.oracle_layer_bwd.argtypes = [I64, I32, I32, I32, I64, P, ctypes.c_int, P, P, P, P, ctypes.c_int, P, D,
                                     P, P, P, P, P]
    lib.oracle_layer_bwd.restype = None
    lib.oracle_router_stats.argtypes = [I64, I32, I64, P, P, P]
    lib.oracle_router_stats.restype = None
    lib.oracle_set_threads.argtypes = [ctypes.c_int]
    lib.oracle_set_threads.restype = None
    return lib


def load(path: Path | None = None) -> ctypes.CDLL:
    """Load the default oracle build, or a given shared object built from a copy."""
    global _lib
    if path is not None:
        return _bind(ctypes.CDLL(str(path)))
    if _lib is None:
        _lib = _bind(ctypes.CDLL(str(build())))
    return _lib


def _ptr(a: np.ndarray | None):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def dtype_code(a: np.ndarray) -> int:
    """float32 arrays hold binary32 values; uint16 arrays hold bfloat16 bit patterns."""
    if a.dtype == np.float32:
        return F32
    if a.dtype == np.uint16:
        return BF16
    raise TypeError(f"oracle element arrays must be float32 or uint16 (bf16 bits), got {a.dtype}")


class Oracle:
    """Thin marshalling layer over one loaded oracle shared object."""

    def __init__(self, lib: ctypes.CDLL | None = None):
        self.lib = lib if lib is not None else load()

    def threads(self) -> int:
        return int(self.lib.oracle_threads())

    def set_threads(self, n: int) -> None:
        """Threads of the OpenMP loops from now on (timing only; results do not depend on it)."""
        self.lib.oracle_set_threads(int(n))

    def capacity(self, T: int, N: int, c: float) -> int:
        return int(self.lib.oracle_capacity(T, N, float(c)))

    def router_logits(self, x: np.ndarray, w_r: np.ndarray, bias: np.ndarray | None = None) -> np.ndarray:
        x = np.ascontiguousarray(x)
        w_r = np.ascontiguousarray(w_r, dtype=np.float32)
        T, d = x.shape
        N = w_r.shape[0]
        assert w_r.shape == (N, d)
        b = None if bias is None else np.ascontiguousarray(bias, dtype=np.float32)
        h = np.empty((T, N), dtype=np.float64)
        self.lib.oracle_router_logits(T, d, N, _ptr(x), dtype_code(x), _ptr(w_r), _ptr(b), _ptr(h))
        return h

    def softmax_top1(self, h: np.ndarray, want_probs: bool = False) -> dict:
        h = np.ascontiguousarray(h, dtype=np.float64)
        T, N = h.shape
        expert = np.empty(T, dtype=np.int32)
        gate = np.empty(T, dtype=np.float64)
        margin = np.empty(T, dtype=np.float64)
        prob_sum = np.empty(N, dtype=np.float64)
        probs = np.empty((T, N), dtype=np.float64) if want_probs else None
        self.lib.oracle_softmax_top1(T, N, _ptr(h), _ptr(expert), _ptr(gate), _ptr(margin),
                                     _ptr(prob_sum), _ptr(probs))
        out = dict(expert=expert, gate=gate, margin=margin, prob_sum=prob_sum)
        if want_probs:
            out["probs"] = probs
        return out

    def assign(self, expert: np.ndarray, N: int, C: int) -> dict:
        expert = np.ascontiguousarray(expert, dtype=np.int32)
        T = expert.shape[0]
        slot = np.empty(T, dtype=np.int32)
        counts = np.empty(N, dtype=np.int32)
        slot_token = np.empty(N * C, dtype=np.int32)
        self.lib.oracle_assign(T, N, C, _ptr(expert), _ptr(slot), _ptr(counts), _ptr(slot_token))
        return dict(slot=slot, counts=counts, slot_token=slot_token.reshape(N, C))

    def aux(self, T: int, counts: np.ndarray, prob_sum: np.ndarray) -> float:
        counts = np.ascontiguousarray(counts, dtype=np.int32)
        prob_sum = np.ascontiguousarray(prob_sum, dtype=np.float64)
        return float(self.lib.oracle_aux(T, counts.shape[0], _ptr(counts), _ptr(prob_sum)))

    def route(self, x, w_r, bias=None, capacity: int | None = None, capacity_factor: float | None = None,
              want_probs: bool = False) -> dict:
        """Router, top-1, capacity assignment and aux loss for all tokens."""
        T = x.shape[0]
        N = w_r.shape[0]
        if capacity is None:
            capacity = self.capacity(T, N, capacity_factor)
        h = self.router_logits(x, w_r, bias)
        r = self.softmax_top1(h, want_probs=want_probs)
        a = self.assign(r["expert"], N, capacity)
        r.update(a)
        r["logits"] = h
        r["capacity"] = capacity
        r["aux"] = self.aux(T, a["counts"], r["prob_sum"])
        return r

    def output_rows(self, rows, x, w_in, w_out, expert, slot, gate) -> np.ndarray:
        """Layer output rows (fp64) for the given token indices."""
        rows = np.ascontiguousarray(rows, dtype=np.int64)
        x = np.ascontiguousarray(x)
        T, d = x.shape
        N, F, d2 = w_in.shape
        assert d2 == d and w_out.shape == (N, d, F)
        assert w_in.flags.c_contiguous and w_out.flags.c_contiguous and w_in.dtype == w_out.dtype
        expert = np.ascontiguousarray(expert, dtype=np.int32)
        slot = np.ascontiguousarray(slot, dtype=np.int32)
        gate = np.ascontiguousarray(gate, dtype=np.float64)
        y = np.empty((rows.shape[0], d), dtype=np.float64)
        self.lib.oracle_output_rows(d, F, rows.shape[0], _ptr(rows), _ptr(x), dtype_code(x), _ptr(w_in),
                                    _ptr(w_out), dtype_code(w_in), _ptr(expert), _ptr(slot), _ptr(gate),
                                    _ptr(y))
        return y

    # ---- top-2 routing (the classic mixture-of-experts variant) ----------
    def softmax_top2(self, h: np.ndarray, want_probs: bool = False) -> dict:
        h = np.ascontiguousarray(h, dtype=np.float64)
        T, N = h.shape
        if N < 2:
            raise ValueError("top-2 routing needs at least two experts")
        expert = np.empty((T, 2), dtype=np.int32)
        gate = np.empty((T, 2), dtype=np.float64)
        margin = np.empty((T, 2), dtype=np.float64)
        prob_sum = np.empty(N, dtype=np.float64)
        probs = np.empty((T, N), dtype=np.float64) if want_probs else None
        self.lib.oracle_softmax_top2(T, N, _ptr(h), _ptr(expert), _ptr(gate), _ptr(margin), _ptr(prob_sum),
                                     _ptr(probs))
        out = dict(expert=expert, gate=gate, margin=margin, prob_sum=prob_sum)
        if want_probs:
            out["probs"] = probs
        return out

    def assign_top2(self, expert: np.ndarray, N: int, C: int) -> dict:
        expert = np.ascontiguousarray(expert, dtype=np.int32)
        T = expert.shape[0]
        assert expert.shape == (T, 2)
        slot = np.empty((T, 2), dtype=np.int32)
        counts = np.empty(N, dtype=np.int32)
        counts_first = np.empty(N, dtype=np.int32)
        slot_token = np.empty(N * C, dtype=np.int32)
        self.lib.oracle_assign_top2(T, N, C, _ptr(expert), _ptr(slot), _ptr(counts), _ptr(counts_first),
                                    _ptr(slot_token))
        return dict(slot=slot, counts=counts, counts_first=counts_first, slot_token=slot_token.reshape(N, C))

    def route_top2(self, x, w_r, bias=None, capacity: int | None = None, capacity_factor: float | None = None,
                   want_probs: bool = False) -> dict:
        """Router, top-2, capacity assignment and aux loss for all tokens."""
        T = x.shape[0]
        N = w_r.shape[0]
        if capacity is None:
            capacity = self.capacity(T, N, capacity_factor)
        h = self.router_logits(x, w_r, bias)
        r = self.softmax_top2(h, want_probs=want_probs)
        a = self.assign_top2(r["expert"], N, capacity)
        r.update(a)
        r["logits"] = h
        r["capacity"] = capacity
        r["aux"] = self.aux(T, a["counts_first"], r["prob_sum"])
        return r

    def output_rows_top2(self, rows, x, w_in, w_out, expert, slot, gate) -> np.ndarray:
        """Top-2 layer output rows (fp64) for the given token indices."""
        rows = np.ascontiguousarray(rows, dtype=np.int64)
        x = np.ascontiguousarray(x)
        T, d = x.shape
        N, F, d2 = w_in.shape
        assert d2 == d and w_out.shape == (N, d, F)
        assert w_in.flags.c_contiguous and w_out.flags.c_contiguous and w_in.dtype == w_out.dtype
        expert = np.ascontiguousarray(expert, dtype=np.int32)
        slot = np.ascontiguousarray(slot, dtype=np.int32)
        gate = np.ascontiguousarray(gate, dtype=np.float64)
        assert expert.shape == (T, 2) and slot.shape == (T, 2) and gate.shape == (T, 2)
        y = np.empty((rows.shape[0], d), dtype=np.float64)
        self.lib.oracle_output_rows_top2(d, F, rows.shape[0], _ptr(rows), _ptr(x), dtype_code(x), _ptr(w_in),
                                         _ptr(w_out), dtype_code(w_in), _ptr(expert), _ptr(slot), _ptr(gate),
                                         _ptr(y))
        return y

    def layer_fwd_top2(self, x, w_r, w_in, w_out, bias=None, capacity=None, capacity_factor=None,
                       want_probs: bool = False) -> dict:
        """The whole top-2 layer for every token."""
        r = self.route_top2(x, w_r, bias, capacity, capacity_factor, want_probs=want_probs)
        rows = np.arange(x.shape[0], dtype=np.int64)
        r["y"] = self.output_rows_top2(rows, x, w_in, w_out, r["expert"], r["slot"], r["gate"])
        return r

    def layer_bwd(self, x, w_r, w_in, w_out, dy, g_aux: float = 0.0, bias=None, capacity=None,
                  capacity_factor=None) -> dict:
        """Gradients of sum(y * dy) + g_aux * aux with respect to x, W_r, the
        logit bias, W_in and W_out (fp64), for the top-1 layer."""
        x = np.ascontiguousarray(x)
        T, d = x.shape
        N, F, d2 = w_in.shape
        assert d2 == d and w_out.shape == (N, d, F) and w_in.dtype == w_out.dtype
        w_r = np.ascontiguousarray(w_r, dtype=np.float32)
        b = None if bias is None else np.ascontiguousarray(bias, dtype=np.float32)
        w_in = np.ascontiguousarray(w_in)
        w_out = np.ascontiguousarray(w_out)
        dy = np.ascontiguousarray(dy, dtype=np.float64)
        assert dy.shape == (T, d)
        if capacity is None:
            capacity = self.capacity(T, N, capacity_factor)
        out = dict(dx=np.empty((T, d)), dw_r=np.empty((N, d)), dbias=np.empty(N) if b is not None else None,
                   dw_in=np.empty((N, F, d)), dw_out=np.empty((N, d, F)))
        self.lib.oracle_layer_bwd(T, d, F, N, capacity, _ptr(x), dtype_code(x), _ptr(w_r), _ptr(b), _ptr(w_in),
                                  _ptr(w_out), dtype_code(w_in), _ptr(dy), float(g_aux), _ptr(out["dx"]),
                                  _ptr(out["dw_r"]), _ptr(out["dbias"]), _ptr(out["dw_in"]), _ptr(out["dw_out"]))
        out["capacity"] = capacity
        return out

    def router_stats(self, probs: np.ndarray, counts: np.ndarray, C: int) -> dict:
        """Mean router entropy, dropped-token fraction, capacity utilisation, busiest-expert load."""
        probs = np.ascontiguousarray(probs, dtype=np.float64)
        counts = np.ascontiguousarray(counts, dtype=np.int32)
        T, N = probs.shape
        out = np.empty(4, dtype=np.float64)
        self.lib.oracle_router_stats(T, N, int(C), _ptr(probs), _ptr(counts), _ptr(out))
        return dict(entropy=out[0], drop_fraction=out[1], capacity_utilisation=out[2], max_load=out[3])

    def expert_row(self, x_row, w_in_e, w_out_e, gate: float) -> np.ndarray:
        x_row = np.ascontiguousarray(x_row)
        F, d = w_in_e.shape
        w_in_e = np.ascontiguousarray(w_in_e)
        w_out_e = np.ascontiguousarray(w_out_e)
        y = np.empty(d, dtype=np.float64)
        self.lib.oracle_expert_row(d, F, _ptr(x_row), dtype_code(x_row), _ptr(w_in_e), _ptr(w_out_e),
                                   dtype_code(w_in_e), float(gate), _ptr(y))
        return y

    def layer_fwd(self, x, w_r, w_in, w_out, bias=None, capacity=None, capacity_factor=None,
                  want_probs: bool = False) -> dict:
        """The whole layer for every token: route() plus all output rows."""
        r = self.route(x, w_r, bias, capacity, capacity_factor, want_probs=want_probs)
        rows = np.arange(x.shape[0], dtype=np.int64)
        r["y"] = self.output_rows(rows, x, w_in, w_out, r["expert"], r["slot"], r["gate"])
        return r
