"""Seeded synthetic inputs for the Switch layer workloads.

This module is shared by the tests, the benchmark and the smoke check, and it
feeds both the CUDA library and the CPU oracle.  It holds none of the layer's
arithmetic: it only draws random numbers, rounds them to the storage type and
builds the optional per-expert logit bias.

Recipe (numpy ``Generator(PCG64)``; one independent stream per tensor):

* activations ``x[T, d]`` ~ N(0, 1), drawn in float32 and rounded to nearest
  even bfloat16 for the bf16 workloads;
* router ``W_r[N, d]`` and expert weights ``W_in[e][F, d]``, ``W_out[e][d, F]``
  ~ N(0, std) truncated at +-2 std by resampling, std = 0.1 / sqrt(fan_in)
  (fan_in = d for W_r and W_in, F for W_out).  The 0.1 factor follows the
  reduced initialisation scale of the Switch Transformer (llm-papers-study
  "精读 06 | Switch Transformers", §3.5, smaller parameter initialisation);
* ``W_r`` and the bias stay float32 (selective precision); expert weights are
  bfloat16, except in the all-float32 tiny workload;
* skewed workloads add ``bias[i] = 0.5 * ln(w_(i+1))`` where
  ``w_k = k^-s / sum_j j^-s`` is the Zipf(s) weight of rank k, so expert 0 is
  the most popular;
* each expert's weights come from their own stream, so any subset of experts
  can be regenerated on its own.

bfloat16 tensors are returned as ``uint16`` arrays of bit patterns.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

F32 = "f32"
BF16 = "bf16"

_STREAM_X, _STREAM_WR, _STREAM_WIN, _STREAM_WOUT = 0, 1, 2, 3


@dataclass(frozen=True)
class Workload:
    name: str
    T: int
    d_model: int
    d_ff: int
    num_experts: int
    capacity_factor: float
    dtype: str
    zipf_s: float | None = None
    bias_scale: float = 0.5
    seed: int = 0
    sweep: tuple = field(default_factory=tuple)
    note: str = ""

    def with_tokens(self, T: int) -> "Workload":
        return Workload(self.name, T, self.d_model, self.d_ff, self.num_experts, self.capacity_factor,
                        self.dtype, self.zipf_s, self.bias_scale, self.seed, self.sweep, self.note)

    def with_capacity_factor(self, c: float) -> "Workload":
        return Workload(self.name, self.T, self.d_model, self.d_ff, self.num_experts, c, self.dtype,
                        self.zipf_s, self.bias_scale, self.seed, self.sweep, self.note)


# The five Switch-layer workloads.  Token counts are whole 512-token sequences
# except for the tiny float32 case.
WORKLOADS = {
    "tiny_fp32": Workload("tiny_fp32", 64, 32, 64, 4, 1.0, F32, seed=1,
                          note="tiny Switch layer, float32 everywhere"),
    "base8": Workload("base8", 8192, 768, 3072, 8, 1.25, BF16, seed=2,
                      note="Switch-Base-8 layer, 16 x 512 tokens"),
    "base128_skew": Workload("base128_skew", 65536, 768, 3072, 128, 1.0, BF16, zipf_s=1.1, seed=3,
                             note="Switch-Base-128 layer, 128 x 512 tokens, Zipf(1.1) logit bias"),
    "large128": Workload("large128", 131072, 1024, 4096, 128, 1.25, BF16, seed=4,
                         note="Switch-Large-shaped layer, 256 x 512 tokens, near-uniform routing"),
    "bigexpert64": Workload("bigexpert64", 32768, 4096, 10240, 64, 1.0, BF16, zipf_s=0.8, seed=5,
                            sweep=(0.5, 1.0, 1.25, 2.0),
                            note="large-expert layer, Zipf(0.8) logit bias, capacity-factor sweep"),
}


def _rng(seed: int, *stream: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, *stream])))


def truncated_normal(rng: np.random.Generator, shape, std: float) -> np.ndarray:
    """N(0, std^2) in float32, values beyond +-2 std redrawn until none remain."""
    z = rng.standard_normal(size=shape, dtype=np.float32)
    flat = z.reshape(-1)
    bad = np.flatnonzero(np.abs(flat) > 2.0)
    while bad.size:
        flat[bad] = rng.standard_normal(size=bad.size, dtype=np.float32)
        bad = bad[np.abs(flat[bad]) > 2.0]
    z *= np.float32(std)
    return z


def to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bfloat16 (ties to even); return the bit patterns."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    rounded = (u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)
    return rounded.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def zipf_bias(N: int, s: float, scale: float = 0.5) -> np.ndarray:
    ranks = np.arange(1, N + 1, dtype=np.float64)
    w = ranks ** (-s)
    w /= w.sum()
    return (scale * np.log(w)).astype(np.float32)


def _store(a: np.ndarray, dtype: str) -> np.ndarray:
    return to_bf16_bits(a) if dtype == BF16 else a


def activations(wl: Workload, seed: int | None = None, T: int | None = None) -> np.ndarray:
    seed = wl.seed if seed is None else seed
    T = wl.T if T is None else T
    x = _rng(seed, _STREAM_X).standard_normal(size=(T, wl.d_model), dtype=np.float32)
    return _store(x, wl.dtype)


def router_weight(wl: Workload, seed: int | None = None) -> np.ndarray:
    seed = wl.seed if seed is None else seed
    return truncated_normal(_rng(seed, _STREAM_WR), (wl.num_experts, wl.d_model), 0.1 / np.sqrt(wl.d_model))


def router_bias(wl: Workload) -> np.ndarray | None:
    if wl.zipf_s is None:
        return None
    return zipf_bias(wl.num_experts, wl.zipf_s, wl.bias_scale)


def expert_weights(wl: Workload, e: int, seed: int | None = None) -> tuple[np.ndarray, np.ndarray]:
    """(W_in[e] of shape [F, d], W_out[e] of shape [d, F]) in the workload's storage type."""
    seed = wl.seed if seed is None else seed
    w_in = truncated_normal(_rng(seed, _STREAM_WIN, e), (wl.d_ff, wl.d_model), 0.1 / np.sqrt(wl.d_model))
    w_out = truncated_normal(_rng(seed, _STREAM_WOUT, e), (wl.d_model, wl.d_ff), 0.1 / np.sqrt(wl.d_ff))
    return _store(w_in, wl.dtype), _store(w_out, wl.dtype)


def all_expert_weights(wl: Workload, seed: int | None = None, experts=None) -> tuple[np.ndarray, np.ndarray]:
    """Stacked [N, F, d] and [N, d, F] expert weights.

    With ``experts`` given, only those experts are drawn and the others are left
    as zeros (allocated lazily), for checks that read only the listed experts.
    """
    N, d, F = wl.num_experts, wl.d_model, wl.d_ff
    np_t = np.uint16 if wl.dtype == BF16 else np.float32
    w_in = np.zeros((N, F, d), dtype=np_t)
    w_out = np.zeros((N, d, F), dtype=np_t)
    for e in (range(N) if experts is None else experts):
        w_in[e], w_out[e] = expert_weights(wl, int(e), seed)
    return w_in, w_out


def inputs(wl: Workload, seed: int | None = None, T: int | None = None, experts=None) -> dict:
    """Everything one layer call needs, as numpy arrays."""
    w_in, w_out = all_expert_weights(wl, seed, experts)
    return dict(x=activations(wl, seed, T), w_r=router_weight(wl, seed), bias=router_bias(wl),
                w_in=w_in, w_out=w_out)
