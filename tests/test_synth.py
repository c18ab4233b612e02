"""The seeded input generator: determinism, storage rounding and the recipe's shape."""
import numpy as np
import torch

from sparse_mixture_experts_fp32_b200 import synth


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(0)
    a = np.concatenate([rng.standard_normal(100000) * 10.0 ** rng.integers(-6, 6, 100000),
                        np.array([0.0, -0.0, 1.0, -1.0, 3.0e38, 1e-40], np.float32)]).astype(np.float32)
    ours = synth.to_bf16_bits(a)
    ref = torch.from_numpy(a).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)
    back = synth.bf16_bits_to_f32(ours)
    assert np.array_equal(back, torch.from_numpy(a).to(torch.bfloat16).float().numpy())


def test_deterministic_and_independent_streams():
    wl = synth.WORKLOADS["base8"].with_tokens(64)
    a = synth.inputs(wl, experts=[1, 3])
    b = synth.inputs(wl, experts=[3])
    assert np.array_equal(a["x"], b["x"]) and np.array_equal(a["w_r"], b["w_r"])
    assert np.array_equal(a["w_in"][3], b["w_in"][3]) and np.array_equal(a["w_out"][3], b["w_out"][3])
    assert not a["w_in"][0].any() and a["w_in"][1].any()
    assert not np.array_equal(a["w_in"][1], a["w_in"][3])


def test_truncation_and_scale():
    rng = np.random.default_rng(1)
    z = synth.truncated_normal(rng, (400000,), 0.5)
    assert np.abs(z).max() <= 1.0 + 1e-7
    # std of N(0,1) truncated at +-2 is 0.8796
    assert abs(z.std() / 0.5 - 0.8796) < 0.01


def test_zipf_bias():
    b = synth.zipf_bias(8, 1.1)
    w = np.arange(1, 9, dtype=np.float64) ** -1.1
    w /= w.sum()
    assert np.allclose(np.exp(b / 0.5), w, rtol=1e-6)
    assert np.all(np.diff(b) < 0)


def test_workload_table():
    w = synth.WORKLOADS
    assert (w["tiny_fp32"].T, w["tiny_fp32"].d_model, w["tiny_fp32"].d_ff, w["tiny_fp32"].num_experts) == (64, 32, 64, 4)
    assert (w["base8"].T, w["base8"].d_model, w["base8"].d_ff, w["base8"].num_experts) == (8192, 768, 3072, 8)
    assert (w["base128_skew"].T, w["base128_skew"].num_experts, w["base128_skew"].zipf_s) == (65536, 128, 1.1)
    assert (w["large128"].T, w["large128"].d_model, w["large128"].d_ff) == (131072, 1024, 4096)
    assert w["bigexpert64"].sweep == (0.5, 1.0, 1.25, 2.0)
    x = synth.activations(w["tiny_fp32"])
    assert x.dtype == np.float32 and x.shape == (64, 32)
    assert synth.activations(w["base8"], T=16).dtype == np.uint16
