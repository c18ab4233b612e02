"""Host-side pieces of bench.py: the kernel work table and the lookup of DRAM
traffic in committed ncu summaries (no GPU needed)."""
import shutil
import sys
from pathlib import Path

import numpy as np

ROOT = Path(__file__).resolve().parents[1]
sys.path.insert(0, str(ROOT))
import bench  # noqa: E402
from sparse_mixture_experts_fp32_b200 import synth  # noqa: E402


def test_kernel_work_base8():
    wl = synth.WORKLOADS["base8"]
    C = 1280
    counts = np.full(wl.num_experts, wl.T // wl.num_experts, dtype=np.int64)
    work = bench.kernel_work(wl, C, counts)
    K = wl.T  # nothing dropped with equal counts below C
    assert work["ffn_tc_fused"] == ("tensor", 4.0 * K * wl.d_model * wl.d_ff, None)
    assert work["_meta"][1]["K"] == K
    # the router reads x once (bf16), W_r, and writes expert + gate per token plus per-tile partials
    tiles = -(-wl.T // 64)
    assert work["router_staged"][1] == wl.T * wl.d_model * 2 + wl.num_experts * wl.d_model * 4 + 8 * wl.T + \
        8 * wl.num_experts * tiles
    # the combine writes y in float32; its activation-dtype figure counts T*d*s written + K*d*s read
    T, d = wl.T, wl.d_model
    assert work["combine"][1] == T * d * 4 + K * d * 4 + 12 * T
    assert work["combine"][2] == T * d * 2 + K * d * 2 + 12 * T


def test_kernel_entry_fractions():
    peaks = {"hbm_gbs": 6000.0, "bf16_tflops": 1500.0, "bf16_tflops_sustained": 1200.0}
    e = bench.kernel_entry("tensor", 3.0e12, None, 2.0, 1, peaks)  # 3 TFLOP in 2 ms = 1500 TFLOP/s
    assert e["frac"] == 1.0 and e["frac_sustained"] == 1.25
    h = bench.kernel_entry("hbm", 6.0e9, 3.0e9, 1.0, 4, peaks)     # 6 GB in 1 ms = 6000 GB/s
    assert h["frac"] == 1.0 and h["frac_act_dtype"] == 0.5 and h["launches"] == 4


def _fake_tree(tmp_path):
    """A copy of the sources and an empty profiles folder under tmp_path."""
    csrc = tmp_path / "sparse_mixture_experts_fp32_b200" / "csrc"
    shutil.copytree(ROOT / "sparse_mixture_experts_fp32_b200" / "csrc", csrc,
                    ignore=shutil.ignore_patterns("_build", "*.o"))
    (tmp_path / "profiles").mkdir()
    return csrc


def test_traffic_lines_follow_the_kernel_source(tmp_path, monkeypatch):
    csrc = _fake_tree(tmp_path)
    monkeypatch.setattr(bench, "ROOT", tmp_path)
    sha = bench.source_sha("router_tc")
    other = bench.source_sha("ffn_tc_fused")
    assert sha != other  # keyed by the kernel's own source file
    (tmp_path / "profiles" / "k.md").write_text(
        f"    traffic[router_tc@base128_skew]: 1234 bytes source_sha={sha}\n"
        f"    traffic[ffn_tc_fused@base128_skew]: 99 bytes source_sha=000000000000\n")
    assert bench.traffic_from_profiles("router_tc", "base128_skew") == 1234.0
    assert bench.traffic_from_profiles("router_tc", "base8") is None          # other workload
    assert bench.traffic_from_profiles("ffn_tc_fused", "base128_skew") is None  # stale hash
    # editing the router's source invalidates only the router's line
    (csrc / "router_tc.cu").write_text((csrc / "router_tc.cu").read_text() + "\n// edit\n")
    assert bench.traffic_from_profiles("router_tc", "base128_skew") is None
    assert bench.source_sha("ffn_tc_fused") == other


def test_ffn_path_rule():
    """The bench reproduces the library's device-side choice of FFN path from the counts: with at
    least twelve waves of 256-wide GEMM2 tiles GEMM1 runs as its own launch and the fused kernel
    does GEMM2 only; otherwise the fused kernel does both and GEMM1's launch (if any) no work."""
    wl = synth.WORKLOADS["large128"]
    C = 1280
    balanced = np.full(wl.num_experts, wl.T // wl.num_experts, dtype=np.int64)
    assert bench.ffn_two_launches(wl, C, balanced)
    work = bench.kernel_work(wl, C, balanced)
    K = int(np.minimum(balanced, C).sum())
    assert work["ffn_tc_fused"] == ("tensor", 2.0 * K * wl.d_ff * wl.d_model, None)
    assert work["ffn_tc_gemm1_relu"][0] == "tensor"
    skewed = np.zeros(wl.num_experts, dtype=np.int64)
    skewed[:2] = C  # two experts at capacity: 10 row blocks x 4 column tiles = 40 tiles
    assert not bench.ffn_two_launches(wl, C, skewed)
    work = bench.kernel_work(wl, C, skewed)
    assert work["ffn_tc_fused"][0] == "tensor" and work["ffn_tc_gemm1_relu"][0] == "?"
    # with SWITCH_FLAG_FFN_TWO_LAUNCHES both GEMMs are real launches and there is no fused kernel
    assert bench.kernel_work(wl, C, skewed, flags=8)["ffn_tc_gemm1_relu"][0] == "tensor"
