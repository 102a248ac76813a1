"""The benchmark's work accounting against the figures the scope table prints.

Algorithmic FLOPs are 6*S*H*I (plus 2*S*r*(H+2I) with LoRA) and algorithmic
bytes count packed nibbles + fp32 absmax of the touched experts in both stacks
(1.6875*H*I bytes per expert), x, out and the routing.  The expected values
below are the rounded figures of the per-workload table (bytes in MB, GFLOP),
not recomputed from bench.py's own formula.  CPU only.
"""
import os
import sys

import pytest

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
import bench  # noqa: E402
from quantized_moe_expert_nf4_b200 import workloads  # noqa: E402

# (config, M, touched experts, algorithmic MB, GFLOP) as tabulated for each workload
TABLE = [
    ("tiny", 64, 8, 0.51, 0.025),
    ("olmoe", 1, 8, 28.3, 0.10),
    ("olmoe", 2048, 64, 243.0, 206.2),
    ("qwen3", 4096, 128, 374.0, 309.2),
    ("qwen3_lora", 4096, 128, 381.0, 311.1),
    ("gptoss", 1, 4, 56.0, 0.20),
]


@pytest.mark.parametrize("name,M,touched,mb,gflop", TABLE)
def test_step_work_matches_the_table(name, M, touched, mb, gflop):
    cfg = workloads.CONFIGS[name]
    flops, nbytes = bench.step_work(cfg, M, touched)
    assert flops / 1e9 == pytest.approx(gflop, rel=0.03)
    # the table leaves out the router logits (M*E*4 bytes): at most 0.6% here
    assert nbytes / 1e6 == pytest.approx(mb, rel=0.006)


def test_decode_roofline_arithmetic():
    """achieved = algorithmic bytes of the launch / its duration; frac = achieved / peak."""
    cfg = workloads.CONFIGS["olmoe"]
    peaks = {"hbm_gbs": 6541.5, "bf16_tflops": 1617.9, "bf16_tflops_sustained": 1374.1, "source": "measured"}
    kt = {"decode.gate_up": (0.010, 100), "decode.down": (0.004, 100)}
    name, r = bench.dominant_roofline(cfg, 1, kt, 8.0, peaks, long_region=False)
    assert name == "decode.gate_up" and r["bound"] == "hbm" and r["unit"] == "GB/s"
    gate_up_bytes = 8 * 2 * 2048 * 1024 * (0.5 + 4 / 64) + 1 * 2048 * 2   # 8 experts' gate_up + x
    assert r["algorithmic_bytes_per_launch"] == pytest.approx(gate_up_bytes)
    assert r["achieved"] == pytest.approx(gate_up_bytes / 10e-6 / 1e9)
    assert r["frac"] == pytest.approx(r["achieved"] / 6541.5)


def test_grouped_roofline_uses_the_sustained_peak_in_a_long_region():
    cfg = workloads.CONFIGS["qwen3"]
    peaks = {"hbm_gbs": 6541.5, "bf16_tflops": 1617.9, "bf16_tflops_sustained": 1374.1, "source": "measured"}
    kt = {"gemm.tc.swiglu": (0.40, 10), "gemm.tc": (0.18, 10), "route.tile": (0.01, 10)}
    name, r = bench.dominant_roofline(cfg, 4096, kt, 128.0, peaks, long_region=True)
    assert name == "gemm.tc.swiglu" and r["bound"] == "tensor"
    flops = 2.0 * 4096 * 8 * 2 * 768 * 2048
    assert r["achieved"] == pytest.approx(flops / 0.40e-3 / 1e12)
    assert r["peak"] == 1374.1 and "sustained" in r["peak_source"]


def test_reference_arm_prints_one_contract_line():
    """`bench.py --impl reference` (the oracle on this host's cores) prints one
    JSON line with the keys the benchmark contract names, its e2e and
    cpu_baseline objects describing the same run."""
    import json
    import subprocess

    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    res = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--impl", "reference", "--workload",
                          "tiny_m64", "--steps", "2", "--warmup", "3"], capture_output=True, text=True, timeout=300,
                         cwd=root)
    assert res.returncode == 0, res.stderr[-2000:]
    lines = [l for l in res.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["steps"] == 2 and d["warmup"] == 3 and d["value"] > 0
    assert d["config"]["workload"] == "tiny_m64"
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
