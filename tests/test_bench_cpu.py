"""bench.py's host side, on CPU: the algorithmic byte counts against the per-config figures
of the measurement table (rms_norm f32 [64, 512]; add_rms_norm bf16 [8192, 4096]; layer_norm
bf16 [16384, 8192]; norm_rope bf16 [8, 32, 2048, 128]), and the reference arm -- the CPU
oracle timed on host cores -- printing one JSON line with every key of the contract.
"""
import json
import os
import subprocess
import sys

import pytest

import bench

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.parametrize("op,rows,D,s,want", [
    ("rms_norm", 64, 512, 4, 264_192),
    ("add_rms_norm", 8192, 4096, 2, 268_443_648),
    ("layer_norm", 16384, 8192, 2, 536_903_680),
    ("norm_rope", 8 * 32 * 2048, 128, 2, 268_435_712),
])
def test_algorithmic_bytes_match_the_config_table(op, rows, D, s, want):
    assert bench.algorithmic_bytes(op, rows, D, s) == want


def test_algorithmic_bytes_of_the_next_rows():
    N, D, s = 8192 * 4096, 4096, 2
    assert bench.algorithmic_bytes("rms_norm_vjp", 8192, D, s) == 3 * N * s + 2 * D * s
    assert bench.algorithmic_bytes("layer_norm_vjp", 8192, D, s) == 3 * N * s + 3 * D * s
    # eight partial outputs read, r read, y and h written, w read once
    assert bench.algorithmic_bytes("allreduce_add_rms_norm", 8192, D, s, nparts=8) == \
        11 * N * s + D * s
    with pytest.raises(ValueError):
        bench.algorithmic_bytes("softmax", 1, 1, 2)


def test_reference_arm_prints_one_contract_line():
    res = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--steps", "3", "--warmup", "3"], capture_output=True, text=True,
                         timeout=600, cwd=ROOT, env={**os.environ, "CUDA_VISIBLE_DEVICES": ""})
    assert res.returncode == 0, res.stderr
    lines = [l for l in res.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, res.stdout
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["metric"] == bench.METRIC
    assert d["unit"] == "GB/s" and d["higher_is_better"] is True and d["value"] > 0
    assert d["steps"] == 3 and d["warmup"] == 3 and d["n_gpus"] == 1
    assert "workload" in d["config"]
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"]
    assert cb["sample"] and cb["unit"] == d["unit"]
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}


def test_nvtx_ranges_nest_and_never_raise():
    with bench.nvtx_range("outer"):
        with bench.nvtx_range("inner") as r:
            assert r.open in (True, False)
    try:
        with bench.nvtx_range("failing body"):
            raise KeyError("body")
    except KeyError:
        pass   # the body's exception propagates; the range is closed on the way out


def test_rotation_keeps_three_l2_between_uses_of_a_buffer_set():
    """Between two uses of one buffer set the other sets hold at least 3x L2, so no line a
    step reads can have survived in L2 from that set's last use; sets too small for that
    within 9 copies (under 3/8 of L2) are flushed instead."""
    l2 = 126 * 2 ** 20
    for set_bytes, want in [(268435456, 3),      # add_rms_norm / norm_rope bf16 sets
                            (536870912, 2),      # layer_norm bf16 [16384, 8192]
                            (201326592, 3),      # rms_norm_vjp
                            (134217728, 4),      # rms_norm bf16 [8192, 4096]
                            (l2, 4), (l2 - 1, 5), (10 * l2, 2), (l2 // 2 + 2 ** 20, 7),
                            (67108864 * 2 // 2, 7),  # add_rms_norm bf16 [4096, 2048]
                            (3 * l2 // 8, 9), (3 * l2 // 8 - 1, 1), (l2 // 4, 1)]:
        n = bench.rotation_sets(set_bytes, l2)
        assert n == want, (set_bytes, n, want)
        if n > 1:
            assert (n - 1) * set_bytes >= 3 * l2 or n == 9
    assert bench.rotation_sets(l2 + 1, l2) == 4     # just over L2: 3 more copies
    assert bench.rotation_sets(l2 // 4 + l2, l2) == 4

