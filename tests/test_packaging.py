"""Host-side contracts that need no GPU: the product path refuses to run
without its CUDA library (no silent CPU fallback), and the benchmark's FLOP
accounting follows the metric's definition for every workload."""
import os
import shutil
import subprocess
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_package_without_cuda_library_fails_loudly(tmp_path):
    pkg = tmp_path / "exact_attention_140_b200"
    shutil.copytree(os.path.join(ROOT, "exact_attention_140_b200"), pkg,
                    ignore=shutil.ignore_patterns("*.so", "__pycache__"))
    r = subprocess.run([sys.executable, "-c", "import exact_attention_140_b200"], cwd=tmp_path,
                       capture_output=True, text=True, timeout=120)
    assert r.returncode != 0
    assert "ImportError" in r.stderr and "libattn.so" in r.stderr


def test_package_never_imports_the_oracle():
    """The product package and its build script name no oracle module."""
    for dirpath, _, files in os.walk(os.path.join(ROOT, "exact_attention_140_b200")):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                text = open(os.path.join(dirpath, f), encoding="utf-8").read()
                assert "import oracle" not in text and "from oracle" not in text, f


def bench_module():
    import importlib.util
    spec = importlib.util.spec_from_file_location("bench", os.path.join(ROOT, "bench.py"))
    b = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(b)
    return b


def test_flop_count_is_the_metric_definition():
    b = bench_module()
    w = b.workloads()
    # 4 * B * Hq * Nq * Nk * d, halved for causal
    assert b.flops(w["gpt2"]) == 4.0 * 8 * 12 * 1024 * 1024 * 64 / 2
    assert b.flops(w["sweep8192"]) == 4.0 * 2 * 16 * 8192 * 8192 * 128
    assert b.flops(w["decode"]) == 4.0 * 4 * 32 * 16 * 32768 * 128
    for name, cfg in w.items():
        assert b.flops(cfg) > 0, name


def test_sampled_row_flops_follow_the_causal_rule():
    """The CPU baseline's per-row work: visible keys of row i are
    min(Nk, i + Nk - Nq + 1) under the bottom-right causal rule."""
    b = bench_module()
    cfg = dict(B=1, Hq=1, Hkv=1, N=300, Nq=100, d=8, causal=True, dtype="bf16")
    rows = np.arange(100)
    expect = float(sum(4 * 8 * min(300, i + 200 + 1) for i in range(100)))
    assert b._row_flops(cfg, rows) == expect
    cfg["causal"] = False
    assert b._row_flops(cfg, rows) == 4.0 * 8 * 300 * 100
