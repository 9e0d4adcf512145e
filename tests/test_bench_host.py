"""Host logic of bench.py, on the CPU: the code digest that keys recorded ncu
traffic, the traffic lookup, the sizing of the oracle's sample, and the JSON
line of the reference arm."""
import json
import os
import shutil
import subprocess
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def test_strip_comments_keeps_code_and_literals():
    src = ('int a = 1;  // trailing\n'
           '/* block\n   over lines */ int b = 2;\n'
           '\n'
           'const char* s = "http://x // not a comment /* nor this */";\n'
           "char c = '/'; char d = '\\'';  /* after */\n"
           '   // a whole-line comment\n'
           'asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));\n')
    assert bench._strip_comments(src).split("\n") == [
        "int a = 1;",
        "int b = 2;",
        'const char* s = "http://x // not a comment /* nor this */";',
        "char c = '/'; char d = '\\'';",
        'asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));',
    ]


@pytest.fixture
def tree(tmp_path, monkeypatch):
    """A copy of the CUDA sources and profiles under a temporary root."""
    pkg = tmp_path / "int8_mixed_precision_outlier_b200"
    shutil.copytree(os.path.join(ROOT, "int8_mixed_precision_outlier_b200", "csrc"), pkg / "csrc",
                    ignore=shutil.ignore_patterns("*.so", "*.o"))
    (tmp_path / "profiles").mkdir()
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    return tmp_path


def test_digest_ignores_comments_but_not_code(tree):
    d0 = bench.source_digest()
    f = tree / "int8_mixed_precision_outlier_b200" / "csrc" / "gemv_kernel.cuh"
    text = f.read_text(encoding="utf-8")
    f.write_text("// a new comment line\n" + text.replace("\n", "  \n", 3) + "\n/* trailing */\n",
                 encoding="utf-8")
    assert bench.source_digest() == d0
    f.write_text(text.replace("constexpr int STAGES = 4;", "constexpr int STAGES = 3;"), encoding="utf-8")
    assert bench.source_digest() != d0


def test_recorded_traffic_needs_the_current_digest(tree):
    d = bench.source_digest()
    (tree / "profiles" / "traffic.txt").write_text(
        "# workload kernel digest bytes\n"
        f"7b_decode decode_call {d} 50921779\n"
        "7b_prefill gemm_pair_kernel 0123456789abcdef 26825984\n", encoding="utf-8")
    assert bench.recorded_traffic("7b_decode", "decode_call") == 50921779.0
    assert bench.recorded_traffic("7b_prefill", "gemm_pair_kernel") is None  # stale digest
    assert bench.recorded_traffic("13b_up", "gemm_pair_kernel") is None


def test_traffic_key_names_the_threshold_sweep(tree):
    d = bench.source_digest()
    (tree / "profiles" / "traffic.txt").write_text(
        f"70b_up gemm_pair_kernel {d} 605212672\n70b_up@4 gemm_pair_kernel {d} 1401019904\n"
        f"70b_up@inf gemm_pair_kernel {d} 584742656\n", encoding="utf-8")
    assert bench.traffic_key("70b_up", bench.THRESHOLD) == "70b_up"
    assert bench.recorded_traffic(bench.traffic_key("70b_up", 4.0), "gemm_pair_kernel") == 1401019904.0
    assert bench.recorded_traffic(bench.traffic_key("70b_up", float("inf")), "gemm_pair_kernel") == 584742656.0
    assert bench.recorded_traffic(bench.traffic_key("70b_up", 6.0), "gemm_pair_kernel") == 605212672.0


def test_shrink_sample_recounts_bytes_and_ops():
    T, N, K, n_out = 4, 1000, 256, 3
    X = np.zeros((T, K), np.float16)
    Wq = np.zeros((N, K), np.int8)
    sw = np.zeros(N, np.float32)
    W = np.zeros((N, K), np.float16)
    nbytes = N * K + 4 * N + 2 * N * n_out + 2 * T * K + 2 * T * N
    fn = object()
    calls, n = bench.shrink_sample([(fn, (X, Wq, sw, W, 6.0), nbytes, 2 * T * N * K)], 0.25)
    fn2, (X2, Wq2, sw2, W2, tau), b2, o2 = calls[0]
    assert fn2 is fn and n == 250 and Wq2.shape == (250, K) and W2.shape == (250, K) and sw2.shape == (250,)
    assert b2 == n * K + 4 * n + 2 * n * n_out + 2 * T * K + 2 * T * n
    assert o2 == 2 * T * n * K
    # prefill samples carry no byte count; a tiny fraction keeps one row
    calls, n = bench.shrink_sample([(fn, (X, Wq, sw, W, 6.0), 0, 2 * T * N * K)], 1e-9)
    assert n == 1 and calls[0][2] == 0 and calls[0][3] == 2 * T * K


def test_reference_arm_prints_the_contract_line():
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "7", "--warmup", "3",
                        "--ref-budget-s", "2"], cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-3000:]
    line = json.loads(r.stdout.strip().splitlines()[-1])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config"):
        assert key in line, key
    assert line["impl"] == "reference" and line["steps"] == 7 and line["warmup"] == 3
    assert line["unit"] == "GB/s" and line["value"] > 0 and line["config"]["workload"] == "7b_decode"
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == line["value"] and cb["cores"] >= 1 and cb["sample"]
    assert line["e2e"] == {"value": line["value"], "unit": "GB/s", "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0}


def test_reference_arm_under_torchrun_prints_once_with_all_cores():
    """Two ranks: rank 0 alone times the oracle, on every host core; rank 1
    exits 0 without work."""
    r = subprocess.run([sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
                        "--master-addr", "127.0.0.1", "--master-port", "29541", "bench.py", "--impl",
                        "reference", "--gpus", "2", "--steps", "3", "--warmup", "3", "--ref-budget-s", "2"],
                       cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-3000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    line = json.loads(lines[0])
    assert line["n_gpus"] == 2 and line["steps"] == 3
    assert line["cpu_baseline"]["cores"] == len(os.sched_getaffinity(0))
