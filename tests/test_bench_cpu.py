"""bench.py on the host: the oracle arm's JSON line and the CPU-sample sizing."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def test_reference_arm_prints_one_contract_line():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload", "tiny",
                          "--steps", "1", "--warmup", "0"], capture_output=True, text=True, timeout=300, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["value"] > 0 and d["higher_is_better"] is True
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0
    assert d["config"]["workload"].startswith("tiny:")


def test_reference_arm_viterbi_mode():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--viterbi",
                          "--workload", "tiny", "--steps", "1", "--warmup", "0"],
                         capture_output=True, text=True, timeout=300, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    d = json.loads(out.stdout.strip().splitlines()[-1])
    assert d["impl"] == "reference" and d["value"] > 0 and "Viterbi" in d["metric"]
    assert "Viterbi decode" in d["config"]["workload"] and d["dtype"] == "f32"


def test_qat_and_viterbi_modes_exclude_each_other():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--qat", "--viterbi"],
                         capture_output=True, text=True, timeout=120, cwd=ROOT)
    assert out.returncode != 0 and "not allowed" in out.stderr


def test_bad_temperature_is_rejected():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--workload", "mlp", "--temp", "0.5"],
                         capture_output=True, text=True, timeout=120, cwd=ROOT)
    assert out.returncode != 0 and "--temp" in out.stderr


def test_oracle_sample_is_bounded_by_cores_and_memory():
    import bench
    from bcjr_sum_product_b200 import inputs as I
    for name, wl in I.WORKLOADS.items():
        n = bench.oracle_sample_rows(wl, wl.n_seq)
        assert 1 <= n <= min(os.cpu_count() or 1, 128, wl.n_seq)
        assert n == 1 or n * 3 * wl.n_steps * wl.S * 8 <= 32 << 30
