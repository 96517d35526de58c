"""bench.py on the CPU: the reference arm (the oracle on a bounded sample)
prints one JSON line with the contract's keys, and the byte counts that the
roofline uses agree with each other."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_prints_the_contract_line():
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "1", "--warmup", "3"],
                       cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    line = json.loads(r.stdout.strip().splitlines()[-1])
    for k in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
              "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert k in line, k
    assert line["impl"] == "reference" and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["value"] == line["value"]
    assert line["config"]["workload"] == "gru_bf16_B1_L65536_D2048"


def test_pass_bytes_sum_to_solve_bytes():
    sys.path.insert(0, ROOT)
    import bench
    from nonlinear_rnn_newton_b200 import workloads as W
    for w in (W.GRU, W.LSTM, W.GRU_SMALL):
        for iters in (1, 2, 4, 7):
            assert sum(bench.pass_bytes(w, k) for k in range(iters)) == bench.solve_bytes(w, iters)
    assert bench.pass_bytes(W.GRU, 0) == W.GRU.N * 10 and bench.pass_bytes(W.GRU, 1) == W.GRU.N * 14
    assert bench.pass_bytes(W.LSTM, 0) == W.LSTM.N * 16 and bench.pass_bytes(W.LSTM, 3) == W.LSTM.N * 24
