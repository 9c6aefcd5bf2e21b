"""bench.py's reference arm (the fp64 oracle on the host cores) keeps the one-JSON-line
contract; it runs without a GPU."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_json_line():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--config", "0",
                          "--steps", "2", "--warmup", "1"], capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.strip()]
    assert len(lines) == 1, out.stdout
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "impl", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["steps"] == 2 and d["warmup"] == 1 and d["n_gpus"] == 1
    assert d["higher_is_better"] is True and d["value"] > 0 and d["unit"] == "TFLOP/s"
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["cpu_baseline"]["cores"] >= 1 and d["cpu_baseline"]["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
    assert d["config"]["workload"].startswith("tiny")


def test_stacked_layer_counts_the_work_of_its_projections():
    """The gate+up layer stacked on one x is measured by the work of the two
    projections: FLOPs are twice gate's, and the bytes are gate's twice less one read
    of the shared x (forward and backward) and with one dX written instead of two; the
    zero blocks of the stacked B and dB count nothing."""
    sys.path.insert(0, ROOT)
    import bench
    from rank_linear_lora_b200 import inputs

    gate, stacked = inputs.workload(2).layers[0], inputs.workload(2).layers[3]
    assert stacked.flops == 2 * gate.flops
    M, di = gate.M, gate.d_in
    x_bytes = M * di * 2
    # forward reads x once; backward reads x once and writes one dX
    assert bench.algorithmic_bytes(stacked) == 2 * bench.algorithmic_bytes(gate) - 3 * x_bytes
