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
    # the same config keys as the GPU arm's line, so the two lines name one workload
    sys.path.insert(0, ROOT)
    import bench
    from rank_linear_lora_b200 import inputs
    spec = inputs.workload(0).layers[0]
    assert d["config"] == bench.config_dict(spec, d["config"]["workload"], 1)
    assert d["cpu_baseline"]["cpu_model"]


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


def test_gpus_2_spawns_two_ranks_and_prints_one_line():
    """`bench.py --gpus 2` with no launcher around it starts two ranks itself; over a gloo
    data plane (--dry-run: no GPU, the oracle on the host) they all-reduce the packed
    [dA | dB] of their token shards, and rank 0 alone prints one JSON line whose reduced
    gradients equal the whole batch's, with n_gpus 2 from the communicator."""
    import json
    import subprocess
    import sys
    env = {k: v for k, v in os.environ.items() if k not in ("RANK", "WORLD_SIZE", "LOCAL_RANK", "MASTER_ADDR",
                                                             "MASTER_PORT")}
    p = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--gpus", "2", "--dry-run", "--backend",
                        "gloo", "--config", "0"], capture_output=True, text=True, timeout=300, env=env)
    assert p.returncode == 0, p.stderr[-2000:]
    lines = [ln for ln in p.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, p.stdout
    out = json.loads(lines[0])
    assert out["n_gpus"] == 2 and out["world_size"] == 2 and out["dry_run"] is True
    assert out["reduced_grads_match_whole_batch"] is True
    assert out["config"]["parallelism"] == "dp2"


def test_traffic_figures_follow_the_kernel_sources(tmp_path, monkeypatch):
    """A stored ncu traffic figure is reported only while the layer's kernel sources are
    the ones it was measured on: a comment or blank-space edit keeps it, a code edit
    voids it (the line then carries null)."""
    import shutil
    sys.path.insert(0, ROOT)
    import bench
    d = json.load(open(os.path.join(ROOT, "profiles", "traffic.json")))
    wl = next(iter(d["workloads"]))
    csrc = tmp_path / "rank_linear_lora_b200" / "csrc"
    csrc.mkdir(parents=True)
    for f in bench.LAYER_SOURCES:
        shutil.copy(os.path.join(ROOT, "rank_linear_lora_b200", "csrc", f), csrc / f)
    (tmp_path / "profiles").mkdir()
    d["kernel_source_hash"] = "0" * 16
    json.dump(d, open(tmp_path / "profiles" / "traffic.json", "w"))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    h0 = bench.kernel_source_hash()
    assert len(h0) == 16 and int(h0, 16) >= 0
    assert bench.stored_traffic("dx_main", wl) is None  # figure of other sources
    d["kernel_source_hash"] = h0
    json.dump(d, open(tmp_path / "profiles" / "traffic.json", "w"))
    want = d["workloads"][wl]["kernels"]["dx_main"]["dram_bytes_per_launch"]
    assert bench.stored_traffic("dx_main", wl) == want
    ptx = csrc / "ptx.cuh"
    text = ptx.read_text()
    ptx.write_text("// an added comment\n\n" + text.replace("\n", "\n  ", 3))
    assert bench.kernel_source_hash() == h0 and bench.stored_traffic("dx_main", wl) == want
    ptx.write_text(text + "\nstatic int an_added_symbol;\n")
    assert bench.kernel_source_hash() != h0 and bench.stored_traffic("dx_main", wl) is None
