#!/usr/bin/env python
"""Benchmark of the fused LoRA linear layer (forward + backward) on B200.

One step = lora_linear_fwd + lora_linear_bwd of one layer over one batch of
synthetic tokens (every row of the hot path: s.xa, the forward main GEMM, s.g,
the dX GEMM, and dB with dA).  Default workload: the attention-projection layer,
M = 4096 tokens (2 x 2048), d_in = d_out = 4096, r = 8, alpha = 32.

Timing: W untimed warm-up steps; then, behind a GPU sleep that lets the host
enqueue all K steps ahead, K back-to-back steps bracketed by CUDA events on the
launch stream (barrier + synchronize on both sides; max over ranks).  Steps rotate
over three independent input sets (3 x 160 MiB > the 126 MB L2), so no step finds
its operands left in L2 by the previous one.

Multi-GPU: data parallel over tokens, weak scaling (each rank its own M tokens);
after the backward the packed [dA | dB] fp32 gradient is summed over ranks with one
NCCL all-reduce inside the timed region.  `--gpus N` with N > 1 and no launcher
around it starts N ranks itself (torch.distributed.run on this node, one per GPU);
under an outside launcher (RANK / WORLD_SIZE set) it runs as one of its ranks.

--impl reference times the fp64 CPU oracle on the host cores instead (a bounded
token sample per step).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "fused LoRA fwd+bwd TFLOP/s & tokens/s per layer; % of BF16 tensor roofline"
UNIT = "TFLOP/s"
N_SETS = 3


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=200)
    p.add_argument("--warmup", type=int, default=10)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--config", type=int, default=1, help="workload index (1: attention projection)")
    p.add_argument("--rank-r", type=int, default=None, help="rank for the rank-sweep workload")
    p.add_argument("--layer", type=int, default=0, help="layer of a multi-layer workload")
    p.add_argument("--fp8", action="store_true",
                   help="store the workload's frozen weight as FP8 (E4M3 codes, one bf16 scale per row)")
    p.add_argument("--nf4", action="store_true",
                   help="store the workload's frozen weight as 4-bit NF4 codes (codebook weight, d_in % 64 == 0)")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--backend", choices=["nccl", "gloo"], default="nccl",
                   help="process-group backend of a multi-rank run (gloo only with --dry-run)")
    p.add_argument("--dry-run", action="store_true",
                   help="no GPU: each rank computes its token shard's dA, dB with the oracle on the host, sums "
                        "them over ranks with one all-reduce of the packed buffer and prints the JSON line; "
                        "checks the multi-rank launch and reduction plumbing on a CPU-only machine")
    p.add_argument("--shape", type=str, default=None,
                   help="M,d_in,d_out: resize the layer (same r, alpha, weight format), e.g. a case small "
                        "enough for a full profiler capture; the line then names the resized workload")
    return p.parse_args()


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        d = json.load(open(path))
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained", d["bf16_tflops"]), "src": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "src": "fallback"}


def algorithmic_bytes(spec) -> float:
    """One read of every operand and one write of every output per fwd + bwd call.  For
    projections stacked on one x only the diagonal blocks of B and dB count (rb = r/proj
    columns per row); A, xa and dA hold every projection's ranks."""
    M, di, do, r = spec.M, spec.d_in, spec.d_out, spec.r
    rb = r // spec.proj
    w = (do * di // 2 + do * (di // 64) * 2 if (spec.q4 or spec.nf4) else do * di + do * 2 if spec.fp8
         else do * di * 2)
    fwd = M * di * 2 + w + r * di * 2 + do * rb * 2 + M * do * 2 + M * r * 2
    bwd = M * do * 2 + M * di * 2 + w + r * di * 2 + do * rb * 2 + M * r * 2 + M * di * 2 + r * di * 4 + do * rb * 4
    return float(fwd + bwd)


# The sources the layer's kernels and their launches are built from: lora_linear.cu and
# every header it includes (the merge and the workspace-free forward are other files).
LAYER_SOURCES = ("lora_linear.cu", "side.cuh", "tc_gemm.cuh", "tc_gemm2.cuh", "ptx.cuh", "tmap.h")


def kernel_source_hash() -> str:
    """Hash of the code of the layer's CUDA sources, comments and blank space removed (a
    stored ncu traffic figure is only reported while the kernels and launches it was
    measured on are unchanged; editing a comment does not change them)."""
    import re
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "rank_linear_lora_b200", "csrc")
    for f in sorted(LAYER_SOURCES):
        with open(os.path.join(csrc, f), encoding="utf-8") as fh:
            text = fh.read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        text = re.sub(r"//[^\n]*", "", text)
        h.update(f.encode())
        h.update(" ".join(text.split()).encode())
    return h.hexdigest()[:16]


def stored_traffic(kind: str, workload: str):
    """DRAM bytes per launch from the committed ncu summary, if the kernels are unchanged."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    d = json.load(open(path))
    if d.get("kernel_source_hash") != kernel_source_hash():
        return None
    e = d.get("workloads", {}).get(workload, {}).get("kernels", {}).get(kind)
    return e.get("dram_bytes_per_launch") if e else None


class ClockSampler:
    """NVML clocks and throttle reasons sampled in a thread while the timed region runs."""

    def __init__(self, dev, period_s: float = 0.0005):
        self.period, self.samples, self._stop = period_s, [], threading.Event()
        self.ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = self._handle(pynvml, dev)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:  # pragma: no cover - no NVML
            self.max_mhz = None

    @staticmethod
    def _handle(nv, dev):
        """The NVML device of torch device ``dev``, matched by PCI address (NVML numbers
        every GPU of the machine and ignores CUDA_VISIBLE_DEVICES)."""
        import torch
        p = torch.cuda.get_device_properties(dev)
        for i in range(nv.nvmlDeviceGetCount()):
            h = nv.nvmlDeviceGetHandleByIndex(i)
            pci = nv.nvmlDeviceGetPciInfo(h)
            if (pci.domain, pci.bus, pci.device) == (p.pci_domain_id, p.pci_bus_id, p.pci_device_id):
                return h
        raise RuntimeError("no NVML device at the PCI address of %s" % dev)

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                mhz = nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)
                reasons = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                self.samples.append((mhz, reasons))
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            # The sampling thread needs the interpreter lock every half millisecond; the
            # default switch interval (5 ms) would leave it one sample per timed region.
            self._switch = sys.getswitchinterval()
            sys.setswitchinterval(1e-4)
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self._stop.set()
            self.t.join()
            sys.setswitchinterval(self._switch)

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unavailable"], "samples": 0}
        nv = self.nv
        names = {
            "gpu_idle": getattr(nv, "nvmlClocksEventReasonGpuIdle", 0x1),
            "sw_power_cap": getattr(nv, "nvmlClocksEventReasonSwPowerCap", 0x4),
            "hw_slowdown": getattr(nv, "nvmlClocksEventReasonHwSlowdown", 0x8),
            "sw_thermal_slowdown": getattr(nv, "nvmlClocksEventReasonSwThermalSlowdown", 0x20),
            "hw_thermal_slowdown": getattr(nv, "nvmlClocksEventReasonHwThermalSlowdown", 0x40),
            "hw_power_brake_slowdown": getattr(nv, "nvmlClocksEventReasonHwPowerBrakeSlowdown", 0x80),
        }
        mhz = sorted(s[0] for s in self.samples)
        seen = sorted({n for _, r in self.samples for n, bit in names.items() if r & bit and n != "gpu_idle"})
        return {"sm_mhz": mhz[len(mhz) // 2], "sm_max_mhz": self.max_mhz, "reasons": seen,
                "samples": len(self.samples)}


def device_spans(step, st, max_ctas: int = 512) -> dict:
    """{kernel kind: us from its first CTA's set-up stamp to its last CTA's exit} over one
    step, from the library's per-CTA device trace (a kind launched more than once in the
    step keeps its last launch).  The set-up stamp follows the kernel's wait for its
    stream predecessor (the dA + dB kernel, which waits only before it exits, stamps it
    on entry), so CTAs that a programmatic launch let in early do not count their wait."""
    import torch
    from rank_linear_lora_b200 import lora_linear as L
    kinds = L.KERNEL_KINDS
    buf = torch.zeros(len(kinds) * max_ctas * L.TRACE_WORDS, dtype=torch.int64, device="cuda")
    torch.cuda.synchronize()
    # timing hooks on: the same launch sequence as the per-kernel event pass
    L.lora_linear_timing_read()
    L.lora_linear_timing_enable(True)
    L.lora_linear_trace_enable(buf)
    try:
        torch.cuda._sleep(int(2e6))  # the host enqueues the whole step ahead of the GPU
        step(st)
        torch.cuda.synchronize()
    finally:
        L.lora_linear_trace_enable(None)
        L.lora_linear_timing_enable(False)
        L.lora_linear_timing_read()
    tr = buf.cpu().numpy().reshape(len(kinds), max_ctas, L.TRACE_WORDS)
    entry, setup, exit_ = (L.TRACE_FIELDS.index(f) for f in ("entry", "setup", "exit"))
    out = {}
    for i, k in enumerate(kinds):
        rows = tr[i][tr[i][:, entry] > 0]
        if len(rows):
            out[k] = float(rows[:, exit_].max() - rows[:, setup].min()) / 1e3
    return out


def config_dict(spec, workload_name: str, world: int) -> dict:
    """The workload as both arms name it (identical keys and values)."""
    return {"workload": workload_name, "M": spec.M, "d_in": spec.d_in, "d_out": spec.d_out, "r": spec.r,
            "alpha": spec.alpha, "q4": spec.q4, "fp8": spec.fp8, "nf4": spec.nf4, "projections": spec.proj,
            "tokens_per_step": spec.M * world,
            "l2": f"{N_SETS} rotating input sets (> L2); no flush inside the timed region",
            "parallelism": f"dp{world}"}


def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform
    return platform.processor() or "unknown"


def free_port() -> int:
    import socket
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as so:
        so.bind(("127.0.0.1", 0))
        return so.getsockname()[1]


def launch_ranks(args) -> int:
    """Run this script as `args.gpus` ranks on this node (torch.distributed.run), one per
    GPU, rendezvous on 127.0.0.1; rank 0 prints the JSON line.  The launcher is bounded
    by a timeout well above the process group's own, after which its process group is
    killed."""
    import signal
    import subprocess
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={args.gpus}",
           "--master-addr=127.0.0.1", f"--master-port={free_port()}", os.path.abspath(__file__)] + sys.argv[1:]
    proc = subprocess.Popen(cmd, start_new_session=True)
    try:
        return proc.wait(timeout=1800)
    except subprocess.TimeoutExpired:
        os.killpg(proc.pid, signal.SIGKILL)
        proc.wait()
        print(f"bench.py: the {args.gpus} ranks did not finish within 1800 s", file=sys.stderr)
        return 1


def run_dry(args, spec, workload_name, rank, world):
    """CPU-only multi-rank run: the plumbing of the data-parallel step without a GPU."""
    import numpy as np
    import torch
    import torch.distributed as dist
    from datetime import timedelta

    import oracle
    from rank_linear_lora_b200 import inputs
    from rank_linear_lora_b200.dp import PackedGrads, token_shard

    if world > 1:
        dist.init_process_group(args.backend, timeout=timedelta(seconds=60))
        assert dist.get_world_size() == world
    tokens = min(spec.M, 64 * max(1, world))
    small = spec.with_(M=tokens, d_in=min(spec.d_in, 256), d_out=min(spec.d_out, 256))
    inp = inputs.make_inputs(small)
    start, count = token_shard(small.M, world, rank)
    grads = PackedGrads(small.r, small.d_in, small.d_out, device="cpu")
    t0 = time.perf_counter()
    if count > 0:
        xa_ = oracle.xa(inp.x[start:start + count], inp.A)
        g_ = oracle.g(inp.dY[start:start + count], inp.B)
        grads.dA.copy_(torch.from_numpy(oracle.da(inp.x[start:start + count], g_, small.s)))
        grads.dB.copy_(torch.from_numpy(oracle.db(inp.dY[start:start + count], xa_, small.s)))
    else:
        grads.zero_()
    if world > 1:
        grads.all_reduce()
    dt = time.perf_counter() - t0
    ok = None
    if rank == 0:
        xa_ = oracle.xa(inp.x, inp.A)
        g_ = oracle.g(inp.dY, inp.B)
        full_dA, full_dB = oracle.da(inp.x, g_, small.s), oracle.db(inp.dY, xa_, small.s)
        ok = bool(np.allclose(grads.dA.double().numpy(), full_dA, rtol=0, atol=1e-5 * np.abs(full_dA).max())
                  and np.allclose(grads.dB.double().numpy(), full_dB, rtol=0, atol=1e-5 * np.abs(full_dB).max()))
        out = {"metric": METRIC, "value": None, "unit": UNIT, "n_gpus": world, "world_size": world,
               "steps": 1, "warmup": 0, "ms_per_step": dt * 1e3, "higher_is_better": True, "scaling": "weak",
               "vs_baseline": None, "dtype": "f64", "data": "synthetic", "dry_run": True,
               "backend": args.backend if world > 1 else None,
               "config": config_dict(small, workload_name + f" (dry run: M{small.M} {small.d_in}->{small.d_out})",
                                     world),
               "reduced_grads_match_whole_batch": ok}
        print(json.dumps(out), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0 if ok in (None, True) else 1


# ---------------------------------------------------------------------- reference arm
def run_reference(args, spec, workload_name, rank, world):
    import numpy as np

    import oracle
    from rank_linear_lora_b200 import inputs

    if rank != 0:
        return None
    inp = inputs.make_inputs(spec)
    per_token = spec.flops / spec.M
    # calibrate, then size the per-step token sample so the whole run takes ~2 minutes
    t0 = time.perf_counter()
    _oracle_step(oracle, inp, spec, 0, 8)
    rate = 8 * per_token / max(1e-6, time.perf_counter() - t0)
    budget = min(20.0, 120.0 / max(1, args.steps + args.warmup))
    tokens = int(max(8, min(spec.M, budget * rate / per_token)))
    for i in range(args.warmup):
        _oracle_step(oracle, inp, spec, i * tokens, tokens)
    t0 = time.perf_counter()
    for i in range(args.steps):
        _oracle_step(oracle, inp, spec, (args.warmup + i) * tokens, tokens)
    dt = time.perf_counter() - t0
    flops = args.steps * tokens * per_token
    value = flops / dt / 1e12
    sample = f"{tokens} of the {spec.M} tokens per step (full d_in, d_out, r), fp64"
    return {
        "metric": METRIC, "value": value, "unit": UNIT, "impl": "reference", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": config_dict(spec, workload_name, world),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": oracle.threads(), "kind": "oracle",
                         "sample": sample, "cpu_model": cpu_model(),
                         "where": "host cores of rank 0 (OpenMP), the other ranks idle"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "tokens_per_s": args.steps * tokens / dt,
    }


def _oracle_step(oracle, inp, spec, start, tokens):
    M = spec.M
    rows = [(start + i) % M for i in range(tokens)]
    x, dY = inp.x[rows], inp.dY[rows]
    wkw = (dict(Wq=inp.Wq, Wscale=inp.Wscale) if spec.q4 else dict(W8=inp.W8, W8scale=inp.W8scale) if spec.fp8
           else dict(Wq=inp.Wq, Wscale=inp.Wscale, codebook=inp.codebook) if spec.nf4 else dict(W=inp.W))
    h, xa = oracle.forward(x, inp.A, inp.B, spec.s, **wkw)
    oracle.backward(dY, x, inp.A, inp.B, spec.s, xa_=xa, **wkw)


def cpu_baseline(spec, seconds=12.0):
    """The oracle as it stands on this host's cores over a bounded token sample."""
    import oracle
    from rank_linear_lora_b200 import inputs

    inp = inputs.make_inputs(spec)
    per_token = spec.flops / spec.M
    t0 = time.perf_counter()
    _oracle_step(oracle, inp, spec, 0, 8)
    rate = 8 * per_token / max(1e-6, time.perf_counter() - t0)
    tokens = int(max(8, min(spec.M, seconds * rate / per_token)))
    t0 = time.perf_counter()
    _oracle_step(oracle, inp, spec, 0, tokens)
    dt = time.perf_counter() - t0
    return {"value": tokens * per_token / dt / 1e12, "unit": UNIT, "cores": oracle.threads(), "kind": "oracle",
            "cpu_model": cpu_model(),
            "sample": f"fwd+bwd of {tokens} of the {spec.M} tokens (full d_in={spec.d_in}, d_out={spec.d_out}, "
                      f"r={spec.r}) in fp64, {dt:.1f} s",
            "single_thread_tiny": single_thread_tiny()}


def single_thread_tiny():
    """The oracle on one host thread, whole tiny workload (M=64, 256x256, r=8)."""
    import oracle
    from rank_linear_lora_b200 import inputs

    spec = inputs.workload(0).layers[0]
    inp = inputs.make_inputs(spec)
    n0 = oracle.threads()
    oracle.set_threads(1)
    try:
        _oracle_step(oracle, inp, spec, 0, spec.M)
        reps, t0 = 0, time.perf_counter()
        while reps < 3 or time.perf_counter() - t0 < 0.5:
            _oracle_step(oracle, inp, spec, 0, spec.M)
            reps += 1
        dt = (time.perf_counter() - t0) / reps
    finally:
        oracle.set_threads(n0)
    return {"workload": "tiny M64 256x256 r8, whole", "threads": 1, "s_per_step": dt,
            "gflops": spec.flops / dt / 1e9}


# ---------------------------------------------------------------------- our arm
def main():
    args = parse()
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        return launch_ranks(args)
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus and not (args.gpus == 1 and world > 1):
        print(f"bench.py: --gpus {args.gpus} but the launcher started {world} ranks", file=sys.stderr)
        return 2

    from rank_linear_lora_b200 import inputs

    wl = inputs.workload(args.config, r=args.rank_r)
    spec = wl.layers[args.layer]
    workload_name = f"{wl.name} / {spec.name}"
    if args.fp8:
        spec = spec.with_(q4=False, fp8=True)
        workload_name += " with the FP8 weight"
    if args.nf4:
        spec = spec.with_(q4=False, nf4=True)
        workload_name += " with the NF4 weight"
    if args.shape:
        M_, di_, do_ = (int(v) for v in args.shape.split(","))
        spec = spec.with_(M=M_, d_in=di_, d_out=do_)
        workload_name += f" resized to M{M_} {di_}->{do_}"

    if args.dry_run:
        return run_dry(args, spec, workload_name, rank, world)
    if args.impl == "reference":
        out = run_reference(args, spec, workload_name, rank, world)
        if out is not None:
            print(json.dumps(out), flush=True)
        return 0

    import numpy as np
    import torch
    import torch.distributed as dist

    from rank_linear_lora_b200 import lora_linear as L
    from rank_linear_lora_b200.dp import PackedGrads

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)
        assert dist.get_world_size() == world

    peaks = load_peaks()
    M, di, do, r, alpha = spec.M, spec.d_in, spec.d_out, spec.r, spec.alpha

    def d16(bits):
        return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(dev)

    # Input sets: set k uses the generator's streams of seed + 1000 * k, shifted by rank.
    sets = []
    host_inputs = None
    for k in range(N_SETS):
        sp = spec.with_(seed=spec.seed + 1000 * k + 7919 * rank)
        inp = inputs.make_inputs(sp)
        if k == 0:
            host_inputs = inp
        s = {"x": d16(inp.x), "A": d16(inp.A), "B": d16(inp.B), "dY": d16(inp.dY)}
        if spec.q4 or spec.nf4:
            s["Wq"] = torch.from_numpy(inp.Wq).to(dev)
            s["Wscale"] = d16(inp.Wscale)
            s["cb"] = inp.codebook
        elif spec.fp8:
            s["W8"] = torch.from_numpy(inp.W8).to(dev)
            s["W8scale"] = d16(inp.W8scale)
        else:
            s["W"] = d16(inp.W)
        s["h"] = torch.empty(M, do, dtype=torch.bfloat16, device=dev)
        s["xa"] = torch.empty(M, r, dtype=torch.bfloat16, device=dev)
        s["dX"] = torch.empty(M, di, dtype=torch.bfloat16, device=dev)
        s["grad"] = PackedGrads(r, di, do, device=dev)  # fp32 [dA | dB], the one all-reduced buffer
        s["dA"], s["dB"] = s["grad"].dA, s["grad"].dB
        fop, bop = ((L.OP_FWD_Q4, L.OP_BWD_Q4) if spec.q4 else (L.OP_FWD_FP8, L.OP_BWD_FP8) if spec.fp8
                    else (L.OP_FWD_NF4, L.OP_BWD_NF4) if spec.nf4 else (L.OP_FWD, L.OP_BWD))
        s["wsf"] = L.workspace(fop, M, di, do, r, device=dev)
        s["wsb"] = L.workspace(bop, M, di, do, r, device=dev)
        sets.append(s)

    def step(s):
        if spec.q4:
            L.lora_linear_fwd_q4(s["x"], s["Wq"], s["Wscale"], s["A"], s["B"], s["h"], s["xa"], alpha, s["wsf"])
            L.lora_linear_bwd_q4(s["dY"], s["x"], s["Wq"], s["Wscale"], s["A"], s["B"], s["xa"], s["dX"], s["dA"],
                                 s["dB"], alpha, s["wsb"])
        elif spec.fp8:
            L.lora_linear_fwd_fp8(s["x"], s["W8"], s["W8scale"], s["A"], s["B"], s["h"], s["xa"], alpha, s["wsf"])
            L.lora_linear_bwd_fp8(s["dY"], s["x"], s["W8"], s["W8scale"], s["A"], s["B"], s["xa"], s["dX"],
                                  s["dA"], s["dB"], alpha, s["wsb"])
        elif spec.nf4:
            L.lora_linear_fwd_nf4(s["x"], s["Wq"], s["Wscale"], s["cb"], s["A"], s["B"], s["h"], s["xa"], alpha,
                                  s["wsf"])
            L.lora_linear_bwd_nf4(s["dY"], s["x"], s["Wq"], s["Wscale"], s["cb"], s["A"], s["B"], s["xa"], s["dX"],
                                  s["dA"], s["dB"], alpha, s["wsb"])
        else:
            L.lora_linear_fwd(s["x"], s["W"], s["A"], s["B"], s["h"], s["xa"], alpha, s["wsf"])
            L.lora_linear_bwd(s["dY"], s["x"], s["W"], s["A"], s["B"], s["xa"], s["dX"], s["dA"], s["dB"], alpha,
                              s["wsb"])
        if world > 1:
            s["grad"].all_reduce()

    def barrier():
        if world > 1:
            dist.barrier(device_ids=[local])

    for i in range(args.warmup):
        step(sets[i % N_SETS])
    torch.cuda.synchronize()
    for s in sets:
        L.lora_linear_check(s["wsf"])
        L.lora_linear_check(s["wsb"])

    stream = torch.cuda.current_stream()
    host_ms = [0.0]

    def timed_region(n_steps, timing_hooks=False):
        barrier()
        torch.cuda.synchronize()
        if timing_hooks:
            L.lora_linear_timing_read()
            L.lora_linear_timing_enable(True)
        # let the host enqueue every step ahead of the GPU (with the timing hooks an event
        # pair per launch costs the host more than a step takes on the GPU)
        torch.cuda._sleep(int(5e6 + (1.5e6 if timing_hooks else 2e5) * n_steps))
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        n0 = L.lora_linear_launch_count()
        th = time.perf_counter()
        e0.record(stream)
        for i in range(n_steps):
            step(sets[i % N_SETS])
        e1.record(stream)
        host_ms[0] = (time.perf_counter() - th) * 1e3
        n1 = L.lora_linear_launch_count()
        torch.cuda.synchronize()
        barrier()
        rec = None
        if timing_hooks:
            L.lora_linear_timing_enable(False)
            rec = L.lora_linear_timing_read()
        return e0.elapsed_time(e1), n1 - n0, rec

    sampler = ClockSampler(dev)
    with sampler:
        ms, launches, _ = timed_region(args.steps)
    clocks = sampler.summary()
    host_enqueue_ms = host_ms[0]
    t = torch.tensor([ms], dtype=torch.float64, device=dev)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    ms_max = float(t.item())

    # Per-kernel device times (separate pass, event pairs around every launch).
    _, _, rec = timed_region(min(args.steps, 100), timing_hooks=True)
    for s in sets:
        L.lora_linear_check(s["wsf"])
        L.lora_linear_check(s["wsb"])

    flops_step = spec.flops
    total_flops = flops_step * args.steps * world
    value = total_flops / (ms_max * 1e-3) / 1e12
    ms_per_step = ms_max / args.steps
    tokens_per_s = M * world * args.steps / (ms_max * 1e-3)

    # roofline of the dominant kernel
    # (stacked projections: each output column of the forward uses its own r/proj ranks)
    kern_flops = {"fwd_main": 2.0 * M * do * (di + r // spec.proj), "dx_main": 2.0 * M * di * (do + r)}
    dom = max(("fwd_main", "dx_main"), key=lambda k: rec[k][0])
    dom_ms = rec[dom][0] / max(1, rec[dom][1])
    achieved = kern_flops[dom] / (dom_ms * 1e-3) / 1e12
    # A kernel timed inside a long, power-capped run is held to the sustained GEMM peak,
    # one timed in a short burst (no power capping seen) to the burst peak.
    sustained = ms_max > 250.0 or "sw_power_cap" in (clocks.get("reasons") or [])
    peak = peaks["bf16_tflops_sustained"] if sustained else peaks["bf16_tflops"]
    peak_kind = "sustained" if sustained else "burst"
    roofline = {"bound": "tensor", "kernel": dom, "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                "frac": achieved / peak,
                "peak_src": f"{peaks['src']} bf16 {peak_kind} (MEASURED_PEAKS.json; timed region {ms_max:.0f} ms)",
                "traffic": stored_traffic(dom, workload_name)}
    t_roof = max(flops_step / (peak * 1e12), algorithmic_bytes(spec) / (peaks["hbm_gbs"] * 1e9))
    step_roof = {"t_roof_us": t_roof * 1e6, "t_meas_us": ms_per_step * 1e3, "frac": t_roof / (ms_per_step * 1e-3),
                 "definition": f"max(FLOP / bf16 {peak_kind} peak, algorithmic bytes / HBM peak) over the measured step time"}
    kernels = {k: {"us_per_launch": (v[0] / v[1] * 1e3) if v[1] else None, "launches": v[1]} for k, v in rec.items()}
    # Each kernel's own device span in one traced step (the library's per-CTA trace:
    # globaltimer at the first CTA's set-up and at the last CTA's exit).  The event pair of
    # the timing pass also brackets the launch, which adds 6-8 us to the side kernels here.
    for k, span in device_spans(step, sets[0]).items():
        if k in kernels:
            kernels[k]["span_us"] = span
    # The same roofline from the dominant kernel's device span.  A main GEMM whose CTAs a
    # programmatic launch made resident early starts work as its predecessor completes,
    # a few us before the stream records the event in front of it, so its event time can
    # read shorter than its span; the span figure is the conservative one.
    dom_span = kernels.get(dom, {}).get("span_us")
    if dom_span:
        roofline["span_us"] = dom_span
        roofline["achieved_span"] = kern_flops[dom] / (dom_span * 1e-6) / 1e12
        roofline["frac_span"] = roofline["achieved_span"] / peak

    # Forward and backward separately: events around each call over 50 steps (the event
    # between them breaks the programmatic-launch overlap of the two, so the parts sum to
    # a little more than the step).
    fb = None
    if world == 1:
        def fwd_call(st):
            if spec.q4:
                L.lora_linear_fwd_q4(st["x"], st["Wq"], st["Wscale"], st["A"], st["B"], st["h"], st["xa"], alpha,
                                     st["wsf"])
            elif spec.fp8:
                L.lora_linear_fwd_fp8(st["x"], st["W8"], st["W8scale"], st["A"], st["B"], st["h"], st["xa"], alpha,
                                      st["wsf"])
            elif spec.nf4:
                L.lora_linear_fwd_nf4(st["x"], st["Wq"], st["Wscale"], st["cb"], st["A"], st["B"], st["h"], st["xa"],
                                      alpha, st["wsf"])
            else:
                L.lora_linear_fwd(st["x"], st["W"], st["A"], st["B"], st["h"], st["xa"], alpha, st["wsf"])

        def bwd_call(st):
            if spec.q4:
                L.lora_linear_bwd_q4(st["dY"], st["x"], st["Wq"], st["Wscale"], st["A"], st["B"], st["xa"], st["dX"],
                                     st["dA"], st["dB"], alpha, st["wsb"])
            elif spec.fp8:
                L.lora_linear_bwd_fp8(st["dY"], st["x"], st["W8"], st["W8scale"], st["A"], st["B"], st["xa"],
                                      st["dX"], st["dA"], st["dB"], alpha, st["wsb"])
            elif spec.nf4:
                L.lora_linear_bwd_nf4(st["dY"], st["x"], st["Wq"], st["Wscale"], st["cb"], st["A"], st["B"],
                                      st["xa"], st["dX"], st["dA"], st["dB"], alpha, st["wsb"])
            else:
                L.lora_linear_bwd(st["dY"], st["x"], st["W"], st["A"], st["B"], st["xa"], st["dX"], st["dA"],
                                  st["dB"], alpha, st["wsb"])

        n_fb = 50
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(n_fb)]
        torch.cuda.synchronize()
        torch.cuda._sleep(int(5e6 + 2e5 * n_fb))
        for i in range(n_fb):
            st = sets[i % N_SETS]
            evs[i][0].record(stream)
            fwd_call(st)
            evs[i][1].record(stream)
            bwd_call(st)
            evs[i][2].record(stream)
        torch.cuda.synchronize()
        f_ms = sorted(e[0].elapsed_time(e[1]) for e in evs)[n_fb // 2]
        b_ms = sorted(e[1].elapsed_time(e[2]) for e in evs)[n_fb // 2]
        fb = {"fwd_us": f_ms * 1e3, "bwd_us": b_ms * 1e3, "note": "medians over 50 steps"}

    # Context, not the reference arm: the unfused composition of the same layer in PyTorch
    # with autograd (x@W.T + s*(x@A.T)@B.T, cuBLAS bf16), same inputs, same GPU.
    context = None
    if world == 1 and not spec.q4 and not spec.fp8 and not spec.nf4:
        st = sets[0]
        xg = st["x"].detach().clone().requires_grad_(True)
        Ag = st["A"].detach().clone().requires_grad_(True)
        Bg = st["B"].detach().clone().requires_grad_(True)
        sc = spec.s

        def torch_step():
            xg.grad = Ag.grad = Bg.grad = None
            hh = xg @ st["W"].t() + sc * ((xg @ Ag.t()) @ Bg.t())
            hh.backward(st["dY"])

        for _ in range(3):
            torch_step()
        n_t = 20
        torch.cuda.synchronize()
        torch.cuda._sleep(int(2e7))
        c0 = torch.cuda.Event(enable_timing=True)
        c1 = torch.cuda.Event(enable_timing=True)
        c0.record(stream)
        for _ in range(n_t):
            torch_step()
        c1.record(stream)
        torch.cuda.synchronize()
        t_ms = c0.elapsed_time(c1) / n_t
        context = {"what": "unfused PyTorch composition with autograd (x@W.T + s*(x@A.T)@B.T), bf16, same inputs",
                   "ms_per_step": t_ms, "tflops": spec.flops / (t_ms * 1e-3) / 1e12}
        del xg, Ag, Bg

    # The deploy-time merge W' = W + s.B.A of the same layer (HBM-bound: one read of the
    # weight, one write of W').  Timed as a model's merge runs: back to back over several
    # copies of the weight and outputs, more than twice L2 in all, so every read comes from
    # DRAM and every write goes back to it during the timed merges; CUDA events on the
    # launch stream around the batch, behind a GPU sleep that covers the host's enqueue.
    merge = None
    if rank == 0:
        s0 = sets[0]
        keys = (("Wq", "Wscale") if (spec.q4 or spec.nf4) else ("W8", "W8scale") if spec.fp8 else ("W",))
        w_one = sum(s0[k].numel() * s0[k].element_size() for k in keys) + do * di * 2
        n_set = max(2, -(-(256 << 20) // w_one))
        msets = [{k: (s0[k] if i == 0 else s0[k].clone()) for k in keys} for i in range(n_set)]
        for m in msets:
            m["out"] = torch.empty(do, di, dtype=torch.bfloat16, device=dev)

        def merge_once(m):
            if spec.q4:
                L.lora_linear_merge_q4(m["Wq"], m["Wscale"], s0["A"], s0["B"], m["out"], alpha)
            elif spec.nf4:
                L.lora_linear_merge_nf4(m["Wq"], m["Wscale"], s0["cb"], s0["A"], s0["B"], m["out"], alpha)
            elif spec.fp8:
                L.lora_linear_merge_fp8(m["W8"], m["W8scale"], s0["A"], s0["B"], m["out"], alpha)
            else:
                L.lora_linear_merge(m["W"], s0["A"], s0["B"], m["out"], alpha)

        for m in msets:
            merge_once(m)
        n_merge = max(16, 4 * n_set)
        times = []
        for _ in range(3):
            m0 = torch.cuda.Event(enable_timing=True)
            m1 = torch.cuda.Event(enable_timing=True)
            torch.cuda._sleep(int(2e7))
            m0.record(stream)
            for i in range(n_merge):
                merge_once(msets[i % n_set])
            m1.record(stream)
            torch.cuda.synchronize()
            times.append(m0.elapsed_time(m1) / n_merge)
        L.lora_linear_merge_check()
        del msets
        t_merge = sorted(times)[1]
        w_bytes = (do * di // 2 + do * (di // 64) * 2 if (spec.q4 or spec.nf4)
                   else do * di + do * 2 if spec.fp8 else do * di * 2)
        m_bytes = w_bytes + r * di * 2 + do * r * 2 + do * di * 2
        ach = m_bytes / (t_merge * 1e-3) / 1e9
        merge = {"us": t_merge * 1e3, "bytes": m_bytes, "achieved_gbs": ach, "peak_gbs": peaks["hbm_gbs"],
                 "frac": ach / peaks["hbm_gbs"], "bound": "hbm",
                 "timing": f"median of 3 batches of {n_merge} merges back to back over {n_set} weight copies",
                 "what": "W' = W + s.B.A" + (" (4-bit W decoded)" if spec.q4 else " (NF4 W decoded)" if spec.nf4
                                             else " (FP8 W decoded)" if spec.fp8 else "")}

    # end to end through the C ABI with host buffers: every step copies its inputs in from
    # pinned host memory and its outputs back out (W stays resident: frozen model state).
    # Steps are pipelined the way a training loop overlaps its data movement: copies in
    # on one stream, fwd + bwd on the launch stream, copies out on a third, over two
    # device buffer sets; events order each step's copy-in -> compute -> copy-out and
    # keep a set from being overwritten before its previous step is done with it.
    e2e = None
    if not args.no_e2e:
        pair = sets[:2]
        names_in = ["x", "dY", "A", "B"]
        names_out = ["h", "dX", "dA", "dB"]
        hin = {k: torch.empty_like(pair[0][k], device="cpu").pin_memory() for k in names_in}
        for k in names_in:
            hin[k].copy_(pair[0][k])
        hout = {k: torch.empty_like(pair[0][k], device="cpu").pin_memory() for k in names_out}
        n_e2e = max(5, min(args.steps, 50))
        s_in, s_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)

        def e2e_run(n):
            computed = [None, None]   # per set: its last step's fwd + bwd finished
            copied_out = [None, None]  # per set: its last step's outputs copied out
            for i in range(n):
                j = i % 2
                st = pair[j]
                if computed[j] is not None:
                    s_in.wait_event(computed[j])
                with torch.cuda.stream(s_in):
                    for k in names_in:
                        st[k].copy_(hin[k], non_blocking=True)
                ev_in = torch.cuda.Event()
                ev_in.record(s_in)
                stream.wait_event(ev_in)
                if copied_out[j] is not None:
                    stream.wait_event(copied_out[j])
                with torch.cuda.stream(stream):
                    step(st)
                ev_c = torch.cuda.Event()
                ev_c.record(stream)
                computed[j] = ev_c
                s_out.wait_event(ev_c)
                with torch.cuda.stream(s_out):
                    for k in names_out:
                        hout[k].copy_(st[k], non_blocking=True)
                ev_o = torch.cuda.Event()
                ev_o.record(s_out)
                copied_out[j] = ev_o

        e2e_run(2)
        barrier()
        torch.cuda.synchronize()
        with torch.cuda.stream(s_in):
            torch.cuda._sleep(int(2e6))
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(s_in)
        e2e_run(n_e2e)
        s_out.wait_stream(stream)
        e1.record(s_out)
        torch.cuda.synchronize()
        barrier()
        te = torch.tensor([e0.elapsed_time(e1)], dtype=torch.float64, device=dev)
        if world > 1:
            dist.all_reduce(te, op=dist.ReduceOp.MAX)
        e2e_ms = float(te.item())
        for st in pair:
            L.lora_linear_check(st["wsf"])
            L.lora_linear_check(st["wsb"])
        e2e = {"value": flops_step * n_e2e * world / (e2e_ms * 1e-3) / 1e12, "unit": UNIT,
               "h2d_bytes_per_step": int(sum(hin[k].numel() * hin[k].element_size() for k in names_in)),
               "d2h_bytes_per_step": int(sum(hout[k].numel() * hout[k].element_size() for k in names_out)),
               "ms_per_step": e2e_ms / n_e2e, "steps": n_e2e,
               "note": "pinned host buffers; frozen W resident on the device; copies in, fwd+bwd and copies "
                       "out pipelined over two device buffer sets on three streams"}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(spec)

    if rank == 0:
        out = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": config_dict(spec, workload_name, world),
            "world_size": dist.get_world_size() if world > 1 else 1,
            "tokens_per_s": tokens_per_s,
            "roofline": roofline,
            "roofline_step": step_roof,
            "kernels": kernels,
            "cpu_baseline": cpu,
            "clocks": clocks,
            "e2e": e2e,
            "gpu_launches": int(launches),
            "merge": merge,
            "fwd_bwd": fb,
            "context_torch_unfused": context,
            "host_enqueue_ms": host_enqueue_ms,
        }
        print(json.dumps(out), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
