"""Per-shape plan tuner for the fused LoRA linear layer.

The library picks a plan for every layer shape from fixed rules and a streaming cost
model (lora_linear_get_plan shows it).  This module measures instead: it times the
layer's forward + backward on the device under candidate plans, keeps the fastest,
and caches the choice on disk per device, so later processes install it with
lora_linear_set_plan before their first call (page "UnSloth加速库集成：编译级优化带来
的性能飞跃", section 技术三: probe the kernel configuration for the GPU, sequence length
and rank, and cache it).  Every plan computes the same function; only the order of fp32
sums differs, so a tuned plan meets the same bounds against the oracle.

The search is coordinate descent from the library's own plan: each field in turn takes
each of its admissible values with the others held, and the best value stays.  A
candidate is timed as the median of `rounds` CUDA-event measurements of `reps`
back-to-back forward + backward calls on the current stream, the calls rotating through
sets of x and dY larger than L2 together, so the streamed operands come from DRAM.
"""
from __future__ import annotations

import json
import os

from . import lora_linear as L

# Values each plan field may take (lora_plan_t); the admissible ones depend on r.
SIDE_MAX_R = 64
SIDE_MAX_R_BWD = 32


def field_options(r: int) -> dict:
    """The values worth trying for each field at rank r, in search order."""
    opts = {
        "side_fwd": [1, 2] if r <= SIDE_MAX_R else [2],
        "xa_cluster": [1, 2, 4],
        "side_bwd": [1, 2] if r <= SIDE_MAX_R_BWD else [2],
        "g_cluster": [1, 2, 4],
        "g_group": [a for a in range(1, 7) if a * r <= 64],
        "da_cluster": [1, 2, 4],
        "fwd_tail": [1, 2, 3],
        "dx_overlap": [1, 2, 3],
    }
    return opts


def _applies(field: str, plan: dict) -> bool:
    """Whether a field matters under the rest of the plan (side-kernel knobs only count
    when the side kernels run)."""
    if field == "xa_cluster":
        return plan.get("side_fwd") == 1
    if field in ("g_cluster", "g_group", "da_cluster"):
        return plan.get("side_bwd") == 1
    return True


def candidates_from(plan: dict, field: str, r: int) -> list:
    """Plans equal to `plan` but for `field`, over its admissible values."""
    out = []
    for v in field_options(r)[field]:
        p = dict(plan)
        p[field] = v
        out.append(p)
    return out


def coordinate_descent(start: dict, r: int, cost) -> tuple:
    """Minimise cost(plan) one field at a time from `start`; returns (best plan, its cost,
    every (plan, cost) tried).  `cost` may return None for a plan the library rejects."""
    best, best_c = dict(start), cost(start)
    tried = [(dict(start), best_c)]
    for field in field_options(r):
        if not _applies(field, best):
            continue
        for cand in candidates_from(best, field, r):
            if cand == best:
                continue
            c = cost(cand)
            tried.append((dict(cand), c))
            if c is not None and (best_c is None or c < best_c):
                best, best_c = cand, c
    return best, best_c, tried


def _op_pair(wf: str):
    return {"bf16": (L.OP_FWD, L.OP_BWD), "q4": (L.OP_FWD_Q4, L.OP_BWD_Q4),
            "fp8": (L.OP_FWD_FP8, L.OP_BWD_FP8), "nf4": (L.OP_FWD_NF4, L.OP_BWD_NF4)}[wf]


# Bytes of the per-call streamed inputs (x and dY) the timed calls rotate through: more
# than twice the B200's 126 MB L2, so each call reads them from DRAM as in training
# (otherwise the HBM-bound side products look as fast as they would from L2).
ROTATE_BYTES = 256 << 20
MAX_SETS = 8


class _Layer:
    """Device buffers of one layer shape (random values: only timing is measured), with
    several sets of x and dY that successive calls rotate through."""

    def __init__(self, M, d_in, d_out, r, wf, alpha, device):
        import torch
        g = torch.Generator(device="cpu").manual_seed(1234)

        def bf(*shape, scale=1.0):
            return (torch.randn(*shape, generator=g) * scale).to(torch.bfloat16).to(device)

        self.shape, self.wf, self.alpha, self.device = (M, d_in, d_out, r), wf, alpha, device
        per_set = M * (d_in + d_out) * 2
        n_sets = max(1, min(MAX_SETS, -(-ROTATE_BYTES // per_set)))
        self.sets = [(bf(M, d_in), bf(M, d_out)) for _ in range(n_sets)]
        self.turn = 0
        self.x, self.dY = self.sets[0]
        self.A, self.B = bf(r, d_in, scale=d_in ** -0.5), bf(d_out, r, scale=0.02)
        if wf in ("q4", "nf4"):
            self.Wq = torch.randint(1, 16, (d_out, d_in // 2), generator=g, dtype=torch.uint8).to(device)
            self.Ws = bf(d_out, d_in // 64, scale=0.01).abs()
            if wf == "nf4":
                from .inputs import nf4_codebook
                self.codebook = nf4_codebook()
        elif wf == "fp8":
            self.W8 = torch.randint(0, 0x7E, (d_out, d_in), generator=g, dtype=torch.uint8).to(device)
            self.W8s = bf(d_out, scale=1e-3).abs()
        else:
            self.W = bf(d_out, d_in, scale=d_in ** -0.5)
        self.h = torch.empty(M, d_out, dtype=torch.bfloat16, device=device)
        self.xa = torch.empty(M, r, dtype=torch.bfloat16, device=device)
        self.dX = torch.empty(M, d_in, dtype=torch.bfloat16, device=device)
        self.dA = torch.empty(r, d_in, dtype=torch.float32, device=device)
        self.dB = torch.empty(d_out, r, dtype=torch.float32, device=device)
        self.ws = None

    def workspaces(self):
        """Workspaces of the plan now in effect (its size follows the plan)."""
        fop, bop = _op_pair(self.wf)
        self.wsf = L.workspace(fop, *self.shape, device=self.device)
        self.wsb = L.workspace(bop, *self.shape, device=self.device)

    def step(self):
        self.x, self.dY = self.sets[self.turn % len(self.sets)]
        self.turn += 1
        a = self.alpha
        if self.wf == "q4":
            L.lora_linear_fwd_q4(self.x, self.Wq, self.Ws, self.A, self.B, self.h, self.xa, a, self.wsf)
            L.lora_linear_bwd_q4(self.dY, self.x, self.Wq, self.Ws, self.A, self.B, self.xa, self.dX, self.dA,
                                 self.dB, a, self.wsb)
        elif self.wf == "nf4":
            cb = self.codebook
            L.lora_linear_fwd_nf4(self.x, self.Wq, self.Ws, cb, self.A, self.B, self.h, self.xa, a, self.wsf)
            L.lora_linear_bwd_nf4(self.dY, self.x, self.Wq, self.Ws, cb, self.A, self.B, self.xa, self.dX, self.dA,
                                  self.dB, a, self.wsb)
        elif self.wf == "fp8":
            L.lora_linear_fwd_fp8(self.x, self.W8, self.W8s, self.A, self.B, self.h, self.xa, a, self.wsf)
            L.lora_linear_bwd_fp8(self.dY, self.x, self.W8, self.W8s, self.A, self.B, self.xa, self.dX, self.dA,
                                  self.dB, a, self.wsb)
        else:
            L.lora_linear_fwd(self.x, self.W, self.A, self.B, self.h, self.xa, a, self.wsf)
            L.lora_linear_bwd(self.dY, self.x, self.W, self.A, self.B, self.xa, self.dX, self.dA, self.dB, a,
                              self.wsb)


def time_plan(layer: _Layer, plan: dict | None, reps: int = 10, rounds: int = 3):
    """Median us per forward + backward under `plan` (None: the library's own), or None
    if the library rejects the plan for this shape."""
    import torch
    try:
        L.lora_linear_set_plan(*layer.shape, plan)
    except L.LoraError:
        return None
    layer.workspaces()
    for _ in range(2):
        layer.step()
    torch.cuda.synchronize()
    L.lora_linear_check(layer.wsf)
    L.lora_linear_check(layer.wsb)
    times = []
    for _ in range(rounds):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda._sleep(int(2e6))  # the host enqueues every call ahead of the timed ones
        e0.record()
        for _ in range(reps):
            layer.step()
        e1.record()
        torch.cuda.synchronize()
        times.append(e0.elapsed_time(e1) * 1e3 / reps)
    L.lora_linear_check(layer.wsf)
    L.lora_linear_check(layer.wsb)
    return sorted(times)[len(times) // 2]


def tune(M: int, d_in: int, d_out: int, r: int, wf: str = "bf16", alpha: float = 16.0, reps: int = 10,
         rounds: int = 3, device=None) -> dict:
    """Search plans for this shape on the current device; installs the best and returns
    {"plan", "us", "default_plan", "default_us", "tried"}."""
    import torch
    device = device or torch.device("cuda", torch.cuda.current_device())
    L.lora_linear_set_plan(M, d_in, d_out, r, None)
    _, bop = _op_pair(wf)
    default = L.lora_linear_get_plan(bop, M, d_in, d_out, r)
    layer = _Layer(M, d_in, d_out, r, wf, alpha, device)
    t_default = time_plan(layer, None, reps, rounds)
    start = {k: default[k] for k in L.lora_plan_t.FIELDS}
    best, best_us, tried = coordinate_descent(start, r, lambda p: time_plan(layer, p, reps, rounds))
    if best_us is None or (t_default is not None and t_default <= best_us):
        best, best_us = start, t_default
    L.lora_linear_set_plan(M, d_in, d_out, r, best)
    # what runs: a field value that does not apply to this shape (a K-split tail where the
    # last wave is not cut, say) reads back as the library's fallback
    effective = L.lora_linear_get_plan(bop, M, d_in, d_out, r)
    best = {k: effective[k] for k in L.lora_plan_t.FIELDS}
    return {"plan": best, "us": best_us, "default_plan": default, "default_us": t_default,
            "tried": [{"plan": p, "us": c} for p, c in tried]}


def device_key() -> str:
    import torch
    p = torch.cuda.get_device_properties(torch.cuda.current_device())
    return f"{p.name} sm{p.major}{p.minor} x{p.multi_processor_count}"


def shape_key(M, d_in, d_out, r, wf) -> str:
    return f"M{M} {d_in}->{d_out} r{r} {wf}"


class PlanCache:
    """Tuned plans on disk: {device key: {shape key: {"plan": ..., "us": ...}}}."""

    def __init__(self, path: str):
        self.path = path
        self.data = {}
        if os.path.exists(path):
            with open(path) as f:
                self.data = json.load(f)

    def get(self, device: str, M, d_in, d_out, r, wf):
        return self.data.get(device, {}).get(shape_key(M, d_in, d_out, r, wf))

    def put(self, device: str, M, d_in, d_out, r, wf, result: dict):
        self.data.setdefault(device, {})[shape_key(M, d_in, d_out, r, wf)] = {
            "shape": [M, d_in, d_out, r], "wf": wf, "plan": result["plan"], "us": result["us"],
            "default_us": result.get("default_us")}

    def save(self):
        tmp = self.path + ".tmp"
        with open(tmp, "w") as f:
            json.dump(self.data, f, indent=1, sort_keys=True)
        os.replace(tmp, self.path)

    def apply(self, device: str) -> int:
        """Install every cached plan of `device` in the library; returns how many."""
        n = 0
        for e in self.data.get(device, {}).values():
            M, d_in, d_out, r = e["shape"]
            L.lora_linear_set_plan(M, d_in, d_out, r, e["plan"])
            n += 1
        return n


def tune_cached(cache_path: str, M, d_in, d_out, r, wf="bf16", **kw) -> dict:
    """The cached plan for this device and shape, installed; tuned and cached first if
    there is none."""
    cache = PlanCache(cache_path)
    dev = device_key()
    hit = cache.get(dev, M, d_in, d_out, r, wf)
    if hit is not None:
        L.lora_linear_set_plan(M, d_in, d_out, r, hit["plan"])
        return hit
    res = tune(M, d_in, d_out, r, wf, **kw)
    cache.put(dev, M, d_in, d_out, r, wf, res)
    cache.save()
    return res
