#!/usr/bin/env python
"""Benchmark of the mixed-head causal attention layer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                    [--impl ours|reference]

One step is the whole hot path on one batch, all through the C ABI with the
inputs resident in HBM: the forward call (the replaced heads' pattern
preparation -- log-normalisers and factored arrays -- in one launch, then the
fused forward) and the backward call (row terms with the pattern preparation
in one launch, the fused backward, the dQ conversion).
Default workload: the 124M-shape layer B=8, H=12 (3 replaced), T=4096,
d_h=64, forward + backward.

Prints one JSON line (rank 0).  Multi-GPU (torchrun): every rank processes
its own batch shard of the same shape (weak scaling, no collective on the
data path); the time is the max over ranks.  `--impl reference` times the
fp64 CPU oracle on a bounded sample of the same workload instead.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

from mixed_head_causal_b200 import inputs as I  # noqa: E402

DEFAULT_WORKLOAD = "124m_b8_t4096_r25"
METRIC = "mixed-head causal attn fwd+bwd tokens/s & TFLOP/s on 1 B200; % of bf16 TC peak"
UNIT = "tokens/s"


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(I.WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--grad-dtype", default="bf16", choices=["bf16", "fp32"])
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extra", action="store_true",
                    help="skip the extra keys (per_config, head_cost) after the headline timing")
    ap.add_argument("--head-cost", action="store_true",
                    help="instead of the headline line, time the workload's shape with 0, 25, 50 and 100%% of "
                         "the heads replaced and fit t = t0 + c_o n_o + c_r n_r per pass")
    ap.add_argument("--pattern-grad", action="store_true",
                    help="instead of the headline line, time the trainable-pattern gradient (dalpha, drho) of "
                         "the workload's replaced heads")
    ap.add_argument("--calibration", action="store_true",
                    help="instead of the headline line, time the calibration statistics (A_hat, s_var) over "
                         "the workload's batch as N samples, every head ordinary")
    ap.add_argument("--fit", action="store_true",
                    help="instead of the headline line, time the fitting of (a, r) (400 Adam steps) to the "
                         "patterns of the workload's replaced heads")
    ap.add_argument("--gqa", type=int, default=0, metavar="H_KV",
                    help="instead of the headline line, time fwd and bwd with K/V shared by groups of "
                         "H / H_KV query heads")
    return ap.parse_args()


# ------------------------------------------------------------------ helpers

def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": p["hbm_gbs"], "bf16_tflops": p["bf16_tflops"],
                "bf16_tflops_sustained": p.get("bf16_tflops_sustained", p["bf16_tflops"]), "src": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "src": "fallback"}


class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = None

    def __enter__(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=self.f, stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.15)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            self.f.close()

    def summary(self):
        if self.proc is None or not self.path or not os.path.exists(self.path):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"]}
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    rows.append((float(parts[1]), float(parts[2]), float(parts[3]), parts[5:9]))
                except ValueError:
                    continue
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        loaded = [r for r in rows if r[2] > 200.0] or rows
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in loaded for i, v in enumerate(r[3]) if v.lower() == "active"})
        return {"sm_mhz": statistics.median(r[0] for r in loaded), "sm_max_mhz": max(r[1] for r in rows),
                "samples": len(loaded), "power_w_max": max(r[2] for r in rows), "reasons": reasons}


# The sources a tensor-core kernel is built from: its own file and the two
# headers every kernel file includes.
KERNEL_SOURCES = {"fwd_tc": "saf_fwd_tc.cu", "bwd_tc": "saf_bwd_tc.cu"}


def kernel_source_hash(kernel):
    csrc = os.path.join(ROOT, "mixed_head_causal_b200", "csrc")
    own = KERNEL_SOURCES.get(kernel)
    if own is None:
        return None
    return source_hash([os.path.join(csrc, f) for f in (own, "saf_common.cuh", "tc_util.cuh")])


def source_hash(paths):
    h = hashlib.sha256()
    for p in sorted(paths):
        with open(p, "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ------------------------------------------------------------------ CPU oracle

def oracle_sample(w, seed=0, groups=1):
    """A bounded sample of (b, h) slices with the workload's head-kind mix,
    `groups` copies of the smallest such group, on batches 0, 1, ..."""
    mask = I.replaced_mask(w, seed).numpy()
    rep = [h for h in range(w.H) if mask[h]]
    ordn = [h for h in range(w.H) if not mask[h]]
    # keep the ordinary:replaced ratio of the layer (e.g. 3:1 for 9:3)
    from math import gcd
    g = gcd(len(ordn), len(rep)) if rep and ordn else 1
    n_o, n_r = (len(ordn) // g, len(rep) // g) if rep and ordn else (min(4, len(ordn)), min(4, len(rep)))
    slices = []
    for gi in range(groups):
        b = gi % w.B
        slices += [(b, ordn[(gi * n_o + i) % len(ordn)]) for i in range(n_o)]
        slices += [(b, rep[(gi * n_r + i) % len(rep)]) for i in range(n_r)]
    return slices


def run_oracle_sample(w, slices, seed=0, threads=None):
    import numpy as np
    import oracle
    a, r = I.make_pattern(w, seed)
    mask = I.replaced_mask(w, seed).numpy()
    q = torch.stack([I.make_slice(w, seed, "q", b, h) for b, h in slices])
    k = torch.stack([I.make_slice(w, seed, "k", b, h) for b, h in slices])
    v = torch.stack([I.make_slice(w, seed, "v", b, h) for b, h in slices])
    ar = np.stack([a[h].double().numpy() for _, h in slices])
    rr = np.stack([r[h].double().numpy() for _, h in slices])
    rep = [int(mask[h]) for _, h in slices]
    threads = threads or oracle.default_threads()
    t0 = time.perf_counter()
    oracle.fwd_slices(q, k, v, ar, rr, rep, threads)
    if w.backward:
        do = torch.stack([I.make_slice(w, seed, "do", b, h) for b, h in slices])
        oracle.bwd_slices(q, k, v, do, ar, rr, rep, threads)
    dt = time.perf_counter() - t0
    frac = len(slices) / float(w.B * w.H)
    return dt, frac, min(threads, len(slices))


def cpu_baseline(w):
    # sixteen groups of the head-kind mix: 64 slices, about eight seconds on
    # 16 host cores at the 124M shape (half a minute on 4)
    slices = oracle_sample(w, groups=16)
    dt, frac, cores = run_oracle_sample(w, slices)
    return {"value": w.tokens * frac / dt, "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": f"{len(slices)} of {w.B * w.H} (batch, head) slices of {w.name} (same head-kind mix), "
                      f"fwd{'+bwd' if w.backward else ''}, {dt:.1f} s, scaled by slice count"}


def arm_config(w, world, grad_dtype):
    """The `config` object of the JSON line (both arms)."""
    return {"workload": w.name, "B": w.B, "H": w.H, "T": w.T, "d_h": w.d, "n_replaced": len(I.replaced_heads(w)),
            "global_batch": w.B * world, "seq_len": w.T, "parallelism": f"dp{world}",
            "passes": "fwd+bwd" if w.backward else "fwd", "grad_dtype": grad_dtype,
            "l2": "inputs larger than L2 (no flush)", "flops_per_step": I.flops(w)["total"] * world}


def reference_arm(args, world, rank):
    w = I.WORKLOADS[args.workload]
    if rank != 0:
        return
    # one slice per step, cycling through one group of the head-kind mix, so
    # that any --steps K --warmup W run stays within a few minutes; the rate is
    # the slices' share of the workload's tokens over their total time
    group = oracle_sample(w)
    for s in range(args.warmup):
        run_oracle_sample(w, [group[s % len(group)]])
    total, done, cores = 0.0, 0.0, 1
    for s in range(args.steps):
        dt, frac, cores = run_oracle_sample(w, [group[s % len(group)]])
        total += dt
        done += frac
    value = w.tokens * done / total
    slices = group
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic",
            "config": arm_config(w, args.gpus, args.grad_dtype),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                             "sample": f"one of {w.B * w.H} (batch, head) slices per step, cycling through "
                                       f"{len(slices)} with the layer's head-kind mix, scaled by slice count"},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ our arm

def algorithmic_flops_per_launch(kernel: str, w, n_r: int) -> float:
    """Algorithmic flops of one launch of `kernel` on workload w (causal
    T^2/2 convention; one unit = d_h * T^2 flops per (batch, head) = one
    T x T x d_h causal contraction)."""
    n_o = w.H - n_r
    unit = float(w.d) * w.T * w.T * w.B
    table = {
        "fwd_mma": unit * (2 * n_o + n_r),     # QK^T + PV (ordinary), PV (replaced)
        "fwd_tc": unit * (2 * n_o + n_r),
        "dkdv_mma": unit * (4 * n_o + n_r),    # S recompute, dV, dP, dK (ordinary); dV (replaced)
        "dq_mma": unit * n_o,                  # dQ (its S/dP recompute is not algorithmic)
        "bwd_tc": unit * (5 * n_o + n_r),
    }
    return table.get(kernel, 0.0)


def device_inputs(w, dev, seed=0):
    """Inputs of workload w drawn on the GPU with the recipe's distributions
    (Q, K, V, dO standard normal rounded to bf16; the pattern vectors and the
    replaced heads exactly as in the seeded recipe).  Used only for timing the
    extra shapes, where building the seeded CPU tensors would take minutes."""
    g = torch.Generator(device=dev)
    g.manual_seed(1000 + seed)
    x = {}
    for name in ("q", "k", "v") + (("do",) if w.backward else ()):
        x[name] = torch.randn(w.B, w.H, w.T, w.d, generator=g, device=dev, dtype=torch.float32).to(torch.bfloat16)
    a, r = I.make_pattern(w, seed)
    x["alpha"], x["rho"] = a.to(dev), r.to(dev)
    x["mask"] = I.replaced_mask(w, seed)
    return x


def _event_ms(fn, reps, stream):
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(reps):
        fn()
    e1.record(stream)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / reps


def time_passes(w, dev, x, reps, gd=torch.bfloat16):
    """Device time of each pass of the layer on workload w (inputs resident):
    forward, backward (each with its pattern preparation), and the whole step
    (forward + backward, as the headline step), each the mean of `reps`
    back-to-back calls after two warm-up calls."""
    from mixed_head_causal_b200 import saf
    stream = torch.cuda.current_stream(dev)
    mask = x["mask"]
    o = torch.empty(w.B, w.H, w.T, w.d, dtype=torch.bfloat16, device=dev)
    lse = torch.empty(w.B, w.H, w.T, dtype=torch.float32, device=dev)
    ws_f = saf.new_workspace(w.B, w.H, w.T, dev, backward=False)
    grads = None
    ws_b = None
    if w.backward:
        grads = [torch.empty(w.B, w.H, w.T, w.d, dtype=gd, device=dev) for _ in range(3)]
        ws_b = saf.new_workspace(w.B, w.H, w.T, dev, backward=True)

    def fwd():
        saf.mixed_attn_fwd(x["q"], x["k"], x["v"], x["alpha"], x["rho"], mask, out=o, lse=lse, workspace=ws_f)

    def bwd():
        saf.mixed_attn_bwd(x["q"], x["k"], x["v"], o, x["do"], lse, x["alpha"], x["rho"], mask,
                           grad_dtype=gd, dq=grads[0], dk=grads[1], dv=grads[2], workspace=ws_b)

    def step():
        fwd()
        if w.backward:
            bwd()

    for _ in range(2):
        step()
    torch.cuda.synchronize()
    out = {"fwd_ms": _event_ms(fwd, reps, stream)}
    if w.backward:
        out["bwd_ms"] = _event_ms(bwd, reps, stream)
    out["step_ms"] = _event_ms(step, reps, stream)
    del o, lse, ws_f, grads, ws_b
    return out


def rates(w, t, pk):
    """tokens/s, TFLOP/s and fraction of the peak of one timed shape."""
    fl = I.flops(w)
    res = {"workload": w.name, "B": w.B, "H": w.H, "T": w.T, "n_replaced": len(I.replaced_heads(w)),
           "passes": "fwd+bwd" if w.backward else "fwd"}
    res.update({k: round(v, 5) for k, v in t.items()})
    res["tokens_per_s"] = w.tokens / (t["step_ms"] * 1e-3)
    res["tflops"] = fl["total"] / (t["step_ms"] * 1e-3) / 1e12
    res["frac_of_peak"] = res["tflops"] / pk["bf16_tflops"]
    if w.backward:  # the ordinary backward's four products, no recompute of Q K^T
        res["tflops_strict"] = I.flops(w, strict=True)["total"] / (t["step_ms"] * 1e-3) / 1e12
    res["fwd_tflops"] = fl["fwd"] / (t["fwd_ms"] * 1e-3) / 1e12
    if w.backward:
        res["bwd_tflops"] = fl["bwd"] / (t["bwd_ms"] * 1e-3) / 1e12
    return res


def per_config(dev, pk, reps=10):
    """The other measured shapes of the layer: the 50%-replaced 124M shape at
    8K, the 1B-scale shape, and the batch-64 / T=4096 prefill sweep (forward
    only); each with its pass split."""
    out = {}
    names = ["124m_b4_t8192_r50", "1b_b4_h32_t8192_r25"] + list(I.PREFILL_SWEEP)
    for name in names:
        w = I.WORKLOADS[name]
        x = device_inputs(w, dev)
        t = time_passes(w, dev, x, reps if w.T * w.B <= 64 * 4096 else max(3, reps // 2))
        out[name] = rates(w, t, pk)
        del x
        torch.cuda.empty_cache()
    return out


def head_cost_fit(base, dev, reps=10):
    """Per-head cost of each head kind on the shape of `base`: n_r = 0, H/4,
    H/2 and H replaced heads (the first n_r), forward and backward timed
    separately, and the least-squares fit t = t0 + c_o n_o + c_r n_r."""
    import numpy as np
    rows = []
    for n_r in sorted({0, base.H // 4, base.H // 2, base.H}):
        w = I.custom(base.B, base.H, base.T, list(range(n_r)))
        x = device_inputs(w, dev)
        t = time_passes(w, dev, x, reps)
        rows.append((w.H - n_r, n_r, t["fwd_ms"], t["bwd_ms"]))
        del x
        torch.cuda.empty_cache()
    A = np.array([[1.0, r[0], r[1]] for r in rows])
    out = {"config": {"workload": base.name, "B": base.B, "H": base.H, "T": base.T,
                      "n_replaced_points": [r[1] for r in rows]},
           "times_ms": [{"n_o": r[0], "n_r": r[1], "fwd": r[2], "bwd": r[3]} for r in rows]}
    for name, col in (("fwd", 2), ("bwd", 3), ("fwd+bwd", None)):
        y = np.array([r[2] + r[3] if col is None else r[col] for r in rows])
        t0, c_o, c_r = np.linalg.lstsq(A, y, rcond=None)[0]
        out[name] = {"t0_ms": float(t0), "c_o_ms": float(c_o), "c_r_ms": float(c_r),
                     "c_r_over_c_o": float(c_r / c_o) if c_o else None}
    return out


def our_arm(args, world, rank, local):
    from mixed_head_causal_b200 import saf
    if not torch.cuda.is_available():
        raise SystemExit("bench.py: no CUDA device (the product path has no CPU fallback)")
    dev = torch.device("cuda", local)
    w = I.WORKLOADS[args.workload]
    gd = torch.bfloat16 if args.grad_dtype == "bf16" else torch.float32
    seed = rank  # each rank's shard of the global batch
    host = I.make_inputs(w, seed, pin=True, threads=min(16, os.cpu_count() or 1))
    mask = host["mask"]
    n_r = int(mask.sum())
    x = {k: (v.to(dev, non_blocking=True) if k != "mask" else v) for k, v in host.items()}
    B, H, T, d = w.B, w.H, w.T, w.d
    o = torch.empty(B, H, T, d, dtype=torch.bfloat16, device=dev)
    lse = torch.empty(B, H, T, dtype=torch.float32, device=dev)
    dq = torch.empty(B, H, T, d, dtype=gd, device=dev)
    dk = torch.empty_like(dq)
    dv = torch.empty_like(dq)
    ws_f = saf.new_workspace(B, H, T, dev, backward=False)
    ws_b = saf.new_workspace(B, H, T, dev, backward=True) if w.backward else None
    stream = torch.cuda.current_stream(dev)

    def step():
        # one training step of the layer: forward and backward, each preparing
        # the replaced heads' patterns (log Z and the factored arrays) in its
        # first launch
        saf.mixed_attn_fwd(x["q"], x["k"], x["v"], x["alpha"], x["rho"], mask, out=o, lse=lse, workspace=ws_f)
        if w.backward:
            saf.mixed_attn_bwd(x["q"], x["k"], x["v"], o, x["do"], lse, x["alpha"], x["rho"], mask,
                               grad_dtype=gd, dq=dq, dk=dk, dv=dv, workspace=ws_b)

    torch.cuda.synchronize()
    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize()

    # ---- headline: device time of K steps, inputs resident (all > L2 in total)
    launches0 = saf.launch_count()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        barrier(world)
        torch.cuda.synchronize()
        ev0.record(stream)
        for _ in range(args.steps):
            step()
        ev1.record(stream)
        torch.cuda.synchronize()
        barrier(world)
    launches = saf.launch_count() - launches0
    ms_total = max_over_ranks(ev0.elapsed_time(ev1), world)
    ms_step = ms_total / args.steps
    tokens = w.tokens * world
    value = tokens / (ms_step * 1e-3)
    fl = I.flops(w)
    tflops = fl["total"] * world / (ms_step * 1e-3) / 1e12
    # the same time against the strict count (ordinary backward without the recompute of Q K^T)
    tflops_strict = I.flops(w, strict=True)["total"] * world / (ms_step * 1e-3) / 1e12

    # ---- per-kernel timing (separate pass, same steps, events around each launch)
    prof_steps = min(args.steps, 20)
    per_step = max(1, launches // max(1, args.steps))
    saf.profile_enable(prof_steps * per_step + 16)
    for _ in range(prof_steps):
        step()
    torch.cuda.synchronize()
    recs = saf.profile_read()
    saf.profile_enable(0)
    per_kernel = {}
    for name, ms in recs:
        e = per_kernel.setdefault(name, [0, 0.0])
        e[0] += 1
        e[1] += ms
    total_ms = sum(v[1] for v in per_kernel.values()) or 1.0
    kernels = {k: {"launches": v[0], "avg_ms": v[1] / v[0], "share": v[1] / total_ms} for k, v in per_kernel.items()}
    dom = max(kernels, key=lambda k: kernels[k]["share"])
    pk = peaks()
    dom_flops = algorithmic_flops_per_launch(dom, w, n_r)
    achieved = dom_flops / (kernels[dom]["avg_ms"] * 1e-3) / 1e12
    traffic = None
    tpath = os.path.join(ROOT, "profiles", "traffic.json")
    if os.path.exists(tpath):
        with open(tpath) as f:
            tj = json.load(f)
        cur = kernel_source_hash(dom)
        ent = tj.get(dom)
        if ent and ent.get("source_hash") == cur and ent.get("workload") == w.name:
            traffic = ent.get("bytes_per_launch")
    roofline = {"bound": "tensor", "achieved": achieved, "peak": pk["bf16_tflops"], "unit": "TFLOP/s",
                "frac": achieved / pk["bf16_tflops"], "traffic": traffic, "kernel": dom,
                "peak_src": f"{pk['src']} (burst bf16 dense)"}

    # ---- end to end: pinned host -> device, both calls, device -> host of the outputs
    e2e = None
    if not args.no_e2e:
        outs_host = {"o": torch.empty(B, H, T, d, dtype=torch.bfloat16, pin_memory=True)}
        if w.backward:
            for k_ in ("dq", "dk", "dv"):
                outs_host[k_] = torch.empty(B, H, T, d, dtype=gd, pin_memory=True)
        in_keys = ["q", "k", "v"] + (["do"] if w.backward else [])
        h2d = sum(host[k_].numel() * host[k_].element_size() for k_ in in_keys)
        h2d += sum(host[k_].numel() * 4 for k_ in ("alpha", "rho"))
        d2h = sum(t.numel() * t.element_size() for t in outs_host.values())
        e2e_steps = max(3, min(args.steps, 20))
        # Two device buffer sets (step k uses set k % 2) and three streams: the
        # input copies of step k + 1 and the output copies of step k - 1 run
        # while step k computes, PCIe carrying both directions at once.  Every
        # step's own copies are inside the timed region.
        bufs = []
        for _ in range(2):
            xi = {k_: torch.empty_like(x[k_]) for k_ in in_keys + ["alpha", "rho"]}
            oi = {"o": torch.empty_like(o), "lse": torch.empty_like(lse)}
            if w.backward:
                oi.update(dq=torch.empty_like(dq), dk=torch.empty_like(dk), dv=torch.empty_like(dv))
            bufs.append((xi, oi))
        s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)

        def e2e_run(n, start_event=None):
            ev_in = [torch.cuda.Event() for _ in range(n)]
            ev_done = [torch.cuda.Event() for _ in range(n)]
            ev_out = [torch.cuda.Event() for _ in range(n)]
            for k_step in range(n):
                xi, oi = bufs[k_step % 2]
                with torch.cuda.stream(s_in):
                    if k_step == 0 and start_event is not None:
                        s_in.wait_event(start_event)
                    if k_step >= 2:
                        s_in.wait_event(ev_done[k_step - 2])  # that step has read this set's inputs
                    for k_ in in_keys + ["alpha", "rho"]:
                        xi[k_].copy_(host[k_], non_blocking=True)
                    ev_in[k_step].record(s_in)
                stream.wait_event(ev_in[k_step])
                if k_step >= 2:
                    stream.wait_event(ev_out[k_step - 2])  # this set's outputs have been copied out
                saf.mixed_attn_fwd(xi["q"], xi["k"], xi["v"], xi["alpha"], xi["rho"], mask, out=oi["o"],
                                   lse=oi["lse"], workspace=ws_f)
                if w.backward:
                    saf.mixed_attn_bwd(xi["q"], xi["k"], xi["v"], oi["o"], xi["do"], oi["lse"], xi["alpha"],
                                       xi["rho"], mask, grad_dtype=gd, dq=oi["dq"], dk=oi["dk"], dv=oi["dv"],
                                       workspace=ws_b)
                ev_done[k_step].record(stream)
                with torch.cuda.stream(s_out):
                    s_out.wait_event(ev_done[k_step])
                    for k_, t in outs_host.items():
                        t.copy_(oi[k_], non_blocking=True)
                    ev_out[k_step].record(s_out)
            stream.wait_event(ev_out[n - 1])

        e2e_run(2)
        torch.cuda.synchronize()
        barrier(world)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        e2e_run(e2e_steps, start_event=e0)
        e1.record(stream)
        torch.cuda.synchronize()
        barrier(world)
        e_ms = max_over_ranks(e0.elapsed_time(e1), world) / e2e_steps
        del bufs
        e2e = {"value": tokens / (e_ms * 1e-3), "unit": UNIT, "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h, "ms_per_step": e_ms}

    # ---- the pass split of the headline shape, the other shapes and the
    # per-head cost (separate timings after the headline; milliseconds each)
    split = rates(w, time_passes(w, dev, x, 20, gd), pk)
    extra, hc, sec = None, None, None
    if rank == 0 and not args.no_extra:
        extra = per_config(dev, pk)
        if w.backward and n_r:
            hc = head_cost_fit(w, dev)
        sec = secondary(w, dev, x)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(w)

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": max(args.warmup, 3), "ms_per_step": ms_step, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "tflops": tflops, "tflops_frac_of_peak": tflops / pk["bf16_tflops"],
            "tflops_strict": tflops_strict, "tflops_strict_frac_of_peak": tflops_strict / pk["bf16_tflops"],
            "config": arm_config(w, world, args.grad_dtype),
            "roofline": roofline, "kernels": kernels, "gpu_launches": launches,
            "clocks": clk.summary(), "e2e": e2e, "cpu_baseline": cpu,
            "passes": split, "per_config": extra, "head_cost": hc, "secondary": sec,
        }
        print(json.dumps(line), flush=True)


def head_cost(args, local):
    """Per-head cost of each head kind (the head_cost key of the headline
    line, printed alone)."""
    dev = torch.device("cuda", local)
    out = {"metric": "per-head cost of ordinary vs replaced heads (ms per head per step)"}
    out.update(head_cost_fit(I.WORKLOADS[args.workload], dev, reps=args.steps))
    print(json.dumps(out), flush=True)


def _time(fn, steps):
    for _ in range(3):
        fn()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    e0.record()
    for _ in range(steps):
        fn()
    e1.record()
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / steps


def pattern_grad_stats(w, x, reps):
    """Trainable-pattern gradient of w's replaced heads on the inputs x (on
    the device): ms per call (log Z given) and the dP contraction's
    algorithmic TFLOP/s (one causal T x T x d unit per replaced (b, h); the
    kernel runs it twice) against the bf16 peak."""
    from mixed_head_causal_b200 import saf
    mask = x["mask"]
    n_r = int(torch.as_tensor(mask).sum())
    lz = saf.replaced_lognorm(x["alpha"], x["rho"], mask)
    da = torch.empty(w.H, w.T, dtype=torch.float32, device=x["v"].device)
    dr = torch.empty_like(da)
    ms = _time(lambda: saf.replaced_pattern_grad(x["v"], x["do"], x["alpha"], x["rho"], mask, logz=lz, da=da,
                                                 dr=dr), reps)
    pk = peaks()
    tf = w.B * n_r * w.d * float(w.T) ** 2 / (ms * 1e-3) / 1e12
    return {"ms": ms, "n_replaced": n_r,
            "roofline": {"bound": "tensor", "achieved": tf, "peak": pk["bf16_tflops"], "unit": "TFLOP/s",
                         "frac": tf / pk["bf16_tflops"], "path": "warp-level mma.sync, two passes"}}


def calibration_stats(w, x, reps):
    """Calibration statistics over w's B sequences of q, k (every head taken
    as ordinary): ms per call and the score contraction's algorithmic TFLOP/s
    (one causal T x T x d unit per (sample, head); the kernel runs it twice)."""
    from mixed_head_causal_b200 import saf
    mask0 = torch.zeros(w.H, dtype=torch.bool)
    _, lse0 = saf.mixed_attn_fwd(x["q"], x["k"], x["v"], x["alpha"], x["rho"], mask0)
    a_hat = torch.empty(w.H, w.T, w.T, dtype=torch.float32, device=x["q"].device)
    svar = torch.empty(w.H, dtype=torch.float32, device=x["q"].device)
    ms = _time(lambda: saf.attn_calibration(x["q"], x["k"], lse0, a_hat=a_hat, svar=svar), reps)
    pk = peaks()
    tf = w.B * w.H * w.d * float(w.T) ** 2 / (ms * 1e-3) / 1e12
    del a_hat
    return {"ms": ms, "N": w.B,
            "roofline": {"bound": "tensor", "achieved": tf, "peak": pk["bf16_tflops"], "unit": "TFLOP/s",
                         "frac": tf / pk["bf16_tflops"], "path": "warp-level mma.sync, two passes",
                         "a_hat_bytes": 4 * w.H * w.T * w.T}}


def fit_stats(w, dev):
    """Pattern fitting (400 Adam steps) of w's replaced heads, the targets
    being their own patterns (dense [T, T] fp32, built on the GPU from the
    pattern vectors): ms per call and the final mean row KL of each head."""
    from mixed_head_causal_b200 import saf
    a, r = I.make_pattern(w, 0)
    heads = I.replaced_heads(w)
    T = w.T
    lz = saf.replaced_lognorm(a.to(dev), r.to(dev), I.replaced_mask(w, 0))
    targets = torch.zeros(len(heads), T, T, dtype=torch.float32, device=dev)
    i = torch.arange(T, device=dev)[:, None]
    j = torch.arange(T, device=dev)[None, :]
    for s_, h in enumerate(heads):
        ah, rh = a[h].to(dev), r[h].to(dev)
        for i0 in range(0, T, 512):
            ii = i[i0:i0 + 512]
            logit = ah[j.expand(ii.shape[0], T)] + rh[(ii - j).clamp(min=0)] - lz[h][ii]
            targets[s_, i0:i0 + 512] = torch.where(j <= ii, torch.exp(logit), torch.zeros((), device=dev))
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    _, _, kl = saf.fit_pattern(targets, steps=400, lr=0.1)
    e1.record()
    torch.cuda.synchronize()
    del targets
    return {"ms": e0.elapsed_time(e1), "heads": len(heads), "steps": 400, "kl": [float(v) for v in kl.cpu()]}


def secondary(w, dev, x, reps=10):
    """The entry points beside the layer (trainable-pattern gradient,
    calibration statistics, pattern fitting) timed on the headline shape."""
    out = {"workload": w.name}
    if w.backward and int(torch.as_tensor(x["mask"]).sum()):
        out["pattern_grad"] = pattern_grad_stats(w, x, reps)
        out["fit"] = fit_stats(w, dev)
    out["calibration"] = calibration_stats(w, x, reps)
    torch.cuda.empty_cache()
    return out


def pattern_grad_cost(args, local):
    """`--pattern-grad`: pattern_grad_stats on the workload's seeded inputs."""
    dev = torch.device("cuda", local)
    w = I.WORKLOADS[args.workload]
    x = {k: (v.to(dev) if k != "mask" else v) for k, v in I.make_inputs(w, 0, threads=16).items()}
    st = pattern_grad_stats(w, x, args.steps)
    print(json.dumps({"metric": "trainable-pattern gradient (dalpha, drho) ms per call", "value": st["ms"],
                      "unit": "ms", "higher_is_better": False,
                      "config": {"workload": w.name, "B": w.B, "H": w.H, "T": w.T, "n_replaced": st["n_replaced"]},
                      "roofline": st["roofline"]}), flush=True)


def calibration_cost(args, local):
    """`--calibration`: calibration_stats over the workload's B sequences."""
    dev = torch.device("cuda", local)
    base = I.WORKLOADS[args.workload]
    w = I.custom(base.B, base.H, base.T, [])
    x = {k: (v.to(dev) if k != "mask" else v) for k, v in I.make_inputs(w, 0, threads=16).items()}
    st = calibration_stats(w, x, args.steps)
    print(json.dumps({"metric": "calibration statistics (A_hat, s_var) ms per call", "value": st["ms"],
                      "unit": "ms", "higher_is_better": False,
                      "config": {"workload": w.name, "N": w.B, "H": w.H, "T": w.T}, "roofline": st["roofline"]}),
          flush=True)


def fit_cost(args, local):
    """`--fit`: fit_stats for the workload's replaced heads."""
    dev = torch.device("cuda", local)
    w = I.WORKLOADS[args.workload]
    t0 = time.perf_counter()
    st = fit_stats(w, dev)
    print(json.dumps({"metric": "pattern fitting, 400 Adam steps, ms per call", "value": st["ms"],
                      "unit": "ms", "higher_is_better": False,
                      "config": {"workload": w.name, "heads": st["heads"], "T": w.T},
                      "kl": st["kl"], "wall_s": time.perf_counter() - t0}), flush=True)


def gqa_cost(args, local):
    """Forward and backward with K/V shared by groups of H / H_kv query heads
    (the workload's shape and head mix): ms and tokens/s per pass."""
    from mixed_head_causal_b200 import saf
    dev = torch.device("cuda", local)
    w = I.WORKLOADS[args.workload]
    hkv = args.gqa
    if w.H % hkv:
        raise SystemExit("--gqa must divide H")
    x = {k: (v.to(dev) if k != "mask" else v) for k, v in I.make_inputs(w, 0, threads=16).items()}
    mask = x["mask"]
    k, v = x["k"][:, :hkv].contiguous(), x["v"][:, :hkv].contiguous()
    lz = saf.replaced_lognorm(x["alpha"], x["rho"], mask)
    o = torch.empty_like(x["q"])
    lse = torch.empty(w.B, w.H, w.T, dtype=torch.float32, device=dev)
    wsf = saf.new_workspace(w.B, w.H, w.T, dev, backward=False, h_kv=hkv)
    wsb = saf.new_workspace(w.B, w.H, w.T, dev, backward=True, h_kv=hkv)
    dq = torch.empty_like(x["q"])
    dk, dv = torch.empty_like(k), torch.empty_like(v)
    fwd = lambda: saf.mixed_attn_fwd(x["q"], k, v, x["alpha"], x["rho"], mask, logz=lz, out=o, lse=lse,  # noqa: E731
                                     workspace=wsf)
    bwd = lambda: saf.mixed_attn_bwd(x["q"], k, v, o, x["do"], lse, x["alpha"], x["rho"], mask, logz=lz,  # noqa: E731
                                     dq=dq, dk=dk, dv=dv, workspace=wsb)
    tf, tb = _time(fwd, args.steps), _time(bwd, args.steps)
    tokens = w.B * w.T
    print(json.dumps({"metric": "mixed-head causal attn with shared K/V heads, ms per pass", "unit": "ms",
                      "config": {"workload": w.name, "B": w.B, "H": w.H, "H_kv": hkv, "T": w.T},
                      "fwd_ms": tf, "bwd_ms": tb, "tokens_per_s": tokens / ((tf + tb) * 1e-3)}), flush=True)


def main():
    args = parse()
    world, rank, local = dist_setup(args)
    try:
        if args.head_cost:
            if rank == 0:
                head_cost(args, local)
        elif args.pattern_grad:
            if rank == 0:
                pattern_grad_cost(args, local)
        elif args.gqa:
            if rank == 0:
                gqa_cost(args, local)
        elif args.calibration:
            if rank == 0:
                calibration_cost(args, local)
        elif args.fit:
            if rank == 0:
                fit_cost(args, local)
        elif args.impl == "reference":
            reference_arm(args, world, rank)
        else:
            our_arm(args, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
