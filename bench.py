#!/usr/bin/env python
"""Benchmark of the Condensate attention hot path on B200.

One step = one call of the library's public entry point for the workload
(decode: score pass + per-chunk Top-k + merge + gather/softmax; prefill:
score + Top-k pass + gather/softmax) over one batch of seeded synthetic
input already resident in device memory.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
    python bench.py --impl reference ...   # the CPU oracle on the host cores

With N > 1 (launched by torch.distributed.run) every rank runs an
independent replica of the workload on its own GPU ("replicas only": the
path has no exchange step); the step time is the maximum over ranks.
Prints one JSON line (rank 0).
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import workloads  # noqa: E402

METRIC = "decode ms @131K/1M ctx; prefill tokens/s; % of HBM / tensor roofline"
DEFAULT_WORKLOAD = "decode_131k"
FLUSH_BYTES = 256 << 20  # > 126 MB L2


def parse_args():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=20)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--workload", default=DEFAULT_WORKLOAD,
                   choices=sorted(workloads.WORKLOADS))
    p.add_argument("--no-cpu-baseline", action="store_true",
                   help="skip the CPU leg (oracle timing and parity)")
    p.add_argument("--no-also", action="store_true",
                   help="time only --workload, not the rest of the metric")
    return p.parse_args()


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        m = json.load(open(path))
        return {"hbm_gbs": m["hbm_gbs"], "bf16_tflops": m["bf16_tflops"],
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "source": "fallback"}


# ----------------------------------------------------------------- work model
def work_model(w):
    """Algorithmic work per launch of each kernel (see the design notes)."""
    es = 2 if w.dtype == "bf16" else 4
    if w.kind == "decode":
        L = w.n
        size = min(L, 1 + w.W + w.k)
        return {
            "decode_score_topk": ("hbm", w.B * w.Hkv * L * w.d * es,
                                  "K bytes scored: B*Hkv*L*d*elem"),
            "decode_merge_attend": ("hbm", w.B * w.Hq * size * 2 * w.d * es,
                                    "K and V rows of C_i: B*Hq*|C|*2*d*elem"),
        }
    n = w.n
    flops = w.B * w.Hq * w.d * n * (n + 1)
    return {
        "prefill_score_topk_tc": ("tensor", flops,
                                  "causal score FLOPs: B*H*d*n*(n+1)"),
        "prefill_score_topk_f32": ("alu", flops,
                                   "causal score FLOPs: B*H*d*n*(n+1)"),
        "prefill_gather": ("hbm", w.B * w.Hq * n * (w.d * es + w.k * 8 +
                                                     w.C_max * 4 + 4 + w.d * 4)
                           + 2 * w.B * w.Hkv * n * w.d * es,
                           "Q, K, V and Top-k keys read; idx, counts and fp32 O "
                           "written: B*H*n*(d*e + 8k + 4*C_max + 4 + 4d) + "
                           "2*B*Hkv*n*d*e"),
    }


def step_units(w):
    return w.B if w.kind == "decode" else w.B * w.n  # tokens per step


# ----------------------------------------------------------------- ranks
def max_over_ranks(values, device=None):
    """Maximum of each value over the ranks of the default process group: a
    replicated job is as slow as its slowest rank."""
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(v) for v in values], dtype=torch.float64,
                     device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.cpu()]


def job_rate(units_per_rank, world, ms):
    """Whole-job throughput: the units all ranks processed in one step over
    the slowest rank's step time (ms)."""
    return units_per_rank * world / (ms * 1e-3)


# The source files a kernel's code comes from (with every shared header).
KERNEL_SOURCES = {
    "decode_score_topk": ("decode_tc.cu", "decode.cu"),
    "decode_merge_attend": ("decode.cu",),
    "prefill_score_topk_tc": ("prefill_tc.cu",),
    "prefill_gather": ("prefill.cu",),
}


def _code_only(text):
    """Source text with C/C++ comments and layout removed, so that the hash
    below follows changes of the code only."""
    text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
    text = re.sub(r"//[^\n]*", " ", text)
    return " ".join(text.split())


def kernel_source_hash(kernel):
    csrc = os.path.join(ROOT, "sparse_transformer_attention_b200", "csrc")
    own = KERNEL_SOURCES.get(kernel)
    h = hashlib.sha256()
    for fn in sorted(os.listdir(csrc)):
        if fn.endswith(".cuh") or (fn.endswith(".cu") and
                                   (own is None or fn in own)):
            h.update(_code_only(open(os.path.join(csrc, fn)).read()).encode())
    return h.hexdigest()[:16]


def traffic_for(kernel, workload):
    """DRAM bytes per launch from a committed ncu capture, if it was taken on
    the current sources of that kernel; else None."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    try:
        t = json.load(open(path))
    except ValueError:
        return None
    e = t.get(f"{kernel}/{workload}")
    if not e or e.get("source_hash") != kernel_source_hash(kernel):
        return None
    return e.get("dram_bytes_per_launch")


# ----------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,"
              "clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, uuid):
        self.uuid = uuid
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}",
                   "--format=csv,noheader,nounits", "-lms", "200"]
            if self.uuid:
                cmd.insert(1, f"--id={self.uuid}")
            self.proc = subprocess.Popen(cmd, stdout=open(self.path, "w"),
                                         stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown",
                 "sw_power_cap"]
        for line in open(self.path):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for nm, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(nm)
        os.unlink(self.path)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": mx, "samples": len(sm),
                "reasons": sorted(reasons)}


# ----------------------------------------------------------------- ours
class L2Flush:
    """Empties the 126 MB L2 between steps: writes a 256 MiB buffer, then
    reads another 256 MiB buffer, so that the step starts with a cold L2 and
    without the write's dirty lines, whose write-back would otherwise land in
    the step's own memory traffic."""

    def __init__(self, dev):
        import torch
        self.w = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
        self.r = torch.zeros(FLUSH_BYTES // 4, dtype=torch.float32, device=dev)

    def zero_(self):
        self.w.zero_()
        self.r.sum()


ALSO = ("decode_1m", "prefill_gpt2s_8k", "prefill_adaptive_32k")


def config_of(w, world):
    return {"workload": w.name, "description": w.description,
            "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "d": w.d,
            ("L" if w.kind == "decode" else "n"): w.n, "W": w.W, "k": w.k,
            "adaptive_window": w.adaptive,
            "parallelism": f"replicas x{world}" if world > 1 else "1 GPU",
            "l2": "flushed before every step, outside the step's events: a "
                  "256 MiB write, then a 256 MiB read of another buffer (so "
                  "that the write's dirty lines are not written back inside "
                  "the step)"}


class Problem:
    """Device-resident inputs, outputs and workspace of one workload."""

    def __init__(self, w, dev):
        import torch
        import sparse_transformer_attention_b200 as ca
        self.w, self.dev = w, dev
        self.x = x = workloads.generate(w)
        tdt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
        to = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(dev).to(tdt)
        self.Q, self.K, self.V = to(x["Q"]), to(x["K"]), to(x["V"])
        self.W_i = None if x["W_i"] is None else \
            torch.from_numpy(x["W_i"]).to(dev)
        self.decode = w.kind == "decode"
        if self.decode:
            self.C_max = min(w.n, 1 + w.W_max + w.k)
            oshape = (w.B, w.Hq, w.d)
            ishape = (w.B, w.Hq)
        else:
            self.C_max = 1 + w.W_max + w.k
            oshape = (w.B, w.Hq, w.n, w.d)
            ishape = (w.B, w.Hq, w.n)
        self.O = torch.empty(oshape, dtype=torch.float32, device=dev)
        self.idx = torch.empty(ishape + (self.C_max,), dtype=torch.int32,
                               device=dev)
        self.cnt = torch.empty(ishape, dtype=torch.int32, device=dev)
        self.ws = torch.empty(ca.condensate_attn_workspace_size(
            self.decode, tdt, w.B, w.n, w.Hq, w.Hkv, w.d, w.W_max, w.k),
            dtype=torch.uint8, device=dev)
        self.fn = (ca.condensate_attn_decode if self.decode
                   else ca.condensate_attn_prefill)
        self.nvtx_name = ("condensate_attn_decode " if self.decode
                          else "condensate_attn_prefill ") + w.name

    def step(self, qin=None):
        import torch
        w = self.w
        # an NVTX range around each library call (seen by nsys / ncu's NVTX
        # filters; next to free without a tool attached)
        torch.cuda.nvtx.range_push(self.nvtx_name)
        try:
            self.fn(self.Q if qin is None else qin, self.K, self.V, w.W, w.k,
                    W_i=self.W_i, O=self.O, idx=self.idx, idx_count=self.cnt,
                    C_max=self.C_max, workspace=self.ws)
        finally:
            torch.cuda.nvtx.range_pop()

    def status(self):
        import sparse_transformer_attention_b200 as ca
        st = ca.condensate_attn_status(self.ws)
        if st != ca.CA_OK:
            raise RuntimeError(f"{self.w.name}: device status: "
                               f"{ca.status_string(st)}")


def timed_steps(p, steps, warmup, flush, dist=None, clocks=None):
    """Device time of each of `steps` steps (CUDA events on the launching
    stream), after at least `warmup` untimed ones; L2 flushed before every
    step.  The clock sampler runs from the start of the warm-up (which goes
    on for at least 0.6 s, so that the samples see the GPU under this load)
    to the end of the timed steps."""
    import torch
    if clocks:
        clocks.start()
    t_w = time.perf_counter()
    done = 0
    while done < warmup or time.perf_counter() - t_w < 0.6:
        flush.zero_()
        p.step()
        done += 1
        if done % 8 == 0:
            torch.cuda.synchronize()
    p.status()
    evs = [(torch.cuda.Event(enable_timing=True),
            torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    for s in range(steps):
        flush.zero_()  # L2 flush, outside the step's events
        evs[s][0].record()
        p.step()
        evs[s][1].record()
    torch.cuda.synchronize()
    wall = time.perf_counter() - t0
    clk = clocks.stop() if clocks else None
    if dist:
        dist.barrier()
    return [a.elapsed_time(b) for a, b in evs], wall, clk


def kernel_times(p, steps, flush):
    """Per-launch device times from the library's own events, in a separate
    pass: event records between the library's launches would otherwise
    serialise the dependent launch of the second kernel inside the timed
    steps."""
    import torch
    from sparse_transformer_attention_b200 import binding
    binding.profile_start(16 * steps + 16)
    for _ in range(steps):
        flush.zero_()
        p.step()
    torch.cuda.synchronize()
    prof = binding.profile_stop(16 * steps + 16)
    per = {}
    for name, t in prof:
        per.setdefault(name, []).append(t)
    return per, len(prof)


def roofline_of(w, per, pk, sm_max_mhz):
    """Roofline of the dominant kernel among those with a work model (the
    exact fallback for overflowing prefill rows has none: its work depends
    on the rows)."""
    model = work_model(w)
    kern_avg = {k_: statistics.mean(v) for k_, v in per.items()}
    dom = max((k_ for k_ in kern_avg if k_ in model),
              key=lambda k_: sum(per[k_]))
    bound, work, what = model[dom]
    t_dom = kern_avg[dom] * 1e-3
    if bound == "tensor":
        achieved = work / t_dom / 1e12
        peak, unit = pk["bf16_tflops"], "TFLOP/s"
    elif bound == "hbm":
        achieved = work / t_dom / 1e9
        peak, unit = pk["hbm_gbs"], "GB/s"
    else:
        achieved = work / t_dom / 1e12
        # fp32 FFMA peak: 148 SMs x 128 lanes x 2 FLOP x max SM clock
        peak = 148 * 128 * 2 * (sm_max_mhz or 1965.0) * 1e6 / 1e12
        unit = "TFLOP/s"
    return {"kernel": dom, "bound": bound, "achieved": achieved, "peak": peak,
            "unit": unit, "frac": achieved / peak,
            "peak_source": pk["source"] + (" burst" if bound != "alu" else
                                           " derived"),
            "work_per_launch": work, "work_definition": what,
            "avg_launch_ms": kern_avg[dom],
            "traffic": traffic_for(dom, w.name)}, kern_avg


def step_roofline_of(w, ms, pk):
    model = work_model(w)
    if w.kind == "decode":
        # whole-step HBM roofline: K scored + K/V rows of C_i gathered
        b = model["decode_score_topk"][1] + model["decode_merge_attend"][1]
        return {"bytes": b, "achieved_gbs": b / (ms * 1e-3) / 1e9,
                "frac": b / (ms * 1e-3) / 1e9 / pk["hbm_gbs"]}
    f = model["prefill_score_topk_tc"][1]
    t = f / (ms * 1e-3) / 1e12
    return {"flops": f, "achieved_tflops": t, "frac": t / pk["bf16_tflops"]}


def e2e_of(p, steps, flush):
    """The same metric through the public call with host buffers: every step
    copies its inputs from pinned host memory and reads the outputs back."""
    import torch
    w = p.w
    pin = lambda t: torch.empty(t.shape, dtype=t.dtype, pin_memory=True)
    if p.decode:
        q_host = pin(p.Q)
        q_host.copy_(p.Q.cpu())
        q_dev = torch.empty_like(p.Q)
        h2d = q_host.numel() * q_host.element_size()
    else:
        # prefill consumes Q, K and V of the step
        hosts = [pin(t) for t in (p.Q, p.K, p.V)]
        for h_, t_ in zip(hosts, (p.Q, p.K, p.V)):
            h_.copy_(t_.cpu())
        h2d = sum(h_.numel() * h_.element_size() for h_ in hosts)
    outs = [pin(p.O), pin(p.idx), pin(p.cnt)]
    d2h = sum(o.numel() * o.element_size() for o in outs)
    evs = [(torch.cuda.Event(enable_timing=True),
            torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    torch.cuda.synchronize()
    for s in range(steps):
        flush.zero_()
        evs[s][0].record()
        if p.decode:
            q_dev.copy_(q_host, non_blocking=True)
            p.step(q_dev)
        else:
            p.Q.copy_(hosts[0], non_blocking=True)
            p.K.copy_(hosts[1], non_blocking=True)
            p.V.copy_(hosts[2], non_blocking=True)
            p.step()
        for o_h, o_d in zip(outs, (p.O, p.idx, p.cnt)):
            o_h.copy_(o_d, non_blocking=True)
        evs[s][1].record()
    torch.cuda.synchronize()
    ms = statistics.mean(a.elapsed_time(b) for a, b in evs)
    return ms, h2d, d2h


def measure(w, dev, steps, warmup, flush, pk, uuid, dist=None, world=1):
    """Timed steps, clocks, per-kernel times and rooflines of one workload."""
    p = Problem(w, dev)
    step_ms, wall, clk = timed_steps(p, steps, warmup, flush, dist,
                                     ClockSampler(uuid))
    per, launches = kernel_times(p, steps, flush)
    p.status()
    ms = statistics.mean(step_ms)
    roof, kern_avg = roofline_of(w, per, pk, clk.get("sm_max_mhz"))
    rec = {"ms_per_step": ms, "tokens_per_s": job_rate(step_units(w), world, ms),
           "roofline": roof, "step_roofline": step_roofline_of(w, ms, pk),
           "kernels_avg_ms": kern_avg,
           "kernel_launches_per_step": launches / steps,
           "clocks": clk, "config": config_of(w, world)}
    return p, rec, step_ms, launches, wall


def run_ours(args, rank, world, local_rank):
    import torch

    dist = None
    if world > 1:
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    w = workloads.get(args.workload)
    pk = peaks()
    flush = L2Flush(dev)

    uuid = None
    try:
        uuid = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:
        pass

    p, rec, step_ms, launches, wall = measure(
        w, dev, args.steps, args.warmup, flush, pk, uuid, dist, world)
    e2e_ms, h2d, d2h = e2e_of(p, args.steps, flush)
    p.status()
    ms = rec["ms_per_step"]
    if dist:
        ms, e2e_ms = max_over_ranks([ms, e2e_ms], device=dev)
    # the rest of the metric, one workload at a time (one GPU only: every
    # rank of a replicated run would otherwise repeat them)
    also = {}
    if world == 1 and not args.no_also:
        headline = p
        for name in ALSO:
            if name == w.name:
                continue
            q, r, *_ = measure(workloads.get(name), dev, args.steps,
                               args.warmup, flush, pk, uuid)
            if rank == 0 and not args.no_cpu_baseline:
                r["parity"] = parity_of(q, sample_rows=2000)
            also[name] = r
            del q
            torch.cuda.empty_cache()
        p = headline

    decode = w.kind == "decode"
    rate = job_rate(step_units(w), world, ms)
    if decode:
        value, unit_v, hib = ms, "ms", False
        e2e_val, e2e_unit = e2e_ms, "ms"
    else:
        value, unit_v, hib = rate, "tokens/s", True
        e2e_val, e2e_unit = job_rate(step_units(w), world, e2e_ms), "tokens/s"
    out = {
        "metric": METRIC, "value": value, "unit": unit_v, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": hib, "scaling": "weak", "vs_baseline": None,
        "dtype": w.dtype, "data": "synthetic (seeded; see workloads/)",
        "config": config_of(w, world),
        "roofline": rec["roofline"],
        "step_roofline": step_roofline_of(w, ms, pk),
        "kernels_avg_ms": rec["kernels_avg_ms"],
        "tokens_per_s": rate,
        "e2e": {"value": e2e_val, "unit": e2e_unit,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "what": ("per-step query H2D (KV cache resident), call, "
                         "O/idx/count D2H" if decode else
                         "Q/K/V H2D, call, O/idx/count D2H")},
        "gpu_launches": launches,
        "clocks": rec["clocks"],
        "wall_s_timed_region": wall,
    }
    if rank == 0 and not args.no_cpu_baseline and world == 1:
        # the CPU leg: the oracle timed on a bounded sample, and the parity
        # of this run's last step against it
        out["cpu_baseline"] = cpu_baseline(w, p.x, budget_s=15.0)
        out["parity"] = parity_of(p, sample_rows=4000)
    if also:
        out["also"] = also
    if dist:
        dist.barrier()
        dist.destroy_process_group()
    return out


def parity_of(p, sample_rows):
    """Rows of the last step compared with the oracle: index sets identical
    outside near-ties (swaps inside the rounding bound), outputs within the
    tolerance.  Decode: every (batch, q-head); prefill: a seeded sample of
    rows plus every row the selector sent to its exact fallback."""
    import oracle
    from oracle.parity import check_rows
    w, x = p.w, p.x
    tol = 1e-2 if w.dtype == "bf16" else 1e-5
    G = w.Hq // w.Hkv
    try:
        if p.decode:
            ref = oracle.decode(x["Q"], x["K"], x["V"], w.W, w.k,
                                W_i=x["W_i"], C_max=p.C_max, with_full=False)
            rows = [(b, h) for b in range(w.B) for h in range(w.Hq)]
            win = [int(x["W_i"][b]) if x["W_i"] is not None else w.W
                   for (b, h) in rows]
            r = check_rows(
                ref, p.idx.cpu().numpy(), p.cnt.cpu().numpy(),
                p.O.float().cpu().numpy(),
                q_rows=[x["Q"][b, h] for (b, h) in rows],
                kv_rows=lambda i: x["K"][rows[i][0], rows[i][1] // G],
                v_rows=lambda i: x["V"][rows[i][0], rows[i][1] // G],
                pos=[w.n - 1] * len(rows), win=win, tol=tol)
            r["what"] = "every (batch, q-head) row"
            return r
        import torch
        rng = np.random.default_rng(0)
        sel = np.stack([rng.integers(w.B, size=sample_rows),
                        rng.integers(w.Hq, size=sample_rows),
                        rng.integers(w.n, size=sample_rows)], 1)
        R = w.B * w.Hq * w.n
        nfb = int(p.ws[16:20].cpu().numpy().view(np.uint32)[0])
        off = 256 + (R * max(w.k, 1) * 8 + 255) // 256 * 256
        fb = p.ws[off:off + 4 * nfb].cpu().numpy().view(np.uint32)
        bh, i_ = np.divmod(fb.astype(np.int64), w.n)
        fb = np.stack([bh // w.Hq, bh % w.Hq, i_], 1)
        sel = np.unique(np.concatenate([sel, fb.reshape(-1, 3)]), axis=0)
        ti = torch.from_numpy(sel).to(p.dev)
        g_idx = p.idx[ti[:, 0], ti[:, 1], ti[:, 2]].cpu().numpy()
        g_cnt = p.cnt[ti[:, 0], ti[:, 1], ti[:, 2]].cpu().numpy()
        g_o = p.O[ti[:, 0], ti[:, 1], ti[:, 2]].float().cpu().numpy()
        ref = oracle.prefill(x["Q"], x["K"], x["V"], w.W, w.k, W_i=x["W_i"],
                             sel=sel, C_max=p.C_max, with_full=False)
        win = [int(x["W_i"][b, i]) if x["W_i"] is not None else w.W
               for (b, h, i) in sel]
        r = check_rows(
            ref, g_idx, g_cnt, g_o,
            q_rows=[x["Q"][b, h, i] for (b, h, i) in sel],
            kv_rows=lambda i: x["K"][sel[i][0], sel[i][1] // G],
            v_rows=lambda i: x["V"][sel[i][0], sel[i][1] // G],
            pos=sel[:, 2], win=win, tol=tol)
        r["what"] = (f"{sample_rows} seeded sample rows + {nfb} exact-"
                     f"fallback rows")
        return r
    except AssertionError as e:
        return {"failed": str(e)[:300]}


# ----------------------------------------------------------------- oracle
def cpu_baseline(w, x, budget_s=15.0, seed=0):
    """Time the CPU oracle, as it stands, on a bounded sample of the workload."""
    import oracle
    threads = oracle.max_threads()
    if w.kind == "decode":
        t0 = time.perf_counter()
        reps = 0
        while True:
            oracle.decode(x["Q"], x["K"], x["V"], w.W, w.k, W_i=x["W_i"],
                          C_max=min(w.n, w.C_max), with_full=False)
            reps += 1
            if time.perf_counter() - t0 > budget_s or reps >= 5:
                break
        per = (time.perf_counter() - t0) / reps
        return {"value": per * 1e3, "unit": "ms", "cores": threads,
                "kind": "oracle",
                "sample": f"{reps} full decode step(s) of {w.name} "
                          f"(all {w.B * w.Hq} q-heads, L={w.n})"}
    rng = np.random.default_rng(seed)
    R = w.B * w.Hq * w.n
    done, rows_total, t_total = 0, 0, 0.0
    batch = 64
    while t_total < budget_s and rows_total < R:
        sel = np.stack([rng.integers(w.B, size=batch),
                        rng.integers(w.Hq, size=batch),
                        rng.integers(w.n, size=batch)], 1)
        t0 = time.perf_counter()
        oracle.prefill(x["Q"], x["K"], x["V"], w.W, w.k, W_i=x["W_i"],
                       sel=sel, C_max=w.C_max, with_full=False)
        t_total += time.perf_counter() - t0
        rows_total += batch
        done += 1
    per_row = t_total / rows_total
    return {"value": 1.0 / per_row, "unit": "tokens/s", "cores": threads,
            "kind": "oracle",
            "sample": f"{rows_total} uniformly drawn query rows of {w.name}; "
                      f"rate extrapolated per row"}


def run_reference(args):
    w = workloads.get(args.workload)
    x = workloads.generate(w)
    vals = []
    for s in range(args.warmup + args.steps):
        cb = cpu_baseline(w, x, budget_s=2.0, seed=s)
        if s >= args.warmup:
            vals.append(cb["value"])
    v = statistics.mean(vals)
    decode = w.kind == "decode"
    cb["value"] = v
    return {
        "impl": "reference", "metric": METRIC, "value": v, "unit": cb["unit"],
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": v if decode else None,
        "higher_is_better": not decode, "scaling": "weak",
        "vs_baseline": None, "dtype": w.dtype,
        "data": "synthetic (seeded; see workloads/)",
        "config": config_of(w, args.gpus),
        "cpu_baseline": cb,
        "e2e": {"value": v, "unit": cb["unit"], "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def main():
    args = parse_args()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        if rank != 0:
            return 0
        print(json.dumps(run_reference(args)), flush=True)
        return 0
    out = run_ours(args, rank, world, local_rank)
    if rank == 0:
        print(json.dumps(out), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
