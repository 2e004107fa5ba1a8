"""Decode-step benchmark of the KIVI packed cache on B200.

One step = for every layer: append one token per sequence (with the residual
flush when due) and run the fused decode attention over the packed cache.
Prints ONE JSON line (rank 0).  `--impl reference` times the CPU oracle on the
host cores instead (bounded samples of the same workload).

Run: python bench.py [--gpus N --steps K --warmup W --workload NAME]
Under torchrun (N > 1) every rank holds its own batch (weak scaling, no
data-path collective); time = max over ranks.
"""
from __future__ import annotations

import argparse
import dataclasses
import hashlib
import json
import math
import os
import re
import statistics
import subprocess
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = ("decode-attention tokens/s and achieved HBM GB/s (% of B200 peak) on packed cache")
FALLBACK_HBM_GBS = 6650.0
DEFAULT_WORKLOAD = "llama3_8b_gqa_8k"
KERNEL_SOURCES = ["decode_attention_kivi_b200/csrc/kivi_attn.cu",
                  "decode_attention_kivi_b200/csrc/kivi_layout.cuh"]


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=64)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", default="kivi", choices=["kivi", "reference"])
    p.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(synth.WORKLOADS))
    p.add_argument("--batch", type=int, default=None, help="override the workload's batch")
    p.add_argument("--layers", type=int, default=None,
                   help="override the workload's layer count (small profiling captures)")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-e2e", action="store_true")
    return p.parse_args()


# ---------------------------------------------------------------------------
# Byte accounting (algorithmic bytes of one decode-attention call)
# ---------------------------------------------------------------------------

def record_bytes(D, bits):
    return 32 * D * bits // 4 + 8 * D


def attention_bytes(w: synth.Workload, S: int) -> int:
    """Group records + bf16 K/V residual + q (bf16) in + out (fp32) of one layer."""
    ng = 0 if S < 128 else (S - 128) // 32
    r = S - 32 * ng
    per_seq = ng * record_bytes(w.head_dim, w.bits) + r * w.head_dim * 4
    return (w.batch * w.num_kv_heads * per_seq
            + w.batch * w.num_q_heads * w.head_dim * (2 + 4))


def max_over_ranks(values, device) -> list:
    """Element-wise max of per-rank timings over the process group (any backend)."""
    t = torch.tensor(list(values), dtype=torch.float64, device=device)
    if torch.distributed.is_initialized() and torch.distributed.get_world_size() > 1:
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return [float(x) for x in t.cpu()]


def weak_scaling_tokens_per_s(world: int, batch: int, steps: int, ms: float) -> float:
    """Whole-job decode throughput: every rank decodes its own batch for `steps` steps."""
    return world * batch * steps / (ms * 1e-3)


def workload_config(w: synth.Workload, s_first: int, s_last: int, l2_note: str) -> dict:
    return {"workload": w.name, "batch_per_gpu": w.batch, "layers": w.num_layers,
            "kv_heads": w.num_kv_heads, "q_heads": w.num_q_heads, "head_dim": w.head_dim,
            "bits": w.bits, "group_size": 32, "residual": 128, "prefill_context": w.context,
            "context_at_timed_steps": [s_first, s_last], "l2": l2_note,
            "step": "per layer: kivi_append_token (flush when due) + kivi_decode_attention"}


def hbm_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_HBM_GBS, "fallback"


def _code_only(text: str) -> str:
    """C++ source without comments or layout: edits to either leave the hash alone."""
    text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
    text = re.sub(r"//[^\n]*", " ", text)
    return " ".join(text.split())


def kernel_hash() -> str:
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES:
        with open(os.path.join(ROOT, rel), encoding="utf-8") as f:
            h.update(_code_only(f.read()).encode())
    return h.hexdigest()[:16]


def recorded_traffic(w: synth.Workload):
    """ncu DRAM bytes per decode-attention launch, if recorded for this kernel source."""
    path = os.path.join(ROOT, "profiles", "decode_traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f)
    except (OSError, ValueError):
        return None
    entry = rec.get(w.name)
    if not entry or entry.get("kernel_hash") != kernel_hash():
        return None
    return entry.get("bytes_per_launch")


# ---------------------------------------------------------------------------
# Clock sampling during the timed region (a separate process: no GIL sharing)
# ---------------------------------------------------------------------------

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.device_index = device_index
        self.proc = None
        self.lines = []
        self.reader = None
        self.t_start = 0.0

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.monotonic(), line))

    def start(self):
        """Starts nvidia-smi and returns once it has printed its first sample, so that
        the (short) timed region that follows is sampled from its start."""
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.device_index}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "20"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self.reader = threading.Thread(target=self._read, daemon=True)
        self.reader.start()
        deadline = time.monotonic() + 5.0
        while not self.lines and self.proc.poll() is None and time.monotonic() < deadline:
            time.sleep(0.005)
        self.t_start = time.monotonic()

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            self.proc.wait()
        self.reader.join(timeout=5)
        timed = [line for t, line in self.lines if t >= self.t_start]
        out = "".join(timed if timed else [line for _, line in self.lines])
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
            except ValueError:
                continue
            for name, val in zip(names, parts[5:9]):
                if val.lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------------------
# The GPU arm
# ---------------------------------------------------------------------------

def build_cache(K, w: synth.Workload, max_tokens: int, device):
    cache = K.KiviCache(batch=w.batch, num_layers=w.num_layers, num_kv_heads=w.num_kv_heads,
                        num_q_heads=w.num_q_heads, head_dim=w.head_dim, bits=w.bits,
                        max_tokens=max_tokens, device=device)
    for layer in range(w.num_layers):
        k, v = synth.prefill_kv(w, layer, device=device)
        cache.prefill(layer, k, v)
        del k, v
    torch.cuda.synchronize()
    return cache


def run_gpu(args, w: synth.Workload, rank: int, world: int):
    import decode_attention_kivi_b200 as K
    from decode_attention_kivi_b200._native import lib

    device = torch.device("cuda", torch.cuda.current_device())
    steps, warmup = args.steps, args.warmup
    total_steps = warmup + steps + (0 if args.no_e2e else warmup + steps)
    cache = build_cache(K, w, w.context + total_steps + 1, device)
    L = lib()
    stream = torch.cuda.current_stream()
    sptr = stream.cuda_stream
    h = cache.handle
    # Step inputs resident in HBM (one set per layer, reused every step).
    q = [synth.query(w, l, 0, device=device) for l in range(w.num_layers)]
    kv = [synth.step_kv(w, l, 0, device=device) for l in range(w.num_layers)]
    out = torch.empty((w.num_layers, w.batch, w.num_q_heads, w.head_dim),
                      dtype=torch.float32, device=device)
    qp = [t.data_ptr() for t in q]
    kp = [a.data_ptr() for a, _ in kv]
    vp = [b.data_ptr() for _, b in kv]
    op = [out[l].data_ptr() for l in range(w.num_layers)]

    def check(rc, what):
        if rc != 0:
            raise RuntimeError(f"{what}: {K.kivi_status_string(rc)}")

    def step(ev=None):
        for l in range(w.num_layers):
            check(L.kivi_append_token(h, l, kp[l], vp[l], sptr), "append")
            if ev is not None:
                ev[l][0].record(stream)
            check(L.kivi_decode_attention(h, l, qp[l], op[l], 0.0, sptr), "attention")
            if ev is not None:
                ev[l][1].record(stream)

    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    s_first = cache.length(0)[0] + 1
    # per-launch events of the attention calls over the timed region
    evs = [[[torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)]
            for _ in range(w.num_layers)] for _ in range(steps)]
    bytes_timed = 0
    for i in range(steps):
        bytes_timed += w.num_layers * attention_bytes(w, s_first + i)
    sampler = ClockSampler(device.index if device.index is not None else 0)
    sampler.start()
    time.sleep(0.05)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    torch.cuda.nvtx.range_push("kivi_timed_steps")  # lets ncu --nvtx-include select these launches
    t0.record(stream)
    for i in range(steps):
        step(evs[i])
    t1.record(stream)
    torch.cuda.nvtx.range_pop()
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    clocks = sampler.stop()
    s_last = cache.length(0)[0]
    ms = t0.elapsed_time(t1)
    attn_ms = sum(e[0].elapsed_time(e[1]) for st in evs for e in st)
    n_attn = steps * w.num_layers
    # device status after the timed region (bounded waits report here)
    if cache.check_device_status() != 0:
        raise RuntimeError("a kernel reported a failure in the device status word")

    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(args, w, cache, L, h, sptr, device, world)

    if world > 1:
        ms, attn_ms = max_over_ranks([ms, attn_ms], device)
        if e2e is not None:
            e2e["_ms"] = max_over_ranks([e2e["_ms"]], device)[0]
    cache.close()
    return dict(ms=ms, attn_ms=attn_ms, n_attn=n_attn, bytes_timed=bytes_timed,
                s_first=s_first, s_last=s_last, clocks=clocks, e2e=e2e)


def run_e2e(args, w, cache, L, h, sptr, device, world):
    """Same steps through the C ABI with the step's inputs copied from pinned host
    memory and the step's outputs read back, copies inside the timed region."""
    nl = w.num_layers
    hq = [synth.query(w, l, 1).pin_memory() for l in range(nl)]
    hk = [synth.step_kv(w, l, 1)[0].pin_memory() for l in range(nl)]
    hv = [synth.step_kv(w, l, 1)[1].pin_memory() for l in range(nl)]
    hout = torch.empty((nl, w.batch, w.num_q_heads, w.head_dim), dtype=torch.float32).pin_memory()
    dq = [torch.empty_like(t, device=device) for t in hq]
    dk = [torch.empty_like(t, device=device) for t in hk]
    dv = [torch.empty_like(t, device=device) for t in hv]
    dout = torch.empty(hout.shape, dtype=torch.float32, device=device)
    h2d = sum(t.numel() * t.element_size() for t in hq + hk + hv)
    d2h = hout.numel() * hout.element_size()

    def step():
        for l in range(nl):
            dq[l].copy_(hq[l], non_blocking=True)
            dk[l].copy_(hk[l], non_blocking=True)
            dv[l].copy_(hv[l], non_blocking=True)
            rc = L.kivi_append_token(h, l, dk[l].data_ptr(), dv[l].data_ptr(), sptr)
            rc |= L.kivi_decode_attention(h, l, dq[l].data_ptr(), dout[l].data_ptr(), 0.0, sptr)
            if rc:
                raise RuntimeError("kivi call failed in the e2e loop")
        hout.copy_(dout, non_blocking=True)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    stream = torch.cuda.current_stream()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for _ in range(args.steps):
        step()
    t1.record(stream)
    torch.cuda.synchronize()
    assert torch.isfinite(hout).all()
    return {"_ms": t0.elapsed_time(t1), "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h}


# ---------------------------------------------------------------------------
# The oracle on the host cores (CPU baseline and the reference arm)
# ---------------------------------------------------------------------------

class OracleSample:
    """One layer of the workload in the oracle, at the prefill context."""

    def __init__(self, w: synth.Workload):
        import numpy as np

        import oracle as O

        self.np, self.O, self.w = np, O, w
        k, v = synth.prefill_kv(w, 0)
        self.cache = O.OracleCache(w.batch, w.num_kv_heads, w.head_dim, w.bits,
                                   w.context + 4096)
        self.cache.prefill(synth.bf16_bits(k), synth.bf16_bits(v))
        kn, vn = synth.step_kv(w, 0, 0)
        self.kn, self.vn = synth.bf16_bits(kn), synth.bf16_bits(vn)
        self.q = synth.bf16_bits(synth.query(w, 0, 0))
        self.rows = [(b, h) for b in range(w.batch) for h in range(w.num_q_heads)]

    def step_seconds(self, n_rows: int, start: int = 0) -> float:
        """Projected seconds of one full decode step from timing n_rows attention
        rows (of B*Hq) and one append of one layer, scaled to all rows and layers."""
        w = self.w
        t0 = time.perf_counter()
        self.cache.append(self.kn, self.vn)
        t_append = time.perf_counter() - t0
        t0 = time.perf_counter()
        for i in range(n_rows):
            b, hh = self.rows[(start + i) % len(self.rows)]
            self.cache.attend(b, hh, self.q[b, hh], w.num_q_heads)
        t_rows = time.perf_counter() - t0
        per_layer = t_append + t_rows * len(self.rows) / n_rows
        return per_layer * w.num_layers


def cpu_baseline(w: synth.Workload, budget_s: float = 12.0) -> dict:
    s = OracleSample(w)
    t_start = time.perf_counter()
    rows_done, proj = 0, []
    while time.perf_counter() - t_start < budget_s and rows_done < len(s.rows):
        n = 8
        proj.append(s.step_seconds(n, rows_done))
        rows_done += n
    step_s = statistics.median(proj)
    return {"value": w.batch / step_s, "unit": "tokens/s", "cores": 1, "kind": "oracle",
            "sample": (f"{rows_done} of {len(s.rows)} (sequence, query head) attention rows of "
                       f"layer 0 at S={w.context}+ plus one append per 8 rows, in "
                       f"{len(proj)} batches; scaled to all rows and {w.num_layers} layers; "
                       "single-threaded plain C oracle")}


def run_reference(args, w: synth.Workload):
    s = OracleSample(w)
    n = 8
    for i in range(args.warmup):
        s.step_seconds(n, i * n)
    total = 0.0
    for i in range(args.steps):
        total += s.step_seconds(n, (args.warmup + i) * n)
    value = w.batch * args.steps / total
    sample = (f"each step: {n} of {w.batch * w.num_q_heads} (sequence, query head) attention "
              f"rows of one layer plus one append, timed and scaled to all rows and "
              f"{w.num_layers} layers; single-threaded plain C oracle")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * total / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_config(w, w.context + 1, w.context + args.steps, "n/a (host)"),
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": 1, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------

def main():
    args = parse()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    w = synth.WORKLOADS[args.workload]
    if args.batch:
        w = w.with_batch(args.batch)
    if args.layers:
        w = dataclasses.replace(w, num_layers=args.layers)
    if args.impl == "reference":
        if rank == 0:
            run_reference(args, w)
        return
    if world > 1:
        import datetime

        local = int(os.environ.get("LOCAL_RANK", "0"))
        torch.cuda.set_device(local)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    res = run_gpu(args, w, rank, world)
    if rank == 0:
        peak, peak_kind = hbm_peak()
        gbs = res["bytes_timed"] / (res["attn_ms"] * 1e-3) / 1e9
        per_launch = res["bytes_timed"] / res["n_attn"]
        value = weak_scaling_tokens_per_s(world, w.batch, args.steps, res["ms"])
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": res["ms"] / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
            "data": "synthetic (seeded; shapes and key-outlier structure of the pages' models)",
            "config": workload_config(w, res["s_first"], res["s_last"],
                                      "inputs larger than L2: one step reads every layer's "
                                      f"cache ({w.num_layers} x ~{per_launch / 1e6:.0f} MB)"),
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": peak, "unit": "GB/s",
                         "frac": gbs / peak, "peak_kind": peak_kind,
                         "traffic": recorded_traffic(w),
                         "algorithmic_bytes_per_launch": per_launch,
                         "kernel": "kivi_decode_attention (split kernel + combine)",
                         "avg_launch_us": 1e3 * res["attn_ms"] / res["n_attn"]},
            "gpu_launches": 3 * w.num_layers * args.steps,
            "clocks": res["clocks"],
        }
        if res["e2e"] is not None:
            e = res["e2e"]
            line["e2e"] = {"value": weak_scaling_tokens_per_s(world, w.batch, args.steps, e["_ms"]),
                           "unit": "tokens/s", "h2d_bytes_per_step": e["h2d_bytes_per_step"],
                           "d2h_bytes_per_step": e["d2h_bytes_per_step"]}
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(w)
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
