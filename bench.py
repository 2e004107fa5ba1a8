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
FALLBACK_BF16_TFLOPS = 1590.0
DEFAULT_WORKLOAD = "llama3_8b_gqa_8k"
KERNEL_SOURCES = ["decode_attention_kivi_b200/csrc/kivi_attn.cu",
                  "decode_attention_kivi_b200/csrc/kivi_layout.cuh",
                  "decode_attention_kivi_b200/csrc/kivi_ptx.cuh"]


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
    p.add_argument("--sweep", choices=["memory-wall", "key-granularity", "prefill"], default=None,
                   help="memory-wall: decode attention of the 2-bit cache and of a bf16 cache "
                        "over growing batches of the Llama-2-13B MHA 4K shape, until a cache "
                        "no longer fits (one JSON line)")
    p.add_argument("--sweep-batches", default="16,32,48,53,64,96,128,160,192,224,240,256")
    p.add_argument("--prefill-batches", default="1,4,16",
                   help="prefill sweep: batches of 8K prompts of one Llama-3-8B GQA layer")
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


def flush_steps(context: int, first: int, count: int) -> list:
    """Indices i in [first, first + count) of the decode steps (step i appends token
    context + i) whose append flushes 32 residual tokens into a new group: the
    residual would reach R + G = 160 tokens."""
    out = []
    for i in range(first, first + count):
        S = context + i
        ng = 0 if S < 128 else (S - 128) // 32
        if S + 1 - 32 * ng == 160:
            out.append(i)
    return out


def timed_window(context: int, warmup: int, steps: int) -> int:
    """Untimed steps before the timed window: at least `warmup`, chosen so that the
    window of `steps` steps holds a residual flush as near its middle as possible (a
    flush comes every 32 steps)."""
    best, best_d = warmup, None
    for pre in range(warmup, warmup + 32):
        fl = flush_steps(context, pre, steps)
        if not fl:
            continue
        d = min(abs(f - (pre + steps // 2)) for f in fl)
        if best_d is None or d < best_d:
            best, best_d = pre, d
    return best


def workload_config(w: synth.Workload, warmup: int, steps: int) -> dict:
    """The workload and the timed window, identical in both arms."""
    pre = timed_window(w.context, warmup, steps)
    return {"workload": w.name, "batch_per_gpu": w.batch, "layers": w.num_layers,
            "kv_heads": w.num_kv_heads, "q_heads": w.num_q_heads, "head_dim": w.head_dim,
            "bits": w.bits, "group_size": 32, "residual": 128, "prefill_context": w.context,
            "untimed_steps_before_window": pre,
            "context_at_timed_steps": [w.context + pre + 1, w.context + pre + steps],
            "residual_flushes_in_window": len(flush_steps(w.context, pre, steps)),
            "step": "per layer: kivi_append_token (flush when due) + kivi_decode_attention"}


def percentiles(xs) -> dict:
    ys = sorted(xs)
    pick = lambda f: ys[min(len(ys) - 1, max(0, int(round(f * (len(ys) - 1)))))]
    return {"median": statistics.median(ys), "p10": pick(0.10), "p90": pick(0.90),
            "mean": sum(ys) / len(ys), "n": len(ys)}


def tensor_peak():
    """Dense bf16 tensor peak (TFLOP/s) for a kernel timed alone: the measured burst."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["bf16_tflops"]), "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_BF16_TFLOPS, "fallback"


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


L2_FLUSH_BYTES = 512 << 20  # more than 4x B200's 126 MB L2


def run_gpu(args, w: synth.Workload, cfg: dict, rank: int, world: int):
    import decode_attention_kivi_b200 as K
    from decode_attention_kivi_b200._native import lib

    device = torch.device("cuda", torch.cuda.current_device())
    steps = args.steps
    pre = cfg["untimed_steps_before_window"]
    e2e_steps = 0 if args.no_e2e else args.warmup + steps
    cache = build_cache(K, w, w.context + pre + steps + e2e_steps + 1, device)
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
    # One step reads every layer's cache; when that is not far above L2, a buffer
    # larger than L2 is written between timed steps (outside their events).
    step_bytes = w.num_layers * attention_bytes(w, w.context + pre)
    flush_l2 = step_bytes < 4 * 126e6
    scratch = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=device) if flush_l2 else None

    def check(rc, what):
        if rc != 0:
            raise RuntimeError(f"{what}: {K.kivi_status_string(rc)}")

    # One step: the appends of every layer, then the decode attention of every
    # layer, each as one burst of back-to-back launches (the layers are
    # independent, so the order changes no result).  One event pair brackets each
    # decode burst: events between the launches would break the programmatic
    # dependent launch chain and add several microseconds to every call.
    def step(ev=None):
        for l in range(w.num_layers):
            check(L.kivi_append_token(h, l, kp[l], vp[l], sptr), "append")
        if ev is not None:
            ev[0].record(stream)
        for l in range(w.num_layers):
            check(L.kivi_decode_attention(h, l, qp[l], op[l], 0.0, sptr), "attention")
        if ev is not None:
            ev[1].record(stream)

    for _ in range(pre):
        step()
    torch.cuda.synchronize()
    s_first = cache.length(0)[0] + 1
    new = lambda: torch.cuda.Event(enable_timing=True)
    evs = [[new(), new()] for _ in range(steps)]  # the decode burst of each step
    st_ev = [[new(), new()] for _ in range(steps)]
    bytes_timed = sum(w.num_layers * attention_bytes(w, s_first + i) for i in range(steps))
    sampler = ClockSampler(device.index if device.index is not None else 0)
    sampler.start()
    time.sleep(0.05)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    t0, t1 = new(), new()
    torch.cuda.nvtx.range_push("kivi_timed_steps")  # lets ncu --nvtx-include select these launches
    t0.record(stream)
    for i in range(steps):
        if scratch is not None:
            scratch.zero_()
        st_ev[i][0].record(stream)
        step(evs[i])
        st_ev[i][1].record(stream)
    t1.record(stream)
    torch.cuda.nvtx.range_pop()
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    clocks = sampler.stop()
    s_last = cache.length(0)[0]
    ms = (sum(a.elapsed_time(b) for a, b in st_ev) if flush_l2 else t0.elapsed_time(t1))
    # average decode-attention launch of each step's burst (one value per step)
    call_us = [1e3 * a.elapsed_time(b) / w.num_layers for a, b in evs]
    attn_ms = 1e-3 * sum(call_us) * w.num_layers
    # device status after the timed region (bounded waits report here)
    if cache.check_device_status() != 0:
        raise RuntimeError("a kernel reported a failure in the device status word")
    del scratch

    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(args, w, cache, L, h, sptr, device, world)

    if world > 1:
        ms, attn_ms = max_over_ranks([ms, attn_ms], device)
        if e2e is not None:
            e2e["_ms"] = max_over_ranks([e2e["_ms"]], device)[0]
    cache.close()
    return dict(ms=ms, attn_ms=attn_ms, call_us=call_us, bytes_timed=bytes_timed,
                s_first=s_first, s_last=s_last, clocks=clocks, e2e=e2e, flush_l2=flush_l2,
                step_bytes=step_bytes)


def run_e2e(args, w, cache, L, h, sptr, device, world):
    """Same steps through the C ABI with the step's inputs copied from pinned host
    memory and the step's outputs read back, copies inside the timed region.  The
    copies run on their own stream with two device buffer sets, ordered by events
    once per step: step i+1's inputs arrive and step i's outputs leave while step
    i computes; the launches of a step stay back to back."""
    nl = w.num_layers
    hq = torch.stack([synth.query(w, l, 1) for l in range(nl)]).pin_memory()
    hk = torch.stack([synth.step_kv(w, l, 1)[0] for l in range(nl)]).pin_memory()
    hv = torch.stack([synth.step_kv(w, l, 1)[1] for l in range(nl)]).pin_memory()
    hout = torch.empty((nl, w.batch, w.num_q_heads, w.head_dim), dtype=torch.float32).pin_memory()
    dq = [torch.empty_like(hq, device=device) for _ in range(2)]
    dk = [torch.empty_like(hk, device=device) for _ in range(2)]
    dv = [torch.empty_like(hv, device=device) for _ in range(2)]
    dout = [torch.empty(hout.shape, dtype=torch.float32, device=device) for _ in range(2)]
    h2d = sum(t.numel() * t.element_size() for t in (hq, hk, hv))
    d2h = hout.numel() * hout.element_size()
    comp = torch.cuda.current_stream()
    copy = torch.cuda.Stream(device=device)
    inputs_in = [torch.cuda.Event() for _ in range(2)]
    step_done = [torch.cuda.Event() for _ in range(2)]
    out_read = [torch.cuda.Event() for _ in range(2)]
    used = [False, False]
    n = [0]

    def step():
        j = n[0] % 2
        with torch.cuda.stream(copy):
            if used[j]:
                copy.wait_event(step_done[j])  # step i-2 is done with buffer set j
            dq[j].copy_(hq, non_blocking=True)
            dk[j].copy_(hk, non_blocking=True)
            dv[j].copy_(hv, non_blocking=True)
            inputs_in[j].record(copy)
        comp.wait_event(inputs_in[j])
        if used[j]:
            comp.wait_event(out_read[j])  # step i-2's outputs have left buffer set j
        rc = 0
        for l in range(nl):
            rc |= L.kivi_append_token(h, l, dk[j][l].data_ptr(), dv[j][l].data_ptr(), sptr)
        for l in range(nl):
            rc |= L.kivi_decode_attention(h, l, dq[j][l].data_ptr(), dout[j][l].data_ptr(), 0.0,
                                          sptr)
        if rc:
            raise RuntimeError("kivi call failed in the e2e loop")
        step_done[j].record(comp)
        with torch.cuda.stream(copy):
            copy.wait_event(step_done[j])
            hout.copy_(dout[j], non_blocking=True)
            out_read[j].record(copy)
        used[j] = True
        n[0] += 1

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(comp)
    copy.wait_stream(comp)  # no copy of the timed steps starts before t0
    for _ in range(args.steps):
        step()
    comp.wait_stream(copy)  # the last step's outputs are on the host
    t1.record(comp)
    torch.cuda.synchronize()
    assert torch.isfinite(hout).all()
    return {"_ms": t0.elapsed_time(t1), "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h}


# ---------------------------------------------------------------------------
# The oracle on the host cores (CPU baseline and the reference arm)
# ---------------------------------------------------------------------------

def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


class OracleSample:
    """One layer of the workload in the oracle, at the prefill context."""

    def __init__(self, w: synth.Workload):
        import oracle as O

        self.O, self.w = O, w
        k, v = synth.prefill_kv(w, 0)
        self.cache = O.OracleCache(w.batch, w.num_kv_heads, w.head_dim, w.bits,
                                   w.context + 4096)
        self.cache.prefill(synth.bf16_bits(k), synth.bf16_bits(v))
        kn, vn = synth.step_kv(w, 0, 0)
        self.kn, self.vn = synth.bf16_bits(kn), synth.bf16_bits(vn)
        self.q = synth.bf16_bits(synth.query(w, 0, 0))
        self.rows = [(b, h) for b in range(w.batch) for h in range(w.num_q_heads)]
        self.next = 0

    def time_rows(self, n_rows: int):
        """Seconds for one append of the layer and n_rows attention rows."""
        t0 = time.perf_counter()
        self.cache.append(self.kn, self.vn)
        t_append = time.perf_counter() - t0
        t0 = time.perf_counter()
        for _ in range(n_rows):
            b, hh = self.rows[self.next % len(self.rows)]
            self.next += 1
            self.cache.attend(b, hh, self.q[b, hh], self.w.num_q_heads)
        return t_append, time.perf_counter() - t0


_WORKER_SAMPLE = None


def _oracle_worker_init(name, batch, layers, worker_index):
    global _WORKER_SAMPLE
    w = dataclasses.replace(synth.WORKLOADS[name], batch=batch, num_layers=layers)
    _WORKER_SAMPLE = OracleSample(w)
    _WORKER_SAMPLE.next = worker_index * 7


def _oracle_worker_rows(n_rows):
    return _WORKER_SAMPLE.time_rows(n_rows)


class OracleTimer:
    """The plain C oracle on the host: single-threaded in this process, and one
    worker process per core (spawned, no CUDA) timing rows side by side."""

    def __init__(self, w: synth.Workload, workers: int):
        import multiprocessing as mp

        self.w = w
        self.rows_per_step = w.num_layers * w.batch * w.num_q_heads
        self.workers = workers
        self.pool = None
        if workers > 1:
            ctx = mp.get_context("spawn")
            # one pool of `workers` processes, each holding its own oracle copy
            self.pool = ctx.Pool(workers, initializer=_oracle_worker_init,
                                 initargs=(w.name, w.batch, w.num_layers, 0))
            self.pool.map(_oracle_worker_rows, [1] * workers)  # builds the copies

    def all_cores(self, rows_each: int) -> dict:
        """Rows/s with every worker timing rows_each rows at once (wall clock)."""
        t0 = time.perf_counter()
        res = self.pool.map(_oracle_worker_rows, [rows_each] * self.workers, chunksize=1)
        wall = time.perf_counter() - t0
        rows = rows_each * self.workers
        return {"rows": rows, "seconds": wall, "rows_per_s": rows / wall,
                "append_s": max(a for a, _ in res)}

    def close(self):
        if self.pool is not None:
            self.pool.close()
            self.pool.join()


def _projection(w, rows_per_s):
    rows_per_step = w.num_layers * w.batch * w.num_q_heads
    step_s = rows_per_step / rows_per_s
    return step_s, w.batch / step_s


def cpu_baseline(w: synth.Workload, budget_s: float = 20.0) -> dict:
    """The oracle as it stands, on a bounded sample of the workload: attention rows
    (sequence, query head) of one layer at the prefill context, timed and projected
    to a full decode step (every row of every layer)."""
    workers = os.cpu_count() or 1
    single = OracleSample(w)
    t_start = time.perf_counter()
    rows1, sec1 = 0, 0.0
    while time.perf_counter() - t_start < 0.3 * budget_s:
        _, t = single.time_rows(4)
        rows1 += 4
        sec1 += t
    timer = OracleTimer(w, workers)
    try:
        done, sec, rows = 0, 0.0, 0
        t_start = time.perf_counter()
        while time.perf_counter() - t_start < 0.5 * budget_s:
            r = timer.all_cores(2)
            rows += r["rows"]
            sec += r["seconds"]
    finally:
        timer.close()
    rate = rows / sec if workers > 1 else rows1 / sec1
    step_s, value = _projection(w, rate)
    step1_s, value1 = _projection(w, rows1 / sec1)
    return {"value": value, "unit": "tokens/s", "cores": workers, "threads": workers,
            "cpu_model": cpu_model(), "kind": "oracle", "projected": True,
            "rows_measured": rows, "rows_per_s": rate,
            "rows_per_step": timer.rows_per_step,
            "scale_factor": timer.rows_per_step / max(rows, 1),
            "single_thread": {"value": value1, "rows_measured": rows1,
                              "rows_per_s": rows1 / sec1},
            "sample": (f"{rows} attention rows (sequence, query head) of layer 0 at S="
                       f"{w.context}+, {workers} worker processes side by side (one per "
                       f"core, {cpu_model()}); a full decode step is "
                       f"{timer.rows_per_step} rows ({w.num_layers} layers), so the "
                       f"figure is projected from the measured rows/s; plain C oracle, "
                       "fp64 accumulation")}


def run_reference(args, w: synth.Workload, cfg: dict):
    workers = os.cpu_count() or 1
    timer = OracleTimer(w, workers) if workers > 1 else None
    single = OracleSample(w) if workers == 1 else None
    rows_each = 2
    try:
        def one_step():
            if timer is not None:
                r = timer.all_cores(rows_each)
                return r["rows"], r["seconds"]
            _, t = single.time_rows(rows_each)
            return rows_each, t
        for _ in range(args.warmup):
            one_step()
        rows, sec = 0, 0.0
        for _ in range(args.steps):
            r, t = one_step()
            rows += r
            sec += t
    finally:
        if timer is not None:
            timer.close()
    rate = rows / sec
    step_s, value = _projection(w, rate)
    rows_per_step = w.num_layers * w.batch * w.num_q_heads
    sample = (f"each step: {rows_each * workers} of the {rows_per_step} attention rows "
              f"(sequence, query head) of a decode step, {workers} worker processes side by "
              f"side (one per core, {cpu_model()}), timed and projected to the full step; "
              "plain C oracle, fp64 accumulation")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * step_s, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": cfg, "projected": True,
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": workers,
                             "threads": workers, "cpu_model": cpu_model(), "kind": "oracle",
                             "projected": True, "rows_measured": rows, "rows_per_s": rate,
                             "rows_per_step": rows_per_step,
                             "scale_factor": rows_per_step * args.steps / rows,
                             "sample": sample},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------

# ---------------------------------------------------------------------------
# Memory-wall sweep: the 2-bit cache against a bf16 cache as the batch grows
# ---------------------------------------------------------------------------

def bf16_attention_bytes(B, H, Hq, D, S) -> int:
    """bf16 K and V of S tokens + q in (bf16) + out (fp32), one layer."""
    return B * H * S * D * 4 + B * Hq * D * (2 + 4)


def _time_layers(call, layers, warmup=3, steps=10):
    """Per-step device time (ms) of `call(layer)` over all layers; median of steps."""
    stream = torch.cuda.current_stream()
    for _ in range(warmup):
        for l in range(layers):
            call(l)
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(steps)]
    for a, b in ev:
        a.record(stream)
        for l in range(layers):
            call(l)
        b.record(stream)
    torch.cuda.synchronize()
    return statistics.median(a.elapsed_time(b) for a, b in ev)


def _sweep_kivi(K, w, B, S, device, peak):
    cfg = K.make_config(batch=B, num_layers=w.num_layers, num_kv_heads=w.num_kv_heads,
                        num_q_heads=w.num_q_heads, head_dim=w.head_dim, bits=w.bits,
                        max_tokens=S)
    need = sum(getattr(K.kivi_required_bytes(cfg), f) for f in
               ("records_bytes", "resid_k_bytes", "resid_v_bytes", "workspace_bytes"))
    free = torch.cuda.mem_get_info()[0]
    entry = {"impl": "kivi-2bit", "batch": B, "cache_gb": need / 1e9}
    if need > free - (2 << 30):
        return dict(entry, fits=False, free_gb=free / 1e9)
    cache = K.KiviCache(batch=B, num_layers=w.num_layers, num_kv_heads=w.num_kv_heads,
                        num_q_heads=w.num_q_heads, head_dim=w.head_dim, bits=w.bits,
                        max_tokens=S, device=device)
    # fill: a short prefill, then appends (no full-context staging buffer, so the
    # cache alone has to fit); tokens cycle through a small seeded pool
    wb = w.with_batch(B)
    S0 = 160
    pool = [synth.step_kv(wb, 0, i, device=device) for i in range(8)]
    for l in range(w.num_layers):
        k, v = synth.prefill_kv(wb, l, S=S0, device=device)
        cache.prefill(l, k, v)
        for t in range(S0, S):
            kn, vn = pool[t % len(pool)]
            cache.append(l, kn, vn)
    q = [synth.query(wb, l, 0, device=device) for l in range(w.num_layers)]
    out = torch.empty((B, w.num_q_heads, w.head_dim), dtype=torch.float32, device=device)
    ms = _time_layers(lambda l: cache.attend(l, q[l], out), w.num_layers)
    assert cache.check_device_status() == 0
    cache.close()
    del cache
    nbytes = w.num_layers * attention_bytes(wb, S)
    gbs = nbytes / (ms * 1e-3) / 1e9
    return dict(entry, fits=True, ms_per_step=ms, tokens_per_s=B / (ms * 1e-3),
                gbs=gbs, frac_of_peak=gbs / peak)


def _sweep_bf16(K, w, B, S, device, peak):
    H, Hq, D, L = w.num_kv_heads, w.num_q_heads, w.head_dim, w.num_layers
    Smax = S
    need = 2 * L * B * H * Smax * D * 2
    free = torch.cuda.mem_get_info()[0]
    entry = {"impl": "bf16", "batch": B, "cache_gb": need / 1e9}
    if need > free - (2 << 30):
        return dict(entry, fits=False, free_gb=free / 1e9)
    kc = torch.empty((L, B, H, Smax, D), dtype=torch.bfloat16, device=device)
    vc = torch.empty_like(kc)
    gen = torch.Generator(device=device).manual_seed(synth.BASE_SEED + 100 + B)
    for l in range(L):
        kc[l].normal_(generator=gen)
        vc[l].normal_(generator=gen)
    wb = w.with_batch(B)
    q = [synth.query(wb, l, 0, device=device) for l in range(L)]
    att = K.Bf16Attention(batch=B, num_kv_heads=H, num_q_heads=Hq, head_dim=D, device=device)
    out = torch.empty((B, Hq, D), dtype=torch.float32, device=device)
    ms = _time_layers(lambda l: att.attend(kc[l], vc[l], S, q[l], out), L)
    assert att.check_device_status() == 0
    del kc, vc
    torch.cuda.empty_cache()
    gbs = L * bf16_attention_bytes(B, H, Hq, D, S) / (ms * 1e-3) / 1e9
    return dict(entry, fits=True, ms_per_step=ms, tokens_per_s=B / (ms * 1e-3),
                gbs=gbs, frac_of_peak=gbs / peak)


def run_memory_wall(args):
    import decode_attention_kivi_b200 as K

    device = torch.device("cuda", torch.cuda.current_device())
    w = synth.WORKLOADS["llama2_13b_mha_sweep"]
    S = w.context + 1
    peak, peak_kind = hbm_peak()
    rows = []
    for impl, fn in (("bf16", _sweep_bf16), ("kivi-2bit", _sweep_kivi)):
        for B in [int(x) for x in args.sweep_batches.split(",")]:
            r = fn(K, w, B, S, device, peak)
            rows.append(r)
            torch.cuda.empty_cache()
            print(json.dumps(r), file=sys.stderr, flush=True)
            if not r["fits"]:
                break
    max_b = {i: max([r["batch"] for r in rows if r["impl"] == i and r["fits"]], default=0)
             for i in ("bf16", "kivi-2bit")}
    print(json.dumps({
        "sweep": "memory-wall", "workload": w.name,
        "shape": {"layers": w.num_layers, "heads": w.num_kv_heads, "head_dim": w.head_dim,
                  "context_at_timed_call": S, "bits": w.bits},
        "metric": "decode-attention tokens/s (all layers, attention calls only) and cache "
                  "bytes that fit on one B200",
        "peak_gbs": peak, "peak_kind": peak_kind, "rows": rows,
        "largest_batch_that_fits": max_b,
        "batch_ratio": max_b["kivi-2bit"] / max_b["bf16"] if max_b["bf16"] else None,
        "data": "synthetic (seeded)",
        "l2": "inputs larger than L2: one step reads every layer's cache"}), flush=True)


# ---------------------------------------------------------------------------
# Key-granularity ablation: per-channel (KIVI) against per-token key quantization
# ---------------------------------------------------------------------------

def run_key_granularity(args):
    """Relative error of the dequantized keys and of the attention output (values
    kept exact, so only the keys' error shows) for keys quantized per channel and
    per token, at 2 and 4 bits, on one layer of each synthetic key distribution."""
    import decode_attention_kivi_b200 as K

    device = torch.device("cuda", torch.cuda.current_device())
    rows = []
    for name in ("llama3_8b_gqa_8k", "tiny"):
        w = synth.WORKLOADS[name]
        k, v = synth.prefill_kv(w, 0, device=device)           # [B][Hkv][S][D]
        q = synth.query(w, 0, 0, device=device)
        B, H, S, D = k.shape
        att = K.Bf16Attention(batch=B, num_kv_heads=H, num_q_heads=w.num_q_heads, head_dim=D,
                              device=device)
        ref = att.attend(k, v, S, q).clone()
        kf = k.float()
        for bits in (2, 4):
            for per_token in (False, True):
                k_hat = K.kivi_fake_quant_keys(k.reshape(-1, D), bits, per_token).view(B, H, S, D)
                k_err = float((k_hat - kf).norm() / kf.norm())
                out = att.attend(k_hat.to(torch.bfloat16).contiguous(), v, S, q)
                o_err = float(((out - ref).norm(dim=-1) / ref.norm(dim=-1)).mean())
                rows.append({"keys": name, "key_distribution": w.key_dist, "bits": bits,
                             "granularity": "per-token" if per_token else "per-channel",
                             "key_rel_l2_error": k_err, "attention_rel_l2_error": o_err})
        assert att.check_device_status() == 0
    print(json.dumps({"sweep": "key-granularity", "rows": rows,
                      "note": "values unquantized; attention over bf16-rounded dequantized keys "
                              "against attention over the original keys, both on the GPU",
                      "data": "synthetic (seeded)"}), flush=True)


# ---------------------------------------------------------------------------
# Prefill: causal attention on the tensor cores, with and without the fused quantize
# ---------------------------------------------------------------------------

def causal_attention_flops(B, Hq, D, S) -> int:
    """Multiply-adds x 2 of the causal attention's two products: position i takes
    i + 1 keys, so sum_i (i + 1) = S (S + 1) / 2 dot products of length D each."""
    return 2 * 2 * B * Hq * D * (S * (S + 1) // 2)


def run_prefill(args):
    """One Llama-3-8B GQA layer's 8K prompt: the causal attention alone, the same
    with the prompt quantized into the cache in its epilogue, and the separate
    quantize kernels, each timed with CUDA events (median of 10 calls)."""
    import decode_attention_kivi_b200 as K

    device = torch.device("cuda", torch.cuda.current_device())
    w0 = synth.WORKLOADS["llama3_8b_gqa_8k"]
    S = w0.context
    peak, peak_kind = tensor_peak()
    rows = []
    for B in [int(x) for x in args.prefill_batches.split(",")]:
        w = w0.with_batch(B)
        q = synth.prompt_query(w, 0, device=device)
        k, v = synth.prefill_kv(w, 0, device=device)
        out = torch.empty(q.shape, dtype=torch.float32, device=device)
        status = torch.zeros(1, dtype=torch.int32, device=device)
        cache = K.KiviCache(batch=B, num_layers=1, num_kv_heads=w.num_kv_heads,
                            num_q_heads=w.num_q_heads, head_dim=w.head_dim, bits=w.bits,
                            max_tokens=S, device=device)

        def fused(_):
            cache.reset(0)
            cache.prefill_attention(0, q, k, v, out)

        def separate_quantize(_):
            cache.reset(0)
            cache.prefill(0, k, v)

        ms_attn = _time_layers(lambda _: K.kivi_causal_attention(q, k, v, out, status=status), 1)
        ms_fused = _time_layers(fused, 1)
        ms_quant = _time_layers(separate_quantize, 1)
        assert cache.check_device_status() == 0 and int(status.item()) == 0
        cache.close()
        flops = causal_attention_flops(B, w.num_q_heads, w.head_dim, S)
        tflops = flops / (ms_attn * 1e-3) / 1e12
        rows.append({"batch": B, "prompt": S, "attention_ms": ms_attn,
                     "attention_tflops": tflops, "frac_of_peak": tflops / peak,
                     "fused_prefill_ms": ms_fused,
                     "fused_tflops": flops / (ms_fused * 1e-3) / 1e12,
                     "separate_quantize_ms": ms_quant,
                     "separate_total_ms": ms_attn + ms_quant,
                     "fused_saves_ms": ms_attn + ms_quant - ms_fused})
        print(json.dumps(rows[-1]), file=sys.stderr, flush=True)
        del q, k, v, out
        torch.cuda.empty_cache()
    print(json.dumps({
        "sweep": "prefill", "workload": "llama3_8b_gqa_8k prompt, one layer",
        "shape": {"kv_heads": w0.num_kv_heads, "q_heads": w0.num_q_heads,
                  "head_dim": w0.head_dim, "prompt": S, "bits": w0.bits},
        "metric": "causal prefill attention TFLOP/s (2 x multiply-adds of the causal "
                  "products) and the time of the fused quantize against the separate kernels",
        "peak_tflops": peak, "peak_kind": peak_kind, "rows": rows,
        "data": "synthetic (seeded)", "l2": "inputs larger than L2"}), flush=True)


def main():
    args = parse()
    if args.sweep == "prefill":
        run_prefill(args)
        return
    if args.sweep == "memory-wall":
        run_memory_wall(args)
        return
    if args.sweep == "key-granularity":
        run_key_granularity(args)
        return
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    w = synth.WORKLOADS[args.workload]
    if args.batch:
        w = w.with_batch(args.batch)
    if args.layers:
        w = dataclasses.replace(w, num_layers=args.layers)
    cfg = workload_config(w, args.warmup, args.steps)
    if args.impl == "reference":
        if rank == 0:
            run_reference(args, w, cfg)
        return
    if world > 1:
        import datetime

        local = int(os.environ.get("LOCAL_RANK", "0"))
        torch.cuda.set_device(local)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    res = run_gpu(args, w, cfg, rank, world)
    if rank == 0:
        peak, peak_kind = hbm_peak()
        n_calls = len(res["call_us"]) * w.num_layers  # one burst of L launches per step
        per_launch = res["bytes_timed"] / n_calls
        gbs = res["bytes_timed"] / (res["attn_ms"] * 1e-3) / 1e9
        value = weak_scaling_tokens_per_s(world, w.batch, args.steps, res["ms"])
        pct = percentiles(res["call_us"])
        l2 = (f"L2 flushed between timed steps ({L2_FLUSH_BYTES >> 20} MB written, outside "
              "the step events)" if res["flush_l2"] else
              f"inputs larger than L2: one step reads every layer's cache "
              f"({w.num_layers} x ~{per_launch / 1e6:.0f} MB)")
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": res["ms"] / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f16 tensor-core operands (codes, q*scale and p*scale as hi+lo pairs; "
                     "bf16 residual), f32 accumulation",
            "data": "synthetic (seeded; shapes and key-outlier structure of the pages' models)",
            "config": cfg, "l2": l2,
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": peak, "unit": "GB/s",
                         "frac": gbs / peak, "peak_kind": peak_kind,
                         "traffic": recorded_traffic(w),
                         "algorithmic_bytes_per_launch": per_launch,
                         "kernel": "decode_kernel (one launch per kivi_decode_attention call)",
                         "avg_launch_us": pct["mean"],
                         "launch_us": {k: pct[k] for k in ("median", "p10", "p90", "n")},
                         "launch_us_basis": "per timed step: CUDA-event time of the step's burst "
                                            "of L back-to-back decode launches / L"},
            "gpu_launches": 2 * w.num_layers * args.steps,
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
