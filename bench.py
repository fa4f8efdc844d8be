#!/usr/bin/env python
"""Benchmark of the causal sliding-window attention forward on B200.

Metric: attention-forward TFLOP/s counted over unmasked (query, key) pairs (4*D flops per pair:
2D for q.k, 2D for p*v), with tokens/s and the fraction of the dense-BF16 tensor peak, on the
nanochat d24 full-window layer with value embeddings (B=16, T=2048, H=12, D=128, W=2048).

One step = one whole layer forward (RoPE + RMS QK-norm + VE gate prologue, then the windowed
attention with its LSE) on inputs already resident in HBM.  Inputs are seeded synthetic
N(0,1) bf16 tensors shaped like the layer; they are larger than the 126 MB L2, so no flush
is needed between steps.  Smaller workloads (the GPT-2 124M layer) flush L2 between steps and
sum the per-step event times instead.

  python bench.py [--gpus N --steps K --warmup W]            # our CUDA path
  python bench.py --impl reference [--steps K --warmup W]    # the fp64 CPU oracle, same metric

With N > 1 (torchrun), every rank runs its own batch shard of 16 sequences (weak scaling, no
collective on the data path); the step time is the max over ranks.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import workloads  # noqa: E402

WORKLOADS = {
    "d24_L_VE": workloads.D24_L_VE,
    "d24_S": workloads.D24_S,
    "gpt2_124m": workloads.GPT2,
    "tiny": workloads.TINY,
}
METRIC = "attention fwd TFLOP/s (unmasked pairs) & tokens/s, d24 T=2048; % of BF16 peak"
UNIT = "TFLOP/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
KERNEL_SOURCES = ["causal_sliding_window_swa_b200/csrc/attn_fwd.cuh",
                  "causal_sliding_window_swa_b200/csrc/ptx.cuh"]
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "attn_fwd_traffic.json")


# ------------------------------------------------------------------ host-side helpers

def flops_per_step(s: workloads.LayerShape) -> float:
    return 4.0 * s.D * s.unmasked_pairs()


def shard_shape(s: workloads.LayerShape, rank: int) -> workloads.LayerShape:
    """Rank r's batch shard: same per-GPU shape, its own seed (rank 0 keeps the workload's)."""
    import dataclasses
    return dataclasses.replace(s, seed=s.seed + 1000 * rank)


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


def kernel_hash() -> str:
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def recorded_traffic(workload: str):
    """dram__bytes_read.sum + dram__bytes_write.sum per launch of the attention kernel from the
    committed ncu summary, or None if absent or taken on a different kernel source."""
    try:
        with open(TRAFFIC_FILE) as f:
            doc = json.load(f)
    except (OSError, ValueError):
        return None
    ent = doc.get(workload)
    if not ent or ent.get("kernel_sha256") != kernel_hash():
        return None
    return ent.get("dram_bytes_per_launch")


class L2Flush:
    """Between timed steps: write a 256 MB buffer (larger than the 126 MB L2), then read another
    256 MB buffer, so that L2 holds neither the step's data nor dirty lines whose write-back would
    otherwise fall inside the next timed step."""

    def __init__(self, dev):
        import torch
        self.w = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
        self.r = torch.ones((256 << 20) // 8, dtype=torch.int64, device=dev)

    def __call__(self, i):
        self.w.fill_(i & 0xff)
        self.r.sum()


L2_NOTE = "flushed between steps (256 MB write, then a 256 MB read of another buffer; outside the timed events)"


def drain(dev):
    """Wait for the device while the clock sampler keeps sampling: poll an event recorded after
    the enqueued work and sleep between polls (one blocking synchronize can keep the sampler
    thread from running until the work is done)."""
    import torch
    ev = torch.cuda.Event()
    ev.record(torch.cuda.current_stream(dev))
    while not ev.query():
        time.sleep(0.0005)
    torch.cuda.synchronize(dev)


def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def reduce_max(x: float, device=None) -> float:
    """Max of a scalar over all ranks (identity when not distributed)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML while the timed region runs."""
    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting"}

    def __init__(self, index: int, period_s: float = 0.001):
        self.index = index
        self.period = period_s
        self.samples = []
        self.reasons = set()
        self.max_mhz = None
        self._stop = threading.Event()
        self._thr = None
        self.ok = False

    def start(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(self.index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            return self
        self._thr = threading.Thread(target=self._run, daemon=True)
        self._thr.start()
        return self

    def _run(self):
        nv = self._nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                get = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                    nv.nvmlDeviceGetCurrentClocksThrottleReasons
                bits = get(self._h)
                for b, name in self.REASONS.items():
                    if bits & b and name != "gpu_idle":
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self.period)

    def stop(self):
        self._stop.set()
        if self._thr is not None:
            self._thr.join()
        return {"sm_mhz": (statistics.median(self.samples) if self.samples else None),
                "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                "samples": len(self.samples)}


def cpu_baseline(s: workloads.LayerShape, d, budget_s: float):
    """The fp64 oracle, as it stands, on whole (b, h) slices of the workload (every query row of
    the slice) until ~budget_s seconds of CPU work are done.  Returns the metric in TFLOP/s."""
    import numpy as np
    import oracle
    W = s.eff_window()
    pairs_per_bh = W * (W + 1) // 2 + (s.T - W) * W
    done = 0
    t0 = time.perf_counter()
    for bh in range(s.B * s.H):
        rows = np.arange(bh * s.T, (bh + 1) * s.T, dtype=np.int64)
        oracle.forward(d, s.window, parity=True, rows=rows)
        done += 1
        if time.perf_counter() - t0 >= budget_s:
            break
    dt = time.perf_counter() - t0
    flops = 4.0 * s.D * pairs_per_bh * done
    return {"value": flops / dt / 1e12, "unit": UNIT, "cores": oracle.threads(), "kind": "oracle",
            "sample": f"{done} of {s.B * s.H} (b,h) slices of {s.name}, every query row of each "
                      f"({done * pairs_per_bh} unmasked pairs), {dt:.1f} s",
            "tokens_per_s": done * s.T / s.H / dt}


L2_BYTES = 126 << 20


def input_bytes(s: workloads.LayerShape) -> int:
    return (4 if s.ve else 3) * s.n_elems * 2


def config_of(s: workloads.LayerShape, world: int):
    mb = input_bytes(s) / 1e6
    names = "q,k,v" + (",ve" if s.ve else "")
    l2 = (f"no flush: inputs ({names}) = {mb:.0f} MB > 126 MB L2" if input_bytes(s) > L2_BYTES
          else f"inputs ({names}) = {mb:.0f} MB fit in L2: " + L2_NOTE + "; step time = sum of "
               "the per-step event times")
    return {"workload": s.name, "B_per_gpu": s.B, "T": s.T, "H": s.H, "D": s.D,
            "window": s.eff_window(), "value_embeddings": s.ve, "global_batch": s.B * world,
            "seq_len": s.T, "parallelism": f"dp{world} (batch shards, no collective)",
            "l2": l2}


# ------------------------------------------------------------------------ reference arm

def run_reference(args, s):
    rank, world, _ = dist_env()
    if rank != 0:
        return 0
    import numpy as np
    import oracle
    d = workloads.make_layer(s)
    W = s.eff_window()
    total_steps = args.steps + args.warmup
    per_step_budget = max(0.02, args.reference_budget_s / max(1, total_steps))
    g = np.random.default_rng(1234)

    def step(n_rows):
        bh = int(g.integers(0, s.B * s.H))
        i = np.sort(g.choice(s.T, size=n_rows, replace=False)).astype(np.int64)
        rows = bh * s.T + i
        t0 = time.perf_counter()
        oracle.forward(d, s.window, parity=True, rows=rows)
        dt = time.perf_counter() - t0
        pairs = int(np.minimum(i + 1, W).sum())
        return dt, pairs

    # calibrate the rows per step to the per-step budget
    dt, _ = step(32)
    n_rows = int(max(1, min(s.T, 32 * per_step_budget / max(dt, 1e-6))))
    for _ in range(args.warmup):
        step(n_rows)
    tot_t, tot_pairs = 0.0, 0
    for _ in range(args.steps):
        dt, pairs = step(n_rows)
        tot_t += dt
        tot_pairs += pairs
    value = 4.0 * s.D * tot_pairs / tot_t / 1e12
    cores = oracle.threads()
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": tot_t / args.steps * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_of(s, world), "impl": "reference",
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": f"each step: {n_rows} seeded query rows of one random (b,h) slice "
                                   f"of {s.name} (with that slice's prologue)"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# --------------------------------------------------------------------------- our arm

def run_ours(args, s0):
    import torch
    import torch.distributed as dist
    import causal_sliding_window_swa_b200 as swa

    rank, world, local = dist_env()
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device (no CPU path)")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    s = shard_shape(s0, rank)

    d = workloads.make_layer(s)
    g = workloads.gpu_side_inputs(d)
    host = {k: (None if v is None else v.contiguous().pin_memory()) for k, v in g.items()}
    x = {k: (None if v is None else v.to(dev, non_blocking=True)) for k, v in host.items()}
    out = torch.empty_like(x["q"])
    lse = torch.empty((s.B, s.H, s.T), dtype=torch.float32, device=dev)
    nbytes = swa.swa_attn_workspace_bytes(s.B, s.T, s.H, s.D, int(s.ve))
    ws = torch.empty(nbytes, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    st = stream.cuda_stream
    P = lambda t: None if t is None else t.data_ptr()
    # the stages of swa_attn_fwd_ws (the same kernels swa_attn_fwd runs): the prologue (with the
    # gate on value-embedding layers), then the attention kernel
    args_pro = (P(x["q"]), P(x["k"]), P(x["v"]), P(x["ve"]), P(x["gate_x"]), P(x["Wg"]),
                s.B, s.T, s.H, s.D, 10000.0, 1e-6, ws.data_ptr(), nbytes, st)
    args_att = (P(x["v"]), int(s.ve), out.data_ptr(), lse.data_ptr(), s.B, s.T, s.H, s.D, s.window,
                ws.data_ptr(), nbytes, st)

    def check(rc, what):
        if rc != 0:
            raise swa.SwaError(rc, what)

    # The RoPE table depends only on (T, D, base): built once, like a model's rotary cache.
    check(swa.swa_attn_rope_table(s.B, s.T, s.H, s.D, int(s.ve), 10000.0, ws.data_ptr(), nbytes, st),
          "swa_attn_rope_table")

    K, Wm = args.steps, args.warmup
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True),
           torch.cuda.Event(enable_timing=True)) for _ in range(K)]

    def step(e=None):
        if e is not None:
            e[0].record(stream)
        check(swa.swa_attn_prologue(*args_pro), "swa_attn_prologue")
        if e is not None:
            e[1].record(stream)
        check(swa.swa_attn_attention(*args_att), "swa_attn_attention")
        if e is not None:
            e[2].record(stream)

    # inputs that fit in L2 would stay there from one step to the next: flush between steps
    flush = L2Flush(dev) if input_bytes(s) <= L2_BYTES else None
    for i in range(Wm):
        if flush is not None:
            flush(i)
        step()
    torch.cuda.synchronize(dev)
    swa.check_device_status(stream)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    sampler = ClockSampler(local).start()
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    t_start.record(stream)
    for i in range(K):
        if flush is not None:
            flush(i)
        step(ev[i])
    t_end.record(stream)
    drain(dev)
    if world > 1:
        dist.barrier()
    clocks = sampler.stop()
    swa.check_device_status(stream)
    if flush is None:
        ms_local = t_start.elapsed_time(t_end) / K
    else:
        ms_local = sum(e[0].elapsed_time(e[2]) for e in ev) / K
    pro_ms = sum(e[0].elapsed_time(e[1]) for e in ev) / K
    att_ms = sum(e[1].elapsed_time(e[2]) for e in ev) / K
    ms = reduce_max(ms_local, dev)
    att_ms_max = reduce_max(att_ms, dev)
    pro_ms_max = reduce_max(pro_ms, dev)

    # ---------------- end to end through the public call, host buffers, copies inside
    # Every step copies all of its inputs in from pinned host memory, runs swa.forward and reads
    # out and lse back.  Two sets of device buffers: step i's copy-in (its own stream) overlaps
    # step i-1's layer call and read-back (a third stream), as a training or serving loop would
    # pipeline them; the link carries both directions at once.
    E = max(1, min(args.e2e_steps, K))
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    bufs = []
    for _ in range(2):
        bufs.append({
            "x": {k: (None if v is None else torch.empty_like(v)) for k, v in x.items()},
            "out": torch.empty_like(out), "lse": torch.empty_like(lse),
            "h_out": torch.empty(out.shape, dtype=out.dtype, pin_memory=True),
            "h_lse": torch.empty(lse.shape, dtype=lse.dtype, pin_memory=True),
            "in": torch.cuda.Event(), "done": torch.cuda.Event(), "read": torch.cuda.Event(),
            "used": False})

    def e2e_step(i):
        b = bufs[i & 1]
        if b["used"]:
            s_in.wait_event(b["done"])          # the layer call two steps back has read these inputs
        with torch.cuda.stream(s_in):
            for k, v in host.items():
                if v is not None:
                    b["x"][k].copy_(v, non_blocking=True)
        b["in"].record(s_in)
        stream.wait_event(b["in"])
        if b["used"]:
            stream.wait_event(b["read"])        # its out / lse have been read back
        xin = b["x"]
        swa.forward(xin["q"], xin["k"], xin["v"], s.window, xin["ve"], xin["gate_x"], xin["Wg"],
                    out=b["out"], lse=b["lse"])
        b["done"].record(stream)
        s_out.wait_event(b["done"])
        with torch.cuda.stream(s_out):
            b["h_out"].copy_(b["out"], non_blocking=True)
            b["h_lse"].copy_(b["lse"], non_blocking=True)
        b["read"].record(s_out)
        b["used"] = True

    for i in range(3):
        e2e_step(i)
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    s_in.wait_event(e0)
    for i in range(E):
        e2e_step(i)
    for b in bufs:
        stream.wait_event(b["read"])
    e1.record(stream)
    torch.cuda.synchronize(dev)
    swa.check_device_status(stream)
    e2e_ms = reduce_max(e0.elapsed_time(e1) / E, dev)
    h2d = sum(v.numel() * v.element_size() for v in host.values() if v is not None)
    d2h = out.numel() * out.element_size() + lse.numel() * lse.element_size()

    # ---------------- roll-up
    fl = flops_per_step(s)
    value = world * fl / (ms * 1e-3) / 1e12
    peaks, peak_src = load_peaks()
    peak = float(peaks["bf16_tflops"])
    achieved = fl / (att_ms_max * 1e-3) / 1e12
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K, "warmup": Wm,
        "ms_per_step": ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16", "data": "synthetic (seeded N(0,1) bf16 q,k,v; VE table/ids/x/Wg as the "
                                  "layer's shapes)",
        "config": config_of(s, world),
        "tokens_per_s": world * s.B * s.T / (ms * 1e-3),
        "pct_bf16_peak": 100.0 * value / world / peak,
        "peak_source": f"{peak_src} bf16_tflops (burst)",
        "stage_ms": {"prologue": pro_ms_max, "attention": att_ms_max},
        "roofline": {"bound": "tensor", "kernel": f"attn_fwd_kernel<{s.D}>", "achieved": achieved,
                     "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
                     "traffic": recorded_traffic(args.workload),
                     "note": f"4*D flops per unmasked pair / mean attention launch time; peak = "
                             f"{peak_src} dense bf16 (burst)"},
        "prologue_roofline": {"bound": "hbm", "achieved": prologue_bytes(s) / (pro_ms_max * 1e-3) / 1e9,
                              "peak": float(peaks["hbm_gbs"]), "unit": "GB/s",
                              "frac": prologue_bytes(s) / (pro_ms_max * 1e-3) / 1e9 / float(peaks["hbm_gbs"])},
        "e2e": {"value": world * fl / (e2e_ms * 1e-3) / 1e12, "unit": UNIT,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms},
        "gpu_launches": (3 if s.ve else 2) * K,   # (gate,) prologue with its repairs, attention
        "clocks": clocks,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(s, d, args.cpu_seconds)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def prologue_bytes(s: workloads.LayerShape) -> float:
    """Algorithmic bytes of the prologue stage: read q, k (+ v, ve, gate_x, Wg), write qhat, khat
    (+ v')."""
    n = s.n_elems * 2
    b = 2 * n + 2 * n           # q, k in; qhat, khat out
    if s.ve:
        b += 3 * n + s.B * s.T * 32 * 2 + 32 * s.H * 2   # v, ve in; v' out; gate_x, Wg
    return float(b)


def run_decode(args, s):
    """One generation step per timed iteration (swa_attn_decode) at the last position of the
    workload's sequence: the new token of each of the B sequences attends to min(W, T) cached keys.
    The caches are filled once by the prefill prologue, so they hold real khat / v'.  Metric: the
    step's algorithmic bytes (K and V window reads, the new token's inputs and cache writes, out)
    per second; HBM-bound."""
    import torch
    import causal_sliding_window_swa_b200 as swa

    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device (no CPU path)")
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    d = workloads.make_layer(s)
    g = {k: (None if v is None else v.to(dev)) for k, v in workloads.gpu_side_inputs(d).items()}
    B, T, H, D = s.B, s.T, s.H, s.D
    stream = torch.cuda.current_stream(dev)
    st = stream.cuda_stream
    P = lambda t: None if t is None else t.data_ptr()
    # caches = the prefill prologue's khat / v' of every position
    nbytes = swa.swa_attn_workspace_bytes(B, T, H, D, int(s.ve))
    ws = torch.empty(nbytes, dtype=torch.uint8, device=dev)
    for rc, what in ((swa.swa_attn_rope_table(B, T, H, D, int(s.ve), 10000.0, ws.data_ptr(), nbytes, st), "rope"),
                     (swa.swa_attn_prologue(P(g["q"]), P(g["k"]), P(g["v"]), P(g["ve"]), P(g["gate_x"]), P(g["Wg"]),
                                            B, T, H, D, 10000.0, 1e-6, ws.data_ptr(), nbytes, st), "prologue")):
        if rc != 0:
            raise swa.SwaError(rc, what)
    sec = lambda i: swa.swa_attn_workspace_offset(B, T, H, D, int(s.ve), i)
    n = B * T * H * D
    k_cache = ws[sec(1):sec(1) + 2 * n].view(torch.bfloat16).view(B, T, H, D).clone()
    v_cache = (ws[sec(2):sec(2) + 2 * n].view(torch.bfloat16).view(B, T, H, D).clone() if s.ve else g["v"].clone())
    pos = T - 1
    tok = {k: (None if g[k] is None else g[k][:, pos].contiguous()) for k in ("q", "k", "v", "ve", "gate_x")}
    out = torch.empty((B, H, D), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((B, H), dtype=torch.float32, device=dev)
    need = swa.swa_attn_decode_workspace_bytes(B, T, H, D, int(s.ve), s.window)
    dws = torch.empty(need, dtype=torch.uint8, device=dev)
    argsd = (P(tok["q"]), P(tok["k"]), P(tok["v"]), P(tok["ve"]), P(tok["gate_x"]), P(g["Wg"]), P(k_cache),
             P(v_cache), pos, P(out), P(lse), B, T, H, D, s.window, 10000.0, 1e-6, P(dws), need, st)

    def step():
        rc = swa.swa_attn_decode(*argsd)
        if rc != 0:
            raise swa.SwaError(rc, "swa_attn_decode")

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    swa.check_device_status(stream)
    # L2 (126 MB) holds part of the 201 MB window: flush it between steps.
    flush = L2Flush(dev)
    K = args.steps
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    sampler = ClockSampler(0).start()
    for i in range(K):
        flush(i)
        evs[i][0].record(stream)
        step()
        evs[i][1].record(stream)
    drain(dev)
    clocks = sampler.stop()
    swa.check_device_status(stream)
    ms = sum(a.elapsed_time(b) for a, b in evs) / K
    W = T if s.window <= 0 or s.window >= T else s.window
    keys = min(W, pos + 1)
    bytes_step = (2.0 * B * keys * H * D * 2          # K and V window reads
                  + B * H * D * 2 * (3 + 2 + 1)       # q, k, v in; khat, v' cache writes; out
                  + (B * H * D * 2 + B * 32 * 2 if s.ve else 0))
    gbs = bytes_step / (ms * 1e-3) / 1e9
    peaks, peak_src = load_peaks()
    line = {
        "metric": "decode step, KV-cache window read bandwidth (d24 shape, last position)",
        "value": gbs, "unit": "GB/s", "n_gpus": 1, "steps": K, "warmup": args.warmup,
        "ms_per_step": ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16 in/out, fp32 scores and sums", "data": "synthetic (seeded), caches from the prefill prologue",
        "config": {"workload": f"decode {args.workload}: B={B} Tmax={T} H={H} D={D} W={W} pos={pos} ve={s.ve}",
                   "l2": L2_NOTE},
        "tokens_per_s": B / (ms * 1e-3),
        "roofline": {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "frac": gbs / peaks["hbm_gbs"], "traffic": None, "peak_source": peak_src},
        "gpu_launches": 2 * K,
        "clocks": clocks,
    }
    print(json.dumps(line), flush=True)
    return 0


def run_backward(args, s):
    """The layer's backward per timed iteration (swa_attn_bwd: prologue recompute, row
    statistics, the dQ and dK/dV tensor-core kernels, the prologue in reverse and the gate
    gradients) on the workload, with out / lse from the forward and seeded dout / dlse.
    Metric: algorithmic backward FLOP/s, 10 D flops per visible (query, key) pair (the five
    products of the gradient, 2.5 times the forward's 4 D)."""
    import torch
    import causal_sliding_window_swa_b200 as swa

    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device (no CPU path)")
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    d = workloads.make_layer(s)
    g = {k: (None if v is None else v.to(dev)) for k, v in workloads.gpu_side_inputs(d).items()}
    B, T, H, D = s.B, s.T, s.H, s.D
    stream = torch.cuda.current_stream(dev)
    out, lse = swa.forward(g["q"], g["k"], g["v"], s.window, ve=g["ve"], gate_x=g["gate_x"], Wg=g["Wg"])
    gen = torch.Generator().manual_seed(s.seed + 1000)
    dout = torch.randn((B, T, H, D), generator=gen).to(torch.bfloat16).to(dev)
    dlse = torch.randn((B, H, T), generator=gen).to(dev)
    need = swa.swa_attn_bwd_workspace_bytes(B, T, H, H, D, int(s.ve))
    ws = torch.empty(need, dtype=torch.uint8, device=dev)

    def step():
        swa.backward(g["q"], g["k"], g["v"], out, lse, dout, s.window, dlse=dlse, ve=g["ve"],
                     gate_x=g["gate_x"], Wg=g["Wg"], workspace=ws)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    swa.check_device_status(stream)
    flush = L2Flush(dev)
    K = args.steps
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    sampler = ClockSampler(0).start()
    for i in range(K):
        flush(i)
        evs[i][0].record(stream)
        step()
        evs[i][1].record(stream)
    drain(dev)
    clocks = sampler.stop()
    swa.check_device_status(stream)
    ms = sum(a.elapsed_time(b) for a, b in evs) / K
    flops = 2.5 * flops_per_step(s)
    tf = flops / (ms * 1e-3) / 1e12
    peaks, peak_src = load_peaks()

    # The same gradient for a caller that keeps the forward's activations: the forward writes
    # qhat, khat, v' and the gates into the backward's workspace, and swa_attn_bwd_saved skips
    # the prologue recompute (its gradients are bit-identical; tests/test_bwd_gpu.py).
    out2, lse2 = swa.forward(g["q"], g["k"], g["v"], s.window, ve=g["ve"], gate_x=g["gate_x"], Wg=g["Wg"],
                             workspace=ws)

    def step_saved():
        swa.backward(g["q"], g["k"], g["v"], out2, lse2, dout, s.window, dlse=dlse, ve=g["ve"],
                     gate_x=g["gate_x"], Wg=g["Wg"], workspace=ws, saved=True)

    for _ in range(args.warmup):
        step_saved()
    torch.cuda.synchronize(dev)
    evs2 = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    for i in range(K):
        flush(i)
        evs2[i][0].record(stream)
        step_saved()
        evs2[i][1].record(stream)
    torch.cuda.synchronize(dev)
    swa.check_device_status(stream)
    ms_saved = sum(a.elapsed_time(b) for a, b in evs2) / K
    tf_saved = flops / (ms_saved * 1e-3) / 1e12
    # RoPE table, prologue, row statistics, dQ, dK/dV; on value-embedding layers also the gate and
    # the three gate-gradient kernels
    launches = 5 + (4 if s.ve else 0)
    line = {
        "metric": "attention backward TFLOP/s (10 D flops per visible pair)",
        "value": tf, "unit": "TFLOP/s", "n_gpus": 1, "steps": K, "warmup": args.warmup,
        "ms_per_step": ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16 operands, fp32 accumulate", "data": "synthetic (seeded)",
        "config": {"workload": f"backward {args.workload}: B={B} T={T} H={H} D={D} W={s.window} ve={s.ve}",
                   "l2": L2_NOTE},
        "roofline": {"bound": "tensor", "achieved": tf, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                     "frac": tf / peaks["bf16_tflops"], "traffic": None, "peak_source": peak_src,
                     "note": "whole backward call; the tensor-core kernels do 7 products per tile pair"},
        "gpu_launches": launches * K,
        "clocks": clocks,
        "saved_activations": {"ms_per_step": ms_saved, "value": tf_saved, "unit": "TFLOP/s",
                              "frac": tf_saved / peaks["bf16_tflops"],
                              "note": "swa_attn_bwd_saved on the workspace the forward wrote: no prologue "
                                      "recompute (rope table, gate and prologue kernels not launched)"},
    }
    print(json.dumps(line), flush=True)
    return 0


def run_forward_x(args, s):
    """The layer from its input x per timed iteration (swa_attn_fwd_x: the fused q/k/v projection +
    prologue kernel, then the attention kernel) on the workload's shapes, x (B, T, H D) and a
    random-init Wqkv [3 H D, H D] (std (H D)^-1/2).  Metric: FLOP/s of the projection
    (2 M N C) plus the attention (4 D per visible pair)."""
    import torch
    import causal_sliding_window_swa_b200 as swa

    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device (no CPU path)")
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    B, T, H, D = s.B, s.T, s.H, s.D
    C = H * D
    gen = torch.Generator().manual_seed(s.seed + 2000)
    x = torch.randn((B, T, C), generator=gen).to(torch.bfloat16).to(dev)
    W = (torch.randn((3 * H * D, C), generator=gen) * C ** -0.5).to(torch.bfloat16).to(dev)
    ve = Wg = None
    if s.ve:
        ve = torch.randn((B, T, H, D), generator=gen).to(torch.bfloat16).to(dev)
        Wg = (torch.randn((32, H), generator=gen) * workloads.WG_STD).to(torch.bfloat16).to(dev)
    need = swa.swa_attn_fwd_x_workspace_bytes(B, T, H, H, D)
    ws = torch.empty(need, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        swa.forward_x(x, W, H, H, D, s.window, ve=ve, Wg=Wg, workspace=ws)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    swa.check_device_status(stream)
    flush = L2Flush(dev)
    K = args.steps
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    sampler = ClockSampler(0).start()
    for i in range(K):
        flush(i)
        evs[i][0].record(stream)
        step()
        evs[i][1].record(stream)
    drain(dev)
    clocks = sampler.stop()
    swa.check_device_status(stream)
    ms = sum(a.elapsed_time(b) for a, b in evs) / K
    proj = 2.0 * B * T * (3 * H * D) * C
    flops = proj + flops_per_step(s)
    tf = flops / (ms * 1e-3) / 1e12
    peaks, peak_src = load_peaks()
    line = {
        "metric": "layer forward from x TFLOP/s (projection 2 M N C + attention 4 D per visible pair)",
        "value": tf, "unit": "TFLOP/s", "n_gpus": 1, "steps": K, "warmup": args.warmup,
        "ms_per_step": ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16 operands, fp32 accumulate", "data": "synthetic (seeded), random-init Wqkv",
        "config": {"workload": f"forward_x {args.workload}: B={B} T={T} C={C} H={H} D={D} W={s.window} ve={s.ve}",
                   "l2": L2_NOTE},
        "roofline": {"bound": "tensor", "achieved": tf, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                     "frac": tf / peaks["bf16_tflops"], "traffic": None, "peak_source": peak_src,
                     "note": "whole call: rope table, gate, fused projection kernel, attention kernel"},
        "gpu_launches": (4 if s.ve else 3) * K,
        "clocks": clocks,
    }
    print(json.dumps(line), flush=True)
    return 0


def run_sssl(args):
    """The SSSL stack of the d24 model at one point of the length sweep: 24 consecutive layer
    calls (swa_attn_fwd, the public call, library workspace) with windows S,S,S,L (S = T/2,
    L = T), value embeddings on even layers, H = 12, D = 128, B = 32768 / T.  Every layer has its
    own inputs (about 0.4 GB per layer, 9.7 GB in all, so L2 never serves a later layer).  One
    timed step = all 24 calls.  Metric: TFLOP/s over the stack's unmasked pairs (4 D per pair)
    and tokens/s = B T / step time.  Inputs are drawn on the device from a seeded generator
    (N(0,1) bf16; ids uniform over the vocabulary; Wg N(0, 0.02)), the shapes and distributions
    of the workload; the parity tests check the same stack drawn on the host."""
    import torch
    import causal_sliding_window_swa_b200 as swa

    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device (no CPU path)")
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    T = args.sssl_T
    B = 32768 // T
    H, D = 12, 128
    shapes = workloads.sssl_layer_shapes(B, T, H, D)
    gen = torch.Generator(device=dev).manual_seed(workloads.SSSL_SEED)
    bf = lambda *shp, std=1.0: (torch.randn(shp, generator=gen, device=dev) * std).to(torch.bfloat16)
    layers = []
    for s in shapes:
        L = dict(q=bf(B, T, H, D), k=bf(B, T, H, D), v=bf(B, T, H, D), ve=None, gate_x=None, Wg=None)
        if s.ve:
            ids = torch.randint(0, workloads.VOCAB, (B, T), generator=gen, device=dev)
            table = bf(workloads.VOCAB, H * D)
            L["ve"] = table[ids].view(B, T, H, D)
            del table
            L["gate_x"] = bf(B, T, workloads.GATE_CHANNELS)
            L["Wg"] = bf(workloads.GATE_CHANNELS, H, std=workloads.WG_STD)
        layers.append((s, L))
    out = torch.empty((B, T, H, D), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((B, H, T), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)
    st = stream.cuda_stream
    P = lambda t: None if t is None else t.data_ptr()
    calls = [(P(L["q"]), P(L["k"]), P(L["v"]), P(L["ve"]), P(L["gate_x"]), P(L["Wg"]), out.data_ptr(),
              lse.data_ptr(), B, T, H, D, s.window, 10000.0, 1e-6, st) for s, L in layers]

    def step():
        for a in calls:
            rc = swa.swa_attn_fwd(*a)
            if rc != 0:
                raise swa.SwaError(rc, "swa_attn_fwd")

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    swa.check_device_status(stream)
    K = args.steps
    sampler = ClockSampler(0).start()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(K):
        step()
    e1.record(stream)
    drain(dev)
    clocks = sampler.stop()
    swa.check_device_status(stream)
    ms = e0.elapsed_time(e1) / K
    flops = sum(flops_per_step(s) for s in shapes)
    tf = flops / (ms * 1e-3) / 1e12
    peaks, peak_src = load_peaks()
    line = {
        "metric": "SSSL stack (24 layers S,S,S,L) attention fwd TFLOP/s (unmasked pairs) & tokens/s",
        "value": tf, "unit": "TFLOP/s", "n_gpus": 1, "steps": K, "warmup": args.warmup,
        "ms_per_step": ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16", "data": "synthetic (seeded N(0,1) bf16 drawn on the device; VE on even layers)",
        "config": {"workload": f"SSSL stack B={B} T={T} H={H} D={D}, 24 layers S={T // 2},S,S,L={T}",
                   "l2": "no flush: each layer's inputs (0.3-0.4 GB) exceed the 126 MB L2"},
        "tokens_per_s": B * T / (ms * 1e-3),
        "stack_tflop": flops / 1e12,
        "roofline": {"bound": "tensor", "achieved": tf, "peak": float(peaks["bf16_tflops"]), "unit": "TFLOP/s",
                     "frac": tf / float(peaks["bf16_tflops"]), "traffic": None,
                     "note": f"whole stack of public calls; peak = {peak_src} dense bf16 (burst)"},
        # per layer: (gate,) prologue with its repairs, attention
        "gpu_launches": sum(3 if ls.ve else 2 for ls in shapes) * K,
        "clocks": clocks,
    }
    print(json.dumps(line), flush=True)
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=sorted(WORKLOADS), default="d24_L_VE")
    ap.add_argument("--e2e-steps", type=int, default=50)
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--reference-budget-s", type=float, default=90.0)
    ap.add_argument("--mode", choices=["forward", "decode", "backward", "forward_x", "sssl"], default="forward",
                    help="decode: time one KV-cache generation step; backward: time the layer's "
                         "gradient; forward_x: the layer from its input x (fused projection); "
                         "sssl: the 24-layer S,S,S,L stack at --sssl-T; default: the layer forward")
    ap.add_argument("--sssl-T", type=int, default=2048, choices=[1024, 2048, 4096, 8192, 16384],
                    help="sequence length of the SSSL stack (B = 32768 / T)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    s = WORKLOADS[args.workload]
    if args.mode != "forward" and (dist_env()[1] > 1 or args.gpus > 1):
        ap.error(f"--mode {args.mode} runs on one GPU (the forward mode shards across ranks)")
    if args.mode == "decode":
        return run_decode(args, s)
    if args.mode == "backward":
        return run_backward(args, s)
    if args.mode == "forward_x":
        return run_forward_x(args, s)
    if args.mode == "sssl":
        return run_sssl(args)
    if args.impl == "reference":
        return run_reference(args, s)
    return run_ours(args, s)


if __name__ == "__main__":
    sys.exit(main())
