#!/usr/bin/env python
"""VSA forward benchmark on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload h3]
    python bench.py --impl reference ...        # the CPU oracle, as a baseline

One step = one whole VSA forward (pool -> coarse attention + top-k ->
block-sparse attention with the fused gated combine) over one batch of seeded
synthetic bf16 inputs already resident in HBM.  Default workload: the
H3-like shape B=1, H=56, D=128, S=15488 (242 blocks of 64), top 20% = 48 KV
blocks per query block, gated.  Metric: effective TFLOP/s over the selected
64x64 tiles (4 * 64 * 64 * D FLOPs per tile) and ms per forward.

With N GPUs (torchrun, one process per GPU) every rank runs its own copy of
the workload (the forward has no exchange step: heads, batches and sequences
are independent), so per-GPU work is fixed and the scaling is weak; the time
is the max over ranks.
"""
from __future__ import annotations

import argparse
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

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from block_sparse_attention_15_b200 import inputs as I  # noqa: E402

METRIC = "VSA fwd ms & effective TFLOPS (selected tiles) at H=56,D=128,S=15488,topk 20%"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
L2_BYTES = 126 * 2**20
SPARSE_SOURCES = ["block_sparse_attention_15_b200/csrc/sparse_fwd.cu",
                  "block_sparse_attention_15_b200/csrc/vsa_device.cuh"]


# ---------------------------------------------------------------------------
# workloads
# ---------------------------------------------------------------------------
def make_workload(name: str) -> I.Workload:
    if name == "tiny":
        return I.workload_tiny()
    if name == "h3":
        return I.workload_h3()
    if name == "vsa128":
        return I.workload_vsa128()
    if name == "vsa256":
        return I.workload_vsa256()
    m = re.fullmatch(r"long(\d+)(-ungated)?", name)
    if m:
        return I.workload_long(int(m.group(1)) / 100.0, gated=m.group(2) is None)
    if name == "video":
        from block_sparse_attention_15_b200 import binding
        meta = binding.build_vsa_metadata(9, 30, 52)
        sizes = [int(s) for s in meta["variable_block_sizes"]]
        wl = I.Workload("video-tiled: 9x30x52 latent (14040 tokens) in 4x4x4 tiles, B1 H12 D128, "
                        "top 25% gated", 1, 12, 128, sizes, sizes,
                        I.topk_count(0.25, len(sizes)), True, 1002)
        wl.extra["meta"] = meta
        return wl
    raise ValueError(f"unknown workload {name}")


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def sparse_source_hash() -> str:
    """SHA-256 of the kernel sources' code: comments and blank lines are
    dropped first, so that an edit of the comments alone keeps a capture's
    record valid (the compiled kernel does not change)."""
    h = hashlib.sha256()
    for rel in SPARSE_SOURCES:
        with open(os.path.join(ROOT, rel)) as f:
            text = re.sub(r"/\*.*?\*/", "", f.read(), flags=re.S)
        lines = [re.sub(r"//.*$", "", ln).rstrip() for ln in text.splitlines()]
        h.update("\n".join(ln for ln in lines if ln).encode())
    return h.hexdigest()


def profiled_traffic(wl):
    """DRAM bytes per launch of the block-sparse kernel, from the committed
    record of an ncu capture (a JSON data file beside the capture's summary),
    if the workload has the recorded shape and the kernel sources still hash
    to what was profiled; else None."""
    path = os.path.join(ROOT, "profiles", "sparse_fwd_h3_traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        rec = json.load(f)
    shape = rec.get("shape", {})
    ours = {"B": wl.B, "H": wl.H, "D": wl.D, "block": wl.block, "n_q_blocks": wl.nq,
            "n_kv_blocks": wl.nkv, "topk": wl.topk}
    if shape != ours or rec.get("kernel_source_sha256") != sparse_source_hash():
        return None
    return int(rec["traffic_bytes_per_launch"])


# ---------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------
class ClockSampler:
    """nvidia-smi samples every 50 ms, started ahead of the timed region (its
    first sample comes ~0.1-0.3 s after launch); only samples that fall inside
    [start(), stop()] are kept, plus, for a region shorter than one period, the
    first sample after it."""
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")
    NAMES = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")

    def __init__(self, device_index: int):
        self.proc = None
        self.lines = []          # (monotonic time, line)
        self.t0 = self.t1 = None
        self.nvml = NvmlSampler(device_index)
        try:
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            ident = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "50", "-i", ident], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL,
                text=True)
        except Exception:  # noqa: BLE001 - clocks are best effort
            self.proc = None
            return
        self.reader = threading.Thread(target=self._read, daemon=True)
        self.reader.start()
        deadline = time.monotonic() + 5.0
        while not self.lines and time.monotonic() < deadline and self.proc.poll() is None:
            time.sleep(0.01)

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.monotonic(), line))

    def start(self):
        self.t0 = time.monotonic()

    def stop(self) -> dict:
        self.t1 = time.monotonic()
        fast = self.nvml.stop(self.t0 if self.t0 is not None else self.t1, self.t1)
        if self.proc is None:
            res = {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
            if fast:
                res["nvml_5ms"] = fast
            return res
        time.sleep(0.12)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.reader.join(timeout=5)
        t0 = self.t0 if self.t0 is not None else self.t1
        res = summarize_clock_lines(self.lines, t0, self.t1, self.NAMES)
        if fast:
            res["nvml_5ms"] = fast
        return res


class NvmlSampler:
    """SM clock and throttle reasons read through NVML every 5 ms on a thread
    (read-only queries), so that a timed region of a few tens of ms still
    holds several samples; None where NVML is unavailable."""
    REASONS = {"hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
               "sw_power_cap": 0x4}

    def __init__(self, device_index: int):
        self.samples = []   # (monotonic time, sm MHz, reason bits)
        self.stop_flag = False
        self.thread = None
        try:
            import pynvml
            pynvml.nvmlInit()
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            ident = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
            self.handle = pynvml.nvmlDeviceGetHandleByUUID(ident)
            self.nv = pynvml
        except Exception:  # noqa: BLE001 - best effort
            self.handle = None
            return
        self.thread = threading.Thread(target=self._run, daemon=True)
        self.thread.start()

    def _run(self):
        nv = self.nv
        while not self.stop_flag:
            try:
                mhz = nv.nvmlDeviceGetClockInfo(self.handle, nv.NVML_CLOCK_SM)
                bits = nv.nvmlDeviceGetCurrentClocksEventReasons(self.handle)
                self.samples.append((time.monotonic(), float(mhz), int(bits)))
            except Exception:  # noqa: BLE001
                return
            time.sleep(0.005)

    def stop(self, t0: float, t1: float):
        if self.thread is None:
            return None
        self.stop_flag = True
        self.thread.join(timeout=2)
        inside = [(m, b) for t, m, b in self.samples if t0 <= t <= t1]
        if not inside:
            return None
        reasons = sorted(n for n, bit in self.REASONS.items() if any(b & bit for _, b in inside))
        return {"sm_mhz": statistics.median(m for m, _ in inside), "samples": len(inside),
                "min_mhz": min(m for m, _ in inside), "reasons": reasons}


def summarize_clock_lines(lines, t0: float, t1: float, names) -> dict:
    """Median SM clock, max clock and power, and the throttle reasons seen, over
    the (time, csv line) samples inside [t0, t1]; for a window shorter than one
    sampling period, the first sample after it."""
    inside = [ln for t, ln in lines if t0 <= t <= t1]
    if not inside:
        inside = [ln for t, ln in lines if t > t1][:1]
    sm, smax, reasons, power = [], [], set(), []
    for line in inside:
        parts = [p.strip() for p in line.split(",")]
        if len(parts) < 3 + len(names):
            continue
        try:
            sm.append(float(parts[0]))
            smax.append(float(parts[1]))
            power.append(float(parts[2]))
        except ValueError:
            continue
        for name, val in zip(names, parts[3:3 + len(names)]):
            if val.lower().startswith("active"):
                reasons.add(name)
    return {"sm_mhz": statistics.median(sm) if sm else None,
            "sm_max_mhz": max(smax) if smax else None,
            "power_w_max": max(power) if power else None,
            "samples": len(sm), "reasons": sorted(reasons)}


# ---------------------------------------------------------------------------
# CPU oracle baseline (bounded sample)
# ---------------------------------------------------------------------------
def _blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [d.get("num_threads", 0) for d in threadpool_info() if d.get("user_api") == "blas"]
        return max(n) if n else os.cpu_count() or 1
    except Exception:  # noqa: BLE001
        return os.cpu_count() or 1


def oracle_sample(wl: I.Workload, q, k, v, gate, head: int, n_items: int):
    """Run the oracle's whole forward for one head restricted to the first
    n_items query blocks; return (seconds, selected-tile FLOPs)."""
    from oracle import vsa_oracle as O
    t0 = time.perf_counter()
    qn = q[:, head:head + 1].float().numpy()
    kn = k[:, head:head + 1].float().numpy()
    vn = v[:, head:head + 1].float().numpy()
    gn = None if gate is None else gate[:, :, head:head + 1].float().numpy()
    items = [(0, 0, a) for a in range(min(n_items, wl.nq))]
    O.vsa_forward(qn, kn, vn, gn, wl.q_block_sizes, wl.kv_block_sizes, wl.topk, items=items,
                  block=wl.block)
    dt = time.perf_counter() - t0
    flops = 4.0 * wl.block * wl.block * wl.D * min(wl.topk, wl.nkv) * len(items)
    return dt, flops


def cpu_baseline(wl, q, k, v, gate, budget_s=15.0):
    total_t, total_f, heads, items = 0.0, 0.0, 0, 0
    h = 0
    while total_t < budget_s and h < wl.H:
        dt, fl = oracle_sample(wl, q, k, v, gate, h, wl.nq)
        total_t += dt
        total_f += fl
        heads += 1
        items += wl.nq
        h += 1
    return {"value": total_f / total_t / 1e12, "unit": "TFLOP/s", "cores": _blas_threads(),
            "kind": "oracle",
            "sample": f"fp64 numpy oracle, whole forward of {heads} head(s) x {wl.nq} query blocks "
                      f"of this workload ({total_t:.1f} s on the host cores)"}


# ---------------------------------------------------------------------------
# inputs
# ---------------------------------------------------------------------------
def host_inputs(wl: I.Workload):
    Sq, Skv = wl.block * wl.nq, wl.block * wl.nkv
    if "meta" in wl.extra:
        meta = wl.extra["meta"]
        N = int(sum(wl.q_block_sizes))
        slot = torch.from_numpy(meta["slot_token"])
        toks = [I.normal_bf16((wl.B, wl.H, N, wl.D), wl.seed, s) for s in range(3)]
        padded = []
        for t in toks:
            x = torch.zeros((wl.B, wl.H, Sq, wl.D), dtype=torch.bfloat16)
            real = slot >= 0
            x[:, :, real] = t[:, :, slot[real]]
            padded.append(x)
        q, k, v = padded
    else:
        q = I.padded_normal_bhsd(wl.B, wl.H, wl.q_block_sizes, wl.D, wl.seed, I.STREAM_Q, block=wl.block)
        k = I.padded_normal_bhsd(wl.B, wl.H, wl.kv_block_sizes, wl.D, wl.seed, I.STREAM_K, block=wl.block)
        v = I.padded_normal_bhsd(wl.B, wl.H, wl.kv_block_sizes, wl.D, wl.seed, I.STREAM_V, block=wl.block)
    gate = I.gate_bf16((wl.B, Sq, wl.H, wl.D), wl.seed) if wl.gated else None
    return q, k, v, gate


def config_of(wl: I.Workload, flushed: bool) -> dict:
    return {"workload": wl.name, "B": wl.B, "H": wl.H, "D": wl.D, "block": wl.block,
            "seq_q_slots": wl.block * wl.nq, "seq_kv_slots": wl.block * wl.nkv,
            "q_blocks": wl.nq, "kv_blocks": wl.nkv,
            "topk": min(wl.topk, wl.nkv), "gated": wl.gated,
            "selected_tiles_per_gpu": wl.selected_tiles,
            "l2": "L2 flushed between steps (a 252 MB write, outside the timed forward)" if flushed else
                  "inputs larger than L2 (126 MB) every step", "per_gpu_work": "fixed (weak)"}


# ---------------------------------------------------------------------------
# the two arms
# ---------------------------------------------------------------------------
def clock_normalised(ms_per_step: float, ms_sparse: float, clocks: dict) -> dict | None:
    """Time x median SM clock over the timed region, and the times that
    product gives at the maximum clock: a run that the power cap slowed
    (sustained behaviour) and one at full clock (burst) then compare like for
    like."""
    fast = clocks.get("nvml_5ms") or {}
    mhz = fast.get("sm_mhz") or clocks.get("sm_mhz")
    mx = clocks.get("sm_max_mhz")
    if not mhz:
        return None
    res = {"sm_mhz_median": mhz, "ms_x_mhz": ms_per_step * mhz, "sparse_ms_x_mhz": ms_sparse * mhz}
    if mx:
        res["ms_per_step_at_max_clock"] = ms_per_step * mhz / mx
        res["sparse_ms_at_max_clock"] = ms_sparse * mhz / mx
    return res


def max_over_ranks(values, world: int, device):
    """Element-wise maximum of per-rank timings (every rank gets the result;
    the slowest rank sets the job's time)."""
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    if world > 1:
        import torch.distributed as dist
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t]


def weak_scaling_value(world: int, flops_per_rank: float, ms_per_step: float) -> float:
    """Whole-job TFLOP/s: every rank runs its own copy of the workload
    (weak scaling), timed as the maximum over ranks."""
    return world * flops_per_rank / (ms_per_step * 1e-3) / 1e12


def a7_timing(wl: I.Workload, dev, vsa, reps: int = 20) -> dict:
    """a7 device token moves of the tiled workload, timed apart from the
    forward: q's tokens into the padded tile layout (gather) and back
    (scatter), L2 flushed before each launch.
    Algorithmic bytes: gather reads the tokens and writes every slot,
    scatter reads and writes the real tokens."""
    meta = wl.extra["meta"]
    n_tok = int(sum(wl.q_block_sizes))
    G = wl.B * wl.H
    tok = I.normal_bf16((wl.B, wl.H, n_tok, wl.D), wl.seed, I.STREAM_Q).view(G, n_tok, wl.D).to(dev)
    slot = torch.from_numpy(meta["slot_token"]).to(dev)
    flush = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device=dev)
    padded = vsa.gather_tokens(tok, slot)
    vsa.scatter_tokens(padded, slot, n_tok)
    torch.cuda.synchronize(dev)
    res = {}
    for name, fn, nbytes in (
            ("gather", lambda: vsa.gather_tokens(tok, slot), 2 * G * wl.D * (n_tok + slot.numel())),
            ("scatter", lambda: vsa.scatter_tokens(padded, slot, n_tok), 2 * G * wl.D * 2 * n_tok)):
        total = 0.0
        for _ in range(reps):
            # write a buffer twice the L2, then read it back: the L2 then
            # holds clean lines, so the timed kernel pays no write-back of the
            # flush's dirty lines
            flush.fill_(1)
            flush.sum()
            # keep the device busy while the host enqueues the call, so the
            # events time the kernels and not the host's launch overhead
            torch.cuda._sleep(400_000)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            fn()
            e1.record()
            torch.cuda.synchronize(dev)
            total += e0.elapsed_time(e1)
        ms = total / reps
        res[name] = {"ms": ms, "gbs": nbytes / (ms * 1e-3) / 1e9, "bytes": nbytes}
    vsa.check_device_status()
    return res


def run_reference(args, wl):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    q, k, v, gate = host_inputs(wl)
    items = max(1, args.ref_items)
    for _ in range(args.warmup):
        oracle_sample(wl, q, k, v, gate, 0, items)
    times, flops = [], 0.0
    for s in range(args.steps):
        dt, fl = oracle_sample(wl, q, k, v, gate, s % wl.H, items)
        times.append(dt)
        flops += fl
    total = sum(times)
    val = flops / total / 1e12
    sample = (f"fp64 numpy oracle on the host cores: per step, one head's pool + coarse + top-k "
              f"and the sparse attention + combine of its first {items} query blocks")
    line = {"impl": "reference", "metric": METRIC, "value": val, "unit": "TFLOP/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * total / args.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config_of(wl, False),
            "cpu_baseline": {"value": val, "unit": "TFLOP/s", "cores": _blas_threads(),
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": val, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def run_ours(args, wl):
    import torch.distributed as dist
    from block_sparse_attention_15_b200 import binding as vsa

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=dev)

    q_h, k_h, v_h, g_h = host_inputs(wl)
    q, k, v = q_h.to(dev), k_h.to(dev), v_h.to(dev)
    gate = None if g_h is None else g_h.to(dev)
    in_bytes = sum(t.numel() * 2 for t in (q, k, v) + ((gate,) if gate is not None else ()))
    flush = None
    if 2 * in_bytes < 2 * L2_BYTES:
        flush = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device=dev)
    qbs = None if all(s == wl.block for s in wl.q_block_sizes) else torch.tensor(wl.q_block_sizes, dtype=torch.int32, device=dev)
    kbs = None if all(s == wl.block for s in wl.kv_block_sizes) else torch.tensor(wl.kv_block_sizes, dtype=torch.int32, device=dev)
    k_eff = min(wl.topk, wl.nkv)
    qbs_list = None if qbs is None else list(wl.q_block_sizes)
    kbs_list = None if kbs is None else list(wl.kv_block_sizes)
    out = torch.empty_like(q)
    ws_bytes = vsa.lib().vsa_forward_workspace_size(wl.B, wl.H, wl.nq, wl.nkv, wl.D)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        if flush is not None:
            flush.fill_(1)
        vsa.vsa_forward(q, k, v, gate, qbs, kbs, topk=wl.topk, out=out, workspace=ws, block=wl.block)

    sampler = ClockSampler(local)  # nvidia-smi starts up during the warm-up
    for _ in range(max(args.warmup, 3) if args.warmup > 0 else 0):
        step()
    torch.cuda.synchronize(dev)
    vsa.check_device_status()

    # timed region: per-step events plus events around each kernel
    K = args.steps
    ev_step = [torch.cuda.Event(enable_timing=True) for _ in range(K + 1)]
    ev_k = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(K)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    sampler.start()
    ev_step[0].record(stream)
    for i in range(K):
        vsa.set_profile_events(ev_k[i])
        step()
    ev_step[K].record(stream)
    vsa.set_profile_events(None)
    torch.cuda.synchronize(dev)
    clocks = sampler.stop()
    if world > 1:
        dist.barrier()
    status = vsa.get_device_status()
    if status != 0:
        raise RuntimeError(f"device status {status} after the timed region")
    total_ms = ev_step[0].elapsed_time(ev_step[K])
    if flush is not None:
        # the L2 flush between steps is not part of the forward
        total_ms = sum(e[0].elapsed_time(e[3]) for e in ev_k)
    k_pool = sum(e[0].elapsed_time(e[1]) for e in ev_k) / K
    k_coarse = sum(e[1].elapsed_time(e[2]) for e in ev_k) / K
    k_sparse = sum(e[2].elapsed_time(e[3]) for e in ev_k) / K
    total_ms, k_sparse_max = max_over_ranks([total_ms, k_sparse], world, dev)
    ms_per_step = total_ms / K
    flops_gpu = wl.flops
    value = weak_scaling_value(world, flops_gpu, ms_per_step)

    # end to end through the public API with host buffers (page-locked): the
    # host-buffer entry point stages chunks of heads in, runs the forward and
    # copies the output back, overlapping the three
    E = max(1, min(K, args.e2e_steps))
    pin = [x.pin_memory() for x in (q_h, k_h, v_h) + ((g_h,) if g_h is not None else ())]
    out_h = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    gh = pin[3] if g_h is not None else None
    host_ws = torch.empty(vsa.lib().vsa_forward_host_workspace_size(
        wl.B, wl.H, wl.nq, wl.nkv, wl.D, k_eff, 1 if gh is not None else 0, 0)
        if wl.block == 64 else 256, dtype=torch.uint8, device=dev)

    def e2e_step():
        vsa.vsa_forward_host(pin[0], pin[1], pin[2], gh, qbs_list, kbs_list, topk=wl.topk, out=out_h,
                             workspace=host_ws, device=dev)

    if wl.block != 64:
        # the host-buffer entry chunks 64-slot forwards; for other block sizes
        # the step copies the pinned inputs in, runs the forward and copies
        # the output back, in sequence on the stream
        def e2e_step():  # noqa: F811
            q.copy_(pin[0], non_blocking=True)
            k.copy_(pin[1], non_blocking=True)
            v.copy_(pin[2], non_blocking=True)
            if gh is not None:
                gate.copy_(gh, non_blocking=True)
            vsa.vsa_forward(q, k, v, gate, qbs, kbs, topk=wl.topk, out=out, workspace=ws,
                            block=wl.block)
            out_h.copy_(out, non_blocking=True)

    e2e_step()
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(E):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = max_over_ranks([e0.elapsed_time(e1) / E], world, dev)[0]
    h2d = sum(x.numel() * x.element_size() for x in pin)
    d2h = out_h.numel() * out_h.element_size()
    vsa.check_device_status()

    a7 = a7_timing(wl, dev, vsa) if "meta" in wl.extra else None
    if rank == 0:
        peaks, peak_kind = load_peaks()
        peak = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
        sustained = float(peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"]))
        achieved = flops_gpu / (k_sparse * 1e-3) / 1e12
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": K,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": config_of(wl, flush is not None),
            "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                         "frac": achieved / peak, "traffic": profiled_traffic(wl),
                         "kernel": ("sparse_fwd_kernel" if wl.block == 64 else "sparse128_fwd_kernel") +
                                   " (block-sparse attention + fused combine)",
                         "peak_kind": f"{peak_kind} dense bf16 burst (cuBLAS)",
                         "frac_of_sustained": achieved / sustained},
            "kernels_ms": {"pool": k_pool, "coarse_topk": k_coarse, "sparse_combine": k_sparse,
                           "sparse_combine_max_over_ranks": k_sparse_max},
            "forward_frac_of_peak": (flops_gpu / (ms_per_step * 1e-3) / 1e12) / peak,
            "e2e": {"value": weak_scaling_value(world, flops_gpu, e2e_ms), "unit": "TFLOP/s",
                    "ms_per_step": e2e_ms, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
            "gpu_launches": 3 * K,
            "clocks": clocks,
        }
        line["clock_normalised"] = clock_normalised(ms_per_step, k_sparse, clocks)
        # pooling streams q, k and v once: algorithmic bytes = their real tokens
        pool_bytes = 2 * wl.B * wl.H * wl.D * (sum(wl.q_block_sizes) + 2 * sum(wl.kv_block_sizes))
        line["pool_gbs"] = pool_bytes / (k_pool * 1e-3) / 1e9
        if a7 is not None:
            line["a7_tile_layout"] = a7
        if not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(wl, q_h, k_h, v_h, g_h, args.cpu_seconds)
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def run_varlen(args):
    """Varlen entry (a6 + a4): four sequences packed virtually, one call per
    step; the whole call is timed (a small host-to-device copy of the block
    tables, the block-norm and logit-bound launches, then the sparse kernel)."""
    import torch.distributed as dist
    from block_sparse_attention_15_b200 import binding as vsa

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=dev)
    H, D, frac, seed = 24, 128, 0.15, 1004
    q_lens, kv_lens = I.VARLEN_Q_LENS, I.VARLEN_KV_LENS
    cu_q, cu_kv = I.cu_seqlens(q_lens), I.cu_seqlens(kv_lens)
    q_h = I.normal_bf16((H, cu_q[-1], D), seed, I.STREAM_Q)
    k_h = I.normal_bf16((H, cu_kv[-1], D), seed, I.STREAM_K)
    v_h = I.normal_bf16((H, cu_kv[-1], D), seed, I.STREAM_V)
    idx_np, num_np, ks = I.varlen_random_selection(q_lens, kv_lens, H, frac, seed)
    tiles = int(num_np.sum())
    flops = 4.0 * 64 * 64 * D * tiles
    q, k, v = q_h.to(dev), k_h.to(dev), v_h.to(dev)
    idx, num = torch.from_numpy(idx_np).to(dev), torch.from_numpy(num_np).to(dev)
    out = torch.empty_like(q)
    stream = torch.cuda.current_stream(dev)

    def step():
        vsa.block_sparse_attn_varlen(q, k, v, cu_q, cu_kv, idx, num, out=out)

    sampler = ClockSampler(local)
    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize(dev)
    vsa.check_device_status()
    K = args.steps
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    sampler.start()
    e0.record(stream)
    for _ in range(K):
        step()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    clocks = sampler.stop()
    vsa.check_device_status()
    ms = max_over_ranks([e0.elapsed_time(e1) / K], world, dev)[0]
    # end to end: page-locked host tensors copied in, the call, the output copied back
    pin = [x.pin_memory() for x in (q_h, k_h, v_h)]
    out_h = torch.empty(out.shape, dtype=out.dtype).pin_memory()

    def e2e_step():
        q.copy_(pin[0], non_blocking=True)
        k.copy_(pin[1], non_blocking=True)
        v.copy_(pin[2], non_blocking=True)
        step()
        out_h.copy_(out, non_blocking=True)

    E = max(1, min(K, args.e2e_steps))
    e2e_step()
    torch.cuda.synchronize(dev)
    e0.record(stream)
    for _ in range(E):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = max_over_ranks([e0.elapsed_time(e1) / E], world, dev)[0]
    if rank == 0:
        peaks, peak_kind = load_peaks()
        peak = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
        value = weak_scaling_value(world, flops, ms)
        line = {
            "metric": "VSA varlen block-sparse attention ms & effective TFLOPS (selected tiles)",
            "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": K, "warmup": args.warmup,
            "ms_per_step": ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16", "data": "synthetic",
            "config": {"workload": f"varlen: 4 sequences, Q {list(q_lens)}, KV {list(kv_lens)}, H{H} D{D}, "
                                   f"top {frac:.0%} per sequence (k = {ks}), uniformly random selections",
                       "selected_tiles_per_gpu": tiles, "l2": "inputs larger than L2 (126 MB) every step",
                       "per_gpu_work": "fixed (weak)"},
            "roofline": {"bound": "tensor", "achieved": flops / (ms * 1e-3) / 1e12, "peak": peak,
                         "unit": "TFLOP/s", "frac": flops / (ms * 1e-3) / 1e12 / peak, "traffic": None,
                         "kernel": "whole varlen call (block-table copy, norm pass, bound, sparse kernel)",
                         "peak_kind": f"{peak_kind} dense bf16 burst (cuBLAS)"},
            "e2e": {"value": weak_scaling_value(world, flops, e2e_ms), "unit": "TFLOP/s",
                    "ms_per_step": e2e_ms,
                    "h2d_bytes_per_step": sum(x.numel() * x.element_size() for x in pin),
                    "d2h_bytes_per_step": out_h.numel() * out_h.element_size()},
            "gpu_launches": 3 * K,
            "clocks": clocks,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def run_entry(args, wl):
    """Other entry points on the same workload, one call per step, the whole
    call timed: ``indices`` = block_sparse_attn_from_indices (with its
    logit-bound pass) on the selection the forward makes; ``bshd`` = the
    whole forward on BSHD tensors (video_sparse_attn_bshd); ``backward`` =
    block_sparse_attn_backward on that selection (TFLOP/s over 2.5 x the
    forward's tile FLOPs: S recomputed, dP, dV, dK and dQ); ``ulysses`` = the
    sequence-parallel wrapper over the job's ranks (strong scaling: the
    sequence is split, the total work is fixed)."""
    from block_sparse_attention_15_b200 import binding as vsa
    local = int(os.environ.get("LOCAL_RANK", "0"))
    world_env = int(os.environ.get("WORLD_SIZE", "1"))
    if world_env > 1 and args.entry != "ulysses":
        raise SystemExit("--entry other than forward and ulysses runs on one GPU")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if args.entry == "ulysses":
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=dev,
                                init_method="env://" if world_env > 1 else
                                f"tcp://127.0.0.1:{29500 + (os.getpid() % 1000)}",
                                rank=int(os.environ.get("RANK", "0")), world_size=world_env)
    q_h, k_h, v_h, g_h = host_inputs(wl)
    q, k, v = q_h.to(dev), k_h.to(dev), v_h.to(dev)
    gate = None if g_h is None else g_h.to(dev)
    qbs = None if all(s == 64 for s in wl.q_block_sizes) else wl.q_block_sizes
    kbs = None if all(s == 64 for s in wl.kv_block_sizes) else wl.kv_block_sizes
    out, idx, num = vsa.vsa_forward(q, k, v, gate, qbs, kbs, topk=wl.topk, block=wl.block)
    flops = wl.flops
    kernels = None
    if args.entry == "backward":
        # the backward of the sparse attention on the forward's selection:
        # algorithmic work 5 tile products (S recomputed, dP, dV, dK, dQ)
        # = 2.5 x the forward's per tile
        o_s, lse = vsa.block_sparse_attn_from_indices(q, k, v, idx, num, qbs, kbs, block=wl.block,
                                                      return_lse=True)
        dout = I.normal_bf16(tuple(q.shape), wl.seed, 7).to(dev)

        def step():
            vsa.block_sparse_attn_backward(q, k, v, o_s, dout, lse, idx, num, qbs, kbs, block=wl.block)
        if wl.block == 64:
            what = "block_sparse_attn_backward (delta, k2q, dq pass, dk/dv pass) on the forward's selection"
            launches = 4
        else:
            what = ("block_sparse_attn_backward_ex (selection rewrite, delta, k2q, dq pass, dk/dv pass) "
                    "on the forward's selection")
            launches = 5
        flops = 2.5 * wl.flops
    elif args.entry == "ulysses":
        # the sequence-parallel wrapper over the ranks of the job (one rank:
        # the exchanges are the identity; the reshards and the forward run)
        from block_sparse_attention_15_b200 import ulysses as U
        world = int(os.environ.get("WORLD_SIZE", "1"))
        qb, kb, vb = (x.transpose(1, 2).contiguous() for x in (q, k, v))
        del q, k, v
        rank = int(os.environ.get("RANK", "0"))
        Sl, Skl = qb.shape[1] // world, kb.shape[1] // world
        sh = lambda x, s_: x[:, rank * s_:(rank + 1) * s_].contiguous()
        qs_, ks_, vs_ = sh(qb, Sl), sh(kb, Skl), sh(vb, Skl)
        gs_ = None if gate is None else sh(gate, Sl)

        def step():
            U.vsa_forward_ulysses(qs_, ks_, vs_, gs_, qbs, kbs, topk=wl.topk, block=wl.block)
        what = "sequence-parallel forward (row reshards + all-to-all + BSHD forward)"
        launches = 11
    elif args.entry == "indices":
        def step():
            vsa.block_sparse_attn_from_indices(q, k, v, idx, num, qbs, kbs, out=out)
        what = "block_sparse_attn_from_indices with its logit-bound pass, on the forward's selection"
        launches = 3
    else:
        qb, kb, vb = (x.transpose(1, 2).contiguous() for x in (q, k, v))
        del q, k, v
        out_b = torch.empty_like(qb)

        def step():
            vsa.video_sparse_attn_bshd(qb, kb, vb, gate, qbs, kbs, topk=wl.topk, out=out_b)
        what = "whole forward on BSHD q/k/v/out (video_sparse_attn_bshd)"
        launches = 3
    sampler = ClockSampler(local)
    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize(dev)
    vsa.check_device_status()
    stream = torch.cuda.current_stream(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler.start()
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    clocks = sampler.stop()
    vsa.check_device_status()
    ms = e0.elapsed_time(e1) / args.steps
    peaks, peak_kind = load_peaks()
    peak = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    tflops = flops / (ms * 1e-3) / 1e12
    line = {"metric": METRIC + f" [{args.entry} entry]", "value": tflops, "unit": "TFLOP/s",
            "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic", "config": {**config_of(wl, False), "entry": what},
            "roofline": {"bound": "tensor", "achieved": tflops, "peak": peak, "unit": "TFLOP/s",
                         "frac": tflops / peak, "traffic": None, "kernel": f"whole call: {what}",
                         "peak_kind": f"{peak_kind} dense bf16 burst (cuBLAS)"},
            "gpu_launches": launches * args.steps, "clocks": clocks}
    if args.entry == "ulysses":
        import torch.distributed as dist
        line["n_gpus"] = dist.get_world_size()
        line["scaling"] = "strong"
        if dist.get_rank() != 0:
            line = None
        dist.barrier()
        dist.destroy_process_group()
    if line is not None:
        print(json.dumps(line), flush=True)
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="h3")
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--ref-items", type=int, default=24,
                    help="query blocks per reference-arm step (bounded CPU sample)")
    ap.add_argument("--entry", choices=["forward", "indices", "bshd", "backward", "ulysses"],
                    default="forward",
                    help="entry point timed on the workload (forward: the headline line)")
    ap.add_argument("--heads", type=int, default=0,
                    help="override the head count (smaller cases for profiler captures)")
    args = ap.parse_args(argv)
    if args.workload == "varlen":
        if args.impl == "reference":
            print(json.dumps({"impl": "reference", "unavailable": "the reference arm covers the "
                              "default workload; the varlen line has no oracle timing"}), flush=True)
            return 0
        return run_varlen(args)
    wl = make_workload(args.workload)
    if args.heads > 0:
        wl.H = args.heads
        wl.name += f" [H overridden to {args.heads}]"
    if args.impl == "reference":
        return run_reference(args, wl)
    if args.entry != "forward":
        return run_entry(args, wl)
    return run_ours(args, wl)


if __name__ == "__main__":
    sys.exit(main())
