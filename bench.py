#!/usr/bin/env python
"""Benchmark of libdcattn: Lightweight DC attention forward + backward on B200.

One step = dc_attn_fwd + dc_attn_bwd_query + dc_attn_bwd_key over one batch of
the GPT-2-small attention shape (B8 x T2048, H6 x d128, W112, one document per
row, bf16, seeded synthetic inputs).  Prints one JSON line (rank 0).

  python bench.py [--gpus N --steps K --warmup W]      # libdcattn
  python bench.py --impl reference ...                 # the fp64 CPU oracle
  python bench.py --sweep [--steps K --warmup W]       # every workload, one line each

Multi-GPU runs are replicas (the path has no cross-GPU exchange): every rank
runs the same workload on its own GPU; value = all tokens / max-over-ranks time.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from cross_head_dynamic_b200.inputs import CONFIGS, generate  # noqa: E402

METRIC = "DC-attn fwd+bwd tokens/sec and % of roofline on 1 B200 (B8×T2048×H6×d128, W112)"
UNIT = "tokens/s"
WORKLOAD = "gpt2_fwdbwd"
N_SETS = 4                                   # rotating input/output sets, each larger than L2
PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "dram_traffic.txt")
KERNEL_SOURCES = {
    "fwd": ["cross_head_dynamic_b200/csrc/tc_fwd.cuh", "cross_head_dynamic_b200/csrc/tc_common.cuh"],
    "bwd_query": ["cross_head_dynamic_b200/csrc/tc_bwd.cuh", "cross_head_dynamic_b200/csrc/tc_common.cuh"],
    "bwd_key": ["cross_head_dynamic_b200/csrc/tc_bwd.cuh", "cross_head_dynamic_b200/csrc/tc_common.cuh"],
}


def algorithmic_bytes_per_token(H: int, d: int, e: int = 2) -> dict:
    """Minimal HBM bytes per token each kernel must move (no LSE, pmap or ds band):
    fwd reads q,k,v,c,g and writes o; bwd_query reads q,k,v,dO,c,g and writes
    dq,dc,dg; bwd_key (given ds from the query side) reads q,dO,g and writes dk,dv.
    The whole step's minimum counts every tensor once: 11*H*d*e + 24*H."""
    return {
        "fwd": 4 * H * d * e + 8 * H,
        "bwd_query": 5 * H * d * e + 16 * H,
        "bwd_key": 4 * H * d * e + 4 * H,
        "step": 11 * H * d * e + 24 * H,
    }


NOMINAL_HBM_GBS = 8000.0        # the ~8 TB/s HBM3e figure the target is stated against
NOMINAL_BF16_TFLOPS = 2250.0    # dense bf16 tensor peak


def window_lengths(cu_seqlens, W: int):
    """Per-token window length min(W, position in document + 1), as a float64 array."""
    import numpy as np
    cu = [int(x) for x in cu_seqlens]
    out = []
    for a, b in zip(cu[:-1], cu[1:]):
        out.append(np.minimum(np.arange(1, b - a + 1, dtype=np.float64), W))
    return np.concatenate(out) if out else np.zeros(0)


def algorithmic_flops(H: int, d: int, weff_sum: float) -> dict:
    """Window FLOPs (only valid (query, key) pairs count): the forward's two products
    (scores, P.V) are 4 H d per pair; the query side's three (score recompute, E, dQ) 6 H d;
    the key side's two (dV, dK) 4 H d; the step 14 H d."""
    return {"fwd": 4 * H * d * weff_sum, "bwd_query": 6 * H * d * weff_sum,
            "bwd_key": 4 * H * d * weff_sum, "step": 14 * H * d * weff_sum}


def roofline(bytes_: float, flops: float, seconds: float, hbm_gbs: float, tflops: float) -> dict:
    """The slower of the two limits (bytes at HBM bandwidth, FLOPs at the bf16 tensor peak)
    is the bound; achieved and peak are given in that limit's unit."""
    t_mem = bytes_ / (hbm_gbs * 1e9)
    t_tc = flops / (tflops * 1e12)
    if t_mem >= t_tc:
        return {"bound": "hbm", "achieved": bytes_ / seconds / 1e9, "peak": hbm_gbs, "unit": "GB/s",
                "frac": t_mem / seconds, "t_hbm_us": t_mem * 1e6, "t_tensor_us": t_tc * 1e6}
    return {"bound": "tensor", "achieved": flops / seconds / 1e12, "peak": tflops, "unit": "TFLOP/s",
            "frac": t_tc / seconds, "t_hbm_us": t_mem * 1e6, "t_tensor_us": t_tc * 1e6}


def step_dram_bytes(tokens: int):
    """Sum over the step's kernels of the committed ncu DRAM bytes (read + write), scaled to
    `tokens`; None unless every kernel's capture matches its current source."""
    tot = 0.0
    for k in KERNEL_SOURCES:
        t = measured_traffic(k, tokens)
        if t is None:
            return None
        tot += t
    return tot


def source_hash(paths) -> str:
    """SHA-1 of the kernel sources' code: comments and whitespace are dropped, so a
    comment edit keeps a DRAM-traffic capture valid while any code change voids it."""
    import re
    h = hashlib.sha1()
    for p in paths:
        with open(os.path.join(ROOT, p)) as f:
            text = f.read()
        text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
        text = re.sub(r"//[^\n]*", " ", text)
        h.update(" ".join(text.split()).encode())
    return h.hexdigest()[:12]


def measured_traffic(kernel: str, tokens: int):
    """dram bytes per launch from the committed ncu summary, scaled to `tokens`,
    or None when absent or taken on a different version of the kernel source."""
    if not os.path.exists(TRAFFIC_FILE):
        return None
    want = source_hash(KERNEL_SOURCES[kernel])
    for line in open(TRAFFIC_FILE):
        parts = line.split()
        if len(parts) >= 4 and not line.startswith("#") and parts[0] == kernel:
            bytes_per_launch, src, cap_tokens = float(parts[1]), parts[2], int(parts[3])
            if src != want:
                return None
            return bytes_per_launch * tokens / cap_tokens
    return None


class ClockSampler:
    """SM clocks and clock-event reasons while the GPU works.  NVML is polled every 2 ms from a
    host thread, so that a timed region of a few milliseconds still holds samples; without
    NVML, nvidia-smi samples every 100 ms.  Both only read the GPU's state."""

    REASONS = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
    SMI_QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
                 "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
                 "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.samples = []   # (time, sm MHz, max sm MHz, active reasons)
        self.dev = device_index
        self.source = None
        self.proc = None
        self._stop = threading.Event()
        self._thread = None

    def start(self):
        if not self._start_nvml():
            self._start_smi()

    def _start_nvml(self) -> bool:
        try:
            import pynvml as nv
            nv.nvmlInit()
            props = torch.cuda.get_device_properties(self.dev)
            if hasattr(props, "pci_bus_id"):
                bus = f"{getattr(props, 'pci_domain_id', 0):08x}:{props.pci_bus_id:02x}:{props.pci_device_id:02x}.0"
                h = nv.nvmlDeviceGetHandleByPciBusId(bus)
            else:
                h = nv.nvmlDeviceGetHandleByIndex(self.dev)
            mx = nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM)
            get_reasons = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                nv.nvmlDeviceGetCurrentClocksThrottleReasons
            bits = []
            for name, key in zip(self.REASONS, ("HwSlowdown", "HwThermalSlowdown", "SwThermalSlowdown", "SwPowerCap")):
                bits.append((name, getattr(nv, "nvmlClocksEventReason" + key, None) or
                             getattr(nv, "nvmlClocksThrottleReason" + key)))
            nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
            get_reasons(h)
        except Exception:
            return False

        def poll():
            while not self._stop.is_set():
                try:
                    sm = nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
                    r = get_reasons(h)
                    self.samples.append((time.time(), float(sm), float(mx), {n for n, b in bits if r & b}))
                except Exception:
                    pass
                time.sleep(0.002)

        self.source = "nvml, every 2 ms"
        self._thread = threading.Thread(target=poll, daemon=True)
        self._thread.start()
        return True

    def _start_smi(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.dev}", f"--query-gpu={self.SMI_QUERY}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, ValueError):
            self.proc = None
            return
        self.source = "nvidia-smi, every 100 ms"
        self._thread = threading.Thread(target=self._read_smi, daemon=True)
        self._thread.start()

    def _read_smi(self):
        def num(x):
            try:
                return float(x)
            except ValueError:
                return None
        for line in self.proc.stdout:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) >= 9:
                active = {self.REASONS[k] for k in range(4) if parts[5 + k].lower().startswith("active")}
                self.samples.append((time.time(), num(parts[1]), num(parts[2]), active))

    def stop(self):
        self._stop.set()
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
        if self._thread is not None:
            self._thread.join(timeout=2)

    def summary(self, t0: float, t1: float):
        win = [x for x in self.samples if t0 <= x[0] <= t1]
        if not win:
            return None
        sm = [x[1] for x in win if x[1] is not None]
        mx = [x[2] for x in win if x[2] is not None]
        reasons = sorted(set().union(*(x[3] for x in win)))
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(win), "source": self.source}


def dist_setup(n_gpus: int):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def allreduce_max(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], device=dev, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def replica_throughput(tokens_per_rank: int, local_ms: float, steps: int, world: int):
    """Whole-job throughput of `world` replicas that each ran `steps` steps of
    `tokens_per_rank` tokens in `local_ms` (device time): every rank's work over the
    slowest rank's time.  Returns (tokens/s, ms per step)."""
    total_ms = allreduce_max(local_ms, world)
    ms_step = total_ms / steps
    return world * tokens_per_rank / (ms_step * 1e-3), ms_step


def oracle_sample_rate(cfg, rows: int, reps: int = 1):
    """fp64 oracle fwd+bwd on the first `rows` batch rows; tokens/s on host cores."""
    import oracle
    oracle.build()
    sub = cfg.replace(batch=rows)
    x = generate(sub)
    t = time.perf_counter()
    for _ in range(reps):
        oracle.forward(x["q"], x["k"], x["v"], x["c"], x["g"], x["cu_seqlens"], x["window"], x["scale"])
        oracle.backward(x["q"], x["k"], x["v"], x["c"], x["g"], x["dO"], x["cu_seqlens"], x["window"], x["scale"])
    dt = time.perf_counter() - t
    return rows * cfg.seqlen * reps / dt, oracle.num_threads(), dt


_ORACLE_SNIPPET = r'''
import json, sys, time
sys.path.insert(0, {root!r})
import oracle
from cross_head_dynamic_b200.inputs import CONFIGS, generate
oracle.build()
cfg = CONFIGS[{name!r}]
x = generate(cfg.replace(batch=1) if cfg.docs == "rows" else cfg)
n = {tokens}
cu = [int(c) for c in x["cu_seqlens"]]
docs = [c for c in cu if c <= n]
if docs[-1] < n:
    docs.append(n)
cut = lambda t: t[:n]
t = time.perf_counter()
oracle.forward(cut(x["q"]), cut(x["k"]), cut(x["v"]), cut(x["c"]), cut(x["g"]), docs, x["window"], x["scale"])
oracle.backward(cut(x["q"]), cut(x["k"]), cut(x["v"]), cut(x["c"]), cut(x["g"]), cut(x["dO"]), docs, x["window"],
                x["scale"])
dt = time.perf_counter() - t
print(json.dumps({{"tokens_per_s": n / dt, "seconds": dt, "threads": oracle.num_threads()}}))
'''


def oracle_sample_subprocess(name: str, tokens: int, threads: int = 0):
    """fp64 oracle fwd+bwd on the first `tokens` tokens of workload `name` (its first batch row;
    the documents cut at that point), in a fresh process (OMP_NUM_THREADS=threads when > 0).
    Returns the parsed JSON result, or None if the sample could not run."""
    env = dict(os.environ)
    if threads > 0:
        env["OMP_NUM_THREADS"] = str(threads)
    code = _ORACLE_SNIPPET.format(root=ROOT, name=name, tokens=int(tokens))
    try:
        res = subprocess.run([sys.executable, "-c", code], env=env, capture_output=True, text=True, timeout=600)
        return json.loads(res.stdout.strip().splitlines()[-1])
    except (subprocess.SubprocessError, ValueError, IndexError):
        return None


def config_block(cfg, n_gpus):
    return {"workload": f"{WORKLOAD}: B{cfg.batch} x T{cfg.seqlen}, H{cfg.heads} x d{cfg.head_dim}, "
                        f"W{cfg.window}, one document per row, bf16 q/k/v/dO, fp32 c/g",
            "tokens_per_gpu": cfg.total_tokens, "global_batch": cfg.batch * n_gpus, "seq_len": cfg.seqlen,
            "heads": cfg.heads, "head_dim": cfg.head_dim, "window": cfg.window,
            "parallelism": f"replicas x{n_gpus}",
            "l2": f"{N_SETS} rotating input/output sets of ~190 MB each (> 126 MB L2)"}


def run_reference(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    cfg = CONFIGS[WORKLOAD]
    rows = 1
    for _ in range(args.warmup):
        oracle_sample_rate(cfg, rows)
    rates, cores = [], 1
    t_all = 0.0
    for _ in range(args.steps):
        r, cores, dt = oracle_sample_rate(cfg, rows)
        rates.append(r)
        t_all += dt
    value = args.steps * rows * cfg.seqlen / t_all
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * t_all / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": config_block(cfg, 1),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                             "sample": f"fwd+bwd of {rows} row x {cfg.seqlen} tokens of the workload per step"},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def run_sweep(args):
    """One JSON line per workload of the inputs module (rank 0 only): the same graph-timed
    step (forward, plus both backward kernels where the workload has a backward) on two
    rotating input sets, with the step's fraction of the HBM roofline.  Shows which kernels
    serve each shape (tcgen05 or SIMT)."""
    from cross_head_dynamic_b200 import build, dcattn
    if int(os.environ.get("RANK", "0")) != 0:
        return 0
    torch.cuda.set_device(0)
    build.build()
    dcattn.load_library()
    dev = torch.device("cuda", 0)
    peaks = json.load(open(PEAKS_FILE)) if os.path.exists(PEAKS_FILE) else {}
    hbm = peaks.get("hbm_gbs") or 6650.0
    tflops = peaks.get("bf16_tflops_sustained") or 1400.0
    for name, cfg in CONFIGS.items():
        if args.workload and name not in args.workload:
            continue
        host = generate(cfg)
        N, H, d, W, scale = cfg.total_tokens, cfg.heads, cfg.head_dim, cfg.window, cfg.softmax_scale
        dt = host["q"].dtype
        impl = dcattn.dc_attn_resolve_impl(host["q"].to(dev), host["cu_seqlens"].to(dev), W, scale)
        sets = []
        for r in range(2):
            x = {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in host.items()}
            if r:
                for k in ("q", "k", "v", "dO"):
                    if isinstance(x.get(k), torch.Tensor):
                        x[k] = x[k].roll(1, dims=0).contiguous()
            x["o"] = torch.empty_like(x["q"])
            x["lse"] = torch.empty(N, H, device=dev)
            x["pmap"] = torch.empty(N, W, device=dev, dtype=dt)
            if cfg.backward:
                x["dq"], x["dk"], x["dv"] = (torch.empty_like(x["q"]) for _ in range(3))
                x["dc"], x["dg"] = torch.empty(N, H, device=dev), torch.empty(N, H, device=dev)
                x["ws"] = torch.empty(max(16, dcattn.dc_attn_bwd_workspace_size(x["q"], x["cu_seqlens"], W, scale)),
                                      device=dev, dtype=torch.uint8)
            sets.append(x)

        def step(x):
            dcattn.dc_attn_fwd(x["q"], x["k"], x["v"], x["c"], x["g"], x["cu_seqlens"], W, scale,
                               o=x["o"], lse=x["lse"], pmap=x["pmap"])
            if cfg.backward:
                dcattn.dc_attn_bwd_query(x["q"], x["k"], x["v"], x["c"], x["g"], x["dO"], x["lse"], x["pmap"],
                                         x["cu_seqlens"], W, scale, dq=x["dq"], dc=x["dc"], dg=x["dg"],
                                         workspace=x["ws"])
                dcattn.dc_attn_bwd_key(x["q"], x["k"], x["c"], x["g"], x["dO"], x["lse"], x["pmap"], x["dc"],
                                       x["ws"], x["cu_seqlens"], W, scale, dk=x["dk"], dv=x["dv"])

        for x in sets:
            step(x)
        torch.cuda.synchronize()
        graphs = []
        for x in sets:
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                step(x)
            graphs.append(g)
        for it in range(args.warmup):
            graphs[it % 2].replay()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        for it in range(args.steps):
            graphs[it % 2].replay()
        b.record()
        torch.cuda.synchronize()
        if dcattn.dc_attn_device_status() != 0:
            raise RuntimeError(f"device status word reports an error on {name}")
        ms = a.elapsed_time(b) / args.steps
        e = 4 if cfg.dtype == "f32" else 2
        per_tok = (11 * H * d * e + 24 * H) if cfg.backward else (4 * H * d * e + 8 * H)
        flops = algorithmic_flops(H, d, float(window_lengths(host["cu_seqlens"], W).sum()))
        rl = roofline(per_tok * N, flops["step"] if cfg.backward else flops["fwd"], ms * 1e-3, hbm, tflops)
        print(json.dumps({"workload": name, "pass": "fwd+bwd" if cfg.backward else "fwd", "kernels": impl,
                          "tokens": N, "heads": H, "head_dim": d, "window": W, "dtype": cfg.dtype,
                          "docs": cfg.docs, "ms_per_step": ms, "tokens_per_s": N / (ms * 1e-3),
                          "roofline": dict(rl, algorithmic_bytes_per_token=per_tok)}), flush=True)
        del graphs, sets
        torch.cuda.empty_cache()
    return 0


# The producer of c and g (assumed per-token affine form), measured beside the headline
# step at the GPT-2 width: x [N][768] bf16 -> c, g [N][6] fp32, and its backward.
CG_SHAPE = (16384, 768, 6)
CG_SETS = 6                                  # rotating x sets: 6 x 25 MB, larger than L2


def cg_measure(dev, hbm_gbs: float, peak_note: str, reps: int = 60) -> dict:
    """Graph-timed forward and backward of the c/g producer; rooflines from algorithmic
    bytes (x read once, c and g written; backward: x and e read, dx written, dweight and
    dbias written; the partial-sum records in the workspace are not algorithmic)."""
    from cross_head_dynamic_b200 import dcattn
    from cross_head_dynamic_b200.inputs import cg_problem
    N, D, H = CG_SHAPE
    sets = []
    for i in range(CG_SETS):
        p = cg_problem(1000 + i, N, D, H, "bf16")
        x = {k: v.to(dev) for k, v in p.items()}
        x["wt"] = x["w"].t().contiguous()
        x["c"], x["gg"] = torch.empty(N, H, device=dev), torch.empty(N, H, device=dev)
        x["dx"], x["dw"], x["db"] = torch.empty_like(x["x"]), torch.empty_like(x["wt"]), torch.empty_like(x["b"])
        x["ws"] = torch.empty(dcattn.dc_attn_cg_bwd_workspace_size(x["x"], H), device=dev, dtype=torch.uint8)
        x["img"] = dcattn.dc_attn_cg_prepare(x["wt"])
        sets.append(x)
    # A training step converts its weight once (prepare) and runs forward and backward on it.
    calls = {
        "fwd": lambda x: dcattn.dc_attn_cg_fwd(x["x"], x["wt"], x["b"], c=x["c"], g=x["gg"], weight_splits=x["img"]),
        "bwd": lambda x: dcattn.dc_attn_cg_bwd(x["x"], x["wt"], x["dc"], x["dg"], dx=x["dx"], dweight=x["dw"],
                                               dbias=x["db"], workspace=x["ws"], weight_splits=x["img"]),
        "prepare": lambda x: dcattn.dc_attn_cg_prepare(x["wt"], splits=x["img"]),
    }
    launches = {}
    out = {}
    stream = torch.cuda.current_stream()
    for name, call in calls.items():   # one direct call of each first: fwd, then the backward's kernels
        call(sets[0])
        launches[name] = dcattn.dc_attn_last_launch_count()
    for name, call in calls.items():
        graphs = []
        for x in sets:
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                call(x)
            graphs.append(g)
        for it in range(2 * CG_SETS):
            graphs[it % CG_SETS].replay()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for it in range(reps):
            graphs[it % CG_SETS].replay()
        b.record(stream)
        torch.cuda.synchronize()
        out[name] = a.elapsed_time(b) / reps * 1e3   # us per call
        del graphs
    if dcattn.dc_attn_device_status() != 0:
        raise RuntimeError("device status word reports an error after the c/g producer")
    xb, eb = N * D * 2, N * 2 * H * 4
    fwd_bytes = xb + eb + 2 * H * D * 4
    bwd_bytes = 2 * xb + eb + 2 * H * D * 4 + 2 * H * 4
    flops = 2.0 * N * D * 2 * H
    res = {"workload": f"x [{N}][{D}] bf16, H = {H} (c, g fp32); {CG_SETS} rotating input sets (> L2)",
           "form": "assumed per-token affine map (the pages give no formula)"}
    res["prepare"] = {"us": out["prepare"], "launches": launches["prepare"],
                      "note": "the weight's bf16 splits for the tensor-core kernels, once per weight update"}
    res["step_us"] = out["prepare"] + out["fwd"] + out["bwd"]
    for name, nbytes, nflops in (("fwd", fwd_bytes, flops), ("bwd", bwd_bytes, 2 * flops)):
        t = out[name] * 1e-6
        res[name] = {"us": out[name], "launches": launches[name], "algorithmic_bytes": nbytes,
                     "fp32_flops": nflops,
                     "roofline": {"bound": "hbm", "achieved": nbytes / t / 1e9, "peak": hbm_gbs, "unit": "GB/s",
                                  "frac": nbytes / t / 1e9 / hbm_gbs, "peak_source": peak_note}}
    return res


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["dcattn", "reference"], default="dcattn")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-next-rows", action="store_true", help="skip the c/g producer measurement")
    ap.add_argument("--cg-only", action="store_true",
                    help="only the c/g producer measurement (--steps graph replays per pass)")
    ap.add_argument("--sweep", action="store_true",
                    help="one JSON line per workload of the inputs module instead of the headline line")
    ap.add_argument("--workload", action="append", choices=list(CONFIGS),
                    help="with --sweep: only these workloads (repeatable)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        return run_reference(args)
    if args.sweep:
        return run_sweep(args)
    if args.cg_only:
        from cross_head_dynamic_b200 import build, dcattn
        torch.cuda.set_device(0)
        build.build()
        dcattn.load_library()
        peaks = json.load(open(PEAKS_FILE)) if os.path.exists(PEAKS_FILE) else {}
        hbm = peaks.get("hbm_gbs")
        note = "of measured" if hbm else "of fallback"
        print(json.dumps({"next_rows": {"cg_producer": cg_measure(torch.device("cuda", 0), hbm or 6650.0, note,
                                                                  reps=max(args.steps, 4))}}), flush=True)
        return 0

    from cross_head_dynamic_b200 import build, dcattn
    world, rank, local = dist_setup(args.gpus)
    if world == 1:
        torch.cuda.set_device(0)
    build.build()
    dcattn.load_library()
    dev = torch.device("cuda", torch.cuda.current_device())
    cfg = CONFIGS[WORKLOAD]
    host = generate(cfg)
    N, H, d, W, scale = cfg.total_tokens, cfg.heads, cfg.head_dim, cfg.window, cfg.softmax_scale
    impl = dcattn.dc_attn_resolve_impl(host["q"].to(dev), host["cu_seqlens"].to(dev), W, scale)

    # rotating sets of device-resident inputs and outputs
    sets = []
    for _ in range(N_SETS):
        x = {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in host.items()}
        x["o"] = torch.empty_like(x["q"])
        x["lse"] = torch.empty(N, H, device=dev)
        x["pmap"] = torch.empty(N, W, device=dev, dtype=torch.bfloat16)
        x["dq"], x["dk"], x["dv"] = (torch.empty_like(x["q"]) for _ in range(3))
        x["dc"], x["dg"] = torch.empty(N, H, device=dev), torch.empty(N, H, device=dev)
        x["ws"] = torch.empty(dcattn.dc_attn_bwd_workspace_size(x["q"], x["cu_seqlens"], W, scale),
                              device=dev, dtype=torch.uint8)
        sets.append(x)
    stream = torch.cuda.current_stream()
    launches = [0]

    def step(x, ev=None):
        # everything on the current stream (the capture stream while a graph is recorded)
        if ev is not None:
            ev[0].record()
        dcattn.dc_attn_fwd(x["q"], x["k"], x["v"], x["c"], x["g"], x["cu_seqlens"], W, scale,
                           o=x["o"], lse=x["lse"], pmap=x["pmap"])
        launches[0] += dcattn.dc_attn_last_launch_count()
        if ev is not None:
            ev[1].record()
        dcattn.dc_attn_bwd_query(x["q"], x["k"], x["v"], x["c"], x["g"], x["dO"], x["lse"], x["pmap"],
                                 x["cu_seqlens"], W, scale, dq=x["dq"], dc=x["dc"], dg=x["dg"], workspace=x["ws"])
        launches[0] += dcattn.dc_attn_last_launch_count()
        if ev is not None:
            ev[2].record()
        dcattn.dc_attn_bwd_key(x["q"], x["k"], x["c"], x["g"], x["dO"], x["lse"], x["pmap"], x["dc"], x["ws"],
                               x["cu_seqlens"], W, scale, dk=x["dk"], dv=x["dv"])
        launches[0] += dcattn.dc_attn_last_launch_count()
        if ev is not None:
            ev[3].record()

    sampler = ClockSampler(local)
    sampler.start()
    time.sleep(0.3)
    for it in range(args.warmup):
        step(sets[it % N_SETS])
    torch.cuda.synchronize()
    if dcattn.dc_attn_device_status() != 0:
        raise RuntimeError("device status word reports an error after warm-up")

    # Timed region: one CUDA graph per input set holds one whole step (the three kernels);
    # the graphs are replayed back to back with nothing between the kernels.
    graphs = []
    launches[0] = 0
    for x in sets:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            step(x)
        graphs.append(g)
    launches_per_step = launches[0] // N_SETS
    torch.cuda.synchronize()
    for it in range(args.warmup):
        graphs[it % N_SETS].replay()
    torch.cuda.synchronize()
    if dcattn.dc_attn_device_status() != 0:
        raise RuntimeError("device status word reports an error after the graph warm-up")
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    t_wall0 = time.time()
    t_start.record(stream)
    for it in range(args.steps):
        graphs[it % N_SETS].replay()
    t_end.record(stream)
    torch.cuda.synchronize()
    t_wall1 = time.time()
    barrier(world)
    total_ms = t_start.elapsed_time(t_end)
    gpu_launches = launches_per_step * args.steps

    # Per-kernel split: a second timed pass of the same steps, launched directly on the
    # stream with CUDA events between the kernels (events inside the timed graphs would
    # themselves slow the step down).
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    torch.cuda.synchronize()
    for it in range(args.steps):
        step(sets[it % N_SETS], evs[it])
    torch.cuda.synchronize()
    names = ("fwd", "bwd_query", "bwd_key")
    per_kernel_eager = {n: sum(ev[j].elapsed_time(ev[j + 1]) for ev in evs) / args.steps
                        for j, n in enumerate(names)}   # ms per launch
    split_ms_step = evs[0][0].elapsed_time(evs[-1][3]) / args.steps
    value, ms_step = replica_throughput(N, total_ms, args.steps, world)

    # Per-kernel time without launch gaps: each kernel alone, one CUDA graph per input set
    # holding 4 launches of it, replayed back to back and timed with CUDA events on the
    # launching stream (the kernels that surround it in a step are absent, so the cache state
    # differs slightly from the step's).
    kernel_calls = {
        "fwd": lambda x: dcattn.dc_attn_fwd(x["q"], x["k"], x["v"], x["c"], x["g"], x["cu_seqlens"], W, scale,
                                            o=x["o"], lse=x["lse"], pmap=x["pmap"]),
        "bwd_query": lambda x: dcattn.dc_attn_bwd_query(x["q"], x["k"], x["v"], x["c"], x["g"], x["dO"], x["lse"],
                                                        x["pmap"], x["cu_seqlens"], W, scale, dq=x["dq"], dc=x["dc"],
                                                        dg=x["dg"], workspace=x["ws"]),
        "bwd_key": lambda x: dcattn.dc_attn_bwd_key(x["q"], x["k"], x["c"], x["g"], x["dO"], x["lse"], x["pmap"],
                                                    x["dc"], x["ws"], x["cu_seqlens"], W, scale, dk=x["dk"],
                                                    dv=x["dv"]),
    }
    per_kernel = {}
    reps_per_graph, kernel_replays = 4, max(8, min(args.steps, 40))
    for kname, call in kernel_calls.items():
        kg = []
        for x in sets:
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                for _ in range(reps_per_graph):
                    call(x)
            kg.append(g)
        for it in range(N_SETS):
            kg[it].replay()
        ka, kb = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ka.record(stream)
        for it in range(kernel_replays):
            kg[it % N_SETS].replay()
        kb.record(stream)
        torch.cuda.synchronize()
        per_kernel[kname] = ka.elapsed_time(kb) / (kernel_replays * reps_per_graph)
        del kg

    clocks = sampler.summary(t_wall0, t_wall1)
    clock_note = "sampled during the timed region"
    if clocks is None or clocks.get("samples", 0) < 3:
        # the timed region was too short for the sampler: keep the same step running
        # (untimed) for about a second and sample that
        t2 = time.time()
        it = 0
        while time.time() - t2 < 1.2:
            graphs[it % N_SETS].replay()
            it += 1
            if it % 50 == 0:
                torch.cuda.synchronize()
        torch.cuda.synchronize()
        clocks = sampler.summary(t2, time.time())
        clock_note = "sampled over ~1 s of the same step right after the timed region"
    sampler.stop()

    # end to end through the public API: pinned host inputs -> device -> fwd+bwd -> host
    # results, every step.  The copies run on their own streams, so step i's upload and
    # step i-1's read-back overlap step i's kernels (as a training loop would pipeline them);
    # each set's buffers are reused only after their previous read-back has finished.
    e2e = None
    pin = {k: host[k].pin_memory() for k in ("q", "k", "v", "c", "g", "dO", "cu_seqlens")}
    out_keys = ("o", "dq", "dk", "dv", "dc", "dg")
    outs_host = [{k: torch.empty(sets[0][k].shape, dtype=sets[0][k].dtype).pin_memory() for k in out_keys}
                 for _ in range(N_SETS)]
    h2d = sum(t.numel() * t.element_size() for t in pin.values())
    d2h = sum(t.numel() * t.element_size() for t in outs_host[0].values())
    up, down = torch.cuda.Stream(), torch.cuda.Stream()
    e2e_steps = max(3, min(args.steps, 20))

    def e2e_run(n):
        freed = [None] * N_SETS            # read-back of the set's previous outputs done
        for it in range(n):
            si = it % N_SETS
            x = sets[si]
            ev_in = torch.cuda.Event()
            with torch.cuda.stream(up):
                if freed[si] is not None:
                    up.wait_event(freed[si])
                for k2 in pin:
                    x[k2].copy_(pin[k2], non_blocking=True)
                ev_in.record(up)
            stream.wait_event(ev_in)
            if freed[si] is not None:
                stream.wait_event(freed[si])
            step(x)
            ev_out = torch.cuda.Event()
            ev_out.record(stream)
            with torch.cuda.stream(down):
                down.wait_event(ev_out)
                for k2 in out_keys:
                    outs_host[si][k2].copy_(x[k2], non_blocking=True)
                done = torch.cuda.Event()
                done.record(down)
            freed[si] = done
        for f in freed:
            if f is not None:
                stream.wait_event(f)

    e2e_run(3)
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    e2e_run(e2e_steps)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = allreduce_max(e0.elapsed_time(e1) / e2e_steps, world)
    e2e = {"value": world * N / (e2e_ms * 1e-3), "unit": UNIT, "h2d_bytes_per_step": h2d,
           "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms,
           "note": "dc_attn_* calls; inputs uploaded and outputs read back every step on copy streams "
                   "that overlap neighbouring steps"}

    # rooflines: the slower of (algorithmic bytes at the measured HBM copy bandwidth) and
    # (window FLOPs at the measured bf16 tensor peak); the dominant kernel and the whole step
    peaks = json.load(open(PEAKS_FILE)) if os.path.exists(PEAKS_FILE) else {}
    hbm = peaks.get("hbm_gbs")
    peak_note = "of measured" if hbm else "of fallback"
    hbm = hbm or 6650.0
    # the kernels run back to back for many steps: the sustained GEMM figure applies
    tflops = peaks.get("bf16_tflops_sustained") or (1400.0 if not peaks else peaks.get("bf16_tflops"))
    abytes = algorithmic_bytes_per_token(H, d)
    weff = float(window_lengths(host["cu_seqlens"], W).sum())
    aflops = algorithmic_flops(H, d, weff)
    dom = max(per_kernel, key=per_kernel.get)
    rl = roofline(abytes[dom] * N, aflops[dom], per_kernel[dom] * 1e-3, hbm, tflops)
    traffic = measured_traffic(dom, N)
    step_rl = roofline(abytes["step"] * N, aflops["step"], ms_step * 1e-3, hbm, tflops)
    step_rl_nominal = roofline(abytes["step"] * N, aflops["step"], ms_step * 1e-3, NOMINAL_HBM_GBS,
                               NOMINAL_BF16_TFLOPS)
    step_dram = step_dram_bytes(N)

    cg = cg_measure(dev, hbm, peak_note) if not args.no_next_rows else None

    cpu = None
    if rank == 0 and not args.no_cpu_baseline:
        rate, cores, dt = oracle_sample_rate(cfg, rows=cfg.batch)
        cpu = {"value": rate, "unit": UNIT, "cores": cores, "kind": "oracle",
               "sample": f"one fwd+bwd of all {cfg.total_tokens} tokens of the workload in fp64 ({dt:.1f} s)"}
        # the same oracle on one thread, and on samples of the packed varlen batch and of the
        # widest-window sweep point (their first 4096 tokens, documents cut there)
        extra = {}
        one = oracle_sample_subprocess(WORKLOAD, 2048, threads=1)
        if one:
            extra["one_thread"] = {"value": one["tokens_per_s"], "unit": UNIT, "cores": 1,
                                   "sample": "fwd+bwd of the first 2048 tokens (one batch row) of the workload"}
        for wname in ("varlen", "sweep_W256_H6_d128"):
            r = oracle_sample_subprocess(wname, 4096)
            if r:
                extra[wname] = {"value": r["tokens_per_s"], "unit": UNIT, "cores": r["threads"],
                                "sample": f"fwd+bwd of the first 4096 tokens of {wname}"}
        cpu["other_samples"] = extra

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic", "impl": "dcattn", "kernels": impl,
            "config": config_block(cfg, world),
            "timing": (f"value: {args.steps} back-to-back replays of one CUDA graph per input set (one graph = "
                       f"one fwd+bwd step, {launches_per_step} kernels), CUDA events on the launching stream; "
                       f"kernel_ms: each kernel alone, {reps_per_graph} launches per graph, {kernel_replays} "
                       f"replays; kernel_ms_eager: a pass of the {args.steps} steps launched directly with "
                       f"CUDA events between the kernels ({split_ms_step * 1e3:.1f} us per step there)"),
            "roofline": dict(rl, kernel=dom, peak_source=peak_note, traffic=traffic,
                             algorithmic_bytes_per_launch=abytes[dom] * N,
                             algorithmic_flops_per_launch=aflops[dom]),
            "step_roofline": dict(step_rl, peak_source=peak_note,
                                  frac_nominal_peaks=step_rl_nominal["frac"],
                                  nominal_peaks={"hbm_gbs": NOMINAL_HBM_GBS, "bf16_tflops": NOMINAL_BF16_TFLOPS},
                                  algorithmic_bytes_per_step=abytes["step"] * N,
                                  algorithmic_flops_per_step=aflops["step"],
                                  dram_bytes_per_step_ncu=step_dram,
                                  roofline_tokens_per_s=hbm * 1e9 / abytes["step"]),
            "kernel_ms": per_kernel,
            "kernel_ms_eager": per_kernel_eager,
            "cpu_baseline": cpu,
            "next_rows": {"cg_producer": cg},
            "e2e": e2e,
            "gpu_launches": gpu_launches,
            "clocks": dict(clocks or {}, note=clock_note),
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
