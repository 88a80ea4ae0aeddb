"""Benchmark of the per-step top-k sparse-attention decode path on B200.

Default workload (one GPU): the Qwen3-8B-shaped 128K decode layer -- 16
requests, 8 KV heads of 4 query heads, d = 128, 131072 keys each, a 92-bit
Fathom budget per key, top-2048 per (request, KV head), a 4096-entry hot
buffer per (request, KV head) holding 80% of the selection. One step is one
fused decode_step over the whole batch: bit allocation, bit-plane scan, top-k,
slot lookup and sparse GQA attention.

metric: keys scored per second by the full decode step (each step scores
R*G*n keys); layer-steps/s and achieved HBM GB/s are reported beside it.
Inputs are synthetic (seeded draws with the pages' shapes and distributions)
and stay resident in HBM; every step reads ~350 MB, more than the 126 MB L2,
so no L2 flush is needed between steps.

--impl reference times the CPU oracle (the only reference this method has) on
a bounded sample of the same workload, on the host cores.
Multi-GPU (torchrun): independent replicas, one per GPU (weak scaling); no
collective is on the data path.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

WORKLOADS = {
    # name: R, G, H, n, B, k, S, miss fraction
    "qwen3-8b-128k": dict(R=16, G=8, H=4, n=131072, B=92, k=2048, S=4096, miss=0.2),
    "qwen3-8b-1m": dict(R=4, G=8, H=4, n=1048576, B=92, k=2048, S=4096, miss=0.2),
    "tiny": dict(R=1, G=1, H=4, n=4096, B=92, k=256, S=512, miss=0.2),
}
METRIC = "index-scan keys/s + sparse decode layer-steps/s; achieved GB/s vs HBM peak"
# the dominant kernel of a step with a plan of <= 144 planes: the byte-indexed
# scan, which reads the plan's planes and writes every score and 16-key maximum
SCAN_KERNEL = "fathom_scan_prmt (scan stage of the step)"

# DRAM bytes (read + write) of one launch of the fused scan + top-k kernel, from
# ncu captures of a smaller case of the same workload scaled to a full launch by
# the keys processed (the capture and scaling are stated under profiles/);
# None where no capture of the current kernel exists.
TRAFFIC: dict = {
    # R=8 capture of fathom_scan_prmt_kernel: 96.56 MB read + 9.77 MB written
    # per launch (the rest of its scores leave L2 later), x2 for R=16
    ("qwen3-8b-128k", 92): 2 * (96_558_080 + 9_770_752),
}


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


def _dist():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    if ws > 1:
        import torch.distributed as dist
        import datetime
        rank = int(os.environ["RANK"])
        local = int(os.environ.get("LOCAL_RANK", rank))
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
        return dist, rank, ws
    return None, 0, 1


def _max_over_ranks(dist, x: float) -> float:
    if dist is None:
        return x
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


class Clocks:
    """SM clock and throttle-reason samples taken every 10 ms by an NVML thread
    while the timed region runs (nvidia-smi is the fallback). The sampler is
    started before the region and must have one sample under load before the
    region starts."""

    REASONS = {"hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
               "sw_power_cap": 0x4}

    def __init__(self):
        self.samples = []
        self.reasons = set()
        self.max_mhz = None
        self._stop = False
        self._thread = None
        self._nvml = None

    def _handle(self):
        import pynvml
        pynvml.nvmlInit()
        props = torch.cuda.get_device_properties(torch.cuda.current_device())
        bus = getattr(props, "pci_bus_id", None)
        dom = getattr(props, "pci_domain_id", 0)
        dev = getattr(props, "pci_device_id", 0)
        if bus is not None:
            try:
                return pynvml, pynvml.nvmlDeviceGetHandleByPciBusId(f"{dom:08x}:{bus:02x}:{dev:02x}.0")
            except Exception:
                pass
        idx = int((os.environ.get("CUDA_VISIBLE_DEVICES", "") or str(torch.cuda.current_device())).split(",")[0])
        return pynvml, pynvml.nvmlDeviceGetHandleByIndex(idx)

    def start(self):
        import threading
        try:
            nv, h = self._handle()
        except Exception as e:  # no NVML
            self.reasons.add(f"nvml unavailable: {type(e).__name__}")
            return
        self.max_mhz = nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM)

        def loop():
            while not self._stop:
                try:
                    self.samples.append(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM))
                    r = (nv.nvmlDeviceGetCurrentClocksEventReasons(h)
                         if hasattr(nv, "nvmlDeviceGetCurrentClocksEventReasons")
                         else nv.nvmlDeviceGetCurrentClocksThrottleReasons(h))
                    for name, bit in self.REASONS.items():
                        if r & bit:
                            self.reasons.add(name)
                except Exception:
                    pass
                time.sleep(0.01)

        self._thread = threading.Thread(target=loop, daemon=True)
        self._thread.start()

    def wait_first(self, timeout=2.0):
        t0 = time.time()
        while self._thread is not None and not self.samples and time.time() - t0 < timeout:
            time.sleep(0.005)
        self.samples.clear()

    def stop(self) -> dict:
        self._stop = True
        if self._thread is not None:
            self._thread.join()
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                "samples": len(self.samples)}


def setup(cfg: dict, device, seed: int = 1):
    """Synthetic inputs resident on the device, a warm-up selection, and the hot
    buffers built around it (80% of the selected rows present)."""
    import kv_index_scan_b200 as kvs
    R, G, H, n, B, k, S = (cfg[x] for x in ("R", "G", "H", "n", "B", "k", "S"))
    K, V, nl = synth.fathom_kv(R, G, 128, n, seed=seed, device=device)
    q = synth.queries(R, G, H, 128, seed=seed, device=device)
    index = kvs.build_fathom_index(K, nl)
    warm = kvs.DecodeStep(index, nl, n, H, B, k, K, V)
    warm(q)
    torch.cuda.synchronize()
    sel = warm.idx.cpu().numpy()
    del warm
    slot_map, hot_tok = synth.slot_map_from_selection(sel, nl, n, S, cfg["miss"], seed=seed)
    hotK, hotV = synth.hot_rows(K, hot_tok), synth.hot_rows(V, hot_tok)
    slot_map_t = torch.from_numpy(slot_map).to(device)
    step = kvs.DecodeStep(index, nl, n, H, B, k, K, V, slot_map_t, hotK, hotV)
    return dict(K=K, V=V, q=q, index=index, step=step, nl=nl, slot_map=slot_map_t, hotK=hotK,
                hotV=hotV, sel=sel)


def algorithmic_bytes(cfg: dict) -> dict:
    R, G, n, B, k = (cfg[x] for x in ("R", "G", "n", "B", "k"))
    keys = R * G * n
    scan = keys * B / 8
    rows = R * G * k * (2 * 128 * 2 + 32)  # K + V rows and one 32-byte slot-map sector
    return dict(keys=keys, scan=scan, rows=rows, total=scan + rows)


def time_steps(fn, steps: int, warmup: int, stream) -> float:
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        fn()
    e1.record(stream)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / steps


def run_ours(args, cfg, dist, rank, ws):
    import kv_index_scan_b200 as kvs
    dev = torch.device("cuda", torch.cuda.current_device())
    data = setup(cfg, dev, seed=1 + rank)
    step, q = data["step"], data["q"]
    stream = torch.cuda.current_stream()
    algo = algorithmic_bytes(cfg)

    # ---- device-resident timed region: whole decode steps ----
    for _ in range(args.warmup):
        step(q)
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    # every 8th step records its stage boundaries (decode_step_timed), so the
    # dominant kernel's launch duration is measured inside the timed region at
    # a negligible cost to the others
    nst = len(step.DECODE_STAGES)
    every = 8
    timed_steps = list(range(0, args.steps, every))
    ev = {i: [torch.cuda.Event(enable_timing=True) for _ in range(nst + 1)] for i in timed_steps}
    clocks = Clocks()
    clocks.start()
    clocks.wait_first()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(args.steps):
        if i in ev:
            step.timed(q, ev[i])
        else:
            step(q)
    e1.record(stream)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / args.steps
    clk = clocks.stop()
    stages_ms = {name: sum(ev[i][j].elapsed_time(ev[i][j + 1]) for i in timed_steps) / len(timed_steps)
                 for j, name in enumerate(step.DECODE_STAGES)}
    if dist:
        dist.barrier()
    ms_max = _max_over_ranks(dist, ms)
    if args.only_step:
        if rank == 0:
            print(json.dumps({"ms_per_step": ms_max, "stages_ms": stages_ms}), flush=True)
        return None

    # ---- the bit-plane scan alone (scores to HBM, no top-k), same stream ----
    scan_scores = torch.empty(cfg["R"], cfg["G"], cfg["n"], dtype=torch.float32, device=dev)
    plan = step.plan

    def scan_once():
        kvs.index_scan_fathom(data["index"], plan, step.n, cfg["n"], scores=scan_scores)

    scan_ms = time_steps(scan_once, max(args.steps, 5), 3, stream)

    # ---- end to end through the C ABI with host buffers ----
    # Every step copies its q from pinned host memory and its out, idx and
    # misses back to pinned host memory. The copies run on two copy streams
    # (the copy engines) beside the compute stream: step i's results are read
    # back while step i + 1 computes, into the other of two output sets (two
    # DecodeSteps over the same index and caches).
    R, G, H = cfg["R"], cfg["G"], cfg["H"]
    step_b = kvs.DecodeStep(data["index"], data["nl"], cfg["n"], H, cfg["B"], cfg["k"], data["K"],
                            data["V"], data["slot_map"], data["hotK"], data["hotV"])
    steps2 = (step, step_b)
    q_host = q.cpu().pin_memory()
    out_host = [torch.empty(R, G, H, 128, dtype=torch.float32).pin_memory() for _ in range(2)]
    idx_host = [torch.empty(R, G, cfg["k"], dtype=torch.int32).pin_memory() for _ in range(2)]
    miss_host = [torch.empty(R, G, dtype=torch.int32).pin_memory() for _ in range(2)]
    q_devs = [torch.empty_like(q) for _ in range(2)]
    h2d_stream, d2h_stream = torch.cuda.Stream(), torch.cuda.Stream()
    ev = lambda: torch.cuda.Event()
    q_ready, done, copied = [ev(), ev()], [ev(), ev()], [ev(), ev()]
    for b in range(2):  # every event exists before its first wait
        for e in (q_ready[b], done[b], copied[b]):
            e.record(stream)

    def e2e_once(i):
        b = i & 1
        st = steps2[b]
        with torch.cuda.stream(h2d_stream):
            h2d_stream.wait_event(done[b])  # step i - 2 has read q_devs[b]
            q_devs[b].copy_(q_host, non_blocking=True)
            q_ready[b].record(h2d_stream)
        stream.wait_event(q_ready[b])
        stream.wait_event(copied[b])  # step i - 2's results are on the host
        st(q_devs[b], stream=stream)
        done[b].record(stream)
        with torch.cuda.stream(d2h_stream):
            d2h_stream.wait_event(done[b])
            out_host[b].copy_(st.out, non_blocking=True)
            idx_host[b].copy_(st.idx, non_blocking=True)
            miss_host[b].copy_(st.misses, non_blocking=True)
            copied[b].record(d2h_stream)

    def time_e2e(steps: int, warmup: int) -> float:
        for i in range(warmup):
            e2e_once(i)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for i in range(steps):
            e2e_once(i)
        for b in range(2):  # the region ends when the last results are on the host
            stream.wait_event(copied[b])
        e1.record(stream)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / steps

    e2e_ms = _max_over_ranks(dist, time_e2e(args.steps, args.warmup))
    assert torch.equal(idx_host[(args.steps - 1) & 1], steps2[(args.steps - 1) & 1].idx.cpu())
    q_host_bytes = q_host.numel() * 4
    h2d = q_host_bytes
    d2h = out_host[0].numel() * 4 + idx_host[0].numel() * 4 + miss_host[0].numel() * 4
    misses = int(step.misses.sum().item())

    peak, peak_kind = _peaks()
    keys_total = algo["keys"] * ws
    value = keys_total / (ms_max / 1e3)
    scan_bytes = algo["scan"]
    scan_gbs = scan_bytes / (scan_ms / 1e3) / 1e9
    launches_per_step = 4 + (1 if step_needs_combine(cfg) else 0)  # plan, scan+top-k, merge, attention (+ split merge)
    res = {
        "metric": METRIC, "value": value, "unit": "keys/s", "n_gpus": ws, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_max, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {"workload": args.workload, "requests": R, "kv_heads": G, "q_heads_per_kv": H,
                   "head_dim": 128, "context": cfg["n"], "bits_per_key": cfg["B"],
                   "topk": cfg["k"], "hot_slots": cfg["S"], "miss_rate": cfg["miss"],
                   "parallelism": f"replicas{ws}" if ws > 1 else "single",
                   "l2": "inputs larger than L2 (>=350 MB read per step)"},
        "layer_steps_per_s": ws * 1e3 / ms_max,
        "achieved_gbs": algo["total"] * ws / (ms_max / 1e3) / 1e9,
        "miss_rate_measured": misses / (R * G * cfg["k"]),
        "roofline": {"bound": "hbm", "kernel": SCAN_KERNEL if cfg["B"] <= 144 else "fathom_scan_topk (scan stage of the step)",
                     "achieved": scan_bytes / (stages_ms["scan"] / 1e3) / 1e9, "peak": peak,
                     "peak_kind": peak_kind, "unit": "GB/s",
                     "frac": scan_bytes / (stages_ms["scan"] / 1e3) / 1e9 / peak,
                     "traffic": TRAFFIC.get((args.workload, cfg["B"])),
                     "algorithmic_bytes": scan_bytes, "ms": stages_ms["scan"],
                     "bytes_moved": scan_bytes + algo["keys"] * (4 + 4 / 16) if cfg["B"] <= 144 else None},
        "stages_ms": stages_ms,
        "scan_only": {"kernel": "fathom_scan_lut (scores written to HBM)", "ms": scan_ms,
                      "achieved_gbs": scan_gbs, "frac": scan_gbs / peak},
        "e2e": {"value": keys_total / (e2e_ms / 1e3), "unit": "keys/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms},
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clk,
    }
    if rank == 0 and not args.no_cpu_baseline:
        res["cpu_baseline"] = cpu_baseline(cfg, data, rows=args.cpu_rows)
    return res


def step_needs_combine(cfg) -> bool:
    import kv_index_scan_b200 as kvs
    return kvs._lib.kvs_attn_workspace_size(cfg["R"], cfg["G"], cfg["H"], cfg["k"]) > 0


def cpu_baseline(cfg, data, rows: int = 8, min_seconds: float = 10.0) -> dict:
    """The CPU oracle, as it stands, on a bounded sample of the same workload:
    `rows` (request, KV head) rows of the decode step, all host cores."""
    import oracle
    R, G, H, n, B, k = (cfg[x] for x in ("R", "G", "H", "n", "B", "k"))
    rows = min(rows, R * G)
    us = list(range(rows))
    rr = [u // G for u in us]
    gg = [u % G for u in us]
    K = data["K"][rr, gg].unsqueeze(0).cpu()
    V = data["V"][rr, gg].unsqueeze(0).cpu()
    q = data["q"][rr, gg].unsqueeze(0).cpu()
    nl = [data["nl"][0]]
    sm = data["slot_map"][rr, gg].unsqueeze(0).cpu()
    hK = data["hotK"][rr, gg].unsqueeze(0).cpu()
    hV = data["hotV"][rr, gg].unsqueeze(0).cpu()
    W = synth.plane_words(n)
    planes, kmin, kstep, kvar = oracle.build_index_batch(K, nl, W)  # data prep, not timed
    cores = os.cpu_count() or 1
    reps, t0 = 0, time.perf_counter()
    while True:  # repeat the bounded sample until ~10 s of CPU work
        oracle.decode_batch(q, planes, kmin, kstep, kvar, nl, B, k, sm, hK, hV, K, V,
                            1 / math.sqrt(128), nthreads=cores)
        reps += 1
        dt = time.perf_counter() - t0
        if dt >= min_seconds or reps >= 5000:
            break
    return {"value": reps * rows * n / dt, "unit": "keys/s", "cores": cores, "kind": "oracle",
            "sample": f"{rows} of {R * G} (request, KV head) rows of one decode step "
                      f"({rows * n} keys) x {reps} repetitions, fp64 C++ oracle on {cores} "
                      f"threads, {dt:.1f} s"}


def run_reference(args, cfg, dist, rank, ws):
    """The CPU oracle timed as the reference arm, on the same workload's shape."""
    import oracle
    dev = torch.device("cuda", torch.cuda.current_device()) if torch.cuda.is_available() else "cpu"
    R, G, H, n, B, k, S = (cfg[x] for x in ("R", "G", "H", "n", "B", "k", "S"))
    rows = min(args.cpu_rows, R * G)
    # a sample of rows of the same workload: (rows requests x 1 head) of length n
    K, V, nl = synth.fathom_kv(rows, 1, 128, n, seed=1)
    q = synth.queries(rows, 1, H, 128, seed=1)
    W = synth.plane_words(n)
    planes, kmin, kstep, kvar = oracle.build_index_batch(K, nl, W)
    cores = os.cpu_count() or 1
    ref0 = oracle.decode_batch(q, planes, kmin, kstep, kvar, nl, B, k, None, None, None, K, V,
                               1 / math.sqrt(128), nthreads=cores)
    slot_map, hot_tok = synth.slot_map_from_selection(ref0["idx"], nl, n, S, cfg["miss"], seed=1)
    hK, hV = synth.hot_rows(K, hot_tok), synth.hot_rows(V, hot_tok)

    def one():
        oracle.decode_batch(q, planes, kmin, kstep, kvar, nl, B, k, slot_map, hK, hV, K, V,
                            1 / math.sqrt(128), nthreads=cores)

    for _ in range(args.warmup):
        one()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        one()
    dt = (time.perf_counter() - t0) / args.steps
    v = rows * n / dt
    return {"metric": METRIC, "value": v, "unit": "keys/s", "n_gpus": ws, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": dt * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "impl": "reference",
            "config": {"workload": args.workload, "requests": R, "kv_heads": G,
                       "q_heads_per_kv": H, "head_dim": 128, "context": n, "bits_per_key": B,
                       "topk": k, "hot_slots": S, "miss_rate": cfg["miss"]},
            "cpu_baseline": {"value": v, "unit": "keys/s", "cores": cores, "kind": "oracle",
                             "sample": f"{rows} (request, KV head) rows of {n} keys per step"},
            "e2e": {"value": v, "unit": "keys/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def _time_ms(fn, steps: int, warmup: int) -> float:
    """Median of per-call CUDA-event times on the current stream."""
    stream = torch.cuda.current_stream()
    for _ in range(warmup):
        fn(0)
    torch.cuda.synchronize()
    ts = []
    for i in range(steps):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        fn(i)
        e1.record(stream)
        torch.cuda.synchronize()
        ts.append(e0.elapsed_time(e1))
    return statistics.median(ts)


def run_row(args) -> dict:
    """Measurements of single rows of the path outside the default decode step
    (one JSON line each; not the benchmark's headline line):
      lightning -- the lightning indexer (a2-L) and its block top-k (a3, block
                   64) at 32 requests x 80000 tokens x 64 index heads;
      host-scan -- the Fathom scan reading its planes from mapped pinned host
                   memory (a2-host) at the 1M layer (4 x 8 x 1048576, B = 92),
                   beside the same scan from HBM and a pinned host-to-device
                   copy of the same size (the link's copy rate)."""
    import kv_index_scan_b200 as kvs
    dev = torch.device("cuda")
    peak, peak_kind = _peaks()
    steps, warmup = max(args.steps, 5), max(args.warmup, 3)
    if args.row == "lightning":
        R, n, Hi, Dl, block, k = 32, 80000, 64, 128, 64, 2048
        # two input sets in turn (each 328 MB of index keys, more than L2)
        sets = [synth.lightning_inputs(R, n, Hi, Dl, seed=3 + j, device=dev) for j in range(2)]
        nb = (n + block - 1) // block
        bs = torch.empty(R, nb, dtype=torch.float32, device=dev)
        scan_ms = _time_ms(lambda i: kvs.index_scan_lightning(*sets[i & 1][:3], sets[i & 1][3],
                                                               block=block, scores=bs), steps, warmup)
        idx = torch.empty(R, 1, k, dtype=torch.int32, device=dev)
        topk_ms = _time_ms(lambda i: kvs.topk_select(bs, sets[0][3], k, block=block, idx=idx),
                           steps, warmup)
        kbytes = R * n * Dl
        flops = 2.0 * R * n * Hi * Dl
        return {"row": "a2-L lightning indexer + a3 block top-k", "requests": R, "tokens": n,
                "index_heads": Hi, "block": block, "k": k,
                "scan_ms": scan_ms, "index_keys_per_s": R * n / (scan_ms / 1e3),
                "scan_gbs": kbytes / (scan_ms / 1e3) / 1e9, "hbm_peak_gbs": peak, "peak_kind": peak_kind,
                "scan_frac_hbm": kbytes / (scan_ms / 1e3) / 1e9 / peak,
                "scan_tflops": flops / (scan_ms / 1e3) / 1e12,
                "block_topk_ms": topk_ms, "algorithmic_bytes": kbytes, "flops": flops}
    if args.row == "host-scan":
        R, G, n, B = 4, 8, 1048576, 92
        K, _, nl = synth.fathom_kv(R, G, 128, n, seed=2, device=dev, with_v=False)
        q = synth.queries(R, G, 4, 128, seed=2, device=dev)
        ix = kvs.build_fathom_index(K, nl)
        del K
        plan = kvs.fathom_plan_bits(q, ix, B)
        scores = torch.empty(R, G, n, dtype=torch.float32, device=dev)
        hbm_ms = _time_ms(lambda i: kvs.index_scan_fathom(ix, plan, nl, n, scores=scores), steps, warmup)
        ref = scores.clone()
        hix = kvs.MappedHostIndex(ix)
        host_ms = _time_ms(lambda i: kvs.index_scan_fathom(hix, plan, nl, n, scores=scores),
                           min(steps, 10), 2)
        host_vs_hbm = float((ref - scores).abs().max())
        plane_bytes = R * G * n * B / 8
        # the link's copy rate for the same byte count, from pinned host memory
        host_buf = torch.empty(int(plane_bytes), dtype=torch.uint8).pin_memory()
        dev_buf = torch.empty(int(plane_bytes), dtype=torch.uint8, device=dev)
        copy_ms = _time_ms(lambda i: dev_buf.copy_(host_buf, non_blocking=True), 5, 2)
        return {"row": "a2-host Fathom scan over mapped pinned host memory", "requests": R,
                "kv_heads": G, "context": n, "bits_per_key": B, "plane_bytes": plane_bytes,
                "hbm_scan_ms": hbm_ms, "hbm_keys_per_s": R * G * n / (hbm_ms / 1e3),
                "hbm_scan_gbs": plane_bytes / (hbm_ms / 1e3) / 1e9, "hbm_frac": plane_bytes / (hbm_ms / 1e3) / 1e9 / peak,
                "host_scan_ms": host_ms, "host_keys_per_s": R * G * n / (host_ms / 1e3),
                "host_link_gbs": plane_bytes / (host_ms / 1e3) / 1e9,
                "pinned_copy_gbs": plane_bytes / (copy_ms / 1e3) / 1e9,
                "host_link_frac_of_copy": copy_ms / host_ms,
                "max_abs_diff_vs_hbm_scan": host_vs_hbm}
    raise ValueError(args.row)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="qwen3-8b-128k", choices=sorted(WORKLOADS))
    ap.add_argument("--B", type=int, default=None, help="bits per key (default: the workload's)")
    ap.add_argument("--cpu-rows", type=int, default=8)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--requests", type=int, default=None,
                    help="override the workload's request count (smaller profiling cases)")
    ap.add_argument("--only-step", action="store_true",
                    help="time the decode steps only (no scan-alone, end-to-end or CPU legs); "
                         "prints the step and stage times, for profiling runs")
    ap.add_argument("--row", default=None, choices=["lightning", "host-scan"],
                    help="measure one row of the path outside the decode step (one JSON line)")
    args = ap.parse_args()
    if args.row is not None:
        print(json.dumps(run_row(args)), flush=True)
        return
    cfg = dict(WORKLOADS[args.workload])
    if args.B is not None:
        cfg["B"] = args.B
    if args.requests is not None:
        cfg["R"] = args.requests
    if args.impl == "reference":
        # the CPU oracle: rank 0 alone runs it; other ranks exit without work
        if int(os.environ.get("RANK", "0")) == 0:
            ws = int(os.environ.get("WORLD_SIZE", "1"))
            print(json.dumps(run_reference(args, cfg, None, 0, ws)), flush=True)
        return
    dist, rank, ws = _dist()
    res = run_ours(args, cfg, dist, rank, ws)
    if rank == 0 and res is not None:
        print(json.dumps(res), flush=True)
    if dist:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
