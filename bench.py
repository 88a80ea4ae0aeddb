"""Benchmark of the per-step top-k sparse-attention decode path on B200.

Headline workload (one GPU): the Qwen3-8B-shaped 128K decode layer -- 16
requests, 8 KV heads of 4 query heads, d = 128, 131072 keys each, a 92-bit
Fathom budget per key, top-2048 per (request, KV head), a 4096-entry hot
buffer per (request, KV head) holding 80% of the selection. One step is one
fused decode_step over the whole batch: bit allocation, bit-plane scan, top-k,
slot lookup and sparse GQA attention.

metric: keys scored per second by the full decode step (each step scores
R*G*n keys); layer-steps/s and achieved HBM GB/s are reported beside it.
Inputs are synthetic (seeded draws with the pages' shapes and distributions)
and stay resident in HBM; every step reads more than the 126 MB L2, so no L2
flush is needed between steps.

The same JSON line carries, under "configs", one entry per other measured
workload, each timed with the same --steps/--warmup and each with its own
roofline (algorithmic bytes of its dominant kernel / that kernel's CUDA-event
time / the measured peak) and a short CPU-oracle sample:
  128k-B68, 128k-B136, 128k-B512  the 128K layer at the other budgets;
  128k-hosttier-miss20, -miss40   the 128K step with the full K/V store in
                                  mapped pinned host memory: the missing
                                  selected rows (20% / 40%) cross the host link
                                  each step; against the all-in-HBM step;
  1m-B92, 1m-B136                 the 1M layer (4 x 8 x 1048576), index in HBM;
  1m-host-B92                     the 1M layer with the index planes in mapped
                                  pinned host memory, read by the scan over
                                  the host link (roofline: a pinned
                                  host-to-device copy measured in the run);
  lightning-pair                  32 requests x 80000 tokens: lightning
                                  indexer (64 heads, tcgen05), block top-k,
                                  and sparse attention for both layers of a
                                  group reusing one selection;
  selection-quality               a diagnostic: top-k recall against the exact
                                  bf16-K top-k and attention error against
                                  dense attention, for the Fathom allocation
                                  at 68/92/136 bits and a SparQ-like scan of
                                  the B/4 largest-|qbar| channels at equal bits;
  sweep-36-layers                 ragged batches of 1 .. 256 requests (lengths
                                  log-uniform in [16K, 128K]) over 36 layers:
                                  each batch's footprint against 180 GB, and for
                                  the batches that fit, one layer's decode step
                                  timed (the 36 layers have the same shape).
--only-headline skips them.

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
import sys
import threading
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
LIGHTNING = dict(R=32, n=80000, Hi=64, Dl=128, block=64, k=2048, G=8, H=4)
# the concurrency sweep: ragged batches over 36 layers, capped by 180 GB of HBM
SWEEP = dict(layers=36, batches=(1, 2, 4, 8, 16, 32, 64, 128, 256), G=8, H=4, B=92, k=2048, S=4096,
             lo=16384, hi=131072, cap_gb=180.0, miss=0.2, seed=4)
METRIC = "index-scan keys/s + sparse decode layer-steps/s; achieved GB/s vs HBM peak"

# DRAM bytes (read + write) of one launch of the scan kernel, from ncu
# captures of a smaller case of the same workload scaled to a full launch by
# the keys processed (the capture and scaling are stated under profiles/);
# keyed by (workload, B, kernel). Absent where no capture of the current kernel
# exists.
TRAFFIC: dict = {
    # R=8 capture of fathom_scan_prmt_kernel: 96.56 MB read + 11.36 MB written
    # per launch (the rest of its scores leave L2 later), x2 for R=16
    ("qwen3-8b-128k", 92, "fathom_scan_prmt"): 2 * (96_562_432 + 11_357_184),
    # full capture of lightning_scan_kernel<4> at 32 x 80000 tokens x 64 heads
    # (the bench's own workload): 328.70 MB read + 4.64 MB written per launch
    ("minimax-lightning-32x80000", 64, "lightning_scan"): 328_696_832 + 4_638_720,
}


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), float(d.get("bf16_tflops", 1590.0)), "measured"
    return 6650.0, 1590.0, "fallback"


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
    """SM clock and throttle-reason samples from an NVML thread, about every
    0.2 ms for as long as the benchmark runs GPU work. Each timed region is
    marked by host timestamps taken just before its first launch and just
    after its closing synchronize; a region's clock record is the samples that
    fall inside it (the headline region of 20 steps lasts a few ms)."""

    REASONS = {"hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
               "sw_power_cap": 0x4}

    def __init__(self):
        self.samples = []  # (host time, sm MHz, reason bits)
        self.max_mhz = None
        self.error = None
        self._stop = False
        self._thread = None

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
        try:
            nv, h = self._handle()
            self.max_mhz = nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM)
        except Exception as e:  # no NVML
            self.error = f"nvml unavailable: {type(e).__name__}"
            return
        reasons_fn = (nv.nvmlDeviceGetCurrentClocksEventReasons
                      if hasattr(nv, "nvmlDeviceGetCurrentClocksEventReasons")
                      else nv.nvmlDeviceGetCurrentClocksThrottleReasons)

        def loop():
            while not self._stop:
                try:
                    mhz = nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
                    self.samples.append((time.perf_counter(), mhz, int(reasons_fn(h))))
                except Exception:
                    pass
                time.sleep(0.0002)

        self._thread = threading.Thread(target=loop, daemon=True)
        self._thread.start()
        t0 = time.time()
        while not self.samples and time.time() - t0 < 2.0:
            time.sleep(0.001)

    def stop(self):
        self._stop = True
        if self._thread is not None:
            self._thread.join()

    def window(self, t0: float, t1: float) -> dict:
        s = [x for x in self.samples if t0 <= x[0] <= t1]
        reasons = sorted({name for _, _, r in s for name, bit in self.REASONS.items() if r & bit})
        out = {"sm_mhz": statistics.median([m for _, m, _ in s]) if s else None,
               "sm_max_mhz": self.max_mhz, "reasons": reasons, "samples": len(s)}
        if self.error:
            out["error"] = self.error
        return out


CLOCKS = Clocks()


class Region:
    """Host timestamps around a timed region (for the clock record)."""

    def __enter__(self):
        self.t0 = time.perf_counter()
        return self

    def __exit__(self, *a):
        self.t1 = time.perf_counter()

    def clocks(self) -> dict:
        return CLOCKS.window(self.t0, self.t1)


# ----------------------------------------------------------------------------- Fathom decode step

def setup_fathom(cfg: dict, device, seed: int = 1, host_index: bool = False):
    """Synthetic caches, queries and the index resident on the device."""
    import kv_index_scan_b200 as kvs
    R, G, H, n = (cfg[x] for x in ("R", "G", "H", "n"))
    K, V, nl = synth.fathom_kv(R, G, 128, n, seed=seed, device=device)
    q = synth.queries(R, G, H, 128, seed=seed, device=device)
    index = kvs.build_fathom_index(K, nl)
    return dict(K=K, V=V, q=q, index=index, nl=nl, seed=seed)


def decode_step_for(cfg: dict, data: dict, B: int, index=None):
    """A DecodeStep at budget B with hot buffers built around a warm-up
    selection of that budget (cfg['miss'] of each selection missing)."""
    import kv_index_scan_b200 as kvs
    R, G, H, n, k, S = (cfg[x] for x in ("R", "G", "H", "n", "k", "S"))
    index = index or data["index"]
    warm = kvs.DecodeStep(index, data["nl"], n, H, B, k, data["K"], data["V"])
    warm(data["q"])
    torch.cuda.synchronize()
    sel = warm.idx.cpu().numpy()
    del warm
    slot_map, hot_tok = synth.slot_map_from_selection(sel, data["nl"], n, S, cfg["miss"],
                                                      seed=data["seed"])
    hotK, hotV = synth.hot_rows(data["K"], hot_tok), synth.hot_rows(data["V"], hot_tok)
    slot_map_t = torch.from_numpy(slot_map).to(data["K"].device)
    step = kvs.DecodeStep(index, data["nl"], n, H, B, k, data["K"], data["V"], slot_map_t, hotK,
                          hotV)
    return step, dict(slot_map=slot_map_t, hotK=hotK, hotV=hotV)


def algorithmic_bytes(cfg: dict, B: int) -> dict:
    R, G, n, k = (cfg[x] for x in ("R", "G", "n", "k"))
    keys = R * G * n
    scan = keys * B / 8
    rows = R * G * k * (2 * 128 * 2 + 32)  # K + V rows and one 32-byte slot-map sector
    return dict(keys=keys, scan=scan, rows=rows, total=scan + rows)


def scan_kernel_name(B: int, host: bool) -> str:
    if host:
        return "fathom_scan_simple"
    return "fathom_scan_prmt" if B <= 144 else "fathom_scan_topk"


def time_decode_steps(step, q, steps: int, warmup: int, dist=None):
    """Warm-up, then exactly `steps` decode steps between CUDA events on the
    launching stream. Every 8th timed step runs decode_step_timed, whose events
    bracket each stage on the same stream, so the dominant kernel's duration is
    measured inside the timed region. Returns (ms per step, stage ms, region)."""
    stream = torch.cuda.current_stream()
    for _ in range(warmup):
        step(q)
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    nst = len(step.DECODE_STAGES)
    timed_steps = list(range(0, steps, 8))
    ev = {i: [torch.cuda.Event(enable_timing=True) for _ in range(nst + 1)] for i in timed_steps}
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with Region() as reg:
        e0.record(stream)
        for i in range(steps):
            if i in ev:
                step.timed(q, ev[i])
            else:
                step(q)
        e1.record(stream)
        torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / steps
    stages = {name: sum(ev[i][j].elapsed_time(ev[i][j + 1]) for i in timed_steps) / len(timed_steps)
              for j, name in enumerate(step.DECODE_STAGES)}
    return ms, stages, reg


def oracle_sample(cfg, data, B, hot, rows: int, min_seconds: float) -> dict:
    """The CPU oracle, as it stands, on a bounded sample of the workload:
    `rows` (request, KV head) rows of one decode step, all host cores."""
    import oracle
    R, G, n, k = (cfg[x] for x in ("R", "G", "n", "k"))
    rows = min(rows, R * G)
    us = list(range(rows))
    rr = [u // G for u in us]
    gg = [u % G for u in us]
    K = data["K"][rr, gg].unsqueeze(0).cpu()
    V = data["V"][rr, gg].unsqueeze(0).cpu()
    q = data["q"][rr, gg].unsqueeze(0).cpu()
    nl = [data["nl"][0]]
    sm = hot["slot_map"][rr, gg].unsqueeze(0).cpu()
    hK = hot["hotK"][rr, gg].unsqueeze(0).cpu()
    hV = hot["hotV"][rr, gg].unsqueeze(0).cpu()
    W = synth.plane_words(n)
    planes, kmin, kstep, kvar = oracle.build_index_batch(K, nl, W)  # data prep, not timed
    cores = os.cpu_count() or 1
    reps, t0 = 0, time.perf_counter()
    while True:  # repeat the bounded sample for about min_seconds of CPU work
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


def decode_entry(name, cfg, data, B, args, dist, ws, peak, peak_kind, cpu_rows, cpu_seconds,
                 host_index=None, link_peak=None):
    """One decode-step measurement at budget B: throughput, stage times, the
    scan's roofline, and a CPU-oracle sample (rank 0)."""
    step, hot = decode_step_for(cfg, data, B, index=host_index)
    ms, stages, reg = time_decode_steps(step, data["q"], args.steps, args.warmup, dist)
    ms = _max_over_ranks(dist, ms)
    algo = algorithmic_bytes(cfg, B)
    kern = scan_kernel_name(B, host_index is not None)
    scan_gbs = algo["scan"] / (stages["scan"] / 1e3) / 1e9
    if host_index is not None:
        roof = {"bound": "host-link", "kernel": kern + " (scan stage of the step, planes over the host link)",
                "achieved": scan_gbs, "peak": link_peak, "peak_kind": "pinned host-to-device copy of the same bytes, measured in this run",
                "unit": "GB/s", "frac": scan_gbs / link_peak, "traffic": None,
                "algorithmic_bytes": algo["scan"], "ms": stages["scan"]}
    else:
        roof = {"bound": "hbm", "kernel": kern + " (scan stage of the step)", "achieved": scan_gbs,
                "peak": peak, "peak_kind": peak_kind, "unit": "GB/s", "frac": scan_gbs / peak,
                "traffic": TRAFFIC.get((cfg["name"], B, kern)), "algorithmic_bytes": algo["scan"],
                "ms": stages["scan"]}
        if B <= 144:  # the scan also writes every score and 16-key maximum
            roof["bytes_moved"] = algo["scan"] + algo["keys"] * (4 + 4 / 16)
    R, G = cfg["R"], cfg["G"]
    res = {"workload": cfg["name"], "bits_per_key": B, "requests": R, "kv_heads": G,
           "context": cfg["n"], "topk": cfg["k"], "hot_slots": cfg["S"], "miss_rate": cfg["miss"],
           "ms_per_step": ms, "keys_per_s": algo["keys"] * ws / (ms / 1e3),
           "layer_steps_per_s": ws * 1e3 / ms,
           "achieved_gbs": algo["total"] * ws / (ms / 1e3) / 1e9,
           "step_frac_hbm": algo["total"] / (ms / 1e3) / 1e9 / peak,
           "bytes_per_key": algo["scan"] / algo["keys"],
           "miss_rate_measured": int(step.misses.sum().item()) / (R * G * cfg["k"]),
           "stages_ms": stages, "roofline": roof, "clocks": reg.clocks(),
           "index": "mapped pinned host memory" if host_index is not None else "hbm"}
    if dist is None or dist.get_rank() == 0:
        if cpu_rows > 0:
            res["cpu_baseline"] = oracle_sample(cfg, data, B, hot, cpu_rows, cpu_seconds)
    res["_step"], res["_hot"] = step, hot
    return res


def _strip(d: dict) -> dict:
    return {k: v for k, v in d.items() if not k.startswith("_")}


def e2e_entry(cfg, data, step, hot, args, dist, B):
    """End to end through the C ABI with host buffers: every step copies its q
    from pinned host memory and its out, idx and misses back to pinned host
    memory. The copies run on two copy streams beside the compute stream: step
    i's results are read back while step i + 1 computes, into the other of two
    output sets (two DecodeSteps over the same index and caches). The timed
    region ends when the last step's results are on the host."""
    import kv_index_scan_b200 as kvs
    R, G, H, k = cfg["R"], cfg["G"], cfg["H"], cfg["k"]
    q = data["q"]
    stream = torch.cuda.current_stream()
    step_b = kvs.DecodeStep(data["index"], data["nl"], cfg["n"], H, B, k, data["K"], data["V"],
                            hot["slot_map"], hot["hotK"], hot["hotV"])
    steps2 = (step, step_b)
    q_host = q.cpu().pin_memory()
    out_host = [torch.empty(R, G, H, 128, dtype=torch.float32).pin_memory() for _ in range(2)]
    idx_host = [torch.empty(R, G, k, dtype=torch.int32).pin_memory() for _ in range(2)]
    miss_host = [torch.empty(R, G, dtype=torch.int32).pin_memory() for _ in range(2)]
    q_devs = [torch.empty_like(q) for _ in range(2)]
    h2d_stream, d2h_stream = torch.cuda.Stream(), torch.cuda.Stream()
    q_ready = [torch.cuda.Event() for _ in range(2)]
    done = [torch.cuda.Event() for _ in range(2)]
    copied = [torch.cuda.Event() for _ in range(2)]
    for b in range(2):  # every event exists before its first wait
        for e in (q_ready[b], done[b], copied[b]):
            e.record(stream)

    def once(i):
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

    for i in range(args.warmup):
        once(i)
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with Region() as reg:
        e0.record(stream)
        for i in range(args.steps):
            once(i)
        for b in range(2):
            stream.wait_event(copied[b])
        e1.record(stream)
        torch.cuda.synchronize()
    ms = _max_over_ranks(dist, e0.elapsed_time(e1) / args.steps)
    last = (args.steps - 1) & 1
    assert torch.equal(idx_host[last], steps2[last].idx.cpu())
    h2d = q_host.numel() * q_host.element_size()
    d2h = sum(t[0].numel() * t[0].element_size() for t in (out_host, idx_host, miss_host))
    return ms, h2d, d2h, reg


def run_ours(args, dist, rank, ws):
    import kv_index_scan_b200 as kvs
    dev = torch.device("cuda", torch.cuda.current_device())
    peak, bf16_peak, peak_kind = _peaks()
    CLOCKS.start()
    stream = torch.cuda.current_stream()
    cfg = dict(WORKLOADS[args.workload], name=args.workload)
    if args.B is not None:
        cfg["B"] = args.B
    if args.requests is not None:
        cfg["R"] = args.requests
    B = cfg["B"]
    data = setup_fathom(cfg, dev, seed=1 + rank)

    # ---- headline: device-resident fused decode steps ----
    head = decode_entry(args.workload, cfg, data, B, args, dist, ws, peak, peak_kind,
                        0 if args.no_cpu_baseline else args.cpu_rows, 10.0)
    step, hot = head["_step"], head["_hot"]
    if args.only_step:
        if rank == 0:
            print(json.dumps({"ms_per_step": head["ms_per_step"], "stages_ms": head["stages_ms"]}),
                  flush=True)
        return None

    # ---- the bit-plane scan alone (scores to HBM, no top-k), same stream ----
    scan_scores = torch.empty(cfg["R"], cfg["G"], cfg["n"], dtype=torch.float32, device=dev)

    def scan_once():
        kvs.index_scan_fathom(data["index"], step.plan, step.n, cfg["n"], scores=scan_scores)

    for _ in range(3):
        scan_once()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    nscan = max(args.steps, 5)
    e0.record(stream)
    for _ in range(nscan):
        scan_once()
    e1.record(stream)
    torch.cuda.synchronize()
    scan_ms = e0.elapsed_time(e1) / nscan
    del scan_scores
    algo = algorithmic_bytes(cfg, B)
    scan_gbs = algo["scan"] / (scan_ms / 1e3) / 1e9

    # ---- end to end through the C ABI with host buffers ----
    e2e_ms, h2d, d2h, _ = e2e_entry(cfg, data, step, hot, args, dist, B)

    keys_total = algo["keys"] * ws
    ms_max = head["ms_per_step"]
    launches_per_step = 4 + (1 if step_needs_combine(cfg) else 0)  # plan, scan, top-k, attention (+ split merge)
    res = {
        "metric": METRIC, "value": keys_total / (ms_max / 1e3), "unit": "keys/s", "n_gpus": ws,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_max,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic",
        "config": {"workload": args.workload, "requests": cfg["R"], "kv_heads": cfg["G"],
                   "q_heads_per_kv": cfg["H"], "head_dim": 128, "context": cfg["n"],
                   "bits_per_key": B, "topk": cfg["k"], "hot_slots": cfg["S"],
                   "miss_rate": cfg["miss"],
                   "parallelism": f"replicas{ws}" if ws > 1 else "single",
                   "l2": "inputs larger than L2 (>=350 MB read per step)"},
        "layer_steps_per_s": head["layer_steps_per_s"],
        "achieved_gbs": head["achieved_gbs"],
        "step_frac_hbm": head["step_frac_hbm"],
        "miss_rate_measured": head["miss_rate_measured"],
        "roofline": head["roofline"],
        "stages_ms": head["stages_ms"],
        "scan_only": {"kernel": scan_kernel_name(B, False) + " (scores written to HBM)", "ms": scan_ms,
                      "achieved_gbs": scan_gbs, "frac": scan_gbs / peak},
        "e2e": {"value": keys_total / (e2e_ms / 1e3), "unit": "keys/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms},
        "gpu_launches": launches_per_step * args.steps,
        "clocks": head["clocks"],
    }
    if "cpu_baseline" in head:
        res["cpu_baseline"] = head["cpu_baseline"]
    del step, hot, head
    torch.cuda.empty_cache()

    if not args.only_headline:
        res["configs"] = other_configs(args, cfg, data, dist, ws, peak, bf16_peak, peak_kind)
    del data
    CLOCKS.stop()
    res["clocks_all_legs"] = CLOCKS.window(-math.inf, math.inf)
    return res


def other_configs(args, cfg128, data128, dist, ws, peak, bf16_peak, peak_kind) -> dict:
    """Every other workload of the scope, each timed like the headline."""
    import kv_index_scan_b200 as kvs
    dev = data128["K"].device
    cpu_rows = 0 if args.no_cpu_baseline else 2
    out = {}
    for B in (68, 136, 512):
        e = decode_entry("128k", cfg128, data128, B, args, dist, ws, peak, peak_kind, cpu_rows, 2.0)
        out[f"128k-B{B}"] = _strip(e)
        del e
    hostK, hostV = kvs.MappedHostStore(data128["K"]), kvs.MappedHostStore(data128["V"])
    for miss in (0.2, 0.4):
        out[f"128k-hosttier-miss{round(100 * miss)}"] = hosttier_entry(cfg128, data128, miss, hostK, hostV,
                                                                       args, dist)
    del hostK, hostV
    data128.clear()
    torch.cuda.empty_cache()

    cfg1m = dict(WORKLOADS["qwen3-8b-1m"], name="qwen3-8b-1m")
    d1 = setup_fathom(cfg1m, dev, seed=2 + (dist.get_rank() if dist else 0))
    for B in (92, 136):
        e = decode_entry("1m", cfg1m, d1, B, args, dist, ws, peak, peak_kind, cpu_rows, 2.0)
        out[f"1m-B{B}"] = _strip(e)
        del e
    # the same layer with the index planes in mapped pinned host memory
    hix = kvs.MappedHostIndex(d1["index"])
    plane_bytes = int(algorithmic_bytes(cfg1m, 92)["scan"])
    host_buf = torch.empty(plane_bytes, dtype=torch.uint8).pin_memory()
    dev_buf = torch.empty(plane_bytes, dtype=torch.uint8, device=dev)
    for _ in range(2):
        dev_buf.copy_(host_buf, non_blocking=True)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(5):
        dev_buf.copy_(host_buf, non_blocking=True)
    e1.record()
    torch.cuda.synchronize()
    link_gbs = 5 * plane_bytes / (e0.elapsed_time(e1) / 1e3) / 1e9
    del host_buf, dev_buf
    e = decode_entry("1m-host", cfg1m, d1, 92, args, dist, ws, peak, peak_kind, 0, 0.0,
                     host_index=hix, link_peak=link_gbs)
    e["pinned_copy_gbs"] = link_gbs
    e["host_link_gbs"] = e["roofline"]["achieved"]
    out["1m-host-B92"] = _strip(e)
    del e, hix
    d1.clear()
    torch.cuda.empty_cache()

    out["lightning-pair"] = lightning_entry(args, dist, peak, bf16_peak, peak_kind, cpu_rows > 0)
    torch.cuda.empty_cache()
    out["sweep-36-layers"] = sweep_entry(args, dist, ws, peak, peak_kind, cpu_rows > 0)
    torch.cuda.empty_cache()
    out["selection-quality"] = quality_entry()
    torch.cuda.empty_cache()
    out["throughput-model"] = model_entry(out["sweep-36-layers"])
    return out


def model_entry(sweep: dict, hbm_budget: float = 150e9, miss: float = 0.2) -> dict:
    """The offloaded system's throughput and capacity model
    (kv_index_scan_b200.capacity) fed with the sweep's measured decode-step
    times: compute = 36 x the measured layer step of each batch (misses read
    from HBM, so no link time in it), plus the fetch of the missing selected
    entries over each link the page models; batches above a configuration's
    capacity (hot buffers + K-index in hbm_budget of HBM, the full KV in the
    link's external memory) get no figure."""
    from kv_index_scan_b200 import capacity as cm
    fp = cm.qwen3_8b_like(layers=SWEEP["layers"])
    rows = []
    for e in sweep["batches"]:
        if e.get("ms_per_layer_step") is None:
            continue
        b, n = e["batch"], int(e["mean_length"])
        tc = SWEEP["layers"] * e["ms_per_layer_step"] / 1e3
        links = {}
        for name, link in cm.LINKS.items():
            bmax = cm.batch_max(fp, n, hbm_budget, link["capacity"])
            links[name] = {"batch_max": bmax,
                           "tokens_per_s": cm.tokens_per_s(tc, fp, b, SWEEP["k"], miss, link["bandwidth"])
                           if b <= bmax else None}
        rows.append({"batch": b, "mean_length": n, "t_compute_ms": tc * 1e3, "ideal_tokens_per_s": b / tc,
                     "links": links})
    return {"model": "T_step = T_compute + batch * layers * k * miss * entry bytes / link bandwidth; "
                     "batch <= min(HBM budget / (hot + index), external capacity / full KV)",
            "layers": SWEEP["layers"], "hbm_budget_gb": hbm_budget / 1e9, "miss_rate": miss,
            "links": {k: {"gbs": v["bandwidth"] / 1e9, "capacity_tb": v["capacity"] / 1e12}
                      for k, v in cm.LINKS.items()},
            "rows": rows}


def sparq_channels(qbar: torch.Tensor, r: int) -> torch.Tensor:
    """The r channels with the largest |qbar_c| per row, ties to the lower
    channel: [..., D] -> [..., r] (ascending)."""
    order = torch.sort(qbar.abs(), dim=-1, descending=True, stable=True).indices
    return torch.sort(order[..., :r], dim=-1).values


def quality_entry(R: int = 4, G: int = 8, H: int = 4, n: int = 131072, k: int = 2048,
                  budgets=(68, 92, 136), seed: int = 5) -> dict:
    """The selection-quality diagnostic of the Fathom abstract's comparison
    (bytes read against attention error and agreement with the exact top-k),
    on synthetic data: for each budget B, the Fathom allocation (decode_step)
    and a SparQ-like scan at the same B bits per key -- all 4 planes of the
    B/4 channels of largest |qbar_c| -- through the same scan and top-k
    kernels. Recall = |selection & exact top-k| / k, where the exact top-k is
    that of qbar . K over the bf16 keys; attention error = relative L2 error
    of the attention output against the output over the exact top-k (the
    target a selection approximates). Against dense attention over all n keys
    every selection's error is large on these synthetic keys (the attention
    mass is spread over all of them), so that figure is reported beside it."""
    import kv_index_scan_b200 as kvs
    dev = torch.device("cuda", torch.cuda.current_device())
    K, V, nl = synth.fathom_kv(R, G, 128, n, seed=seed, device=dev)
    q = synth.queries(R, G, H, 128, seed=seed, device=dev)
    ix = kvs.build_fathom_index(K, nl)
    qbar = ((q[:, :, 0] + q[:, :, 1]) + q[:, :, 2]) + q[:, :, 3]  # [R][G][D]
    exact = torch.einsum("rgd,rgnd->rgn", qbar, K.float())
    o_star = torch.topk(exact, k, dim=2).indices
    scale = 1 / math.sqrt(128)
    logits = torch.einsum("rghd,rgnd->rghn", q, K.float()) * scale
    dense = torch.einsum("rghn,rgnd->rghd", torch.softmax(logits, dim=-1), V.float())
    attn = kvs.DecodeStep(ix, nl, n, H, 92, k, K, V)  # attention over a given selection

    def recall(sel):
        hits = torch.zeros(R, G, device=dev)
        for r in range(R):
            for g in range(G):
                hits[r, g] = torch.isin(sel[r, g], o_star[r, g]).sum()
        return float(hits.mean() / k)

    def attn_out(sel):
        return attn(q, idx_in=sel.to(torch.int32).contiguous()).clone()

    def rel(out, ref):
        return float(((out - ref).norm(dim=-1) / ref.norm(dim=-1)).mean())

    exact_out = attn_out(torch.sort(o_star, dim=2).values)
    res = {"requests": R, "kv_heads": G, "context": n, "topk": k,
           "exact_topk_error_vs_dense": rel(exact_out, dense), "budgets": []}
    for B in budgets:
        step = kvs.DecodeStep(ix, nl, n, H, B, k, K, V)
        step(q)
        fathom_sel = step.idx.clone()
        # the SparQ-like plan: all 4 planes of the B/4 largest-|qbar| channels
        r = B // 4
        ch = sparq_channels(qbar, r)  # [R][G][r]
        pidx = (4 * ch.unsqueeze(-1) + torch.arange(4, device=dev)).reshape(R, G, 4 * r)
        kst = torch.gather(ix.kstep, 2, ch)
        kmn = torch.gather(ix.kmin, 2, ch)
        qc = torch.gather(qbar, 2, ch)
        pw = (qc * kst).unsqueeze(-1) * torch.tensor([8.0, 4.0, 2.0, 1.0], device=dev)
        plan = kvs.Plan(R, G, 128, 4 * r, dev)
        plan.plane_idx.copy_(pidx.to(torch.int16))
        plan.plane_w.copy_(pw.reshape(R, G, 4 * r))
        plan.C.copy_((qc * kmn).sum(-1))
        sc = kvs.index_scan_fathom(ix, plan, nl, n)
        sparq_sel = kvs.topk_select(sc, nl, k)
        fo, so = attn_out(fathom_sel), attn_out(sparq_sel)
        res["budgets"].append({"bits_per_key": B, "bytes_per_key": B / 8,
                               "fathom_recall": recall(fathom_sel), "sparq_like_recall": recall(sparq_sel),
                               "fathom_attention_error": rel(fo, exact_out),
                               "sparq_like_attention_error": rel(so, exact_out),
                               "fathom_error_vs_dense": rel(fo, dense),
                               "sparq_like_error_vs_dense": rel(so, dense),
                               "sparq_like_channels": r})
    torch.cuda.synchronize()
    return res


def hosttier_entry(cfg, data, miss, hostK, hostV, args, dist) -> dict:
    """The decode step with its full K/V store in the host tier (mapped
    pinned host memory): each step fetches the missing selected rows over the
    host link into HBM, then attends. Timed beside the same step with the
    store in HBM; the fetch rate is the miss bytes over the extra time."""
    import kv_index_scan_b200 as kvs
    c = dict(cfg, miss=miss)
    step_hbm, hot = decode_step_for(c, data, cfg["B"])
    ms_hbm, _, _ = time_decode_steps(step_hbm, data["q"], args.steps, args.warmup, dist)
    step = kvs.DecodeStep(data["index"], data["nl"], cfg["n"], cfg["H"], cfg["B"], cfg["k"], hostK, hostV,
                          hot["slot_map"], hot["hotK"], hot["hotV"])
    ms, stages, reg = time_decode_steps(step, data["q"], args.steps, args.warmup, dist)
    ms_hbm, ms = _max_over_ranks(dist, ms_hbm), _max_over_ranks(dist, ms)
    torch.cuda.synchronize()
    same = bool(torch.equal(step.out, step_hbm.out) and torch.equal(step.idx, step_hbm.idx))
    misses = int(step.misses.sum().item())
    miss_bytes = misses * 2 * 128 * 2
    extra = max(ms - ms_hbm, 1e-6)
    return {"workload": cfg["name"], "full_store": "mapped pinned host memory", "miss_rate": miss,
            "miss_rate_measured": misses / (cfg["R"] * cfg["G"] * cfg["k"]),
            "ms_per_step": ms, "ms_per_step_all_in_hbm": ms_hbm, "layer_steps_per_s": 1e3 / ms,
            "miss_bytes_per_step": miss_bytes, "fetch_gbs": miss_bytes / (extra / 1e3) / 1e9,
            "stages_ms": stages, "outputs_equal_hbm_step": same, "clocks": reg.clocks()}


def sweep_footprint(nl, c=SWEEP) -> dict:
    """HBM bytes of a batch with lengths nl over c['layers'] layers: per
    request and layer the index planes (4 planes of D channels, W words each),
    the slot map and the hot K/V buffers; per request one full K/V store that
    the layers share (it only serves the misses: a synthetic shortcut)."""
    G, S = c["G"], c["S"]
    per_layer = sum(G * 128 * 4 * synth.plane_words(n) * 4 + G * n * 4 + 2 * G * S * 128 * 2 for n in nl)
    full = sum(2 * G * n * 128 * 2 for n in nl)
    total = c["layers"] * per_layer + full
    return {"bytes": total, "gb": total / 1e9, "over_capacity": total / 1e9 > c["cap_gb"]}


def sweep_entry(args, dist, ws, peak, peak_kind, with_cpu: bool) -> dict:
    """The concurrency sweep of the fused decode step (a6) over ragged
    batches: layer-steps/s, 36-layer token steps/s and GB/s per batch size."""
    import kv_index_scan_b200 as kvs
    c = SWEEP
    dev = torch.device("cuda", torch.cuda.current_device())
    rank = dist.get_rank() if dist else 0
    out = {"layers": c["layers"], "cap_gb": c["cap_gb"], "bits_per_key": c["B"], "topk": c["k"],
           "hot_slots": c["S"], "miss_rate": c["miss"], "lengths": "floor(exp(U(ln 16384, ln 131072)))",
           "timed": "one layer's fused decode step over the whole batch; the 36 layers have the same shape",
           "batches": []}
    for b in c["batches"]:
        nl = synth.ragged_lengths(b, seed=c["seed"] * 1000 + b + 7919 * rank)
        fp = sweep_footprint(nl)
        e = {"batch": b, "mean_length": sum(nl) / b, "footprint_gb": fp["gb"],
             "over_capacity": fp["over_capacity"]}
        # every rank takes the same collective steps, fit or not
        if fp["over_capacity"]:
            out["batches"].append(e)
            continue
        n_max = max(nl)
        K, V, _ = synth.fathom_kv(b, c["G"], 128, nl, n_max=n_max, seed=c["seed"] + 10 * rank, device=dev)
        q = synth.queries(b, c["G"], c["H"], 128, seed=c["seed"] + 10 * rank, device=dev)
        index = kvs.build_fathom_index(K, nl)
        cfg = dict(R=b, G=c["G"], H=c["H"], n=n_max, B=c["B"], k=c["k"], S=c["S"], miss=c["miss"])
        step, _ = decode_step_for(cfg, dict(K=K, V=V, q=q, index=index, nl=nl, seed=c["seed"]), c["B"])
        ms, stages, reg = time_decode_steps(step, q, args.steps, args.warmup, dist)
        ms = _max_over_ranks(dist, ms)
        keys = c["G"] * sum(nl)
        scan_bytes = keys * c["B"] / 8
        rows = b * c["G"] * c["k"] * (2 * 128 * 2 + 32)
        e.update({"ms_per_layer_step": ms, "layer_steps_per_s": 1e3 / ms,
                  "token_steps_per_s": 1e3 / (ms * c["layers"]),
                  "keys_per_s": keys * ws / (ms / 1e3),
                  "achieved_gbs": (scan_bytes + rows) * ws / (ms / 1e3) / 1e9,
                  "frac_hbm": (scan_bytes + rows) / (ms / 1e3) / 1e9 / peak,
                  "stages_ms": stages, "clocks": reg.clocks()})
        out["batches"].append(e)
        if with_cpu and rank == 0 and b == 1:
            data = dict(K=K, V=V, q=q, nl=nl, seed=c["seed"])
            hot = {"slot_map": step.slot_map, "hotK": step.hotK, "hotV": step.hotV}
            cb = oracle_sample(cfg, data, c["B"], hot, rows=2, min_seconds=2.0)
            cb["sample"] += " (batch 1, one layer)"
            out["cpu_baseline"] = cb
        del K, V, q, index, step
        torch.cuda.empty_cache()
    fits = [e["batch"] for e in out["batches"] if not e["over_capacity"]]
    out["largest_batch_that_fits"] = max(fits) if fits else 0
    out["peak_kind"] = peak_kind
    return out


def lightning_entry(args, dist, peak, bf16_peak, peak_kind, with_cpu: bool) -> dict:
    """The lightning layer pair: indexer (a2-L) + block top-k (a3) on layer 2j,
    and the sparse attention of both layers of the group over that one
    selection (a7), all KV heads of a request sharing it."""
    import kv_index_scan_b200 as kvs
    c = LIGHTNING
    dev = torch.device("cuda", torch.cuda.current_device())
    R, n, Hi, Dl, block, k, G, H = (c[x] for x in ("R", "n", "Hi", "Dl", "block", "k", "G", "H"))
    kidx, qidx, w, nl = synth.lightning_inputs(R, n, Hi=Hi, Dl=Dl, seed=3, device=dev)
    nl_dev = torch.tensor(nl, dtype=torch.int32, device=dev)  # resident: no copy inside the step
    layers = []
    for layer in range(2):
        K, V, _ = synth.fathom_kv(R, G, 128, n, seed=40, layer=layer, device=dev)
        q = synth.queries(R, G, H, 128, seed=40, layer=layer, device=dev, dtype=torch.bfloat16)
        # the step takes its R x G rows from the index (whose planes are not
        # read when the selection is given), so the index covers every row
        ix = kvs.build_fathom_index(K, nl)
        st = kvs.DecodeStep(ix, nl, n, H, 92, k, K, V, q_dtype=torch.bfloat16)
        assert (st.R, st.G) == (R, G)
        layers.append((q, st))
    nb = (n + block - 1) // block
    bs = torch.empty(R, nb, dtype=torch.float32, device=dev)
    idx = torch.empty(R, 1, k, dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream()

    def pair(ev=None):
        if ev:
            ev[0].record(stream)
        kvs.index_scan_lightning(kidx, qidx, w, nl_dev, block=block, scores=bs)
        if ev:
            ev[1].record(stream)
        kvs.topk_select(bs, nl_dev, k, block=block, idx=idx)
        if ev:
            ev[2].record(stream)
        for j, (q, st) in enumerate(layers):
            st(q, idx_in=idx, idx_shared=True)
            if ev:
                ev[3 + j].record(stream)

    for _ in range(args.warmup):
        pair()
    torch.cuda.synchronize()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(args.steps)]
    with Region() as reg:
        for i in range(args.steps):
            pair(evs[i])
        torch.cuda.synchronize()
    t = lambda a, b: statistics.mean(e[a].elapsed_time(e[b]) for e in evs)
    scan_ms, topk_ms, a1_ms, a2_ms, eager_ms = t(0, 1), t(1, 2), t(2, 3), t(3, 4), t(0, 4)
    # host time to enqueue one pair (four library calls), no synchronisation
    torch.cuda.synchronize()
    h0 = time.perf_counter()
    for _ in range(args.steps):
        pair()
    host_us = (time.perf_counter() - h0) / args.steps * 1e6
    torch.cuda.synchronize()
    # the pair captured once as a CUDA graph (no allocation inside, as the
    # layer-shared top-k buffer is persistent) and replayed: device time
    # without the host's launch cost between the four calls
    graph_ms = None
    try:
        side = torch.cuda.Stream()
        side.wait_stream(stream)
        with torch.cuda.stream(side):
            pair()  # warm the side stream (function attributes, tensor maps)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            pair()
        for _ in range(args.warmup):
            g.replay()
        torch.cuda.synchronize()
        ge = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(args.steps)]
        with Region() as greg:
            for a, b in ge:
                a.record(stream)
                g.replay()
                b.record(stream)
            torch.cuda.synchronize()
        graph_ms = statistics.mean(a.elapsed_time(b) for a, b in ge)
        del g
    except RuntimeError as e:  # capture refused: keep the eager number
        print(f"lightning pair: graph capture failed ({e}); eager timing only", file=sys.stderr)
    pair_ms = graph_ms if graph_ms is not None else eager_ms
    kbytes = R * n * Dl
    flops = 2.0 * R * n * Hi * Dl
    rows = R * G * k * 2 * 128 * 2  # K and V rows of one layer
    pair_bytes = kbytes + 2 * rows
    scan_gbs = kbytes / (scan_ms / 1e3) / 1e9
    res = {"workload": "minimax-lightning-32x80000", "requests": R, "tokens": n,
           "index_heads": Hi, "block": block, "topk": k, "kv_heads": G, "q_heads_per_kv": H,
           "ms_per_layer_pair": pair_ms, "layer_pairs_per_s": 1e3 / pair_ms,
           "timing": ("one CUDA graph of the pair, replayed" if graph_ms is not None
                      else "the four calls issued one by one"),
           "ms_per_layer_pair_eager": eager_ms, "host_us_per_pair": host_us,
           "index_keys_per_s": R * n / (scan_ms / 1e3),
           "stages_ms": {"indexer": scan_ms, "block_topk": topk_ms, "attention_layer0": a1_ms,
                         "attention_layer1": a2_ms},
           "pair_achieved_gbs": pair_bytes / (pair_ms / 1e3) / 1e9,
           "pair_frac_hbm": pair_bytes / (pair_ms / 1e3) / 1e9 / peak,
           "indexer_tflops": flops / (scan_ms / 1e3) / 1e12,
           # the e4m3 contraction against the measured bf16 peak x 2 (the nominal
           # fp8 : bf16 ratio); hi and lo query parts make two passes
           "indexer_frac_tensor": 2 * flops / (scan_ms / 1e3) / 1e12 / (2 * bf16_peak),
           "roofline": {"bound": "hbm", "kernel": "lightning_scan (tcgen05 kind::f8f6f4)",
                        "achieved": scan_gbs, "peak": peak, "peak_kind": peak_kind, "unit": "GB/s",
                        "frac": scan_gbs / peak,
                        "traffic": TRAFFIC.get(("minimax-lightning-32x80000", Hi, "lightning_scan")),
                        "algorithmic_bytes": kbytes,
                        "ms": scan_ms},
           "clocks": reg.clocks()}
    if with_cpu and (dist is None or dist.get_rank() == 0):
        import oracle
        cores = os.cpu_count() or 1
        reps, t0 = 0, time.perf_counter()
        sub_k = kidx[:1].cpu()
        sub_q, sub_w = qidx[:1].cpu(), w[:1].cpu()
        while True:
            oracle.lightning_batch(sub_k, sub_q, sub_w, [n], block, k, nthreads=cores)
            reps += 1
            dt = time.perf_counter() - t0
            if dt >= 2.0:
                break
        res["cpu_baseline"] = {"value": reps * n / dt, "unit": "index keys/s", "cores": cores,
                               "kind": "oracle",
                               "sample": f"the indexer and block top-k of 1 of {R} requests "
                                         f"({n} tokens x {Hi} heads) x {reps} repetitions, fp64 "
                                         f"C++ oracle, {dt:.1f} s"}
    del layers
    return res


def step_needs_combine(cfg) -> bool:
    import kv_index_scan_b200 as kvs
    return kvs._lib.kvs_attn_workspace_size(cfg["R"], cfg["G"], cfg["H"], cfg["k"]) > 0


def run_reference(args, cfg, dist, rank, ws):
    """The CPU oracle timed as the reference arm, on the same workload's shape."""
    import oracle
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
    if args.row == "quality":
        return quality_entry()
    return _run_row(args)


def _run_row(args) -> dict:
    """Measurements of single rows of the path outside the decode step (one
    JSON line each; not the benchmark's headline line):
      lightning -- the lightning indexer (a2-L) alone and its block top-k (a3,
                   block 64) at 32 requests x 80000 tokens x 64 index heads,
                   two input sets in turn;
      host-scan -- the Fathom scan reading its planes from mapped pinned host
                   memory (a2-host) at the 1M layer (4 x 8 x 1048576, B = 92),
                   beside the same scan from HBM and a pinned host-to-device
                   copy of the same size (the link's copy rate)."""
    import kv_index_scan_b200 as kvs
    dev = torch.device("cuda")
    peak, bf16_peak, peak_kind = _peaks()
    steps, warmup = max(args.steps, 5), max(args.warmup, 3)
    if args.row == "lightning":
        c = LIGHTNING
        R, n, Hi, Dl, block, k = (c[x] for x in ("R", "n", "Hi", "Dl", "block", "k"))
        sets = [synth.lightning_inputs(R, n, Hi, Dl, seed=3 + j, device=dev) for j in range(2)]
        # request lengths resident on the device, so that no copy falls inside the timing
        sets = [(kk, qq, ww, torch.tensor(nn, dtype=torch.int32, device=dev)) for kk, qq, ww, nn in sets]
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
        nl = torch.tensor(nl, dtype=torch.int32, device=dev)  # resident: no copy inside the timing
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
                    help="time the decode steps only (no scan-alone, end-to-end, CPU or other "
                         "workloads); prints the step and stage times, for profiling runs")
    ap.add_argument("--only-headline", action="store_true",
                    help="measure the headline workload only (no other workloads)")
    ap.add_argument("--row", default=None, choices=["lightning", "host-scan", "quality"],
                    help="measure one row of the path outside the decode step (one JSON line)")
    args = ap.parse_args()
    if args.row is not None:
        print(json.dumps(run_row(args)), flush=True)
        return
    if args.impl == "reference":
        cfg = dict(WORKLOADS[args.workload])
        if args.B is not None:
            cfg["B"] = args.B
        if args.requests is not None:
            cfg["R"] = args.requests
        # the CPU oracle: rank 0 alone runs it; other ranks exit without work
        if int(os.environ.get("RANK", "0")) == 0:
            ws = int(os.environ.get("WORLD_SIZE", "1"))
            print(json.dumps(run_reference(args, cfg, None, 0, ws)), flush=True)
        return
    dist, rank, ws = _dist()
    res = run_ours(args, dist, rank, ws)
    if rank == 0 and res is not None:
        print(json.dumps(res), flush=True)
    if dist:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
