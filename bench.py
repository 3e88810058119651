"""Benchmark of the trie-constrained wide beam-search decode on B200.

One benchmark step = one full decode of one batch of requests (depth beam
steps + finalize) over a resident catalog trie, with every step's logits
already in HBM when the timed region starts (they are produced beforehand by
an untimed decode; each step has its own 1.9-5 GB buffer, far larger than the
126 MB L2, so no step re-reads cached logits).

Metric: constrained beam candidates per second, B*K*depth per decode, summed
over ranks (requests shard across GPUs with no collective: weak scaling).
The timed decodes replay one decode captured in a CUDA graph from the library
calls (`--eager` times the calls issued from Python instead); the per-kernel
breakdown and the end-to-end leg use the calls themselves.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config serving]
    python bench.py --impl reference     # the CPU oracle on a bounded sample
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

from trie_constrained_beam_fr_b200 import synth  # noqa: E402

METRIC = "constrained beam candidates/sec (B·K·steps/s) and logits HBM GB/s vs 8 TB/s"
UNIT = "candidates/s"
# the streaming kernel's translation unit: its source and the headers it includes
STREAM_KERNEL_SRC = [os.path.join(ROOT, "trie_constrained_beam_fr_b200", "csrc", f)
                     for f in ("fr_step.cu", "fr_step.cuh", "fr_internal.cuh", "fr_topk.cuh")]
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "traffic.json")


def parse_args():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=10)
    p.add_argument("--warmup", type=int, default=3)
    p.add_argument("--impl", default="fr", choices=["fr", "reference"])
    p.add_argument("--config", default="serving", choices=[k for k in synth.WORKLOADS if k != "tiny"])
    p.add_argument("--e2e-steps", type=int, default=2)
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--eager", action="store_true",
                   help="time the library calls issued from Python instead of replays of one decode captured "
                        "in a CUDA graph (the default; graph replay keeps host launch overhead out of small "
                        "decodes, as a serving engine's captured decode does)")
    p.add_argument("--no-workloads", action="store_true",
                   help="with --config serving: skip the records of the other catalog-scale workloads")
    p.add_argument("--ref-requests", type=int, default=1, help="requests per reference-arm sample")
    p.add_argument("--batch", type=int, default=0, help="override B (requests per GPU), e.g. for profiling")
    p.add_argument("--norm", default="full", choices=["full", "sid_range", "candidates"],
                   help="log-softmax normalisation set (full vocabulary by default)")
    p.add_argument("--temperature", type=float, default=0.0,
                   help="0: deterministic top-K; > 0: Gumbel top-K sampling at this temperature")
    p.add_argument("--lmhead", type=int, default=0, metavar="D",
                   help="the lm_head path: hidden states of size D instead of logits (fused tensor-core "
                        "lm_head + log-sum-exp, then the step from the SID-range slice)")
    return p.parse_args()


def dist_env():
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def rank_requests(rank: int, world: int, B: int):
    """Requests are independent, so ranks shard them: rank r decodes the
    global requests r*B .. r*B+B-1 (the hash logits take the global index)."""
    if not (0 <= rank < world) or B < 1:
        raise ValueError("bad rank layout")
    return rank * B, B


def max_over_ranks(x: float, world: int, dist=None, device=None) -> float:
    """The job's time is its slowest rank's (one all-reduce, not on the data path)."""
    if world == 1:
        return float(x)
    import torch

    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(world: int, candidates_per_decode: int, decodes: int, elapsed_ms: float) -> float:
    """Whole-job candidates/s: every rank's decodes over the slowest rank's time."""
    return world * candidates_per_decode * decodes / (elapsed_ms / 1e3)


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


def kernel_source_hash() -> str:
    """Hash of the streaming kernel's sources (its file and the headers it
    includes) with comments and blank lines removed: recorded counters stay
    valid across comment-only edits and are dropped as soon as any code
    changes."""
    import re

    src = ""
    for path in STREAM_KERNEL_SRC:
        with open(path) as f:
            src += f.read() + "\n"
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    src = re.sub(r"//[^\n]*", "", src)
    code = "\n".join(line.rstrip() for line in src.splitlines() if line.strip())
    return hashlib.sha256(code.encode()).hexdigest()[:16]


def recorded_traffic(config: str, live_rows_per_launch: float):
    """Per-launch DRAM bytes (read + written) of the streaming kernel: the
    committed ncu capture's bytes per live row, times the launch's average
    live rows, if the capture was taken on the current kernel source."""
    if not os.path.exists(TRAFFIC_FILE):
        return None
    with open(TRAFFIC_FILE) as f:
        d = json.load(f)
    e = d.get(config)
    if not e or e.get("kernel_sha") != kernel_source_hash():
        return None
    return e["bytes_per_live_row"] * live_rows_per_launch


class ClockSampler:
    """SM clock and throttle-reason samples (NVML, every 5 ms, in a thread)
    during the timed region.  Reading clocks changes nothing on the GPU."""

    REASONS = {"hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
               "sw_power_cap": 0x4, "hw_power_brake_slowdown": 0x80}

    def __init__(self, device_index: int, period_s: float = 0.005):
        self.device_index = device_index
        self.period_s = period_s
        self.samples = []
        self.max_mhz = None
        self.error = None

    def _handle(self):
        import pynvml
        import torch

        pynvml.nvmlInit()
        props = torch.cuda.get_device_properties(self.device_index)
        bus = "%08X:%02X:%02X.0" % (getattr(props, "pci_domain_id", 0), props.pci_bus_id, props.pci_device_id)
        try:
            return pynvml.nvmlDeviceGetHandleByPciBusId(bus)
        except Exception:
            return pynvml.nvmlDeviceGetHandleByIndex(self.device_index)

    def _run(self):
        import pynvml

        get_reasons = getattr(pynvml, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            pynvml.nvmlDeviceGetCurrentClocksThrottleReasons
        while not self._stop.is_set():
            try:
                sm = pynvml.nvmlDeviceGetClockInfo(self.h, pynvml.NVML_CLOCK_SM)
                rs = get_reasons(self.h)
                pw = pynvml.nvmlDeviceGetPowerUsage(self.h) / 1000.0
                self.samples.append((sm, rs, pw))
            except Exception as e:  # keep the benchmark running
                self.error = str(e)
                return
            self._stop.wait(self.period_s)

    def __enter__(self):
        import threading

        try:
            import pynvml

            self.h = self._handle()
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self._stop = threading.Event()
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()
        except Exception as e:
            self.error = str(e)
            self._thread = None
        return self

    def __exit__(self, *exc):
        if self._thread is not None:
            self._stop.set()
            self._thread.join(timeout=2)

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0,
                    "error": self.error}
        reasons = sorted({n for _, rs, _ in self.samples for n, bit in self.REASONS.items() if rs & bit})
        return {"sm_mhz": statistics.median([s for s, _, _ in self.samples]), "sm_max_mhz": self.max_mhz,
                "reasons": reasons, "samples": len(self.samples),
                "power_w_max": max(p for _, _, p in self.samples), "source": "nvml, 5 ms"}


# ---------------------------------------------------------------------------
# CPU oracle timing (reference arm and cpu_baseline)


NORM_CODES = {"full": 0, "sid_range": 1, "candidates": 2}  # fr_norm values (include/fr.h)


def catalog_level_sizes(sids: np.ndarray) -> list:
    """Nodes per trie level of a catalog: the root, then the distinct SID
    prefixes of each length (the level sizes the device trie build reports)."""
    u = np.unique(sids, axis=0)
    return [1] + [int(np.unique(u[:, : l + 1], axis=0).shape[0]) for l in range(u.shape[1])]


def logits_config(w: synth.Workload, args, levels) -> dict:
    """`config` of a bench line on the logits path (both arms)."""
    return {"workload": w.name, "norm": args.norm, "temperature": args.temperature, "B_per_gpu": w.B, "K": w.K,
            "depth": w.depth, "V": w.V, "codes_per_level": w.C, "catalog": w.n_items, "logits": w.dtype,
            "trie_levels": list(levels),
            "l2": "inputs larger than L2: one distinct %.2f GB logits buffer per step, read once"
                  % (w.B * w.K * w.V * w.elt_size / 1e9),
            "step": "one full decode: depth beam steps + finalize",
            "launch": "library calls from Python, stream-ordered" if getattr(args, "eager", False) else
                      "CUDA graph replay of one decode (captured from the library calls)"}


def lmhead_config(w: synth.Workload, args) -> dict:
    """`config` of a bench line on the lm_head path (both arms)."""
    dh = args.lmhead
    return {"workload": w.name, "path": "lm_head", "hidden_size": dh, "norm": args.norm,
            "temperature": args.temperature, "B_per_gpu": w.B, "K": w.K, "depth": w.depth, "V": w.V,
            "codes_per_level": w.C, "catalog": w.n_items,
            "l2": "per step a distinct %.0f MB hidden-state buffer; the %.0f MB lm_head is re-read "
                  "every step (larger than L2)" % (w.B * w.K * dh * 2 / 1e6, w.V * dh * 2 / 1e6),
            "step": "one full decode: depth x (fused lm_head + beam step) + finalize"}


def lmhead_oracle_sample(w: synth.Workload, hidden: np.ndarray, weight: np.ndarray) -> dict:
    """The oracle's lm_head rows for the given rows of one request, timed, and
    scaled to that request's decode: 1 row at step 0, K at every later step.
    The selection's cost is negligible next to the rows."""
    import oracle

    span = sum(w.codebook_sizes)
    t0 = time.perf_counter()
    oracle.lmhead_rows(hidden, weight, w.sid_base, span)
    per_row = (time.perf_counter() - t0) / hidden.shape[0]
    rows_per_request = 1 + (w.depth - 1) * w.K
    return {"candidates": w.K * w.depth, "method_s": rows_per_request * per_row, "per_row_s": per_row,
            "rows_per_request": rows_per_request}


def oracle_sample(w: synth.Workload, n_requests: int, first_request: int = 0, sids=None, cat=None,
                  norm: str = "full", temperature: float = 0.0):
    import oracle

    if sids is None:
        sids = synth.workload_catalog(w)
    if cat is None:
        cat = oracle.Catalog(sids, w.codebook_sizes)
    cfg = oracle.Config.from_workload(w, B=n_requests, b_offset=first_request, norm=NORM_CODES[norm])
    cfg.temperature = temperature
    cfg.gseed = 0x5EED
    t0 = time.perf_counter()
    r = oracle.decode(cfg, cat)
    wall = time.perf_counter() - t0
    method = wall - r.gen_seconds
    return {"candidates": n_requests * w.K * w.depth, "method_s": method, "gen_s": r.gen_seconds, "wall_s": wall}


CPU_SAMPLE_S = 10.0  # CPU work of a cpu_baseline sample (the oracle is slow by design)


def cpu_baseline_logits(w: synth.Workload, sids: np.ndarray, norm: str, temperature: float,
                        min_s: float = CPU_SAMPLE_S) -> dict:
    """cpu_baseline on the logits path: whole decodes of requests 0, 1, ...
    by the single-threaded oracle until about min_s seconds of CPU work (at
    least one request, at most B), timing the method without the oracle's
    own logits generation."""
    import oracle

    cat = oracle.Catalog(sids, w.codebook_sizes)
    cand, method, gen, n = 0, 0.0, 0.0, 0
    t0 = time.perf_counter()
    while n < w.B and (n == 0 or time.perf_counter() - t0 < min_s):
        smp = oracle_sample(w, 1, first_request=n, sids=sids, cat=cat, norm=norm, temperature=temperature)
        cand += smp["candidates"]
        method += smp["method_s"]
        gen += smp["gen_s"]
        n += 1
    return {"value": cand / method, "unit": UNIT, "cores": 1, "kind": "oracle", "host": host_description(),
            "sample": "requests 0..%d of %s (%d of B=%d), a full decode each, single-threaded C oracle in double, "
                      "time excluding its logits generation (%.1f s method, %.1f s generation)"
                      % (n - 1, w.name, n, w.B, method, gen)}


def cpu_baseline_lmhead(w: synth.Workload, rows: np.ndarray, weight: np.ndarray,
                        min_s: float = CPU_SAMPLE_S) -> dict:
    """cpu_baseline on the lm_head path: the oracle's lm_head rows (float32
    rows [r, d] of one request) 4 at a time until about min_s seconds, the
    mean time per row scaled to one request's decode."""
    done, secs = 0, 0.0
    per_req = None
    while done < rows.shape[0] and (done == 0 or secs < min_s):
        smp = lmhead_oracle_sample(w, rows[done:done + 4], weight)
        n = min(4, rows.shape[0] - done)
        secs += smp["per_row_s"] * n
        done += n
        per_req = smp["rows_per_request"]
    per_row = secs / done
    return {"value": w.K * w.depth / (per_req * per_row), "unit": UNIT, "cores": 1, "kind": "oracle",
            "host": host_description(),
            "sample": "oracle lm_head rows (hidden . W^T over V = %d, d = %d, in double) for %d rows of "
                      "request 0, %.2f s per row, scaled to one request's decode (%d rows: 1 at step 0, "
                      "K afterwards); the selection's cost is negligible next to the rows"
                      % (w.V, weight.shape[1], done, per_row, per_req)}


def run_reference(args):
    """The oracle on host cores, on the same workload, config, metric and
    unit as the GPU arm; each step a bounded sample of that workload."""
    rank, world, _ = dist_env()
    if rank != 0:
        return
    import oracle

    w = synth.WORKLOADS[args.config]
    if args.batch:
        w = synth.scaled(w, B=args.batch)
    sids = synth.workload_catalog(w)
    if args.lmhead:
        dh = args.lmhead
        rng = np.random.default_rng(1234)
        # bf16-representable values of the GPU arm's scale; only the timing is used
        weight = (rng.integers(-128, 128, size=(w.V, dh), dtype=np.int16).astype(np.float32) / 8192.0)
        n_rows = 4
        hid = [rng.integers(-128, 128, size=(n_rows, dh), dtype=np.int16).astype(np.float32) / 64.0
               for _ in range(args.warmup + args.steps)]
        for i in range(args.warmup):
            lmhead_oracle_sample(w, hid[i], weight)
        samples = [lmhead_oracle_sample(w, hid[args.warmup + i], weight) for i in range(args.steps)]
        config = lmhead_config(w, args)
        sample = ("oracle lm_head rows (hidden . W^T over V = %d, d = %d, in double) for %d rows of one request "
                  "per step, scaled to that request's decode (%d rows)"
                  % (w.V, dh, n_rows, samples[0]["rows_per_request"]))
    else:
        cat = oracle.Catalog(sids, w.codebook_sizes)
        for i in range(args.warmup):
            oracle_sample(w, args.ref_requests, first_request=i % w.B, sids=sids, cat=cat, norm=args.norm,
                          temperature=args.temperature)
        samples = [oracle_sample(w, args.ref_requests, first_request=i % w.B, sids=sids, cat=cat, norm=args.norm,
                                 temperature=args.temperature)
                   for i in range(args.steps)]
        config = logits_config(w, args, catalog_level_sizes(sids))
        sample = ("%d request(s) of %s per step (of B=%d), full decode, oracle time excluding its logits generation"
                  % (args.ref_requests, w.name, w.B))
    cand = sum(s["candidates"] for s in samples)
    secs = sum(s["method_s"] for s in samples)
    value = cand / secs
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * secs / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config,
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": 1, "kind": "oracle", "sample": sample,
                         "host": host_description()},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------
# GPU arm


def run_lmhead(args):
    """The lm_head path: per step, the live beams' hidden states [rows, D]
    (bf16, random, resident in HBM) go through fr_lmhead_run (every row's
    log-sum-exp over V and its SID-range logits, on the tensor cores) and
    fr_beam_step_lse; one benchmark step is one full decode."""
    import torch
    import torch.distributed as dist

    from trie_constrained_beam_fr_b200 import fr

    rank, world, local_rank = dist_env()
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    if world > 1:
        import datetime

        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    def barrier():
        if world > 1:
            dist.barrier()

    w = synth.WORKLOADS[args.config]
    if args.batch:
        w = synth.scaled(w, B=args.batch)
    B, K, D, V, dh = w.B, w.K, w.depth, w.V, args.lmhead
    b_offset, _ = rank_requests(rank, world, B)
    span = sum(w.codebook_sizes)
    sids = torch.from_numpy(synth.workload_catalog(w)).to(dev)
    trie = fr.fr_trie_build(sids, w.codebook_sizes, w.sid_base)
    beam = fr.fr_beam_init(trie, B, K, V, "bf16")
    fr.fr_beam_set_normalization(beam, NORM_CODES[args.norm])
    if args.temperature > 0:
        fr.fr_beam_set_sampling(beam, args.temperature, 0x5EED, b_offset)
    g = torch.Generator(device=dev).manual_seed(1234 + rank)
    weight = (torch.randn(V, dh, device=dev, generator=g) / dh ** 0.5).to(torch.bfloat16)
    hidden = [torch.randn(B, K, dh, device=dev, generator=g).to(torch.bfloat16) for _ in range(D)]
    lm = fr.fr_lmhead_init(weight, max_rows=B * K, sid_base=w.sid_base, sid_span=span)
    lse = torch.empty(B * K, device=dev)
    sl = torch.empty(B * K, span, device=dev)
    out_sids = torch.empty((B, K, D), dtype=torch.int32, device=dev)
    out_scores = torch.empty((B, K), dtype=torch.float32, device=dev)
    out_items = torch.empty((B, K), dtype=torch.int32, device=dev)
    rows_per_step = [B] + [B * K] * (D - 1)  # step 0: slot 0 of each request is the only live beam

    def decode(hid, lm_events=None):
        fr.fr_beam_reset(beam)
        for t in range(D):
            rows = rows_per_step[t]
            h = hid[t][:, 0, :] if t == 0 else hid[t].view(B * K, dh)
            if lm_events is not None:
                lm_events[t][0].record()
            fr.fr_lmhead_run(lm, h, lse[:rows], sl[:rows])
            if lm_events is not None:
                lm_events[t][1].record()
            fr.fr_beam_step_lse(beam, lse[:rows], sl[:rows], 1 if t == 0 else K)
        fr.fr_beam_finalize(beam, out_sids, out_scores, out_items)

    for _ in range(args.warmup):
        decode(hidden)
    torch.cuda.synchronize()
    for st in (fr.fr_lmhead_status(lm), fr.fr_beam_status(beam)):
        if st != fr.FR_OK:
            raise RuntimeError("lm_head decode failed: " + fr.fr_status_string(st))
    barrier()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    lm_ms = [[] for _ in range(D)]
    with ClockSampler(torch.cuda.current_device()) as clocks:
        t0.record()
        for _ in range(args.steps):
            decode(hidden)
        t1.record()
        torch.cuda.synchronize()
        barrier()
        for _ in range(args.steps):
            ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(D)]
            decode(hidden, ev)
            torch.cuda.synchronize()
            for t in range(D):
                lm_ms[t].append(ev[t][0].elapsed_time(ev[t][1]))
    barrier()
    elapsed_ms = max_over_ranks(t0.elapsed_time(t1), world, dist, dev)
    ms_per_decode = elapsed_ms / args.steps
    value = job_throughput(world, B * K * D, args.steps, elapsed_ms)
    flops = [2.0 * r * dh * V for r in rows_per_step]
    lm_avg = [float(np.mean(x)) for x in lm_ms]
    achieved = sum(flops) / (sum(lm_avg) / 1e3) / 1e12
    # The sustained GEMM figure applies once the power cap holds the clocks
    # down during the timed region; a short run at full clock is held to the
    # burst figure.
    clk = clocks.summary()
    capped = "sw_power_cap" in (clk.get("reasons") or [])
    kind = "sustained" if capped else "burst"
    why = "power cap active during the timed region" if capped else "no power cap during the timed region"
    peak = 1400.0 if capped else 1590.0
    peak_src = "fallback, %s bf16 (cuBLAS) of this pool's B200s; %s" % (kind, why)
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            peaks = json.load(f)
        key = "bf16_tflops_sustained" if capped else "bf16_tflops"
        if key in peaks:
            peak = float(peaks[key])
            peak_src = "measured, %s bf16 (cuBLAS); %s" % (kind, why)
    roofline = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
                "traffic": None, "kernel": "k_lmhead (+ k_lmhead_combine)",
                "peak_source": peak_src,
                "flops_per_launch": sum(flops) / D, "ms_per_launch": sum(lm_avg) / D,
                "timing": "CUDA events around fr_lmhead_run, second timed pass of the same decodes"}
    per_step = [{"t": t, "rows": rows_per_step[t], "lmhead_ms": lm_avg[t],
                 "tflops": flops[t] / (lm_avg[t] / 1e3) / 1e12} for t in range(D)]

    e2e = None
    if not args.no_e2e:
        host = [h.cpu().pin_memory() for h in hidden]
        dev_h = [torch.empty_like(h) for h in hidden]
        h_sids = torch.empty((B, K, D), dtype=torch.int32, pin_memory=True)
        h_scores = torch.empty((B, K), dtype=torch.float32, pin_memory=True)

        def e2e_decode():
            for t in range(D):
                dev_h[t].copy_(host[t], non_blocking=True)
            decode(dev_h)
            h_sids.copy_(out_sids, non_blocking=True)
            h_scores.copy_(out_scores, non_blocking=True)

        e2e_decode()
        torch.cuda.synchronize()
        barrier()
        a, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        for _ in range(args.e2e_steps):
            e2e_decode()
        b_.record()
        torch.cuda.synchronize()
        barrier()
        e2e_ms = max_over_ranks(a.elapsed_time(b_), world, dist, dev) / args.e2e_steps
        e2e = {"value": world * B * K * D / (e2e_ms / 1e3), "unit": UNIT,
               "h2d_bytes_per_step": sum(h.numel() * 2 for h in hidden),
               "d2h_bytes_per_step": B * K * D * 4 + B * K * 4, "ms_per_step": e2e_ms, "steps": args.e2e_steps}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline_lmhead(w, hidden[1][0].float().cpu().numpy(), weight.float().cpu().numpy())

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_decode, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16 x bf16 -> f32", "data": "synthetic",
            "config": lmhead_config(w, args),
            "roofline": roofline, "per_step": per_step, "gpu_launches": args.steps * (4 * D + 2),
            "clocks": clk, "e2e": e2e, "cpu_baseline": cpu,
        }
        print(json.dumps(line), flush=True)
    fr.fr_lmhead_destroy(lm)
    fr.fr_beam_destroy(beam)
    fr.fr_trie_destroy(trie)
    if world > 1:
        dist.destroy_process_group()


def host_description() -> dict:
    """The host the CPU legs ran on: logical cores and CPU model."""
    model = None
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return {"nproc": os.cpu_count(), "cpu_model": model}


def measure_logits_workload(w: synth.Workload, args, dev, world: int, b_offset: int, barrier, slowest,
                            with_e2e: bool) -> dict:
    """One logits-path workload on this rank's GPU: build the trie (timed on
    its own), produce every step's logits with an untimed decode, then time
    `args.steps` whole decodes twice (the headline with nothing recorded
    between kernels, then with the library's per-kernel events for the
    roofline and the per-step breakdown), and optionally the end-to-end
    decode through host buffers.  Frees everything it allocated."""
    import torch

    from trie_constrained_beam_fr_b200 import fr

    B, K, D, V = w.B, w.K, w.depth, w.V
    tdt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    elt = w.elt_size
    sids_np = synth.workload_catalog(w)
    sids = torch.from_numpy(sids_np).to(dev)

    # catalog trie (off the per-decode path; timed on its own)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    trie = fr.fr_trie_build(sids, w.codebook_sizes, w.sid_base)  # warm (allocations, first launch)
    fr.fr_trie_destroy(trie)
    torch.cuda.synchronize()
    e0.record()
    trie = fr.fr_trie_build(sids, w.codebook_sizes, w.sid_base)
    e1.record()
    torch.cuda.synchronize()
    trie_ms = e0.elapsed_time(e1)
    del sids
    levels = fr.fr_trie_level_sizes(trie)
    beam = fr.fr_beam_init(trie, B, K, V, w.dtype)
    norm_code = {"full": fr.FR_NORM_FULL, "sid_range": fr.FR_NORM_SID_RANGE,
                 "candidates": fr.FR_NORM_CANDIDATES}[args.norm]
    fr.fr_beam_set_normalization(beam, norm_code)
    if args.temperature > 0:
        fr.fr_beam_set_sampling(beam, args.temperature, 0x5EED, b_offset)
    # columns each live row's log-sum-exp streams (none over the candidate slice)
    row_cols = {"full": V, "sid_range": sum(w.codebook_sizes), "candidates": 0}[args.norm]
    # the first step runs as one kernel (root rows + selection) under these settings
    fused0 = fr.fr_beam_fused_first_step(beam)

    # one untimed decode produces every step's logits (prefix-dependent)
    bufs = [torch.empty((B, K, V), dtype=tdt, device=dev) for _ in range(D)]
    rows = []
    fr.fr_beam_reset(beam)
    for t in range(D):
        o = fr.fr_beam_outputs(beam, B, K, D)
        rows.append(int(o["live"].sum().item()))
        fr.fr_gen_hash_logits(w.seed, b_offset, B, K, V, bufs[t], w.dtype, prefix=o["prefix"], t=t, live=o["live"])
        fr.fr_beam_step(beam, bufs[t])
    out_sids = torch.empty((B, K, D), dtype=torch.int32, device=dev)
    out_scores = torch.empty((B, K), dtype=torch.float32, device=dev)
    out_items = torch.empty((B, K), dtype=torch.int32, device=dev)
    fr.fr_beam_finalize(beam, out_sids, out_scores, out_items)
    st = fr.fr_beam_status(beam)
    if st != fr.FR_OK:
        raise RuntimeError("decode failed: " + fr.fr_status_string(st))
    bytes_per_decode = sum(r * row_cols * elt for r in rows)

    def decode():
        fr.fr_beam_reset(beam)
        for t in range(D):
            fr.fr_beam_step(beam, bufs[t])
        fr.fr_beam_finalize(beam, out_sids, out_scores, out_items)

    for _ in range(args.warmup):
        decode()
    torch.cuda.synchronize()
    graph = None
    if not args.eager:
        # one whole decode (reset, steps, finalize) as a CUDA graph: the
        # library calls allocate nothing and never synchronise
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            decode()
        for _ in range(args.warmup):
            graph.replay()
        torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(torch.cuda.current_device()) as clocks:
        # the headline: K decodes back to back, nothing recorded between the
        # kernels (an event between two kernels would stop the next one from
        # launching while the previous one drains)
        t_start.record()
        for _ in range(args.steps):
            if graph is not None:
                graph.replay()
            else:
                decode()
        t_end.record()
        torch.cuda.synchronize()
        barrier()
        # the same K decodes again with the library's per-kernel events: the
        # kernel durations of the roofline and the per-step breakdown
        fr.fr_beam_read_timing(beam)  # clear
        fr.fr_beam_set_timing(beam, True)
        k_start, k_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        k_start.record()
        for _ in range(args.steps):
            decode()
        k_end.record()
        torch.cuda.synchronize()
        fr.fr_beam_set_timing(beam, False)
    barrier()
    elapsed_ms = slowest(t_start.elapsed_time(t_end))
    evented_ms = k_start.elapsed_time(k_end)
    stream_ms, select_ms = fr.fr_beam_read_timing(beam)
    st = fr.fr_beam_status(beam)
    if st != fr.FR_OK:
        raise RuntimeError("timed decode failed: " + fr.fr_status_string(st))
    ms_per_decode = elapsed_ms / args.steps
    cands_per_decode = B * K * D
    value = job_throughput(world, cands_per_decode, args.steps, elapsed_ms)

    # roofline of the dominant kernel: the streaming log-sum-exp / candidate
    # kernel, over its own launches (not the fused first step's)
    peak, peak_kind = measured_peaks()
    n_launch = len(stream_ms)
    per_step_bytes = [r * row_cols * elt for r in rows]
    row_kernel = ("k_slice_candidates" if not row_cols else
                  "k_rows_short" if row_cols * elt <= 16384 else "k_stream")
    idx = [i for i in range(n_launch) if not (fused0 and i % D == 0)]
    alg_bytes = sum(per_step_bytes[i % D] for i in idx)
    stream_total_ms = float(sum(stream_ms[i] for i in idx))
    achieved = alg_bytes / (stream_total_ms / 1e3) / 1e9 if stream_total_ms > 0 else 0.0
    live_rows_per_launch = sum(rows[i % D] for i in idx) / max(1, len(idx))
    # the committed counters are for k_stream over the full vocabulary
    traffic = (recorded_traffic(w.name, live_rows_per_launch)
               if (args.norm == "full" and row_kernel == "k_stream") else None)
    roofline = {"bound": "hbm" if row_cols else "latency", "achieved": achieved, "peak": peak, "unit": "GB/s",
                "frac": achieved / peak, "traffic": traffic, "peak_source": peak_kind,
                "kernel": row_kernel, "timing": "per-kernel CUDA events, second timed pass of the same decodes",
                "launches": "steps %s of each decode" % ("1.." + str(D - 1) if fused0 else "0.." + str(D - 1)),
                "alg_bytes_per_launch": alg_bytes / max(1, len(idx)),
                "ms_per_launch": stream_total_ms / max(1, len(idx)),
                "frac_of_8tbs": achieved / 8000.0}
    per_step = []
    for t in range(D):
        sm = [stream_ms[i] for i in range(t, n_launch, D)]
        se = [select_ms[i] for i in range(t, n_launch, D)]
        one = fused0 and t == 0
        per_step.append({"t": t, "live_rows": rows[t],
                         "kernels": ("k_root_step (rows and selection in one kernel)" if one else
                                     "%s + selection" % row_kernel),
                         "stream_us": 1e3 * float(np.mean(sm)),
                         "select_us": None if one else 1e3 * float(np.mean(se)),
                         "stream_gbs": per_step_bytes[t] / (float(np.mean(sm)) / 1e3) / 1e9 if sm else 0.0})
    hbm_gbs_decode = bytes_per_decode / (ms_per_decode / 1e3) / 1e9

    # end to end through the public API with host buffers
    e2e = None
    if with_e2e:
        host = []
        try:
            for t in range(D):
                h = torch.empty((B, K, V), dtype=tdt, pin_memory=True)
                h.copy_(bufs[t])
                host.append(h)
        except RuntimeError:
            host = [torch.empty((B, K, V), dtype=tdt, pin_memory=True).copy_(bufs[1 % D])] * D
        h_sids = torch.empty((B, K, D), dtype=torch.int32, pin_memory=True)
        h_scores = torch.empty((B, K), dtype=torch.float32, pin_memory=True)
        h_items = torch.empty((B, K), dtype=torch.int32, pin_memory=True)

        def e2e_decode():
            fr.fr_beam_reset(beam)
            for t in range(D):
                bufs[t].copy_(host[t], non_blocking=True)
                fr.fr_beam_step(beam, bufs[t])
            fr.fr_beam_finalize(beam, out_sids, out_scores, out_items)
            h_sids.copy_(out_sids, non_blocking=True)
            h_scores.copy_(out_scores, non_blocking=True)
            h_items.copy_(out_items, non_blocking=True)

        e2e_decode()
        torch.cuda.synchronize()
        barrier()
        a, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        for _ in range(args.e2e_steps):
            e2e_decode()
        b_.record()
        torch.cuda.synchronize()
        barrier()
        e2e_ms = slowest(a.elapsed_time(b_)) / args.e2e_steps
        e2e = {"value": world * cands_per_decode / (e2e_ms / 1e3), "unit": UNIT,
               "h2d_bytes_per_step": D * B * K * V * elt,
               "d2h_bytes_per_step": B * K * D * 4 + B * K * 4 + B * K * 4,
               "ms_per_step": e2e_ms, "steps": args.e2e_steps}
        del host

    graph = None  # release the captured decode before the buffers it names
    fr.fr_beam_destroy(beam)
    fr.fr_trie_destroy(trie)
    del bufs, out_sids, out_scores, out_items
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    return {"config": logits_config(w, args, levels), "value": value, "ms_per_step": ms_per_decode,
            "hbm_gbs": hbm_gbs_decode, "hbm_frac_of_8tbs": hbm_gbs_decode / 8000.0,
            "ms_per_step_with_kernel_events": evented_ms / args.steps, "roofline": roofline,
            "per_step": per_step, "trie_build_ms": trie_ms, "clocks": clocks.summary(), "e2e": e2e,
            "gpu_launches": args.steps * (2 * D + 2 - (1 if fused0 else 0)), "sids_np": sids_np}


# The catalog-scale workloads recorded beside the serving headline.
OTHER_CATALOG_WORKLOADS = ["wide_deep", "narrow", "skewed"]


def main():
    args = parse_args()
    if args.impl == "reference":
        run_reference(args)
        return
    if args.lmhead:
        run_lmhead(args)
        return
    import torch
    import torch.distributed as dist

    rank, world, local_rank = dist_env()
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    if world > 1:
        import datetime

        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    def barrier():
        if world > 1:
            dist.barrier()

    def slowest(x: float) -> float:
        return max_over_ranks(x, world, dist, dev)

    def workload(name: str) -> synth.Workload:
        w = synth.WORKLOADS[name]
        return synth.scaled(w, B=args.batch) if args.batch else w

    w = workload(args.config)
    b_offset, _ = rank_requests(rank, world, w.B)  # each rank decodes its own requests
    head = measure_logits_workload(w, args, dev, world, b_offset, barrier, slowest, with_e2e=not args.no_e2e)
    sids_np = head.pop("sids_np")

    # the other catalog-scale workloads at full size (same timing, no e2e /
    # CPU leg), each one's buffers freed before the next
    others = {}
    if args.config == "serving" and not args.no_workloads:
        for name in OTHER_CATALOG_WORKLOADS:
            wo = workload(name)
            bo, _ = rank_requests(rank, world, wo.B)
            r = measure_logits_workload(wo, args, dev, world, bo, barrier, slowest, with_e2e=False)
            r.pop("sids_np")
            r.pop("e2e")
            others[name] = r

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline_logits(w, sids_np, args.norm, args.temperature)

    if rank == 0:
        line = {
            "metric": METRIC, "value": head["value"], "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": head["ms_per_step"], "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f32",
            "data": "synthetic",
            "config": head["config"],
            "hbm_gbs": head["hbm_gbs"], "hbm_frac_of_8tbs": head["hbm_frac_of_8tbs"],
            "ms_per_step_with_kernel_events": head["ms_per_step_with_kernel_events"],
            "roofline": head["roofline"], "per_step": head["per_step"], "trie_build_ms": head["trie_build_ms"],
            "gpu_launches": head["gpu_launches"],
            "clocks": head["clocks"], "e2e": head["e2e"], "cpu_baseline": cpu,
        }
        if others:
            line["workloads"] = others
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
