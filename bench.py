#!/usr/bin/env python
"""Throughput of the routed MoE FFN on B200: tokens/s, with the dominant
kernel's fraction of its roofline.

A step is one pass of the whole hot path (router, top-k, experts, fixed-order
combine) over the workload's batches; the default workload is decode: three
calls at T = 1, 4 and 8 rows (13 tokens), H=4096, E=128, top_k=8, I=1536, one
shared expert, plan of 8 bands.  Inputs are seeded synthetic tensors resident
in HBM; 16 distinct x batches per row count cycle so that routing varies; the
L2 cache is flushed (a 512 MiB write) before every step, outside the timed
events.  `value` = tokens / device time (CUDA events around each step, max over
ranks); `e2e` repeats the measurement through the public API with the inputs
copied from pinned host memory and y copied back inside the timed region.

The default run also measures the prefill (T=512), load-imbalanced (T=2048)
and large (T=4096) workloads, each with its own steps, and reports them under
detail.configs: tokens/s, step time, the whole step's HBM and tensor-core
fractions and the dominant kernel's roofline.

  python bench.py [--gpus N --steps K --warmup W] [--config decode|prefill|...]
  python bench.py --impl reference ...   # the fp64 CPU oracle on the host cores

With N > 1 (torchrun) every rank runs an independent replica on its own GPU:
the tokens of a MoE layer are independent problems, so the ranks share no data
and the reported throughput is the sum over ranks (weak scaling).
"""
import argparse
import datetime
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

import workloads  # noqa: E402

METRIC = "routed MoE FFN tokens/s; decode HBM GB/s and prefill TFLOPS as % of B200 peak"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
N_BATCHES = 16
FLUSH_BYTES = 512 << 20
DETAIL_CONFIGS = ("prefill", "imbalanced", "large")
# a step shorter than this is graded against the burst GEMM peak
SUSTAINED_AFTER_S = 1.0


def whole_job_throughput(tokens, seconds, dist=None, device="cpu"):
    """Units per second of the whole job: the tokens of every rank over the
    slowest rank's time (sum and max over the ranks of the process group;
    this rank alone when dist is None).  Returns (throughput, max seconds)."""
    if dist is None:
        return tokens / seconds, seconds
    t = torch.tensor([float(tokens), seconds], device=device, dtype=torch.float64)
    tokens_t = t[:1].clone()
    seconds_t = t[1:].clone()
    dist.all_reduce(tokens_t, op=dist.ReduceOp.SUM)
    dist.all_reduce(seconds_t, op=dist.ReduceOp.MAX)
    return float(tokens_t.item()) / float(seconds_t.item()), float(seconds_t.item())


def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--config", choices=tuple(workloads.WORKLOADS), default="decode")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=500)
    ap.add_argument("--graph-steps", type=int, default=200,
                    help="steps replayed from CUDA graphs (one graph per input batch); 0 skips")
    ap.add_argument("--detail", default=None,
                    help="comma-separated workloads measured after the headline one "
                         "(default with --config decode: prefill,imbalanced,large; 'none' skips)")
    ap.add_argument("--detail-steps", type=int, default=50,
                    help="timed steps of each detail workload (at most --steps)")
    ap.add_argument("--experts", type=int, default=0,
                    help="profiling only: fewer experts (same H, I, top_k) to keep an ncu "
                         "capture to a few GB on the device")
    ap.add_argument("--flush-mib", type=int, default=FLUSH_BYTES >> 20)
    ap.add_argument("--router-only", action="store_true",
                    help="profiling only: run moe_route alone on the workload's router weights, "
                         "bias and activations (no expert weights on the device) and print its "
                         "per-call time; no bench line")
    ap.add_argument("--ep", action="store_true",
                    help="expert parallel across the ranks: rank r holds band r of the experts "
                         "(ep_plan(E, N)), every rank routes the same tokens, and the partials "
                         "are exchanged by the rank-order reduce-scatter (strong scaling)")
    ap.add_argument("--dispatch", default="auto",
                    choices=("auto", "streaming", "tensor", "streaming_tc", "streaming_simt"),
                    help="tuning: the path moe_ffn_forward takes (ep_set_dispatch)")
    ap.add_argument("--reference-budget-s", type=float, default=150.0,
                    help="wall-time budget of the reference arm's warm-up and timed steps")
    return ap.parse_args(argv)


def read_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return {k: float(p[k]) for k in FALLBACK_PEAKS}, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


# --------------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi read-only queries of this GPU's SM clock and throttle
    reasons every 100 ms, each sample stamped with the host time."""
    FIELDS = ("timestamp,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")
    NAMES = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")

    def __init__(self, device):
        self.proc = None
        uuid = str(torch.cuda.get_device_properties(device).uuid)
        self.gpu = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
        self.out = os.path.join("/tmp", f"clocks_{os.getpid()}_{id(self)}.csv")

    def start(self, wait_first_s=5.0):
        """Start sampling and wait (up to wait_first_s) for the first sample, so
        that the region measured next is covered from its start."""
        try:
            self.fh = open(self.out, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.gpu, "--query-gpu=" + self.FIELDS,
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=self.fh, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
            return
        t0 = time.time()
        while time.time() - t0 < wait_first_s and self.proc.poll() is None:
            if os.path.getsize(self.out) > 0:
                break
            time.sleep(0.02)

    def _samples(self):
        rows = []
        for line in open(self.out):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 8:
                continue
            try:
                ts = datetime.datetime.strptime(parts[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
                sm, mx = float(parts[1]), float(parts[2])
            except ValueError:
                continue
            reasons = {n for n, v in zip(self.NAMES, parts[4:8]) if v.lower() == "active"}
            rows.append((ts, sm, mx, reasons))
        return rows

    def stop(self, window=None, min_after_s=0.25):
        """Stop and summarise.  window = (t0, t1) host times: the summary keeps
        the samples taken in it, or, when the window is shorter than the
        sampling period, the samples nearest to it on either side."""
        if self.proc is None:
            return None
        if window is not None:
            time.sleep(max(0.0, window[1] + min_after_s - time.time()))
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.fh.close()
        rows = self._samples()
        os.unlink(self.out)
        if not rows:
            return None
        scope = "whole run"
        if window is not None:
            inside = [r for r in rows if window[0] <= r[0] <= window[1]]
            if inside:
                rows, scope = inside, "timed region"
            else:
                before = [r for r in rows if r[0] < window[0]][-1:]
                after = [r for r in rows if r[0] > window[1]][:1]
                if before or after:
                    rows = before + after
                    scope = "samples adjacent to the timed region (shorter than 100 ms)"
        reasons = set().union(*(r[3] for r in rows))
        return {"sm_mhz": statistics.median(r[1] for r in rows),
                "sm_max_mhz": max(r[2] for r in rows), "reasons": sorted(reasons),
                "samples": len(rows), "scope": scope}


# ------------------------------------------------------------------ workload
class Layer:
    """One MoE layer's weights on the device plus per-row-count buffers."""

    def __init__(self, wl, device, seed):
        import expert_decode_b200 as ed
        self.ed = ed
        self.wl = wl
        self.W = workloads.make_weights(wl, device=device, seed=workloads.SEED_BASE)
        self.shared = (None if self.W["ws_gate"] is None
                       else (self.W["ws_gate"], self.W["ws_up"], self.W["ws_down"]))
        self.plan = ed.ep_plan(wl.E, wl.bands[0])
        self.xs = {T: [workloads.make_x(wl, T, device=device, seed=seed, batch=b + 100 * T)
                       for b in range(N_BATCHES if T <= 8 else 2)] for T in wl.T}
        self.ids = {T: torch.empty((T, wl.top_k), dtype=torch.int32, device=device)
                    for T in wl.T}
        self.wts = {T: torch.empty((T, wl.top_k), dtype=torch.float32, device=device)
                    for T in wl.T}
        self.y = {T: torch.empty((T, wl.H), dtype=torch.float32, device=device) for T in wl.T}
        ws = max(ed.moe_ffn_workspace_size(T, wl.H, wl.E, wl.top_k, wl.I, wl.I_s)
                 for T in wl.T)
        self.workspace = torch.empty(ws, dtype=torch.uint8, device=device)
        self.launches = 0
        self.ffn_kernels = {}  # kernels of the last forward call per row count

    def call(self, T, b, x=None):
        ed = self.ed
        x = self.xs[T][b % len(self.xs[T])] if x is None else x
        ed.moe_route(x, self.W["w_router"], self.W["bias"], self.wl.top_k, ids=self.ids[T],
                     weights=self.wts[T])
        self.launches += ed.ep_last_launch_count()

    def ffn(self, T, b, x=None, y=None):
        ed = self.ed
        x = self.xs[T][b % len(self.xs[T])] if x is None else x
        ed.moe_ffn_forward(x, self.ids[T], self.wts[T], self.W["w_gate"], self.W["w_up"],
                           self.W["w_down"], self.shared, self.plan,
                           y=self.y[T] if y is None else y, workspace=self.workspace)
        n = ed.ep_last_launch_count()
        self.launches += n
        self.ffn_kernels[T] = n

    def distinct_experts(self, T, b):
        self.call(T, b)
        torch.cuda.synchronize()
        return int(torch.unique(self.ids[T]).numel())


# ---------------------------------------------------------------- bytes/flops
def kernel_cost(wl, T, n_distinct, tensor_path):
    """Algorithmic bytes / flops of the dominant kernel (gate/up) of one call,
    and of the whole call.  Weights: only the picked experts plus the shared
    one, each read once; activations at their stored widths."""
    H, I, I_s, k = wl.H, wl.I, wl.I_s, wl.top_k
    xb = 4 if wl.x_dtype == "f32" else 2
    n_exp = n_distinct + (1 if I_s else 0)
    w_gu = (n_distinct * 2 * H * I + (2 * H * I_s if I_s else 0)) * 2
    w_dn = (n_distinct * H * I + (H * I_s if I_s else 0)) * 2
    P = T * k
    flops_gu = 2 * (P * 2 * H * I + (T * 2 * H * I_s if I_s else 0))
    flops_dn = 2 * (P * H * I + (T * H * I_s if I_s else 0))
    if tensor_path:
        gu_bytes = w_gu + (P + (T if I_s else 0)) * H * 2 + (P * I + T * I_s) * 2
    else:
        gu_bytes = w_gu + T * H * xb
    call_bytes = (wl.E * H * 2 + T * H * xb + T * k * 8) + w_gu + w_dn + T * H * 4
    call_flops = 2 * T * H * wl.E + flops_gu + flops_dn
    return {"gu_bytes": gu_bytes, "gu_flops": flops_gu, "call_bytes": call_bytes,
            "call_flops": call_flops, "n_experts": n_exp}


def _code_only(text):
    """C/C++/CUDA source with its comments removed and runs of white space
    collapsed (string and character literals are kept as they are)."""
    out, i, n = [], 0, len(text)
    while i < n:
        c = text[i]
        if c in "\"'":
            j = i + 1
            while j < n and text[j] != c:
                j += 2 if text[j] == "\\" else 1
            out.append(text[i:j + 1])
            i = j + 1
        elif text.startswith("//", i):
            j = text.find("\n", i)
            i = n if j < 0 else j
        elif text.startswith("/*", i):
            j = text.find("*/", i + 2)
            i = n if j < 0 else j + 2
            out.append(" ")
        else:
            out.append(c)
            i += 1
    return " ".join("".join(out).split())


def source_digest():
    """Digest of the kernel sources' code (comments excluded): the ncu counters
    committed under profiles/ stand for the kernels while it matches."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "expert_decode_b200", "csrc")
    for f in sorted(os.listdir(csrc)):
        with open(os.path.join(csrc, f), encoding="utf-8") as fh:
            h.update(f.encode() + b"\0" + _code_only(fh.read()).encode())
    return h.hexdigest()[:16]


def traffic_for(kernel, workload):
    """DRAM bytes per launch from the committed ncu summary, if it was taken
    on the current kernel sources."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        d = json.load(f)
    e = d.get(f"{kernel}:{workload}")
    if not e or e.get("source_digest") != source_digest():
        return None
    return e.get("dram_bytes_per_launch")




# ------------------------------------------------------------------- CPU legs
class HostDecode:
    """The oracle's view of a workload, drawn on the host from the same seeded
    recipe (the host generator's numbers differ from the device generator's;
    shapes, distributions and biases are the workload's).  Only the router,
    the shared expert and the experts that the batches pick are drawn."""

    def __init__(self, wl, n_batches=2, seed=workloads.SEED_BASE):
        import oracle
        self.o = oracle.load()
        self.wl = wl
        w_router, bias = workloads.make_router(wl, "cpu", seed)
        self.wr = workloads.bits(w_router)
        self.bias = None if bias is None else bias.numpy()
        sh = workloads.make_shared(wl, "cpu", seed)
        self.shared = None if sh is None else tuple(workloads.bits(t) for t in sh)
        self.batches = [(T, workloads.bits(workloads.make_x(wl, T, "cpu", seed,
                                                            batch=b + 100 * T)))
                        for b in range(n_batches) for T in wl.T]
        self.mats = ({}, {}, {})
        self.seed = seed

    def route(self, xh, threads):
        return self.o.route(xh, self.wr, self.bias, self.wl.top_k, threads=threads)

    def ensure(self, experts):
        for e in experts:
            if e not in self.mats[0]:
                for m, which in zip(self.mats, ("w_gate", "w_up", "w_down")):
                    m[e] = workloads.bits(workloads.make_expert(self.wl, which, e, "cpu",
                                                                self.seed))

    def ffn(self, xh, ids, w, threads):
        return self.o.moe_ffn_monolith(xh, ids, w, *self.mats, self.wl.E, shared=self.shared,
                                       threads=threads)


def oracle_tokens(host, tokens, threads):
    """Route + monolith FFN of the given tokens (rows of the host batches,
    concatenated) in one oracle call each, OpenMP over tokens.  The experts'
    host copies are drawn before the clock starts.  Returns seconds."""
    xh = np.concatenate([x for _, x in host.batches], axis=0)[tokens]
    ids, w, _ = host.route(xh, threads)
    host.ensure(sorted(set(int(e) for e in ids.ravel())))
    t0 = time.perf_counter()
    ids, w, _ = host.route(xh, threads)
    host.ffn(xh, ids, w, threads)
    return time.perf_counter() - t0


def cpu_baseline(wl):
    """The oracle as it stands on all of this host's cores: the first two
    batches of every row count in one route and one FFN call (OpenMP over the
    tokens), and one token alone on one thread."""
    host = HostDecode(wl, n_batches=2)
    n_tok = sum(x.shape[0] for _, x in host.batches)
    cores = os.cpu_count() or 1
    threads = min(cores, n_tok)
    sec = oracle_tokens(host, np.arange(n_tok), threads)
    sec1 = oracle_tokens(host, np.arange(1), 1)
    return {"value": n_tok / sec, "unit": "tokens/s", "cores": threads, "kind": "oracle",
            "sample": f"{n_tok} tokens: the first 2 batches of each row count "
                      f"({', '.join(f'T={T}' for T in wl.T)}), fp64 route + monolith FFN in "
                      f"one call each, OpenMP over tokens; inputs drawn on the host from "
                      f"the workload's recipe",
            "host_cores": cores, "cpu_model": cpu_model(),
            "one_thread": {"value": 1.0 / sec1, "unit": "tokens/s", "sample": "1 token"}}


def run_reference(args, wl):
    """The reference arm: the fp64 CPU oracle, as it stands, on this host's
    cores.  Nothing here loads the CUDA library or touches a GPU.

    The work is the workload's own tokens: the decode step's batches (T = 1,
    4 and 8, drawn on the host).  A token of the workload costs its routing
    plus top_k + 1 expert evaluations (routed picks and the shared expert).
    When W + K whole steps fit the wall-time budget, a step is the workload's
    tokens in one route and one FFN call; otherwise a step is one oracle FFN
    call over a bounded number n of (token, expert) evaluations, each counted
    as 1 / (top_k + 1) token, with a token's routing timed when it is first
    met; n = the host's cores (at most the workload's evaluations), which run
    side by side in about one evaluation's time."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    host = HostDecode(wl, n_batches=1)
    cores = os.cpu_count() or 1
    xh = np.concatenate([x for _, x in host.batches], axis=0)
    n_tok = xh.shape[0]
    ids, w, _ = host.route(xh, min(cores, n_tok))
    host.ensure(sorted(set(int(e) for e in ids.ravel())))
    per_token = wl.top_k + (1 if host.shared is not None else 0)
    steps = args.warmup + args.steps
    # one whole step, timed once, decides the form of the steps
    t_whole = oracle_tokens(host, np.arange(n_tok), min(cores, n_tok))
    if steps * t_whole <= args.reference_budget_s:
        mode = "whole"
        threads = min(cores, n_tok)
        sample = (f"each step: the workload's {n_tok} tokens (one batch each of "
                  f"{', '.join(f'T={T}' for T in wl.T)}) through one fp64 route and one "
                  f"monolith FFN call, OpenMP over tokens")
    else:
        # n <= cores evaluations run side by side in about one evaluation's
        # time, so every core takes one
        mode = "evaluations"
        n = min(cores, n_tok * per_token)
        threads = n
        sample = (f"each step: {n} (token, expert) evaluations of the workload's {n_tok} "
                  f"tokens (one batch each of {', '.join(f'T={T}' for T in wl.T)}) in one "
                  f"oracle FFN call (OpenMP over rows), each 1/{per_token} token, a token's "
                  f"routing timed when it is first met")
    evals = [(t, int(ids[t, j]), float(w[t, j])) for t in range(n_tok) for j in range(wl.top_k)]
    if host.shared is not None:
        evals += [(t, wl.E, 1.0) for t in range(n_tok)]
        tables = tuple({**m, wl.E: s} for m, s in zip(host.mats, host.shared))
    else:
        tables = host.mats
    total_tok, total_s = 0.0, 0.0
    seen = set()
    for i in range(steps):
        if mode == "whole":
            sec = oracle_tokens(host, np.arange(n_tok), threads)
            tok = float(n_tok)
        else:
            batch = [evals[(i * threads + q) % len(evals)] for q in range(threads)]
            rows = np.array([t for t, _, _ in batch])
            new = sorted(set(rows.tolist()) - seen)
            t0 = time.perf_counter()
            if new:
                host.route(xh[new], min(cores, len(new)))
            host.o.moe_ffn_monolith(xh[rows], np.array([[e] for _, e, _ in batch], dtype=np.int32),
                                    np.array([[wt] for _, _, wt in batch]), *tables, wl.E + 1,
                                    threads=threads)
            sec = time.perf_counter() - t0
            seen.update(new)
            if len(seen) == n_tok:
                seen = set()
            tok = threads / per_token
        if i >= args.warmup:
            total_tok += tok
            total_s += sec
    value = total_tok / total_s
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * total_s / max(args.steps, 1), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": wl.description, "bands": wl.bands[0]},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": threads, "kind": "oracle",
                         "sample": sample, "host_cores": cores, "cpu_model": cpu_model()},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# -------------------------------------------------------------------- our arm
def measure(args, wl, device, rank, dist, peaks, K, warmup, sampler=None, with_graph=True,
            e2e_steps=0):
    """Every measurement of one workload: the timed steps, the per-kernel and
    per-call passes, CUDA-graph replay and the end-to-end pass."""
    import expert_decode_b200 as ed
    layer = Layer(wl, device, workloads.SEED_BASE + 7919 * rank)
    Ts = wl.T
    tensor_path = {T: T > 8 for T in Ts}
    flush = torch.empty(args.flush_mib << 20, dtype=torch.uint8, device=device)

    # per (T, batch): distinct experts picked (fixed for a given batch)
    n_batches = {T: len(layer.xs[T]) for T in Ts}
    distinct = {(T, b): layer.distinct_experts(T, b) for T in Ts for b in range(n_batches[T])}
    dom_index = {T: (2 if tensor_path[T] else 0) for T in Ts}   # kernel j of the ffn call

    def step(i, prof=None):
        for T in Ts:
            if prof is not None:
                ed.ep_profile_events(prof[("route", T)])
            layer.call(T, i)
            if prof is not None:
                ed.ep_profile_events(prof[T])
            layer.ffn(T, i)
            if prof is not None:
                ed.ep_profile_events(None)

    for i in range(warmup):
        flush.zero_()
        step(i)
    torch.cuda.synchronize()
    ed.ep_check_status()

    ev_s = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    ev_e = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    layer.launches = 0
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    if sampler is not None:
        sampler.start()
    t_wall0 = time.time()
    # an NVTX range marks the timed launches for a profiler's launch filter
    # (ncu --nvtx --nvtx-include timed/)
    torch.cuda.nvtx.range_push("timed")
    for i in range(K):
        flush.zero_()
        ev_s[i].record()
        step(warmup + i)
        ev_e[i].record()
    torch.cuda.nvtx.range_pop()
    torch.cuda.synchronize()
    t_wall1 = time.time()
    clocks = sampler.stop((t_wall0, t_wall1)) if sampler is not None else None
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    ed.ep_check_status()
    launches = layer.launches

    # per-call pass: events around each row count's route + forward only, so
    # the kernels inside a call keep their early (programmatic) launches
    call_s = {T: [torch.cuda.Event(enable_timing=True) for _ in range(K)] for T in Ts}
    call_e = {T: [torch.cuda.Event(enable_timing=True) for _ in range(K)] for T in Ts}
    for i in range(K):
        flush.zero_()
        for T in Ts:
            call_s[T][i].record()
            layer.call(T, warmup + i)
            layer.ffn(T, warmup + i)
            call_e[T][i].record()
    torch.cuda.synchronize()

    # per-kernel pass: every kernel bracketed by its own events, for the
    # dominant kernel's duration (events between launches stop the early
    # launch of the next kernel, so the throughput above is taken without them)
    nk = 10
    prof = [{key: [torch.cuda.Event(enable_timing=True) for _ in range(2 * nk)]
             for key in list(Ts) + [("route", T) for T in Ts]} for _ in range(K)]
    for p in prof:
        for evs in p.values():
            for e in evs:
                e.record()
    torch.cuda.synchronize()
    for i in range(K):
        flush.zero_()
        step(warmup + i, prof[i])
    torch.cuda.synchronize()

    step_ms = [ev_s[i].elapsed_time(ev_e[i]) for i in range(K)]
    dev_s = sum(step_ms) / 1e3
    tokens_rank = K * sum(Ts)
    # dominant kernel: summed algorithmic bytes over summed durations
    dom_bytes = dom_flops = dom_s = 0.0
    step_bytes = step_flops = 0.0
    per_T = {}
    for T in Ts:
        j = dom_index[T]
        durs, byts, fl, cbytes, cflops = [], 0.0, 0.0, 0.0, 0.0
        for i in range(K):
            b = warmup + i
            c = kernel_cost(wl, T, distinct[(T, b % n_batches[T])], tensor_path[T])
            durs.append(prof[i][T][2 * j].elapsed_time(prof[i][T][2 * j + 1]) / 1e3)
            byts += c["gu_bytes"]
            fl += c["gu_flops"]
            cbytes += c["call_bytes"]
            cflops += c["call_flops"]
        step_bytes += cbytes
        step_flops += cflops
        dom_bytes += byts
        dom_flops += fl
        dom_s += sum(durs)
        call_sec = sum(call_s[T][i].elapsed_time(call_e[T][i]) for i in range(K)) / 1e3
        per_T[f"T={T}"] = {
            "call_us": 1e6 * call_sec / K,
            "call_hbm_GBps": cbytes / call_sec / 1e9,
            "call_hbm_frac": cbytes / call_sec / 1e9 / peaks["hbm_gbs"],
            "call_bytes": cbytes / K,
            "dominant_kernel_us": 1e6 * sum(durs) / K,
            "dominant_kernel_GBps": byts / sum(durs) / 1e9}
        # mean duration of every kernel of the route and forward calls
        if tensor_path[T]:
            names = ["plan", "gather", "gate_up", "down", "combine"]
        elif layer.ffn_kernels.get(T) == 3:
            names = ["gate_up", "down", "fold"]
        else:
            names = ["gate_up", "down_fold"]
        kus = {}
        for jj, name in enumerate(names):
            kus[name] = 1e3 * sum(prof[i][T][2 * jj].elapsed_time(prof[i][T][2 * jj + 1])
                                  for i in range(K)) / K
        kus["router"] = 1e3 * sum(prof[i][("route", T)][0].elapsed_time(prof[i][("route", T)][1])
                                  for i in range(K)) / K
        per_T[f"T={T}"]["kernels_us"] = {k: round(v, 2) for k, v in kus.items()}

    value, dev_s_max = whole_job_throughput(tokens_rank, dev_s, dist, device)

    # roofline of the dominant kernel: the burst GEMM peak for short steps
    peak_tf_key = "bf16_tflops_sustained" if dev_s / K >= SUSTAINED_AFTER_S else "bf16_tflops"
    peak_tf = peaks[peak_tf_key]
    t_hbm = dom_bytes / (peaks["hbm_gbs"] * 1e9)
    t_tc = dom_flops / (peak_tf * 1e12)
    if t_hbm >= t_tc:
        roof = {"bound": "hbm", "achieved": dom_bytes / dom_s / 1e9, "peak": peaks["hbm_gbs"],
                "unit": "GB/s"}
    else:
        roof = {"bound": "tensor", "achieved": dom_flops / dom_s / 1e12, "peak": peak_tf,
                "unit": "TFLOP/s"}
    roof["frac"] = roof["achieved"] / roof["peak"]
    kname = "grouped_gemm_kernel<true>" if any(tensor_path.values()) else "decode_gate_up"
    roof["traffic"] = traffic_for(kname, wl.name)
    roof["kernel"] = kname
    roof["peak_source"] = "measured" if peaks.get("_source") == "measured" else "fallback"
    roof["peak_key"] = "hbm_gbs" if roof["bound"] == "hbm" else peak_tf_key

    # the same steps replayed from CUDA graphs, one per input batch (the
    # kernels' launch attributes, programmatic dependent launch included, are
    # captured with them); the L2 flush stays outside the graphs
    graph = None
    if with_graph and args.graph_steps > 0:
        nb = min(len(layer.xs[T]) for T in Ts)
        graphs = []
        for b in range(nb):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                step(b)
            graphs.append(g)
        torch.cuda.synchronize()
        KG = min(args.graph_steps, K) if wl.T[0] > 8 else args.graph_steps
        gs = [torch.cuda.Event(enable_timing=True) for _ in range(KG)]
        ge = [torch.cuda.Event(enable_timing=True) for _ in range(KG)]
        for i in range(KG):
            flush.zero_()
            gs[i].record()
            graphs[i % nb].replay()
            ge[i].record()
        torch.cuda.synchronize()
        ed.ep_check_status()
        g_s = sum(gs[i].elapsed_time(ge[i]) for i in range(KG)) / 1e3
        graph = {"value": KG * sum(Ts) / g_s, "unit": "tokens/s", "ms_per_step": 1e3 * g_s / KG,
                 "steps": KG, "graphs": nb}
        del graphs

    # e2e: inputs from pinned host memory, y back to pinned host, in the region.
    # The copies run on their own streams with two device buffers per row
    # count, so that step i + 1's inputs arrive and step i - 1's outputs leave
    # while step i computes (as a serving loop would do); every step's copies
    # are inside the timed region, which ends when the last output is on the
    # host.
    e2e = None
    if e2e_steps > 0:
        KE = e2e_steps
        hx = {T: [x.cpu().pin_memory() for x in layer.xs[T]] for T in Ts}
        dx = {T: [torch.empty_like(layer.xs[T][0]) for _ in range(2)] for T in Ts}
        dy = {T: [torch.empty((T, wl.H), dtype=torch.float32, device=device) for _ in range(2)]
              for T in Ts}
        hy = {T: [torch.empty((T, wl.H), dtype=torch.float32).pin_memory() for _ in range(2)]
              for T in Ts}
        s_in, s_out = torch.cuda.Stream(device), torch.cuda.Stream(device)
        comp = torch.cuda.current_stream(device)
        ev = lambda: torch.cuda.Event()
        ev_in = {T: [ev(), ev()] for T in Ts}
        ev_done = {T: [ev(), ev()] for T in Ts}
        ev_out = {T: [ev(), ev()] for T in Ts}
        es = torch.cuda.Event(enable_timing=True)
        ee = torch.cuda.Event(enable_timing=True)
        h2d = sum(hx[T][0].numel() * hx[T][0].element_size() for T in Ts)
        d2h = sum(hy[T][0].numel() * 4 for T in Ts)
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize()
        es.record(comp)
        for i in range(KE):
            q = i % 2
            for T in Ts:
                b = i % len(hx[T])
                with torch.cuda.stream(s_in):
                    if i >= 2:
                        s_in.wait_event(ev_done[T][q])  # dx[T][q] is free again
                    dx[T][q].copy_(hx[T][b], non_blocking=True)
                    ev_in[T][q].record(s_in)
                comp.wait_event(ev_in[T][q])
                if i >= 2:
                    comp.wait_event(ev_out[T][q])  # dy[T][q] has left for the host
                layer.call(T, 0, x=dx[T][q])
                layer.ffn(T, 0, x=dx[T][q], y=dy[T][q])
                ev_done[T][q].record(comp)
                with torch.cuda.stream(s_out):
                    s_out.wait_event(ev_done[T][q])
                    hy[T][q].copy_(dy[T][q], non_blocking=True)
                    ev_out[T][q].record(s_out)
        for T in Ts:
            for q in range(2):
                comp.wait_event(ev_out[T][q])
        ee.record(comp)
        torch.cuda.synchronize()
        e2e_s = es.elapsed_time(ee) / 1e3
        e2e_value, e2e_s = whole_job_throughput(KE * sum(Ts), e2e_s, dist, device)
        e2e = {"value": e2e_value, "unit": "tokens/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": KE,
               "l2": "not flushed",
               "copies": "own streams, two buffers per row count: a step's input copy and "
                         "the previous step's output copy overlap its compute"}

    step_s = dev_s / K
    out = {
        "value": value, "ms_per_step": 1e3 * dev_s_max / K, "steps": K, "warmup": warmup,
        "roofline": roof, "e2e": e2e, "gpu_launches": launches, "clocks": clocks,
        "per_T": per_T, "cuda_graph": graph,
        "step_hbm_GBps": step_bytes / dev_s / 1e9,
        "step_hbm_frac": step_bytes / dev_s / 1e9 / peaks["hbm_gbs"],
        "step_tflops": step_flops / dev_s / 1e12,
        "step_tensor_frac": step_flops / dev_s / 1e12 / peak_tf,
        "step_tensor_peak_key": peak_tf_key,
        "step_roofline_frac": max(step_bytes / (peaks["hbm_gbs"] * 1e9),
                                  step_flops / (peak_tf * 1e12)) / step_s,
        "wall_s": t_wall1 - t_wall0,
    }
    del layer, flush
    torch.cuda.empty_cache()
    return out


def nvfp4_cost(wl, T, n_distinct):
    """Algorithmic bytes of one NVFP4 decode call: the picked experts' and the
    shared expert's codes (half a byte per weight) and block scales (one byte
    per 16 weights) read once, the activations and h at their stored widths
    (fp16 hi/lo for h), the contributions and y in fp32.  Returns the gate/up
    kernel's bytes and the call's (router included)."""
    H, I, I_s, k = wl.H, wl.I, wl.I_s, wl.top_k
    per_w = 0.5 + 1.0 / 16
    w_gu = (n_distinct * 2 * H * I + 2 * H * I_s) * per_w
    w_dn = (n_distinct * H * I + H * I_s) * per_w
    P = T * k
    h_bytes = (P * I + T * I_s) * 2 * 2
    gu_bytes = w_gu + T * H * 2 + h_bytes
    call_bytes = (wl.E * H * 2 + T * H * 2 + T * k * 8) + w_gu + w_dn + T * H * 4
    return gu_bytes, call_bytes


def measure_nvfp4(args, wl, device, peaks, K, warmup):
    """The decode workload with every expert matrix in NVFP4 (moe_ffn_forward_nvfp4
    after the same bf16 router): tokens/s over the row counts, per-call and
    per-kernel times, and the gate/up kernel's roofline at the stored bytes."""
    import expert_decode_b200 as ed
    seed = workloads.SEED_BASE
    mats = [workloads.make_nvfp4_experts(wl.E, rows, cols, seed + 11 + j, device=device)
            for j, (rows, cols) in enumerate(((wl.I, wl.H), (wl.I, wl.H), (wl.H, wl.I)))]
    shared = tuple({"packed": m["packed"][0], "scales": m["scales"][0],
                    "tensor_scale": m["tensor_scale"]}
                   for m in (workloads.make_nvfp4_experts(1, rows, cols, seed + 14 + j, device)
                             for j, (rows, cols) in enumerate(((wl.I_s, wl.H), (wl.I_s, wl.H),
                                                               (wl.H, wl.I_s)))))
    w_router, bias = workloads.make_router(wl, device)
    plan = ed.ep_plan(wl.E, wl.bands[0])
    Ts = wl.T
    xs = {T: [workloads.make_x(wl, T, device=device, seed=seed, batch=b + 100 * T)
              for b in range(N_BATCHES)] for T in Ts}
    ids = {T: torch.empty((T, wl.top_k), dtype=torch.int32, device=device) for T in Ts}
    wts = {T: torch.empty((T, wl.top_k), dtype=torch.float32, device=device) for T in Ts}
    ys = {T: torch.empty((T, wl.H), dtype=torch.float32, device=device) for T in Ts}
    ws = torch.empty(max(ed.moe_ffn_nvfp4_workspace_size(T, wl.H, wl.E, wl.top_k, wl.I, wl.I_s)
                         for T in Ts), dtype=torch.uint8, device=device)
    flush = torch.empty(args.flush_mib << 20, dtype=torch.uint8, device=device)
    launches = [0]

    def call(T, i, prof=None):
        x = xs[T][i % N_BATCHES]
        if prof is not None:
            ed.ep_profile_events(prof[("route", T)])
        ed.moe_route(x, w_router, bias, wl.top_k, ids=ids[T], weights=wts[T])
        launches[0] += ed.ep_last_launch_count()
        if prof is not None:
            ed.ep_profile_events(prof[T])
        ed.moe_ffn_forward_nvfp4(x, ids[T], wts[T], *mats, shared, plan, y=ys[T], workspace=ws)
        launches[0] += ed.ep_last_launch_count()
        if prof is not None:
            ed.ep_profile_events(None)

    for i in range(warmup):
        flush.zero_()
        for T in Ts:
            call(T, i)
    torch.cuda.synchronize()
    ed.ep_check_status()
    distinct = {}
    for T in Ts:
        for b in range(N_BATCHES):
            call(T, b)
            torch.cuda.synchronize()
            distinct[(T, b)] = int(torch.unique(ids[T]).numel())
    ev_s = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    ev_e = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    call_s = {T: [torch.cuda.Event(enable_timing=True) for _ in range(K)] for T in Ts}
    call_e = {T: [torch.cuda.Event(enable_timing=True) for _ in range(K)] for T in Ts}
    launches[0] = 0
    torch.cuda.synchronize()
    for i in range(K):
        flush.zero_()
        ev_s[i].record()
        for T in Ts:
            call_s[T][i].record()
            call(T, warmup + i)
            call_e[T][i].record()
        ev_e[i].record()
    torch.cuda.synchronize()
    ed.ep_check_status()
    n_launch = launches[0]
    nk = 4
    prof = [{key: [torch.cuda.Event(enable_timing=True) for _ in range(2 * nk)]
             for key in list(Ts) + [("route", T) for T in Ts]} for _ in range(K)]
    for p in prof:
        for evs in p.values():
            for e in evs:
                e.record()
    torch.cuda.synchronize()
    for i in range(K):
        flush.zero_()
        for T in Ts:
            call(T, warmup + i, prof[i])
    torch.cuda.synchronize()
    dev_s = sum(ev_s[i].elapsed_time(ev_e[i]) for i in range(K)) / 1e3
    per_T = {}
    gu_b = gu_s = 0.0
    for T in Ts:
        names = ["to_f16", "gate_up", "down", "combine"]
        kus = {nm: 1e3 * sum(prof[i][T][2 * j].elapsed_time(prof[i][T][2 * j + 1])
                             for i in range(K)) / K for j, nm in enumerate(names)}
        kus["router"] = 1e3 * sum(prof[i][("route", T)][0].elapsed_time(prof[i][("route", T)][1])
                                  for i in range(K)) / K
        costs = [nvfp4_cost(wl, T, distinct[(T, (warmup + i) % N_BATCHES)]) for i in range(K)]
        call_sec = sum(call_s[T][i].elapsed_time(call_e[T][i]) for i in range(K)) / 1e3
        cb = sum(c[1] for c in costs)
        gb = sum(c[0] for c in costs)
        gs = sum(prof[i][T][2].elapsed_time(prof[i][T][3]) for i in range(K)) / 1e3
        gu_b += gb
        gu_s += gs
        per_T[f"T={T}"] = {"call_us": 1e6 * call_sec / K, "call_bytes": cb / K,
                           "call_hbm_GBps": cb / call_sec / 1e9,
                           "call_hbm_frac": cb / call_sec / 1e9 / peaks["hbm_gbs"],
                           "gate_up_GBps": gb / gs / 1e9,
                           "kernels_us": {k: round(v, 2) for k, v in kus.items()}}
    achieved = gu_b / gu_s / 1e9
    roof = {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
            "frac": achieved / peaks["hbm_gbs"], "kernel": "stream_gate_up_fp4_kernel",
            "traffic": traffic_for("stream_gate_up_fp4_kernel", "decode_nvfp4"),
            "peak_source": "measured" if peaks.get("_source") == "measured" else "fallback",
            "bytes": "codes 0.5 B + block scales 1/16 B per weight, x fp16, h fp16 hi/lo"}
    out = {"workload": wl.description + ", every expert matrix NVFP4 (E2M1 codes, E4M3 "
                                        "scales per 16, fp32 tensor scale)",
           "value": K * sum(Ts) / dev_s, "unit": "tokens/s", "ms_per_step": 1e3 * dev_s / K,
           "steps": K, "warmup": warmup, "gpu_launches": n_launch, "roofline": roof,
           "per_T": per_T}
    del mats, shared, flush, ws
    torch.cuda.empty_cache()
    return out


def run_ours(args, wl):
    import expert_decode_b200 as ed  # the library must load
    ed.ep_set_dispatch(args.dispatch)
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    dist = None
    if world > 1:
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=device)
    peaks, peak_src = read_peaks()
    peaks["_source"] = peak_src
    K = args.steps
    sampler = ClockSampler(device) if rank == 0 else None
    head = measure(args, wl, device, rank, dist, peaks, K, args.warmup, sampler,
                   e2e_steps=min(args.e2e_steps, K))

    if args.detail is None:
        detail_names = list(DETAIL_CONFIGS) if wl.name == "decode" else []
    elif args.detail == "none":
        detail_names = []
    else:
        detail_names = [n for n in args.detail.split(",") if n]
    configs = {}
    for name in detail_names:
        dwl = workloads.WORKLOADS[name]
        KD = max(1, min(args.detail_steps, K))
        s2 = ClockSampler(device) if rank == 0 else None
        r = measure(args, dwl, device, rank, dist, peaks, KD, max(3, min(args.warmup, 10)), s2,
                    with_graph=False, e2e_steps=min(args.e2e_steps, KD))
        per = r["per_T"][f"T={dwl.T[0]}"]
        configs[name] = {
            "workload": dwl.description, "bands": dwl.bands[0], "value": r["value"],
            "unit": "tokens/s", "ms_per_step": r["ms_per_step"], "steps": KD,
            "warmup": r["warmup"], "e2e": r["e2e"],
            "step_hbm_frac": r["step_hbm_frac"], "step_tflops": r["step_tflops"],
            "step_tensor_frac": r["step_tensor_frac"],
            "step_tensor_peak_key": r["step_tensor_peak_key"],
            "step_roofline_frac": r["step_roofline_frac"], "roofline": r["roofline"],
            "kernels_us": per["kernels_us"], "call_us": per["call_us"], "clocks": r["clocks"]}

    if wl.name == "decode" and args.detail != "none":
        KD = max(1, min(args.detail_steps, K))
        configs["decode_nvfp4"] = measure_nvfp4(args, wl, device, peaks, KD,
                                                max(3, min(args.warmup, 10)))

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(wl)

    if dist is not None:
        dist.destroy_process_group()
    if rank != 0:
        return
    line = {
        "metric": METRIC, "value": head["value"], "unit": "tokens/s", "n_gpus": world,
        "steps": K, "warmup": args.warmup, "ms_per_step": head["ms_per_step"],
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": wl.description, "bands": wl.bands[0],
                   "dispatch": args.dispatch,
                   "l2": "flushed before every step (512 MiB write)",
                   "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                   "batches": "16 distinct x batches per row count, cycled",
                   "roofline_timing": "dominant kernel timed in a second pass of K steps "
                                      "with events around each kernel"},
        "roofline": head["roofline"],
        "cpu_baseline": cpu,
        "e2e": head["e2e"],
        "gpu_launches": head["gpu_launches"],
        "clocks": head["clocks"],
        "detail": {"per_T": head["per_T"], "wall_s": head["wall_s"],
                   "cuda_graph": head["cuda_graph"],
                   "step_hbm_GBps": head["step_hbm_GBps"],
                   "step_hbm_frac": head["step_hbm_frac"],
                   "step_tflops": head["step_tflops"],
                   "step_tensor_frac": head["step_tensor_frac"],
                   "peak_source": peak_src,
                   "dominant_kernel": ("gate/up GEMM (tcgen05)" if wl.T[0] > 8 else
                                       "decode gate/up (tcgen05 from 2 tokens with bf16 x, "
                                       "CUDA cores below)"),
                   "configs": configs},
    }
    print(json.dumps(line), flush=True)


def run_ep(args, wl):
    """Band-resident expert parallelism across the ranks of one node: rank r
    holds the experts of band r of ep_plan(E, N) only, every rank routes the
    same batch, computes its band's partial, and the partials are folded in
    rank order by the reduce-scatter exchange (expert_decode_b200.ep).  The
    whole job processes each token once: value = tokens / slowest rank's
    device time (strong scaling).  Collectives are NCCL's; the kernels read
    this GPU's memory only."""
    import expert_decode_b200 as ed
    from expert_decode_b200 import ep
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    dist = None
    if world > 1:
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=device)
    plan = ed.ep_plan(wl.E, world)
    lo, hi = plan.band_start[rank], plan.band_start[rank + 1]
    band = tuple(torch.stack([workloads.make_expert(wl, which, e, device) for e in range(lo, hi)])
                 for which in ("w_gate", "w_up", "w_down"))
    w_router, bias = workloads.make_router(wl, device)
    shared = workloads.make_shared(wl, device)
    xs = {T: [workloads.make_x(wl, T, device=device, batch=b + 100 * T)
              for b in range(N_BATCHES if T <= 8 else 2)] for T in wl.T}
    flush = torch.empty(args.flush_mib << 20, dtype=torch.uint8, device=device)

    def step(i):
        for T in wl.T:
            x = xs[T][i % len(xs[T])]
            ids, w = ed.moe_route(x, w_router, bias, wl.top_k)
            if dist is None:
                ed.moe_ffn_forward(x, ids, w, *band, shared, plan)
            else:
                ep.ep_forward(x, ids, w, band, shared, plan, rank)

    for i in range(args.warmup):
        flush.zero_()
        step(i)
    torch.cuda.synchronize()
    ed.ep_check_status()
    K = args.steps
    ev_s = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    ev_e = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    for i in range(K):
        flush.zero_()
        ev_s[i].record()
        step(args.warmup + i)
        ev_e[i].record()
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    ed.ep_check_status()
    dev_s = sum(ev_s[i].elapsed_time(ev_e[i]) for i in range(K)) / 1e3
    tokens = K * sum(wl.T)
    if dist is not None:
        t = torch.tensor([dev_s], device=device, dtype=torch.float64)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        dev_s = float(t.item())
        dist.destroy_process_group()
    if rank != 0:
        return
    line = {
        "metric": METRIC, "value": tokens / dev_s, "unit": "tokens/s", "n_gpus": world,
        "steps": K, "warmup": args.warmup, "ms_per_step": 1e3 * dev_s / K,
        "higher_is_better": True, "scaling": "strong", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": wl.description, "bands": world,
                   "parallelism": f"expert-parallel bands x{world} (rank-order reduce-scatter)",
                   "l2": "flushed before every step (512 MiB write)"},
        "roofline": None, "cpu_baseline": None, "e2e": None, "gpu_launches": None,
        "clocks": None,
    }
    print(json.dumps(line), flush=True)


def run_router_only(args, wl):
    """Profiling aid: moe_route alone, W warm-up and K timed calls per token count."""
    import expert_decode_b200 as ed
    device = torch.device("cuda", 0)
    torch.cuda.set_device(device)
    w_router, bias = workloads.make_router(wl, device)
    for T in wl.T:
        x = workloads.make_x(wl, T, device=device)
        ids = torch.empty((T, wl.top_k), dtype=torch.int32, device=device)
        w = torch.empty((T, wl.top_k), dtype=torch.float32, device=device)
        for _ in range(args.warmup):
            ed.moe_route(x, w_router, bias, wl.top_k, ids=ids, weights=w)
        torch.cuda.synchronize()
        ed.ep_check_status()
        es, ee = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        es.record()
        for _ in range(args.steps):
            ed.moe_route(x, w_router, bias, wl.top_k, ids=ids, weights=w)
        ee.record()
        torch.cuda.synchronize()
        ed.ep_check_status()
        print(f"router {wl.name} T={T}: {es.elapsed_time(ee) * 1e3 / max(args.steps, 1):.2f} us "
              f"per call (back to back, weights L2-resident)", flush=True)


def main():
    args = parse_args()
    wl = workloads.WORKLOADS[args.config]
    if args.experts:
        import dataclasses
        wl = dataclasses.replace(wl, E=args.experts, bands=(min(wl.bands[0], args.experts),),
                                 description=wl.description + f" (E reduced to {args.experts})")
    if args.impl == "reference":
        run_reference(args, wl)
    elif args.router_only:
        run_router_only(args, wl)
    elif args.ep:
        run_ep(args, wl)
    else:
        run_ours(args, wl)


if __name__ == "__main__":
    main()
