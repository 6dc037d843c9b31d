#!/usr/bin/env python3
"""Benchmark of the sparse latent-MoE decode layer step on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

A step is one decode layer step (router, top-k, latent down-projection, routed MXFP4 experts,
combine, up-projection, shared expert) for one batch of tokens.  A timed region replays a
CUDA graph of exactly K steps that cycles through `--layers` layers of distinct seeded weights
(32 by default, ~99 GB), so every step streams its weights from HBM: the per-step working set
(>= 148 MB) exceeds the 126 MB L2 and the same layer returns only after 31 others.  The reported
time is the median of `--reps` (5) such regions, each bracketed by a synchronise (and a barrier
under torchrun); every layer's device error word is read after them, so a step that gave up on
a bounded wait fails the run instead of being timed.  The headline is `--workload` (full_b1);
`per_config` repeats the measurement for the metric's other batches (B = 2, 16, 64) and for a
speculative-decoding batch (B = 256 = 32 sequences x 8 tokens), each over
32 layers of its own weights.  Rank 0 prints one JSON line.  Under torchrun every rank runs an
independent replica (the step does not shard; no collective touches the data path); value =
all ranks' steps / max time.

--impl reference times the CPU oracle (the plain fp64 C implementation) on this host's cores
for a bounded sample of the same workload, on the same metric and configuration: the reference
arm that this bench's throughput is compared against.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "MoE layer-steps/s & µs/step at B=1..64; achieved HBM GB/s vs B200 peak"
PER_CONFIG = ("full_b1", "full_b2", "full_b16", "full_b64_skewed", "full_b256")  # the metric's batches, and a speculative-decoding batch
UNIT = "layer-steps/s"


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=200)
    p.add_argument("--warmup", type=int, default=10)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--workload", default="full_b1", choices=sorted(synth.WORKLOADS))
    p.add_argument("--layers", type=int, default=0, help="distinct layers cycled through (default 32)")
    p.add_argument("--schedule", choices=["fused", "multi", "stream"], default="fused",
                   help="one persistent kernel per step (default) or eight stream-ordered kernels")
    p.add_argument("--reps", type=int, default=5, help="timed replays of the K-step graph (median)")
    p.add_argument("--no-per-config", action="store_true", help="skip the B=2/16/64 entries of per_config")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--fp4-stream", action="store_true",
                   help="build and run bench_fp4_stream.cu (streaming rate of the MXFP4 tile path, piece by piece)")
    p.add_argument("--ncu", action="store_true",
                   help="profiling case for ncu: --steps eager steps over --layers resident layers, no timing")
    p.add_argument("--cpu-seconds", type=float, default=12.0, help="CPU oracle sample length")
    p.add_argument("--ep-emulate", type=int, default=0, metavar="G",
                   help="time the expert-parallel step's ranks (G shards of every layer) one at a time on "
                        "this GPU, and the exchange kernels; prints its own JSON line")
    return p.parse_args()


def dist_env():
    return int(os.environ.get("RANK", "0")), int(os.environ.get("LOCAL_RANK", "0")), int(os.environ.get("WORLD_SIZE", "1"))


def max_over_ranks(v: float, dist, device) -> float:
    """The largest of every rank's v (v itself without a process group): a multi-rank time is the
    slowest rank's."""
    if dist is None:
        return v
    import torch
    t = torch.tensor([v], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def replica_throughput(world: int, steps: int, max_ms: float) -> float:
    """Whole-job layer-steps/s of `world` independent replicas that each ran `steps` steps, the
    slowest in max_ms milliseconds."""
    return world * steps / (max_ms / 1e3)


def log(*a):
    print(*a, file=sys.stderr, flush=True)


# ---------------------------------------------------------------------------------------------
# byte accounting (algorithmic bytes: every weight byte the step must read once, plus tokens)

def kernel_bytes(d: synth.Dims, unique_experts: float, B: int) -> dict:
    H, L, E, I, Is = d.hidden, d.latent, d.n_experts, d.expert_inter, d.shared_inter
    fp4 = lambda n, k: n * k // 2 + n * k // 32
    return {
        "router_dn": 2 * E * H + 2 * L * H + 2 * B * H,
        "topk": 4 * B * E,
        "expert_gate_up": unique_experts * 2 * fp4(I, L),
        "expert_down": unique_experts * fp4(L, I),
        "combine": 4 * B * d.top_k * L,
        "up": 2 * H * L + 2 * B * H,
        "shared_gate_up": 2 * fp4(Is, H),
        "shared_down": fp4(H, Is),
        "fused_step_splitk": step_bytes(d, unique_experts, B),
        "fused_step_small": step_bytes(d, unique_experts, B),
        "fused_step_stream": step_bytes(d, unique_experts, B),
    }


def step_bytes(d: synth.Dims, unique_experts: float, B: int) -> float:
    """Algorithmic HBM bytes of one step: fixed weights + touched experts + tokens in and out."""
    return d.fixed_bytes() + unique_experts * d.expert_bytes() + 2 * 2 * B * d.hidden


# ---------------------------------------------------------------------------------------------
# clocks during the timed region

class ClockSampler:
    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
             "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
             "clocks_event_reasons.sw_power_cap")
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.index}", f"--query-gpu={q}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        rows = []
        try:
            for line in open(self.path):
                f = [x.strip() for x in line.split(",")]
                if len(f) >= 9:
                    rows.append(f)
        except OSError:
            pass
        finally:
            try:
                os.unlink(self.path)
            except OSError:
                pass
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["clock sampling unavailable"]}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        smax = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        reasons = set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            for n, v in zip(names, r[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        busy = [s for s in sm if smax and s > 0.5 * max(smax)] or sm
        return {"sm_mhz": statistics.median(busy) if busy else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(rows)}


# the files that decide what a kernel reads and writes: its code, and moedec_api.cu, which sizes
# its work items (the plan of K splits)
KERNEL_SOURCES = {
    "fused_step_stream": ["moedec_stream.cu", "moedec_items.cuh", "moedec_tiles.cuh", "moedec_device.cuh",
                          "moedec_router.cuh", "moedec_internal.h", "moedec_api.cu"],
    "fused_step_small": ["moedec_fused_small.cu", "moedec_ring.cuh", "moedec_experts.cuh", "moedec_items.cuh",
                         "moedec_tiles.cuh", "moedec_device.cuh", "moedec_router.cuh", "moedec_internal.h",
                         "moedec_api.cu"],
    "fused_step_splitk": ["moedec_fused.cu", "moedec_ring.cuh", "moedec_experts.cuh", "moedec_items.cuh",
                          "moedec_tiles.cuh", "moedec_device.cuh", "moedec_router.cuh", "moedec_internal.h",
                          "moedec_api.cu"],
}


def profiled_traffic(kernel: str, workload: str):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on this workload from
    the kernel's current sources (else None: the counters no longer describe the kernel)."""
    import hashlib
    try:
        rec = json.load(open(os.path.join(ROOT, "profiles", "traffic.json")))[kernel]
        h = hashlib.sha256()
        for f in KERNEL_SOURCES[kernel]:
            h.update(open(os.path.join(ROOT, "moe_decode_layer_moedec_b200", "csrc", f), "rb").read())
        if rec["workload"] == workload and h.hexdigest()[:16] == rec["source_sha256_16"]:
            return float(rec["bytes_per_launch"])
    except Exception:
        pass
    return None


def measured_peak_hbm():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        v = json.load(open(p))["hbm_gbs"]
        return float(v), "measured (MEASURED_PEAKS.json hbm_gbs, copy)"
    except Exception:
        return 6650.0, "fallback 6.65 TB/s (no MEASURED_PEAKS.json)"


# ---------------------------------------------------------------------------------------------
# CPU oracle timing (the baseline; also the reference arm)

def cpu_oracle_rate(w: synth.Workload, seconds: float):
    import oracle
    W = synth.layer_weights(w, 0)
    x = synth.tokens(w)
    n = 0
    t0 = time.perf_counter()
    while True:
        oracle.step(w.dims, W, x)
        n += 1
        if time.perf_counter() - t0 >= seconds:
            break
    dt = time.perf_counter() - t0
    return {"value": n / dt, "unit": UNIT, "cores": oracle.threads(), "kind": "oracle",
            "sample": f"{n} oracle steps of {w.name} layer 0 (B={w.batch}, all {w.batch} tokens), {dt:.1f} s"}


def workload_config(w: synth.Workload, n_layers: int, schedule: str, world: int) -> dict:
    """The `config` object of both arms' JSON lines (same workload, same keys)."""
    d = w.dims
    return {"workload": w.name, "batch": w.batch, "hidden": d.hidden, "latent": d.latent, "experts": d.n_experts,
            "top_k": d.top_k, "expert_inter": d.expert_inter, "shared_inter": d.shared_inter,
            "layers_cycled": n_layers,
            "l2": "inputs larger than L2: each step streams one of %d distinct layers (>= 148 MB)" % n_layers,
            "arith": "MXFP4/bf16 weights; tensor-core MMA operands fp16 (MXFP4 parts) and bf16 (dense parts), tokens "
                     "as hi/lo operand pairs at B <= 4 and for W_up, single fp16 with a per-token power-of-two "
                     "scale otherwise; fp32 accumulation; router exact products summed in fp64",
            "parallelism": "replicas" if world > 1 else "single GPU", "schedule": schedule}


def default_layers(w: synth.Workload, requested: int) -> int:
    return requested or (32 if w.dims is synth.FULL else 4)


def run_reference(args):
    rank, _, world = dist_env()
    if rank != 0:
        return
    w = synth.WORKLOADS[args.workload]
    import oracle
    W = synth.layer_weights(w, 0)
    x = synth.tokens(w)
    t0 = time.perf_counter()
    for _ in range(max(args.warmup, 1)):
        oracle.step(w.dims, W, x)
    est = (time.perf_counter() - t0) / max(args.warmup, 1)
    # bounded sample: at most ~150 s of timed oracle steps whatever K is
    n = max(1, min(args.steps, int(150.0 / max(est, 1e-6))))
    t0 = time.perf_counter()
    for _ in range(n):
        oracle.step(w.dims, W, x)
    dt = time.perf_counter() - t0
    v = n / dt
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": UNIT, "n_gpus": args.gpus, "steps": n,
            "warmup": args.warmup, "ms_per_step": 1e3 * dt / n, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_config(w, default_layers(w, args.layers), args.schedule, world),
            "cpu_baseline": {"value": v, "unit": UNIT, "cores": oracle.threads(), "kind": "oracle",
                             "sample": f"{n} timed oracle steps (of {args.steps} requested, capped at ~150 s) of "
                                       f"{w.name} layer 0 after {args.warmup} warm-up"},
            "e2e": {"value": v, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------------------------
# our arm

def load_layers(w, n_layers, schedule, local_rank, rank):
    """n_layers handles of distinct seeded layers of workload w, weights resident in HBM."""
    import torch
    from moe_decode_layer_moedec_b200 import FLAG_MULTI_KERNEL, FLAG_SKIP_SCALE_CHECK, FLAG_STREAM, LayerDims, \
        MoeDecodeLayer
    d = w.dims
    dims = LayerDims(d.hidden, d.latent, d.n_experts, d.top_k, d.expert_inter, d.shared_inter, 1)
    t0 = time.time()
    layers, dev_weights = [], []
    for l in range(n_layers):
        W = synth.layer_weights(w, l)
        Wd = {}
        for k, v in W.items():
            t = torch.from_numpy(v.view(np.int16) if v.dtype == np.uint16 else v)
            Wd[k] = t.to(f"cuda:{local_rank}", non_blocking=False)
        del W
        flags = 0 if l == 0 else FLAG_SKIP_SCALE_CHECK  # layer 0 runs the create-time scale scan
        if schedule == "multi":
            flags |= FLAG_MULTI_KERNEL
        if schedule == "stream":
            flags |= FLAG_STREAM
        layers.append(MoeDecodeLayer(dims, Wd, max_batch=w.batch, flags=flags))
        dev_weights.append(Wd)
        if rank == 0 and (l % 8 == 7 or l == n_layers - 1):
            log(f"[bench] {w.name}: {l + 1}/{n_layers} layers resident ({time.time() - t0:.0f} s)")
    return layers, dev_weights


def check_device_errors(layers, B, stream):
    """Every layer's sticky device error word: a bounded wait that ran out, or a bad bucket, makes
    the CTAs leave early and would otherwise be timed as a fast step.  Raises on any."""
    for L_ in layers:
        L_.routing(B, stream=stream)


class Timed:
    """Graph replays of `steps` steps over the resident layers, timed with CUDA events on the
    launching stream; median over `reps` replays, max over ranks."""

    def __init__(self, layers, x, out, stream, steps, warmup, dist, device):
        import torch
        self.torch, self.layers, self.x, self.out, self.stream = torch, layers, x, out, stream
        self.steps, self.warmup, self.dist, self.device = steps, warmup, dist, device
        n = len(layers)
        B = x.shape[0]
        with torch.cuda.stream(stream):
            for i in range(max(warmup, 3)):   # eager warm-up (module load, caches)
                layers[i % n].step(x, out=out, stream=stream)
        torch.cuda.synchronize()
        check_device_errors(layers, B, stream)
        self.g_warm = self.capture(max(warmup, 1), 0)
        self.g_main = self.capture(steps, warmup)

    def capture(self, n_steps, first):
        torch = self.torch
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=self.stream, capture_error_mode="thread_local"):
            for i in range(n_steps):
                self.layers[(first + i) % len(self.layers)].step(self.x, out=self.out, stream=self.stream)
        return g

    def replay_ms(self, g):
        torch = self.torch
        ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        if self.dist:
            self.dist.barrier()
        torch.cuda.synchronize()
        ev0.record(self.stream)
        with torch.cuda.stream(self.stream):
            g.replay()
        ev1.record(self.stream)
        torch.cuda.synchronize()
        if self.dist:
            self.dist.barrier()
        return ev0.elapsed_time(ev1)

    def run(self, reps, local_rank):
        """Median ms of `reps` timed replays (each exactly `steps` steps), with untimed replays of
        the same graph for ~0.5 s on each side so that the clock samples see the step running."""
        torch = self.torch
        self.g_warm.replay()
        torch.cuda.synchronize()
        t_probe = time.perf_counter()
        with torch.cuda.stream(self.stream):
            self.g_main.replay()
        torch.cuda.synchronize()
        pad = max(1, min(200, int(0.5 / max(time.perf_counter() - t_probe, 1e-4))))
        with ClockSampler(local_rank) as clk:
            with torch.cuda.stream(self.stream):
                for _ in range(pad):
                    self.g_main.replay()
            times = [self.replay_ms(self.g_main) for _ in range(reps)]
            with torch.cuda.stream(self.stream):
                for _ in range(pad):
                    self.g_main.replay()
            torch.cuda.synchronize()
        check_device_errors(self.layers, self.x.shape[0], self.stream)
        ms = max_over_ranks(statistics.median(times), self.dist, self.device)
        return ms, times, clk.summary()

    def run_hinted(self, reps, local_rank):
        """The same measurement with the cross-layer prefetch hint set: layer l's steps prefetch the
        router of layer l + 1 (the one the graph steps next).  The hints are cleared afterwards."""
        n = len(self.layers)
        for l, L_ in enumerate(self.layers):
            L_.set_next(self.layers[(l + 1) % n])
        self.g_warm, self.g_main = self.capture(max(self.warmup, 1), 0), self.capture(self.steps, self.warmup)
        try:
            return self.run(reps, local_rank)
        finally:
            for L_ in self.layers:
                L_.set_next(None)
            self.g_warm, self.g_main = self.capture(max(self.warmup, 1), 0), self.capture(self.steps, self.warmup)

    def close(self):
        del self.g_main, self.g_warm
        self.layers = self.x = self.out = None


def unique_experts(layers, x, out, stream, B):
    """Mean number of distinct experts a step touches (routing of every layer, untimed)."""
    import torch
    uniq = []
    with torch.cuda.stream(stream):
        for L_ in layers:
            L_.step(x, out=out, stream=stream)
            idx, _ = L_.routing(B, stream=stream)
            uniq.append(len(np.unique(idx.cpu().numpy())))
    torch.cuda.synchronize()
    return float(np.mean(uniq))


def config_entry(w, ms, times, clocks, steps, world, unique_mean, peak, hinted=None):
    """One per_config record: time per step, throughput, algorithmic bytes and their HBM fraction;
    `hinted` = (ms, times, clocks) of the same steps with the cross-layer prefetch hint."""
    ms_per_step = ms / steps
    sb = step_bytes(w.dims, unique_mean, w.batch)
    r = {"workload": w.name, "batch": w.batch, "us_per_step": 1e3 * ms_per_step,
         "layer_steps_per_s": replica_throughput(world, steps, ms), "unique_experts_per_step": unique_mean,
         "bytes_per_step": sb, "hbm_gbs": sb / (ms_per_step / 1e3) / 1e9,
         "hbm_frac": sb / (ms_per_step / 1e3) / 1e9 / peak,
         "replay_ms": [round(t, 4) for t in times], "clocks": clocks}
    if hinted:
        hms = hinted[0] / steps
        r["next_layer_hint"] = {"us_per_step": 1e3 * hms, "layer_steps_per_s": replica_throughput(world, steps, hinted[0]),
                                "hbm_frac": sb / (hms / 1e3) / 1e9 / peak, "replay_ms": [round(t, 4) for t in hinted[1]],
                                "clocks": hinted[2]}
    return r


def profile_case(args, w, n_layers, local_rank, rank):
    """The small case an ncu capture runs: step i on layer i mod n_layers, eagerly, then every
    layer's device error word is read (the run exits non-zero on a device-side error)."""
    import torch
    layers, dev_weights = load_layers(w, n_layers, args.schedule, local_rank, rank)
    x = torch.from_numpy(synth.tokens(w).view(np.int16)).to(f"cuda:{local_rank}")
    out = torch.empty_like(x)
    for i in range(args.steps):
        layers[i % n_layers].step(x, out=out)
    torch.cuda.synchronize()
    for L_ in layers:
        L_.routing(w.batch)
        L_.close()
    log(f"[bench] profiling case done: {args.steps} steps of {w.name} over {n_layers} layers")


def fp4_stream():
    """Compile bench_fp4_stream.cu for sm_100a (under _build/) and run it; prints its table."""
    exe = os.path.join(ROOT, "_build", "bench_fp4_stream")
    os.makedirs(os.path.dirname(exe), exist_ok=True)
    subprocess.check_call(["nvcc", "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-std=c++17",
                           "--expt-relaxed-constexpr", "-I", ROOT, "-I", os.path.join(ROOT, "include"),
                           os.path.join(ROOT, "bench_fp4_stream.cu"), "-o", exe])
    subprocess.check_call([exe])


def ep_emulated(args, w, n_layers, local_rank):
    """Each rank of a G-way expert-parallel split of the workload's layers, timed alone on this GPU
    (graph replays of K partial steps over the resident layers, CUDA events, median of the reps),
    and the exchange (publish + combine over G partials, with flags already set, so no waiting).
    On a node of G GPUs the ranks run at once; the exchange there reads peer memory over NVLink,
    which this one-GPU measurement does not include."""
    import torch
    from moe_decode_layer_moedec_b200 import FLAG_SKIP_SCALE_CHECK, LayerDims, ep
    d, B, G = w.dims, w.batch, args.ep_emulate
    dims = LayerDims(d.hidden, d.latent, d.n_experts, d.top_k, d.expert_inter, d.shared_inter, 1)
    full, dev_weights = load_layers(w, n_layers, "fused", local_rank, 0)
    for L_ in full:
        L_.close()
    groups = [ep.EmulatedExpertParallel(dims, Wd, G, max_batch=B, flags=FLAG_SKIP_SCALE_CHECK) for Wd in dev_weights]
    x = torch.from_numpy(synth.tokens(w).view(np.int16)).to(f"cuda:{local_rank}")
    stream = torch.cuda.Stream()
    with torch.cuda.stream(stream):
        for g in groups:
            g.step(x, stream=stream)
    torch.cuda.synchronize()
    for g in groups:
        check_device_errors(g.layers, B, stream)

    def timed(fn):
        gr = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gr, stream=stream, capture_error_mode="thread_local"):
            for i in range(args.steps):
                fn(i)
        for _ in range(max(args.warmup, 3)):
            with torch.cuda.stream(stream):
                gr.replay()
        ts = []
        for _ in range(args.reps):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            torch.cuda.synchronize()
            e0.record(stream)
            with torch.cuda.stream(stream):
                gr.replay()
            e1.record(stream)
            torch.cuda.synchronize()
            ts.append(e0.elapsed_time(e1))
        del gr
        return 1e3 * statistics.median(ts) / args.steps

    n = len(groups)
    per_rank = []
    for r in range(G):
        per_rank.append(timed(lambda i, r=r: groups[i % n].layers[r].step_partial(x, groups[i % n].parts[r, 0],
                                                                                   stream=stream)))
    out = torch.empty((B, d.hidden), dtype=torch.int16, device=x.device)

    def exchange(i):
        g = groups[i % n]
        e = g.clock.epoch  # already published by every rank: the combine does not wait
        g.layers[0].ep_publish([g.flag_ptr(q, 0) for q in range(G)], e, stream=stream)
        g.layers[0].ep_combine([g.parts[q, e % 2].data_ptr() for q in range(G)], g.flag_ptr(0, 0), e, B, out,
                               stream=stream)
    xch = timed(exchange)
    for g in groups:
        check_device_errors(g.layers, B, stream)
        g.close()
    line = {"metric": "ep_emulated", "workload": w.name, "world": G, "batch": B, "layers": n,
            "steps": args.steps, "reps": args.reps,
            "per_rank_partial_us": [round(v, 2) for v in per_rank],
            "exchange_us": round(xch, 2), "slowest_rank_plus_exchange_us": round(max(per_rank) + xch, 2),
            "note": "ranks timed one at a time on one GPU; the exchange reads local memory, so NVLink "
                    "transfer time is not included"}
    print(json.dumps(line), flush=True)


def main():
    args = parse()
    if args.fp4_stream:
        return fp4_stream()
    if args.impl == "reference":
        return run_reference(args)
    rank, local_rank, world = dist_env()
    import torch
    torch.cuda.set_device(local_rank)
    device = f"cuda:{local_rank}"
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=600),
                                device_id=torch.device("cuda", local_rank))

    w = synth.WORKLOADS[args.workload]
    d = w.dims
    B = w.batch
    n_layers = default_layers(w, args.layers)
    if args.ncu:
        return profile_case(args, w, n_layers, local_rank, rank)
    if args.ep_emulate:
        if world > 1:
            raise SystemExit("--ep-emulate runs on one GPU")
        return ep_emulated(args, w, n_layers, local_rank)
    peak, peak_src = measured_peak_hbm()
    layers, dev_weights = load_layers(w, n_layers, args.schedule, local_rank, rank)
    x_host = torch.from_numpy(synth.tokens(w).view(np.int16)).pin_memory()
    x = x_host.to(device)
    out = torch.empty_like(x)
    stream = torch.cuda.Stream()
    unique_mean = unique_experts(layers, x, out, stream, B)

    tm = Timed(layers, x, out, stream, args.steps, args.warmup, dist, device)
    ms, times, clocks = tm.run(args.reps, local_rank)
    hinted = tm.run_hinted(args.reps, local_rank)
    ms_per_step = ms / args.steps
    value = replica_throughput(world, args.steps, ms)
    kps = layers[0].kernels_per_step(B)

    # per-kernel durations: a replay of the same K steps with an event pair around every kernel on
    # the stream it runs on (main or side stream).  With one kernel per step the dominant kernel's
    # time per launch is the timed replay's time per step; the bracketed pass (which slows the
    # kernels it brackets) only splits the time of a multi-kernel step.
    for L_ in layers:
        L_.profile(True)
    g_prof = tm.capture(args.steps, args.warmup)
    for L_ in layers:
        L_.profile(False)
    tm.g_warm.replay()
    ms_prof = tm.replay_ms(g_prof)
    check_device_errors(layers, B, stream)
    per_kernel = {}
    for L_ in layers:
        for name, (kms, n) in L_.profile_read().items():
            a, b = per_kernel.get(name, (0.0, 0))
            per_kernel[name] = (a + kms, b + n)
    del g_prof
    kb = kernel_bytes(d, unique_mean, B)
    if not any(v[0] > 0 for v in per_kernel.values()):
        raise RuntimeError(f"per-kernel profile is empty: {per_kernel}")
    dom = max(per_kernel, key=lambda k: per_kernel[k][0])
    dom_ms, dom_n = per_kernel[dom]
    dom_avg_s = ms_per_step / 1e3 if kps == 1 else dom_ms / 1e3 / max(dom_n, 1)
    achieved = kb[dom] / dom_avg_s / 1e9
    kernels_table = {k: {"avg_us": 1e3 * v[0] / max(v[1], 1), "launches": v[1],
                         "share": v[0] / max(sum(x_[0] for x_ in per_kernel.values()), 1e-12),
                         "gbs": kb[k] / (v[0] / 1e3 / max(v[1], 1)) / 1e9 if v[0] > 0 else None}
                     for k, v in per_kernel.items() if v[1] > 0}

    # end to end through the public API: pinned host tokens in, step, result back to pinned host
    out_host = torch.empty_like(x_host).pin_memory()
    with torch.cuda.stream(stream):
        for i in range(3):
            x.copy_(x_host, non_blocking=True)
            layers[i % n_layers].step(x, out=out, stream=stream)
            out_host.copy_(out, non_blocking=True)
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    with torch.cuda.stream(stream):
        for i in range(args.steps):
            x.copy_(x_host, non_blocking=True)
            layers[i % n_layers].step(x, out=out, stream=stream)
            out_host.copy_(out, non_blocking=True)
    e1.record(stream)
    torch.cuda.synchronize()
    check_device_errors(layers, B, stream)
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), dist, device)
    e2e_value = replica_throughput(world, args.steps, e2e_ms)
    per_config = {w.name: config_entry(w, ms, times, clocks, args.steps, world, unique_mean, peak, hinted)}
    tm.close()
    for L_ in layers:
        L_.close()
    del layers, dev_weights
    torch.cuda.empty_cache()

    # the metric's other batches (B = 2, 16, 64), each over its own resident layers, same K and W
    if not args.no_per_config:
        for name in PER_CONFIG:
            if name == w.name:
                continue
            wc = synth.WORKLOADS[name]
            lc, wd = load_layers(wc, default_layers(wc, args.layers), args.schedule, local_rank, rank)
            xc = torch.from_numpy(synth.tokens(wc).view(np.int16)).to(device)
            oc = torch.empty_like(xc)
            uc = unique_experts(lc, xc, oc, stream, wc.batch)
            tc = Timed(lc, xc, oc, stream, args.steps, args.warmup, dist, device)
            mc, tsc, cc = tc.run(args.reps, local_rank)
            hc = tc.run_hinted(args.reps, local_rank)
            per_config[name] = config_entry(wc, mc, tsc, cc, args.steps, world, uc, peak, hc)
            tc.close()
            for L_ in lc:
                L_.close()
            del lc, wd, xc, oc
            torch.cuda.empty_cache()

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_oracle_rate(w, args.cpu_seconds)

    sb = step_bytes(d, unique_mean, B)
    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f16", "data": "synthetic",
            "config": workload_config(w, n_layers, args.schedule, world),
            "us_per_step": 1e3 * ms_per_step, "unique_experts_per_step": unique_mean,
            "timed_replays": args.reps, "replay_ms": [round(t, 4) for t in times],
            "step_hbm": {"bytes_per_step": sb, "gbs": sb / (ms_per_step / 1e3) / 1e9,
                         "frac": sb / (ms_per_step / 1e3) / 1e9 / peak, "peak_gbs": peak, "peak": peak_src},
            "clocks": clocks,
            "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": int(x_host.numel() * 2),
                    "d2h_bytes_per_step": int(out_host.numel() * 2)},
            "gpu_launches": kps * args.steps,
            "roofline": {"bound": "hbm", "kernel": dom, "achieved": achieved, "peak": peak, "unit": "GB/s",
                         "frac": achieved / peak, "traffic": profiled_traffic(dom, w.name), "bytes_per_launch": kb[dom],
                         "avg_launch_us": dom_avg_s * 1e6, "peak_source": peak_src,
                         "time_source": "timed replay (one kernel per step)" if kps == 1 else
                                        "per-kernel CUDA events of a bracketed replay"},
            "kernels": kernels_table,
            "profiled_pass_ms_per_step": ms_prof / args.steps,
            "per_config": per_config,
            "cpu_baseline": cpu,
        }
        print(json.dumps(line), flush=True)
    if dist:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
