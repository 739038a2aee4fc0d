"""Benchmark of the co-activation / deduplicated-dispatch hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                    [--placement correlated|uniform|capacity|capped] [--no-shuffle]
                    [--balanced-shuffle] [--prereduce] [--replicas N]
                    [--coact-method auto|histogram|tensor] [--no-overlap] [--no-graph]
                    [--out-dtype f32|bf16] [--ep] [--ep-emulate W] [--impl reference]

A step is one pass of the whole path over one batch: co-activation counts,
Ochiai and transitions for every layer, then per layer the dispatch plan, the
row permute, identity experts, the weighted combine and the shuffle targets
for the next layer.  Plans, shuffle targets and statistics run on a second
stream beside the row traffic (--no-overlap: in line); the timed steps are
replayed from one CUDA graph (--no-graph: eager launches).  The default
workload is large EP64 (T=131072, E=256, k=8, G=64 in 8 nodes, d=7168 bf16,
4 layers), the largest workload with hidden states; its inputs (x = 1.88 GB)
exceed the 126 MB L2, so no flush is needed between steps.  Workloads whose
inputs fit in L2 (one node, tiny) time each step on its own after a write of
twice the L2 size.  With N GPUs each rank runs its own batch (seed + rank): weak
scaling, no collective on the data path.

value = dispatch+combine algorithmic bytes of the step / device time of the
whole step (max over ranks), in GB/s.  Algorithmic bytes are the minimum HBM
traffic: permute reads each token row once and writes R rows; combine reads
the U distinct rows and writes T output rows (U = R for identity experts).
"""
from __future__ import annotations

import argparse
import json
import os
import platform
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "dedup dispatch+combine GB/s (frac of HBM peak); co-activation tokens/s"
FALLBACK_HBM_GBS = 6650.0
SM_MAX_MHZ = 1965.0            # B200 clocks.max.sm


def measured_peak(key):
    """A positive number under `key` in MEASURED_PEAKS.json (written per pool:
    hbm_gbs, bf16_tflops, bf16_tflops_sustained; a value may also sit in a
    {"value": ...} object), else None: no file, unreadable, or no such key."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if not os.path.exists(p):
        return None
    try:
        with open(p) as f:
            v = json.load(f).get(key)
        if isinstance(v, dict):
            v = v.get("value")
        v = float(v)
    except (OSError, ValueError, TypeError, AttributeError):
        return None
    return v if v > 0 else None


def peaks():
    v = measured_peak("hbm_gbs")
    return (v, "measured") if v is not None else (FALLBACK_HBM_GBS, "fallback")


def tensor_peak():
    """Dense bf16 TFLOP/s for a kernel timed alone: the measured burst figure."""
    v = measured_peak("bf16_tflops")
    return (v, "measured") if v is not None else (1590.0, "fallback")


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default="large_ep64")
    ap.add_argument("--placement", default=None, choices=["correlated", "uniform", "capacity", "capped"],
                    help="default: uniform for the tiny workload (its stated placement), correlated otherwise; "
                         "capped: correlated with every rank's load within 1.1 x the average")
    ap.add_argument("--no-shuffle", action="store_true")
    ap.add_argument("--balanced-shuffle", action="store_true",
                    help="cap every rank's shard at T/G tokens (capacity-balanced shuffle targets)")
    ap.add_argument("--out-dtype", default="f32", choices=["f32", "bf16"])
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-graph", action="store_true", help="time eager launches instead of one CUDA graph")
    ap.add_argument("--no-overlap", action="store_true",
                    help="run plans, shuffle targets and statistics in line instead of on a second stream "
                         "(the same as --schedule inline)")
    ap.add_argument("--row-chunks", type=int, default=1, metavar="C",
                    help="pipeline each layer's permute and combine over C token chunks (the combine of a chunk "
                         "beside the permute of the next); the per-kernel times then overlap")
    ap.add_argument("--schedule", default=None, choices=["overlap", "forward", "inline"],
                    help="overlap (default): all control work ahead on a second stream; forward: the order of a "
                         "forward pass, each layer's plan in line before its rows, shuffle targets and statistics "
                         "beside them; inline: everything in line")
    ap.add_argument("--replicas", type=int, default=0, metavar="EXTRA",
                    help="replicate experts (EXTRA more per rank) and assign tasks to the fewest remote nodes")
    ap.add_argument("--replica-eps", type=float, default=None, metavar="EPS",
                    help="with --replicas: cap every rank's tasks at (1 + EPS) T k / G in the assignment")
    ap.add_argument("--prereduce", action="store_true",
                    help="receiver-side pre-reduced combine with stand-in experts (gates dispatched with rows)")
    ap.add_argument("--seed", type=int, default=None,
                    help="seed of the evaluation batch (calibration: seed + 1); the cluster layout stays the workload's")
    ap.add_argument("--coact-method", default="auto", choices=["auto", "histogram", "tensor"],
                    help="how the co-activation statistics count: per call, shared-memory histograms, tensor cores")
    ap.add_argument("--ep", action="store_true",
                    help="expert parallelism over the job's GPUs: the G ranks spread over the N processes "
                         "(rows stored to and loaded from the other GPUs' buffers)")
    ap.add_argument("--ep-emulate", type=int, default=0, metavar="W",
                    help="also time the several-device path with W virtual devices on this GPU")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-sweep", action="store_true")
    ap.add_argument("--sweep-only", action="store_true", help="only the co-activation statistics sweep")
    ap.add_argument("--cpu-seconds", type=float, default=15.0, help="target oracle time for the CPU baseline")
    return ap.parse_args()


def rank_seed(base, rank):
    """Each rank draws its own batch (weak scaling); the cluster layout (the
    stand-in for the trained router) is the workload's, shared by all ranks."""
    return base + 1000 * rank


def reduce_max(x, pg, device):
    """Max over ranks of a per-rank time (the only collective in the bench)."""
    if pg is None:
        return x
    import torch
    t = torch.tensor([float(x)], device=device, dtype=torch.float64)
    pg.all_reduce(t, op=pg.ReduceOp.MAX)
    return float(t.item())


def weak_value(world, bytes_per_rank, ms_step):
    """Whole-job GB/s: all ranks' bytes over the slowest rank's step time."""
    return world * bytes_per_rank / (ms_step * 1e-3) / 1e9


def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


# ------------------------------------------------------------------ clocks

class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons while running."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, uuid=None, period_ms=100):
        self.uuid = uuid
        self.period = period_ms
        self.proc = None

    def __enter__(self):
        self.tmp = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        cmd = ["nvidia-smi", "--query-gpu=" + self.FIELDS, "--format=csv,noheader,nounits", "-lms", str(self.period)]
        if self.uuid:
            cmd += ["-i", self.uuid]
        try:
            self.proc = subprocess.Popen(cmd, stdout=self.tmp, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            time.sleep(0.15)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
        self.tmp.flush()

    def summary(self):
        try:
            with open(self.tmp.name) as f:
                rows = [r.strip().split(", ") for r in f if r.strip()]
        finally:
            os.unlink(self.tmp.name)
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            if len(r) < 9:
                continue
            try:
                sm.append(float(r[1]))
                mx.append(float(r[2]))
            except ValueError:
                continue
            for n, v in zip(names, r[5:9]):
                if v.strip().lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


# ------------------------------------------------------------------ reference arm / CPU baseline

def oracle_pass(w, ids, ids_cal, gates, x, placement, shuffle, balanced=False):
    """One pass of the path through the CPU oracle on a token sample.
    Returns (seconds, algorithmic dispatch+combine bytes)."""
    import oracle as orc
    from synth import bf16_bits_to_f32
    L, T, k = ids.shape
    t0 = time.perf_counter()
    orc.coact(ids, w.E)
    cal = orc.coact(ids_cal, w.E)
    if placement == "correlated":
        e2r = [orc.place_correlated(cal["coact"][l], w.G, w.rpn) for l in range(L)]
    elif placement == "capacity":
        e2r = [orc.place_capacity(np.diag(cal["coact"][l]).astype(np.float64), w.G)[0] for l in range(L)]
    elif placement == "capped":
        e2r = [orc.place_correlated_capped(cal["coact"][l], w.G, w.rpn, 0.1) for l in range(L)]
    else:
        e2r = [orc.place_uniform(w.E, w.G) for _ in range(L)]
    rs = [orc.rank_score(cal["trans"][l], e2r[l + 1], w.G) for l in range(L - 1)] if shuffle else []
    src = None
    rowB = w.d * w.elem_bytes
    nbytes = 0
    for l in range(L):
        p = orc.plan(ids[l], w.E, w.G, w.rpn, e2r[l], src_rank=src)
        send = orc.permute(x, p["row_token"])
        Y = bf16_bits_to_f32(send) if w.dtype == "bf16" else send
        orc.combine(Y, p["row_of"], gates[l], y_is_bf16=False)
        R = p["R"]
        nbytes += T * rowB + R * rowB + 4 * T * k + R * rowB + T * w.d * 4 + 8 * T * k
        if shuffle and l + 1 < L:
            src = orc.shuffle_balanced(ids[l], w.E, w.G, rs[l], T // w.G) if balanced else \
                orc.shuffle_targets(ids[l], w.E, w.G, rs[l])
    return time.perf_counter() - t0, nbytes


def cpu_sample(w, T_s, seed):
    from synth import make_routing, make_gates, make_hidden
    ids = make_routing(w, seed=seed, T=T_s)
    cal = make_routing(w, seed=seed + 1, T=T_s)
    gates = make_gates(w, seed=seed, T=T_s)
    x = make_hidden(w, seed=seed, T=T_s)
    return ids, cal, gates, x


def sized_sample(w, target_s, shuffle, balanced=False, base_seed=None):
    """Choose a token count (a multiple of G) whose oracle pass takes about target_s."""
    base_seed = w.seed if base_seed is None else base_seed
    T_probe = max(w.G, (1024 // w.G) * w.G)
    ids, cal, gates, x = cpu_sample(w, T_probe, base_seed)
    sec, _ = oracle_pass(w, ids, cal, gates, x, "correlated", shuffle, balanced)
    T_s = int(T_probe * target_s / max(sec, 1e-6))
    T_s = max(w.G, min(w.T, (T_s // w.G) * w.G))
    return T_s


def cpu_baseline(w, placement, shuffle, target_s, balanced=False, base_seed=None):
    base_seed = w.seed if base_seed is None else base_seed
    T_s = sized_sample(w, target_s, shuffle, balanced, base_seed)
    ids, cal, gates, x = cpu_sample(w, T_s, base_seed)
    sec, nbytes = oracle_pass(w, ids, cal, gates, x, placement, shuffle, balanced)
    model = platform.processor() or platform.machine()
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return {"value": nbytes / sec / 1e9, "unit": "GB/s", "cores": 1, "kind": "oracle",
            "sample": "%d of %d tokens of %s, all %d layers (stats, calibration, placement, plan, permute, "
                      "fp64 combine, shuffle), single-threaded C oracle on 1 of %d host cores (%s); %.1f s"
                      % (T_s, w.T, w.name, w.L, os.cpu_count() or 0, model, sec)}


def run_reference(a, w):
    rank, world, local = dist_env()
    if rank != 0:
        return
    shuffle = not a.no_shuffle
    bal = shuffle and a.balanced_shuffle
    # each step: a bounded sample, so that warmup + steps end within a few minutes
    per_step = max(0.5, min(10.0, 150.0 / max(1, a.steps + a.warmup)))
    base_seed = a.seed if getattr(a, "seed", None) is not None else w.seed
    T_s = sized_sample(w, per_step, shuffle, bal, base_seed)
    ids, cal, gates, x = cpu_sample(w, T_s, base_seed)
    for _ in range(a.warmup):
        oracle_pass(w, ids, cal, gates, x, a.placement, shuffle, bal)
    secs, nb = [], 0
    for _ in range(a.steps):
        s, nb = oracle_pass(w, ids, cal, gates, x, a.placement, shuffle, bal)
        secs.append(s)
    tot = sum(secs)
    value = nb * a.steps / tot / 1e9
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": a.gpus,
            "steps": a.steps, "warmup": a.warmup, "ms_per_step": 1e3 * tot / a.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": w.name, "tokens_per_step": T_s, "T": w.T, "E": w.E, "k": w.k, "G": w.G,
                       "rpn": w.rpn, "d": w.d, "L": w.L, "placement": a.placement,
                       "shuffle": ("balanced" if bal else True) if shuffle else False},
            "cpu_baseline": {"value": value, "unit": "GB/s", "cores": 1, "kind": "oracle",
                             "sample": "%d of %d tokens per step, single-threaded C oracle" % (T_s, w.T)},
            "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ native arm

def traffic_record(kernel_name, algorithmic_bytes_per_launch, k=None):
    """DRAM bytes per launch for the dominant kernel, from the committed ncu
    capture (profiles/traffic.json): the capture's DRAM bytes over its
    algorithmic bytes, scaled to this launch's algorithmic bytes (both kernels
    stream, so traffic grows in proportion).  The record of the same top-k
    instantiation ("combine_k8") is preferred to the kernel's general one.
    None when the kernel's source changed since the capture."""
    import hashlib
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        recs = json.load(f)
    rec = recs.get("%s_k%d" % (kernel_name, k)) if k is not None else None
    rec = rec or recs.get(kernel_name)
    if not rec:
        return None
    names = rec["source"].split("+")              # the kernel's file and the headers it is built from
    blob = b"".join(open(os.path.join(ROOT, "co_activation_placement_b200", "csrc", n), "rb").read() for n in names)
    h = hashlib.sha256(blob).hexdigest()[:16]
    if h != rec["source_sha256_16"]:
        return None
    return int(rec["traffic_over_algorithmic"] * algorithmic_bytes_per_launch)


def main():
    a = parse()
    from synth import WORKLOADS
    w = WORKLOADS[a.workload]
    if a.placement is None:
        a.placement = "uniform" if w.name == "tiny" else "correlated"
    if a.impl == "reference":
        run_reference(a, w)
        return
    import torch
    import co_activation_placement_b200 as cap
    from co_activation_placement_b200 import pipeline
    from synth import make_routing, make_gates, make_hidden, make_expert_scales

    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    pg = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=device)
        pg = dist
    seed = rank_seed(a.seed if a.seed is not None else w.seed, rank)
    cap.coact_stats_method({"auto": 0, "histogram": 1, "tensor": 2}[a.coact_method])
    if a.ep:
        run_ep(a, w, rank, world, device, seed)
        return
    if a.sweep_only:
        hbm, _ = peaks()
        sweep = run_sweep(cap, pipeline, device, seed, a.steps, a.warmup, hbm, pg)
        if rank == 0:
            print(json.dumps({"coact_sweep": sweep}), flush=True)
        if pg is not None:
            pg.destroy_process_group()
        return
    shuffle = (not a.no_shuffle) and w.L > 1
    balanced = shuffle and a.balanced_shuffle
    out_dtype = torch.float32 if a.out_dtype == "f32" else torch.bfloat16
    if w.d == 0:
        raise SystemExit("workload %s has no hidden states; it is measured as the co-activation sweep" % w.name)

    ids = make_routing(w, seed=seed)
    ids_cal = make_routing(w, seed=seed + 1)
    gates = make_gates(w, seed=seed)
    x = make_hidden(w, seed=seed)
    hp = pipeline.prepare(w.E, w.G, w.rpn, ids, gates, x, w.dtype, ids_cal, placement=a.placement,
                          shuffle=shuffle, out_dtype=out_dtype, device=device, timers=True,
                          scales=make_expert_scales(w, seed=seed) if a.prereduce else None,
                          replica_extra=a.replicas, shuffle_capacity=w.T // w.G if balanced else 0,
                          overlap=not a.no_overlap, replica_eps=a.replica_eps,
                          schedule="inline" if a.no_overlap else a.schedule, row_chunks=a.row_chunks)
    place = time_placement(cap, ids_cal, w, a.placement, device)

    def barrier():
        if pg is not None:
            pg.barrier()

    for _ in range(a.warmup):
        hp.step()
    torch.cuda.synchronize()
    if int(hp.err.item()) != 0:
        raise SystemExit("device data error %d" % int(hp.err.item()))
    summaries = hp.summaries()
    sb = hp.step_bytes(summaries)

    uuid = None
    try:
        uuid = "GPU-" + str(torch.cuda.get_device_properties(device).uuid)
    except Exception:
        pass
    # the timed steps: captured once into a CUDA graph (launch gaps between
    # the small kernels vanish), or launched eagerly with --no-graph.  The
    # timed graph carries no per-call timing events; a second graph with them
    # is replayed afterwards for the per-kernel breakdown.
    # inputs that fit in L2 would stay cached from one step to the next: then
    # every step is timed on its own, after a write of twice the L2 size
    l2_bytes = int(getattr(torch.cuda.get_device_properties(device), "L2_cache_size", 0) or (126 << 20))
    in_bytes = x.nbytes + ids.nbytes + gates.nbytes
    flush = None if in_bytes > l2_bytes else torch.empty(2 * l2_bytes, dtype=torch.uint8, device=device)
    per_graph = a.steps if flush is None else 1      # steps recorded in one graph
    graph = None
    graph_note = None
    hp.timers = False
    if not a.no_graph:
        try:
            n0 = cap.launch_count()
            graph = hp.capture(per_graph)
            n_launch = (cap.launch_count() - n0) * (a.steps // per_graph)   # kernels the replays run
        except Exception as ex:                    # capture unsupported here: time eagerly
            graph, graph_note = None, "graph capture failed: %s" % str(ex).splitlines()[0][:120]
            torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()
    if graph is None:
        n0 = cap.launch_count()

    def run(n):
        if graph is not None:
            graph.replay()
        else:
            for _ in range(n):
                hp.step()

    with ClockSampler(uuid) as clk:
        if flush is None:
            start = torch.cuda.Event(enable_timing=True)
            stop = torch.cuda.Event(enable_timing=True)
            start.record()
            run(a.steps)
            stop.record()
            torch.cuda.synchronize()
            ms_total = start.elapsed_time(stop)
        else:
            pairs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                     for _ in range(a.steps)]
            for s0, s1 in pairs:
                flush.zero_()
                s0.record()
                run(1)
                s1.record()
            torch.cuda.synchronize()
            ms_total = sum(s0.elapsed_time(s1) for s0, s1 in pairs)
    if graph is None:
        n_launch = cap.launch_count() - n0
    barrier()
    # per-kernel device times: the same steps again, with events around every
    # call (a replayed graph re-records its events: they hold its last replay)
    graphed = graph is not None
    hp.timers = True
    hp.reset_events()
    if graphed:
        del graph
        timed = hp.capture(per_graph)
        for _ in range(a.steps // per_graph):
            if flush is not None:
                flush.zero_()
            timed.replay()
        torch.cuda.synchronize()
        del timed
        ev_steps = per_graph
    else:
        for _ in range(a.steps):
            if flush is not None:
                flush.zero_()
            hp.step()
        torch.cuda.synchronize()
        ev_steps = a.steps
    per_kernel = hp.kernel_times_ms()
    hp.reset_events()
    if int(hp.err.item()) != 0:
        raise SystemExit("device data error %d in the timed steps" % int(hp.err.item()))
    ms_step = ms_total / a.steps
    ms_step = reduce_max(ms_step, pg, device)
    clocks = clk.summary()

    hbm, hbm_kind = peaks()
    value = weak_value(world, sb.dispatch_combine, ms_step)
    kern = {}
    # the source order computed ahead (forward schedule): src_rank read, perm written
    presort = bool(getattr(hp, "presort", False))
    bytes_of = {"stats": sb.stats, "plan": sb.plan, "permute": sb.permute, "combine": sb.combine,
                "shuffle": sb.shuffle, "gates": sb.gates, "reduce": sb.reduce,
                "sources": (w.L - 1) * 8 * w.T if presort else 0}
    rc = getattr(hp, "row_chunks", 1)
    launches_of = {"stats": 1, "plan": w.L, "permute": w.L * rc, "combine": w.L * rc,
                   "shuffle": (w.L - 1) if shuffle else 0,
                   "gates": w.L, "reduce": w.L, "sources": (w.L - 1) if presort else 0}
    for name, tot_ms in per_kernel.items():
        ms = tot_ms / ev_steps                        # per step
        gbs = bytes_of[name] / (ms * 1e-3) / 1e9 if ms > 0 else 0.0
        kern[name] = {"ms_per_step": ms, "launches_per_step": launches_of[name], "gbs": gbs,
                      "frac_of_hbm": gbs / hbm}
    # with the overlap the control calls' event times include waiting for SM
    # slots beside the row traffic: the dominant kernel is taken among the
    # calls on the main stream, whose chain is the step
    side_calls = hp.side_calls
    dom = max((n for n in kern if n not in side_calls), key=lambda n: kern[n]["ms_per_step"])
    nl = launches_of[dom]
    per_launch_ms = kern[dom]["ms_per_step"] / nl
    traffic = traffic_record(dom, bytes_of[dom] // nl, w.k)
    roofline = {"bound": "hbm", "kernel": dom, "achieved": kern[dom]["gbs"], "peak": hbm, "unit": "GB/s",
                "frac": kern[dom]["gbs"] / hbm, "peak_kind": hbm_kind,
                "algorithmic_bytes_per_launch": bytes_of[dom] // nl, "ms_per_launch": per_launch_ms,
                "traffic": traffic}

    # co-activation tokens/s on this step and on the statistics sweep
    stats_ms = kern["stats"]["ms_per_step"]
    # in line only: with the overlap the statistics share the SMs with the
    # row kernels and their event time is not their own (the sweep times them alone)
    coact_tps = None if "stats" in hp.side_calls else world * w.L * w.T / (stats_ms * 1e-3)
    sweep = None
    if not a.no_sweep:
        sweep = run_sweep(cap, pipeline, device, seed, a.steps, a.warmup, hbm, pg)

    ep_emu = None
    if a.ep_emulate > 0 and not a.prereduce and a.replicas == 0:
        ep_emu = run_ep_emulated(hp, w, a.ep_emulate, a.steps, a.warmup, hbm, sb, pg)

    e2e = None
    if not a.no_e2e:
        e2e = run_e2e(hp, ids, gates, x, w, a, device, sb, pg, world)

    cpu = None
    if rank == 0 and world == 1 and not a.no_cpu_baseline:
        cpu = cpu_baseline(w, a.placement, shuffle, a.cpu_seconds, balanced, seed)

    if rank == 0:
        R = [int(s[0]) for s in summaries]
        line = {
            "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": a.steps,
            "warmup": a.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "dtype_note": "the combine accumulates in fp32; rows (x_dtype) are moved bit for bit; counts and plans are integer",
            "config": {"workload": w.name, "seed": seed, "T": w.T, "E": w.E, "k": w.k, "G": w.G, "rpn": w.rpn, "d": w.d,
                       "L": w.L, "x_dtype": w.dtype, "out_dtype": a.out_dtype, "placement": a.placement,
                       "combine": "receiver-side pre-reduced (stand-in experts)" if a.prereduce
                                  else "source-side weighted (identity experts)",
                       "replicas_per_rank": a.replicas,
                       "replica_eps": a.replica_eps if a.replicas else None,
                       "schedule": hp.schedule,
                       "row_chunks": hp.row_chunks,
                       "overlap": (", ".join({"stats": "statistics", "plan": "plans", "shuffle": "shuffle targets",
                                              "sources": "the next layer's source order"}[c]
                                             for c in hp.side_calls) + " on a second stream" +
                                   ("; its cooperative launches on fewer blocks than SMs"
                                    if (balanced and "shuffle" in hp.side_calls) or
                                    (a.replicas and a.replica_eps is not None and "plan" in hp.side_calls) else ""))
                                  if hp.overlap else "none",
                       "shuffle": ("balanced (T/G tokens per rank)" if balanced else True) if shuffle else False,
                       "parallelism": "replicas (weak scaling, one batch per GPU)",
                       "l2": ("inputs larger than L2 (%.2f GB per GPU; no flush)" % (in_bytes / 1e9))
                             if flush is None else
                             ("inputs within L2 (%.3f GB per GPU): L2 flushed (%d MB write) before every "
                              "step, steps timed one by one" % (in_bytes / 1e9, flush.nbytes >> 20))},
            "frac_of_hbm_peak": value / hbm,
            "roofline": roofline,
            "kernels": kern,
            "coact_tokens_per_s": coact_tps,
            "coact_tokens_per_s_source": "the statistics sweep (coact_sweep.tokens_per_s) times the statistics alone"
                                         if hp.overlap else "this step's statistics call",
            "coact_sweep": sweep,
            "rows": {"R": R, "T_k": w.T * w.k, "dedup_removed": [1 - r / (w.T * w.k) for r in R],
                     "R_remote": [int(s[1]) for s in summaries],
                     "local_share": [int(s[2]) / (w.T * w.k) for s in summaries],
                     "V": [int(s[3]) for s in summaries]},
            "replica_load": replica_load(hp, w),
            "clocks": clocks,
            "balanced_shuffle": {
                "rounds": hp.shuffle_info[:, 0].tolist(), "proposals": hp.shuffle_info[:, 1].tolist(),
                "phase_us": {n: (hp.shuffle_info[:, 2 + i].double() / 1e3).tolist()
                              for i, n in enumerate(["propose", "gather", "select", "barrier_wait"])}}
            if balanced else None,
            "e2e": e2e,
            "placement_host": place,
            "ep_emulated": ep_emu,
            "gpu_launches": int(n_launch),
            "gpu_launches_per_step": n_launch / a.steps,
            "kernel_times": "CUDA events around each library call on its stream; plans, shuffle targets and "
                            "statistics run on a second stream beside the row traffic, so their times include "
                            "waiting for SM slots and the kernel times add up to more than the step"
                            if hp.overlap else "CUDA events around each library call",
            "timing": ("one CUDA graph of the %d steps" % a.steps if flush is None else
                       "one CUDA graph of one step, replayed %d times between L2 flushes" % a.steps)
                      + ", without per-call events (a second graph with them gives the kernel breakdown)"
                      if graphed else ("eager launches" + ("; " + graph_note if graph_note else "")),
            "cpu_baseline": cpu,
        }
        print(json.dumps(line), flush=True)
    if pg is not None:
        pg.destroy_process_group()


def run_sweep(cap, pipeline, device, seed, steps, warmup, hbm, pg):
    """Co-activation statistics on the 1M-token, 8-layer sweep: tokens/s and
    the fraction of HBM the statistics kernels reach on their input bytes,
    for the default counting method and, beside it, for each method alone
    (shared-memory histograms; the one-hot contraction on the tensor cores),
    each against its own ceiling."""
    import torch
    from synth import WORKLOADS, make_routing
    w = WORKLOADS["stats_sweep"]
    ids = make_routing(w, seed=seed)
    ids_d = torch.from_numpy(ids).to(device)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=device)
    world = pg.get_world_size() if pg is not None else 1
    sms = torch.cuda.get_device_properties(device).multi_processor_count
    n = max(steps, 10)

    def timed(method):
        prev = cap.coact_stats_method(method)
        try:
            hp = pipeline.HotPath(E=w.E, G=1, rpn=1, ids=ids_d, gates=None, x=None, e2r=[], rank_scores=[],
                                  rows=False)
            path = cap.coact_stats_path(w.L, w.T, w.k, w.E, True)
            for _ in range(warmup):
                hp.step()
            torch.cuda.synchronize()
            tot = 0.0
            for _ in range(n):
                flush.zero_()                         # ids (268 MB) exceed L2; flush anyway
                s_ = torch.cuda.Event(enable_timing=True)
                e_ = torch.cuda.Event(enable_timing=True)
                s_.record()
                hp.step()
                e_.record()
                torch.cuda.synchronize()
                tot += s_.elapsed_time(e_)
            err = int(hp.err.item())
        finally:
            cap.coact_stats_method(prev)
        return reduce_max(tot / n, pg, device), path, hp, err

    def record(ms, path, nbytes):
        incs = (w.L * w.T * w.k * (w.k + 1) // 2 + (w.L - 1) * w.T * w.k * w.k) / (ms * 1e-3)
        r = {"ms": ms, "method": path, "tokens_per_s": world * w.L * w.T / (ms * 1e-3),
             "gbs": nbytes / (ms * 1e-3) / 1e9, "frac_of_hbm": nbytes / (ms * 1e-3) / 1e9 / hbm}
        if path == "tensor":
            # C_l = X_l X_l^T and M_l = X_l X_{l+1}^T: 2 E^2 T int8 operations each
            ops = 2.0 * w.E * w.E * w.T * (2 * w.L - 1) / (ms * 1e-3)
            bf16, kind = tensor_peak()
            r["tensor_roofline"] = {
                "bound": "tensor", "achieved": ops / 1e12, "unit": "TOP/s (int8)", "peak": 2 * bf16,
                "frac": ops / 1e12 / (2 * bf16),
                "peak_note": "%s bf16 dense %.1f TFLOP/s x 2 (nominal int8 / bf16 ratio 4.5 / 2.25)" % (kind, bf16)}
        else:
            # shared memory serves 32 4-byte accesses per clock per SM, so at
            # most 32 counter increments per clock per SM
            peak_inc = 32.0 * sms * SM_MAX_MHZ * 1e6
            r["increments_per_s"] = world * incs
            r["atomic_roofline"] = {"bound": "shared-memory atomics", "achieved": incs, "unit": "increments/s",
                                    "peak": peak_inc, "frac": incs / peak_inc,
                                    "peak_note": "32 per clock per SM x %d SMs x %.0f MHz" % (sms, SM_MAX_MHZ)}
        return r

    ms, path, hp, err = timed(0)
    nbytes = hp.step_bytes(None).stats
    methods = {}
    for name, m in (("histogram", 1), ("tensor", 2)):
        ms_m, path_m, _, err_m = timed(m)
        methods[name] = record(ms_m, path_m, nbytes)
        methods[name]["err"] = err_m
    # what the placements do on this batch: local share, V per token and rank
    # load balance at each rank count (8 ranks per node), placements from a
    # calibration batch
    effect = {}
    ids_cal = torch.from_numpy(make_routing(w, seed=seed + 1)).to(device)
    for G in w.sweep_G:
        row = {}
        for placement in ("uniform", "correlated", "capped", "capacity"):
            sm, rl = pipeline.placement_effect(hp.ids, ids_cal, w.E, G, w.rpn, placement, loads=True)
            row[placement] = {"local_share": [round(int(r[2]) / int(r[4]), 5) for r in sm],
                              "V_per_token": [round(int(r[3]) / w.T, 4) for r in sm],
                              "rows_removed": [round(1 - int(r[0]) / int(r[4]), 4) for r in sm],
                              # per-rank load: token-expert assignments served
                              "load_max_over_mean": [round(float(x.max() / x.mean()), 4) for x in rl],
                              "load_cv": [round(float(x.std() / x.mean()), 4) for x in rl]}
        effect["G=%d" % G] = row
    del ids_cal
    out = {"workload": w.name, "T": w.T, "E": w.E, "k": w.k, "L": w.L}
    out.update(record(ms, path, nbytes))
    out.update({"methods": methods, "algorithmic_bytes": nbytes, "err": err, "placement_effect": effect})
    return out


def replica_load(hp, w):
    """Per-rank task loads the capped replica assignment returned (one row
    per layer): busiest rank over the mean, next to V in "rows"; beside them
    the same assignment without a cap (eps = inf) on the same inputs, and
    the ranks whose tasks reach the cap."""
    if not hp.replicas or hp.replica_eps is None:
        return None
    import torch
    import co_activation_placement_b200 as cap
    ld = hp.rank_load.cpu().double()
    free = torch.zeros_like(hp.rank_load)
    pick = torch.empty_like(hp.pick_rank)
    for l in range(hp.L):
        src = hp.targets[l - 1] if (hp.shuffle and l > 0) else None
        rr, nr = hp.replicas[l]
        cap.assign_replicas_capped(hp.ids[l], hp.E, hp.G, hp.rpn, rr, nr, float("inf"), src_rank=src,
                                   pick_rank=pick, rank_load=free[l], err=hp.err, ws=hp.capped_ws)
    torch.cuda.synchronize()
    fr = free.cpu().double()
    limit = int(((1.0 + hp.replica_eps) * hp.T * hp.k) // hp.G)
    return {"eps": hp.replica_eps, "cap": limit,
            "max_over_mean": [float(r.max() / r.mean()) for r in ld],
            "max": [int(r.max()) for r in ld], "mean": [float(r.mean()) for r in ld],
            "ranks_at_cap": [int((r >= limit).sum()) for r in ld],
            "uncapped_max_over_mean": [float(r.max() / r.mean()) for r in fr],
            "uncapped_ranks_over_cap": [int((r > limit).sum()) for r in fr]}


def time_placement(cap, ids_cal, w, placement, device):
    """Host time of the placement from the calibration batch's counts (the
    step that runs once per re-layout, on one CPU thread): per layer, and the
    counts' device-to-host read beside it."""
    import torch
    cal = torch.from_numpy(ids_cal).to(device)
    st = cap.coact_stats(cal, w.E, want=("coact",))
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    coact = st["coact"].cpu().numpy()
    t1 = time.perf_counter()
    for l in range(w.L):
        c = coact[l]
        if placement == "uniform":
            cap.place_uniform(w.E, w.G)
        elif placement == "correlated":
            cap.place_correlated(c, w.G, w.rpn)
        elif placement == "capped":
            cap.place_correlated_capped(c, w.G, w.rpn, 0.1)
        else:
            cap.place_capacity(np.diag(c).astype(np.float64), w.G)
    t2 = time.perf_counter()
    return {"kind": placement, "ms_per_layer": (t2 - t1) * 1e3 / w.L, "counts_readback_ms": (t1 - t0) * 1e3,
            "threads": 1, "E": w.E, "G": w.G}


def run_ep(a, w, rank, world, device, seed):
    """--ep: one process per GPU, the workload's G ranks spread over the N
    GPUs (G/N each), every GPU with its own batch of T tokens (weak scaling:
    N*T tokens over the G ranks).  A step: the statistics of all GPUs' tokens
    (local counts, one all-reduce) and, per layer, the plan of this GPU's
    tokens, the counts all-gather, the route table, the rows stored into the
    receiving GPUs' buffers, identity experts and the combine loading them
    back (EPGroup).  The placement comes from one calibration batch that every
    GPU draws alike.  Timed eagerly with CUDA events, max over the GPUs."""
    import datetime
    import socket
    import torch
    import torch.distributed as dist
    import co_activation_placement_b200 as cap
    from co_activation_placement_b200 import pipeline
    from co_activation_placement_b200.ep import EPGroup
    from synth import make_routing, make_gates, make_hidden
    if not dist.is_initialized():                 # one GPU: a one-process group
        with socket.socket() as so:
            so.bind(("127.0.0.1", 0))
            port = so.getsockname()[1]
        dist.init_process_group("nccl", init_method="tcp://127.0.0.1:%d" % port, rank=0, world_size=1,
                                timeout=datetime.timedelta(seconds=120), device_id=device)
    if w.G % world or w.d == 0:
        raise SystemExit("--ep needs hidden states and N dividing G")
    base = a.seed if a.seed is not None else w.seed
    ids = torch.from_numpy(make_routing(w, seed=seed)).to(device)
    gates = torch.from_numpy(make_gates(w, seed=seed)).to(device)
    xh = make_hidden(w, seed=seed)
    x = (torch.from_numpy(xh.view(np.int16)).to(device).view(torch.bfloat16) if w.dtype == "bf16"
         else torch.from_numpy(xh).to(device))
    cal = torch.from_numpy(make_routing(w, seed=base + 1)).to(device)
    e2r = pipeline.calibrate(cal, w.E, w.G, w.rpn, a.placement, False)[0]
    Gl = w.G // world
    # receive capacity and row counts: every layer planned once, counts gathered
    from co_activation_placement_b200.ep import EPShard, gather_counts
    sh = EPShard(world, rank, w.E, w.G, w.rpn, w.T, w.k, w.d, x.dtype, device)
    need, R, counts = 0, [], []
    for l in range(w.L):
        sh.plan_layer(ids[l], e2r[l])
        gather_counts(sh.counts_all, sh.my_counts())
        c = sh.counts_all.cpu().numpy().astype(np.int64)
        counts.append(c.astype(np.int32))
        need = max(need, int(c[:, rank * Gl:(rank + 1) * Gl].sum()))
        R.append(int(sh.plan.summary[0].item()))
    del sh
    t = torch.tensor([need], dtype=torch.int64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    recv_cap = int(t.item()) + 64
    out_dtype = torch.float32 if a.out_dtype == "f32" else torch.bfloat16
    grp = EPGroup(w.E, w.G, w.rpn, w.T, w.k, w.d, x.dtype, device, recv_cap, out_dtype=out_dtype)

    def step():
        grp.stats(ids, w.E)
        for l in range(w.L):
            grp.step(ids[l], x, gates[l], e2r[l])

    for _ in range(a.warmup):
        step()
    torch.cuda.synchronize()
    if int(grp.shard.err.item()):
        raise SystemExit("device data error %d" % int(grp.shard.err.item()))
    dist.barrier()
    torch.cuda.synchronize()
    n0 = cap.launch_count()
    uuid = None
    try:
        uuid = "GPU-" + str(torch.cuda.get_device_properties(device).uuid)
    except Exception:
        pass
    with ClockSampler(uuid) as clk:
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(a.steps):
            step()
        e1.record()
        torch.cuda.synchronize()
    n_launch = cap.launch_count() - n0
    dist.barrier()
    ms = reduce_max(e0.elapsed_time(e1) / a.steps, dist, device)
    rowB = w.d * x.element_size()
    ob = w.d * (4 if a.out_dtype == "f32" else 2)
    mine = sum(w.T * rowB + r * rowB + 4 * w.T * w.k + r * rowB + w.T * ob + 8 * w.T * w.k for r in R)
    tb = torch.tensor([float(mine)], dtype=torch.float64, device=device)
    dist.all_reduce(tb)
    hbm, hbm_kind = peaks()
    value = float(tb.item()) / (ms * 1e-3) / 1e9
    if rank == 0:
        print(json.dumps({
            "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": a.steps,
            "warmup": a.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "dtype_note": "the combine accumulates in fp32; rows (x_dtype) are moved bit for bit; counts and plans are integer",
            "config": {"workload": w.name, "seed": seed, "T_per_gpu": w.T, "E": w.E, "k": w.k, "G": w.G, "rpn": w.rpn,
                       "d": w.d, "L": w.L, "x_dtype": w.dtype, "out_dtype": a.out_dtype, "placement": a.placement,
                       "parallelism": "expert parallel over %d GPU(s), %d ranks each" % (world, Gl),
                       "recv_rows_capacity": recv_cap,
                       "l2": "inputs larger than L2" if x.nbytes > (126 << 20) else "inputs within L2 (no flush)"},
            "frac_of_hbm_peak": value / hbm if world == 1 else None,
            "roofline": None,
            "roofline_note": "per-kernel events are not taken in this mode; the one-GPU path reports the kernels",
            "clocks": clk.summary(), "gpu_launches": int(n_launch), "e2e": None, "cpu_baseline": None,
            "cross_device": exchange_record(cap, counts, w.G, world, w.d * x.element_size(), ms),
            "timing": "eager launches between two CUDA events, max over the GPUs",
        }), flush=True)
    del grp
    dist.destroy_process_group()


NVLINK_GBS = 770.0   # measured peer copy per direction per GPU on this machine (the profiling recipe's figure)


def exchange_record(cap, counts_layers, G, W, rowB, ms_step, crossed=True):
    """Rows and bytes that cross devices in the exchange with the G ranks on W
    devices (moe_ep_exchange_rows on each layer's gathered counts), and the
    NVLink floor they set: per layer the busiest device sends or receives
    max(sent_h, received_h) rows in the dispatch and again in the combine, at
    NVLINK_GBS per direction.  crossed: the rows did cross NVLink in the timed
    steps (several GPUs); else (virtual devices on one GPU) only the floor is
    reported, beside the measured step."""
    rows, busiest = [], []
    for c in counts_layers:
        sent, recv = cap.ep_exchange_rows(c, G, W)
        rows.append(int(sent.sum()))
        busiest.append(int(max(sent.max(), recv.max())))
    floor_ms = sum(2.0 * b * rowB / (NVLINK_GBS * 1e9) * 1e3 for b in busiest)
    busiest_bytes = sum(2 * b * rowB for b in busiest)
    nv = {"bound": "nvlink", "peak": NVLINK_GBS, "unit": "GB/s",
          "peak_kind": "measured peer copy per direction (pool figure)",
          "busiest_device_bytes_per_step": busiest_bytes, "floor_ms_per_step": floor_ms}
    if crossed and ms_step > 0 and W > 1:
        nv["achieved"] = busiest_bytes / (ms_step * 1e-3) / 1e9
        nv["frac"] = nv["achieved"] / NVLINK_GBS
    else:
        nv["floor_over_measured_step"] = floor_ms / ms_step if ms_step > 0 else None
    return {"devices": W, "rows_crossing_per_layer": rows, "bytes_each_way_per_step": sum(rows) * rowB,
            "busiest_device_rows_per_layer": busiest, "nvlink": nv}


def run_ep_emulated(hp, w, W, steps, warmup, hbm, sb, pg):
    """The several-device path (moe_ep_routes / moe_ep_permute / moe_ep_combine)
    with W virtual devices on this GPU, each with its own receive buffer and
    T/W tokens, over all layers with identity experts; one CUDA graph of the
    steps.  The bytes are the step's dispatch+combine bytes: R does not depend
    on which rank a token starts from."""
    import torch
    import co_activation_placement_b200 as cap
    from co_activation_placement_b200.ep import EPEmulation
    if w.G % W or w.T % W:
        return {"devices": W, "skipped": "W must divide G and T"}
    Gl = w.G // W
    rows = 0
    for l in range(w.L):                      # receive capacity from the contiguous-source plans
        p = cap.plan_dispatch(hp.ids[l], w.E, w.G, w.rpn, hp.e2r[l])
        off = p.offsets.cpu().numpy().astype(np.int64)
        rows = max(rows, max(int(off[(h + 1) * Gl * w.G] - off[h * Gl * w.G]) for h in range(W)))
        del p
    emu = EPEmulation(W, w.E, w.G, w.rpn, w.T, w.k, w.d, hp.x.dtype, hp.x.device, rows, out_dtype=hp.out_dtype)

    def step():
        for l in range(w.L):
            emu.step(hp.ids[l], hp.x, hp.gates[l], hp.e2r[l])

    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    if any(emu.errors()):
        raise SystemExit("device data error in the several-device path: %s" % emu.errors())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, capture_error_mode="thread_local"):
        for _ in range(steps):
            step()
    if pg is not None:
        pg.barrier()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    g.replay()
    b.record()
    torch.cuda.synchronize()
    ms = a.elapsed_time(b) / steps
    del g
    counts = []
    for l in range(w.L):                      # each layer's gathered counts, for the exchange record
        emu.step(hp.ids[l], hp.x, hp.gates[l], hp.e2r[l])
        counts.append(emu.shards[0].counts_all.cpu().numpy())
    nbytes = sb.permute + sb.combine
    return {"devices": W, "ranks_per_device": Gl, "tokens_per_device": w.T // W, "recv_rows_max": rows,
            "exchange": exchange_record(cap, counts, w.G, W, w.d * hp.x.element_size(), ms, crossed=False),
            "exchange_note": "the rows that would cross NVLink with the W devices on W GPUs; here they move "
                             "within one GPU's memory: floor_over_measured_step > 1 means W GPUs would be "
                             "NVLink-bound at the measured peer bandwidth",
            "ms_per_step": ms, "gbs": nbytes / (ms * 1e-3) / 1e9, "frac_of_hbm": nbytes / (ms * 1e-3) / 1e9 / hbm,
            "errors": emu.errors(),
            "note": "W virtual devices on this GPU, each with its own receive buffer and stream (a phase of the W devices runs side by side, each meeting joins the streams); "
                    "rows move through the peer-addressed kernels within this GPU's memory; per layer and "
                    "device: plan, routes, permute, combine (the counts gathered with one device-side copy)"}


def run_e2e(hp, ids, gates, x, w, a, device, sb, pg, world):
    """The same metric through the public API with host buffers: every step
    copies its inputs from pinned host memory and reads its results back
    (statistics, plan summaries, shuffle targets and the last layer's combine
    output).  Steps are pipelined: inputs and the big output are double
    buffered, so step i+1's host-to-device copy and step i-1's device-to-host
    copy run on their own streams while step i computes."""
    import torch
    from co_activation_placement_b200.pipeline import bf16_from_bits
    ids_h = torch.from_numpy(ids).pin_memory()
    gates_h = torch.from_numpy(gates).pin_memory()
    x_h = (bf16_from_bits(x) if w.dtype == "bf16" else torch.from_numpy(x)).pin_memory()
    out_h = torch.empty(hp.outs[-1].shape, dtype=hp.outs[-1].dtype).pin_memory()
    small = {k: v for k, v in hp.stats.items() if v is not None}
    small_h = {k: torch.empty(v.shape, dtype=v.dtype).pin_memory() for k, v in small.items()}
    sum_h = torch.empty((w.L, 5), dtype=torch.int64).pin_memory()
    tgt_h = [torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in hp.targets]
    sets = [dict(ids=hp.ids, gates=hp.gates, x=hp.x, out=hp.outs[-1]),
            dict(ids=torch.empty_like(hp.ids), gates=torch.empty_like(hp.gates), x=torch.empty_like(hp.x),
                 out=torch.empty_like(hp.outs[-1]))]
    comp = torch.cuda.current_stream()
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    ev = lambda: torch.cuda.Event()
    ready, done, read = [ev(), ev()], [ev(), ev()], [ev(), ev()]
    for e in done + read:
        e.record(comp)
    hp.timers = False

    def upload(j):
        s_in.wait_event(done[j])                  # the step that last read set j is over
        with torch.cuda.stream(s_in):
            sets[j]["ids"].copy_(ids_h, non_blocking=True)
            sets[j]["gates"].copy_(gates_h, non_blocking=True)
            sets[j]["x"].copy_(x_h, non_blocking=True)
        ready[j].record(s_in)

    def run(n, t0=None):
        if t0 is not None:
            t0.record(s_in)                       # before the first upload
        upload(0)
        for i in range(n):
            j = i % 2
            if i + 1 < n:
                upload(1 - j)
            comp.wait_event(ready[j])
            comp.wait_event(read[j])              # set j's output was read back
            hp.ids, hp.gates, hp.x, hp.outs[-1] = sets[j]["ids"], sets[j]["gates"], sets[j]["x"], sets[j]["out"]
            hp.step()
            for k_, v in small.items():           # small results, in stream order
                small_h[k_].copy_(v, non_blocking=True)
            sum_h.copy_(torch.stack([p.summary for p in hp.plans]), non_blocking=True)
            for th, td in zip(tgt_h, hp.targets):
                th.copy_(td, non_blocking=True)
            done[j].record(comp)
            s_out.wait_event(done[j])
            with torch.cuda.stream(s_out):
                out_h.copy_(sets[j]["out"], non_blocking=True)
            read[j].record(s_out)

    run(2)
    torch.cuda.synchronize()
    n = max(4, min(a.steps, 12))
    if pg is not None:
        pg.barrier()
    s = torch.cuda.Event(enable_timing=True)
    e = torch.cuda.Event(enable_timing=True)
    run(n, t0=s)
    e.record(s_out)
    torch.cuda.synchronize()
    ms = reduce_max(s.elapsed_time(e) / n, pg, device)
    hp.ids, hp.gates, hp.x, hp.outs[-1] = sets[0]["ids"], sets[0]["gates"], sets[0]["x"], sets[0]["out"]
    hp.timers = True
    h2d = ids_h.numel() * 4 + gates_h.numel() * 4 + x_h.numel() * x_h.element_size()
    d2h = (out_h.numel() * out_h.element_size() + sum(v.numel() * v.element_size() for v in small_h.values())
           + sum_h.numel() * 8 + sum(t.numel() * 4 for t in tgt_h))
    return {"value": weak_value(world, sb.dispatch_combine, ms), "unit": "GB/s", "ms_per_step": ms,
            "steps": n, "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
            "pipelined": "inputs and output double buffered; copies overlap compute across steps"}


if __name__ == "__main__":
    main()
