"""One step of the hot path over a batch, on preallocated device buffers.

A step is, for a batch of top-k routing decisions over L MoE layers:

  1. co-activation counts, Ochiai and cross-layer transitions for all layers
     (moe_coact_stats);
  2. per layer l: the deduplicated dispatch plan under that layer's placement,
     with source ranks = the previous layer's shuffle targets when token
     shuffling is on (moe_plan_dispatch); the row permute of the hidden states
     into the rank-major send buffer (moe_permute); identity experts (the
     expert output of a row is the row); the weighted combine back to token
     order (moe_combine); and, before layer l+1, the shuffle targets from
     layer l's picks (moe_shuffle_targets, or moe_shuffle_balanced when every
     rank's shard is capped).

Every step is a library call on torch's current stream; this module only
allocates buffers and sequences the calls.  Placements and rank-score tables
are inputs: they are computed from a calibration batch (a re-layout happens
every so many training steps, not every step).
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import List, Optional

import numpy as np
import torch

import co_activation_placement_b200 as cap


def bf16_from_bits(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16)


@dataclass
class StepBytes:
    """Algorithmic HBM bytes of one step (minimum traffic of each kernel)."""
    permute: int = 0
    combine: int = 0
    plan: int = 0
    stats: int = 0
    shuffle: int = 0
    gates: int = 0
    reduce: int = 0

    @property
    def dispatch_combine(self) -> int:
        return self.permute + self.gates + self.reduce + self.combine


@dataclass
class HotPath:
    E: int
    G: int
    rpn: int
    ids: torch.Tensor                  # int32 [L][T][k]
    gates: Optional[torch.Tensor]      # f32 [L][T][k]
    x: Optional[torch.Tensor]          # [T][d] f32 or bf16
    e2r: List[torch.Tensor]            # int32 [E] per layer
    rank_scores: List[torch.Tensor]    # uint32 [E][G] per layer pair (empty: no shuffle)
    out_dtype: torch.dtype = torch.bfloat16
    rows: bool = True                  # run plan/permute/combine (False: statistics only)
    timers: bool = False               # record CUDA events around each library call
    prereduce: bool = False            # receiver-side pre-reduced combine with stand-in experts
    scales: List[torch.Tensor] = field(default_factory=list)   # f32 [E] per layer (prereduce)
    replicas: list = field(default_factory=list)   # per layer (replica_rank [E][1+nodes], n_rep [E]) or empty
    shuffle_capacity: int = 0          # > 0: at most this many tokens per rank (moe_shuffle_balanced)
    replica_eps: Optional[float] = None   # load tolerance of the replica assignment (None: no cap)
    overlap: bool = True               # control work on a second stream beside the row traffic
    # "overlap": every layer's plan, shuffle and the statistics ahead on a
    # second stream (all routing known up front); "forward": the order of a
    # forward pass -- layer l's plan in line before its rows, its shuffle
    # targets and the statistics beside them; "inline": everything in line.
    # None: "overlap" if overlap else "inline".
    schedule: Optional[str] = None
    # blocks of the cooperative launches (balanced shuffle, capped assignment)
    # when they run beside the row traffic.  None: the balanced shuffle takes
    # min(G, 32) blocks and the capped assignment 48 (the rest of the SMs
    # stream rows; on large_ep64 these gave the shortest steps: 24, 48 and 64
    # blocks for the shuffle, 64, 96 and 148 for the assignment were slower,
    # 32 as fast)
    side_coop_blocks: Optional[int] = None
    side_priority: int = 0             # priority of the second stream (lower = higher priority)
    # > 1: a layer's permute and combine pipelined over this many token
    # chunks (the combine of chunk c beside the permute of chunk c + 1: a
    # token's combine reads only that token's rows), mixing the permute's
    # writes with the combine's reads in HBM; not with the pre-reduced combine
    row_chunks: int = 1
    # buffers
    stats: dict = field(default_factory=dict)
    plans: List[cap.Plan] = field(default_factory=list)
    send: Optional[torch.Tensor] = None
    outs: List[torch.Tensor] = field(default_factory=list)
    targets: List[torch.Tensor] = field(default_factory=list)
    err: Optional[torch.Tensor] = None
    events: list = field(default_factory=list)

    def __post_init__(self):
        L, T, k = self.ids.shape
        dev = self.ids.device
        E = self.E
        self.L, self.T, self.k = L, T, k
        self.err = cap.new_err(dev)
        if self.schedule is None:
            self.schedule = "overlap" if self.overlap else "inline"
        if self.schedule not in ("overlap", "forward", "inline"):
            raise ValueError("schedule must be overlap, forward or inline")
        self.overlap = self.schedule != "inline"
        self.presort = False
        self.stats = dict(coact=torch.empty((L, E, E), dtype=torch.uint32, device=dev),
                          ochiai=torch.empty((L, E, E), dtype=torch.float32, device=dev),
                          trans=torch.empty((max(L - 1, 1), E, E), dtype=torch.uint32, device=dev) if L > 1 else None)
        self.stats_ws = torch.empty(max(cap.coact_stats_workspace(L, T, k, E, L > 1), 1), dtype=torch.uint8, device=dev)
        if not self.rows:
            return
        self.shuffle = len(self.rank_scores) > 0
        self.plans = [cap.Plan.empty(T, k, self.G, dev) for _ in range(L)]
        self.plan_ws = torch.empty(max(cap.plan_dispatch_workspace(T, k, self.G, True), 1), dtype=torch.uint8, device=dev)
        # forward schedule: the next layer's source order (a counting sort of
        # the shuffle targets) is computed beside the rows, into that layer's
        # own plan workspace, so its plan on the critical path skips it
        self.presort = (self.schedule == "forward" and self.shuffle and not self.replicas and L > 1)
        self.plan_ws_l = [torch.empty_like(self.plan_ws) for _ in range(L)] if self.presort else []
        d = self.x.shape[1]
        self.send = torch.empty((T * k, d), dtype=self.x.dtype, device=dev)
        self.outs = [torch.empty((T, d), dtype=self.out_dtype, device=dev) for _ in range(L)]
        self.targets = [torch.empty(T, dtype=torch.int32, device=dev) for _ in range(max(L - 1, 0))] if self.shuffle else []
        if self.shuffle and self.shuffle_capacity > 0:
            self.shuffle_ws = torch.empty(max(cap.shuffle_balanced_workspace(T, self.G, self.shuffle_capacity), 1),
                                          dtype=torch.uint8, device=dev)
            # rounds and proposals of each balanced shuffle
            self.shuffle_info = torch.zeros((max(L - 1, 1), 6), dtype=torch.int64, device=dev)
        if self.prereduce or self.row_chunks < 1:
            self.row_chunks = 1
        if self.row_chunks > 1:
            self.comb_stream = torch.cuda.Stream(device=dev)
            self.chunk_ev = [torch.cuda.Event() for _ in range(self.row_chunks)]
        if self.overlap:
            self.side = torch.cuda.Stream(device=dev, priority=self.side_priority)
            self.fork_ev = torch.cuda.Event()
            self.join_ev = torch.cuda.Event()
            self.plan_ev = [torch.cuda.Event() for _ in range(L)]
            self.shuffle_ev = [torch.cuda.Event() for _ in range(L)]
        if self.replicas:
            self.pick_rank = torch.empty((T, k), dtype=torch.int32, device=dev)
            self.n_remote = torch.empty(T, dtype=torch.int32, device=dev)
            if self.replica_eps is not None:
                self.rank_load = torch.zeros((L, self.G), dtype=torch.int64, device=dev)
                self.capped_ws = torch.empty(cap.assign_replicas_capped_workspace(self.G), dtype=torch.uint8,
                                             device=dev)
        if self.prereduce:
            if len(self.scales) != L:
                raise ValueError("prereduce needs one scale vector per layer")
            self.send_e = torch.empty((T * k, k), dtype=torch.int32, device=dev)
            self.send_w = torch.empty((T * k, k), dtype=torch.float32, device=dev)
            self.y = torch.empty((T * k, d), dtype=self.x.dtype, device=dev)

    # ------------------------------------------------------------------ step
    def _call(self, name, fn):
        """Run one library call on torch's current stream inside an NVTX range
        (visible in Nsight timelines), bracketed by timing events when timers
        are on (external events: inside a captured graph they are real
        event-record nodes)."""
        with torch.cuda.nvtx.range("moe_" + name):
            if self.timers:
                a = torch.cuda.Event(enable_timing=True, external=True)
                a.record()
            out = fn()
            if self.timers:
                b = torch.cuda.Event(enable_timing=True, external=True)
                b.record()
                self.events.append((name, a, b))
        return out

    @property
    def side_calls(self):
        """The calls that run on the second stream, beside the row traffic."""
        return {"overlap": ("stats", "plan", "shuffle"), "forward": ("stats", "shuffle", "sources"),
                "inline": ()}[self.schedule]

    def _coop(self, fn, name):
        """Run a call that makes a cooperative launch; beside the row traffic
        the balanced shuffle takes fewer blocks than SMs, leaving the other
        SMs to the rows."""
        if name not in self.side_calls:
            return fn()
        n = self.side_coop_blocks
        if n is None:
            n = min(self.G, 32) if name == "shuffle" else 48
        prev = cap.cooperative_blocks(n)
        try:
            return fn()
        finally:
            cap.cooperative_blocks(prev)

    def reset_events(self):
        self.events = []

    # the parts of a step
    def _stats(self):
        self._call("stats", lambda: cap.coact_stats(self.ids, self.E, coact=self.stats["coact"],
                                                     ochiai=self.stats["ochiai"], trans=self.stats["trans"],
                                                     err=self.err, ws=self.stats_ws))

    def _plan(self, l):
        src = self.targets[l - 1] if (self.shuffle and l > 0) else None
        if self.replicas:
            # each task to a replica of its expert: fewest remote nodes per token
            rr, nr = self.replicas[l]

            def go():
                if self.replica_eps is not None:
                    self._coop(lambda: cap.assign_replicas_capped(
                        self.ids[l], self.E, self.G, self.rpn, rr, nr, self.replica_eps, src_rank=src,
                        pick_rank=self.pick_rank, n_remote=self.n_remote, rank_load=self.rank_load[l], err=self.err,
                        ws=self.capped_ws), "plan")
                else:
                    cap.assign_replicas(self.ids[l], self.E, self.G, self.rpn, rr, nr, src_rank=src,
                                        pick_rank=self.pick_rank, n_remote=self.n_remote, err=self.err)
                cap.plan_dispatch_ranks(self.ids[l], self.E, self.G, self.rpn, self.pick_rank, src_rank=src,
                                        plan=self.plans[l], ws=self.plan_ws)
            self._call("plan", go)
        elif self.presort and src is not None:
            self._call("plan", lambda: cap.plan_dispatch(self.ids[l], self.E, self.G, self.rpn, self.e2r[l],
                                                         src_rank=src, plan=self.plans[l], ws=self.plan_ws_l[l],
                                                         presorted=True))
        else:
            self._call("plan", lambda: cap.plan_dispatch(self.ids[l], self.E, self.G, self.rpn, self.e2r[l],
                                                         src_rank=src, plan=self.plans[l], ws=self.plan_ws))

    def _sources(self, l):
        """Layer l's source order from layer l - 1's shuffle targets."""
        self._call("sources", lambda: cap.plan_sources(self.targets[l - 1], self.G, self.plan_ws_l[l],
                                                        self.plans[l].err))

    def _rows(self, l):
        p = self.plans[l]
        if self.row_chunks > 1 and not self.prereduce:
            # chunk c's combine waits only for chunk c's permute; the next
            # layer's permute (which rewrites the send buffer) waits for all
            main = torch.cuda.current_stream(self.ids.device)
            C, T = self.row_chunks, self.T
            b = [T * c // C for c in range(C + 1)]
            for c in range(C):
                t0, t1 = b[c], b[c + 1]
                self._call("permute", lambda: cap.permute(self.x[t0:t1], p.row_of[t0:t1], p.R_max, send=self.send,
                                                          err=self.err))
                self.chunk_ev[c].record(main)
            for c in range(C):
                t0, t1 = b[c], b[c + 1]
                self.comb_stream.wait_event(self.chunk_ev[c])
                with torch.cuda.stream(self.comb_stream):
                    self._call("combine", lambda: cap.combine(self.send, p.row_of[t0:t1], self.gates[l][t0:t1],
                                                              out=self.outs[l][t0:t1], err=self.err))
            main.wait_stream(self.comb_stream)
            return
        self._call("permute", lambda: cap.permute(self.x, p.row_of, p.R_max, send=self.send, err=self.err))
        if self.prereduce:
            # gates travel with the rows; the receiving rank applies its
            # experts and returns one row per (token, rank); the source sums
            self._call("gates", lambda: cap.dispatch_gates(self.ids[l], self.gates[l], p, send_e=self.send_e,
                                                           send_w=self.send_w, err=self.err))
            self._call("reduce", lambda: cap.expert_reduce(self.send, p.summary, self.send_e, self.send_w,
                                                           self.scales[l], y=self.y, err=self.err))
            self._call("combine", lambda: cap.combine_rows(self.y, p.row_of, out=self.outs[l], err=self.err))
        else:
            self._call("combine", lambda: cap.combine(self.send, p.row_of, self.gates[l], out=self.outs[l],
                                                      err=self.err))

    def _shuffle(self, l):
        if not (self.shuffle and l + 1 < self.L):
            return
        if self.shuffle_capacity > 0:
            self._call("shuffle", lambda: self._coop(lambda: cap.shuffle_balanced(
                self.ids[l], self.E, self.G, self.rank_scores[l], self.shuffle_capacity, target=self.targets[l],
                info=self.shuffle_info[l], err=self.err, ws=self.shuffle_ws), "shuffle"))
        else:
            self._call("shuffle", lambda: cap.shuffle_targets(self.ids[l], self.E, self.G, self.rank_scores[l],
                                                              target=self.targets[l], err=self.err))

    def step(self):
        """One step.  With the overlap schedule, the control work -- plans,
        shuffle targets and statistics, which read only routing ids and tables
        -- runs on a second stream that starts when everything before the
        step is done and keeps ahead of the row traffic; the permute and
        combine of layer l wait only for layer l's plan.  The forward schedule
        keeps each plan on the critical path (see the field's comment)."""
        if not self.rows:
            self._stats()
            return
        if self.schedule == "inline":
            self._stats()
            for l in range(self.L):
                self._plan(l)
                self._rows(l)
                self._shuffle(l)
            return
        main = torch.cuda.current_stream(self.ids.device)
        if self.schedule == "forward":
            # layer l's routing exists once layer l - 1's rows are done: its
            # plan runs in line before its rows; its shuffle targets (needed
            # by the next layer's plan) and, after the last layer, the
            # statistics run beside the rows on the second stream
            for l in range(self.L):
                if l > 0 and self.shuffle:
                    main.wait_event(self.shuffle_ev[l - 1])
                self._plan(l)
                # layer l's routing is known from its plan on; the side work
                # starts after the plan so that it does not delay it
                self.plan_ev[l].record(main)
                if self.shuffle and l + 1 < self.L:
                    self.side.wait_event(self.plan_ev[l])
                    with torch.cuda.stream(self.side):
                        self._shuffle(l)
                        if self.presort:
                            self._sources(l + 1)
                        self.shuffle_ev[l].record(self.side)
                if l == self.L - 1:
                    self.side.wait_event(self.plan_ev[l])
                    with torch.cuda.stream(self.side):
                        self._stats()
                        self.join_ev.record(self.side)
                self._rows(l)
            main.wait_event(self.join_ev)
            return
        self.fork_ev.record(main)
        self.side.wait_event(self.fork_ev)
        with torch.cuda.stream(self.side):
            for l in range(self.L):
                self._plan(l)
                self.plan_ev[l].record(self.side)
                self._shuffle(l)
            self._stats()                       # nothing in the step waits for the statistics
            self.join_ev.record(self.side)
        for l in range(self.L):
            main.wait_event(self.plan_ev[l])
            self._rows(l)
        main.wait_event(self.join_ev)

    def capture(self, n_steps: int) -> torch.cuda.CUDAGraph:
        """Capture n_steps consecutive steps into one CUDA graph.  The library
        allocates nothing and every buffer is preallocated, so replaying the
        graph reruns exactly these steps.  Timing events (if on) are captured
        as event-record nodes; read them with kernel_times_ms() after a replay."""
        g = torch.cuda.CUDAGraph()
        torch.cuda.synchronize()
        self.reset_events()
        with torch.cuda.graph(g, capture_error_mode="thread_local"):
            for _ in range(n_steps):
                self.step()
        return g

    def kernel_times_ms(self):
        """Device time (ms) of each kind of call, summed over all steps run
        since reset_events() (call after synchronising).  With overlap the
        control calls run beside the row traffic, so the times add up to more
        than the step."""
        out = {}
        for name, a, b in self.events:
            out[name] = out.get(name, 0.0) + a.elapsed_time(b)
        return out

    # ------------------------------------------------------------------ bytes
    def step_bytes(self, summaries: np.ndarray) -> StepBytes:
        """summaries int64 [L][5] as read back from the plans."""
        L, T, k, E = self.L, self.T, self.k, self.E
        b = StepBytes()
        b.stats = L * T * k * 4 + (2 * L + max(L - 1, 0)) * E * E * 4
        if not self.rows:
            return b
        d = self.x.shape[1]
        rowB = d * self.x.element_size()
        outB = d * torch.tensor([], dtype=self.out_dtype).element_size()
        for l in range(L):
            R = int(summaries[l][0])
            src_b = 4 * T if (self.shuffle and l > 0) else 0
            b.plan += T * k * 4 + E * 4 + src_b + 8 * T + 5 * R + 4 * T * k + 8 * self.G * self.G
            if self.replicas:   # the assignment reads ids, writes pick ranks; the plan reads them back
                b.plan += T * k * 4 + T * k * 4 + 4 * T + T * k * 4
            b.permute += T * rowB + R * rowB + 4 * T * k
            if self.prereduce:
                # gates: row_token + jmask read, (e, w) gathered and written per row slot
                b.gates += 5 * R + 8 * T * k + 8 * R * k
                b.reduce += R * rowB + R * rowB + 8 * R * k + 4 * self.E
                b.combine += R * rowB + T * outB + 4 * T * k
            else:
                b.combine += R * rowB + T * outB + 8 * T * k
            if self.shuffle and l + 1 < L:
                b.shuffle += T * k * 4 + E * self.G * 4 + 4 * T
        return b

    def summaries(self) -> np.ndarray:
        return torch.stack([p.summary for p in self.plans]).cpu().numpy()


def calibrate(ids_cal: torch.Tensor, E: int, G: int, rpn: int, placement: str, shuffle: bool,
              replica_extra: int = 0, load_tolerance: float = 0.1):
    """Placements and rank-score tables from a calibration batch (int32
    [L][T][k] on the device): its statistics come from moe_coact_stats, the
    placement from the host greedy, the tables from moe_rank_score.
    Returns (list of e2r int32 [E] device tensors, list of rank_score uint32
    [E][G] device tensors, host coact of the calibration batch)."""
    L = ids_cal.shape[0]
    st = cap.coact_stats(ids_cal, E, want=("coact", "trans"))
    torch.cuda.current_stream(ids_cal.device).synchronize()
    if int(st["err"].item()):
        raise ValueError("calibration batch has invalid ids (device code %d)" % int(st["err"].item()))
    coact_h = st["coact"].cpu().numpy()
    if placement == "uniform":
        e2r_h = [cap.place_uniform(E, G) for _ in range(L)]
    elif placement == "correlated":
        e2r_h = [cap.place_correlated(coact_h[l], G, rpn) for l in range(L)]
    elif placement == "capped":
        # correlated grouping with every rank's load within (1 + tolerance) x the average
        e2r_h = [cap.place_correlated_capped(coact_h[l], G, rpn, load_tolerance) for l in range(L)]
    elif placement == "capacity":
        # first-fit decreasing on the calibration loads n_e = C_ee
        e2r_h = [cap.place_capacity(np.diag(coact_h[l]).astype(np.float64), G)[0] for l in range(L)]
    else:
        raise ValueError("placement must be uniform, correlated, capped or capacity")
    e2r = [torch.from_numpy(a).to(ids_cal.device) for a in e2r_h]
    rs = []
    if shuffle:
        for l in range(L - 1):
            rs.append(cap.rank_score(st["trans"][l], e2r[l + 1], G))
    reps = []
    if replica_extra > 0:
        for l in range(L):
            rr, nr = cap.place_replicas(coact_h[l], G, rpn, e2r_h[l], replica_extra)
            reps.append((torch.from_numpy(rr).to(ids_cal.device), torch.from_numpy(nr).to(ids_cal.device)))
    return e2r, rs, coact_h, reps


def prepare(E: int, G: int, rpn: int, ids: np.ndarray, gates: Optional[np.ndarray], x: Optional[np.ndarray],
            x_dtype: str, ids_cal: np.ndarray, placement: str = "correlated", shuffle: bool = True,
            out_dtype=torch.bfloat16, device="cuda", rows: bool = True, timers: bool = False,
            scales: Optional[np.ndarray] = None, replica_extra: int = 0, shuffle_capacity: int = 0,
            overlap: bool = True, replica_eps: Optional[float] = None, schedule: Optional[str] = None,
            row_chunks: int = 1) -> HotPath:
    """Upload a batch (host numpy arrays; x as float32 or bf16 bit patterns)
    and its calibration batch, calibrate, and return the step's HotPath."""
    dev = torch.device(device)
    ids_d = torch.from_numpy(np.ascontiguousarray(ids, dtype=np.int32)).to(dev)
    cal_d = torch.from_numpy(np.ascontiguousarray(ids_cal, dtype=np.int32)).to(dev)
    e2r, rs, _, reps = calibrate(cal_d, E, G, rpn, placement, shuffle and ids.shape[0] > 1, replica_extra) \
        if rows else ([], [], None, [])
    gates_d = torch.from_numpy(np.ascontiguousarray(gates, dtype=np.float32)).to(dev) if rows else None
    if rows:
        x_d = (bf16_from_bits(x) if x_dtype == "bf16" else torch.from_numpy(np.ascontiguousarray(x, np.float32))).to(dev)
    else:
        x_d = None
    scales_d = [torch.from_numpy(np.ascontiguousarray(s_, dtype=np.float32)).to(dev) for s_ in scales] \
        if scales is not None else []
    return HotPath(E=E, G=G, rpn=rpn, ids=ids_d, gates=gates_d, x=x_d, e2r=e2r, rank_scores=rs,
                   out_dtype=out_dtype, rows=rows, timers=timers, prereduce=scales is not None, scales=scales_d,
                   replicas=reps, shuffle_capacity=shuffle_capacity, overlap=overlap, schedule=schedule,
                   row_chunks=row_chunks,
                   replica_eps=replica_eps if replica_extra > 0 else None)


def placement_effect(ids: torch.Tensor, ids_cal: torch.Tensor, E: int, G: int, rpn: int,
                     placement: str = "correlated", loads: bool = False):
    """What a placement does to a batch without hidden states: the placement
    is computed from the calibration batch (as calibrate() does), then every
    layer's dispatch plan of the evaluation batch (contiguous shards of T/G
    tokens) is built on the device.  Returns int64 [L][5]: R, R_remote, local,
    V, T*k per layer (local share = local / (T*k), V per token = V / T).
    With loads=True also returns float64 [L][G]: the token-expert
    assignments each rank serves in the evaluation batch (sum of n_e = C_ee
    over its experts)."""
    e2r, _, _, _ = calibrate(ids_cal, E, G, rpn, placement, False)
    L, T, k = ids.shape
    ws = torch.empty(max(cap.plan_dispatch_workspace(T, k, G, False), 1), dtype=torch.uint8, device=ids.device)
    plan = cap.Plan.empty(T, k, G, ids.device)
    out = []
    for l in range(L):
        p = cap.plan_dispatch(ids[l], E, G, rpn, e2r[l], plan=plan, ws=ws)
        out.append(p.summary.cpu().numpy().copy())
        if int(p.err.item()):
            raise ValueError("device data error %d" % int(p.err.item()))
    if not loads:
        return np.stack(out)
    n = cap.coact_stats(ids, E, want=("coact",))["coact"].cpu().numpy()
    rank_load = np.stack([cap.rank_loads(n[l], e2r[l].cpu().numpy(), G) for l in range(L)]).astype(np.float64)
    return np.stack(out), rank_load


def save_layout(path: str, expert_to_rank, rank_scores=(), replicas=(), stats=None):
    """Write a placement (and what was derived with it) to one .npz file: the
    expert-to-rank map per layer, rank-score tables per layer pair, replica
    tables per layer and, optionally, the statistics they came from.  Accepts
    numpy arrays or tensors (device tensors are copied to the host)."""
    def h(a):
        return a.detach().cpu().numpy() if isinstance(a, torch.Tensor) else np.asarray(a)
    arrays = {"expert_to_rank": np.stack([h(a) for a in expert_to_rank]).astype(np.int32)}
    if len(rank_scores):
        arrays["rank_score"] = np.stack([h(a) for a in rank_scores]).astype(np.uint32)
    if len(replicas):
        arrays["replica_rank"] = np.stack([h(r) for r, _ in replicas]).astype(np.int32)
        arrays["n_rep"] = np.stack([h(n) for _, n in replicas]).astype(np.int32)
    for k_, v in (stats or {}).items():
        if v is not None:
            arrays["stats_" + k_] = h(v)
    np.savez(path, **arrays)


def load_layout(path: str, device=None) -> dict:
    """Read save_layout's file: lists per layer (tensors on `device` when
    given, else numpy arrays) under the same names, statistics under 'stats'."""
    with np.load(path) as z:
        d = {k_: z[k_] for k_ in z.files}
    conv = (lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(device)) if device is not None else (lambda a: a)
    out = {"expert_to_rank": [conv(a) for a in d["expert_to_rank"]],
           "rank_score": [conv(a) for a in d.get("rank_score", [])],
           "replicas": [(conv(r), conv(n)) for r, n in zip(d.get("replica_rank", []), d.get("n_rep", []))],
           "stats": {k_[6:]: d[k_] for k_ in d if k_.startswith("stats_")}}
    return out
