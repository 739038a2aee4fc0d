"""Single library calls on seeded workload inputs, for kernel profiles.

    python -m co_activation_placement_b200.cases CASE [--workload W] [--tokens T] [--reps N]

Each case builds its inputs with the workload generators (synth), runs one
library entry point ``--reps`` times on the current CUDA device (the first
call warms up; a profiler skips it with ``-s``) and synchronises.  Only what
the call needs is allocated, so a capture of one kernel holds a few GB of
device memory at most: the row cases take the first ``--tokens`` tokens of
the workload (default: all of them when the rows fit in 4 GB, else as many
as do).  Placements and rank-score tables come from the workload's
calibration batch, as in the step.  Nothing is checked here: the tests
compare every call with the oracle.

Cases: stats, plan, plan_src, plan_single, plan_single_src, shuffle,
balanced, assign, assign_capped, ema, rows, prereduce, ep.
"""
from __future__ import annotations

import argparse
import os
import sys

import numpy as np
import torch

_ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if _ROOT not in sys.path:
    sys.path.insert(0, _ROOT)

import co_activation_placement_b200 as cap  # noqa: E402
from co_activation_placement_b200 import pipeline  # noqa: E402
from synth import WORKLOADS, make_routing, make_gates, make_hidden, make_expert_scales  # noqa: E402

CASES = ("stats", "plan", "plan_src", "plan_single", "plan_single_src", "shuffle", "balanced", "assign",
         "assign_capped", "ema", "rows", "prereduce", "ep")


def _tokens_for_rows(w, limit_bytes=4 << 30):
    """Tokens whose worst-case send buffer (T k rows) and input fit the limit."""
    rowB = w.d * (2 if w.dtype == "bf16" else 4)
    per_token = (w.k + 1) * rowB + w.d * 4
    t = min(w.T, limit_bytes // per_token)
    return max(w.G, t // w.G * w.G)


def run(case: str, workload: str, tokens: int, reps: int, eps: float, W: int, coact_method: int = 0) -> None:
    w = WORKLOADS[workload]
    cap.coact_stats_method(coact_method)
    dev = torch.device("cuda")
    rows = case in ("rows", "prereduce", "ep")
    T = tokens or (_tokens_for_rows(w) if rows else w.T)
    T = T // w.G * w.G if w.G else T
    ids_h = make_routing(w, T=T)
    ids = torch.from_numpy(ids_h).to(dev)
    L = ids.shape[0]
    cal = torch.from_numpy(make_routing(w, seed=w.seed + 1, T=T)).to(dev)
    if case in ("stats", "ema"):
        st = cap.coact_stats(ids, w.E)
        ema = None
        for _ in range(reps):
            if case == "stats":
                cap.coact_stats(ids, w.E, coact=st["coact"], ochiai=st["ochiai"], trans=st["trans"], err=st["err"])
            else:
                ema, _ = cap.coact_ema(st["coact"], 0.1, ema_in=ema)
        torch.cuda.synchronize()
        return
    e2r, rs, coact_h, reps_ = pipeline.calibrate(cal, w.E, w.G, w.rpn, "correlated", L > 1,
                                                 1 if case.startswith("assign") else 0)
    if case.startswith("plan"):
        single = case.startswith("plan_single")
        src = None
        if case.endswith("src"):
            src = cap.shuffle_targets(ids[0], w.E, w.G, rs[0]) if rs else None
        prev = cap.plan_dispatch_method(1 if single else 0)
        plan = cap.Plan.empty(T, w.k, w.G, dev)
        try:
            for _ in range(reps):
                cap.plan_dispatch(ids[min(1, L - 1)], w.E, w.G, w.rpn, e2r[min(1, L - 1)], src_rank=src, plan=plan)
        finally:
            cap.plan_dispatch_method(prev)
        torch.cuda.synchronize()
        return
    if case == "shuffle":
        tg = torch.empty(T, dtype=torch.int32, device=dev)
        for _ in range(reps):
            tab = cap.rank_score(cap.coact_stats(cal, w.E, want=("trans",))["trans"][0], e2r[1], w.G)
            cap.shuffle_targets(ids[0], w.E, w.G, tab, target=tg)
        torch.cuda.synchronize()
        return
    if case == "balanced":
        tg = torch.empty(T, dtype=torch.int32, device=dev)
        info = torch.zeros(6, dtype=torch.int64, device=dev)
        for _ in range(reps):
            cap.shuffle_balanced(ids[0], w.E, w.G, rs[0], T // w.G, target=tg, info=info)
        torch.cuda.synchronize()
        return
    if case.startswith("assign"):
        rr, nr = reps_[0]
        for _ in range(reps):
            if case == "assign":
                cap.assign_replicas(ids[0], w.E, w.G, w.rpn, rr, nr)
            else:
                cap.assign_replicas_capped(ids[0], w.E, w.G, w.rpn, rr, nr, eps)
        torch.cuda.synchronize()
        return
    # row cases: the first T tokens of the workload's first layer
    gates = torch.from_numpy(make_gates(w, T=T)).to(dev)
    xh = make_hidden(w, T=T)
    x = pipeline.bf16_from_bits(xh).to(dev) if w.dtype == "bf16" else torch.from_numpy(xh).to(dev)
    if case == "ep":
        from co_activation_placement_b200.ep import EPEmulation
        p = cap.plan_dispatch(ids[0], w.E, w.G, w.rpn, e2r[0])
        off = p.offsets.cpu().numpy().astype(np.int64)
        Gl = w.G // W
        cap_rows = max(int(off[(h + 1) * Gl * w.G] - off[h * Gl * w.G]) for h in range(W)) + 64
        del p
        emu = EPEmulation(W, w.E, w.G, w.rpn, T, w.k, w.d, x.dtype, dev, cap_rows)
        for _ in range(reps):
            emu.step(ids[0], x, gates[0], e2r[0])
        torch.cuda.synchronize()
        return
    p = cap.plan_dispatch(ids[0], w.E, w.G, w.rpn, e2r[0])
    send = torch.empty((T * w.k, w.d), dtype=x.dtype, device=dev)
    out = torch.empty((T, w.d), dtype=torch.float32, device=dev)
    if case == "rows":
        for _ in range(reps):
            cap.permute(x, p.row_of, p.R_max, send=send, err=p.err)
            cap.combine(send, p.row_of, gates[0], out=out, err=p.err)
    else:
        scale = torch.from_numpy(make_expert_scales(w)[0]).to(dev)
        y = torch.empty_like(send)
        for _ in range(reps):
            cap.permute(x, p.row_of, p.R_max, send=send, err=p.err)
            se, sw = cap.dispatch_gates(ids[0], gates[0], p, err=p.err)
            cap.expert_reduce(send, p.summary, se, sw, scale, y=y, err=p.err)
            cap.combine_rows(y, p.row_of, out=out, err=p.err)
    torch.cuda.synchronize()


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("case", choices=CASES)
    ap.add_argument("--workload", default="large_ep64")
    ap.add_argument("--tokens", type=int, default=0, help="tokens (default: the workload's, or what 4 GB of rows hold)")
    ap.add_argument("--reps", type=int, default=3)
    ap.add_argument("--eps", type=float, default=0.1, help="load tolerance of assign_capped")
    ap.add_argument("--devices", type=int, default=4, help="virtual devices of the ep case")
    ap.add_argument("--coact-method", type=int, default=0, choices=[0, 1, 2],
                    help="counting method of the statistics (moe_coact_stats_method)")
    a = ap.parse_args(argv)
    if not torch.cuda.is_available():
        raise SystemExit("needs a CUDA device")
    run(a.case, a.workload, a.tokens, a.reps, a.eps, a.devices, a.coact_method)
    print("case %s on %s: done" % (a.case, a.workload))


if __name__ == "__main__":
    main()
