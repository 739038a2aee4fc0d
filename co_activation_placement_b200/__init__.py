"""Co-activation statistics and deduplicated expert-parallel dispatch on B200.

Python binding of libmoecoact.so (C ABI in include/moe_coact.h).  Every
function here only marshals torch tensors into pointers and sizes and enqueues
the library's sm_100a kernels on torch's current CUDA stream; no step of the
path is computed in Python or by torch.  If the shared library is missing the
import of any entry point raises: there is no fallback.

Entry points (names follow the C ABI without the ``moe_`` prefix):
  coact_stats, coact_stats_method, coact_stats_path, coact_ema,
  plan_dispatch, plan_sources, plan_dispatch_method, permute, combine, rank_score, shuffle_targets, shuffle_balanced,
  dispatch_gates, expert_reduce, combine_rows,
  place_replicas, assign_replicas, assign_replicas_capped, plan_dispatch_ranks,
  ep_routes, ep_permute, ep_combine, ep_scatter_rows, ep_exchange_rows (ranks over several devices),
  place_uniform, place_capacity, place_correlated, place_correlated_capped, rank_loads,
  cooperative_blocks, selftest_wait_timeout, launch_count.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from typing import Optional

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoecoact.so")

MOE_OK, MOE_ERR_ARG, MOE_ERR_DATA, MOE_ERR_WORKSPACE, MOE_ERR_CUDA, MOE_ERR_UNSUPPORTED = range(6)
DERR_ID_RANGE, DERR_ID_REPEAT, DERR_RANK_RANGE, DERR_ROW_RANGE, DERR_TIMEOUT = 1, 2, 3, 4, 5
MOE_F32, MOE_BF16 = 0, 1

_lib = None


class MoeError(RuntimeError):
    def __init__(self, fn: str, status: int):
        msg = lib().moe_status_string(status).decode() if _lib is not None else str(status)
        super().__init__("%s: %s (status %d)" % (fn, msg, status))
        self.status = status


class _Plan(ctypes.Structure):
    _fields_ = [("dest_mask", ctypes.c_void_p), ("counts", ctypes.c_void_p), ("offsets", ctypes.c_void_p),
                ("row_token", ctypes.c_void_p), ("row_jmask", ctypes.c_void_p), ("row_of", ctypes.c_void_p),
                ("summary", ctypes.c_void_p)]


def lib() -> ctypes.CDLL:
    """Load libmoecoact.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError("libmoecoact.so is not built (run python -m co_activation_placement_b200.build)")
        L = ctypes.CDLL(LIB_PATH)
        P, i, i64, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t
        sigs = {
            "moe_status_string": ([i], ctypes.c_char_p),
            "moe_launch_count": ([], ctypes.c_uint64),
            "moe_coact_stats_workspace": ([i, i, i, i, i], sz),
            "moe_coact_stats_method": ([i], i),
            "moe_coact_stats_path": ([i, i, i, i, i], i),
            "moe_coact_ema": ([P, i, i, ctypes.c_double, P, P, P, P], i),
            "moe_selftest_workspace": ([], sz),
            "moe_selftest_wait_timeout": ([i, P, P, sz, P], i),
            "moe_coact_stats": ([P, i, i, i, i, P, P, P, P, P, sz, P], i),
            "moe_plan_dispatch_workspace": ([i, i, i, i], sz),
            "moe_plan_dispatch_method": ([i], i),
            "moe_cooperative_blocks": ([i], i),
            "moe_plan_dispatch": ([P, i, i, i, i, i, P, P, ctypes.POINTER(_Plan), P, P, sz, P], i),
            "moe_plan_sources": ([P, i, i, P, P, sz, P], i),
            "moe_plan_dispatch_presorted": ([P, i, i, i, i, i, P, P, ctypes.POINTER(_Plan), P, P, sz, P], i),
            "moe_permute": ([P, i, i, i, i, P, i64, P, P, P], i),
            "moe_combine": ([P, i, i64, i, P, P, i, i, P, i, P, P], i),
            "moe_dispatch_gates": ([P, P, i, i, P, P, P, i64, P, P, P, P], i),
            "moe_expert_reduce": ([P, i, i64, i, P, P, P, i, P, i, P, i, P, P], i),
            "moe_combine_rows": ([P, i, i64, i, P, i, i, P, i, P, P], i),
            "moe_rank_score": ([P, P, i, i, P, P, P], i),
            "moe_shuffle_targets": ([P, i, i, i, i, P, P, P, P], i),
            "moe_shuffle_balanced_workspace": ([i, i, i], sz),
            "moe_shuffle_balanced": ([P, i, i, i, i, P, i, P, P, P, sz, P, P], i),
            "moe_place_uniform": ([i, i, P], i),
            "moe_place_capacity": ([P, i, i, P, P], i),
            "moe_place_correlated": ([P, i, i, i, P], i),
            "moe_place_correlated_capped": ([P, i, i, i, ctypes.c_double, P], i),
            "moe_place_replicas": ([P, i, i, i, P, i, P, P], i),
            "moe_assign_replicas": ([P, i, i, i, i, i, P, P, P, P, P, P, P], i),
            "moe_assign_replicas_capped_workspace": ([i], sz),
            "moe_assign_replicas_capped": ([P, i, i, i, i, i, P, P, P, ctypes.c_double, P, P, P, P, P, sz, P], i),
            "moe_rank_loads": ([P, i, i, P, P], i),
            "moe_ep_exchange_rows": ([P, i, i, P, P], i),
            "moe_plan_dispatch_ranks": ([P, i, i, i, i, i, P, P, ctypes.POINTER(_Plan), P, P, sz, P], i),
            "moe_ep_routes": ([P, P, i, i, i, P, P, P], i),
            "moe_ep_permute": ([P, i, i, i, i, P, i64, P, i, i, P, i64, P, P], i),
            "moe_ep_combine": ([P, i, i64, i, P, i, i, i64, P, P, i, i, P, i, P, P], i),
            "moe_ep_scatter_rows": ([P, i64, i64, P, i, i, P, i64, P, P], i),
        }
        for name, (args, res) in sigs.items():
            f = getattr(L, name)
            f.argtypes = args
            f.restype = res
        _lib = L
    return _lib


def launch_count() -> int:
    return int(lib().moe_launch_count())


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(t: torch.Tensor):
    return ctypes.c_void_p(torch.cuda.current_stream(t.device).cuda_stream)


def _check(fn: str, st: int):
    if st != MOE_OK:
        raise MoeError(fn, st)


def _dev(t: torch.Tensor, dtype, name: str, ndim: Optional[int] = None):
    if not t.is_cuda:
        raise ValueError("%s must be a CUDA tensor" % name)
    if t.dtype != dtype:
        raise ValueError("%s must be %s, got %s" % (name, dtype, t.dtype))
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous" % name)
    if ndim is not None and t.dim() != ndim:
        raise ValueError("%s must have %d dims" % (name, ndim))
    return t


def _need(cond: bool, what: str):
    """Shape agreement between the tensors of one call (checked before anything is enqueued)."""
    if not cond:
        raise ValueError(what)


class Workspace:
    """A growable device byte buffer, 256-byte aligned (torch allocations are)."""

    def __init__(self, device):
        self.device = torch.device(device)
        self.buf = torch.empty(0, dtype=torch.uint8, device=self.device)

    def get(self, nbytes: int) -> torch.Tensor:
        if self.buf.numel() < nbytes:
            self.buf = torch.empty(max(nbytes, 1), dtype=torch.uint8, device=self.device)
        return self.buf


_ws = {}


def _workspace(device, slot: str) -> Workspace:
    key = (str(torch.device(device)), slot)
    if key not in _ws:
        _ws[key] = Workspace(device)
    return _ws[key]


def new_err(device) -> torch.Tensor:
    return torch.zeros(1, dtype=torch.int32, device=device)


# ---------------------------------------------------------------- statistics

def coact_stats_method(method: int) -> int:
    """0 = choose per call, 1 = shared-memory histograms, 2 = tensor cores
    where the shape allows; returns the previous setting (process-wide)."""
    prev = int(lib().moe_coact_stats_method(int(method)))
    if prev < 0:
        raise ValueError("method must be 0, 1 or 2")
    return prev


def coact_stats_path(L: int, T: int, k: int, E: int, with_trans: bool = True) -> str:
    """'tensor' or 'histogram': the method moe_coact_stats would use now."""
    return {1: "histogram", 2: "tensor"}.get(int(lib().moe_coact_stats_path(L, T, k, E, int(bool(with_trans)))), "none")


def coact_stats_workspace(L: int, T: int, k: int, E: int, with_trans: bool = True) -> int:
    return int(lib().moe_coact_stats_workspace(L, T, k, E, int(bool(with_trans))))


def coact_stats(ids: torch.Tensor, E: int, coact=None, ochiai=None, trans=None, err=None,
                want=("coact", "ochiai", "trans"), ws: Optional[torch.Tensor] = None):
    """ids int32 [L][T][k] -> dict(coact uint32 [L][E][E], ochiai f32 [L][E][E], trans uint32 [L-1][E][E], err)."""
    _dev(ids, torch.int32, "ids", 3)
    L, T, k = ids.shape
    dev = ids.device
    if coact is None and "coact" in want:
        coact = torch.empty((L, E, E), dtype=torch.uint32, device=dev)
    if ochiai is None and "ochiai" in want:
        ochiai = torch.empty((L, E, E), dtype=torch.float32, device=dev)
    if trans is None and "trans" in want and L > 1:
        trans = torch.empty((L - 1, E, E), dtype=torch.uint32, device=dev)
    err = new_err(dev) if err is None else err
    need = coact_stats_workspace(L, T, k, E, trans is not None)
    if ws is None:
        ws = _workspace(dev, "stats").get(need)
    st = lib().moe_coact_stats(_ptr(ids), L, T, k, E, _ptr(coact), _ptr(ochiai), _ptr(trans), _ptr(err),
                               _ptr(ws), ws.numel(), _stream(ids))
    _check("moe_coact_stats", st)
    return dict(coact=coact, ochiai=ochiai, trans=trans, err=err)


def coact_ema(coact: torch.Tensor, alpha: float, ema_in: Optional[torch.Tensor] = None,
              ema_out: Optional[torch.Tensor] = None, ochiai: Optional[torch.Tensor] = None, want_ochiai: bool = True):
    """EMA of co-activation counts (float64 [L][E][E], out of place) and
    Ochiai on it.  ema_in None: the first batch.  Returns (ema_out, ochiai)."""
    _dev(coact, torch.uint32, "coact", 3)
    L, E, _ = coact.shape
    if ema_out is None:
        ema_out = torch.empty((L, E, E), dtype=torch.float64, device=coact.device)
    if ochiai is None and want_ochiai:
        ochiai = torch.empty((L, E, E), dtype=torch.float32, device=coact.device)
    st = lib().moe_coact_ema(_ptr(coact), L, E, float(alpha), _ptr(ema_in), _ptr(ema_out), _ptr(ochiai),
                             _stream(coact))
    _check("moe_coact_ema", st)
    return ema_out, ochiai


def selftest_wait_timeout(kind: int, device="cuda") -> torch.Tensor:
    """Make one kind of bounded device wait run out on purpose (0: a grid
    barrier one block never reaches; 1: an mbarrier phase nothing completes);
    returns the error word (device int32 [1]), MOE_DERR_TIMEOUT when the wait
    gave up as designed."""
    err = new_err(device)
    ws = torch.empty(max(int(lib().moe_selftest_workspace()), 1), dtype=torch.uint8, device=device)
    _check("moe_selftest_wait_timeout", lib().moe_selftest_wait_timeout(int(kind), _ptr(err), _ptr(ws), ws.numel(),
                                                                        _stream(err)))
    return err


# ---------------------------------------------------------------- dispatch plan

@dataclass
class Plan:
    dest_mask: torch.Tensor   # uint64 [T]
    counts: torch.Tensor      # int32 [G][G]
    offsets: torch.Tensor     # int32 [G*G+1]
    row_token: torch.Tensor   # int32 [T*k]
    row_jmask: torch.Tensor   # uint8 [T*k]
    row_of: torch.Tensor      # int32 [T][k]
    summary: torch.Tensor     # int64 [5]
    err: torch.Tensor         # int32 [1]
    T: int
    k: int
    G: int

    @property
    def R_max(self) -> int:
        return self.T * self.k

    @staticmethod
    def empty(T: int, k: int, G: int, device) -> "Plan":
        n = max(T * k, 1)
        return Plan(dest_mask=torch.empty(max(T, 1), dtype=torch.uint64, device=device),
                    counts=torch.empty((G, G), dtype=torch.int32, device=device),
                    offsets=torch.empty(G * G + 1, dtype=torch.int32, device=device),
                    row_token=torch.empty(n, dtype=torch.int32, device=device),
                    row_jmask=torch.empty(n, dtype=torch.uint8, device=device),
                    row_of=torch.empty((max(T, 1), k), dtype=torch.int32, device=device),
                    summary=torch.empty(5, dtype=torch.int64, device=device),
                    err=new_err(device), T=T, k=k, G=G)

    def c_struct(self) -> _Plan:
        return _Plan(self.dest_mask.data_ptr(), self.counts.data_ptr(), self.offsets.data_ptr(),
                     self.row_token.data_ptr(), self.row_jmask.data_ptr(), self.row_of.data_ptr(),
                     self.summary.data_ptr())


def plan_dispatch_method(method: int) -> int:
    """0 = separate kernels (default), 1 = one cooperative launch when the
    plan has at most 512 chunks; returns the previous setting (process-wide)."""
    prev = int(lib().moe_plan_dispatch_method(int(method)))
    if prev < 0:
        raise ValueError("method must be 0 or 1")
    return prev


def cooperative_blocks(blocks: int) -> int:
    """Blocks of the cooperative launches (shuffle_balanced,
    assign_replicas_capped): 0 = one per SM (default), n > 0 = n blocks;
    returns the previous setting (process-wide)."""
    prev = int(lib().moe_cooperative_blocks(int(blocks)))
    if prev < 0:
        raise ValueError("blocks must be >= 0")
    return prev


def plan_dispatch_workspace(T: int, k: int, G: int, with_src_rank: bool) -> int:
    return int(lib().moe_plan_dispatch_workspace(T, k, G, int(bool(with_src_rank))))


def plan_sources(src_rank: torch.Tensor, G: int, ws: torch.Tensor, err: torch.Tensor) -> None:
    """The first step of a plan with source ranks (the tokens' order by source
    rank) into ws, ahead of plan_dispatch(..., presorted=True) with the same
    src_rank and ws; err: the plan's device error word."""
    _dev(src_rank, torch.int32, "src_rank", 1)
    _dev(ws, torch.uint8, "ws", 1)
    T = src_rank.shape[0]
    st = lib().moe_plan_sources(_ptr(src_rank), T, G, _ptr(err), _ptr(ws), ws.numel(), _stream(src_rank))
    _check("moe_plan_sources", st)


def plan_dispatch(ids: torch.Tensor, E: int, G: int, rpn: int, expert_to_rank: torch.Tensor,
                  src_rank: Optional[torch.Tensor] = None, plan: Optional[Plan] = None,
                  ws: Optional[torch.Tensor] = None, presorted: bool = False) -> Plan:
    """ids int32 [T][k] (one layer) -> Plan (device tensors; row arrays sized T*k).
    presorted: plan_sources already put src_rank's order into ws."""
    _dev(ids, torch.int32, "ids", 2)
    _dev(expert_to_rank, torch.int32, "expert_to_rank", 1)
    if src_rank is not None:
        _dev(src_rank, torch.int32, "src_rank", 1)
    T, k = ids.shape
    dev = ids.device
    if plan is None:
        plan = Plan.empty(T, k, G, dev)
    need = plan_dispatch_workspace(T, k, G, src_rank is not None)
    if ws is None:
        ws = _workspace(dev, "plan").get(need)
    if presorted and ws is None:
        raise ValueError("a presorted plan needs the workspace plan_sources filled")
    cs = plan.c_struct()
    fn = lib().moe_plan_dispatch_presorted if presorted else lib().moe_plan_dispatch
    st = fn(_ptr(ids), T, k, E, G, rpn, _ptr(expert_to_rank), _ptr(src_rank),
            ctypes.byref(cs), _ptr(plan.err), _ptr(ws), ws.numel(), _stream(ids))
    _check("moe_plan_dispatch_presorted" if presorted else "moe_plan_dispatch", st)
    return plan


def plan_dispatch_ranks(ids: torch.Tensor, E: int, G: int, rpn: int, pick_rank: torch.Tensor,
                        src_rank: Optional[torch.Tensor] = None, plan: Optional[Plan] = None,
                        ws: Optional[torch.Tensor] = None) -> Plan:
    """The dispatch plan with the serving rank of every pick given (replicated experts)."""
    _dev(ids, torch.int32, "ids", 2)
    _dev(pick_rank, torch.int32, "pick_rank", 2)
    if src_rank is not None:
        _dev(src_rank, torch.int32, "src_rank", 1)
    T, k = ids.shape
    dev = ids.device
    if plan is None:
        plan = Plan.empty(T, k, G, dev)
    need = plan_dispatch_workspace(T, k, G, src_rank is not None)
    if ws is None:
        ws = _workspace(dev, "plan").get(need)
    cs = plan.c_struct()
    st = lib().moe_plan_dispatch_ranks(_ptr(ids), T, k, E, G, rpn, _ptr(pick_rank), _ptr(src_rank),
                                       ctypes.byref(cs), _ptr(plan.err), _ptr(ws), ws.numel(), _stream(ids))
    _check("moe_plan_dispatch_ranks", st)
    return plan


def assign_replicas(ids: torch.Tensor, E: int, G: int, rpn: int, replica_rank: torch.Tensor, n_rep: torch.Tensor,
                    src_rank: Optional[torch.Tensor] = None, pick_rank: Optional[torch.Tensor] = None,
                    n_remote: Optional[torch.Tensor] = None, err: Optional[torch.Tensor] = None):
    """(pick_rank int32 [T][k], n_remote int32 [T]): fewest remote nodes per token over the replicas."""
    _dev(ids, torch.int32, "ids", 2)
    _dev(replica_rank, torch.int32, "replica_rank", 2)
    _dev(n_rep, torch.int32, "n_rep", 1)
    T, k = ids.shape
    if pick_rank is None:
        pick_rank = torch.empty((max(T, 1), k), dtype=torch.int32, device=ids.device)
    if n_remote is None:
        n_remote = torch.empty(max(T, 1), dtype=torch.int32, device=ids.device)
    err = new_err(ids.device) if err is None else err
    st = lib().moe_assign_replicas(_ptr(ids), T, k, E, G, rpn, _ptr(replica_rank), _ptr(n_rep), _ptr(src_rank),
                                   _ptr(pick_rank), _ptr(n_remote), _ptr(err), _stream(ids))
    _check("moe_assign_replicas", st)
    return pick_rank, n_remote


def assign_replicas_capped_workspace(G: int) -> int:
    return int(lib().moe_assign_replicas_capped_workspace(G))


def assign_replicas_capped(ids: torch.Tensor, E: int, G: int, rpn: int, replica_rank: torch.Tensor,
                           n_rep: torch.Tensor, eps: float, src_rank: Optional[torch.Tensor] = None,
                           pick_rank: Optional[torch.Tensor] = None, n_remote: Optional[torch.Tensor] = None,
                           rank_load: Optional[torch.Tensor] = None, err: Optional[torch.Tensor] = None,
                           ws: Optional[torch.Tensor] = None):
    """(pick_rank int32 [T][k], n_remote int32 [T], rank_load int64 [G]): the
    fewest-remote-nodes assignment with each rank's tasks capped at
    floor((1 + eps) T k / G), tokens taken in id order."""
    _dev(ids, torch.int32, "ids", 2)
    _dev(replica_rank, torch.int32, "replica_rank", 2)
    _dev(n_rep, torch.int32, "n_rep", 1)
    T, k = ids.shape
    dev = ids.device
    if pick_rank is None:
        pick_rank = torch.empty((max(T, 1), k), dtype=torch.int32, device=dev)
    if n_remote is None:
        n_remote = torch.empty(max(T, 1), dtype=torch.int32, device=dev)
    if rank_load is None:
        rank_load = torch.empty(G, dtype=torch.int64, device=dev)
    err = new_err(dev) if err is None else err
    need = int(lib().moe_assign_replicas_capped_workspace(G))
    if ws is None:
        ws = _workspace(dev, "capped").get(need)
    st = lib().moe_assign_replicas_capped(_ptr(ids), T, k, E, G, rpn, _ptr(replica_rank), _ptr(n_rep),
                                          _ptr(src_rank), float(eps), _ptr(pick_rank), _ptr(n_remote),
                                          _ptr(rank_load), _ptr(err), _ptr(ws), ws.numel(), _stream(ids))
    _check("moe_assign_replicas_capped", st)
    return pick_rank, n_remote, rank_load


# ---------------------------------------------------------------- rows

def _dtype_code(dt) -> int:
    if dt == torch.float32:
        return MOE_F32
    if dt == torch.bfloat16:
        return MOE_BF16
    raise ValueError("dtype must be float32 or bfloat16")


def permute(x: torch.Tensor, row_of: torch.Tensor, R_max: int, send: Optional[torch.Tensor] = None,
            err: Optional[torch.Tensor] = None) -> torch.Tensor:
    """send[row_of[t][j]] = x[t]; send is [R_max][d] (rows >= R untouched)."""
    if x.dim() != 2:
        raise ValueError("x must be [T][d]")
    _dev(x, x.dtype, "x")
    _dev(row_of, torch.int32, "row_of", 2)
    T, d = x.shape
    k = row_of.shape[1]
    _need(row_of.shape[0] >= T, "row_of needs a row per token of x")
    if send is None:
        send = torch.empty((max(R_max, 1), d), dtype=x.dtype, device=x.device)
    _need(send.dim() == 2 and send.shape[0] >= R_max and send.shape[1] == d and send.dtype == x.dtype
          and send.is_contiguous(), "send must be a contiguous [R_max][d] tensor of x's dtype")
    err = new_err(x.device) if err is None else err
    st = lib().moe_permute(_ptr(x), _dtype_code(x.dtype), T, d, k, _ptr(row_of), R_max, _ptr(send), _ptr(err),
                           _stream(x))
    _check("moe_permute", st)
    return send


def combine(Y: torch.Tensor, idx: torch.Tensor, w: torch.Tensor, out_dtype=torch.float32,
            out: Optional[torch.Tensor] = None, err: Optional[torch.Tensor] = None) -> torch.Tensor:
    """out[t] = sum_j w[t][j] * Y[idx[t][j]] (fp32 FMA accumulation; out fp32 or bf16)."""
    _dev(Y, Y.dtype, "Y", 2)
    _dev(idx, torch.int32, "idx", 2)
    _dev(w, torch.float32, "w", 2)
    T, k = idx.shape
    R_max, d = Y.shape
    _need(w.shape[0] >= T and w.shape[1] == k, "w needs a weight per (token, pick) of idx")
    if out is None:
        out = torch.empty((T, d), dtype=out_dtype, device=Y.device)
    _need(out.dim() == 2 and out.shape[0] >= T and out.shape[1] == d and out.is_contiguous(),
          "out must be a contiguous [T][d] tensor")
    err = new_err(Y.device) if err is None else err
    st = lib().moe_combine(_ptr(Y), _dtype_code(Y.dtype), R_max, d, _ptr(idx), _ptr(w), T, k, _ptr(out),
                           _dtype_code(out.dtype), _ptr(err), _stream(Y))
    _check("moe_combine", st)
    return out


# ---------------------------------------------------------------- receiver-side pre-reduced combine

def dispatch_gates(ids: torch.Tensor, w: torch.Tensor, plan: Plan, send_e: Optional[torch.Tensor] = None,
                   send_w: Optional[torch.Tensor] = None, err: Optional[torch.Tensor] = None):
    """(send_e int32 [R_max][k], send_w f32 [R_max][k]) for the plan's rows (rows >= R untouched)."""
    _dev(ids, torch.int32, "ids", 2)
    _dev(w, torch.float32, "w", 2)
    T, k = ids.shape
    R_max = plan.R_max
    _need(w.shape[0] >= T and w.shape[1] == k, "w needs a weight per (token, pick) of ids")
    if send_e is None:
        send_e = torch.empty((max(R_max, 1), k), dtype=torch.int32, device=ids.device)
    if send_w is None:
        send_w = torch.empty((max(R_max, 1), k), dtype=torch.float32, device=ids.device)
    err = plan.err if err is None else err
    st = lib().moe_dispatch_gates(_ptr(ids), _ptr(w), T, k, _ptr(plan.row_token), _ptr(plan.row_jmask),
                                  _ptr(plan.summary), R_max, _ptr(send_e), _ptr(send_w), _ptr(err), _stream(ids))
    _check("moe_dispatch_gates", st)
    return send_e, send_w


def expert_reduce(send: torch.Tensor, summary: torch.Tensor, send_e: torch.Tensor, send_w: torch.Tensor,
                  scale: torch.Tensor, y_dtype=None, y: Optional[torch.Tensor] = None,
                  err: Optional[torch.Tensor] = None) -> torch.Tensor:
    """y[i] = sum_j send_w[i][j] * scale[send_e[i][j]] * send[i] for the rows i < summary[0]."""
    _dev(send, send.dtype, "send", 2)
    _dev(send_e, torch.int32, "send_e", 2)
    _dev(send_w, torch.float32, "send_w", 2)
    _dev(scale, torch.float32, "scale", 1)
    R_max, d = send.shape
    k = send_e.shape[1]
    _need(send_e.shape[0] >= R_max and tuple(send_w.shape) == tuple(send_e.shape),
          "send_e and send_w need k entries per row of send")
    if y is None:
        y = torch.empty((R_max, d), dtype=y_dtype or send.dtype, device=send.device)
    _need(y.dim() == 2 and y.shape[0] >= R_max and y.shape[1] == d and y.is_contiguous(),
          "y must be a contiguous [R_max][d] tensor")
    err = new_err(send.device) if err is None else err
    st = lib().moe_expert_reduce(_ptr(send), _dtype_code(send.dtype), R_max, d, _ptr(summary), _ptr(send_e),
                                 _ptr(send_w), k, _ptr(scale), scale.numel(), _ptr(y), _dtype_code(y.dtype),
                                 _ptr(err), _stream(send))
    _check("moe_expert_reduce", st)
    return y


def combine_rows(Y: torch.Tensor, row_of: torch.Tensor, out_dtype=torch.float32, out: Optional[torch.Tensor] = None,
                 err: Optional[torch.Tensor] = None) -> torch.Tensor:
    """out[t] = sum of the distinct rows {row_of[t][j]} of Y, each once."""
    _dev(Y, Y.dtype, "Y", 2)
    _dev(row_of, torch.int32, "row_of", 2)
    T, k = row_of.shape
    R_max, d = Y.shape
    if out is None:
        out = torch.empty((T, d), dtype=out_dtype, device=Y.device)
    _need(out.dim() == 2 and out.shape[0] >= T and out.shape[1] == d and out.is_contiguous(),
          "out must be a contiguous [T][d] tensor")
    err = new_err(Y.device) if err is None else err
    st = lib().moe_combine_rows(_ptr(Y), _dtype_code(Y.dtype), R_max, d, _ptr(row_of), T, k, _ptr(out),
                                _dtype_code(out.dtype), _ptr(err), _stream(Y))
    _check("moe_combine_rows", st)
    return out


# ---------------------------------------------------------------- several devices

def ep_route_len(G: int, W: int) -> int:
    """Entries (int64) of a route table for G ranks over W devices."""
    return 2 * G * (G // W) + 2


def ep_routes(counts_all: torch.Tensor, offsets: torch.Tensor, G: int, W: int, me: int,
              route: Optional[torch.Tensor] = None, err: Optional[torch.Tensor] = None) -> torch.Tensor:
    """route int64 [2*G*(G/W) + 2]: where this device's rows land in the receiving devices' buffers."""
    _dev(counts_all, torch.int32, "counts_all", 2)
    _dev(offsets, torch.int32, "offsets", 1)
    if route is None:
        route = torch.empty(ep_route_len(G, W), dtype=torch.int64, device=counts_all.device)
    err = new_err(counts_all.device) if err is None else err
    st = lib().moe_ep_routes(_ptr(counts_all), _ptr(offsets), G, W, me, _ptr(route), _ptr(err), _stream(counts_all))
    _check("moe_ep_routes", st)
    return route


def ep_permute(x: torch.Tensor, row_of: torch.Tensor, R_max: int, route: torch.Tensor, G: int, W: int,
               recv_base: torch.Tensor, recv_cap: int, err: Optional[torch.Tensor] = None):
    """Store every local row x[t] into its receiving device's buffer (recv_base: int64 [W] addresses)."""
    _dev(x, x.dtype, "x", 2)
    _dev(row_of, torch.int32, "row_of", 2)
    _dev(route, torch.int64, "route", 1)
    _dev(recv_base, torch.int64, "recv_base", 1)
    T, d = x.shape
    k = row_of.shape[1]
    _need(row_of.shape[0] >= T, "row_of needs a row per token of x")
    _need(recv_base.numel() == W, "recv_base needs one address per device")
    err = new_err(x.device) if err is None else err
    st = lib().moe_ep_permute(_ptr(x), _dtype_code(x.dtype), T, d, k, _ptr(row_of), R_max, _ptr(route), G, W,
                              _ptr(recv_base), recv_cap, _ptr(err), _stream(x))
    _check("moe_ep_permute", st)


def ep_combine(y_base: torch.Tensor, y_dtype, y_cap: int, d: int, route: torch.Tensor, G: int, W: int,
               R_max: int, idx: torch.Tensor, w: Optional[torch.Tensor], out: torch.Tensor,
               err: Optional[torch.Tensor] = None) -> torch.Tensor:
    """out[t] = sum_j w[t][j] * Y[idx[t][j]] (w None: distinct rows once), rows read from the devices' buffers."""
    _dev(y_base, torch.int64, "y_base", 1)
    _dev(route, torch.int64, "route", 1)
    _dev(idx, torch.int32, "idx", 2)
    if w is not None:
        _dev(w, torch.float32, "w", 2)
    _dev(out, out.dtype, "out", 2)
    T, k = idx.shape
    _need(w is None or (w.shape[0] >= T and w.shape[1] == k), "w needs a weight per (token, pick) of idx")
    _need(out.shape[0] >= T and out.shape[1] == d, "out must be a [T][d] tensor")
    _need(y_base.numel() == W, "y_base needs one address per device")
    err = new_err(out.device) if err is None else err
    st = lib().moe_ep_combine(_ptr(y_base), _dtype_code(y_dtype), y_cap, d, _ptr(route), G, W, R_max, _ptr(idx),
                              _ptr(w), T, k, _ptr(out), _dtype_code(out.dtype), _ptr(err), _stream(out))
    _check("moe_ep_combine", st)
    return out


def ep_scatter_rows(src: torch.Tensor, route: torch.Tensor, G: int, W: int, dst_base: torch.Tensor, dst_cap: int,
                    err: Optional[torch.Tensor] = None):
    """Per-row records src [R_max][...] (4-byte elements) stored to the receiving devices' buffers."""
    _dev(src, src.dtype, "src")
    _dev(route, torch.int64, "route", 1)
    _dev(dst_base, torch.int64, "dst_base", 1)
    R_max = src.shape[0]
    row_bytes = src[0].numel() * src.element_size() if R_max else 4
    _need(dst_base.numel() == W, "dst_base needs one address per device")
    err = new_err(src.device) if err is None else err
    st = lib().moe_ep_scatter_rows(_ptr(src), row_bytes, R_max, _ptr(route), G, W, _ptr(dst_base), dst_cap,
                                   _ptr(err), _stream(src))
    _check("moe_ep_scatter_rows", st)


# ---------------------------------------------------------------- token shuffle

def rank_score(trans_l: torch.Tensor, next_expert_to_rank: torch.Tensor, G: int,
               out: Optional[torch.Tensor] = None, err: Optional[torch.Tensor] = None) -> torch.Tensor:
    _dev(trans_l, torch.uint32, "trans_l", 2)
    _dev(next_expert_to_rank, torch.int32, "next_expert_to_rank", 1)
    E = trans_l.shape[0]
    if out is None:
        out = torch.empty((E, G), dtype=torch.uint32, device=trans_l.device)
    err = new_err(trans_l.device) if err is None else err
    st = lib().moe_rank_score(_ptr(trans_l), _ptr(next_expert_to_rank), E, G, _ptr(out), _ptr(err), _stream(trans_l))
    _check("moe_rank_score", st)
    return out


def shuffle_targets(ids: torch.Tensor, E: int, G: int, rank_score_tab: torch.Tensor,
                    target: Optional[torch.Tensor] = None, err: Optional[torch.Tensor] = None) -> torch.Tensor:
    _dev(ids, torch.int32, "ids", 2)
    _dev(rank_score_tab, torch.uint32, "rank_score", 2)
    T, k = ids.shape
    if target is None:
        target = torch.empty(max(T, 1), dtype=torch.int32, device=ids.device)
    err = new_err(ids.device) if err is None else err
    st = lib().moe_shuffle_targets(_ptr(ids), T, k, E, G, _ptr(rank_score_tab), _ptr(target), _ptr(err), _stream(ids))
    _check("moe_shuffle_targets", st)
    return target


def shuffle_balanced_workspace(T: int, G: int, capacity: int) -> int:
    return int(lib().moe_shuffle_balanced_workspace(T, G, capacity))


def shuffle_balanced(ids: torch.Tensor, E: int, G: int, rank_score_tab: torch.Tensor, capacity: int,
                     target: Optional[torch.Tensor] = None, info: Optional[torch.Tensor] = None,
                     err: Optional[torch.Tensor] = None, ws: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Shuffle targets with at most `capacity` tokens per rank (the unique
    stable assignment under score desc, token asc, rank asc).  `info`, when
    given (device int64 [6]), receives the rounds taken, the proposals made
    and the nanoseconds spent proposing, gathering, selecting (slowest block)
    and waiting at barriers."""
    _dev(ids, torch.int32, "ids", 2)
    _dev(rank_score_tab, torch.uint32, "rank_score", 2)
    T, k = ids.shape
    if target is None:
        target = torch.empty(max(T, 1), dtype=torch.int32, device=ids.device)
    err = new_err(ids.device) if err is None else err
    need = shuffle_balanced_workspace(T, G, capacity)
    if ws is None:
        ws = _workspace(ids.device, "shuffle").get(need)
    st = lib().moe_shuffle_balanced(_ptr(ids), T, k, E, G, _ptr(rank_score_tab), int(capacity), _ptr(target),
                                    _ptr(info) if info is not None else None, _ptr(ws), ws.numel(), _ptr(err),
                                    _stream(ids))
    _check("moe_shuffle_balanced", st)
    return target


# ---------------------------------------------------------------- placement (host)

def _np_ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def place_uniform(E: int, G: int) -> np.ndarray:
    out = np.empty(E, np.int32)
    _check("moe_place_uniform", lib().moe_place_uniform(E, G, _np_ptr(out)))
    return out


def place_capacity(load, G: int):
    load = np.ascontiguousarray(load, dtype=np.float64)
    out = np.empty(load.size, np.int32)
    dev = np.empty(G, np.float64)
    _check("moe_place_capacity", lib().moe_place_capacity(_np_ptr(load), load.size, G, _np_ptr(out), _np_ptr(dev)))
    return out, dev


def ep_exchange_rows(counts_all, G: int, W: int):
    """(sent int64 [W], received int64 [W]): rows that cross devices when the
    G ranks are spread over W devices, from host counts int32 [G][G]."""
    c = np.ascontiguousarray(counts_all, dtype=np.int32)
    sent = np.empty(W, np.int64)
    recv = np.empty(W, np.int64)
    _check("moe_ep_exchange_rows", lib().moe_ep_exchange_rows(_np_ptr(c), G, W, _np_ptr(sent), _np_ptr(recv)))
    return sent, recv


def rank_loads(coact_l, expert_to_rank, G: int) -> np.ndarray:
    """int64 [G]: tasks each rank serves under a one-replica placement (the
    sum of n_e = C_ee over its experts), from host arrays."""
    c = np.ascontiguousarray(coact_l, dtype=np.uint32)
    E = c.shape[0]
    e2r = np.ascontiguousarray(expert_to_rank, dtype=np.int32)
    out = np.empty(G, np.int64)
    _check("moe_rank_loads", lib().moe_rank_loads(_np_ptr(c), E, G, _np_ptr(e2r), _np_ptr(out)))
    return out


def place_correlated(coact_l, G: int, rpn: int) -> np.ndarray:
    c = np.ascontiguousarray(coact_l, dtype=np.uint32)
    E = c.shape[0]
    out = np.empty(E, np.int32)
    _check("moe_place_correlated", lib().moe_place_correlated(_np_ptr(c), E, G, rpn, _np_ptr(out)))
    return out


def place_correlated_capped(coact_l: np.ndarray, G: int, rpn: int, eps: float) -> np.ndarray:
    """Correlated placement with load tolerance eps (eps < 0: none)."""
    c = np.ascontiguousarray(coact_l, dtype=np.uint32)
    E = c.shape[0]
    out = np.empty(E, np.int32)
    _check("moe_place_correlated_capped", lib().moe_place_correlated_capped(_np_ptr(c), E, G, rpn, float(eps),
                                                                           _np_ptr(out)))
    return out


def place_replicas(coact_l, G: int, rpn: int, expert_to_rank, extra: int):
    """(replica_rank int32 [E][1 + G/rpn], n_rep int32 [E]) on the host."""
    c = np.ascontiguousarray(coact_l, dtype=np.uint32)
    E = c.shape[0]
    e2r = np.ascontiguousarray(expert_to_rank, dtype=np.int32)
    rr = np.empty((E, 1 + G // rpn), np.int32)
    nr = np.empty(E, np.int32)
    _check("moe_place_replicas", lib().moe_place_replicas(_np_ptr(c), E, G, rpn, _np_ptr(e2r), extra,
                                                          _np_ptr(rr), _np_ptr(nr)))
    return rr, nr
