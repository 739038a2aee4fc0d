"""ORACLE -- test infrastructure only.

numpy front end over ``oracle.c`` (a plain single-threaded C statement of the
path) plus the pure-Python brute force in ``brute.py``.  Only the tests, the
build entry's smoke check and bench.py's CPU-baseline leg may import this
package; the product library never does and shares no code with it.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

OK, ERR_ARG, ERR_DATA = 0, 1, 2


def build(force: bool = False) -> str:
    """Compile oracle.c with gcc (-O2, no FP contraction) into liboracle.so."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp%d" % os.getpid()
        subprocess.check_call(["gcc", "-O2", "-ffp-contract=off", "-fno-fast-math", "-std=c11",
                               "-fPIC", "-shared", _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def lib():
    global _lib
    if _lib is None:
        # ORACLE_LIB points the pins at another build of oracle.c (the
        # mutation test plants mistakes in copies and expects the pins to fail)
        _lib = ctypes.CDLL(os.environ.get("ORACLE_LIB") or build())
        P = ctypes.c_void_p
        i = ctypes.c_int
        i64 = ctypes.c_int64
        sig = {
            "orc_coact": [P, i, i, i, i, P, P, P],
            "orc_place_uniform": [i, i, P],
            "orc_place_capacity": [P, i, i, P, P],
            "orc_place_correlated": [P, i, i, i, P],
            "orc_place_correlated_capped": [P, i, i, i, ctypes.c_double, P],
            "orc_plan": [P, i, i, i, i, i, P, P, P, P, P, P, P, P, P],
            "orc_permute": [P, i, i, i, P, i64, P],
            "orc_combine": [P, i, i64, i, P, P, i, i, P],
            "orc_rank_score": [P, P, i, i, P],
            "orc_shuffle_targets": [P, i, i, i, i, P, P],
            "orc_shuffle_balanced": [P, i, i, i, i, P, i, P],
            "orc_coact_ema": [P, i, i, ctypes.c_double, P, P, P],
            "orc_dispatch_gates": [P, P, i, i, P, P, i64, P, P],
            "orc_expert_reduce": [P, i, i64, i, P, P, i, P, i, P],
            "orc_combine_rows": [P, i, i64, i, P, i, i, P],
            "orc_plan_ranks": [P, i, i, i, i, i, P, P, P, P, P, P, P, P, P],
            "orc_place_replicas": [P, i, i, i, P, i, P, P],
            "orc_assign_replicas": [P, i, i, i, i, i, P, P, P, P, P],
            "orc_assign_replicas_capped": [P, i, i, i, i, i, P, P, P, ctypes.c_double, P, P, P],
            "orc_rank_loads": [P, i, i, P, P],
            "orc_ep_routes": [P, P, i, i, i, P],
            "orc_ep_exchange_rows": [P, i, i, P, P],
        }
        for name, args in sig.items():
            f = getattr(_lib, name)
            f.argtypes = args
            f.restype = ctypes.c_int
        _lib.orc_load_cap.argtypes = [i, i, i, ctypes.c_double]
        _lib.orc_load_cap.restype = i64
    return _lib


class OracleError(RuntimeError):
    def __init__(self, fn, code):
        super().__init__("%s returned %d" % (fn, code))
        self.code = code


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _check(fn, rc):
    if rc != OK:
        raise OracleError(fn, rc)


def coact(ids: np.ndarray, E: int, want=("coact", "ochiai", "trans")):
    """ids int32 [L][T][k] -> dict of coact uint32 [L][E][E], ochiai f32 [L][E][E], trans uint32 [L-1][E][E]."""
    ids = np.ascontiguousarray(ids, dtype=np.int32)
    L, T, k = ids.shape
    out = {}
    c = np.empty((L, E, E), np.uint32) if "coact" in want else None
    o = np.empty((L, E, E), np.float32) if "ochiai" in want else None
    tr = np.empty((max(L - 1, 0), E, E), np.uint32) if ("trans" in want and L > 1) else None
    _check("orc_coact", lib().orc_coact(_p(ids), L, T, k, E, _p(c), _p(o), _p(tr)))
    if c is not None:
        out["coact"] = c
    if o is not None:
        out["ochiai"] = o
    if tr is not None:
        out["trans"] = tr
    return out


def place_uniform(E: int, G: int) -> np.ndarray:
    e2r = np.empty(E, np.int32)
    _check("orc_place_uniform", lib().orc_place_uniform(E, G, _p(e2r)))
    return e2r


def place_capacity(load: np.ndarray, G: int):
    load = np.ascontiguousarray(load, dtype=np.float64)
    e2r = np.empty(load.size, np.int32)
    dev = np.empty(G, np.float64)
    _check("orc_place_capacity", lib().orc_place_capacity(_p(load), load.size, G, _p(e2r), _p(dev)))
    return e2r, dev


def place_correlated(coact_l: np.ndarray, G: int, rpn: int) -> np.ndarray:
    c = np.ascontiguousarray(coact_l, dtype=np.uint32)
    E = c.shape[0]
    e2r = np.empty(E, np.int32)
    _check("orc_place_correlated", lib().orc_place_correlated(_p(c), E, G, rpn, _p(e2r)))
    return e2r


def place_correlated_capped(coact_l: np.ndarray, G: int, rpn: int, eps: float) -> np.ndarray:
    """Correlated placement with load tolerance eps (eps < 0: none)."""
    c = np.ascontiguousarray(coact_l, dtype=np.uint32)
    E = c.shape[0]
    e2r = np.empty(E, np.int32)
    _check("orc_place_correlated_capped", lib().orc_place_correlated_capped(_p(c), E, G, rpn, float(eps), _p(e2r)))
    return e2r


def plan(ids_l: np.ndarray, E: int, G: int, rpn: int, expert_to_rank: np.ndarray, src_rank=None, pick_rank=None):
    """ids_l int32 [T][k] (one layer) -> dict of plan arrays (row arrays trimmed to R).
    With pick_rank int32 [T][k] the serving rank of every pick is given (expert_to_rank ignored)."""
    ids_l = np.ascontiguousarray(ids_l, dtype=np.int32)
    T, k = ids_l.shape
    e2r = None if expert_to_rank is None else np.ascontiguousarray(expert_to_rank, dtype=np.int32)
    pr = None if pick_rank is None else np.ascontiguousarray(pick_rank, dtype=np.int32)
    src = None if src_rank is None else np.ascontiguousarray(src_rank, dtype=np.int32)
    dm = np.empty(T, np.uint64)
    counts = np.empty((G, G), np.int32)
    offsets = np.empty(G * G + 1, np.int32)
    row_token = np.empty(max(T * k, 1), np.int32)
    row_jmask = np.empty(max(T * k, 1), np.uint8)
    row_of = np.empty((T, k), np.int32)
    summary = np.empty(5, np.int64)
    if pr is None:
        _check("orc_plan", lib().orc_plan(_p(ids_l), T, k, E, G, rpn, _p(e2r), _p(src), _p(dm), _p(counts),
                                          _p(offsets), _p(row_token), _p(row_jmask), _p(row_of), _p(summary)))
    else:
        _check("orc_plan_ranks", lib().orc_plan_ranks(_p(ids_l), T, k, E, G, rpn, _p(pr), _p(src), _p(dm),
                                                      _p(counts), _p(offsets), _p(row_token), _p(row_jmask),
                                                      _p(row_of), _p(summary)))
    R = int(summary[0])
    return dict(dest_mask=dm, counts=counts, offsets=offsets, row_token=row_token[:R].copy(),
                row_jmask=row_jmask[:R].copy(), row_of=row_of, summary=summary,
                R=R, R_remote=int(summary[1]), local=int(summary[2]), V=int(summary[3]))


def permute(x: np.ndarray, row_token: np.ndarray) -> np.ndarray:
    x = np.ascontiguousarray(x)
    T, d = x.shape
    rt = np.ascontiguousarray(row_token, dtype=np.int32)
    send = np.empty((rt.size, d), x.dtype)
    _check("orc_permute", lib().orc_permute(_p(x), x.itemsize, T, d, _p(rt), rt.size, _p(send)))
    return send


def combine(Y: np.ndarray, idx: np.ndarray, w: np.ndarray, y_is_bf16: bool) -> np.ndarray:
    """fp64 combine: Y [R_max][d] (float32, or uint16 bf16 bits), idx int32 [T][k], w f32 [T][k]."""
    Y = np.ascontiguousarray(Y)
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    w = np.ascontiguousarray(w, dtype=np.float32)
    T, k = idx.shape
    Rm, d = Y.shape
    out = np.empty((T, d), np.float64)
    _check("orc_combine", lib().orc_combine(_p(Y), int(bool(y_is_bf16)), Rm, d, _p(idx), _p(w), T, k, _p(out)))
    return out


def rank_score(trans_l: np.ndarray, next_expert_to_rank: np.ndarray, G: int) -> np.ndarray:
    tr = np.ascontiguousarray(trans_l, dtype=np.uint32)
    E = tr.shape[0]
    e2r = np.ascontiguousarray(next_expert_to_rank, dtype=np.int32)
    rs = np.empty((E, G), np.uint32)
    _check("orc_rank_score", lib().orc_rank_score(_p(tr), _p(e2r), E, G, _p(rs)))
    return rs


def shuffle_targets(ids_l: np.ndarray, E: int, G: int, rank_score_tab: np.ndarray) -> np.ndarray:
    ids_l = np.ascontiguousarray(ids_l, dtype=np.int32)
    T, k = ids_l.shape
    rs = np.ascontiguousarray(rank_score_tab, dtype=np.uint32)
    tgt = np.empty(T, np.int32)
    _check("orc_shuffle_targets", lib().orc_shuffle_targets(_p(ids_l), T, k, E, G, _p(rs), _p(tgt)))
    return tgt


def shuffle_balanced(ids_l: np.ndarray, E: int, G: int, rank_score_tab: np.ndarray, capacity: int) -> np.ndarray:
    """Shuffle targets with at most `capacity` tokens per rank: pairs (t, r)
    accepted greedily in the order score desc, t asc, r asc."""
    ids_l = np.ascontiguousarray(ids_l, dtype=np.int32)
    T, k = ids_l.shape
    rs = np.ascontiguousarray(rank_score_tab, dtype=np.uint32)
    tgt = np.empty(T, np.int32)
    _check("orc_shuffle_balanced", lib().orc_shuffle_balanced(_p(ids_l), T, k, E, G, _p(rs), int(capacity), _p(tgt)))
    return tgt


def coact_ema(coact, alpha: float, ema_in=None):
    """(ema fp64 [L][E][E], ochiai f32 [L][E][E]) after one batch's counts."""
    c = np.ascontiguousarray(coact, dtype=np.uint32)
    L, E, _ = c.shape
    out = np.empty(c.shape, np.float64)
    och = np.empty(c.shape, np.float32)
    ein = None if ema_in is None else np.ascontiguousarray(ema_in, dtype=np.float64)
    _check("orc_coact_ema", lib().orc_coact_ema(_p(c), L, E, float(alpha), _p(ein) if ein is not None else None,
                                                _p(out), _p(och)))
    return out, och


def dispatch_gates(ids_l, w_l, row_token, row_jmask):
    """(send_e int32 [R][k], send_w f32 [R][k]) for the plan's rows."""
    ids_l = np.ascontiguousarray(ids_l, dtype=np.int32)
    w_l = np.ascontiguousarray(w_l, dtype=np.float32)
    T, k = ids_l.shape
    rt = np.ascontiguousarray(row_token, dtype=np.int32)
    jm = np.ascontiguousarray(row_jmask, dtype=np.uint8)
    R = rt.size
    se = np.empty((R, k), np.int32)
    sw = np.empty((R, k), np.float32)
    _check("orc_dispatch_gates", lib().orc_dispatch_gates(_p(ids_l), _p(w_l), T, k, _p(rt), _p(jm), R, _p(se), _p(sw)))
    return se, sw


def expert_reduce(send, send_e, send_w, scale, y_is_bf16):
    """fp64 y [R][d]: per row, the gate-weighted sum of the stand-in experts' outputs."""
    send = np.ascontiguousarray(send)
    R, d = send.shape
    se = np.ascontiguousarray(send_e, dtype=np.int32)
    sw = np.ascontiguousarray(send_w, dtype=np.float32)
    sc = np.ascontiguousarray(scale, dtype=np.float32)
    y = np.empty((R, d), np.float64)
    _check("orc_expert_reduce", lib().orc_expert_reduce(_p(send), int(bool(y_is_bf16)), R, d, _p(se), _p(sw),
                                                        se.shape[1], _p(sc), sc.size, _p(y)))
    return y


def combine_rows(y, row_of, y_is_bf16=False):
    """fp64 out [T][d]: each token's distinct pre-reduced rows summed once (y float32 or bf16 bits)."""
    y = np.ascontiguousarray(y)
    R, d = y.shape
    ro = np.ascontiguousarray(row_of, dtype=np.int32)
    T, k = ro.shape
    out = np.empty((T, d), np.float64)
    _check("orc_combine_rows", lib().orc_combine_rows(_p(y), int(bool(y_is_bf16)), R, d, _p(ro), T, k, _p(out)))
    return out


def place_replicas(coact_l, G: int, rpn: int, expert_to_rank, extra: int):
    """(replica_rank int32 [E][1 + G/rpn], n_rep int32 [E])."""
    c = np.ascontiguousarray(coact_l, dtype=np.uint32)
    E = c.shape[0]
    e2r = np.ascontiguousarray(expert_to_rank, dtype=np.int32)
    rr = np.empty((E, 1 + G // rpn), np.int32)
    nr = np.empty(E, np.int32)
    _check("orc_place_replicas", lib().orc_place_replicas(_p(c), E, G, rpn, _p(e2r), extra, _p(rr), _p(nr)))
    return rr, nr


def assign_replicas(ids_l, E: int, G: int, rpn: int, replica_rank, n_rep, src_rank=None):
    """(pick_rank int32 [T][k], n_remote int32 [T])."""
    ids_l = np.ascontiguousarray(ids_l, dtype=np.int32)
    T, k = ids_l.shape
    rr = np.ascontiguousarray(replica_rank, dtype=np.int32)
    nr = np.ascontiguousarray(n_rep, dtype=np.int32)
    src = None if src_rank is None else np.ascontiguousarray(src_rank, dtype=np.int32)
    pr = np.empty((T, k), np.int32)
    nrem = np.empty(T, np.int32)
    _check("orc_assign_replicas", lib().orc_assign_replicas(_p(ids_l), T, k, E, G, rpn, _p(rr), _p(nr), _p(src),
                                                            _p(pr), _p(nrem)))
    return pr, nrem


def assign_replicas_capped(ids_l, E: int, G: int, rpn: int, replica_rank, n_rep, eps: float, src_rank=None):
    """(pick_rank int32 [T][k], n_remote int32 [T], rank_load int64 [G]) under
    the per-rank task cap floor((1 + eps) T k / G), tokens in id order."""
    ids_l = np.ascontiguousarray(ids_l, dtype=np.int32)
    T, k = ids_l.shape
    rr = np.ascontiguousarray(replica_rank, dtype=np.int32)
    nr = np.ascontiguousarray(n_rep, dtype=np.int32)
    src = None if src_rank is None else np.ascontiguousarray(src_rank, dtype=np.int32)
    pr = np.empty((T, k), np.int32)
    nrem = np.empty(T, np.int32)
    load = np.empty(G, np.int64)
    _check("orc_assign_replicas_capped",
           lib().orc_assign_replicas_capped(_p(ids_l), T, k, E, G, rpn, _p(rr), _p(nr), _p(src), float(eps),
                                            _p(pr), _p(nrem), _p(load)))
    return pr, nrem, load


def load_cap(T: int, k: int, G: int, eps: float) -> int:
    """floor((1 + eps) T k / G) in fp64 (the per-rank task cap)."""
    return int(lib().orc_load_cap(T, k, G, float(eps)))


def rank_loads(coact_l, expert_to_rank, G: int) -> np.ndarray:
    """int64 [G]: the tasks each rank serves under a one-replica placement
    (sum of n_e = C_ee over its experts)."""
    c = np.ascontiguousarray(coact_l, dtype=np.uint32)
    E = c.shape[0]
    e2r = np.ascontiguousarray(expert_to_rank, dtype=np.int32)
    load = np.empty(G, np.int64)
    _check("orc_rank_loads", lib().orc_rank_loads(_p(c), E, G, _p(e2r), _p(load)))
    return load


def ep_routes(counts_all, offsets, G: int, W: int, me: int) -> np.ndarray:
    """int64 [2*G*(G/W) + 2]: device me's route table (rows received, its
    segments' first local rows, its R, the shifts to the receiving buffers)."""
    c = np.ascontiguousarray(counts_all, dtype=np.int32)
    o = np.ascontiguousarray(offsets, dtype=np.int32)
    route = np.empty(2 * G * (G // W) + 2, np.int64)
    _check("orc_ep_routes", lib().orc_ep_routes(_p(c), _p(o), G, W, me, _p(route)))
    return route


def ep_exchange_rows(counts_all, G: int, W: int):
    """(sent int64 [W], received int64 [W]): rows crossing devices per device."""
    c = np.ascontiguousarray(counts_all, dtype=np.int32)
    sent = np.empty(W, np.int64)
    recv = np.empty(W, np.int64)
    _check("orc_ep_exchange_rows", lib().orc_ep_exchange_rows(_p(c), G, W, _p(sent), _p(recv)))
    return sent, recv
