"""The C ABI without a GPU: the library builds and loads, exports every entry
point that include/*.h declares, the host placement entry points agree with
the oracle exactly, and argument checks fail before any device work."""
import ctypes
import glob
import os
import re

import numpy as np
import pytest

from conftest import ROOT


@pytest.fixture(scope="module")
def cap():
    from co_activation_placement_b200 import build
    build.build()
    import co_activation_placement_b200 as cap
    cap.lib()
    return cap


def declared_functions():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        src = open(h).read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        for m in re.finditer(r"\b(moe_[a-z_0-9]+)\s*\(", src):
            names.add(m.group(1))
    return sorted(names)


def test_header_declares_the_path():
    names = declared_functions()
    for want in ["moe_coact_stats", "moe_plan_dispatch", "moe_permute", "moe_combine",
                 "moe_shuffle_targets", "moe_rank_score", "moe_place_uniform", "moe_place_correlated"]:
        assert want in names


def test_every_declared_symbol_is_exported(cap):
    lib = ctypes.CDLL(cap.LIB_PATH)
    missing = [n for n in declared_functions() if not hasattr(lib, n)]
    assert not missing, missing


def test_process_wide_settings(cap):
    """The method and grid settings return the previous value and reject bad
    arguments without touching a device."""
    prev = cap.cooperative_blocks(7)
    assert cap.cooperative_blocks(prev) == 7
    with pytest.raises(ValueError):
        cap.cooperative_blocks(-1)
    prev = cap.plan_dispatch_method(1)
    assert cap.plan_dispatch_method(prev) == 1
    with pytest.raises(ValueError):
        cap.plan_dispatch_method(2)


def test_status_strings(cap):
    assert cap.lib().moe_status_string(0) == b"ok"
    assert cap.lib().moe_status_string(3).startswith(b"workspace")


@pytest.mark.parametrize("E,G", [(64, 8), (8, 4), (256, 64), (12, 12), (5, 1)])
def test_place_uniform_matches_oracle(cap, orc, E, G):
    assert (cap.place_uniform(E, G) == orc.place_uniform(E, G)).all()


def test_place_uniform_rejects_uneven(cap):
    with pytest.raises(cap.MoeError) as ei:
        cap.place_uniform(10, 4)
    assert ei.value.status == cap.MOE_ERR_ARG


def test_place_capacity_matches_oracle(cap, orc):
    rng = np.random.default_rng(0)
    for E, G in [(64, 8), (256, 64), (13, 4)]:
        load = rng.random(E) * rng.integers(1, 100, E)
        load[3] = load[5]                    # a tie: lower id first
        a, da = cap.place_capacity(load, G)
        b, db = orc.place_capacity(load, G)
        assert (a == b).all() and (da == db).all()


def test_place_correlated_matches_oracle(cap, orc):
    from synth import WORKLOADS, make_routing
    for name in ["tiny", "one_node", "ep32"]:
        w = WORKLOADS[name]
        ids = make_routing(w, seed=1, T=min(w.T, 20000))
        C = orc.coact(ids[:1], w.E, want=("coact",))["coact"][0]
        for G, rpn in [(w.G, w.rpn), (w.G, 1), (w.G, w.G)]:
            if G % rpn:
                continue
            assert (cap.place_correlated(C, G, rpn) == orc.place_correlated(C, G, rpn)).all()


def test_place_correlated_large_matches_oracle(cap, orc):
    rng = np.random.default_rng(1)
    E = 256
    C = rng.integers(0, 1000, (E, E)).astype(np.uint32)
    C = np.triu(C, 1)
    C = C + C.T
    np.fill_diagonal(C, 5000 + rng.integers(0, 3, E))
    C = C.astype(np.uint32)
    assert (cap.place_correlated(C, 64, 8) == orc.place_correlated(C, 64, 8)).all()


def test_workspace_queries(cap):
    assert cap.coact_stats_workspace(8, 1 << 20, 8, 128) > 0
    assert cap.coact_stats_workspace(1, 10, 9, 128) == 0          # k > 8
    assert cap.plan_dispatch_workspace(131072, 8, 64, True) > cap.plan_dispatch_workspace(131072, 8, 64, False)
    assert cap.plan_dispatch_workspace(16, 2, 65, False) == 0     # G > 64


def test_argument_errors_return_before_device_work(cap):
    L = cap.lib()
    P = ctypes.c_void_p
    fake = P(256)   # never dereferenced: each call below fails its host checks first
    # k out of range
    assert L.moe_coact_stats(fake, 1, 10, 9, 16, fake, None, None, fake, fake, 1 << 20, None) == cap.MOE_ERR_ARG
    # workspace too small
    assert L.moe_coact_stats(fake, 2, 4096, 2, 8, fake, None, None, fake, fake, 16, None) == cap.MOE_ERR_WORKSPACE
    # G > 64, rpn not dividing G, T not a multiple of G without src_rank
    pl = cap._Plan(256, 256, 256, 256, 256, 256, 256)
    assert L.moe_plan_dispatch(fake, 64, 2, 8, 65, 1, fake, None, ctypes.byref(pl), fake, fake, 1 << 20, None) == cap.MOE_ERR_ARG
    assert L.moe_plan_dispatch(fake, 64, 2, 8, 8, 3, fake, None, ctypes.byref(pl), fake, fake, 1 << 20, None) == cap.MOE_ERR_ARG
    assert L.moe_plan_dispatch(fake, 63, 2, 8, 8, 8, fake, None, ctypes.byref(pl), fake, fake, 1 << 20, None) == cap.MOE_ERR_ARG
    # the plan in two calls: no source ranks, G out of range, a short workspace
    assert L.moe_plan_dispatch_presorted(fake, 64, 2, 8, 8, 8, fake, None, ctypes.byref(pl), fake, fake, 1 << 20,
                                         None) == cap.MOE_ERR_ARG
    assert L.moe_plan_sources(None, 64, 8, fake, fake, 1 << 20, None) == cap.MOE_ERR_ARG
    assert L.moe_plan_sources(fake, 64, 65, fake, fake, 1 << 20, None) == cap.MOE_ERR_ARG
    assert L.moe_plan_sources(fake, 4096, 8, fake, fake, 64, None) == cap.MOE_ERR_WORKSPACE
    # misaligned rows / unsupported row size / bad dtype
    assert L.moe_permute(P(264), cap.MOE_BF16, 4, 8, 2, fake, 8, fake, fake, None) == cap.MOE_ERR_ARG
    assert L.moe_permute(fake, cap.MOE_BF16, 4, 7, 2, fake, 8, fake, fake, None) == cap.MOE_ERR_UNSUPPORTED
    assert L.moe_combine(fake, 7, 8, 8, fake, fake, 4, 2, fake, 0, fake, None) == cap.MOE_ERR_ARG
    assert L.moe_shuffle_targets(fake, 4, 2, 1024, 64, fake, fake, fake, None) == cap.MOE_ERR_UNSUPPORTED
    # balanced shuffle: shards that cannot hold T, a table too large, a short workspace
    assert L.moe_shuffle_balanced(fake, 9, 1, 4, 4, fake, 2, fake, None, fake, 1 << 30, fake, None) == cap.MOE_ERR_ARG
    assert L.moe_shuffle_balanced(fake, 64, 2, 1024, 64, fake, 1, fake, None, fake, 1 << 30, fake, None) \
        == cap.MOE_ERR_UNSUPPORTED
    assert L.moe_shuffle_balanced(fake, 64, 2, 8, 4, fake, 16, fake, None, fake, 64, fake, None) == cap.MOE_ERR_WORKSPACE
    assert cap.shuffle_balanced_workspace(1000, 8, 125) < cap.shuffle_balanced_workspace(1000, 8, 1000)
    # EMA: alpha outside [0, 1], in place
    assert L.moe_coact_ema(fake, 1, 4, ctypes.c_double(1.5), None, fake, None, None) == cap.MOE_ERR_ARG
    assert L.moe_coact_ema(fake, 1, 4, ctypes.c_double(0.5), fake, fake, None, None) == cap.MOE_ERR_ARG
    # several devices: W not dividing G, me outside [0, W), G > 64, misaligned x, odd row sizes, records
    assert L.moe_ep_routes(fake, fake, 8, 3, 0, fake, fake, None) == cap.MOE_ERR_ARG
    assert L.moe_ep_routes(fake, fake, 8, 4, 4, fake, fake, None) == cap.MOE_ERR_ARG
    assert L.moe_ep_routes(fake, fake, 128, 2, 0, fake, fake, None) == cap.MOE_ERR_ARG
    assert L.moe_ep_permute(P(264), cap.MOE_BF16, 4, 8, 2, fake, 8, fake, 8, 2, fake, 8, fake, None) == cap.MOE_ERR_ARG
    assert L.moe_ep_permute(fake, cap.MOE_BF16, 4, 7, 2, fake, 8, fake, 8, 2, fake, 8, fake, None) \
        == cap.MOE_ERR_UNSUPPORTED
    assert L.moe_ep_permute(fake, cap.MOE_F32, 4, 8, 9, fake, 8, fake, 8, 2, fake, 8, fake, None) == cap.MOE_ERR_ARG
    assert L.moe_ep_combine(fake, cap.MOE_F32, 8, 8, fake, 8, 3, 8, fake, fake, 4, 2, fake, 0, fake, None) \
        == cap.MOE_ERR_ARG
    assert L.moe_ep_combine(fake, cap.MOE_F32, 8, 8, fake, 8, 2, 8, fake, fake, 4, 2, P(260), 0, fake, None) \
        == cap.MOE_ERR_ARG
    assert L.moe_ep_scatter_rows(fake, 6, 8, fake, 8, 2, fake, 8, fake, None) == cap.MOE_ERR_ARG
    assert L.moe_ep_scatter_rows(P(258), 8, 8, fake, 8, 2, fake, 8, fake, None) == cap.MOE_ERR_ARG
    assert cap.ep_route_len(64, 8) == 2 * 64 * 8 + 2
    # capped task assignment: eps < 0, T k past int32 task counts
    assert L.moe_assign_replicas_capped(fake, 64, 2, 8, 8, 8, fake, fake, None, ctypes.c_double(-0.5), fake, None,
                                        None, fake, fake, 1 << 20, None) == cap.MOE_ERR_ARG
    assert L.moe_assign_replicas_capped(fake, 1 << 28, 8, 64, 8, 8, fake, fake, fake, ctypes.c_double(0.1), fake,
                                        None, None, fake, fake, 1 << 20, None) == cap.MOE_ERR_ARG


@pytest.mark.parametrize("E,G,rpn,extra", [(16, 8, 2, 1), (64, 8, 8, 2), (64, 32, 8, 1), (256, 64, 8, 1), (24, 6, 1, 3)])
def test_place_replicas_matches_oracle(cap, orc, E, G, rpn, extra):
    rng = np.random.default_rng(E + G + extra)
    C = rng.integers(0, 200, (E, E)) * (rng.random((E, E)) < 0.3)
    C = np.triu(C, 1)
    C = (C + C.T + np.diag(rng.integers(100, 300, E))).astype(np.uint32)
    C[3, 5] = C[5, 3] = C[3, 7] = C[7, 3] = 777                  # equal scores: ties by (e, node)
    e2r = orc.place_correlated(C, G, rpn)
    a = cap.place_replicas(C, G, rpn, e2r, extra)
    b = orc.place_replicas(C, G, rpn, e2r, extra)
    assert (a[0] == b[0]).all() and (a[1] == b[1]).all()


@pytest.mark.parametrize("eps", [-1.0, 0.0, 0.1, 0.5])
def test_place_correlated_capped_matches_oracle(cap, orc, eps):
    from synth import WORKLOADS, make_routing
    for name in ["one_node", "ep32"]:
        w = WORKLOADS[name]
        ids = make_routing(w, seed=1, T=min(w.T, 20000))
        C = orc.coact(ids[:1], w.E, want=("coact",))["coact"][0]
        assert (cap.place_correlated_capped(C, w.G, w.rpn, eps) == orc.place_correlated_capped(C, w.G, w.rpn, eps)).all()
    rng = np.random.default_rng(3)
    C = rng.integers(0, 1000, (256, 256)).astype(np.uint32)
    C = np.triu(C, 1)
    C = (C + C.T + np.diag(rng.integers(1000, 90000, 256))).astype(np.uint32)
    assert (cap.place_correlated_capped(C, 64, 8, eps) == orc.place_correlated_capped(C, 64, 8, eps)).all()


def test_header_is_plain_c(tmp_path):
    """include/moe_coact.h is a C header: a C99 translation unit that includes
    it and names its types and entry points compiles with warnings as errors."""
    import shutil
    import subprocess
    gcc = shutil.which("gcc")
    cuda_inc = "/usr/local/cuda/include"
    if not gcc or not os.path.isdir(cuda_inc):
        pytest.skip("gcc or the CUDA headers are not installed")
    src = tmp_path / "use_header.c"
    src.write_text('#include "moe_coact.h"\n'
                   "int use(void) {\n"
                   "    moe_plan p = {0};\n"
                   "    moe_status (*f)(const int32_t *, int, int, int, int, uint32_t *, float *, uint32_t *,\n"
                   "                    int32_t *, void *, size_t, cudaStream_t) = moe_coact_stats;\n"
                   "    return (int)(p.counts == 0) + (f != 0) + (int)moe_launch_count();\n"
                   "}\n")
    r = subprocess.run([gcc, "-std=c99", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"),
                        "-I", cuda_inc, "-c", str(src), "-o", str(tmp_path / "use_header.o")],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr


def test_c_program_links_and_calls_the_library(cap, tmp_path):
    """A plain C program linked against libmoecoact.so calls a host entry
    point through the C ABI alone (no Python): the uniform placement of 64
    experts on 8 ranks, the pages' worked example (rank d holds 8d..8d+7)."""
    import shutil
    import subprocess
    gcc = shutil.which("gcc")
    cuda_inc = "/usr/local/cuda/include"
    if not gcc or not os.path.isdir(cuda_inc):
        pytest.skip("gcc or the CUDA headers are not installed")
    libdir = os.path.dirname(cap.LIB_PATH)
    src = tmp_path / "place.c"
    src.write_text('#include <stdio.h>\n#include "moe_coact.h"\n'
                   "int main(void) {\n"
                   "    int32_t e2r[64];\n"
                   "    if (moe_place_uniform(64, 8, e2r) != MOE_OK) return 1;\n"
                   "    if (moe_place_uniform(63, 8, e2r) != MOE_ERR_ARG) return 2;\n"
                   "    for (int e = 0; e < 64; ++e) printf(\"%d \", e2r[e]);\n"
                   "    printf(\"\\n%s\\n\", moe_status_string(MOE_ERR_ARG));\n"
                   "    return 0;\n"
                   "}\n")
    exe = tmp_path / "place"
    r = subprocess.run([gcc, "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"), "-I", cuda_inc,
                        str(src), "-o", str(exe), "-L", libdir, "-l:libmoecoact.so", "-Wl,-rpath," + libdir],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    run = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert run.returncode == 0, run.stderr
    ranks = [int(v) for v in run.stdout.split("\n")[0].split()]
    assert ranks == [e // 8 for e in range(64)]
    assert run.stdout.split("\n")[1].strip() != ""


def test_host_placements_match_oracle_on_random_inputs(cap, orc):
    """The library's host placements (C++) against the oracle on 120 seeded
    random shapes and co-activation matrices: uniform, capacity-aware,
    correlated, capped, and replica layouts, bit for bit."""
    rng = np.random.default_rng(2024)
    for _ in range(120):
        G = int(rng.choice([1, 2, 4, 6, 8, 16]))
        rpn = int(rng.choice([r for r in range(1, G + 1) if G % r == 0]))
        E = G * int(rng.integers(1, 6))
        k = int(rng.integers(1, min(E, 6) + 1))
        T = int(rng.integers(1, 300))
        hot = rng.permutation(E)[: min(E, k + 2)]
        ids = np.where((rng.random(T) < 0.6)[:, None],
                       hot[np.argsort(rng.random((T, hot.size)), axis=1)[:, :k]],
                       np.argsort(rng.random((T, E)), axis=1)[:, :k]).astype(np.int32)[None]
        C = orc.coact(ids, E)["coact"][0]
        assert (cap.place_uniform(E, G) == orc.place_uniform(E, G)).all()
        load = np.diag(C).astype(np.float64)
        assert (cap.place_capacity(load, G)[0] == orc.place_capacity(load, G)[0]).all()
        assert (cap.place_correlated(C, G, rpn) == orc.place_correlated(C, G, rpn)).all()
        eps = float(rng.choice([0.0, 0.05, 0.2]))
        assert (cap.place_correlated_capped(C, G, rpn, eps) == orc.place_correlated_capped(C, G, rpn, eps)).all()
        e2r = orc.place_correlated(C, G, rpn)
        extra = int(rng.integers(0, 3))
        got = cap.place_replicas(C, G, rpn, e2r, extra)
        want = orc.place_replicas(C, G, rpn, e2r, extra)
        assert (got[0] == want[0]).all() and (got[1] == want[1]).all()
        assert (cap.rank_loads(C, e2r, G) == orc.rank_loads(C, e2r, G)).all()
