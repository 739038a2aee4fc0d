"""moe_plan_dispatch_static: the dispatch plan for callers that cannot
allocate device memory (code inside another framework's allocator hook,
processes with a fixed device-memory budget, latency-critical loops that
cannot accept cudaMalloc's possible device synchronisation).  Its output must
equal moe_plan_dispatch's, computed with caller-provided workspace, on two
calls in a row (the static scratch keeps the previous call's contents, so the
second call checks that everything that must start at zero is cleared).

Called through the C ABI directly.  This file is collected last, so that a run
stopping at the first failure has already run every other test."""
import ctypes

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

SCRATCH_BYTES = 4 << 20   # MOE_PLAN_STATIC_SCRATCH_BYTES in include/moe_coact.h


@pytest.fixture(scope="module")
def lib():
    from co_activation_placement_b200 import build
    build.build()
    import co_activation_placement_b200 as cap
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    L = cap.lib()
    P, i = ctypes.c_void_p, ctypes.c_int
    f = L.moe_plan_dispatch_static
    f.argtypes = [P, i, i, i, i, i, P, P, ctypes.POINTER(cap._Plan), P, P]
    f.restype = i
    return cap, L


def _plan_arrays(p, T, k):
    torch.cuda.synchronize()
    R = int(p.summary[0].item())
    return dict(summary=p.summary.cpu().numpy(), dest_mask=p.dest_mask[:T].cpu().numpy(),
                counts=p.counts.cpu().numpy(), offsets=p.offsets.cpu().numpy(),
                row_token=p.row_token[:R].cpu().numpy(), row_jmask=p.row_jmask[:R].cpu().numpy(),
                row_of=p.row_of[:T].cpu().numpy(), err=int(p.err.item()))


def _inputs(seed, T, E, k, G, with_src):
    rng = np.random.default_rng(seed)
    hot = rng.permutation(E)[: k + 2]
    ids = np.where((rng.random(T) < 0.6)[:, None],
                   hot[np.argsort(rng.random((T, hot.size)), axis=1)[:, :k]],
                   np.argsort(rng.random((T, E)), axis=1)[:, :k]).astype(np.int32)
    e2r = rng.permutation(np.arange(E, dtype=np.int32) // (E // G)).astype(np.int32)
    src = rng.integers(0, G, T).astype(np.int32) if with_src else None
    dev = lambda a: None if a is None else torch.from_numpy(a).cuda()
    return dev(ids), dev(e2r), dev(src)


@pytest.mark.parametrize("T,E,k,G,rpn,with_src", [(4096, 8, 2, 4, 2, False), (131072, 256, 8, 64, 8, True),
                                                  (65536, 64, 6, 32, 8, False), (5000, 40, 5, 8, 4, True)])
def test_static_plan_equals_workspace_plan(lib, T, E, k, G, rpn, with_src):
    cap, L = lib
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for call in range(2):
        ids, e2r, src = _inputs(1000 * call + T, T, E, k, G, with_src)
        ref = cap.plan_dispatch(ids, E, G, rpn, e2r, src_rank=src)
        got = cap.Plan.empty(T, k, G, "cuda")
        cs = got.c_struct()
        st = L.moe_plan_dispatch_static(ids.data_ptr(), T, k, E, G, rpn, e2r.data_ptr(),
                                        None if src is None else src.data_ptr(), ctypes.byref(cs),
                                        got.err.data_ptr(), stream)
        assert st == cap.MOE_OK
        a, b = _plan_arrays(ref, T, k), _plan_arrays(got, T, k)
        assert a["err"] == 0 and b["err"] == 0
        for key in a:
            assert np.array_equal(a[key], b[key]), (call, key)


def test_static_plan_rejects_sizes_beyond_its_scratch(lib):
    cap, L = lib
    T, k, G = 1 << 21, 8, 64
    assert cap.plan_dispatch_workspace(T, k, G, True) > SCRATCH_BYTES
    before = cap.launch_count()
    fake = ctypes.c_void_p(256)          # never dereferenced: the size check fails first
    pl = cap._Plan(256, 256, 256, 256, 256, 256, 256)
    st = L.moe_plan_dispatch_static(fake, T, k, 256, G, 8, fake, fake, ctypes.byref(pl), fake, None)
    assert st == cap.MOE_ERR_WORKSPACE
    assert cap.launch_count() == before
