"""The bounded device waits give up instead of hanging: each self-test makes
one kind of wait run out on purpose (a grid barrier that one block never
reaches, an mbarrier phase that nothing completes).  The kernel must return
after about the 2 s limit with MOE_DERR_TIMEOUT in the error word, and the
context must stay usable for the next call."""
import time

import numpy as np
import pytest
import torch

import oracle as orc

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def cap():
    from co_activation_placement_b200 import build
    build.build()
    import co_activation_placement_b200 as cap
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    cap.lib()
    return cap


@pytest.mark.parametrize("kind", [0, 1])
def test_wait_runs_out_and_reports(cap, kind):
    torch.cuda.synchronize()
    t0 = time.time()
    err = cap.selftest_wait_timeout(kind)
    torch.cuda.synchronize()
    dt = time.time() - t0
    assert int(err.item()) == cap.DERR_TIMEOUT
    assert 1.5 < dt < 30.0
    # the context is still usable
    ids = np.array([[[0, 1], [2, 3], [1, 2]]], np.int32)
    g = cap.coact_stats(torch.from_numpy(ids).cuda(), 4)
    assert int(g["err"].item()) == 0
    assert (g["coact"].cpu().numpy() == orc.coact(ids, 4)["coact"]).all()
