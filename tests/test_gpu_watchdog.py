"""The device watchdog: a wait that can never complete ends with an error
status that the host reads, and the CUDA context stays usable.  The wait is
made to run out on purpose (an mbarrier nothing arrives at, a short limit);
nothing faults, traps or hangs."""
import numpy as np
import pytest

import block_sparse_attention_mask_b200 as vsa
import workloads as W
from _helpers import PathRun

pytestmark = pytest.mark.gpu


def test_watchdog_reports_timeout_and_context_survives():
    import torch
    w = W.tiny()
    plan = vsa.Plan(list(w.specs), (w.T, w.H, w.W), w.unit, w.q_tile, w.kv_tile)
    plan.check()                                        # clean to start with
    vsa.vsa_selftest_watchdog(plan.handle, 2_000_000)   # about 1 ms of SM cycles
    torch.cuda.synchronize()
    with pytest.raises(vsa.VsaError) as e:
        plan.check()
    assert e.value.code == -6                           # VSA_ERR_TIMEOUT
    plan.check()                                        # the status word was cleared
    plan.close()
    # the context still runs the real path correctly
    r = PathRun(w)
    for h in range(w.heads):
        r.check_rows(h, np.arange(w.N))
    r.close()


def test_watchdog_rejects_bad_limits():
    w = W.tiny()
    plan = vsa.Plan(list(w.specs), (w.T, w.H, w.W), w.unit, w.q_tile, w.kv_tile)
    for bad in (0, -5, 1 << 40):
        with pytest.raises(vsa.VsaError):
            vsa.vsa_selftest_watchdog(plan.handle, bad)
    plan.close()
