"""The timeout path of the bounded mbarrier waits, on the GPU, without a fault or a hang:
a wait on a barrier that nothing arrives at gives up after its limit, the status word
records it, and the context keeps working."""
import time

import numpy as np
import pytest
import torch

from block_scaled_moe_sigmoid_b200 import api, synth

from .gpu_helpers import Case

pytestmark = pytest.mark.gpu


def test_bounded_wait_times_out_and_context_survives():
    wl = synth.custom(seed=19, T=32, d=256, E=8, k=2, I=128)
    case = Case(wl)
    assert case.plan.check()[0] == 0
    t0 = time.time()
    api.moe_debug_timeout_probe(case.plan.handle)
    code, bits = case.plan.check()
    elapsed = time.time() - t0
    assert code == 5 and bits & 1, (code, bits)          # MOE_ERR_TIMEOUT, bit MOE_DEV_ERR_TIMEOUT
    assert 0.9 < elapsed < 30.0                           # the 1 s limit, not a hang
    assert case.plan.check()[0] == 0                      # cleared by the check
    # the context is intact: a full layer call still runs and is deterministic
    idx, w = case.plan.route(case.x, case.W_r, case.bias)
    y1 = case.plan.forward(case.x, idx, w, case.experts, case.shared)
    y2 = case.plan.forward(case.x, idx, w, case.experts, case.shared)
    torch.cuda.synchronize()
    assert torch.equal(y1, y2) and torch.isfinite(y1.float()).all()
    assert case.plan.check()[0] == 0
