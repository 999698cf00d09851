"""Quantile Balancing inputs on the GPU against the oracle (reading R23).

The margins are fp32 differences of fp32 keys and the quantiles are order statistics
(selections, no arithmetic), so the comparison on the GPU's own logits is bit-exact.  The
bias-update rule is the caller's (the pages do not publish it): the tests hand in a rule
of their own and check that the library calls it with this step's quantiles."""
import ctypes

import numpy as np
import pytest
import torch

from block_scaled_moe_sigmoid_b200 import api, synth
from oracle import router

pytestmark = pytest.mark.gpu

LEVELS = [0.0, 0.1, 0.5, 1.0 - 16 / 896, 0.999, 1.0]


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    api.lib()


def _plan(T, E, k, select_only=False):
    return api.Plan(T, 128, E, k, 128,
                    bias_mode=api.MOE_BIAS_SELECT_ONLY if select_only else api.MOE_BIAS_LOGIT)


def _oracle(z, k, levels, b=None):
    return router.margin_quantiles(router.routing_margins(z, k, select_bias=b), levels)


@pytest.mark.parametrize("T,E,k", [(1000, 896, 16), (1, 64, 4), (257, 32, 32), (33, 8, 1)])
def test_margin_quantiles_bit_exact(T, E, k):
    g = torch.Generator().manual_seed(T * 7 + E)
    z = torch.randn((T, E), generator=g) * 1.7
    plan = _plan(T, E, k)
    q = api.moe_route_margin_quantiles(plan.handle, z.cuda(), E, LEVELS)
    ref = _oracle(z.numpy(), k, LEVELS)
    assert ref.dtype == np.float32
    assert np.array_equal(q.cpu().numpy(), ref)


def test_margin_quantiles_select_only_key_and_ties():
    """Select-only key z + b (fp32) on logits with many exact ties (small integers): the
    k-th key and the order statistics are unaffected by which tied index is taken."""
    T, E, k = 300, 96, 8
    g = torch.Generator().manual_seed(3)
    z = torch.randint(-3, 4, (T, E), generator=g).float() * 0.5
    b = (torch.randint(-2, 3, (E,), generator=g).float() * 0.25)
    plan = _plan(T, E, k, select_only=True)
    q = api.moe_route_margin_quantiles(plan.handle, z.cuda(), E, LEVELS, select_bias=b.cuda())
    assert np.array_equal(q.cpu().numpy(), _oracle(z.numpy(), k, LEVELS, b.numpy()))


def test_margin_quantiles_on_routed_logits():
    """The logits moe_route writes for the toy layer, then the quantiles of its margins."""
    wl = synth.WORKLOADS["toy"]
    x = synth.draw_x(wl).cuda()
    W_r, b = synth.draw_router(wl)
    plan = _plan(wl.T, wl.E, wl.k)
    logits = torch.empty((wl.T, wl.E), dtype=torch.float32, device="cuda")
    plan.route(x, W_r.cuda(), b.cuda(), logits=logits)
    q = api.moe_route_margin_quantiles(plan.handle, logits, wl.E, LEVELS)
    ref = _oracle(logits.cpu().numpy(), wl.k, LEVELS)
    assert np.array_equal(q.cpu().numpy(), ref)
    m = router.routing_margins(logits.cpu().numpy(), wl.k)
    assert np.array_equal(q[0].cpu().numpy(), m.min(axis=0))      # level 0: the minimum
    assert np.array_equal(q[-1].cpu().numpy(), m.max(axis=0))     # level 1: the maximum


def test_quantile_balance_calls_the_rule_with_this_steps_quantiles():
    T, E, k = 512, 128, 8
    g = torch.Generator().manual_seed(9)
    z = (torch.randn((T, E), generator=g) * 1.3).cuda()
    bias = (torch.randn(E, generator=g) * 0.1).cuda()
    plan = _plan(T, E, k, select_only=True)
    levels = [1.0 - k / E, 0.5]
    qview = plan.debug_tensor(7, torch.float32, (len(levels), E))   # the buffer the rule reads
    nxt = torch.full((E,), 123.0, device="cuda")
    seen = {}

    def rule(q_ptr, n_levels, n_experts, b_ptr, next_ptr, stream_ptr, user):
        # the test's own rule (the pages publish none): move each expert's bias half way
        # towards putting its (1 - k/E)-quantile margin at zero, on the call's stream
        seen.update(q=q_ptr, n=n_levels, E=n_experts, b=b_ptr, nxt=next_ptr, user=user)
        # a NULL stream is the legacy default stream, which torch calls its default stream
        st = torch.cuda.ExternalStream(stream_ptr) if stream_ptr else torch.cuda.default_stream()
        with torch.cuda.stream(st):
            nxt.copy_(bias - 0.5 * qview[0])

    cb = api.BIAS_RULE(rule)
    api.moe_quantile_balance(plan.handle, z, bias, levels, cb, bias_next=nxt, user=ctypes.c_void_p(77))
    torch.cuda.synchronize()
    assert seen["n"] == 2 and seen["E"] == E and seen["user"] == 77
    assert seen["q"] == qview.data_ptr() and seen["b"] == bias.data_ptr() and seen["nxt"] == nxt.data_ptr()
    # the rule saw this step's quantiles of the key z + b ...
    q_ref = _oracle(z.cpu().numpy(), k, levels, bias.cpu().numpy())
    assert np.array_equal(qview.cpu().numpy(), q_ref)
    # ... and its own arithmetic ran after the quantile kernels, in stream order
    assert torch.equal(nxt.cpu(), (bias - 0.5 * torch.from_numpy(q_ref[0]).cuda()).cpu())


def test_margin_quantiles_reject_bad_arguments():
    plan = _plan(16, 32, 4)
    z = torch.zeros((16, 32), device="cuda")
    with pytest.raises(api.MoeError):
        api.moe_route_margin_quantiles(plan.handle, z, 32, [1.5])           # level outside [0, 1]
    with pytest.raises(api.MoeError):
        api.moe_route_margin_quantiles(plan.handle, z, 32, [0.5] * 17)      # more than 16 levels
    with pytest.raises(api.MoeError):
        api.moe_route_margin_quantiles(plan.handle, torch.zeros((17, 32), device="cuda"), 32, [0.5])  # T > T_max
