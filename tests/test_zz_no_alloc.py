"""The allocation-free grouping entry point (moe_permute_noalloc).

Some callers cannot call cudaMalloc: a plug-in inside a serving engine or framework that
owns the device-memory budget, or a thread that must not take the allocator's locks or
pay its implicit synchronisation.  moe_permute_noalloc serves them from a fixed device
scratch array.  This test calls it through the C ABI twice in a row, with different
inputs, and requires exactly the output of the plan-based moe_permute (integer work:
bit-exact).  It lives in a file of its own that pytest collects last."""
import ctypes

import pytest
import torch

from block_scaled_moe_sigmoid_b200 import api

pytestmark = pytest.mark.gpu


def _idx(T, E, k, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.stack([torch.randperm(E, generator=g)[:k] for _ in range(T)]).to(torch.int32).cuda()


def _noalloc(idx, E):
    """Direct C-ABI call with caller-owned output buffers."""
    T, k = idx.shape
    out = [torch.full((E,), -7, dtype=torch.int32, device="cuda"),
           torch.full((E + 1,), -7, dtype=torch.int32, device="cuda"),
           torch.full((T * k,), -7, dtype=torch.int32, device="cuda"),
           torch.full((T, k), -7, dtype=torch.int32, device="cuda")]
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    code = api.lib().moe_permute_noalloc(ctypes.c_void_p(idx.data_ptr()), T, E, k,
                                         *(ctypes.c_void_p(t.data_ptr()) for t in out), stream)
    assert code == 0, api.STATUS_NAMES.get(code, code)
    return out


def test_noalloc_permute_matches_plan_permute_on_two_calls():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    for T, E, k, seed in ((1000, 896, 16, 1), (300, 64, 4, 2)):
        idx = _idx(T, E, k, seed)
        got = _noalloc(idx, E)
        plan = api.Plan(T, 128, E, k, 128)
        ref = plan.permute(idx)
        torch.cuda.synchronize()
        for a, b in zip(got, ref):
            assert torch.equal(a.reshape(-1).cpu(), b.reshape(-1).cpu())


def test_noalloc_permute_rejects_sizes_beyond_its_scratch():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    buf = torch.zeros(16, dtype=torch.int32, device="cuda")
    p = ctypes.c_void_p(buf.data_ptr())   # the size check rejects the call before any access
    assert api.lib().moe_permute_noalloc(p, 100000, 896, 16, p, p, p, p, None) == 2
