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


def _noalloc_code(idx, T, E, k, out):
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return api.lib().moe_permute_noalloc(None if idx is None else ctypes.c_void_p(idx.data_ptr()), T, E, k,
                                         *(ctypes.c_void_p(t.data_ptr()) for t in out), stream)


def test_noalloc_permute_empty_batch_zeroes_counts_and_offsets():
    """T = 0: only the counts and offsets are written (all zero)."""
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    E, k = 40, 4
    out = [torch.full((E,), -7, dtype=torch.int32, device="cuda"),
           torch.full((E + 1,), -7, dtype=torch.int32, device="cuda"),
           torch.full((4,), -7, dtype=torch.int32, device="cuda"),
           torch.full((4,), -7, dtype=torch.int32, device="cuda")]
    assert _noalloc_code(None, 0, E, k, out) == 0
    torch.cuda.synchronize()
    assert torch.all(out[0] == 0) and torch.all(out[1] == 0)
    assert torch.all(out[2] == -7) and torch.all(out[3] == -7)


def test_noalloc_permute_skips_out_of_range_ids():
    """Ids outside [0, E) are skipped: their inv entry is -1, and the counts, offsets and
    the written part of perm_tok equal the plan-based entry point's (which skips them the
    same way) and a host count of the valid ids."""
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    T, E, k = 200, 48, 6
    idx = _idx(T, E, k, 9)
    bad = [(3, 1, E), (17, 0, -1), (150, 5, E + 100)]
    for t, j, v in bad:
        idx[t, j] = v
    got = _noalloc(idx, E)
    plan = api.Plan(T, 128, E, k, 128)
    ref = plan.permute(idx)
    torch.cuda.synchronize()
    inv = got[3].cpu()
    for t, j, _ in bad:
        assert inv[t, j].item() == -1
    ids = idx.cpu().reshape(-1)
    valid = ids[(ids >= 0) & (ids < E)].long()
    assert torch.equal(got[0].cpu(), torch.bincount(valid, minlength=E).to(torch.int32))
    n_valid = valid.numel()
    assert got[1][E].item() == n_valid
    for a, b in zip(got[:2], ref[:2]):
        assert torch.equal(a.cpu(), b.cpu())
    assert torch.equal(got[2][:n_valid].cpu(), ref[2][:n_valid].cpu())
    assert torch.equal(inv, ref[3].cpu())
    code, bits = plan.check()
    assert code == 7 and bits & 2          # the plan-based call flags them; this one cannot


def test_noalloc_permute_at_its_size_limit():
    """T = 18432 at E = 896, k = 16 fills the scratch array exactly as far as it goes (the
    largest accepted batch): bit-exact against the plan-based call.  One token more is
    rejected with MOE_ERR_UNSUPPORTED_SHAPE before anything is launched."""
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    E, k, T = 896, 16, 18432
    g = torch.Generator(device="cuda").manual_seed(5)
    idx = torch.argsort(torch.rand((T, E), generator=g, device="cuda"), dim=1)[:, :k].to(torch.int32).contiguous()
    got = _noalloc(idx, E)
    plan = api.Plan(T, 128, E, k, 128)
    ref = plan.permute(idx)
    torch.cuda.synchronize()
    for a, b in zip(got, ref):
        assert torch.equal(a.reshape(-1).cpu(), b.reshape(-1).cpu())
    out = [torch.empty(n, dtype=torch.int32, device="cuda") for n in (E, E + 1, (T + 1) * k, (T + 1) * k)]
    big = torch.zeros(((T + 1), k), dtype=torch.int32, device="cuda")
    assert _noalloc_code(big, T + 1, E, k, out) == 2
