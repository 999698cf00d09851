"""GPU parity at the full Kimi-K3 shapes (d=7168, 896 experts, top-16, I=3072, one bf16
shared expert), in the launch configuration the benchmark times.

Checked on every token: router logits against fp64 (sampled rows), bit-exact top-k on
the GPU's own logits (all rows), bit-exact permutation and MXFP8 bytes (all rows), finite
outputs.  Checked on sampled tokens: the layer output against the fp64 oracle (the
oracle quantises each touched expert's fp32 masters itself, in a process pool)."""
import multiprocessing as mp
import os

import numpy as np
import pytest
import torch

from block_scaled_moe_sigmoid_b200 import api, synth
from oracle import layer, mx, permute as operm, router

from .gpu_helpers import layer_stats

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

MAX_REL, MEAN_REL = 2e-2, 2e-3


class K3Case:
    def __init__(self, wl, T):
        self.wl, self.T = wl, T
        self.x = synth.draw_x(wl, T, device="cuda")
        self.W_r, self.bias = synth.draw_router(wl, device="cuda")
        self.plan = api.Plan(T, wl.d, wl.E, wl.k, wl.I, wl.I_shared)
        self.experts = api.Experts(wl.d, wl.I, wl.E)
        for e in range(wl.E):
            self.experts.pack(e, *synth.draw_expert(wl, e, device="cuda"))
        self.shared = api.Shared(wl.d, wl.I_shared)
        self.shared_w = synth.draw_shared(wl, device="cuda")
        self.shared.pack(*self.shared_w)
        torch.cuda.synchronize()

    def run(self):
        wl, T = self.wl, self.T
        self.logits = torch.empty((T, wl.E), dtype=torch.float32, device="cuda")
        self.idx, self.w = self.plan.route(self.x, self.W_r, self.bias, logits=self.logits)
        self.y = self.plan.forward(self.x, self.idx, self.w, self.experts, self.shared)
        code, bits = self.plan.check()
        assert code == 0, (code, bits)

    def free(self):
        for name in ("experts", "shared", "plan", "x", "logits", "y"):
            if hasattr(self, name):
                delattr(self, name)
        torch.cuda.empty_cache()


def _check(case, sample_tokens, logit_rows=64):
    wl, T = case.wl, case.T
    case.run()
    x = case.x.float().cpu().numpy().astype(np.float64)
    z_gpu = case.logits.cpu().numpy().astype(np.float64)
    idx = case.idx.cpu().numpy()
    w = case.w.cpu().numpy()
    y = case.y.float().cpu().numpy().astype(np.float64)
    assert np.all(np.isfinite(y))

    # router: fp64 logits on sampled rows; bit-exact top-k on the GPU logits for every row
    W_r, bias = case.W_r.cpu().numpy(), case.bias.cpu().numpy()
    g = np.random.default_rng(T)
    rows = np.unique(np.concatenate([g.choice(T, size=min(logit_rows, T), replace=False), sample_tokens]))
    z_ref = router.router_logits(x[rows], W_r, bias)
    assert np.max(np.abs(z_gpu[rows] - z_ref)) < 5e-5
    idx_g, w_g, _ = router.route(z_gpu, wl.k)
    assert np.array_equal(idx, idx_g)
    assert np.allclose(w, w_g, rtol=2e-6, atol=1e-7)
    idx_o, w_o, gap = router.route(z_ref, wl.k)
    assert not np.any(np.any(idx[rows] != idx_o, axis=1) & (gap >= 1e-6))

    # permutation (bit-exact, every assignment) and the MXFP8 activations in expert order
    counts, offsets, perm_tok, inv = case.plan.permute(case.idx)
    c_ref, o_ref, p_ref, i_ref = operm.permute(idx, wl.E)
    assert np.array_equal(counts.cpu().numpy(), c_ref) and np.array_equal(offsets.cpu().numpy(), o_ref)
    assert np.array_equal(perm_tok.cpu().numpy(), p_ref) and np.array_equal(inv.cpu().numpy(), i_ref)
    qrows = rows if T > 8192 else np.arange(T)          # every row up to the prefill size
    xq_ref, xs_ref = mx.quantize_mx(x[qrows], "e4m3")
    q_gpu, s_gpu = api.moe_quant_mxfp8(case.x)
    assert np.array_equal(q_gpu.cpu().numpy()[qrows], xq_ref)
    assert np.array_equal(s_gpu.cpu().numpy()[qrows], xs_ref)
    # the forward pass's own copy in expert order (first row of each sampled token's slots)
    xq_perm = case.plan.debug_tensor(0, torch.uint8, (T * wl.k, wl.d))
    for t in sample_tokens:
        pos = i_ref[t]
        ref_q, _ = mx.quantize_mx(x[t:t + 1], "e4m3")
        assert np.array_equal(xq_perm[torch.as_tensor(pos, device="cuda").long()].cpu().numpy(),
                              np.repeat(ref_q, len(pos), axis=0))

    # layer output on the sampled tokens
    st_rows = np.asarray(sample_tokens)
    need = sorted(set(int(e) for e in idx_o[np.searchsorted(rows, st_rows)].ravel()))
    masters = {e: tuple(t.cpu().numpy() for t in synth.draw_expert(wl, e, device="cuda")) for e in need}
    ctx = mp.get_context("spawn")
    with ctx.Pool(min(8, os.cpu_count() or 1)) as pool:
        quant = dict(zip(need, pool.starmap(layer.quantize_expert, [masters[e] for e in need])))
    del masters
    shared = tuple(t.float().cpu().numpy().astype(np.float64) for t in case.shared_w)
    y_ref = layer.moe_layer(x[st_rows], idx_o[np.searchsorted(rows, st_rows)],
                            w_o[np.searchsorted(rows, st_rows)],
                            lambda e: layer.decode_expert(quant[e]), shared)
    st = layer_stats(y[st_rows], y_ref, gap[np.searchsorted(rows, st_rows)])
    print(wl.name, T, st)
    assert st["max_rel"] <= MAX_REL and st["mean_rel"] <= MEAN_REL, st
    return st


@pytest.fixture(autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")


def test_k3_decode_t64():
    case = K3Case(synth.WORKLOADS["k3_decode_t64"], 64)
    try:
        _check(case, sample_tokens=[5, 63])
    finally:
        case.free()


def test_k3_prefill_t8192():
    case = K3Case(synth.WORKLOADS["k3_prefill_t8192"], 8192)
    try:
        _check(case, sample_tokens=[0, 8191])
    finally:
        case.free()


def test_k3_skewed_t32768():
    """Zipf-like logit bias: hot experts get thousands of rows (many GEMM tiles each)."""
    wl = synth.WORKLOADS["k3_skewed_t32768"]
    case = K3Case(wl, 32768)
    try:
        st = _check(case, sample_tokens=[12345], logit_rows=32)
        counts = np.bincount(case.idx.cpu().numpy().ravel(), minlength=wl.E)
        assert counts.max() > 5 * counts.mean()       # the load really is skewed
        print("skewed load: max", counts.max(), "experts used", int((counts > 0).sum()))
    finally:
        case.free()
