"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle.

Bit-exact: MXFP8 quantised bytes and scales, packed MXFP4 weights, routing indices
given identical logits, the permutation.  Within tolerance: logits, routing weights, the
layer output (max relative error <= 2e-2, mean <= 2e-3 over tokens whose k/k+1 score
gap is >= 1e-6; the others are counted)."""
import numpy as np
import pytest
import torch

from block_scaled_moe_sigmoid_b200 import api, synth
from oracle import layer, mx, permute as operm, router

from .gpu_helpers import Case, decode_tile_major_scales, layer_stats, unpack_expert_codes

pytestmark = pytest.mark.gpu

MAX_REL, MEAN_REL = 2e-2, 2e-3


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    api.lib()


# ------------------------------------------------------------------ a1: MXFP8 quantiser
def _quant_inputs():
    g = torch.Generator().manual_seed(11)
    x = torch.randn(37, 224, generator=g) * torch.logspace(-30, 30, 224).float()  # ragged rows, wide range
    x[0] = 0.0
    x[1, :32] = -0.0
    x[2, :32] = 448.0 * 2.0 ** 10
    x[3, :32] *= 1e-38                 # a block of bf16 subnormals and zeros
    x[3, 5] = float(2.0 ** -133)
    x[4, :32] = torch.tensor([17.0, 19.0, -17.0, 480.0] * 8)
    return x.to(torch.bfloat16)


def test_quant_mxfp8_bit_exact():
    x = _quant_inputs()
    q, s = api.moe_quant_mxfp8(x.cuda())
    q_ref, s_ref = mx.quantize_mx(x.float().numpy().astype(np.float64), "e4m3")
    assert np.array_equal(s.cpu().numpy(), s_ref)
    assert np.array_equal(q.cpu().numpy(), q_ref)


def test_quant_mxfp8_toy_and_empty():
    wl = synth.WORKLOADS["toy"]
    x = synth.draw_x(wl)
    q, s = api.moe_quant_mxfp8(x.cuda())
    q_ref, s_ref = mx.quantize_mx(x.float().numpy().astype(np.float64), "e4m3")
    assert np.array_equal(q.cpu().numpy(), q_ref) and np.array_equal(s.cpu().numpy(), s_ref)
    q0, s0 = api.moe_quant_mxfp8(torch.empty((0, 64), dtype=torch.bfloat16, device="cuda"))
    assert q0.shape == (0, 64)


# ------------------------------------------------------------------ a0: MXFP4 packing
def test_pack_mxfp4_bit_exact():
    wl = synth.custom(seed=5, d=384, I=256, E=3)
    ex = api.Experts(wl.d, wl.I, wl.E)
    for e in range(wl.E):
        ms = synth.draw_expert(wl, e)
        ex.pack(e, *(t.cuda() for t in ms))
        torch.cuda.synchronize()
        got = unpack_expert_codes(ex, e, wl.d, wl.I)
        ref = layer.quantize_expert(*(t.numpy() for t in ms))
        for name in ("gate", "up", "down"):
            assert np.array_equal(got[name][1], ref[name][1]), (e, name, "scales")
            assert np.array_equal(got[name][0], ref[name][0]), (e, name, "codes")


# ------------------------------------------------------------------ a4: permutation
@pytest.mark.parametrize("T,E,k", [(128, 32, 4), (1, 8, 2), (1000, 896, 16), (513, 5, 5)])
def test_permute_bit_exact(T, E, k):
    g = torch.Generator().manual_seed(T + E)
    idx = torch.stack([torch.randperm(E, generator=g)[:k] for _ in range(T)]).to(torch.int32)
    plan = api.Plan(T, 128, E, k, 128)
    counts, offsets, perm_tok, inv = plan.permute(idx.cuda())
    c_ref, o_ref, p_ref, i_ref = operm.permute(idx.numpy(), E)
    assert np.array_equal(counts.cpu().numpy(), c_ref)
    assert np.array_equal(offsets.cpu().numpy(), o_ref)
    assert np.array_equal(perm_tok.cpu().numpy(), p_ref)
    assert np.array_equal(inv.cpu().numpy(), i_ref)
    assert plan.check()[0] == 0


def test_permute_flags_bad_ids():
    plan = api.Plan(4, 128, 8, 2, 128)
    idx = torch.tensor([[0, 1], [2, 9], [3, 4], [5, 6]], dtype=torch.int32, device="cuda")
    _, _, _, inv = plan.permute(idx)
    code, bits = plan.check()
    assert code == 7 and bits & 2
    assert inv[1, 1].item() == -1


# ------------------------------------------------------------------ a2/a3: router
def _check_route(case, atol_z=2e-5):
    T, E, k = case.T, case.wl.E, case.wl.k
    logits = torch.empty((T, E), dtype=torch.float32, device="cuda")
    idx, w = case.plan.route(case.x, case.W_r, case.bias, logits=logits)
    torch.cuda.synchronize()
    z_gpu = logits.cpu().numpy().astype(np.float64)
    z_ref, (idx_o, w_o, gap) = case.oracle_route()
    assert np.max(np.abs(z_gpu - z_ref)) < atol_z
    # bit-exact selection given identical scores (select-only: the key z + b in fp32, as
    # the kernel forms it)
    if case.select_only:
        idx_g, w_g, _ = router.route(logits.cpu().numpy(), k, select_bias=case.bias.cpu().numpy())
    else:
        idx_g, w_g, _ = router.route(z_gpu, k)
    assert np.array_equal(idx.cpu().numpy(), idx_g)
    assert np.allclose(w.cpu().numpy(), w_g, rtol=2e-6, atol=1e-7)
    # against the oracle's own fp64 routing, mismatches only on near ties
    mism = np.any(idx.cpu().numpy() != idx_o, axis=1)
    assert not np.any(mism & (gap >= 1e-6))
    return idx, w, idx_o, w_o, gap


def test_route_toy():
    case = Case(synth.WORKLOADS["toy"])
    _check_route(case)


def test_route_ragged_and_biased():
    wl = synth.custom(seed=3, T=333, d=256, E=40, k=7, I=128)
    bias = -2.4 * torch.log(torch.randperm(40, generator=torch.Generator().manual_seed(1)).double() + 1)
    case = Case(wl, bias=bias)
    _check_route(case)


# ------------------------------------------------------------------ the layer
def _check_layer(case, tokens=None, stage_checks=False):
    idx, w, idx_o, w_o, gap = _check_route(case)
    y = case.plan.forward(case.x, idx, w, case.experts, case.shared)
    assert case.plan.check()[0] == 0
    y = y.float().cpu().numpy().astype(np.float64)
    x = case.x_np()
    rows = np.arange(case.T) if tokens is None else np.asarray(tokens)
    y_ref = layer.moe_layer(x, idx_o, w_o, case.oracle_expert, case.oracle_shared(), tokens=rows, act=case.act)
    st = layer_stats(y[rows], y_ref, gap[rows])
    assert st["max_rel"] <= MAX_REL and st["mean_rel"] <= MEAN_REL, st
    if stage_checks:
        _stage_checks(case, idx.cpu().numpy(), w.cpu().numpy())
    return st


def _stage_checks(case, idx, w):
    """Intermediates in expert order against the oracle on the same routing."""
    wl, T = case.wl, case.T
    A = T * wl.k
    counts, offs, perm_tok, inv = operm.permute(idx, wl.E)
    x = case.x_np()
    xq_ref, xs_ref = mx.quantize_mx(x, "e4m3")
    xq = case.plan.debug_tensor(0, torch.uint8, (A, wl.d)).cpu().numpy()
    bn = api.moe_plan_get_option(case.plan.handle, api.MOE_OPT_TILE_N)
    assert bn in (32, 128, 160, 176)
    ptr, nbytes = api.moe_debug_buffer(case.plan.handle, 1)
    xs = decode_tile_major_scales(case.plan.debug_tensor(1, torch.uint8, (nbytes,)).cpu().numpy(),
                                  counts, wl.d // 128, bn)
    assert np.array_equal(xq, xq_ref[perm_tok])
    assert np.array_equal(xs, xs_ref[perm_tok])
    # GLU output (MXFP8): decoded values agree up to one E4M3 step where fp32 and fp64
    # land on different sides of a rounding boundary
    hq = case.plan.debug_tensor(2, torch.uint8, (A, wl.I)).cpu().numpy()
    ptr, nbytes = api.moe_debug_buffer(case.plan.handle, 3)
    hs = decode_tile_major_scales(case.plan.debug_tensor(3, torch.uint8, (nbytes,)).cpu().numpy(),
                                  counts, wl.I // 128, bn)
    H = mx.dequantize_mx(hq, hs, "e4m3")
    X = mx.dequantize_mx(xq_ref, xs_ref, "e4m3")
    worst, mism = 0.0, 0
    O = case.plan.debug_tensor(4, torch.bfloat16, (A, wl.d)).float().cpu().numpy()
    for e in range(wl.E):
        rows = np.arange(offs[e], offs[e + 1])
        if len(rows) == 0:
            continue
        Wg, Wu, Wd = case.oracle_expert(e)
        o_ref, a_ref, hq_ref, hs_ref = layer.expert_forward(X[perm_tok[rows]], Wg, Wu, Wd, case.act)
        H_ref = mx.dequantize_mx(hq_ref, hs_ref, "e4m3")
        diff = np.abs(H[rows] - H_ref)
        scale = np.repeat(mx.e8m0_value(hs_ref), 32, axis=1)
        mism += int(np.sum(diff > 0))
        worst = max(worst, float(np.max(diff / (np.abs(H_ref) + scale * 2.0 ** -9))))
        # expert outputs (bf16, expert order) against the oracle's, row-normwise
        rel = np.linalg.norm(O[rows] - o_ref, axis=1) / np.linalg.norm(o_ref, axis=1)
        assert rel.max() < 1e-2, (e, rel.max())
    assert worst <= 0.13, worst                      # at most one E4M3 step (2^-3 relative)
    assert mism <= 0.01 * A * wl.I, mism


def test_layer_toy():
    case = Case(synth.WORKLOADS["toy"])
    st = _check_layer(case, stage_checks=True)
    print("toy", st)


def test_layer_with_shared_ragged():
    wl = synth.custom(seed=7, T=203, d=384, E=12, k=3, I=256, I_shared=384)
    case = Case(wl)
    _check_layer(case, stage_checks=True)


def test_layer_single_token_and_empty_experts():
    wl = synth.custom(seed=8, T=1, d=256, E=64, k=4, I=128)
    case = Case(wl)
    _check_layer(case)


def test_layer_hot_experts_span_several_tiles():
    """A bias sends every token to the same experts: each carries T=400 rows, which the
    GEMMs split over 3 tiles of <= 176 rows."""
    wl = synth.custom(seed=9, T=400, d=256, E=16, k=4, I=128, I_shared=128)
    bias = torch.zeros(16)
    bias[[3, 7, 11, 12]] = 40.0
    case = Case(wl, bias=bias)
    _check_layer(case, stage_checks=True)


def test_layer_tile_configs_agree():
    """The three routed-GEMM tile configurations (32 and 176 token rows with the weights on
    the MMA's M side, 128 with the tokens on M) on one input whose hot experts span several
    tiles in each (400 rows: 13 tiles of <= 32 rows, 4 of <= 128, 3 of <= 176): each matches
    the oracle, and all three give the same bytes: the K loop runs in the same order, and
    the tensor core accumulates an output the same way in either orientation."""
    wl = synth.custom(seed=11, T=400, d=256, E=16, k=4, I=128, I_shared=128)
    bias = torch.zeros(16)
    bias[[1, 5, 6, 14]] = 40.0
    case = Case(wl, bias=bias)
    outs = []
    for bn in (32, 128, 176):
        api.moe_plan_set_option(case.plan.handle, api.MOE_OPT_TILE_N, bn)
        _check_layer(case, stage_checks=True)
        assert api.moe_plan_get_option(case.plan.handle, api.MOE_OPT_TILE_N) == bn
        idx, w = case.plan.route(case.x, case.W_r, case.bias)
        outs.append(case.plan.forward(case.x, idx, w, case.experts, case.shared).cpu())
    assert torch.equal(outs[0], outs[1]) and torch.equal(outs[1], outs[2])
    api.moe_plan_set_option(case.plan.handle, api.MOE_OPT_TILE_N, 0)
    with pytest.raises(api.MoeError):
        api.moe_plan_set_option(case.plan.handle, api.MOE_OPT_TILE_N, 64)


def test_layer_cta_pair_config_agrees():
    """The CTA-pair routed GEMM (MOE_OPT_TILE_N = 160: clusters of two CTAs, M=256 MMAs
    over both CTAs' weight rows, the token tile split between them) on a layer with even
    m-tile counts (2I = 512 and d = 512: two 256-row m-tiles each).  Hot experts carry 400
    rows, split into tiles of 144, 144 and 112 rows (MMA N 160, 160, 128); the others a few
    rows (MMA N 32).  The result matches the oracle with the stage checks, and equals the
    single-CTA 176-row configuration byte for byte: each output's K loop runs in the same
    order."""
    wl = synth.custom(seed=25, T=400, d=512, E=16, k=4, I=256, I_shared=128)
    bias = torch.zeros(16)
    bias[[2, 4, 9, 13]] = 40.0
    case = Case(wl, bias=bias)
    outs = []
    for bn in (176, 160):
        api.moe_plan_set_option(case.plan.handle, api.MOE_OPT_TILE_N, bn)
        _check_layer(case, stage_checks=True)
        assert api.moe_plan_get_option(case.plan.handle, api.MOE_OPT_TILE_N) == bn
        idx, w = case.plan.route(case.x, case.W_r, case.bias)
        outs.append(case.plan.forward(case.x, idx, w, case.experts, case.shared).cpu())
    assert torch.equal(outs[0], outs[1])
    api.moe_plan_set_option(case.plan.handle, api.MOE_OPT_TILE_N, 0)


def test_route_select_only_bias():
    """Select-only bias: logits exclude b, experts are chosen by z + b (fp32), weights from
    sigmoid(z).  A strong bias makes the chosen set differ from the unbiased top-k."""
    wl = synth.custom(seed=12, T=300, d=256, E=48, k=6, I=128)
    bias = torch.zeros(48)
    bias[torch.randperm(48, generator=torch.Generator().manual_seed(5))[:10]] = 0.5
    case = Case(wl, bias=bias, select_only=True)
    idx, w, idx_o, w_o, gap = _check_route(case)
    z = router.router_logits(case.x_np(), case.W_r.cpu().numpy())
    plain, _, _ = router.route(z, wl.k)
    assert not np.array_equal(idx.cpu().numpy(), plain)


def test_layer_select_only_bias():
    wl = synth.custom(seed=13, T=160, d=256, E=16, k=4, I=128, I_shared=128)
    bias = torch.linspace(-0.5, 0.5, 16)
    case = Case(wl, bias=bias, select_only=True)
    _check_layer(case, stage_checks=True)


def test_layer_clamped_swiglu():
    """The clamped SwiGLU on routed and shared experts.  x is scaled by 32 (exact in bf16
    and MXFP8) so that many pre-activations pass both clamps (|g|, |u| > 7)."""
    wl = synth.custom(seed=14, T=203, d=384, E=12, k=3, I=256, I_shared=128)
    case = Case(wl, act="clamped_swiglu", x_scale=32.0)
    st = _check_layer(case, stage_checks=True)
    # the clamps are reached: some g of the first expert's rows exceed 7
    Wg, Wu, _ = case.oracle_expert(0)
    xq, xs = mx.quantize_mx(case.x_np(), "e4m3")
    g = mx.dequantize_mx(xq, xs, "e4m3") @ Wg.T
    assert (g > 7).mean() > 0.01 and (np.abs(mx.dequantize_mx(xq, xs, "e4m3") @ Wu.T) > 7).mean() > 0.01
    print("clamped", st)


def test_layer_fused_double_shared_expert():
    """The pages' shared expert is two full-width experts fused into one GLU of twice the
    intermediate size; here I_shared = 2 I."""
    wl = synth.custom(seed=16, T=130, d=256, E=8, k=2, I=128, I_shared=256)
    case = Case(wl)
    _check_layer(case, stage_checks=True)


def test_static_router_flag_reuses_and_refreshes_planes():
    """MOE_FLAG_STATIC_ROUTER: the second call with the same W_r skips the split and gives
    the same logits; a call with another W_r pointer splits that matrix."""
    wl = synth.custom(seed=17, T=64, d=256, E=24, k=4, I=128)
    case = Case(wl)
    plan = api.Plan(wl.T, wl.d, wl.E, wl.k, wl.I, flags=api.MOE_FLAG_STATIC_ROUTER)
    z0 = torch.empty((wl.T, wl.E), device="cuda")
    z1 = torch.empty_like(z0)
    i0, w0 = plan.route(case.x, case.W_r, case.bias, logits=z0)
    i1, w1 = plan.route(case.x, case.W_r, case.bias, logits=z1)
    assert torch.equal(z0, z1) and torch.equal(i0, i1) and torch.equal(w0, w1)
    W2 = (case.W_r * 2.0).contiguous()          # exact scaling: logits double exactly
    z2 = torch.empty_like(z0)
    plan.route(case.x, W2, None, logits=z2)
    zb = torch.empty_like(z0)
    plan.route(case.x, case.W_r, None, logits=zb)
    assert torch.equal(z2, 2.0 * zb)
    assert plan.check()[0] == 0


def test_layer_max_top_k_32():
    """The largest supported k (32) with more experts than one 128-lane router tile."""
    wl = synth.custom(seed=18, T=40, d=256, E=160, k=32, I=128, I_shared=128)
    case = Case(wl)
    _check_layer(case, stage_checks=True)


def _check_latent_layer(case):
    idx, w, idx_o, w_o, gap = _check_route(case)
    y = case.plan.forward(case.x, idx, w, case.experts, case.shared, latent=case.latent)
    assert case.plan.check()[0] == 0
    y = y.float().cpu().numpy().astype(np.float64)
    y_ref = layer.latent_moe_layer(case.x_np(), idx_o, w_o, case.oracle_expert, case.oracle_latent(),
                                   case.oracle_shared(), act=case.act)
    st = layer_stats(y, y_ref, gap)
    assert st["max_rel"] <= MAX_REL and st["mean_rel"] <= MEAN_REL, st
    return st


def test_layer_latent_option():
    """The latent option (experts on a d/2 latent, RMSNorm before them, projections back),
    with a shared expert on the un-projected input and a ragged token count."""
    wl = synth.custom(seed=20, T=150, d=256, E=12, k=3, I=128, I_shared=128, d_latent=128)
    case = Case(wl)
    print("latent", _check_latent_layer(case))


def test_layer_latent_option_wide_and_small_tiles():
    """d_latent spanning two 256-row output tiles of the expert down GEMM (d_latent = 384 of
    d = 512), no shared expert, both GEMM tile configurations."""
    wl = synth.custom(seed=21, T=64, d=512, E=8, k=2, I=128, d_latent=384)
    case = Case(wl)
    for bn in (32, 128, 176):
        api.moe_plan_set_option(case.plan.handle, api.MOE_OPT_TILE_N, bn)
        _check_latent_layer(case)


def test_latent_plan_rejects_the_plain_call_and_bad_shapes():
    wl = synth.custom(seed=22, T=8, d=256, E=4, k=2, I=128, d_latent=128)
    case = Case(wl)
    idx, w = case.plan.route(case.x, case.W_r, case.bias)
    with pytest.raises(api.MoeError):
        api.moe_forward(case.plan.handle, case.x, idx, w, case.experts, None)
    h = api.moe_plan_create(8, 256, 4, 2, 128)
    L = api.lib()
    import ctypes
    assert L.moe_plan_set_latent(h, 100, ctypes.c_float(1e-5)) == 2     # not a multiple of 128
    assert L.moe_plan_set_latent(h, 384, ctypes.c_float(1e-5)) == 1     # wider than d
    assert L.moe_plan_set_latent(h, 128, ctypes.c_float(0.0)) == 1      # eps must be > 0
    api.moe_plan_destroy(h)


def test_layer_shared_expert_split_k():
    """Few tokens and a wide d: the shared expert's dense GEMMs split K over the SMs (fp32
    partials, then sum + GLU, and sum); the layer still matches the oracle and repeats
    bit for bit."""
    wl = synth.custom(seed=23, T=40, d=1024, E=8, k=2, I=128, I_shared=1024)
    case = Case(wl)
    st = _check_layer(case)
    assert api.moe_plan_get_option(case.plan.handle, api.MOE_OPT_SHARED_SPLIT) > 1
    assert api.moe_plan_get_option(case.plan.handle, api.MOE_OPT_SHARED_SPLIT_DOWN) > 1
    idx, w = case.plan.route(case.x, case.W_r, case.bias)
    y1 = case.plan.forward(case.x, idx, w, case.experts, case.shared).clone()
    y2 = case.plan.forward(case.x, idx, w, case.experts, case.shared)
    assert torch.equal(y1, y2)
    print("shared split", st)


def test_layer_clamped_swiglu_with_shared_split_k():
    """The clamped SwiGLU through the split-K shared expert (partials summed, then the
    clamped GLU in the reduction kernel)."""
    wl = synth.custom(seed=24, T=40, d=1024, E=8, k=2, I=128, I_shared=1024)
    case = Case(wl, act="clamped_swiglu", x_scale=8.0)
    _check_layer(case)
    assert api.moe_plan_get_option(case.plan.handle, api.MOE_OPT_SHARED_SPLIT) > 1


def test_layer_dense_mixture_k_equals_e():
    wl = synth.custom(seed=10, T=50, d=256, E=4, k=4, I=128)
    case = Case(wl)
    _check_layer(case)


def test_forward_t0_is_noop():
    wl = synth.custom(seed=1, T=4, d=128, E=4, k=2, I=128)
    case = Case(wl)
    y = torch.full((0, 128), 1.0, dtype=torch.bfloat16, device="cuda")
    idx = torch.zeros((0, 2), dtype=torch.int32, device="cuda")
    w = torch.zeros((0, 2), dtype=torch.float32, device="cuda")
    case.plan.forward(y, idx, w, case.experts, None, y=y)


def test_forward_rejects_bad_arguments():
    wl = synth.custom(seed=1, T=4, d=128, E=4, k=2, I=128)
    case = Case(wl)
    idx = torch.zeros((4, 2), dtype=torch.int32, device="cuda")
    w = torch.zeros((4, 2), dtype=torch.float32, device="cuda")
    with pytest.raises(api.MoeError) as e:        # T > T_max
        big = torch.zeros((8, 128), dtype=torch.bfloat16, device="cuda")
        case.plan.forward(big, torch.zeros((8, 2), dtype=torch.int32, device="cuda"),
                          torch.zeros((8, 2), device="cuda"), case.experts)
    assert e.value.code == 2
    with pytest.raises(api.MoeError) as e:        # misaligned x
        raw = torch.zeros(4 * 128 + 8, dtype=torch.bfloat16, device="cuda")
        case.plan.forward(raw[1:1 + 512].view(4, 128), idx, w, case.experts)
    assert e.value.code == 3


def test_route_and_forward_replay_from_a_cuda_graph():
    """moe_route + moe_forward make no host synchronisation and allocate nothing, so a
    whole layer step can be captured into a CUDA graph; replays reproduce the eager bytes."""
    wl = synth.custom(seed=15, T=96, d=256, E=16, k=4, I=128, I_shared=128)
    case = Case(wl)
    idx = torch.empty((wl.T, wl.k), dtype=torch.int32, device="cuda")
    w = torch.empty((wl.T, wl.k), dtype=torch.float32, device="cuda")
    y = torch.empty((wl.T, wl.d), dtype=torch.bfloat16, device="cuda")
    s = torch.cuda.Stream()

    def step():
        api.moe_route(case.plan.handle, case.x, case.W_r, case.bias, wl.k, idx=idx, w=w, stream=s)
        api.moe_forward(case.plan.handle, case.x, idx, w, case.experts, case.shared, y, stream=s)

    with torch.cuda.stream(s):
        step()                              # eager run (also sets the kernels' attributes)
    s.synchronize()
    y_eager = y.clone()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        step()
    y.zero_()
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    assert torch.equal(y, y_eager)
    assert case.plan.check()[0] == 0


@pytest.mark.parametrize("E,k,select_only,T", [(96, 8, False, 40), (600, 16, False, 40), (1100, 32, False, 40),
                                                 (2100, 16, False, 40), (64, 4, True, 40), (300, 24, True, 40),
                                                 (896, 16, False, 1301), (160, 32, True, 1301)])
def test_route_exact_ties_lower_index_wins(E, k, select_only, T):
    """Exact ties in the selection key: duplicated router columns give equal logits, an
    all-zero token gives every expert the logit +0 (and -0 where the bias is -0), and in the
    select-only mode equal keys come from different (z, b) pairs.  The selection on the
    GPU's own logits must equal the oracle's (descending key, lower index first) for every
    width of the selection kernel's first stage (1, 2, 4, 8 and 16 experts per lane: E up
    to 256, 512, 1024, 2048, 4096), through both forms of its second stage (candidates
    above the lane-maxima threshold; and, for the all-zero token, whose keys all tie, the
    scan of every key), and with T = 1301 in 8-token groups, a ragged last group
    included."""
    d = 128
    g = torch.Generator().manual_seed(E + k)
    x = torch.randn((T, d), generator=g).to(torch.bfloat16)
    x[3] = 0.0
    W_r = torch.randn((d, E), generator=g) * 0.02
    W_r[:, 1::3] = W_r[:, 0::3][:, :W_r[:, 1::3].shape[1]]       # every third pair of experts ties
    b = torch.zeros(E)
    b[::5] = -0.0
    if select_only:
        b = torch.randint(-2, 3, (E,), generator=g).float() * 0.5
    plan = api.Plan(T, d, E, k, 128, bias_mode=api.MOE_BIAS_SELECT_ONLY if select_only else api.MOE_BIAS_LOGIT)
    logits = torch.empty((T, E), dtype=torch.float32, device="cuda")
    idx, w = plan.route(x.cuda(), W_r.cuda(), b.cuda(), logits=logits)
    z = logits.cpu().numpy()
    if select_only:
        idx_g, w_g, _ = router.route(z, k, select_bias=b.numpy())
    else:
        idx_g, w_g, _ = router.route(z.astype(np.float64), k)
    assert np.array_equal(idx.cpu().numpy(), idx_g)
    assert np.allclose(w.cpu().numpy(), w_g, rtol=2e-6, atol=1e-7)
    if not select_only:
        assert list(idx[3].cpu().numpy()) == list(range(k))     # all logits tie at zero
