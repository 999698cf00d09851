"""Pins for the oracle's layer (oracle/layer.py): brute-force scalar loops on a
tiny shape, special cases that reduce to a dense GLU MLP (checked against
torch.nn.functional in float64), routing invariance when all experts are equal,
and the dense-mixture case k = E."""
import math

import numpy as np
import torch
import torch.nn.functional as F

from oracle import layer, mx, router

T, D, E, K, I = 3, 64, 4, 2, 32          # d != I so a transposed operand fails


def _experts(rng, E_, d, I_):
    Ws = []
    for _ in range(E_):
        q = layer.quantize_expert(rng.standard_normal((I_, d)) * 0.02,
                                  rng.standard_normal((I_, d)) * 0.02,
                                  rng.standard_normal((d, I_)) * 0.02)
        Ws.append(layer.decode_expert(q))
    return Ws


def _bf16(a):
    return torch.from_numpy(np.asarray(a, np.float32)).to(torch.bfloat16).to(torch.float64).numpy()


def _brute_force_mismatch(seed=0):
    """Largest |oracle - scalar-loop reference| in bf16 ulps of the reference, on
    the tiny shape, with a shared expert."""
    rng = np.random.default_rng(seed)
    x = _bf16(rng.standard_normal((T, D)))
    Ws = _experts(rng, E, D, I)
    shared = tuple(_bf16(rng.standard_normal(s) * 0.02) for s in ((I, D), (I, D), (D, I)))
    z = rng.standard_normal((T, E))
    idx, w, _ = router.route(z, K)
    y = layer.moe_layer(x, idx, w, lambda e: Ws[e], shared)

    xq, xs = mx.quantize_mx(x, "e4m3")
    X = mx.dequantize_mx(xq, xs, "e4m3")
    worst = 0.0
    for t in range(T):
        acc = [0.0] * D
        h = []                                   # shared expert, scalar loops
        for n in range(I):
            g = sum(x[t, i] * shared[0][n, i] for i in range(D))
            u = sum(x[t, i] * shared[1][n, i] for i in range(D))
            h.append(g / (1 + math.exp(-g)) * u)
        h = list(mx.bf16_round(np.array(h)))
        for c in range(D):
            acc[c] += sum(h[n] * shared[2][c, n] for n in range(I))
        for j in range(K):
            Wg, Wu, Wd = Ws[idx[t, j]]
            a = []
            for n in range(I):
                g = sum(X[t, i] * Wg[n, i] for i in range(D))
                u = sum(X[t, i] * Wu[n, i] for i in range(D))
                a.append(g / (1 + math.exp(-g)) * u)
            hq, hs = mx.quantize_mx(np.array(a)[None], "e4m3")
            H = mx.dequantize_mx(hq, hs, "e4m3")[0]
            for c in range(D):
                acc[c] += w[t, j] * sum(H[n] * Wd[c, n] for n in range(I))
        ref = mx.bf16_round(np.array(acc))
        ulp = 2.0 ** (np.floor(np.log2(np.maximum(np.abs(ref), 2.0 ** -126))) - 7)
        worst = max(worst, float(np.max(np.abs(y[t] - ref) / ulp)))
    return worst


def test_brute_force_tiny():
    # summation order differs (BLAS vs scalar loops) only in the last fp64 bits,
    # so the bf16 outputs agree to at most one ulp on a rounding boundary
    for seed in range(3):
        assert _brute_force_mismatch(seed) <= 1.0


def test_planted_mistakes_are_caught(monkeypatch):
    """Plausible oracle bugs, planted on the CPU, each break the brute-force pin."""
    good_hidden = layer.expert_hidden
    mutants = {
        "gate/up swapped": lambda X, Wg, Wu, act="silu": good_hidden(X, Wu, Wg, act),
        "sigmoid sign": lambda X, Wg, Wu, act="silu": (lambda g: g / (1 + np.exp(g)))(X @ Wg.T) * (X @ Wu.T),
        "no activation": lambda X, Wg, Wu, act="silu": (X @ Wg.T) * (X @ Wu.T),
    }
    for name, fn in mutants.items():
        monkeypatch.setattr(layer, "expert_hidden", fn)
        assert _brute_force_mismatch(0) > 1.0, name
    monkeypatch.setattr(layer, "expert_hidden", good_hidden)

    def no_requant(X, Wg, Wu, Wd, act="silu"):
        a = good_hidden(X, Wg, Wu, act)
        hq, hs = mx.quantize_mx(a, "e4m3")
        return a @ Wd.T, a, hq, hs
    monkeypatch.setattr(layer, "expert_forward", no_requant)
    assert _brute_force_mismatch(0) > 1.0, "requant dropped"


def test_single_expert_is_dense_glu_mlp_torch():
    rng = np.random.default_rng(1)
    x = _bf16(rng.standard_normal((16, 128)))
    Ws = _experts(rng, 1, 128, 64)
    idx = np.zeros((16, 1), np.int32)
    w = np.ones((16, 1))
    y = layer.moe_layer(x, idx, w, lambda e: Ws[0])
    xq, xs = mx.quantize_mx(x, "e4m3")
    X = torch.from_numpy(mx.dequantize_mx(xq, xs, "e4m3"))
    Wg, Wu, Wd = (torch.from_numpy(a) for a in Ws[0])
    a = F.silu(F.linear(X, Wg)) * F.linear(X, Wu)
    hq, hs = mx.quantize_mx(a.numpy(), "e4m3")
    o = F.linear(torch.from_numpy(mx.dequantize_mx(hq, hs, "e4m3")), Wd).numpy()
    assert np.array_equal(y, mx.bf16_round(o))


def test_shared_expert_torch():
    rng = np.random.default_rng(2)
    x = _bf16(rng.standard_normal((8, 96)))
    Wsg, Wsu, Wsd = (_bf16(rng.standard_normal(s) * 0.02) for s in ((48, 96), (48, 96), (96, 48)))
    ys, h = layer.shared_expert(x, Wsg, Wsu, Wsd)
    xt = torch.from_numpy(x)
    ht = F.silu(F.linear(xt, torch.from_numpy(Wsg))) * F.linear(xt, torch.from_numpy(Wsu))
    hb = ht.to(torch.bfloat16).to(torch.float64)
    # torch may round through fp32; allow a one-ulp bf16 difference on rare ties
    assert np.all(np.abs(h - hb.numpy()) <= 2.0 ** -7 * np.abs(hb.numpy()))
    assert np.allclose(ys, F.linear(torch.from_numpy(h), torch.from_numpy(Wsd)).numpy(), rtol=1e-12, atol=1e-15)


def test_equal_experts_make_routing_irrelevant():
    rng = np.random.default_rng(3)
    x = _bf16(rng.standard_normal((10, 64)))
    W = _experts(rng, 1, 64, 32)[0]
    z1, z2 = rng.standard_normal((10, 6)), rng.standard_normal((10, 6))
    i1, w1, _ = router.route(z1, 3)
    i2, w2, _ = router.route(z2, 3)
    y1 = layer.moe_layer(x, i1, w1, lambda e: W)
    y2 = layer.moe_layer(x, i2, w2, lambda e: W)
    y0 = layer.moe_layer(x, np.zeros((10, 1), np.int32), np.ones((10, 1)), lambda e: W)
    # weights sum to one, so every routing gives the single expert's output (up to fp64 sums)
    assert np.max(np.abs(y1 - y0)) <= 2.0 ** -7 * np.max(np.abs(y0))
    assert np.max(np.abs(y2 - y0)) <= 2.0 ** -7 * np.max(np.abs(y0))


def test_dense_mixture_k_equals_e():
    rng = np.random.default_rng(4)
    x = _bf16(rng.standard_normal((5, 64)))
    Ws = _experts(rng, 4, 64, 32)
    z = rng.standard_normal((5, 4))
    idx, w, _ = router.route(z, 4)
    y, inter = layer.moe_layer(x, idx, w, lambda e: Ws[e], want_intermediates=True)
    s = router.sigmoid(z)
    wd = s / s.sum(1, keepdims=True)
    for t in range(5):
        acc = np.zeros(64)
        for e in range(4):
            j = list(idx[t]).index(e)
            acc += wd[t, e] * inter["o"][t, j]
        assert np.array_equal(y[t], mx.bf16_round(acc)) or np.max(np.abs(y[t] - mx.bf16_round(acc))) <= 2 ** -8 * np.max(np.abs(acc))


def test_token_subset_matches_full():
    rng = np.random.default_rng(5)
    x = _bf16(rng.standard_normal((12, 64)))
    Ws = _experts(rng, 5, 64, 32)
    idx, w, _ = router.route(rng.standard_normal((12, 5)), 2)
    y = layer.moe_layer(x, idx, w, lambda e: Ws[e])
    ys = layer.moe_layer(x, idx, w, lambda e: Ws[e], tokens=[3, 7, 11])
    assert np.array_equal(ys, y[[3, 7, 11]])


def test_relative_error_definition():
    y_ref = np.array([[1.0, -2.0, 0.0, 0.5]])
    y = y_ref + np.array([[0.01, 0.0, 0.001, 0.0]])
    r, nw = layer.relative_errors(y, y_ref)
    rms = math.sqrt((1 + 4 + 0 + 0.25) / 4)
    assert abs(r[0, 0] - 0.01 / max(1.0, rms)) < 1e-15
    assert abs(r[0, 2] - 0.001 / rms) < 1e-15
    assert abs(nw[0] - math.sqrt(0.01 ** 2 + 0.001 ** 2) / math.sqrt(5.25)) < 1e-15


# ------------------------------------------------------------------ clamped SwiGLU (R21)
def test_clamped_swiglu_inside_the_clamps_is_scaled_torch_silu():
    """Inside the clamps, (u + 1) * g * sigmoid(1.702 g) equals (u + 1) * silu(1.702 g) / 1.702.
    torch's silu (a library routine) pins the sigmoid factor and which operand is the gate."""
    rng = np.random.default_rng(11)
    g = rng.uniform(-12.0, 7.0, 4096)
    u = rng.uniform(-7.0, 7.0, 4096)
    a = layer.ACTIVATIONS["clamped_swiglu"](g, u)
    ref = (torch.from_numpy(u) + 1.0) * F.silu(1.702 * torch.from_numpy(g)) / 1.702
    assert np.allclose(a, ref.numpy(), rtol=1e-14, atol=1e-300)
    # a gate/linear swap fails the pin (the two operands play different roles)
    assert not np.allclose(layer.ACTIVATIONS["clamped_swiglu"](u, g), ref.numpy(), rtol=1e-6)


def test_clamped_swiglu_clamps_and_zeros():
    f = layer.ACTIVATIONS["clamped_swiglu"]
    g = np.array([7.0, 7.5, 100.0, 1e30])
    u = np.array([0.3, 0.3, 0.3, 0.3])
    assert np.all(f(g, u) == f(np.full(4, 7.0), u))          # gate clamped from above at 7
    assert f(-50.0, 1.0) != f(-7.0, 1.0)                      # ... but not from below
    assert f(2.0, 9.0) == f(2.0, 7.0) and f(2.0, -9.0) == f(2.0, -7.0)   # linear branch to [-7, 7]
    assert f(3.0, -1.0) == 0.0 and f(0.0, 5.0) == 0.0        # (u + 1) and g factors
    assert f(2.0, -7.0) == -6.0 * f(2.0, 0.0)                 # (u + 1) is linear in u


def test_single_expert_clamped_swiglu_torch():
    """E = k = 1 with the clamped SwiGLU reduces to one dense MLP (torch float64 GEMMs)."""
    rng = np.random.default_rng(12)
    x = _bf16(rng.standard_normal((16, 128)) * 3.0)
    Ws = _experts(rng, 1, 128, 64)
    Ws = [tuple(W * 40.0 for W in Ws[0])]       # large pre-activations reach both clamps
    idx = np.zeros((16, 1), np.int32)
    w = np.ones((16, 1))
    y = layer.moe_layer(x, idx, w, lambda e: Ws[0], act="clamped_swiglu")
    xq, xs = mx.quantize_mx(x, "e4m3")
    X = torch.from_numpy(mx.dequantize_mx(xq, xs, "e4m3"))
    Wg, Wu, Wd = (torch.from_numpy(a) for a in Ws[0])
    g, u = F.linear(X, Wg), F.linear(X, Wu)
    assert (g > 7).any() and (u.abs() > 7).any()
    gc, uc = g.clamp(max=7.0), u.clamp(-7.0, 7.0)
    a = (uc + 1.0) * F.silu(1.702 * gc) / 1.702
    hq, hs = mx.quantize_mx(a.numpy(), "e4m3")
    o = F.linear(torch.from_numpy(mx.dequantize_mx(hq, hs, "e4m3")), Wd).numpy()
    assert np.allclose(y, mx.bf16_round(o), rtol=2 ** -7, atol=0)


# ------------------------------------------------------------------ latent option (R22)
def test_rms_norm_matches_torch():
    rng = np.random.default_rng(31)
    v = rng.standard_normal((9, 96)) * rng.uniform(0.01, 30.0, (9, 1))
    gamma = rng.uniform(0.5, 1.5, 96)
    ref = F.rms_norm(torch.from_numpy(v), (96,), torch.from_numpy(gamma), eps=1e-5).numpy()
    assert np.allclose(layer.rms_norm(v, gamma), ref, rtol=1e-13, atol=0)


def test_latent_single_expert_is_dense_pipeline_torch():
    """E = k = 1 in the latent option: x -> W_ld -> RMSNorm -> bf16 -> one quantised GLU MLP
    -> bf16 -> W_lu, plus the shared expert, all through torch float64 linears."""
    rng = np.random.default_rng(32)
    T, d, dl, I = 12, 128, 64, 32
    x = _bf16(rng.standard_normal((T, d)))
    W_ld = _bf16(rng.standard_normal((dl, d)) * 0.05)
    W_lu = _bf16(rng.standard_normal((d, dl)) * 0.05)
    gamma = rng.uniform(0.5, 1.5, dl)
    Ws = _experts(rng, 1, dl, I)
    shared = tuple(_bf16(rng.standard_normal(sh) * 0.02) for sh in ((48, d), (48, d), (d, 48)))
    idx = np.zeros((T, 1), np.int32)
    w = np.ones((T, 1))
    y = layer.latent_moe_layer(x, idx, w, lambda e: Ws[0], (W_ld, gamma, W_lu), shared)

    xt = torch.from_numpy(x)
    xl = F.linear(xt, torch.from_numpy(W_ld))
    xn = F.rms_norm(xl, (dl,), torch.from_numpy(gamma), eps=1e-5).to(torch.bfloat16).to(torch.float64)
    xq, xs = mx.quantize_mx(xn.numpy(), "e4m3")
    X = torch.from_numpy(mx.dequantize_mx(xq, xs, "e4m3"))
    Wg, Wu, Wd = (torch.from_numpy(a) for a in Ws[0])
    a = F.silu(F.linear(X, Wg)) * F.linear(X, Wu)
    hq, hs = mx.quantize_mx(a.numpy(), "e4m3")
    o = F.linear(torch.from_numpy(mx.dequantize_mx(hq, hs, "e4m3")), Wd)
    yl = o.to(torch.bfloat16).to(torch.float64)
    yr = F.linear(yl, torch.from_numpy(W_lu))
    ys, _ = layer.shared_expert(x, *shared)
    ref = mx.bf16_round(yr.numpy() + ys)
    # torch's rms_norm and the bf16 casts may round a few elements differently from fp64
    assert np.mean(y == ref) > 0.98
    assert np.allclose(y, ref, rtol=2 ** -6, atol=1e-6)


def test_latent_routing_slices_and_token_subset():
    """Rows of a token subset equal the same rows of the full computation."""
    rng = np.random.default_rng(33)
    T, d, dl, I, E, k = 20, 128, 64, 32, 4, 2
    x = _bf16(rng.standard_normal((T, d)))
    lat = (_bf16(rng.standard_normal((dl, d)) * 0.05), rng.uniform(0.5, 1.5, dl),
           _bf16(rng.standard_normal((d, dl)) * 0.05))
    Ws = _experts(rng, E, dl, I)
    idx = np.stack([rng.choice(E, k, replace=False) for _ in range(T)]).astype(np.int32)
    w = rng.uniform(0.1, 1.0, (T, k))
    full = layer.latent_moe_layer(x, idx, w, lambda e: Ws[e], lat)
    rows = np.array([3, 7, 19])
    assert np.array_equal(layer.latent_moe_layer(x, idx, w, lambda e: Ws[e], lat, tokens=rows), full[rows])
