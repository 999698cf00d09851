"""The parallel oracle harness used by the Kimi-K3-shape GPU parity tests, checked on CPU
against the oracle's own single-process layer (small shapes, no GPU)."""
import numpy as np

from block_scaled_moe_sigmoid_b200 import synth
from oracle import layer, mx, router

from . import k3_oracle


def test_fast_expert_quantiser_matches_the_oracle():
    g = np.random.default_rng(3)
    ms = [(g.standard_normal(s) * 0.02).astype(np.float32) for s in ((96, 256), (96, 256), (256, 96))]
    a = k3_oracle.quantize_expert_fast(*ms)
    b = layer.quantize_expert(*ms)
    for name in ("gate", "up", "down"):
        assert np.array_equal(a[name][0], b[name][0]) and np.array_equal(a[name][1], b[name][1])


def test_fast_expert_decoder_matches_the_oracle():
    g = np.random.default_rng(4)
    ms = [(g.standard_normal(s) * 0.02).astype(np.float32) for s in ((64, 256), (64, 256), (256, 64))]
    q = layer.quantize_expert(*ms)
    for a, b in zip(k3_oracle.decode_expert_fast(q), layer.decode_expert(q)):
        assert np.array_equal(a, b)


def test_pool_layer_outputs_match_single_process_oracle():
    wl = synth.custom(seed=8, T=40, d=256, E=8, k=3, I=128, I_shared=128)
    x = synth.draw_x(wl).float().numpy().astype(np.float64)
    W_r, b = synth.draw_router(wl)
    z = router.router_logits(x, W_r.numpy(), b.numpy())
    idx, w, _ = router.route(z, wl.k)
    shared = tuple(t.float().numpy().astype(np.float64) for t in synth.draw_shared(wl))
    q = {e: layer.quantize_expert(*(t.numpy() for t in synth.draw_expert(wl, e))) for e in range(wl.E)}
    tokens = np.array([0, 3, 17, 39])
    y_ref = layer.moe_layer(x, idx, w, lambda e: layer.decode_expert(q[e]), shared, tokens=tokens)
    # one expert's whole row block, with intermediates
    e_st = int(idx[0, 0])
    rows = np.sort(np.argwhere(idx == e_st)[:, 0])
    xq, xs = mx.quantize_mx(x[rows], "e4m3")
    blk = mx.dequantize_mx(xq, xs, "e4m3")
    y, extra = k3_oracle.layer_outputs(wl, x[tokens], idx[tokens], w[tokens], shared,
                                       stage_experts={e_st}, extra_rows={e_st: blk})
    assert np.array_equal(y, y_ref)
    o, a, hq, hs = extra[e_st]
    o2, a2, hq2, hs2 = layer.expert_forward(blk, *layer.decode_expert(q[e_st]))
    assert np.array_equal(o, o2) and np.array_equal(hq, hq2) and np.array_equal(hs, hs2)
