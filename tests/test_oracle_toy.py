"""The oracle runs the whole toy workload (T=128, d=512, E=32, k=4, I=256) in seconds."""
import time

import numpy as np

from block_scaled_moe_sigmoid_b200 import synth
from oracle import layer, router


def test_toy_workload_end_to_end():
    wl = synth.WORKLOADS["toy"]
    t0 = time.time()
    x = synth.draw_x(wl).float().numpy()
    W_r, b = (a.numpy() for a in synth.draw_router(wl))
    z = router.router_logits(x, W_r, b)
    idx, w, gap = router.route(z, wl.k)
    cache = {}

    def weights(e):
        if e not in cache:
            cache[e] = layer.decode_expert(layer.quantize_expert(*(a.numpy() for a in synth.draw_expert(wl, e))))
        return cache[e]
    y = layer.moe_layer(x, idx, w, weights)
    assert y.shape == (wl.T, wl.d) and np.all(np.isfinite(y))
    assert np.allclose(w.sum(1), 1.0)
    assert time.time() - t0 < 120
    # outputs are O(0.02^2 * sqrt(d) * sqrt(I)) in size: a sanity bound on the scale
    assert 1e-4 < np.sqrt(np.mean(y ** 2)) < 1.0
