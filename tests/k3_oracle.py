"""Parallel fp64 oracle evaluation at the Kimi-K3 shapes, for the GPU parity tests.

At d=7168, I=3072 one expert costs the oracle a few seconds (MXFP4-quantising and decoding
its 66M weights), and a full-shape parity case touches hundreds of experts.  This module
spreads the per-expert work over a process pool (spawn start method):

  * the parent draws each needed expert's fp32 masters with the shared seeded generator
    (on the GPU, as the workload defines) and hands them to a worker in shared memory;
  * the worker quantises them with the oracle's C restatement of the MX quantiser
    (``oracle.cmx``, pinned bit-exact against ``oracle.mx``), decodes them with
    ``oracle.layer`` and runs ``oracle.layer.expert_forward`` on the MXFP8-decoded token
    rows routed to that expert;
  * the parent assembles the per-slot outputs and finishes with ``oracle.layer`` (shared
    expert, combine).

Nothing here reads kernel output: the token rows, routing and weights are the oracle's own
(routing from fp64 logits), so the only thing compared against the GPU is the result.
"""
import os
from collections import deque

import numpy as np
import torch

from block_scaled_moe_sigmoid_b200 import synth
from oracle import cmx, layer, mx

def pool_size():
    """Worker processes: the usable cores, bounded by host memory (~1.5 GB per worker)."""
    try:
        cores = len(os.sched_getaffinity(0))
    except AttributeError:
        cores = os.cpu_count() or 1
    n = max(1, min(cores, 48))
    try:
        import psutil
        n = max(1, min(n, int(psutil.virtual_memory().available / 1.5e9) - 2))
    except Exception:
        pass
    return n


def quantize_expert_fast(W_gate, W_up, W_down):
    """The same dict as oracle.layer.quantize_expert for fp32 masters, from the C
    restatement of the MX quantiser (oracle/cmx.c, pinned bit-exact against
    oracle.mx.quantize_mx)."""
    return {"gate": cmx.quantize_mx_f32(W_gate, "e2m1"), "up": cmx.quantize_mx_f32(W_up, "e2m1"),
            "down": cmx.quantize_mx_f32(W_down, "e2m1")}


def expert_job(w_gate, w_up, w_down, blocks, want_stage, act):
    """Worker: one expert's oracle outputs for several blocks of decoded token rows.

    w_*: fp32 masters (torch CPU tensors in shared memory); blocks: list of fp64 [R, d]
    arrays.  Returns, per block, (o,) or, with want_stage, (o, a, hq, hs)."""
    torch.set_num_threads(1)
    q = quantize_expert_fast(w_gate.numpy(), w_up.numpy(), w_down.numpy())
    Wg, Wu, Wd = layer.decode_expert(q)
    out = []
    for X in blocks:
        o, a, hq, hs = layer.expert_forward(X, Wg, Wu, Wd, act)
        out.append((o, a, hq, hs) if want_stage else (o,))
    return out


def run_experts(wl, jobs, stage_experts=(), act="silu", device=None):
    """jobs: {expert: [fp64 [R, d] token-row block, ...]} -> {expert: [result per block]}.

    Results are expert_job's tuples; experts in `stage_experts` also return the GLU values
    and their MXFP8 codes and scales."""
    import torch.multiprocessing as tmp
    device = wl.device if device is None else device
    n = pool_size()
    ctx = tmp.get_context("spawn")
    results = {}
    with ctx.Pool(n) as pool:
        inflight = deque()
        for e in sorted(jobs):
            while len(inflight) >= 2 * n:            # bound the masters held in shared memory
                e0, r0 = inflight.popleft()
                results[e0] = r0.get()
            ms = [t.cpu().share_memory_() for t in synth.draw_expert(wl, e, device=device)]
            inflight.append((e, pool.apply_async(expert_job, (*ms, jobs[e], e in stage_experts, act))))
            del ms
        while inflight:
            e0, r0 = inflight.popleft()
            results[e0] = r0.get()
    return results


def layer_outputs(wl, x_rows, idx, w, shared, act="silu", stage_experts=(), extra_rows=None):
    """Oracle layer output for the given tokens.

    x_rows: fp64 [n, d] bf16 token values; idx, w: [n, k] oracle routing of those tokens;
    shared: None or the shared expert's (Wsg, Wsu, Wsd) bf16 values.  extra_rows maps an
    expert to an fp64 [R, d] block of MXFP8-decoded rows whose outputs (and, for experts
    in stage_experts, GLU values / codes / scales) are returned as well.
    Returns (y fp64 [n, d] holding bf16 values, {expert: result of its extra block})."""
    n, k = idx.shape
    xq, xs = mx.quantize_mx(x_rows, "e4m3")
    X = mx.dequantize_mx(xq, xs, "e4m3")
    jobs, where = {}, {}
    for e in np.unique(idx):
        sel = np.argwhere(idx == e)                   # (row, slot) pairs
        jobs[int(e)] = [X[sel[:, 0]]]
        where[int(e)] = sel
    extra_rows = extra_rows or {}
    for e, blk in extra_rows.items():
        jobs.setdefault(int(e), []).append(blk)
    res = run_experts(wl, jobs, stage_experts=stage_experts, act=act)
    o = np.zeros((n, k, x_rows.shape[1]))
    for e, sel in where.items():
        o[sel[:, 0], sel[:, 1]] = res[e][0][0]
    ys = layer.shared_expert(x_rows, *shared, act=act)[0] if shared is not None else np.zeros_like(x_rows)
    y = layer.combine(ys, w, o)
    extra = {int(e): res[int(e)][-1] for e in extra_rows}
    return y, extra
