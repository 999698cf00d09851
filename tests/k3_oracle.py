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
from multiprocessing import shared_memory

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


def decode_expert_fast(q):
    """oracle.layer.decode_expert with the C restatement of the MX decoder (pinned
    bit-exact against oracle.mx.dequantize_mx)."""
    return tuple(cmx.dequantize_mx_f64(*q[name], "e2m1") for name in ("gate", "up", "down"))


# worker side: shared-memory blocks attached once per process, by name
_attached = {}


def _masters(name, shapes):
    if name not in _attached:
        _attached[name] = shared_memory.SharedMemory(name=name)
    buf = _attached[name].buf
    out, off = [], 0
    for shp in shapes:
        n = int(np.prod(shp))
        out.append(np.ndarray(shp, dtype=np.float32, buffer=buf, offset=off))
        off += 4 * n
    return out


def expert_job(shm_name, shapes, blocks, want_stage, act):
    """Worker: one expert's oracle outputs for several blocks of decoded token rows.

    shm_name/shapes: the fp32 masters (gate, up, down) in a shared-memory block; blocks:
    list of fp64 [R, d] arrays.  Returns, per block, (o,) or, with want_stage,
    (o, a, hq, hs)."""
    torch.set_num_threads(1)
    w_gate, w_up, w_down = _masters(shm_name, shapes)
    q = quantize_expert_fast(w_gate, w_up, w_down)
    Wg, Wu, Wd = decode_expert_fast(q)
    out = []
    for X in blocks:
        o, a, hq, hs = layer.expert_forward(X, Wg, Wu, Wd, act)
        out.append((o, a, hq, hs) if want_stage else (o,))
    return out


def run_experts(wl, jobs, stage_experts=(), act="silu", device=None):
    """jobs: {expert: [fp64 [R, d] token-row block, ...]} -> {expert: [result per block]}.

    Results are expert_job's tuples; experts in `stage_experts` also return the GLU values
    and their MXFP8 codes and scales.  The parent draws each expert's masters straight into
    one of 2 x pool-size shared-memory blocks, reused round robin (a block is rewritten only
    after the job that read it has returned)."""
    import torch.multiprocessing as tmp
    device = wl.device if device is None else device
    n = pool_size()
    ctx = tmp.get_context("spawn")
    de = wl.d_expert
    shapes = ((wl.I, de), (wl.I, de), (de, wl.I))
    nbytes = 4 * sum(a * b for a, b in shapes)
    blocks_shm = [shared_memory.SharedMemory(create=True, size=nbytes) for _ in range(2 * n)]
    results = {}
    try:
        with ctx.Pool(n) as pool:
            inflight = deque()
            for i, e in enumerate(sorted(jobs)):
                while len(inflight) >= 2 * n:            # frees the block this job reuses
                    e0, r0 = inflight.popleft()
                    results[e0] = r0.get()
                blk = blocks_shm[i % (2 * n)]
                off = 0
                for t, shp in zip(synth.draw_expert(wl, e, device=device), shapes):
                    cnt = shp[0] * shp[1]
                    dst = torch.from_numpy(np.ndarray(shp, dtype=np.float32, buffer=blk.buf, offset=off))
                    dst.copy_(t)
                    off += 4 * cnt
                inflight.append((e, pool.apply_async(expert_job, (blk.name, shapes, jobs[e], e in stage_experts, act))))
            while inflight:
                e0, r0 = inflight.popleft()
                results[e0] = r0.get()
    finally:
        for b in blocks_shm:
            b.close()
            b.unlink()
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
