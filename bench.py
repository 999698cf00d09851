"""Benchmark of the Kimi-K3 MoE feed-forward layer on B200.

One step = the whole hot path on one batch: moe_route (router GEMM, sigmoid top-k) and
moe_forward (grouping, MXFP8 quantise, gate/up grouped GEMM + GLU + requant, down grouped
GEMM, shared expert, combine), inputs resident in HBM.  Default workload: Kimi-K3 prefill,
T=8192 tokens, d=7168, 896 experts, top-16, I=3072, one bf16 shared expert (I=3072).  The
default line also carries a `decode` object: the Kimi-K3 decode step (T=64, seed 1, same
shapes) timed the same way, with its fraction of the measured HBM bandwidth.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Multi-GPU: token batches are independent, so N ranks run N replicas of the workload
(weak scaling, no collective on the data path); the timing is the max over ranks.
`--impl reference` times the fp64 CPU oracle on a bounded sample of the same workload
(rank 0 only) and extrapolates to the full batch.
"""
import argparse
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "MoE-layer tokens/s at K3 shape (T=8192); % FP4 tensor peak, decode % HBM BW"
UNIT = "tokens/s"

# The GEMM sources whose hash (over their code, comments dropped) keys a recorded
# DRAM-traffic figure.
GEMM_SOURCES = ("gemm.cuh", "ptx.cuh", "tiling.cuh")
# DRAM bytes (read + write) of one launch of the routed gate/up GEMM, from an ncu capture
# (`--metrics dram__bytes_read.sum,dram__bytes_write.sum`, one pass) of the kernel built
# from the GEMM sources with the given hash.  A figure whose hash no longer matches the
# sources is not reported.
GATE_UP_TRAFFIC = {
    ("k3_prefill_t8192", 8192): {"bytes": 22092875264 + 408987392, "sha16": "a78528257fadb9ff",
                                  "how": "timed-step launch of the full T=8192 workload"},
}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="k3_prefill_t8192")
    ap.add_argument("--T", type=int, default=None, help="override the token count")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-decode", action="store_true",
                    help="skip the decode (T=64) measurement that the default workload adds")
    ap.add_argument("--tile-n", type=int, default=0, choices=[0, 32, 128, 160, 176],
                    help="grouped-GEMM token rows per tile (0 = the library's per-call choice)")
    return ap.parse_args()


# ---------------------------------------------------------------- oracle timing (CPU)
def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return os.cpu_count() or 1


def oracle_sample_seconds(wl, T, x_dev, W_r_dev, bias_dev, n_router, n_experts, n_shared, seed=0):
    """Time the fp64 oracle on a bounded sample and extrapolate to the full batch of T tokens:
    router logits + top-k for n_router tokens (scaled by T / n_router), n_experts experts
    each with the mean load T*k/E rows (scaled by E / n_experts; includes quantising and
    decoding the expert's MXFP4 weights), and the shared expert on n_shared tokens
    (scaled by T / n_shared).  Returns (seconds for T tokens, sample description)."""
    import numpy as np
    import torch

    from block_scaled_moe_sigmoid_b200 import synth
    from oracle import layer, mx, router

    g = np.random.default_rng(seed)
    rows = np.sort(g.choice(T, size=min(n_router, T), replace=False))
    x = x_dev.float().cpu().numpy().astype(np.float64)
    W_r = W_r_dev.cpu().numpy()
    b = bias_dev.cpu().numpy()
    t0 = time.perf_counter()
    z = router.router_logits(x[rows], W_r, b)
    router.route(z, wl.k)
    t_router = (time.perf_counter() - t0) * T / len(rows)

    # latent option: x -> latent projection + RMSNorm (and the projection back) per token
    t_lat = 0.0
    xe = x                                       # what the experts read
    if wl.d_latent:
        W_ld, gamma, W_lu = (t.float().cpu().numpy().astype(np.float64)
                             for t in synth.draw_latent(wl, device=x_dev.device.type))
        lrows = rows[:min(n_shared, len(rows))]
        t0 = time.perf_counter()
        xn = mx.bf16_round(layer.rms_norm(x[lrows] @ W_ld.T, gamma))
        mx.bf16_round(xn) @ W_lu.T
        t_lat = (time.perf_counter() - t0) * T / len(lrows)
        # the experts' inputs: the latent rows of a token sample (enough for the mean load)
        xe = np.zeros((T, wl.d_latent))
        xe[lrows] = xn

    load = max(1, int(round(T * wl.k / wl.E)))
    t_exp = 0.0
    for i in range(n_experts):
        e = int(g.integers(wl.E))
        masters = [t.cpu().numpy() for t in synth.draw_expert(wl, e, device=x_dev.device.type)]
        tok = g.choice(rows[:min(n_shared, len(rows))] if wl.d_latent else np.arange(T), size=load, replace=True)
        t0 = time.perf_counter()
        Wg, Wu, Wd = layer.decode_expert(layer.quantize_expert(*masters))
        xq, xs = mx.quantize_mx(xe[tok], "e4m3")
        layer.expert_forward(mx.dequantize_mx(xq, xs, "e4m3"), Wg, Wu, Wd)
        t_exp += time.perf_counter() - t0
    t_exp *= wl.E / max(n_experts, 1)

    t_sh = 0.0
    if wl.I_shared:
        sw = tuple(t.float().cpu().numpy().astype(np.float64)
                   for t in synth.draw_shared(wl, device=x_dev.device.type))
        srows = rows[:min(n_shared, len(rows))]
        t0 = time.perf_counter()
        layer.shared_expert(x[srows], *sw)
        t_sh = (time.perf_counter() - t0) * T / len(srows)
    desc = (f"router on {len(rows)} of {T} tokens, {n_experts} of {wl.E} experts at the mean "
            f"load of {load} rows (weights quantised+decoded per expert), shared expert"
            f"{' and latent projections' if wl.d_latent else ''} on "
            f"{min(n_shared, len(rows))} tokens; each part scaled linearly to T={T}")
    return t_router + t_exp + t_sh + t_lat, desc


# ---------------------------------------------------------------- clocks
class ClockSampler:
    def __init__(self, index):
        self.index = index
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={q}", "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        self.proc.wait(timeout=10)
        sms, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            f = [c.strip() for c in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sms.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        os.unlink(self.path)
        load = [s for s in sms if mx and s > 0.3 * mx] or sms
        return {"sm_mhz": statistics.median(load) if load else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sms)}


# ---------------------------------------------------------------- multi-rank helpers
def max_over_ranks_(v, world, device):
    """The largest of the ranks' values (every rank gets it); v itself when world == 1."""
    if world == 1:
        return v
    import torch
    import torch.distributed as dist
    t = torch.tensor([v], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.item()


def job_throughput(T, steps, world, ms_max):
    """Whole-job tokens/s: every rank runs `steps` steps of T tokens; the job takes the
    slowest rank's time."""
    return world * T * steps / (ms_max / 1e3)


# ---------------------------------------------------------------- our arm
def setup(wl, T, device):
    import torch

    from block_scaled_moe_sigmoid_b200 import api, synth
    x = synth.draw_x(wl, T, device=device)
    W_r, bias = synth.draw_router(wl, device=device)
    plan = api.Plan(T, wl.d, wl.E, wl.k, wl.I, wl.I_shared, device=device, d_latent=wl.d_latent)
    ex = api.Experts(wl.d_expert, wl.I, wl.E, device=device)
    for e in range(wl.E):
        g, u, dn = synth.draw_expert(wl, e, device=device)
        ex.pack(e, g, u, dn)
        del g, u, dn
    sh = None
    if wl.I_shared:
        sh = api.Shared(wl.d, wl.I_shared, device=device)
        sh.pack(*synth.draw_shared(wl, device=device))
    lat = None
    if wl.d_latent:
        lat = api.Latent(*synth.draw_latent(wl, device=device))
    torch.cuda.synchronize()
    plan.latent = lat
    return x, W_r, bias, plan, ex, sh


_C_COMMENT = re.compile(r"//[^\n]*|/\*.*?\*/", re.S)


def source_sha16(*names, csrc=None):
    """First 16 hex digits of the sha256 of the named CUDA sources of the package (or of
    the directory `csrc`), taken over their code only: comments, trailing blanks and empty
    lines are dropped, so that a recorded figure follows the kernels and not the wording of
    their comments."""
    csrc = csrc or os.path.join(ROOT, "block_scaled_moe_sigmoid_b200", "csrc")
    h = hashlib.sha256()
    for n in names:
        with open(os.path.join(csrc, n), encoding="utf-8") as f:
            code = _C_COMMENT.sub("", f.read())
        lines = [ln.rstrip() for ln in code.splitlines()]
        h.update("\n".join(ln for ln in lines if ln).encode())
        h.update(b"\0")
    return h.hexdigest()[:16]


def peaks_from_file():
    peaks = {}
    pk_path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(pk_path):
        peaks = json.load(open(pk_path))
    if peaks.get("bf16_tflops_sustained"):
        bf16, peak_src = peaks["bf16_tflops_sustained"], "measured"
    else:
        bf16, peak_src = 1400.0, "fallback"
    hbm, hbm_src = (peaks["hbm_gbs"], "measured") if peaks.get("hbm_gbs") else (6650.0, "fallback")
    return bf16, peak_src, hbm, hbm_src


def count_launches(api, plan, stages):
    """Kernels launched by the recorded stage instances (profiled pass)."""
    launches = sum(cnt * api.STAGE_KERNELS.get(name, 1) for name, (_, cnt) in stages.items())
    if api.moe_plan_get_option(plan.handle, api.MOE_OPT_SHARED_SPLIT) > 1:
        launches += stages["shared_gate_up"][1]
    if api.moe_plan_get_option(plan.handle, api.MOE_OPT_SHARED_SPLIT_DOWN) > 1:
        launches += stages["shared_down"][1]
    return launches


def measure(args, wl, T, world, local_rank, e2e_on):
    """Time `args.steps` steps of the workload (route + forward) on resident inputs.

    1. Timed pass: CUDA events on the launching stream around the K steps, stage profiler
       off, barrier + synchronize on both sides, max over ranks.
    2. Profiled pass: the same K steps again with the per-stage event profiler on, for the
       per-kernel launch times (roofline) and the launch count.
    3. Optionally the end-to-end pass with host buffers."""
    import torch
    import torch.distributed as dist

    from block_scaled_moe_sigmoid_b200 import api
    dev = torch.device("cuda", local_rank)
    x, W_r, bias, plan, ex, sh = setup(wl, T, "cuda")
    api.moe_plan_set_option(plan.handle, api.MOE_OPT_TILE_N, args.tile_n)
    idx = torch.empty((T, wl.k), dtype=torch.int32, device=dev)
    w = torch.empty((T, wl.k), dtype=torch.float32, device=dev)
    y = torch.empty((T, wl.d), dtype=torch.bfloat16, device=dev)
    stream = torch.cuda.current_stream()

    def one_step():
        api.moe_route(plan.handle, x, W_r, bias, wl.k, idx=idx, w=w)
        plan.forward(x, idx, w, ex, sh, y, latent=plan.latent)

    for _ in range(args.warmup):
        one_step()
    code, bits = plan.check()
    if code != 0:
        raise RuntimeError(f"device status {code} bits {bits} after warm-up")

    def barrier():
        if world > 1:
            dist.barrier()

    def max_over_ranks(v):
        return max_over_ranks_(v, world, dev)

    # ---- 1. timed pass (device time, CUDA events on the launching stream)
    clocks = ClockSampler(local_rank)
    clocks.start()
    barrier()
    torch.cuda.synchronize()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record(stream)
    for _ in range(args.steps):
        one_step()
    ev1.record(stream)
    torch.cuda.synchronize()
    barrier()
    ms = max_over_ranks(ev0.elapsed_time(ev1))
    clk = clocks.stop()
    code, bits = plan.check()
    if code != 0:
        raise RuntimeError(f"device status {code} bits {bits} in the timed region")

    # ---- 2. profiled pass: per-stage launch times and the launch count
    api.moe_plan_set_profiling(plan.handle, True)
    barrier()
    torch.cuda.synchronize()
    for _ in range(args.steps):
        one_step()
    torch.cuda.synchronize()
    barrier()
    stages = api.moe_plan_stage_ms(plan.handle)
    api.moe_plan_set_profiling(plan.handle, False)
    launches = count_launches(api, plan, stages)

    # ---- 3. end to end through the public API with host buffers
    # Every step copies its input x from pinned host memory and its output y back, inside
    # the timed region.  The copies run on their own streams, double-buffered, so step i's
    # output copy and step i+1's input copy overlap the compute of the neighbouring steps,
    # as a serving loop would run them.  Each step's compute waits for its own input copy,
    # and the first input copy of the timed region waits for its start event.
    e2e = None
    if e2e_on:
        x_host = x.cpu().pin_memory()
        y_host = [torch.empty((T, wl.d), dtype=torch.bfloat16).pin_memory() for _ in range(2)]
        x_dev = [torch.empty_like(x) for _ in range(2)]
        y_dev = [torch.empty_like(y) for _ in range(2)]
        h2d, d2h = torch.cuda.Stream(), torch.cuda.Stream()
        ev = {n: [torch.cuda.Event() for _ in range(2)] for n in ("h2d", "comp", "d2h")}

        def e2e_step(i, start=None):
            b = i % 2
            with torch.cuda.stream(h2d):
                if start is not None:
                    h2d.wait_event(start)                # nothing of the step before the window
                if i >= 2:
                    h2d.wait_event(ev["comp"][b])        # step i-2 is done with x_dev[b]
                x_dev[b].copy_(x_host, non_blocking=True)
                ev["h2d"][b].record(h2d)
            stream.wait_event(ev["h2d"][b])
            if i >= 2:
                stream.wait_event(ev["d2h"][b])          # step i-2's y_dev[b] has been read
            api.moe_route(plan.handle, x_dev[b], W_r, bias, wl.k, idx=idx, w=w)
            plan.forward(x_dev[b], idx, w, ex, sh, y_dev[b], latent=plan.latent)
            ev["comp"][b].record(stream)
            with torch.cuda.stream(d2h):
                d2h.wait_event(ev["comp"][b])
                y_host[b].copy_(y_dev[b], non_blocking=True)
                ev["d2h"][b].record(d2h)

        for i in range(max(2, args.warmup)):
            e2e_step(i)
        barrier()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for i in range(args.steps):
            e2e_step(i, start=e0 if i == 0 else None)
        for b in range(2):
            stream.wait_event(ev["d2h"][b])              # the last outputs are on the host
        e1.record(stream)
        torch.cuda.synchronize()
        barrier()
        e_ms = max_over_ranks(e0.elapsed_time(e1))
        e2e = {"value": world * T * args.steps / (e_ms / 1e3), "unit": UNIT,
               "h2d_bytes_per_step": x.numel() * x.element_size(),
               "d2h_bytes_per_step": y.numel() * y.element_size(),
               "overlap": "copies on their own streams, double-buffered across steps"}

    touched = int(torch.unique(idx).numel())
    load = torch.bincount(idx.reshape(-1).long(), minlength=wl.E).cpu()
    tile_rows = api.moe_plan_get_option(plan.handle, api.MOE_OPT_TILE_N)
    res = {"ms": ms, "stages": stages, "launches": launches, "clocks": clk, "e2e": e2e,
           "touched": touched, "load": load, "tile_rows": tile_rows}
    # the host copies the CPU baseline needs (the oracle reads the same draws)
    res["data"] = (x, W_r, bias)
    del plan, ex, sh, y, idx, w
    torch.cuda.empty_cache()
    return res


def gate_up_roofline(wl, T, m, traffic):
    """Roofline object of the routed gate/up GEMM, the dominant kernel.

    Its bound is the slower of two terms: the block-scaled MMAs at the tensor pipe's rate
    for MXFP4 x MXFP8 operands (kind::mxf8f6f4 issues at the FP8 rate, twice bf16), and the
    algorithmic HBM bytes (the touched experts' codes and scales, the MXFP8 token rows read
    once, the MXFP8 GLU output written once) at the measured copy bandwidth."""
    bf16, peak_src, hbm, hbm_src = peaks_from_file()
    gu_ms, gu_n = m["stages"]["gate_up_glu"]
    t_launch = gu_ms / gu_n / 1e3 if gu_n else None
    A = T * wl.k
    de = wl.d_expert                                           # expert input width (d, or d_latent)
    flops = 2.0 * A * de * (2 * wl.I)
    gu_bytes = (m["touched"] * 2 * wl.I * de * 17 / 32        # E2M1 codes + E8M0 scales
                + A * de * 33 / 32 + A * wl.I * 33 / 32)       # MXFP8 rows in, GLU rows out
    tc_peak = 2.0 * bf16
    tensor_bound = flops / tc_peak / 1e12 >= gu_bytes / hbm / 1e9
    if tensor_bound:
        achieved = flops / t_launch / 1e12 if t_launch else None
        peak, unit = tc_peak, "TFLOP/s"
    else:
        achieved = gu_bytes / t_launch / 1e9 if t_launch else None
        peak, unit = hbm, "GB/s"
    return {"kernel": "gemm_kernel<KIND_MX, EPI_GLU_MX8> (routed gate/up + SiLU-GLU + MXFP8 requant)",
            "bound": "tensor" if tensor_bound else "hbm", "achieved": achieved, "peak": peak,
            "unit": unit, "frac": achieved / peak if achieved else None,
            "traffic": traffic["bytes"] if traffic else None,
            "traffic_unit": "bytes per launch (ncu dram__bytes_read.sum + dram__bytes_write.sum)",
            "traffic_source": traffic["source"] if traffic else
            "none recorded for this kernel source and workload",
            "peak_note": (f"tensor: FP8-rate pipe = 2 x {peak_src} sustained bf16 GEMM "
                          f"(kind::mxf8f6f4 issues at the FP8 rate); hbm: {hbm_src} copy bandwidth"),
            "ms_per_launch": gu_ms / gu_n if gu_n else None,
            "launch_time_source": "per-stage CUDA events on the launching stream, profiled pass "
                                  "of the same steps",
            "flops_per_launch": flops, "algorithmic_bytes_per_launch": gu_bytes,
            "hbm_frac_of_algorithmic_bytes": (gu_bytes / t_launch / 1e9 / hbm) if t_launch else None,
            "touched_experts": m["touched"],
            "tflops_per_launch": flops / t_launch / 1e12 if t_launch else None,
            "frac_of_nominal_fp4_rate": (flops / t_launch / 1e12 / (4.0 * bf16)) if t_launch else None,
            "fp4_note": "FP4-rate MMAs (kind::mxf4) need both operands in E2M1; MXFP8 "
                        "activations run at the FP8 rate, so the FP4 figure is context"}


def weight_bytes(wl, touched):
    """Touched experts' MXFP4 weights + bf16 shared expert + fp32 router matrix (+ latent
    projections) streamed per step."""
    de = wl.d_expert
    return (touched * 3 * de * wl.I * 17 / 32 + 3 * wl.d * wl.I_shared * 2
            + wl.d * wl.E * 4 + 2 * wl.d * wl.d_latent * 2)


def traffic_record(workload, T):
    """The recorded ncu DRAM bytes of one gate/up launch, when they were captured on the
    current GEMM source; None otherwise (a stale figure is not reported)."""
    rec = GATE_UP_TRAFFIC.get((workload, T))
    if not rec:
        return None
    sha = source_sha16(*GEMM_SOURCES)
    if rec["sha16"] != sha:
        return None
    return {"bytes": rec["bytes"],
            "source": f"ncu capture of this gate/up kernel (csrc sha {sha}), {rec['how']}"}


def run_ours(args, rank, world, local_rank):
    import torch

    from block_scaled_moe_sigmoid_b200 import synth
    wl = synth.WORKLOADS[args.workload]
    T = args.T or (wl.sweep[-1] if wl.sweep else wl.T)
    torch.cuda.set_device(torch.device("cuda", local_rank))
    m = measure(args, wl, T, world, local_rank, e2e_on=not args.no_e2e)
    ms = m["ms"]
    _, _, hbm, _ = peaks_from_file()
    roofline = gate_up_roofline(wl, T, m, traffic_record(args.workload, T))
    w_bytes = weight_bytes(wl, m["touched"])
    stage_ms = {k: round(v[0] / max(v[1], 1), 4) for k, v in m["stages"].items()}
    load = m["load"]
    ls = torch.sort(load, descending=True).values
    expert_load = {"mean": float(load.float().mean()), "max": int(ls[0]), "min": int(ls[-1]),
                   "p50": int(ls[wl.E // 2]), "p90": int(ls[wl.E // 10]), "zero_experts": int((load == 0).sum()),
                   "top8": [int(v) for v in ls[:8]],
                   "share_of_top_1pct": float(ls[:max(1, wl.E // 100)].sum()) / max(1, int(load.sum()))}

    # ---- the decode half of the metric: the Kimi-K3 decode step (T=64), same shapes
    decode = None
    if args.workload == "k3_prefill_t8192" and not args.no_decode:
        dwl = synth.WORKLOADS["k3_decode_t64"]
        dm = measure(args, dwl, dwl.T, world, local_rank, e2e_on=False)
        d_ms = dm["ms"] / args.steps
        d_bytes = weight_bytes(dwl, dm["touched"])
        d_roof = gate_up_roofline(dwl, dwl.T, dm, None)
        decode = {"workload": dwl.name, "T": dwl.T, "seed": dwl.seed, "ms_per_step": d_ms,
                  "value": world * dwl.T / (d_ms / 1e3), "unit": UNIT,
                  "touched_experts": dm["touched"], "weight_bytes_per_step": d_bytes,
                  "frac_hbm": d_bytes / (d_ms / 1e3) / 1e9 / hbm,
                  "gate_up_frac_hbm": d_roof["hbm_frac_of_algorithmic_bytes"],
                  "gate_up_ms_per_launch": d_roof["ms_per_launch"],
                  "stage_ms_per_launch": {k: round(v[0] / max(v[1], 1), 4) for k, v in dm["stages"].items()},
                  "gpu_launches": dm["launches"], "clocks": dm["clocks"],
                  "note": "frac_hbm = touched experts' MXFP4 weights + shared expert + router "
                          "matrix per step over the step's device time, against the measured "
                          "copy bandwidth; 20 GB+ of weights per step, so no L2 reuse between steps"}

    out = None
    if rank == 0:
        value = job_throughput(T, args.steps, world, ms)
        out = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "mxfp4xmxfp8 (fp32 acc); bf16 shared/router",
            "data": "synthetic (seeded N(0,1) x, N(0,0.02) weights, random-init)",
            "config": {"workload": args.workload, "T": T, "d": wl.d, "d_latent": wl.d_latent, "E": wl.E,
                       "k": wl.k, "I": wl.I,
                       "I_shared": wl.I_shared, "seed": wl.seed, "parallelism": f"replicas x{world}",
                       "l2": "inputs larger than L2: every step streams "
                             f"{w_bytes / 1e9:.1f} GB of weights ({m['touched']} touched experts)"},
            "roofline": roofline,
            "decode": decode,
            "gemm_tile_rows": m["tile_rows"],
            "expert_load": expert_load,
            "hbm_view": {"weight_bytes_per_step": w_bytes, "touched_experts": m["touched"],
                         "achieved_gbs": w_bytes / (ms / args.steps / 1e3) / 1e9,
                         "peak_gbs": hbm, "frac": w_bytes / (ms / args.steps / 1e3) / 1e9 / hbm,
                         "note": "touched experts' MXFP4 weights + bf16 shared expert + fp32 "
                                 "router matrix per step, over the whole step's time"},
            "stage_ms_per_launch": stage_ms,
            "clocks": m["clocks"], "e2e": m["e2e"], "gpu_launches": m["launches"],
        }
    x, W_r, bias = m["data"]
    return out, (x, W_r, bias, wl, T)


def main():
    args = parse()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        return run_reference(args, rank, world)
    import torch
    import torch.distributed as dist
    if world > 1:
        torch.cuda.set_device(local_rank)
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=600),
                                device_id=torch.device("cuda", local_rank))
    out, data = run_ours(args, rank, world, local_rank)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        x, W_r, bias, wl, T = data
        secs, desc = oracle_sample_seconds(wl, T, x, W_r, bias, n_router=256, n_experts=2, n_shared=64)
        out["cpu_baseline"] = {"value": T / secs, "unit": UNIT, "cores": blas_threads(),
                               "kind": "oracle", "sample": desc}
    if rank == 0:
        print(json.dumps(out))
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def run_reference(args, rank, world):
    """The reference arm: the fp64 oracle, as it stands, on the host cores."""
    if rank != 0:
        return
    import torch

    from block_scaled_moe_sigmoid_b200 import synth
    wl = synth.WORKLOADS[args.workload]
    T = args.T or (wl.sweep[-1] if wl.sweep else wl.T)
    gen = "cuda" if torch.cuda.is_available() else "cpu"
    x = synth.draw_x(wl, T, device=gen)
    W_r, bias = synth.draw_router(wl, device=gen)
    secs = []
    desc = ""
    for i in range(args.warmup + args.steps):
        s, desc = oracle_sample_seconds(wl, T, x, W_r, bias, n_router=32, n_experts=1, n_shared=8, seed=i)
        if i >= args.warmup:
            secs.append(s)
    total = sum(secs)
    value = T * len(secs) / total
    out = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
           "warmup": args.warmup, "ms_per_step": 1e3 * total / len(secs), "higher_is_better": True,
           "scaling": "weak", "vs_baseline": None, "dtype": "f64", "impl": "reference",
           "data": "synthetic (seeded)",
           "config": {"workload": args.workload, "T": T, "d": wl.d, "E": wl.E, "k": wl.k, "I": wl.I,
                      "I_shared": wl.I_shared, "seed": wl.seed},
           "cpu_baseline": {"value": value, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
                            "sample": desc},
           "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(out))


if __name__ == "__main__":
    main()
