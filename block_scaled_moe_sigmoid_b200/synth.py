"""Seeded synthetic inputs for the MoE layer workloads.

This module draws random numbers and nothing else: it holds none of the
layer's arithmetic (no quantisation, no routing, no products), so both the CPU
oracle and the CUDA path can take their inputs from it.

Generator: ``torch.randn`` / ``torch.randperm`` from a ``torch.Generator`` seeded
with a 63-bit mix of (workload seed, tensor id, sub-index).  Each tensor, and
each expert's matrix, has its own stream, so any one expert can be redrawn
alone.  Draws depend on the device type of the generator (CPU and CUDA produce
different streams), so each workload fixes where it is drawn: small shapes on
the CPU, Kimi-K3-shaped tensors on the GPU.  A consumer on the other side gets a
copy of the drawn values.

Distributions (the workload table of the layer's specification):
  x      ~ N(0, 1) rounded to bf16
  W_r    ~ N(0, 0.02) fp32, bias 0 (or the skewed-load bias below)
  W_gate, W_up [I, d], W_down [d, I] per expert ~ N(0, 0.02) fp32 masters
         (quantised to MXFP4 by each side on its own)
  shared W_gate, W_up [I_s, d], W_down [d, I_s] ~ N(0, 0.02) rounded to bf16
  skewed-load bias b_e = 2.0 * ln(1 / (rank_e + 1)^1.2) = -2.4 ln(rank_e + 1),
         rank = a seeded random permutation of 0..E-1
  latent option (d_latent > 0): experts act on d_latent; projections W_ld [d_latent, d]
         and W_lu [d, d_latent] ~ N(0, 0.02) rounded to bf16; the RMSNorm gain
         gamma [d_latent] = 1 + N(0, 0.1) fp32 (the spec gives no distribution)
The std 0.02 is the config's initializer_range ("Kimi K3" (llm-atlas), raw
config fields).
"""
from dataclasses import dataclass, field

import torch

STD = 0.02

# tensor ids of the independent streams
TID_X, TID_WR, TID_RANK = 0, 1, 2
TID_GATE, TID_UP, TID_DOWN = 3, 4, 5
TID_SGATE, TID_SUP, TID_SDOWN = 6, 7, 8
TID_LDOWN, TID_LUP, TID_LGAMMA = 9, 10, 11


def stream_seed(seed, tid, sub=0):
    return ((int(seed) * 1000003 + int(tid)) * 1000033 + int(sub)) & ((1 << 63) - 1)


def _gen(device, seed, tid, sub=0):
    g = torch.Generator(device=torch.device(device).type)
    g.manual_seed(stream_seed(seed, tid, sub))
    return g


def normal(shape, seed, tid, sub=0, std=1.0, device="cpu"):
    """fp32 N(0, std^2) draws (the product randn * std is rounded to fp32)."""
    t = torch.randn(shape, generator=_gen(device, seed, tid, sub), device=device,
                    dtype=torch.float32)
    if std != 1.0:
        t.mul_(std)
    return t


@dataclass
class Workload:
    name: str
    seed: int
    T: int
    d: int
    E: int
    k: int
    I: int
    I_shared: int            # 0 = no shared expert
    skew_bias: bool = False
    device: str = "cpu"      # where the generator runs
    sweep: tuple = field(default_factory=tuple)
    d_latent: int = 0        # > 0: the latent option (experts act on d_latent)

    @property
    def d_expert(self):
        return self.d_latent or self.d


WORKLOADS = {
    # toy layer the oracle finishes in seconds
    "toy": Workload("toy", 0, 128, 512, 32, 4, 256, 0, device="cpu"),
    # Kimi-K3 shape: decode step (T=64) and prefill (T=8192)
    "k3_decode_t64": Workload("k3_decode_t64", 1, 64, 7168, 896, 16, 3072, 3072, device="cuda"),
    "k3_prefill_t8192": Workload("k3_prefill_t8192", 2, 8192, 7168, 896, 16, 3072, 3072, device="cuda"),
    # skewed routing through a Zipf-like logit bias
    "k3_skewed_t32768": Workload("k3_skewed_t32768", 3, 32768, 7168, 896, 16, 3072, 3072,
                                 skew_bias=True, device="cuda"),
    # Kimi-K3 expert shapes on a 64-expert slice (2.2 GB of weights): a profiling case that
    # keeps the device footprint to a few GB while the weights still exceed L2
    "k3_slice_e64_t1024": Workload("k3_slice_e64_t1024", 2, 1024, 7168, 64, 16, 3072, 3072, device="cuda"),
    # the pages' shared expert: two full-width experts stored fused as one GLU with
    # intermediate size 6144 ("Kimi K3.1 Pro vs gpt-oss-120b", component table, shared-expert row)
    "k3_prefill_t8192_shared6144": Workload("k3_prefill_t8192_shared6144", 2, 8192, 7168, 896, 16, 3072, 6144,
                                            device="cuda"),
    # the latent option at Kimi-K3 shape: experts on a 3584-dim latent (half of d)
    "k3_latent_prefill_t8192": Workload("k3_latent_prefill_t8192", 2, 8192, 7168, 896, 16, 3072, 3072,
                                        device="cuda", d_latent=3584),
    # token-count sweep (T is given per run)
    "k3_sweep": Workload("k3_sweep", 4, 1, 7168, 896, 16, 3072, 3072, device="cuda",
                         sweep=(1, 16, 256, 2048, 16384)),
}


def draw_x(wl, T=None, device=None):
    T = wl.T if T is None else T
    dev = wl.device if device is None else device
    return normal((T, wl.d), wl.seed, TID_X, device=dev).to(torch.bfloat16)


def draw_router(wl, device=None):
    """(W_r fp32 [d, E], bias fp32 [E])."""
    dev = wl.device if device is None else device
    W_r = normal((wl.d, wl.E), wl.seed, TID_WR, std=STD, device=dev)
    if wl.skew_bias:
        rank = torch.randperm(wl.E, generator=_gen(dev, wl.seed, TID_RANK), device=dev)
        bias = -2.4 * torch.log(rank.to(torch.float64) + 1.0)
        bias = bias.to(torch.float32)
    else:
        bias = torch.zeros(wl.E, dtype=torch.float32, device=dev)
    return W_r, bias


def draw_expert(wl, e, device=None):
    """fp32 masters of expert e: (W_gate [I, de], W_up [I, de], W_down [de, I]) with
    de = d, or d_latent for the latent option."""
    dev = wl.device if device is None else device
    de = wl.d_expert
    return (normal((wl.I, de), wl.seed, TID_GATE, e, STD, dev),
            normal((wl.I, de), wl.seed, TID_UP, e, STD, dev),
            normal((de, wl.I), wl.seed, TID_DOWN, e, STD, dev))


def draw_latent(wl, device=None):
    """Latent option: (W_ld bf16 [d_latent, d], gamma fp32 [d_latent], W_lu bf16 [d, d_latent])."""
    if not wl.d_latent:
        return None
    dev = wl.device if device is None else device
    dl = wl.d_latent
    gamma = normal((dl,), wl.seed, TID_LGAMMA, 0, 0.1, dev).add_(1.0)
    return (normal((dl, wl.d), wl.seed, TID_LDOWN, 0, STD, dev).to(torch.bfloat16), gamma,
            normal((wl.d, dl), wl.seed, TID_LUP, 0, STD, dev).to(torch.bfloat16))


def draw_shared(wl, device=None):
    """bf16 shared expert: (W_gate [I_s, d], W_up [I_s, d], W_down [d, I_s]) or None."""
    if not wl.I_shared:
        return None
    dev = wl.device if device is None else device
    Is = wl.I_shared
    return (normal((Is, wl.d), wl.seed, TID_SGATE, 0, STD, dev).to(torch.bfloat16),
            normal((Is, wl.d), wl.seed, TID_SUP, 0, STD, dev).to(torch.bfloat16),
            normal((wl.d, Is), wl.seed, TID_SDOWN, 0, STD, dev).to(torch.bfloat16))


def custom(name="custom", seed=0, T=8, d=256, E=8, k=2, I=128, I_shared=0,
           skew_bias=False, device="cpu", d_latent=0):
    """A workload of arbitrary (small) shape for tests."""
    return Workload(name, seed, T, d, E, k, I, I_shared, skew_bias, device, d_latent=d_latent)
