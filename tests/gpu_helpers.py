"""Helpers for the GPU parity tests: build a workload on the device through the C ABI
and the matching oracle inputs from the same generator draws (never from kernel output),
plus decoders for the library's documented packed layouts."""
import numpy as np
import torch

from block_scaled_moe_sigmoid_b200 import api, synth
from oracle import layer, mx, router


def unpack_expert_codes(ex, e, d, I):
    """Packed w_gu / s_gu / w_dn / s_dn of expert e -> plain (codes, scales) per matrix,
    following the tile-major layouts documented in include/moe.h."""
    mt_dn = (d + 255) // 256
    gu_w = 2 * I * d // 2
    gu_s = (2 * I // 256) * (d // 128) * 1024
    dn_w = mt_dn * 256 * I // 2
    dn_s = mt_dn * (I // 128) * 1024
    wgu = ex.w_gu[e * gu_w:(e + 1) * gu_w].cpu().numpy()
    sgu = ex.s_gu[e * gu_s:(e + 1) * gu_s].cpu().numpy()
    wdn = ex.w_dn[e * dn_w:(e + 1) * dn_w].cpu().numpy()
    sdn = ex.s_dn[e * dn_s:(e + 1) * dn_s].cpu().numpy()

    def codes(buf, rows, K):
        # [m-tile][k-tile][256][64 B] -> [rows][K/2]
        mt = -(-rows // 256)
        t = buf.reshape(mt, K // 128, 256, 64).transpose(0, 2, 1, 3).reshape(mt * 256, K // 2)
        return t[:rows]

    def scales(buf, rows, K):
        pr = np.arange(rows)[:, None]
        b = np.arange(K // 32)[None, :]
        mt, half, rr = pr >> 8, (pr >> 7) & 1, pr & 127
        off = ((mt * (K // 128) + (b >> 2)) * 2 + half) * 512 + (rr & 31) * 16 + (rr >> 5) * 4 + (b & 3)
        return buf[off]

    codes_gu = mx.unpack_e2m1(codes(wgu, 2 * I, d))
    sc_gu = scales(sgu, 2 * I, d)
    # rows are interleaved in 128-row blocks: gate[0:128], up[0:128], gate[128:256], ...
    c = np.arange(I)
    g_rows = 256 * (c // 128) + c % 128
    u_rows = g_rows + 128
    return {
        "gate": (codes_gu[g_rows], sc_gu[g_rows]),
        "up": (codes_gu[u_rows], sc_gu[u_rows]),
        "down": (mx.unpack_e2m1(codes(wdn, d, I)), scales(sdn, d, I)),
    }


def decode_tile_major_scales(buf, counts, k_tiles, bn=176):
    """Token-side scale bytes [A][k_tiles*4] from the tile-major layout documented in
    include/moe.h (debug buffers 1 and 3), using the expert row counts."""
    buf = np.asarray(buf, dtype=np.uint8)
    rows = []
    gt = 0
    for c in counts:
        c = int(c)
        if c == 0:
            continue
        ntiles = -(-c // bn)
        n_per = -(-c // ntiles)
        n_per = (n_per + 15) // 16 * 16
        for r in range(c):
            nt, n = divmod(r, n_per)
            off = (n >> 7) * 512 + (n & 31) * 16 + ((n & 127) >> 5) * 4
            base = (gt + nt) * k_tiles * 1024 + off
            rows.append(np.concatenate([buf[base + kt * 1024: base + kt * 1024 + 4] for kt in range(k_tiles)]))
        gt += ntiles
    return np.stack(rows) if rows else np.zeros((0, 4 * k_tiles), np.uint8)


class Case:
    """A workload: generator draws on `gen_device`, copied to the GPU for the kernels and
    to the CPU for the oracle."""

    def __init__(self, wl, T=None, gen_device=None, bias=None, act="silu", select_only=False,
                 x_scale=1.0):
        self.wl = wl
        self.act = act
        self.select_only = select_only
        self.T = wl.T if T is None else T
        gd = wl.device if gen_device is None else gen_device
        self.gen_device = gd
        dev = "cuda"
        self.x = (synth.draw_x(wl, self.T, device=gd) * x_scale).to(dev)   # x_scale: power of two
        W_r, b = synth.draw_router(wl, device=gd)
        if bias is not None:
            b = bias.to(torch.float32)
        self.W_r, self.bias = W_r.to(dev).contiguous(), b.to(dev).contiguous()
        self.plan = api.Plan(max(self.T, 1), wl.d, wl.E, wl.k, wl.I, wl.I_shared,
                             act={"silu": api.MOE_ACT_SILU_GLU, "clamped_swiglu": api.MOE_ACT_CLAMPED_SWIGLU}[act],
                             bias_mode=api.MOE_BIAS_SELECT_ONLY if select_only else api.MOE_BIAS_LOGIT,
                             d_latent=wl.d_latent)
        self.latent_w = synth.draw_latent(wl, device=gd)
        self.latent = api.Latent(*(t.to(dev) for t in self.latent_w)) if self.latent_w else None
        self.experts = api.Experts(wl.d_expert, wl.I, wl.E)
        for e in range(wl.E):
            g, u, dn = (t.to(dev) for t in synth.draw_expert(wl, e, device=gd))
            self.experts.pack(e, g, u, dn)
        self.shared = None
        self.shared_w = None
        if wl.I_shared:
            sw = synth.draw_shared(wl, device=gd)
            self.shared_w = sw
            self.shared = api.Shared(wl.d, wl.I_shared)
            self.shared.pack(*(t.to(dev) for t in sw))
        torch.cuda.synchronize()
        self._oracle_w = {}

    # ---------------------------------------------------------------- oracle side
    def x_np(self):
        return self.x.float().cpu().numpy().astype(np.float64)

    def oracle_expert(self, e):
        """Exact decoded weights of expert e, quantised by the oracle from the generator's
        fp32 masters."""
        if e not in self._oracle_w:
            ms = [t.cpu().numpy() for t in synth.draw_expert(self.wl, e, device=self.gen_device)]
            self._oracle_w[e] = layer.decode_expert(layer.quantize_expert(*ms))
        return self._oracle_w[e]

    def oracle_latent(self):
        if self.latent_w is None:
            return None
        return tuple(t.float().cpu().numpy().astype(np.float64) for t in self.latent_w)

    def oracle_shared(self):
        if self.shared_w is None:
            return None
        return tuple(t.float().cpu().numpy().astype(np.float64) for t in self.shared_w)

    def oracle_route(self):
        b = self.bias.cpu().numpy()
        if self.select_only:
            z = router.router_logits(self.x_np(), self.W_r.cpu().numpy())
            return z, router.route(z, self.wl.k, select_bias=b)
        z = router.router_logits(self.x_np(), self.W_r.cpu().numpy(), b)
        return z, router.route(z, self.wl.k)


def layer_stats(y_gpu, y_ref, gap, thresh=1e-6):
    """Relative error statistics over tokens with gap >= thresh (reading R17)."""
    keep = gap >= thresh
    r, nw = layer.relative_errors(y_gpu[keep], y_ref[keep])
    return {"max_rel": float(r.max()) if r.size else 0.0, "mean_rel": float(r.mean()) if r.size else 0.0,
            "max_normwise": float(nw.max()) if nw.size else 0.0, "near_ties": int((~keep).sum())}
