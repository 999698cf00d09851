"""MoE feed-forward layer, fp64 reference.  TEST INFRASTRUCTURE ONLY.

What the pages fix:
  * Routed experts: "Kimi K3.1 Pro vs gpt-oss-120b" (archdiff), component table,
    row "Stable LatentMoE routed experts (SiTU-GLU)": 896 GLU experts, 16 fire
    per token.  "Kimi K3" (llm-atlas), raw config fields: moe_intermediate_size
    3072, hidden_size 7168.
  * Shared expert: same table, row "Shared expert": always active, ungated,
    reads the un-projected input, kept in BF16.
  * Precision: "Kimi K3" (llm-atlas), Key facts, Dtype row (experts MXFP4, shared
    expert high precision); "Kimi K3, previewed" (embedl blog), specifications
    figure caption (MXFP4 weights with MXFP8 activations).
  * Combine: the block diagram of "Kimi K3.1 Pro vs gpt-oss-120b" adds the
    routed and the shared expert outputs (circled-plus node), and the raw config
    has routed_scaling_factor 1.

Readings (the pages leave these open):
  R11 Activation: the pages name SiTU-GLU but give no formula, only the config
      betas (activation_situ_beta 4, activation_situ_linear_beta 25).  The
      activation is a pluggable GLU, act(g) * u, defaulting to SiLU:
      silu(g) = g / (1 + exp(-g)).
  R12 Experts act directly on d_model (the latent projection, RMSNorm placement
      and its weights are unpublished).
  R13 Expert weights are stored out x in, W[n, k], so g_n = sum_k x_k W_g[n, k].
      They are MXFP4-quantised in blocks of 32 along k (the reduction axis).
  R14 The routed input is x quantised to MXFP8 along d; the GLU output
      a = act(g) * u is requantised to MXFP8 along I before the down projection.
      This is the only requantisation; accumulation is exact (fp64 here).
  R15 Shared expert: bf16 x and weights, accumulation in fp64, the GLU output
      rounded to bf16 (the precision of the operand of the second product).
  R16 Output: y = y_shared + sum_j w_j * o_j accumulated in fp64, then rounded
      once to bf16 (ties to even).
  R21 Second GLU (an option, not the Kimi default): the clamped SwiGLU that
      "Kimi K3.1 Pro vs gpt-oss-120b" (archdiff), component table, routed-experts
      row, describes for gpt-oss.  The gate is clamped from above at 7.0, the
      linear branch to [-7, 7], and a = (u_c + 1) * g_c * sigmoid(1.702 g_c).
      Reading: "gate" is the first projection g and "linear branch" the second u.
      The plan's activation applies to every GLU of the layer, routed and shared.
  R22 Latent option (not the default; unpinned placement).  The component tables of
      "Kimi K3.1 Pro vs gpt-oss-120b" and "Gemma 4 31B vs Kimi K3" have the routed
      experts run in a 3,584-dim latent (half of d) with an RMSNorm before the
      up-projection.  The raw config of "Kimi K3" (llm-atlas) gives
      routed_expert_hidden_size 3584, latent_moe_use_norm true and rms_norm_eps 1e-5.
      The projections' placement, weights and precision are not published.  Plainest
      reading, built as an option:
        x_l = x W_ld^T (bf16 weights, fp32/fp64 accumulation)
        x_n = bf16(x_l / sqrt(mean(x_l^2) + eps) * gamma)   (the norm before the experts' up-projection)
        y_l = bf16(sum_j w_j expert_j(x_n))                  (experts act on the latent)
        y   = bf16(y_l W_lu^T + shared(x))                   (the shared expert reads the un-projected x)
"""
import numpy as np

from . import mx


def silu(g):
    g = np.asarray(g, dtype=np.float64)
    return g / (1.0 + np.exp(-g))


def glu_silu(g, u):
    """SiLU-GLU (R11): silu(g) * u."""
    return silu(g) * np.asarray(u, dtype=np.float64)


def glu_clamped_swiglu(g, u, limit=7.0, alpha=1.702):
    """Clamped SwiGLU (R21): (clip(u, -7, 7) + 1) * g_c * sigmoid(1.702 g_c), g_c = min(g, 7)."""
    gc = np.minimum(np.asarray(g, dtype=np.float64), limit)
    uc = np.clip(np.asarray(u, dtype=np.float64), -limit, limit)
    return (uc + 1.0) * gc / (1.0 + np.exp(-alpha * gc))


# GLU activations by name: a = glu(g, u)
ACTIVATIONS = {"silu": glu_silu, "clamped_swiglu": glu_clamped_swiglu}


def quantize_expert(W_gate, W_up, W_down):
    """MXFP4 codes/scales of one expert's fp32 master weights (R13).

    W_gate, W_up: [I, d]; W_down: [d, I].  Returns dict of (codes, scales) pairs.
    """
    return {
        "gate": mx.quantize_mx(W_gate, "e2m1"),
        "up": mx.quantize_mx(W_up, "e2m1"),
        "down": mx.quantize_mx(W_down, "e2m1"),
    }


def decode_expert(q):
    """Exact fp64 weights of a quantised expert: (Wg [I,d], Wu [I,d], Wd [d,I])."""
    return (mx.dequantize_mx(*q["gate"], "e2m1"),
            mx.dequantize_mx(*q["up"], "e2m1"),
            mx.dequantize_mx(*q["down"], "e2m1"))


def expert_hidden(X, Wg, Wu, act="silu"):
    """a = glu(X Wg^T, X Wu^T) in fp64 (R11, R13, R21).  X: [M, d] exact values."""
    g = X @ Wg.T
    u = X @ Wu.T
    return ACTIVATIONS[act](g, u)


def expert_forward(X, Wg, Wu, Wd, act="silu"):
    """One expert on the (already MXFP8-decoded) rows X [M, d].

    Returns (o fp64 [M, d], a fp64 [M, I], hq uint8 [M, I], hs uint8 [M, I/32]).
    """
    a = expert_hidden(X, Wg, Wu, act)
    hq, hs = mx.quantize_mx(a, "e4m3")                     # R14
    H = mx.dequantize_mx(hq, hs, "e4m3")
    return H @ Wd.T, a, hq, hs


def shared_expert(x, Wsg, Wsu, Wsd, act="silu"):
    """y_s = bf16(act(x Wsg^T) * (x Wsu^T)) Wsd^T, fp64 accumulation (R15).

    x: [T, d]; Wsg, Wsu: [I_s, d]; Wsd: [d, I_s]; all bf16 values (exact in fp64).
    Returns (y_s fp64 [T, d], h fp64 [T, I_s] holding bf16 values).
    """
    h = mx.bf16_round(expert_hidden(np.asarray(x, np.float64), Wsg, Wsu, act))
    return h @ np.asarray(Wsd, np.float64).T, h


def moe_layer(x, idx, w, expert_weights, shared=None, tokens=None, act="silu",
              want_intermediates=False):
    """Full layer output for the rows `tokens` of x (all rows when None).

    x:      [T, d] bf16 values (as float array)
    idx, w: [T, k] routing (expert ids, weights), e.g. from oracle.router.route
    expert_weights(e) -> (Wg [I,d], Wu [I,d], Wd [d,I]) exact fp64 decoded MXFP4
            weights of expert e (see decode_expert)
    shared: None or (Wsg, Wsu, Wsd) bf16 values
    Returns y fp64 [len(tokens), d] holding bf16 values (R16); with
    want_intermediates also a dict with the per-slot expert outputs o [n,k,d],
    the GLU values a [n,k,I] and their MXFP8 codes hq / scales hs.
    """
    x = np.asarray(x, dtype=np.float64)
    idx = np.asarray(idx)
    w = np.asarray(w, dtype=np.float64)
    T, d = x.shape
    k = idx.shape[1]
    rows = np.arange(T) if tokens is None else np.asarray(tokens)
    n = len(rows)
    xq, xs = mx.quantize_mx(x[rows], "e4m3")              # R14: MXFP8 activations
    X = mx.dequantize_mx(xq, xs, "e4m3")
    o = np.zeros((n, k, d))
    inter = {}
    sub_idx = idx[rows]
    for e in np.unique(sub_idx):
        sel = np.argwhere(sub_idx == e)                  # (row position, slot) pairs
        Wg, Wu, Wd = expert_weights(int(e))
        oe, a, hq, hs = expert_forward(X[sel[:, 0]], Wg, Wu, Wd, act)
        o[sel[:, 0], sel[:, 1]] = oe
        if want_intermediates:
            if "a" not in inter:
                I = a.shape[1]
                inter["a"] = np.zeros((n, k, I))
                inter["hq"] = np.zeros((n, k, I), np.uint8)
                inter["hs"] = np.zeros((n, k, I // mx.BLOCK), np.uint8)
            inter["a"][sel[:, 0], sel[:, 1]] = a
            inter["hq"][sel[:, 0], sel[:, 1]] = hq
            inter["hs"][sel[:, 0], sel[:, 1]] = hs
    if shared is not None:
        ys, _ = shared_expert(x[rows], *shared, act=act)
    else:
        ys = np.zeros((n, d))
    y = combine(ys, w[rows], o)
    if want_intermediates:
        inter["o"] = o
        inter["y_shared"] = ys
        inter["xq"], inter["xs"] = xq, xs
        return y, inter
    return y


def combine(y_shared, w, o):
    """y = bf16(y_shared + sum_j w_j o_j), summed in fp64 and rounded once (R16).

    y_shared: [n, d]; w: [n, k] routing weights; o: [n, k, d] expert outputs per slot.
    """
    acc = np.asarray(y_shared, np.float64) + np.einsum("nk,nkd->nd", np.asarray(w, np.float64),
                                                       np.asarray(o, np.float64))
    return mx.bf16_round(acc)


def rms_norm(v, gamma, eps=1e-5):
    """v / sqrt(mean(v^2) + eps) * gamma over the last axis, in fp64 (R22)."""
    v = np.asarray(v, dtype=np.float64)
    ms = np.mean(v * v, axis=-1, keepdims=True)
    return v / np.sqrt(ms + eps) * np.asarray(gamma, dtype=np.float64)


def latent_moe_layer(x, idx, w, expert_weights, latent, shared=None, tokens=None, act="silu",
                     eps=1e-5):
    """The latent option (R22) for the rows `tokens` of x.

    latent: (W_ld [dl, d] bf16 values, gamma [dl], W_lu [d, dl] bf16 values);
    expert_weights(e) -> decoded expert weights acting on the dl-dim latent.
    Returns y fp64 [len(tokens), d] holding bf16 values.
    """
    x = np.asarray(x, dtype=np.float64)
    W_ld, gamma, W_lu = (np.asarray(a, dtype=np.float64) for a in latent)
    T = x.shape[0]
    rows = np.arange(T) if tokens is None else np.asarray(tokens)
    xn = np.zeros((T, W_ld.shape[0]))
    xn[rows] = mx.bf16_round(rms_norm(x[rows] @ W_ld.T, gamma, eps))
    y_l = moe_layer(xn, idx, w, expert_weights, None, tokens=rows, act=act)   # bf16(sum_j w_j o_j)
    y_r = y_l @ W_lu.T
    if shared is not None:
        ys, _ = shared_expert(x[rows], *shared, act=act)
    else:
        ys = np.zeros_like(y_r)
    return mx.bf16_round(y_r + ys)


def relative_errors(y, y_ref):
    """Per-element error |y - y_ref| / max(|y_ref|, rms of the token's row of y_ref).

    Reading R17: the acceptance criteria name a "relative error" without a
    denominator; the row rms floor keeps entries near zero from dominating.
    Returns (r [n, d], per-token normwise relative error [n]).
    """
    y = np.asarray(y, np.float64)
    y_ref = np.asarray(y_ref, np.float64)
    rms = np.sqrt(np.mean(y_ref ** 2, axis=1, keepdims=True))
    denom = np.maximum(np.abs(y_ref), rms)
    denom = np.where(denom == 0, 1.0, denom)
    r = np.abs(y - y_ref) / denom
    nrm = np.linalg.norm(y_ref, axis=1)
    nw = np.linalg.norm(y - y_ref, axis=1) / np.where(nrm == 0, 1.0, nrm)
    return r, nw
