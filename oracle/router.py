"""Sigmoid top-k router, fp64 reference.  TEST INFRASTRUCTURE ONLY.

What the pages fix:
  * "Kimi K3.1 Pro vs gpt-oss-120b" (archdiff), component table, row
    "Sigmoid router with Quantile Balancing": sigmoid scores pick 16 of 896
    experts.  The same row appears in "Gemma 4 31B vs Kimi K3" (archdiff).
  * "Kimi K3" (llm-atlas), raw config fields: moe_router_activation_func
    sigmoid, num_experts 896, num_experts_per_token 16, moe_renormalize true,
    routed_scaling_factor 1, use_grouped_topk true with num_expert_group 1 and
    topk_group 1.  One group makes grouped top-k plain top-k.

Readings (the pages leave these open):
  R6 The bias is added to the logit, z = x.W_r + b, and both selection and
     weights come from s = sigmoid(z).  The per-step Quantile Balancing rule is
     unpublished, so b is an input.
  R7 Selection is by z in descending order; on equal z the lower expert index
     wins.  sigmoid is monotone, so this is selection by s in exact arithmetic,
     and it avoids ties created by rounding s.
  R8 Weights: w_j = s_j / sum of the selected s (renormalise, scale factor 1).
     The output order is the selection order.
  R9 The "16th/17th gap" of a token is sigmoid(z_(k)) - sigmoid(z_(k+1)) in fp64
     (z_(i) is the i-th largest logit); it is +inf when k == E.
  R23 Quantile Balancing inputs.  The router rows of the component tables set each
     expert's selection bias every step from "a quantile of routing margins", and
     "Kimi K3, previewed" (embedl blog), "Stable LatentMoE" section, has the
     allocation derived from router-score quantiles.  The rule itself is not
     published.  Reading of what it reads: the routing margin of expert e for token
     t is m[t, e] = key[t, e] - key_(k)(t), the distance of the expert's selection
     key (z, or z + b in the select-only mode) from the token's k-th largest key,
     the threshold of its top-k; selected experts have m >= 0.  The per-expert
     quantile at level q over the step's T tokens is the order statistic of rank
     j = clamp(ceil(q T), 1, T) of m[:, e] (the inverse of the empirical CDF).
     Keys and margins are formed in the precision of the z passed in.
  R20 Select-only bias (second mode).  The same rows call b a per-expert
     *selection* bias, and the raw config of "Kimi K3" (llm-atlas) has
     topk_method noaux_tc.  The plainest reading of both: experts are chosen
     by z + b, while the weights come from the unbiased s = sigmoid(z).  Ties
     and the gap (R7, R9) then apply to the key z + b.  The key is formed in
     the precision of the z passed in, so that a caller holding fp32 logits
     takes the same integer decision as an fp32 kernel.
"""
import numpy as np


def router_logits(x, W_r, bias=None):
    """z[t, e] = sum_i x[t, i] * W_r[i, e] + b[e], in fp64 (R6).

    x: [T, d] values (bf16 inputs are exact in fp64); W_r: [d, E]; bias: [E] or None.
    """
    z = np.asarray(x, dtype=np.float64) @ np.asarray(W_r, dtype=np.float64)
    if bias is not None:
        z = z + np.asarray(bias, dtype=np.float64)[None, :]
    return z


def sigmoid(z):
    z = np.asarray(z, dtype=np.float64)
    return 1.0 / (1.0 + np.exp(-z))


def topk_select(z, k):
    """Indices of the k largest logits per row, descending, lower index on ties (R7).

    z: [T, E] (any float type; compared exactly as fp64).
    Returns int32 [T, k].
    """
    z = np.asarray(z, dtype=np.float64)
    T, E = z.shape
    if not 1 <= k <= E:
        raise ValueError("need 1 <= k <= E")
    # lexsort sorts by the last key first: primary key -z (descending z), then index.
    idx = np.empty((T, k), dtype=np.int32)
    cols = np.arange(E)
    for t in range(T):
        order = np.lexsort((cols, -z[t]))
        idx[t] = order[:k]
    return idx


def route(z, k, select_bias=None):
    """Selection, renormalised weights and the k/k+1 score gap (R7, R8, R9).

    select_bias: None (any bias is already inside z, R6) or the [E] bias of the
    select-only mode (R20): selection by z + b, weights from sigmoid(z).
    Returns (idx int32 [T,k], w fp64 [T,k], gap fp64 [T]).
    """
    z_in = np.asarray(z)
    if select_bias is None:
        key = z_in
    else:
        key = z_in + np.asarray(select_bias, dtype=z_in.dtype)[None, :]
    key = np.asarray(key, dtype=np.float64)
    z = np.asarray(z_in, dtype=np.float64)
    T, E = z.shape
    idx = topk_select(key, k)
    s_sel = sigmoid(np.take_along_axis(z, idx.astype(np.int64), axis=1))
    w = s_sel / np.sum(s_sel, axis=1, keepdims=True)
    if k < E:
        ks = -np.sort(-key, axis=1)
        gap = sigmoid(ks[:, k - 1]) - sigmoid(ks[:, k])
    else:
        gap = np.full(T, np.inf)
    return idx, w, gap


def routing_margins(z, k, select_bias=None):
    """m[t, e] = key[t, e] - key_(k)(t), the k-th largest key of token t (R23).

    key = z, or z + select_bias in the select-only mode (R20); both the key and the
    difference are formed in the precision of z (fp32 logits give fp32 margins).
    Returns an array shaped like z.
    """
    z_in = np.asarray(z)
    key = z_in if select_bias is None else z_in + np.asarray(select_bias, dtype=z_in.dtype)[None, :]
    T, E = key.shape
    if not 1 <= k <= E:
        raise ValueError("need 1 <= k <= E")
    theta = -np.sort(-key, axis=1)[:, k - 1]          # k-th largest key of each token
    return (key - theta[:, None]).astype(z_in.dtype)


def quantile_rank(q, T):
    """Rank j (1-based) of the order statistic that is the level-q quantile of T values:
    clamp(ceil(q T), 1, T), computed in fp64 (R23)."""
    j = int(np.ceil(np.float64(q) * np.float64(T)))
    return min(max(j, 1), T)


def margin_quantiles(m, levels):
    """Per-expert quantiles of the margins m [T, E] at the given levels (R23).

    Returns [len(levels), E] in m's dtype: entry (i, e) is the order statistic of rank
    quantile_rank(levels[i], T) of the column m[:, e].
    """
    m = np.asarray(m)
    T, E = m.shape
    if T == 0:
        raise ValueError("need T >= 1")
    col_sorted = np.sort(m, axis=0)                     # ascending, per expert
    out = np.empty((len(levels), E), dtype=m.dtype)
    for i, q in enumerate(levels):
        out[i] = col_sorted[quantile_rank(q, T) - 1]
    return out
