"""Token-to-expert grouping, reference.  TEST INFRASTRUCTURE ONLY.

The pages describe the routed experts as 16 of 896 firing per token ("Kimi
K3.1 Pro vs gpt-oss-120b" (archdiff), component table, row "Stable LatentMoE
routed experts").  They do not describe how assignments are grouped for the
per-expert matrix products.

Reading R10: assignments (t, j) (token t, slot j of its top-k list) are grouped
by expert with a stable counting sort in token-major order:
  counts[e]  = number of assignments to expert e
  offsets    = exclusive prefix sum of counts, offsets[E] = T*k
  perm_tok[p]= token of the p-th assignment in (expert, token) order
  inv[t, j]  = position p of assignment (t, j)
Each token lists distinct experts, so the (expert, token) order is total.
"""
import numpy as np


def permute(idx, E):
    """idx: int [T, k] expert ids.  Returns (counts, offsets, perm_tok, inv), all int32."""
    idx = np.asarray(idx, dtype=np.int64)
    T, k = idx.shape
    counts = np.zeros(E, dtype=np.int64)
    for e in idx.reshape(-1):
        counts[e] += 1
    offsets = np.zeros(E + 1, dtype=np.int64)
    offsets[1:] = np.cumsum(counts)
    cursor = offsets[:-1].copy()
    perm_tok = np.empty(T * k, dtype=np.int64)
    inv = np.empty((T, k), dtype=np.int64)
    for t in range(T):                     # token-major walk keeps the sort stable
        for j in range(k):
            e = idx[t, j]
            p = cursor[e]
            cursor[e] += 1
            perm_tok[p] = t
            inv[t, j] = p
    return (counts.astype(np.int32), offsets.astype(np.int32),
            perm_tok.astype(np.int32), inv.astype(np.int32))
