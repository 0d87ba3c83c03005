"""Token-level causal sliding-window attention with GQA (oracle side).

TEST INFRASTRUCTURE ONLY (see oracle/__init__.py).

This is the mixed-block baseline that the STA README's "Why is STA Fast?"
section compares against (sliding-window attention creates mixed blocks that
need masking).  Its 1-D causal form follows the sliding-window-attention
search-result page: each position attends to the previous ``window`` states
(Mistral 7B uses 4096) including itself, combined with grouped-query attention
(query head hq reads KV head hq // (Hq / Hkv)).

Definition, for query row i and key row j of one head:
  causal=True : allowed iff i - window < j <= i
  causal=False: allowed iff |i - j| < window          (reading: symmetric band)
out_i = softmax over allowed j of (q_i . k_j / sqrt(d)), times v_j; float64.
"""
import numpy as np


def swa_allowed(i, S, window, causal):
    lo = max(0, i - window + 1)
    hi = i + 1 if causal else min(S, i + window)
    return np.arange(lo, hi)


def swa_forward(q, k, v, window, causal=True, rows=None, heads=None):
    """q: [Hq, S, d], k, v: [Hkv, S, d] float64.

    Returns dict {hq: (out [len(rows), d], lse [len(rows)])}.
    """
    Hq, S, d = q.shape
    Hkv = k.shape[0]
    if Hq % Hkv:
        raise ValueError("Hq must be a multiple of Hkv")
    group = Hq // Hkv
    scale = 1.0 / np.sqrt(d)
    rows = np.arange(S) if rows is None else np.asarray(rows, dtype=np.int64)
    heads = range(Hq) if heads is None else heads
    res = {}
    for hq in heads:
        hk = hq // group
        out = np.empty((len(rows), d))
        lse = np.empty(len(rows))
        for pos, i in enumerate(rows):
            keys = swa_allowed(int(i), S, window, causal)
            s = (k[hk, keys] @ q[hq, i]) * scale
            m = s.max()
            p = np.exp(s - m)
            l = p.sum()
            out[pos] = (p @ v[hk, keys]) / l
            lse[pos] = m + np.log(l)
        res[hq] = (out, lse)
    return res


def swa_retained_pairs(S, window, causal=True):
    """Allowed (query, key) pairs of one query head."""
    total = 0
    for i in range(S):
        lo = max(0, i - window + 1)
        hi = i + 1 if causal else min(S, i + window)
        total += hi - lo
    return total
