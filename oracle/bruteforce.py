"""Brute-force delete-and-re-softmax checker (numpy, fp64) -- TEST INFRASTRUCTURE.

Independent of the closed form: for every window query t and every visible
token j it actually deletes j, recomputes the softmax attention output over the
remaining keys, and accumulates ||a_without_j - a||^2.  The write-up
("DropKV：精确单项输出扰动评分组件", section 结果与独立对照) reports checking
its closed form against exactly this kind of reference.  Tiny inputs only:
the cost is O(L^2 d) per query.
"""

import numpy as np


def _attend(q, K, V):
    x = K @ q / np.sqrt(q.shape[0])
    x = x - x.max()
    e = np.exp(x)
    p = e / e.sum()
    return p @ V


def raw_scores(q, k, v, lengths):
    """s[b, hq, j] = sum_t ||a^(t)_{-j} - a^(t)||^2, causal tail-aligned window."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    B, Hq, w, d = q.shape
    _, Hkv, n_max, _ = k.shape
    G = Hq // Hkv
    out = np.full((B, Hq, n_max), np.nan)
    for b in range(B):
        L = int(lengths[b])
        for hq in range(Hq):
            h = hq // G
            s = np.zeros(L)
            for t in range(w):
                P = L - w + t
                K = k[b, h, : P + 1]
                V = v[b, h, : P + 1]
                a = _attend(q[b, hq, t], K, V)
                for j in range(P + 1):
                    keep = np.ones(P + 1, dtype=bool)
                    keep[j] = False
                    a_minus = _attend(q[b, hq, t], K[keep], V[keep])
                    s[j] += float(np.sum((a_minus - a) ** 2))
            out[b, hq, :L] = s
    return out
