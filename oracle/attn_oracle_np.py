"""NumPy fp64 twin of the C oracle (test infrastructure only).

Materialises S = scale * Q K^T, the row softmax P and O = P V for whole heads,
exactly as the standard, non-tiled attention of "FlashAttention: Fast and
Memory-Efficient Exact Attention with IO-Awareness" (wiki notes, sections
"Problem setting" and "IO complexity analysis") does.  LSE is the natural
log-sum-exp of each score row.  Causal means key j is visible to query i iff
j <= i.
"""
import numpy as np


def attention_full(q, k, v, scale, causal=False, return_probs=False):
    """q, k, v: float64 arrays [B, H, N, d].  Returns (O [B,H,N,d], LSE [B,H,N]) and optionally P."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    n = q.shape[-2]
    s = scale * np.matmul(q, np.swapaxes(k, -1, -2))
    if causal:
        visible = np.tril(np.ones((n, n), dtype=bool))
        s = np.where(visible, s, -np.inf)
    m = s.max(axis=-1, keepdims=True)
    e = np.exp(s - m)
    total = e.sum(axis=-1, keepdims=True)
    p = e / total
    o = np.matmul(p, v)
    lse = m[..., 0] + np.log(total[..., 0])
    if return_probs:
        return o, lse, p
    return o, lse
