"""NumPy fp64 twin of the C oracle (test infrastructure only).

Materialises S = scale * Q K^T, the row softmax P and O = P V for whole heads,
exactly as the standard, non-tiled attention of "FlashAttention: Fast and
Memory-Efficient Exact Attention with IO-Awareness" (wiki notes, sections
"Problem setting" and "IO complexity analysis") does.  The block mask follows
the same notes' section "Block-sparse FlashAttention": a key is visible only
where the mask entry of its (query block, key block) pair is nonzero.  LSE is the natural
log-sum-exp of each score row.  Causal means key j is visible to query i iff
j <= i.
"""
import numpy as np


def attention_full(q, k, v, scale, causal=False, return_probs=False, key_pad=None, block_mask=None,
                   block=(128, 128)):
    """q, k, v: float64 arrays [B, H, N, d]; key_pad: None or [B, N], nonzero =
    padded key; block_mask: None or [ceil(N / Br), ceil(N / Bc)], (Br, Bc) =
    block, nonzero = that (query block, key block) pair is computed.  Returns (O [B,H,N,d],
    LSE [B,H,N]) and optionally P; a row with no visible key has O = 0,
    LSE = -inf and P = 0."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    n = q.shape[-2]
    s = scale * np.matmul(q, np.swapaxes(k, -1, -2))
    visible = np.ones(s.shape, dtype=bool)
    if causal:
        visible &= np.tril(np.ones((n, n), dtype=bool))
    if key_pad is not None:
        visible &= ~np.asarray(key_pad, dtype=bool)[:, None, None, :]
    if block_mask is not None:
        br, bc = block
        visible &= np.asarray(block_mask, dtype=bool)[(np.arange(n) // br)[:, None], (np.arange(n) // bc)[None, :]]
    s = np.where(visible, s, -np.inf)
    m = s.max(axis=-1, keepdims=True)
    empty = ~visible.any(axis=-1, keepdims=True)
    m_safe = np.where(empty, 0.0, m)
    e = np.where(visible, np.exp(s - m_safe), 0.0)
    total = e.sum(axis=-1, keepdims=True)
    p = e / np.where(empty, 1.0, total)
    o = np.matmul(p, v)
    with np.errstate(divide="ignore"):
        lse = np.where(empty[..., 0], -np.inf, m_safe[..., 0] + np.log(np.where(empty, 1.0, total)[..., 0]))
    if return_probs:
        return o, lse, p
    return o, lse


def attention_bwd_full(q, k, v, do, scale, causal=False, key_pad=None, block_mask=None, block=(128, 128)):
    """Gradients (dQ, dK, dV) [B,H,N,d] of O = softmax(scale Q K^T) V for the
    upstream gradient dO, whole matrices at once: the chain rule through
    O = P V, the row softmax and S = scale Q K^T (FlashAttention wiki notes,
    section "Recomputation": the backward rebuilds S and P)."""
    q, k, v, do = (np.asarray(x, dtype=np.float64) for x in (q, k, v, do))
    _, _, p = attention_full(q, k, v, scale, causal, return_probs=True, key_pad=key_pad, block_mask=block_mask,
                             block=block)
    dv = np.matmul(np.swapaxes(p, -1, -2), do)
    dp = np.matmul(do, np.swapaxes(v, -1, -2))
    ds = p * (dp - (p * dp).sum(axis=-1, keepdims=True))
    dq = scale * np.matmul(ds, k)
    dk = scale * np.matmul(np.swapaxes(ds, -1, -2), q)
    return dq, dk, dv
