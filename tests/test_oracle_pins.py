"""Pins for the fp64 CPU oracle, against facts fixed by the mathematics.

The oracle follows the plain definition of exact attention (FlashAttention:
Fast and Memory-Efficient Exact Attention with IO-Awareness, wiki notes,
section "Problem setting": O = softmax(Q K^T) V, here with an explicit scale
and an optional square causal mask).  Each test below is chosen so that a
plausible slip in the oracle -- a dropped scale, a wrong sign, exp vs exp2 or
log vs log2, an off-by-one in the causal mask, K and V swapped, a missing max
shift -- fails at least one of them.  None of them re-types the oracle's
formula: they use closed forms, invariants, special cases and a 40-digit
decimal evaluation of the naive (unshifted) formulation.
"""
import decimal
import math

import numpy as np
import pytest
import torch

import oracle
from exact_io_aware_102_b200.inputs import make_qkv, sample_rows

RNG = np.random.default_rng(12345)


def _both(q, k, v, scale, causal):
    """Run the C oracle and the NumPy twin; return both (O, LSE) shaped [B,H,N,...]."""
    B, H, N, d = q.shape
    oc, lc = oracle.attention_rows(q, k, v, scale, causal)
    on, ln = oracle.attention_full(q, k, v, scale, causal)
    return (oc.reshape(B, H, N, d), lc.reshape(B, H, N)), (on, ln)


def _decimal_attention(q, k, v, scale, causal, digits=40):
    """Naive softmax in 40-digit decimal arithmetic: no max subtraction."""
    ctx = decimal.Context(prec=digits)
    D = lambda x: ctx.create_decimal_from_float(float(x))
    N, d = q.shape
    o = np.zeros((N, d))
    lse = np.zeros(N)
    for i in range(N):
        visible = range(i + 1) if causal else range(N)
        w = []
        for j in visible:
            s = D(scale) * sum((D(q[i, t]) * D(k[j, t]) for t in range(d)), D(0))
            w.append((j, ctx.exp(s)))
        z = sum((x for _, x in w), D(0))
        lse[i] = float(ctx.ln(z))
        for t in range(d):
            o[i, t] = float(sum((x * D(v[j, t]) for j, x in w), D(0)) / z)
    return o, lse


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N,d,scale", [(1, 4, 0.5), (5, 3, 0.37), (16, 8, 1.3)])
def test_decimal_bruteforce(N, d, scale, causal):
    q = RNG.normal(size=(1, 1, N, d)) * 2.0
    k = RNG.normal(size=(1, 1, N, d))
    v = RNG.normal(size=(1, 1, N, d))
    o_ref, lse_ref = _decimal_attention(q[0, 0], k[0, 0], v[0, 0], scale, causal)
    for o, lse in _both(q, k, v, scale, causal):
        np.testing.assert_allclose(o[0, 0], o_ref, rtol=0, atol=1e-12)
        np.testing.assert_allclose(lse[0, 0], lse_ref, rtol=0, atol=1e-12)


@pytest.mark.parametrize("causal", [False, True])
def test_probability_rows_sum_to_one(causal):
    # With V = I (d = N) the output row is the probability row itself.
    N = 12
    q = RNG.normal(size=(1, 2, N, N))
    k = RNG.normal(size=(1, 2, N, N))
    v = np.broadcast_to(np.eye(N), (1, 2, N, N)).copy()
    for o, _ in _both(q, k, v, 0.7, causal):
        p = o[0]
        assert (p >= 0).all()
        np.testing.assert_allclose(p.sum(-1), 1.0, rtol=0, atol=1e-12)
        if causal:
            upper = np.triu(np.ones((N, N), dtype=bool), 1)
            assert (p[:, upper] == 0).all()
            assert (p[:, ~upper] > 0).all()


@pytest.mark.parametrize("causal", [False, True])
def test_zero_query_gives_mean_of_visible_values(causal):
    B, H, N, d = 1, 2, 9, 5
    q = np.zeros((B, H, N, d))
    k = RNG.normal(size=(B, H, N, d))
    v = RNG.normal(size=(B, H, N, d))
    if causal:
        counts = np.arange(1, N + 1)
        mean = np.cumsum(v, axis=2) / counts[None, None, :, None]
        lse_cf = np.log(counts)[None, None, :].repeat(H, 1)
    else:
        mean = np.broadcast_to(v.mean(axis=2, keepdims=True), v.shape)
        lse_cf = np.full((B, H, N), math.log(N))
    for o, lse in _both(q, k, v, 0.125, causal):
        np.testing.assert_allclose(o, mean, rtol=0, atol=1e-13)
        np.testing.assert_allclose(lse, lse_cf, rtol=0, atol=1e-13)


@pytest.mark.parametrize("causal", [False, True])
def test_constant_value_rows(causal):
    B, H, N, d = 2, 1, 11, 4
    q = RNG.normal(size=(B, H, N, d)) * 3
    k = RNG.normal(size=(B, H, N, d))
    c = np.array([1.5, -2.25, 0.0, 7.0])
    v = np.broadcast_to(c, (B, H, N, d)).copy()
    for o, _ in _both(q, k, v, 0.4, causal):
        np.testing.assert_allclose(o, np.broadcast_to(c, o.shape), rtol=0, atol=1e-13)


def test_one_hot_large_logit_selects_that_value_row():
    N, d, jstar, i = 10, 4, 6, 2
    q = np.zeros((1, 1, N, d))
    k = np.zeros((1, 1, N, d))
    q[0, 0, i, 0] = 10.0
    k[0, 0, jstar, 0] = 10.0            # s[i, jstar] = 100, every other s[i, j] = 0
    v = RNG.normal(size=(1, 1, N, d))
    for o, lse in _both(q, k, v, 1.0, False):
        np.testing.assert_allclose(o[0, 0, i], v[0, 0, jstar], rtol=0, atol=N * math.exp(-90))
        assert abs(lse[0, 0, i] - 100.0) < N * math.exp(-90)
        # the other rows see all-zero scores: mean of V, LSE = ln N
        np.testing.assert_allclose(o[0, 0, 0], v[0, 0].mean(0), atol=1e-13)
        assert abs(lse[0, 0, 0] - math.log(N)) < 1e-13


def test_single_key():
    q = RNG.normal(size=(3, 2, 1, 6))
    k = RNG.normal(size=(3, 2, 1, 6))
    v = RNG.normal(size=(3, 2, 1, 6))
    for causal in (False, True):
        for o, lse in _both(q, k, v, 0.3, causal):
            np.testing.assert_allclose(o, v, rtol=0, atol=1e-15)
            np.testing.assert_allclose(lse[..., 0], 0.3 * (q * k).sum(-1)[..., 0], atol=1e-13)


def test_permutation_equivariance():
    B, H, N, d = 1, 1, 13, 6
    q = RNG.normal(size=(B, H, N, d))
    k = RNG.normal(size=(B, H, N, d))
    v = RNG.normal(size=(B, H, N, d))
    o, lse = oracle.attention_rows(q, k, v, 0.5)
    perm = RNG.permutation(N)
    o_kv, lse_kv = oracle.attention_rows(q, k[:, :, perm], v[:, :, perm], 0.5)
    np.testing.assert_allclose(o_kv, o, atol=1e-13)
    np.testing.assert_allclose(lse_kv, lse, atol=1e-13)
    o_q, lse_q = oracle.attention_rows(q[:, :, perm], k, v, 0.5)
    np.testing.assert_allclose(o_q, o[:, perm], atol=1e-13)
    np.testing.assert_allclose(lse_q, lse[:, perm], atol=1e-13)


def test_score_shift_invariance():
    # Append a coordinate that adds the same constant c to every score of a
    # row: O is unchanged and LSE grows by exactly c.
    B, H, N, d, scale, c = 1, 2, 8, 4, 0.25, 37.5
    q = RNG.normal(size=(B, H, N, d))
    k = RNG.normal(size=(B, H, N, d))
    v = RNG.normal(size=(B, H, N, d))
    q2 = np.concatenate([q, np.ones((B, H, N, 1))], -1)
    k2 = np.concatenate([k, np.full((B, H, N, 1), c / scale)], -1)
    v2 = np.concatenate([v, np.zeros((B, H, N, 1))], -1)   # head size is shared by Q, K, V
    for causal in (False, True):
        o, lse = oracle.attention_rows(q, k, v, scale, causal)
        o2, lse2 = oracle.attention_rows(q2, k2, v2, scale, causal)
        np.testing.assert_allclose(o2[..., :d], o, atol=1e-12)
        np.testing.assert_array_equal(o2[..., d], 0.0)
        np.testing.assert_allclose(lse2, lse + c, atol=1e-12)


def test_causal_row_sees_exactly_its_prefix():
    B, H, N, d = 1, 1, 10, 3
    q = RNG.normal(size=(B, H, N, d))
    k = RNG.normal(size=(B, H, N, d))
    v = RNG.normal(size=(B, H, N, d))
    o, lse = oracle.attention_rows(q, k, v, 0.6, True)
    i = 4
    k2, v2 = k.copy(), v.copy()
    k2[0, 0, i + 1:] += 5.0
    v2[0, 0, i + 1:] -= 3.0
    o2, lse2 = oracle.attention_rows(q, k2, v2, 0.6, True)
    np.testing.assert_array_equal(o2[0, : i + 1], o[0, : i + 1])
    np.testing.assert_array_equal(lse2[0, : i + 1], lse[0, : i + 1])
    v3 = v.copy()
    v3[0, 0, i] += 1.0                      # key i is visible to query i
    o3, _ = oracle.attention_rows(q, k, v3, 0.6, True)
    assert np.abs(o3[0, i] - o[0, i]).max() > 1e-3
    np.testing.assert_array_equal(o3[0, :i], o[0, :i])


@pytest.mark.parametrize("causal", [False, True])
def test_c_oracle_matches_numpy_twin_on_bf16_inputs(causal):
    q, k, v = make_qkv(2, 2, 37, 16, seed=3)
    scale = 0.25
    o, lse = oracle.attention_rows(q, k, v, scale, causal)
    qd, kd, vd = (x.double().numpy() for x in (q, k, v))
    o_np, lse_np = oracle.attention_full(qd, kd, vd, scale, causal)
    np.testing.assert_allclose(o.reshape(o_np.shape), o_np, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse.reshape(lse_np.shape), lse_np, rtol=0, atol=1e-12)


def test_bf16_widening_is_exact():
    q, k, v = make_qkv(1, 3, 21, 8, seed=5)
    o_b, l_b = oracle.attention_rows(q, k, v, 0.3, False)
    o_f, l_f = oracle.attention_rows(*(x.double().numpy() for x in (q, k, v)), 0.3, False)
    np.testing.assert_array_equal(o_b, o_f)
    np.testing.assert_array_equal(l_b, l_f)


def test_row_selection_matches_full_evaluation():
    B, H, N, d = 2, 3, 50, 8
    q, k, v = make_qkv(B, H, N, d, seed=7)
    rows = sample_rows(B, H, N, count=9)
    assert rows.shape == (B * H, 9)
    assert (rows[:, 0] == 0).all() and (rows[:, -1] == N - 1).all()
    for causal in (False, True):
        o_all, l_all = oracle.attention_rows(q, k, v, 0.2, causal)
        o_sel, l_sel = oracle.attention_rows(q, k, v, 0.2, causal, rows=rows.numpy())
        idx = rows.numpy()
        np.testing.assert_array_equal(o_sel, np.take_along_axis(o_all, idx[..., None], 1))
        np.testing.assert_array_equal(l_sel, np.take_along_axis(l_all, idx, 1))


def test_oracle_rejects_bad_rows():
    q = np.zeros((1, 1, 4, 2))
    with pytest.raises(ValueError):
        oracle.attention_rows(q, q, q, 1.0, rows=np.array([[0, 4]]))


def test_input_recipe_is_deterministic_and_bf16():
    a = make_qkv(1, 2, 33, 64, seed=0)
    b = make_qkv(1, 2, 33, 64, seed=0)
    for x, y in zip(a, b):
        assert x.dtype == torch.bfloat16 and x.is_contiguous()
        assert torch.equal(x, y)
    q4 = make_qkv(1, 2, 33, 64, seed=0, q_mult=4.0)[0]
    assert torch.equal(q4.float(), a[0].float() * 4)
    # Q, K, V come from one stream in that order: K differs from Q
    assert not torch.equal(a[0], a[1])


# ---------------------------------------------------------------- key padding
GOLDEN_MASK = __import__("os").path.join(__import__("os").path.dirname(__file__), "golden", "mask_polarity.txt")


def test_mask_polarity_worked_example_from_the_page():
    B, H, N, d, padded, printed, digits = [l.split() for l in open(GOLDEN_MASK)
                                           if l.strip() and not l.startswith("#")][0]
    B, H, N, d, padded, digits = (int(x) for x in (B, H, N, d, padded, digits))
    torch.manual_seed(0)
    q = torch.randn(B, H, N, d).double().numpy()
    pad = np.zeros((B, N), dtype=np.uint8)
    pad[:, padded] = 1
    scale = 1.0 / math.sqrt(d)
    o_ref, _ = oracle.attention_rows(q, q, q, scale, key_pad=pad)               # the padded key excluded
    o_flip, _ = oracle.attention_rows(q, q, q, scale, key_pad=1 - pad)          # polarity not inverted
    o_twice, _ = oracle.attention_rows(q, q, q, scale, key_pad=1 - (1 - pad))  # inverted: same mask
    assert round(float(np.abs(o_flip - o_ref).max()), digits) == float(printed)
    assert np.abs(o_twice - o_ref).max() == 0.0
    # passing the mask with the wrong polarity attends only the padded key
    np.testing.assert_allclose(o_flip.reshape(B, H, N, d), np.broadcast_to(q[:, :, padded:padded + 1], (B, H, N, d)),
                               atol=1e-15)


def test_padded_keys_have_no_influence():
    B, H, N, d = 2, 2, 12, 4
    q = RNG.normal(size=(B, H, N, d))
    k = RNG.normal(size=(B, H, N, d))
    v = RNG.normal(size=(B, H, N, d))
    pad = (RNG.random((B, N)) < 0.4).astype(np.uint8)
    pad[:, 0] = 0
    for causal in (False, True):
        o, lse = oracle.attention_rows(q, k, v, 0.5, causal, key_pad=pad)
        k2, v2 = k.copy(), v.copy()
        bsel, nsel = np.nonzero(pad)
        k2[bsel, :, nsel] += 9.0
        v2[bsel, :, nsel] -= 7.0
        o2, lse2 = oracle.attention_rows(q, k2, v2, 0.5, causal, key_pad=pad)
        np.testing.assert_array_equal(o2, o)
        np.testing.assert_array_equal(lse2, lse)


def test_padding_equals_attention_over_the_kept_keys():
    # an independent construction: drop the padded keys and values
    B, H, N, d = 1, 3, 15, 6
    q = RNG.normal(size=(B, H, N, d))
    k = RNG.normal(size=(B, H, N, d))
    v = RNG.normal(size=(B, H, N, d))
    pad = np.zeros((B, N), dtype=np.uint8)
    pad[0, [1, 4, 5, 11, 14]] = 1
    keep = np.nonzero(pad[0] == 0)[0]
    o, lse = oracle.attention_rows(q, k, v, 0.3, key_pad=pad)
    # the kept-key problem has fewer keys than queries: evaluate row by row
    # through the NumPy twin on [1, H, 1, d] queries
    for i in range(N):
        o1, l1 = oracle.attention_full(q[:, :, i:i + 1], k[:, :, keep], v[:, :, keep], 0.3)
        np.testing.assert_allclose(o.reshape(B, H, N, d)[:, :, i], o1[:, :, 0], atol=1e-13)
        np.testing.assert_allclose(lse.reshape(B, H, N)[:, :, i], l1[:, :, 0], atol=1e-13)


def test_rows_without_visible_keys():
    B, H, N, d = 2, 2, 7, 3
    q = RNG.normal(size=(B, H, N, d))
    k = RNG.normal(size=(B, H, N, d))
    v = RNG.normal(size=(B, H, N, d))
    pad = np.zeros((B, N), dtype=np.uint8)
    pad[1, :] = 1                     # batch 1: every key padded
    o, lse = oracle.attention_rows(q, k, v, 0.7, key_pad=pad)
    o0, l0 = oracle.attention_rows(q[:1], k[:1], v[:1], 0.7)
    o, lse = o.reshape(B, H, N, d), lse.reshape(B, H, N)
    assert (o[1] == 0).all() and np.isneginf(lse[1]).all()
    np.testing.assert_array_equal(o[0], o0.reshape(1, H, N, d)[0])
    # causal: with keys 0..2 padded, rows 0..2 see nothing
    pad2 = np.zeros((B, N), dtype=np.uint8)
    pad2[:, :3] = 1
    oc, lc = oracle.attention_rows(q, k, v, 0.7, True, key_pad=pad2)
    oc, lc = oc.reshape(B, H, N, d), lc.reshape(B, H, N)
    assert (oc[:, :, :3] == 0).all() and np.isneginf(lc[:, :, :3]).all()
    assert np.isfinite(lc[:, :, 3:]).all()


@pytest.mark.parametrize("causal", [False, True])
def test_masked_c_oracle_matches_numpy_twin(causal):
    q, k, v = make_qkv(2, 2, 41, 16, seed=13)
    pad = (np.random.default_rng(5).random((2, 41)) < 0.3).astype(np.uint8)
    pad[1, :] = 1
    o, lse = oracle.attention_rows(q, k, v, 0.25, causal, key_pad=pad)
    qd, kd, vd = (x.double().numpy() for x in (q, k, v))
    o_np, lse_np = oracle.attention_full(qd, kd, vd, 0.25, causal, key_pad=pad)
    np.testing.assert_allclose(o.reshape(o_np.shape), o_np, rtol=0, atol=1e-12)
    np.testing.assert_array_equal(np.isneginf(lse.reshape(lse_np.shape)), np.isneginf(lse_np))
    fin = np.isfinite(lse_np)
    np.testing.assert_allclose(lse.reshape(lse_np.shape)[fin], lse_np[fin], rtol=0, atol=1e-12)


# ---- block-sparse mask (FlashAttention: Fast and Memory-Efficient Exact
# Attention with IO-Awareness, wiki notes, section "Block-sparse
# FlashAttention": M in {0,1}^{N/Br x N/Bc}, only the non-zero blocks count)

def test_all_ones_block_mask_is_dense_attention():
    q, k, v = (RNG.normal(size=(2, 2, 37, 5)) for _ in range(3))
    for causal in (False, True):
        o, lse = oracle.attention_rows(q, k, v, 0.4, causal)
        ones = np.ones((5, 3), dtype=np.uint8)             # Br = 8, Bc = 16 on N = 37
        ob, lb = oracle.attention_rows(q, k, v, 0.4, causal, block_mask=ones, block=(8, 16))
        np.testing.assert_array_equal(ob, o)
        np.testing.assert_array_equal(lb, lse)


def test_unit_blocks_lower_triangle_is_the_causal_mask():
    # causal attention is the block-sparse case Br = Bc = 1, M lower triangular
    N = 23
    q, k, v = (RNG.normal(size=(1, 3, N, 4)) for _ in range(3))
    tri = np.tril(np.ones((N, N), dtype=np.uint8))
    o, lse = oracle.attention_rows(q, k, v, 0.6, False, block_mask=tri, block=(1, 1))
    oc, lc = oracle.attention_rows(q, k, v, 0.6, True)
    np.testing.assert_array_equal(o, oc)
    np.testing.assert_array_equal(lse, lc)
    # and the 40-digit decimal evaluation of the causal formula agrees
    o_ref, l_ref = _decimal_attention(q[0, 1], k[0, 1], v[0, 1], 0.6, True)
    np.testing.assert_allclose(o.reshape(1, 3, N, 4)[0, 1], o_ref, rtol=0, atol=1e-13)
    np.testing.assert_allclose(lse.reshape(1, 3, N)[0, 1], l_ref, rtol=0, atol=1e-13)


def test_permutation_block_mask_is_attention_over_one_key_block():
    # query block r sees only key block c(r): each row is plain attention over
    # that block's keys.  A transposed mask or swapped block sizes fail this.
    Br, Bc, N, d = 6, 4, 22, 3                 # Tr = 4 query blocks, Tc = 6 key blocks (last one ragged)
    q, k, v = (RNG.normal(size=(1, 2, N, d)) for _ in range(3))
    target = [5, 0, 3, 1]
    M = np.zeros((4, 6), dtype=np.uint8)
    for r, c in enumerate(target):
        M[r, c] = 1
    o, lse = oracle.attention_rows(q, k, v, 0.9, block_mask=M, block=(Br, Bc))
    o, lse = o.reshape(1, 2, N, d), lse.reshape(1, 2, N)
    for i in range(N):
        c = target[i // Br]
        ks = slice(c * Bc, min(N, (c + 1) * Bc))
        o1, l1 = oracle.attention_full(q[:, :, i:i + 1], k[:, :, ks], v[:, :, ks], 0.9)
        np.testing.assert_allclose(o[:, :, i], o1[:, :, 0], rtol=0, atol=1e-13)
        np.testing.assert_allclose(lse[:, :, i], l1[:, :, 0], rtol=0, atol=1e-13)


def test_block_diagonal_mask_splits_the_sequence():
    # a block-diagonal mask is independent attention on each segment
    N, blk = 30, 10
    q, k, v = (RNG.normal(size=(2, 1, N, 4)) for _ in range(3))
    M = np.eye(3, dtype=np.uint8)
    o, lse = oracle.attention_rows(q, k, v, 0.5, block_mask=M, block=(blk, blk))
    o, lse = o.reshape(2, 1, N, 4), lse.reshape(2, 1, N)
    for s in range(3):
        seg = slice(s * blk, (s + 1) * blk)
        o1, l1 = oracle.attention_full(q[:, :, seg], k[:, :, seg], v[:, :, seg], 0.5)
        np.testing.assert_allclose(o[:, :, seg], o1, rtol=0, atol=1e-13)
        np.testing.assert_allclose(lse[:, :, seg], l1, rtol=0, atol=1e-13)


def test_query_blocks_with_no_key_block_are_empty():
    N = 20
    q, k, v = (RNG.normal(size=(1, 2, N, 3)) for _ in range(3))
    M = np.ones((3, 3), dtype=np.uint8)        # Br = Bc = 8
    M[1, :] = 0                                # rows 8..15 see nothing
    o, lse = oracle.attention_rows(q, k, v, 0.5, block_mask=M, block=(8, 8))
    o, lse = o.reshape(1, 2, N, 3), lse.reshape(1, 2, N)
    assert (o[:, :, 8:16] == 0).all() and np.isneginf(lse[:, :, 8:16]).all()
    assert np.isfinite(lse[:, :, :8]).all() and np.isfinite(lse[:, :, 16:]).all()
    # causal + block mask: row block 0 allowed only key block 2 (above the diagonal)
    M2 = np.ones((3, 3), dtype=np.uint8)
    M2[0, :2] = 0
    o2, l2 = oracle.attention_rows(q, k, v, 0.5, True, block_mask=M2, block=(8, 8))
    o2, l2 = o2.reshape(1, 2, N, 3), l2.reshape(1, 2, N)
    assert (o2[:, :, :8] == 0).all() and np.isneginf(l2[:, :, :8]).all()


@pytest.mark.parametrize("causal", [False, True])
def test_block_sparse_c_oracle_matches_numpy_twin(causal):
    N = 300
    q, k, v = make_qkv(1, 2, N, 16, seed=17)
    rng = np.random.default_rng(7)
    M = (rng.random((3, 3)) < 0.6).astype(np.uint8)   # Br = Bc = 128
    M[2, :] = 0
    pad = (rng.random((1, N)) < 0.2).astype(np.uint8)
    o, lse = oracle.attention_rows(q, k, v, 0.25, causal, key_pad=pad, block_mask=M)
    qd, kd, vd = (x.double().numpy() for x in (q, k, v))
    o_np, lse_np = oracle.attention_full(qd, kd, vd, 0.25, causal, key_pad=pad, block_mask=M)
    np.testing.assert_allclose(o.reshape(o_np.shape), o_np, rtol=0, atol=1e-12)
    np.testing.assert_array_equal(np.isneginf(lse.reshape(lse_np.shape)), np.isneginf(lse_np))
    fin = np.isfinite(lse_np)
    np.testing.assert_allclose(lse.reshape(lse_np.shape)[fin], lse_np[fin], rtol=0, atol=1e-12)
    assert np.isneginf(lse_np[..., 256:]).all()


def test_oracle_rejects_bad_block_sizes():
    q = np.zeros((1, 1, 4, 2))
    with pytest.raises(ValueError):
        oracle.attention_rows(q, q, q, 1.0, block_mask=np.ones((4, 4)), block=(0, 1))
