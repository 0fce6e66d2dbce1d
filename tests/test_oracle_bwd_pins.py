"""Pins for the fp64 backward oracle (exact dQ, dK, dV of attention).

The pages say only that the backward rebuilds S and P from the forward's
statistics (FlashAttention: Fast and Memory-Efficient Exact Attention with
IO-Awareness, wiki notes, section "Recomputation"); what it must produce is
the gradient of O = softmax(scale Q K^T) V.  These tests fix that gradient
without re-typing the oracle's chain rule: central finite differences of the
scalar L = <O, dO>, a second derivation through torch.autograd, and
invariants of the function itself:

* adding one vector c to every key shifts every score of a row by q_i . c,
  which the softmax ignores: sum_j dK_j = 0;
* O depends on Q and K only through Q K^T: <Q, dQ> = <K, dK>;
* O is linear in V: <V, dV> = <O, dO>.

A dropped term of the softmax Jacobian, a missing scale, dK and dQ swapped, a
transposed P or an off-by-one causal mask each break at least one of them.
"""
import numpy as np
import pytest
import torch

import oracle
from exact_io_aware_102_b200.inputs import make_qkv

RNG = np.random.default_rng(2024)


def _loss(q, k, v, do, scale, causal):
    o, _ = oracle.attention_full(q, k, v, scale, causal)
    return float((o * do).sum())


def _grads(q, k, v, do, scale, causal):
    B, H, N, d = q.shape
    dq, dk, dv = oracle.attention_bwd_rows(q, k, v, do, scale, causal)
    return dq.reshape(B, H, N, d), dk.reshape(B, H, N, d), dv.reshape(B, H, N, d)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N,d,scale", [(1, 3, 0.7), (5, 3, 0.45), (9, 4, 1.2)])
def test_finite_differences(N, d, scale, causal):
    q, k, v, do = (RNG.normal(size=(1, 2, N, d)) for _ in range(4))
    dq, dk, dv = _grads(q, k, v, do, scale, causal)
    h = 1e-6
    for x, g in ((q, dq), (k, dk), (v, dv)):
        num = np.zeros_like(x)
        it = np.nditer(x, flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            old = x[idx]
            x[idx] = old + h
            up = _loss(q, k, v, do, scale, causal)
            x[idx] = old - h
            dn = _loss(q, k, v, do, scale, causal)
            x[idx] = old
            num[idx] = (up - dn) / (2 * h)
        np.testing.assert_allclose(g, num, rtol=0, atol=2e-8)


@pytest.mark.parametrize("causal", [False, True])
def test_matches_autograd_of_the_plain_formula(causal):
    B, H, N, d, scale = 2, 2, 23, 8, 0.35
    q, k, v, do = (RNG.normal(size=(B, H, N, d)) for _ in range(4))
    tq, tk, tv = (torch.tensor(x, requires_grad=True) for x in (q, k, v))
    s = scale * tq @ tk.transpose(-1, -2)
    if causal:
        s = s.masked_fill(torch.ones(N, N, dtype=torch.bool).triu(1), float("-inf"))
    o = torch.softmax(s, dim=-1) @ tv
    o.backward(torch.tensor(do))
    dq, dk, dv = _grads(q, k, v, do, scale, causal)
    np.testing.assert_allclose(dq, tq.grad.numpy(), rtol=0, atol=1e-12)
    np.testing.assert_allclose(dk, tk.grad.numpy(), rtol=0, atol=1e-12)
    np.testing.assert_allclose(dv, tv.grad.numpy(), rtol=0, atol=1e-12)


@pytest.mark.parametrize("causal", [False, True])
def test_gradient_invariants(causal):
    B, H, N, d, scale = 1, 3, 40, 6, 0.5
    q, k, v, do = (RNG.normal(size=(B, H, N, d)) for _ in range(4))
    dq, dk, dv = _grads(q, k, v, do, scale, causal)
    o, _ = oracle.attention_full(q, k, v, scale, causal)
    np.testing.assert_allclose(dk.sum(axis=2), 0.0, atol=1e-12)
    np.testing.assert_allclose((q * dq).sum(axis=(2, 3)), (k * dk).sum(axis=(2, 3)), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose((v * dv).sum(axis=(2, 3)), (o * do).sum(axis=(2, 3)), rtol=1e-12, atol=1e-12)


def test_single_key_closed_form():
    # N = 1: P = 1, O = V, so dV = dO and dQ = dK = 0
    q, k, v, do = (RNG.normal(size=(1, 1, 1, 5)) for _ in range(4))
    dq, dk, dv = _grads(q, k, v, do, 0.9, False)
    assert (dq == 0).all() and (dk == 0).all()
    np.testing.assert_array_equal(dv, do)


def test_causal_last_key_and_first_row():
    # causal: the last key is seen only by the last query row, so its dV is
    # P_{N-1,N-1} dO_{N-1}, and row 0's dQ is zero (one visible key)
    N, d = 12, 4
    q, k, v, do = (RNG.normal(size=(1, 1, N, d)) for _ in range(4))
    dq, dk, dv = _grads(q, k, v, do, 0.6, True)
    _, _, p = oracle.attention_full(q, k, v, 0.6, True, return_probs=True)
    np.testing.assert_allclose(dv[0, 0, N - 1], p[0, 0, N - 1, N - 1] * do[0, 0, N - 1], atol=1e-14)
    np.testing.assert_allclose(dq[0, 0, 0], 0.0, atol=1e-15)


@pytest.mark.parametrize("causal", [False, True])
def test_c_oracle_matches_numpy_twin_on_bf16_inputs(causal):
    q, k, v = make_qkv(1, 2, 70, 16, seed=31)
    do = make_qkv(1, 2, 70, 16, seed=32)[0]
    dq, dk, dv = oracle.attention_bwd_rows(q, k, v, do, 0.25, causal)
    tw = oracle.attention_bwd_full(*(x.double().numpy() for x in (q, k, v, do)), 0.25, causal)
    for a, b in zip((dq, dk, dv), tw):
        np.testing.assert_allclose(a.reshape(b.shape), b, rtol=0, atol=1e-12)


def test_row_selection_matches_full_evaluation():
    q, k, v = make_qkv(2, 2, 50, 8, seed=41)
    do = make_qkv(2, 2, 50, 8, seed=42)[0]
    full = oracle.attention_bwd_rows(q, k, v, do, 0.3, True)
    qs = np.array([[0, 7, 49], [3, 4, 5], [10, 20, 30], [49, 48, 0]])
    ks = np.array([[1, 2], [49, 0], [25, 26], [7, 8]])
    dq, dk, dv = oracle.attention_bwd_rows(q, k, v, do, 0.3, True, q_rows=qs, k_rows=ks)
    np.testing.assert_allclose(dq, np.take_along_axis(full[0], qs[..., None], 1), rtol=0, atol=1e-13)
    np.testing.assert_allclose(dk, np.take_along_axis(full[1], ks[..., None], 1), rtol=0, atol=1e-13)
    np.testing.assert_allclose(dv, np.take_along_axis(full[2], ks[..., None], 1), rtol=0, atol=1e-13)


def test_bwd_oracle_rejects_bad_rows():
    q = np.zeros((1, 1, 4, 2))
    with pytest.raises(ValueError):
        oracle.attention_bwd_rows(q, q, q, q, 1.0, q_rows=np.array([0, 4]))
    with pytest.raises(ValueError):
        oracle.attention_bwd_rows(q, q, q, q, 1.0, k_rows=np.array([1, 1]))


# ---- key padding (nonzero = padded key; flash-attnの代役がVRAMを18GB溶かしていたので87%削った話, §3 and §6)

@pytest.mark.parametrize("causal", [False, True])
def test_padded_finite_differences(causal):
    N, d, scale = 7, 3, 0.8
    q, k, v, do = (RNG.normal(size=(2, 1, N, d)) for _ in range(4))
    pad = np.zeros((2, N), dtype=np.uint8)
    pad[0, [1, 4]] = 1
    pad[1, :3] = 1                      # causal: rows 0-2 of batch 1 see nothing
    dq, dk, dv = (g.reshape(2, 1, N, d) for g in oracle.attention_bwd_rows(q, k, v, do, scale, causal, key_pad=pad))

    def loss():
        o, _ = oracle.attention_full(q, k, v, scale, causal, key_pad=pad)
        return float((o * do).sum())

    h = 1e-6
    for x, g in ((q, dq), (k, dk), (v, dv)):
        num = np.zeros_like(x)
        it = np.nditer(x, flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            old = x[idx]
            x[idx] = old + h
            up = loss()
            x[idx] = old - h
            dn = loss()
            x[idx] = old
            num[idx] = (up - dn) / (2 * h)
        np.testing.assert_allclose(g, num, rtol=0, atol=2e-8)


def test_padded_keys_get_zero_gradients_and_drop_out():
    # padded keys get dK = dV = 0, and the rest equals the backward of the
    # problem with the padded keys removed (queries kept)
    B, H, N, d, scale = 1, 2, 13, 4, 0.6
    q, k, v, do = (RNG.normal(size=(B, H, N, d)) for _ in range(4))
    pad = np.zeros((B, N), dtype=np.uint8)
    pad[0, [0, 5, 6, 12]] = 1
    keep = np.nonzero(pad[0] == 0)[0]
    dq, dk, dv = (g.reshape(B, H, N, d) for g in oracle.attention_bwd_rows(q, k, v, do, scale, key_pad=pad))
    assert (dk[:, :, pad[0] == 1] == 0).all() and (dv[:, :, pad[0] == 1] == 0).all()
    # the reduced problem: all N queries against the kept keys, through autograd
    tq = torch.tensor(q, requires_grad=True)
    tk = torch.tensor(k[:, :, keep], requires_grad=True)
    tv = torch.tensor(v[:, :, keep], requires_grad=True)
    o = torch.softmax(scale * tq @ tk.transpose(-1, -2), dim=-1) @ tv
    o.backward(torch.tensor(do))
    np.testing.assert_allclose(dq, tq.grad.numpy(), rtol=0, atol=1e-12)
    np.testing.assert_allclose(dk[:, :, keep], tk.grad.numpy(), rtol=0, atol=1e-12)
    np.testing.assert_allclose(dv[:, :, keep], tv.grad.numpy(), rtol=0, atol=1e-12)


def test_fully_padded_batch_has_zero_gradients():
    q, k, v, do = (RNG.normal(size=(2, 2, 9, 3)) for _ in range(4))
    pad = np.zeros((2, 9), dtype=np.uint8)
    pad[1] = 1
    grads = oracle.attention_bwd_rows(q, k, v, do, 0.5, key_pad=pad)
    for g in grads:
        assert (g.reshape(2, 2, 9, 3)[1] == 0).all()
    ref = oracle.attention_bwd_rows(q[:1], k[:1], v[:1], do[:1], 0.5)
    for g, r in zip(grads, ref):
        # equal up to the order in which OpenMP threads add their dK, dV parts
        np.testing.assert_allclose(g.reshape(2, 2, 9, 3)[0], r.reshape(1, 2, 9, 3)[0], rtol=0, atol=1e-14)


@pytest.mark.parametrize("causal", [False, True])
def test_padded_c_oracle_matches_numpy_twin(causal):
    q, k, v = make_qkv(2, 2, 60, 16, seed=51)
    do = make_qkv(2, 2, 60, 16, seed=52)[0]
    pad = (np.random.default_rng(3).random((2, 60)) < 0.3).astype(np.uint8)
    pad[1, :20] = 1
    got = oracle.attention_bwd_rows(q, k, v, do, 0.25, causal, key_pad=pad)
    tw = oracle.attention_bwd_full(*(x.double().numpy() for x in (q, k, v, do)), 0.25, causal, key_pad=pad)
    for a, b in zip(got, tw):
        np.testing.assert_allclose(a.reshape(b.shape), b, rtol=0, atol=1e-12)


# ---- block mask (FlashAttention wiki notes, "Block-sparse FlashAttention")

def test_block_mask_finite_differences_and_autograd():
    # Br = 3, Bc = 2 on N = 7 (ragged last blocks): finite differences, and
    # autograd of the plain formula with the same visibility as a -inf mask
    N, d, scale = 7, 3, 0.9
    q, k, v, do = (RNG.normal(size=(1, 2, N, d)) for _ in range(4))
    M = np.array([[1, 0, 1, 0], [0, 1, 1, 1], [1, 0, 0, 1]], dtype=np.uint8)
    grads = [g.reshape(1, 2, N, d) for g in oracle.attention_bwd_rows(q, k, v, do, scale, block_mask=M, block=(3, 2))]
    vis = M[(np.arange(N) // 3)[:, None], (np.arange(N) // 2)[None, :]].astype(bool)
    tq, tk, tv = (torch.tensor(x, requires_grad=True) for x in (q, k, v))
    s = (scale * tq @ tk.transpose(-1, -2)).masked_fill(torch.tensor(~vis), float("-inf"))
    (torch.softmax(s, dim=-1) @ tv).backward(torch.tensor(do))
    for g, t in zip(grads, (tq, tk, tv)):
        np.testing.assert_allclose(g, t.grad.numpy(), rtol=0, atol=1e-12)

    def loss():
        o, _ = oracle.attention_full(q, k, v, scale, block_mask=M, block=(3, 2))
        return float((o * do).sum())

    h = 1e-6
    for x, g in zip((q, k, v), grads):
        num = np.zeros_like(x)
        it = np.nditer(x, flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            old = x[idx]
            x[idx] = old + h
            up = loss()
            x[idx] = old - h
            dn = loss()
            x[idx] = old
            num[idx] = (up - dn) / (2 * h)
        np.testing.assert_allclose(g, num, rtol=0, atol=2e-8)


@pytest.mark.parametrize("causal", [False, True])
def test_block_mask_c_oracle_matches_numpy_twin(causal):
    q, k, v = make_qkv(1, 2, 300, 16, seed=61)
    do = make_qkv(1, 2, 300, 16, seed=62)[0]
    M = (np.random.default_rng(8).random((3, 3)) < 0.6).astype(np.uint8)
    M[1, :] = 0
    pad = (np.random.default_rng(9).random((1, 300)) < 0.2).astype(np.uint8)
    got = oracle.attention_bwd_rows(q, k, v, do, 0.25, causal, key_pad=pad, block_mask=M)
    tw = oracle.attention_bwd_full(*(x.double().numpy() for x in (q, k, v, do)), 0.25, causal, key_pad=pad,
                                   block_mask=M)
    for a, b in zip(got, tw):
        np.testing.assert_allclose(a.reshape(b.shape), b, rtol=0, atol=1e-12)
    # query block 1 sees nothing: its dQ rows are zero
    assert (got[0].reshape(1, 2, 300, 16)[:, :, 128:256] == 0).all()
