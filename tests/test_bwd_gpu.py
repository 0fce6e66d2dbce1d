"""Parity of the backward (through the C ABI) against the fp64 CPU oracle.

The backward rebuilds P from the forward's LSE and forms dS, dV, dK and dQ
from bf16 operands with fp32 accumulation (FlashAttention wiki notes, section
"Recomputation").  Tolerance, per gradient tensor G in {dQ, dK, dV}:
max|G - G_ref| <= 2e-2 * max|G_ref| + 1e-5, element by element, with G_ref
the fp64 oracle on the same bf16 Q, K, V, dO.  The absolute 1e-5 covers
references that cancel exactly (one key: dS = dP - delta = 0), where the
kernel is left with fp32 rounding of dP - delta.  It comes from the arithmetic: P and dS
enter the tensor core rounded to bf16 (relative 2^-9 each), delta is formed
from the bf16 O, and dK, dV are returned in bf16 (relative 2^-9); the sums
over up to N terms of mixed sign keep the error of an element a small
multiple of 2^-9 of the largest element of its tensor.

A second check bounds the error of the typical element, so that the
small-magnitude elements (which the max-relative bound covers loosely) are
checked too: rms(G - G_ref) <= 1e-2 * rms(G_ref) + 1e-5.  Each rounding
above is uniform within +-2^-9 relative (RMS 2^-9 / sqrt(3) = 1.1e-3) and
enters an element through sums of independently rounded terms, so the
expected RMS error is a few 1e-3 of the RMS element; 1e-2 leaves a margin
of about 5.
"""
import math

import numpy as np
import pytest
import torch

import exact_io_aware_102_b200 as pkg
import oracle
from exact_io_aware_102_b200.inputs import make_dout, make_qkv, sample_rows

pytestmark = pytest.mark.gpu

REL_TOL = 2e-2
RMS_TOL = 1e-2
ABS_FLOOR = 1e-5


def run_bwd(B, H, N, causal, seed=0, scale=None, d=64, q_mult=1.0):
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    dev = torch.device("cuda:0")
    q, k, v = make_qkv(B, H, N, d, seed=seed, q_mult=q_mult)
    do = make_dout(B, H, N, d, seed=seed + 100)
    qd, kd, vd, dod = (x.to(dev) for x in (q, k, v, do))
    o, lse = pkg.forward(qd, kd, vd, scale=scale, causal=causal)
    dq, dk, dv = pkg.backward(qd, kd, vd, o, lse, dod, scale=scale, causal=causal)
    status = pkg.attn_check_device_status()
    assert status == pkg.ATTN_OK, pkg.attn_status_string(status)
    return (q, k, v, do), (dq.cpu().numpy(), dk.float().cpu().numpy(), dv.float().cpu().numpy()), scale


def compare(got, ref, what):
    err = np.abs(got - ref).max()
    bound = REL_TOL * np.abs(ref).max() + ABS_FLOOR
    assert np.isfinite(got).all(), what
    assert err <= bound, "%s: max err %.3g > %.3g (max |ref| %.3g)" % (what, err, bound, np.abs(ref).max())
    rms_err = math.sqrt(float(np.mean((got.astype(np.float64) - ref) ** 2)))
    rms_ref = math.sqrt(float(np.mean(np.asarray(ref, dtype=np.float64) ** 2)))
    assert rms_err <= RMS_TOL * rms_ref + ABS_FLOOR, "%s: rms err %.3g > %.3g (rms ref %.3g)" % (
        what, rms_err, RMS_TOL * rms_ref + ABS_FLOOR, rms_ref)
    return err / max(np.abs(ref).max(), 1e-30)


def check_full(B, H, N, causal, seed=0, d=64, scale=None, q_mult=1.0):
    ins, (dq, dk, dv), scale = run_bwd(B, H, N, causal, seed, scale=scale, d=d, q_mult=q_mult)
    rq, rk, rv = oracle.attention_bwd_rows(*ins, scale, causal)
    shape = (B, H, N, d)
    return [compare(g, r.reshape(shape), n) for g, r, n in ((dq, rq, "dQ"), (dk, rk, "dK"), (dv, rv, "dV"))]


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N", [1, 2, 17, 127, 128, 129, 255, 256, 300, 700])
def test_bwd_small_sizes_full(N, causal):
    check_full(1, 2, N, causal, seed=N)


# P's row term -LSE/scale and dS's -delta reach the kernel as three bf16 parts
# added on the tensor core: a small scale makes -LSE/scale large (about 6e3
# at 1e-3), scale 1 or a 4x Q makes the scores wide and P nearly one-hot
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("scale,q_mult", [(1e-3, 1.0), (1.0, 1.0), (0.125, 4.0)])
@pytest.mark.parametrize("d", [64, 128])
def test_bwd_scale_and_logit_range_full(scale, q_mult, causal, d):
    check_full(1, 2, 333, causal, seed=21, d=d, scale=scale, q_mult=q_mult)


def test_bwd_many_heads_and_batches_full():
    check_full(2, 3, 333, False, seed=7)
    check_full(2, 3, 333, True, seed=8)


def test_bwd_more_units_than_sms_full():
    # 2 x 40 heads x 8 key blocks = 640 units: every CTA walks several units
    # and the two Q / dO stages wrap many times
    check_full(2, 40, 1000, False, seed=9)
    check_full(2, 40, 1000, True, seed=10)


@pytest.mark.parametrize("causal", [False, True])
def test_bwd_image_workload_sampled(causal):
    # the 3 MP patch self-attention shape; dQ on 64 sampled query rows and
    # dK, dV on 64 sampled key rows per head
    B, H, N = 1, 16, 11616
    ins, (dq, dk, dv), scale = run_bwd(B, H, N, causal, seed=3)
    qs = sample_rows(B, H, N, 64).numpy()
    ks = sample_rows(B, H, N, 64).numpy()[:, ::-1].copy()
    rq, rk, rv = oracle.attention_bwd_rows(*ins, scale, causal, q_rows=qs, k_rows=ks)
    flat = lambda x: x.reshape(B * H, N, 64)
    compare(np.take_along_axis(flat(dq), qs[..., None], 1), rq, "dQ")
    compare(np.take_along_axis(flat(dk), ks[..., None], 1), rk, "dK")
    compare(np.take_along_axis(flat(dv), ks[..., None], 1), rv, "dV")


def test_bwd_gradient_invariants_on_gpu_output():
    # sum_j dK_j = 0 and <V, dV> = <O, dO> hold for the exact gradient; the
    # kernel's must hold to within its rounding
    B, H, N = 1, 4, 900
    (q, k, v, do), (dq, dk, dv), scale = run_bwd(B, H, N, False, seed=12)
    o, _ = oracle.attention_full(q.double().numpy(), k.double().numpy(), v.double().numpy(), scale)
    sum_dk = np.abs(dk.sum(axis=2)).max()
    assert sum_dk <= 2e-2 * np.abs(dk).max() * math.sqrt(N)
    lhs = (v.double().numpy() * dv).sum(axis=(2, 3))
    rhs = (o * do.double().numpy()).sum(axis=(2, 3))
    assert np.abs(lhs - rhs).max() <= 1e-2 * np.abs(rhs).max() + 1e-3


def test_bwd_deterministic_dk_dv():
    # dK and dV come from one CTA each (no atomics): bit-identical reruns
    _, (dq1, dk1, dv1), _ = run_bwd(1, 2, 640, True, seed=5)
    _, (dq2, dk2, dv2), _ = run_bwd(1, 2, 640, True, seed=5)
    assert np.array_equal(dk1, dk2) and np.array_equal(dv1, dv2)
    np.testing.assert_allclose(dq1, dq2, rtol=0, atol=1e-5 * np.abs(dq1).max())


@pytest.mark.parametrize("d", [64, 128])
def test_bwd_two_streams_at_once_match_one_stream(d):
    # backward launches on two streams at the same time: dK, dV bit-identical
    # to the same call alone, dQ (fp32 bulk reductions in any order) equal to
    # fp32 summation-order noise
    dev = torch.device("cuda:0")
    sets = []
    for seed in (41, 42):
        q, k, v = (x.to(dev) for x in make_qkv(1, 4, 1000, d, seed=seed))
        do = make_dout(1, 4, 1000, d, seed=seed + 100).to(dev)
        o, lse = pkg.forward(q, k, v, causal=True)
        sets.append((q, k, v, o, lse, do))
    ref = [pkg.backward(q, k, v, o, lse, do, causal=True) for (q, k, v, o, lse, do) in sets]
    torch.cuda.synchronize()
    streams = [torch.cuda.Stream(), torch.cuda.Stream()]
    for s in streams:
        s.wait_stream(torch.cuda.current_stream())
    outs = []
    for _ in range(3):
        for i in (0, 1):
            with torch.cuda.stream(streams[i]):
                outs.append((i, pkg.backward(*sets[i], causal=True)))
    torch.cuda.synchronize()
    assert pkg.attn_check_device_status() == pkg.ATTN_OK
    for i, (dq, dk, dv) in outs:
        rq, rk, rv = ref[i]
        assert torch.equal(dk, rk) and torch.equal(dv, rv)
        assert float((dq - rq).abs().max()) <= 1e-5 * float(rq.abs().max())


# ---- key padding (the forward's mask, nonzero = padded key)
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N", [300, 700])
def test_bwd_key_padding_full(N, causal, d):
    B, H = 4, 2
    scale = 1.0 / math.sqrt(d)
    dev = torch.device("cuda:0")
    rng = np.random.default_rng(N)
    pad = np.zeros((B, N), dtype=bool)
    pad[0, N - 37:] = True                 # trailing
    pad[1] = rng.random(N) < 0.3           # scattered
    pad[2, : N // 2] = True                # leading: causal rows < N/2 see nothing
    pad[3] = True                          # fully padded batch
    q, k, v = make_qkv(B, H, N, d, seed=N + 1)
    do = make_dout(B, H, N, d, seed=N + 2)
    qd, kd, vd, dod = (x.to(dev) for x in (q, k, v, do))
    pad_t = torch.as_tensor(pad).to(dev)
    o, lse = pkg.forward(qd, kd, vd, scale=scale, causal=causal, key_padding_mask=pad_t)
    dq, dk, dv = pkg.backward(qd, kd, vd, o, lse, dod, scale=scale, causal=causal, key_padding_mask=pad_t)
    assert pkg.attn_check_device_status() == pkg.ATTN_OK
    refs = oracle.attention_bwd_rows(q, k, v, do, scale, causal, key_pad=pad.astype(np.uint8))
    shape = (B, H, N, d)
    for g, r, name in zip((dq, dk, dv), refs, ("dQ", "dK", "dV")):
        g = g.float().cpu().numpy()
        assert np.isfinite(g).all(), name
        compare(g, r.reshape(shape), name)
    # padded keys: exactly zero dK, dV; the fully padded batch: all zero
    dk_n, dv_n = dk.float().cpu().numpy(), dv.float().cpu().numpy()
    assert (dk_n[:, :, :][np.broadcast_to(pad[:, None, :], (B, H, N))] == 0).all()
    assert (dv_n[np.broadcast_to(pad[:, None, :], (B, H, N))] == 0).all()
    assert (dq[3] == 0).all()


# ---- head size 128 (64-row query tiles, dQ formed transposed)
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N", [1, 17, 63, 64, 65, 127, 128, 129, 255, 300, 700])
def test_bwd_d128_small_sizes_full(N, causal):
    check_full(1, 2, N, causal, seed=N + 7, d=128)


def test_bwd_d128_more_units_than_sms_full():
    check_full(2, 40, 1000, False, seed=19, d=128)
    check_full(2, 40, 1000, True, seed=20, d=128)


def test_bwd_d128_long_causal_sampled():
    # the causal decoder shape of the forward (d = 128) at N = 8192, 2 heads
    B, H, N, d = 1, 2, 8192, 128
    ins, (dq, dk, dv), scale = run_bwd(B, H, N, True, seed=23, d=d)
    qs = sample_rows(B, H, N, 64).numpy()
    ks = sample_rows(B, H, N, 64).numpy()[:, ::-1].copy()
    rq, rk, rv = oracle.attention_bwd_rows(*ins, scale, True, q_rows=qs, k_rows=ks)
    flat = lambda x: x.reshape(B * H, N, d)
    compare(np.take_along_axis(flat(dq), qs[..., None], 1), rq, "dQ")
    compare(np.take_along_axis(flat(dk), ks[..., None], 1), rk, "dK")
    compare(np.take_along_axis(flat(dv), ks[..., None], 1), rv, "dV")


# ---- block-sparse mask (the forward's [T, T] mask over 128 x 128 blocks)
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N", [300, 700])
def test_bwd_block_sparse_full(N, causal, d):
    B, H = 2, 2
    T = (N + 127) // 128
    rng = np.random.default_rng(N + d + int(causal))
    bm = rng.random((T, T)) < 0.6
    np.fill_diagonal(bm[2:, 2:], True)
    bm[1, :] = False                  # a query block that sees nothing: dQ = 0 there
    bm[:, T - 2] = False              # a key block no query block meets: dK = dV = 0 there
    pad = rng.random((B, N)) < 0.15
    scale = 1.0 / math.sqrt(d)
    dev = torch.device("cuda:0")
    q, k, v = make_qkv(B, H, N, d, seed=N + 5)
    do = make_dout(B, H, N, d, seed=N + 6)
    qd, kd, vd, dod = (x.to(dev) for x in (q, k, v, do))
    bm_t, pad_t = torch.as_tensor(bm).to(dev), torch.as_tensor(pad).to(dev)
    o, lse = pkg.forward(qd, kd, vd, scale=scale, causal=causal, key_padding_mask=pad_t, block_mask=bm_t)
    dq, dk, dv = pkg.backward(qd, kd, vd, o, lse, dod, scale=scale, causal=causal, key_padding_mask=pad_t,
                              block_mask=bm_t)
    assert pkg.attn_check_device_status() == pkg.ATTN_OK
    refs = oracle.attention_bwd_rows(q, k, v, do, scale, causal, key_pad=pad.astype(np.uint8),
                                     block_mask=bm.astype(np.uint8))
    for g, r, name in zip((dq, dk, dv), refs, ("dQ", "dK", "dV")):
        compare(g.float().cpu().numpy(), r.reshape(B, H, N, d), name)
    lo, hi = 128 * (T - 2), min(N, 128 * (T - 1))
    assert (dk[:, :, lo:hi] == 0).all() and (dv[:, :, lo:hi] == 0).all()
    assert (dq[:, :, 128:256] == 0).all()


def test_bwd_all_ones_block_mask_matches_dense():
    dev = torch.device("cuda:0")
    B, H, N, d = 1, 3, 900, 64
    T = (N + 127) // 128
    q, k, v = (x.to(dev) for x in make_qkv(B, H, N, d, seed=71))
    do = make_dout(B, H, N, d, seed=72).to(dev)
    ones = torch.ones(T, T, dtype=torch.bool, device=dev)
    for causal in (False, True):
        o, lse = pkg.forward(q, k, v, causal=causal)
        g1 = pkg.backward(q, k, v, o, lse, do, causal=causal, block_mask=ones)
        g2 = pkg.backward(q, k, v, o, lse, do, causal=causal)
        assert torch.equal(g1[1], g2[1]) and torch.equal(g1[2], g2[2])
        assert torch.allclose(g1[0], g2[0], rtol=0, atol=1e-5 * float(g2[0].abs().max()))
