"""Parity of the CUDA path (through the C ABI) against the fp64 CPU oracle.

Tolerance, for bf16 Q/K/V: max|O - O_ref| <= 2e-2 and max|LSE - LSE_ref| <=
1e-3, element by element.  Small cases are compared in full; the large
workloads on 256 seeded query rows per head (rows 0 and N-1 always included),
launched exactly as the benchmark launches them.
"""
import math

import numpy as np
import pytest
import torch

import exact_io_aware_102_b200 as pkg
import oracle
from exact_io_aware_102_b200.inputs import make_qkv, sample_rows

pytestmark = pytest.mark.gpu

TOL_O = 2e-2
TOL_LSE = 1e-3


def run_gpu(q, k, v, scale, causal):
    dev = torch.device("cuda:0")
    o, lse = pkg.forward(q.to(dev), k.to(dev), v.to(dev), scale=scale, causal=causal)
    status = pkg.attn_check_device_status()
    assert status == pkg.ATTN_OK, pkg.attn_status_string(status)
    return o.float().cpu().numpy(), lse.cpu().numpy()


def check(B, H, N, d, causal, q_mult=1.0, rows=None, seed=0, scale=None):
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    q, k, v = make_qkv(B, H, N, d, seed=seed, q_mult=q_mult)
    o, lse = run_gpu(q, k, v, scale, causal)
    assert np.isfinite(o).all() and np.isfinite(lse).all()
    if rows is None:
        o_ref, lse_ref = oracle.attention_rows(q, k, v, scale, causal)
        o_gpu = o.reshape(B * H, N, d)
        l_gpu = lse.reshape(B * H, N)
    else:
        idx = sample_rows(B, H, N, rows).numpy()
        o_ref, lse_ref = oracle.attention_rows(q, k, v, scale, causal, rows=idx)
        o_gpu = np.take_along_axis(o.reshape(B * H, N, d), idx[..., None], 1)
        l_gpu = np.take_along_axis(lse.reshape(B * H, N), idx, 1)
    err_o = np.abs(o_gpu - o_ref).max()
    err_l = np.abs(l_gpu - lse_ref).max()
    assert err_o <= TOL_O and err_l <= TOL_LSE, (err_o, err_l)
    return err_o, err_l


# ---- tiny exact attention: full comparison
def test_tiny_config_full():
    check(1, 2, 128, 64, False)


# ---- the 12-argument entry point itself, attn_fwd(q, k, v, o, lse, B, H, N, d,
# scale, causal, stream), on contiguous device buffers, against the oracle
@pytest.mark.parametrize("B,H,N,d", [(1, 2, 128, 64), (1, 16, 1944, 64), (2, 3, 700, 128)])
@pytest.mark.parametrize("causal", [False, True])
def test_attn_fwd_entry_point_full(B, H, N, d, causal):
    dev = torch.device("cuda:0")
    q, k, v = make_qkv(B, H, N, d, seed=N + d)
    qd, kd, vd = (x.to(dev).contiguous() for x in (q, k, v))
    o = torch.full((B, H, N, d), 7.0, dtype=torch.bfloat16, device=dev)
    lse = torch.full((B, H, N), 7.0, dtype=torch.float32, device=dev)
    scale = 1.0 / math.sqrt(d)
    st = pkg.attn_fwd(qd.data_ptr(), kd.data_ptr(), vd.data_ptr(), o.data_ptr(), lse.data_ptr(), B, H, N, d, scale,
                      causal, torch.cuda.current_stream().cuda_stream)
    assert st == pkg.ATTN_OK
    assert pkg.attn_check_device_status() == pkg.ATTN_OK
    o_ref, lse_ref = oracle.attention_rows(q, k, v, scale, causal)
    assert np.abs(o.float().cpu().numpy().reshape(o_ref.shape) - o_ref).max() <= TOL_O
    assert np.abs(lse.cpu().numpy().reshape(lse_ref.shape) - lse_ref).max() <= TOL_LSE


# ---- several tiles plus ragged tails, both head sizes, both masks: full comparison
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N", [1, 2, 17, 127, 128, 129, 255, 256, 257, 300, 511, 700])
def test_small_sizes_full(N, d, causal):
    check(1, 2, N, d, causal, seed=N)


@pytest.mark.parametrize("d", [64, 128])
def test_many_heads_and_batches_full(d):
    check(3, 5, 333, d, False, seed=11)
    check(3, 5, 333, d, True, seed=12)


# ---- patch self-attention 0.5 MP and its stability variant (logit std ~4)
@pytest.mark.parametrize("q_mult", [1.0, 4.0])
def test_half_megapixel_full(q_mult):
    check(1, 16, 1944, 64, False, q_mult=q_mult)


# ---- the image-size sweep and the 8 MP case: sampled rows
@pytest.mark.parametrize("N", [3952, 7776, 11616])
def test_image_sweep_sampled(N):
    check(1, 16, N, 64, False, rows=256)


def test_eight_megapixel_sampled():
    check(1, 16, 38400, 64, False, rows=256)


# ---- causal decoder-style configurations
def test_causal_decoder_full():
    check(8, 12, 1024, 64, True)


def test_causal_long_d128_sampled():
    check(1, 16, 16384, 128, True, rows=256)


# ---- degenerate cases with closed forms
def test_zero_query_gives_mean_and_log_n():
    dev = torch.device("cuda:0")
    B, H, N, d = 1, 2, 300, 64
    _, k, v = make_qkv(B, H, N, d, seed=4)
    q = torch.zeros_like(k)
    for causal in (False, True):
        o, lse = pkg.forward(q.to(dev), k.to(dev), v.to(dev), causal=causal)
        vd = v.double().numpy()
        if causal:
            cnt = np.arange(1, N + 1)
            mean = np.cumsum(vd, 2) / cnt[None, None, :, None]
            lse_cf = np.broadcast_to(np.log(cnt), (B, H, N))
        else:
            mean = np.broadcast_to(vd.mean(2, keepdims=True), vd.shape)
            lse_cf = np.full((B, H, N), math.log(N))
        assert np.abs(o.float().cpu().numpy() - mean).max() <= TOL_O
        assert np.abs(lse.cpu().numpy() - lse_cf).max() <= TOL_LSE


def test_constant_values_reproduced():
    dev = torch.device("cuda:0")
    q, k, _ = make_qkv(1, 2, 515, 128, seed=8)
    c = torch.randn(128, generator=torch.Generator().manual_seed(3)).to(torch.bfloat16)
    v = c.expand(1, 2, 515, 128).contiguous()
    o, _ = pkg.forward(q.to(dev), k.to(dev), v.to(dev), causal=False)
    assert np.abs(o.float().cpu().numpy() - c.float().numpy()).max() <= TOL_O


def test_deterministic_and_stream_ordered():
    dev = torch.device("cuda:0")
    q, k, v = (x.to(dev) for x in make_qkv(1, 4, 1000, 64, seed=9))
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        o1, l1 = pkg.forward(q, k, v)
        o2, l2 = pkg.forward(q, k, v)
    s.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


@pytest.mark.parametrize("d,causal", [(64, False), (128, True)])
def test_two_streams_at_once_match_one_stream(d, causal):
    # launches on two streams run at the same time (each kernel keeps its state
    # in its own shared memory and TMEM; no atomics on the outputs): every
    # result is bit-identical to the same call alone
    dev = torch.device("cuda:0")
    ins = [[x.to(dev) for x in make_qkv(1, 8, 2000, d, seed=s)] for s in (31, 32)]
    ref = [pkg.forward(*t, causal=causal) for t in ins]
    torch.cuda.synchronize()
    streams = [torch.cuda.Stream(), torch.cuda.Stream()]
    for s in streams:
        s.wait_stream(torch.cuda.current_stream())
    outs = []
    for _ in range(4):
        for i in (0, 1):
            with torch.cuda.stream(streams[i]):
                outs.append((i, pkg.forward(*ins[i], causal=causal)))
    torch.cuda.synchronize()
    assert pkg.attn_check_device_status() == pkg.ATTN_OK
    for i, (o, lse) in outs:
        assert torch.equal(o, ref[i][0]) and torch.equal(lse, ref[i][1])


def test_permuting_keys_and_values_leaves_output_unchanged():
    # a property that holds at any size: exact attention is invariant to a
    # joint permutation of the keys and values
    dev = torch.device("cuda:0")
    q, k, v = make_qkv(1, 4, 2000, 64, seed=10)
    perm = torch.randperm(2000, generator=torch.Generator().manual_seed(1))
    o1, l1 = pkg.forward(q.to(dev), k.to(dev), v.to(dev))
    o2, l2 = pkg.forward(q.to(dev), k[:, :, perm].contiguous().to(dev), v[:, :, perm].contiguous().to(dev))
    assert (o1.float() - o2.float()).abs().max().item() <= TOL_O
    assert (l1 - l2).abs().max().item() <= TOL_LSE


# ---- strided inputs and outputs: the patch self-attention module's layout
@pytest.mark.parametrize("d,causal", [(64, False), (64, True), (128, False), (128, True)])
def test_packed_projection_layout_matches_contiguous(d, causal):
    # Q, K, V as views of one packed projection output [B, N, 3, H, d] and O
    # written straight into a [B, N, H, d] buffer: no transpose copies.
    dev = torch.device("cuda:0")
    B, H, N = 2, 3, 333
    g = torch.Generator().manual_seed(21)
    packed = torch.randn(B, N, 3, H, d, generator=g).to(torch.bfloat16).to(dev)
    q, k, v = (packed[:, :, i].permute(0, 2, 1, 3) for i in range(3))
    assert not q.is_contiguous()
    o_buf = torch.full((B, N, H, d), 7.0, dtype=torch.bfloat16, device=dev)
    o_view = o_buf.permute(0, 2, 1, 3)
    o, lse = pkg.forward(q, k, v, causal=causal, out=o_view)
    assert o.data_ptr() == o_buf.data_ptr()
    o_ref, lse_ref = pkg.forward(q.contiguous(), k.contiguous(), v.contiguous(), causal=causal)
    assert pkg.attn_check_device_status() == pkg.ATTN_OK
    # the same kernel on the same values: identical results
    assert torch.equal(o, o_ref) and torch.equal(lse, lse_ref)
    # and against the oracle on the logical [B, H, N, d] tensors
    qc, kc, vc = (x.contiguous().cpu() for x in (q, k, v))
    oo, lo = oracle.attention_rows(qc, kc, vc, 1.0 / math.sqrt(d), causal)
    assert np.abs(o.float().cpu().numpy().reshape(oo.shape) - oo).max() <= TOL_O
    assert np.abs(lse.cpu().numpy().reshape(lo.shape) - lo).max() <= TOL_LSE


def test_strided_headline_layout_sampled():
    # the 3 MP workload in the module's packed layout, checked on sampled rows
    dev = torch.device("cuda:0")
    B, H, N, d = 1, 16, 11616, 64
    q0, k0, v0 = make_qkv(B, H, N, d, seed=0)
    packed = torch.stack([x.permute(0, 2, 1, 3) for x in (q0, k0, v0)], dim=2).to(dev)  # [B, N, 3, H, d]
    q, k, v = (packed[:, :, i].permute(0, 2, 1, 3) for i in range(3))
    o, lse = pkg.forward(q, k, v)
    assert pkg.attn_check_device_status() == pkg.ATTN_OK
    idx = sample_rows(B, H, N, 64).numpy()
    o_ref, lse_ref = oracle.attention_rows(q0, k0, v0, 1.0 / 8, False, rows=idx)
    o_gpu = np.take_along_axis(o.float().cpu().numpy().reshape(B * H, N, d), idx[..., None], 1)
    l_gpu = np.take_along_axis(lse.cpu().numpy().reshape(B * H, N), idx, 1)
    assert np.abs(o_gpu - o_ref).max() <= TOL_O and np.abs(l_gpu - lse_ref).max() <= TOL_LSE


# ---- key padding (the pages' mask pass): nonzero = padded key
def masked_check(B, H, N, d, causal, pad, seed=0):
    dev = torch.device("cuda:0")
    q, k, v = make_qkv(B, H, N, d, seed=seed)
    pad_t = torch.as_tensor(pad, dtype=torch.bool)
    o, lse = pkg.forward(q.to(dev), k.to(dev), v.to(dev), causal=causal, key_padding_mask=pad_t.to(dev))
    assert pkg.attn_check_device_status() == pkg.ATTN_OK
    o_ref, lse_ref = oracle.attention_rows(q, k, v, 1.0 / math.sqrt(d), causal, key_pad=pad.astype(np.uint8))
    o = o.float().cpu().numpy().reshape(o_ref.shape)
    lse = lse.cpu().numpy().reshape(lse_ref.shape)
    assert np.abs(o - o_ref).max() <= TOL_O
    empty = np.isneginf(lse_ref)
    assert (np.isneginf(lse) == empty).all()
    assert np.abs(lse[~empty] - lse_ref[~empty]).max() <= TOL_LSE if (~empty).any() else True
    assert (o.reshape(-1, d)[empty.reshape(-1)] == 0).all()


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N", [300, 512, 1000])   # 512: the 16-byte mask path; 300, 1000: bytewise
def test_key_padding_trailing_and_scattered(N, d, causal):
    B = 3
    rng = np.random.default_rng(N + d)
    pad = np.zeros((B, N), dtype=bool)
    pad[0, N - 37:] = True                            # trailing padding
    pad[1] = rng.random(N) < 0.3                      # scattered padding
    pad[1, 0] = False
    pad[2, : N // 2] = True                           # leading padding: causal rows < N/2 see nothing
    masked_check(B, 2, N, d, causal, pad, seed=N)


def test_key_padding_fully_padded_batch_and_no_padding():
    dev = torch.device("cuda:0")
    B, H, N, d = 2, 2, 640, 64
    pad = np.zeros((B, N), dtype=bool)
    pad[1] = True
    masked_check(B, H, N, d, False, pad, seed=3)
    # an all-False mask is the same computation as no mask
    q, k, v = (x.to(dev) for x in make_qkv(B, H, N, d, seed=4))
    none = torch.zeros(B, N, dtype=torch.bool, device=dev)
    o1, l1 = pkg.forward(q, k, v, key_padding_mask=none)
    o2, l2 = pkg.forward(q, k, v)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


@pytest.mark.parametrize("causal", [False, True])
def test_key_padding_skips_padded_tiles_full(causal):
    # the 0.5 MP shape with two batches, the second one's last 1024 patches
    # padded: 8 of its 16 key tiles hold only padded keys and are skipped
    # (never loaded or multiplied); the partly padded tile is masked per key.
    # Full element-wise comparison with the oracle.
    B, H, N, d = 2, 16, 1944, 64
    pad = np.zeros((B, N), dtype=bool)
    pad[1, N - 1024:] = True
    masked_check(B, H, N, d, causal, pad, seed=5)


def test_key_padding_skipped_tiles_in_the_middle_full():
    # whole padded key tiles between visible ones, at both head sizes, and a
    # batch whose only visible keys sit in its last (ragged) tile
    for d in (64, 128):
        B, H, N = 3, 2, 1000
        pad = np.zeros((B, N), dtype=bool)
        pad[0, 128:512] = True            # key tiles 1-3 skipped
        pad[1, :896] = True               # only the ragged last tile is visible
        pad[2, 256:384] = True
        pad[2, 640:] = True               # tiles 2, 5, 6, 7 skipped
        for causal in (False, True):
            masked_check(B, H, N, d, causal, pad, seed=d + int(causal))


def test_key_padding_image_workload_sampled():
    # 0.5 MP patch self-attention with its last 200 patches padded
    dev = torch.device("cuda:0")
    B, H, N, d = 2, 16, 1944, 64
    q, k, v = make_qkv(B, H, N, d, seed=0)
    pad = np.zeros((B, N), dtype=bool)
    pad[1, N - 200:] = True
    pad_t = torch.as_tensor(pad).to(dev)
    o, lse = pkg.forward(q.to(dev), k.to(dev), v.to(dev), key_padding_mask=pad_t)
    idx = sample_rows(B, H, N, 128).numpy()
    o_ref, lse_ref = oracle.attention_rows(q, k, v, 1.0 / 8, False, rows=idx, key_pad=pad.astype(np.uint8))
    o_gpu = np.take_along_axis(o.float().cpu().numpy().reshape(B * H, N, d), idx[..., None], 1)
    l_gpu = np.take_along_axis(lse.cpu().numpy().reshape(B * H, N), idx, 1)
    assert np.abs(o_gpu - o_ref).max() <= TOL_O and np.abs(l_gpu - lse_ref).max() <= TOL_LSE


# ---- block-sparse mask (FlashAttention wiki notes, "Block-sparse
# FlashAttention"): [T, T] over 128-row query blocks x 128-key blocks
def sparse_check(B, H, N, d, causal, bm, pad=None, seed=0, rows=None):
    dev = torch.device("cuda:0")
    q, k, v = make_qkv(B, H, N, d, seed=seed)
    bm_t = torch.as_tensor(bm, dtype=torch.bool).to(dev)
    pad_t = None if pad is None else torch.as_tensor(pad, dtype=torch.bool).to(dev)
    o, lse = pkg.forward(q.to(dev), k.to(dev), v.to(dev), causal=causal, key_padding_mask=pad_t, block_mask=bm_t)
    assert pkg.attn_check_device_status() == pkg.ATTN_OK
    kp = None if pad is None else pad.astype(np.uint8)
    o = o.float().cpu().numpy().reshape(B * H, N, d)
    lse = lse.cpu().numpy().reshape(B * H, N)
    if rows is None:
        o_ref, lse_ref = oracle.attention_rows(q, k, v, 1.0 / math.sqrt(d), causal, key_pad=kp,
                                               block_mask=bm.astype(np.uint8))
    else:
        idx = sample_rows(B, H, N, rows).numpy()
        o_ref, lse_ref = oracle.attention_rows(q, k, v, 1.0 / math.sqrt(d), causal, rows=idx, key_pad=kp,
                                               block_mask=bm.astype(np.uint8))
        o = np.take_along_axis(o, idx[..., None], 1)
        lse = np.take_along_axis(lse, idx, 1)
    assert np.abs(o - o_ref).max() <= TOL_O
    empty = np.isneginf(lse_ref)
    assert (np.isneginf(lse) == empty).all()
    if (~empty).any():
        assert np.abs(lse[~empty] - lse_ref[~empty]).max() <= TOL_LSE
    assert (o.reshape(-1, d)[empty.reshape(-1)] == 0).all()
    return empty.mean()


def random_block_mask(T, density, seed):
    rng = np.random.default_rng(seed)
    bm = rng.random((T, T)) < density
    if T >= 4:
        bm[1, :] = False          # a query block with no key block at all
        bm[2, :] = False
        bm[2, T - 1] = True       # only the last (ragged) key block
    return bm


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N", [129, 300, 700, 1000])
def test_block_sparse_random_full(N, d, causal):
    T = (N + 127) // 128
    sparse_check(2, 3, N, d, causal, random_block_mask(T, 0.5, N + d), seed=N)


@pytest.mark.parametrize("d", [64, 128])
def test_block_sparse_with_key_padding_full(d):
    N, B = 777, 2
    T = (N + 127) // 128
    rng = np.random.default_rng(d)
    pad = rng.random((B, N)) < 0.25
    pad[1, 256:512] = True            # a whole key block padded for batch 1
    for causal in (False, True):
        sparse_check(B, 2, N, d, causal, random_block_mask(T, 0.6, d + 1), pad=pad, seed=d)


@pytest.mark.parametrize("d", [64, 128])
def test_block_sparse_empty_units_between_busy_ones(d):
    # 256 work units (more than one per CTA): whole pairs of query blocks
    # without any key block sit between busy ones, and pairs whose two query
    # blocks use disjoint key blocks
    N = 1000
    bm = np.zeros((8, 8), dtype=bool)
    bm[0, [0, 3]] = True
    bm[1, [1, 6, 7]] = True           # pair 0: disjoint key blocks
    bm[4, :] = True                   # pair 2: only its first query block; pair 1 empty
    bm[7, 2] = True                   # pair 3: only its second query block
    sparse_check(2, 32, N, d, False, bm, seed=5)
    sparse_check(2, 32, N, d, True, bm, seed=6)


@pytest.mark.parametrize("d", [64, 128])
def test_all_ones_and_lower_triangle_block_masks_match_the_dense_kernel(d):
    dev = torch.device("cuda:0")
    B, H, N = 2, 3, 900
    T = (N + 127) // 128
    q, k, v = (x.to(dev) for x in make_qkv(B, H, N, d, seed=21))
    ones = torch.ones(T, T, dtype=torch.bool, device=dev)
    tri = torch.tril(ones)
    for causal, bm in ((False, ones), (True, ones), (True, tri)):
        o1, l1 = pkg.forward(q, k, v, causal=causal, block_mask=bm)
        o2, l2 = pkg.forward(q, k, v, causal=causal)
        assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_block_sparse_local_global_pattern_image_workload_sampled():
    # the 3 MP patch self-attention shape with a local band (3 key blocks on
    # each side) plus one global key block: about 8% of the blocks
    N = 11616
    T = (N + 127) // 128
    bm = np.zeros((T, T), dtype=bool)
    for r in range(T):
        bm[r, max(0, r - 3):r + 4] = True
    bm[:, 0] = True
    sparse_check(1, 16, N, 64, False, bm, rows=256)


def test_block_sparse_largest_mask_d128_sampled():
    # T = 512 (N = 65536): the largest mask, at the head size with the least
    # shared memory to spare
    N = 65536
    bm = random_block_mask(512, 0.05, 9)
    np.fill_diagonal(bm, True)
    sparse_check(1, 2, N, 128, True, bm, rows=64)


# ---- host-memory entry point: chunked transfers overlapping the kernel
@pytest.mark.parametrize("chunks", [1, 3, 8])
def test_forward_host_equals_device_forward(chunks):
    dev = torch.device("cuda:0")
    for (B, H, N, d, causal) in ((2, 3, 500, 64, True), (1, 16, 1944, 64, False), (1, 4, 700, 128, True)):
        q, k, v = make_qkv(B, H, N, d, seed=N + chunks)
        qh, kh, vh = (x.pin_memory() for x in (q, k, v))
        oh, lh = pkg.forward_host(qh, kh, vh, causal=causal, chunks=chunks)
        torch.cuda.synchronize()
        o, lse = pkg.forward(q.to(dev), k.to(dev), v.to(dev), causal=causal)
        assert pkg.attn_check_device_status() == pkg.ATTN_OK
        assert torch.equal(oh, o.cpu()) and torch.equal(lh, lse.cpu())


# ---- everything at once: packed-projection strides, key padding and a block mask
@pytest.mark.parametrize("d,causal", [(64, False), (64, True), (128, False), (128, True)])
def test_strided_padded_block_sparse_together(d, causal):
    dev = torch.device("cuda:0")
    B, H, N = 2, 3, 600
    T = (N + 127) // 128
    g = torch.Generator().manual_seed(31 + d)
    packed = torch.randn(B, N, 3, H, d, generator=g).to(torch.bfloat16).to(dev)
    q, k, v = (packed[:, :, i].permute(0, 2, 1, 3) for i in range(3))
    rng = np.random.default_rng(d + int(causal))
    pad = rng.random((B, N)) < 0.2
    pad[1, N - 100:] = True
    bm = random_block_mask(T, 0.6, 77 + d)
    o_buf = torch.zeros((B, N, H, d), dtype=torch.bfloat16, device=dev)
    o, lse = pkg.forward(q, k, v, causal=causal, out=o_buf.permute(0, 2, 1, 3),
                         key_padding_mask=torch.as_tensor(pad).to(dev), block_mask=torch.as_tensor(bm).to(dev))
    assert pkg.attn_check_device_status() == pkg.ATTN_OK
    qc, kc, vc = (x.contiguous().cpu() for x in (q, k, v))
    o_ref, lse_ref = oracle.attention_rows(qc, kc, vc, 1.0 / math.sqrt(d), causal, key_pad=pad.astype(np.uint8),
                                           block_mask=bm.astype(np.uint8))
    o_n = o.float().cpu().numpy().reshape(o_ref.shape)
    lse_n = lse.cpu().numpy().reshape(lse_ref.shape)
    assert np.abs(o_n - o_ref).max() <= TOL_O
    empty = np.isneginf(lse_ref)
    assert (np.isneginf(lse_n) == empty).all()
    assert np.abs(lse_n[~empty] - lse_ref[~empty]).max() <= TOL_LSE


def test_many_small_heads_full():
    # 1024 (batch, head) pairs of 200 rows: 1024 work units over 148 CTAs
    check(64, 16, 200, 64, False, seed=41)
    check(64, 16, 200, 64, True, seed=42)
