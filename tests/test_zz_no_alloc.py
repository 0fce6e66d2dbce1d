"""attn_bwd_noalloc: the backward with its delta workspace in the library's
static device array, so the call allocates nothing.

Collected last (file name) and independent of the order: every test resolves
what it needs itself.  The first call on a device looks up the array's
address; the capture test makes that call before capturing.
"""
import math

import numpy as np
import pytest
import torch

import exact_io_aware_102_b200 as pkg
import oracle
from exact_io_aware_102_b200.inputs import make_dout, make_qkv

CAPACITY = 1 << 20  # B * H * N rows of delta in the static array
GIB = 1 << 30


def test_noalloc_rejects_oversize_on_host():
    dense = [GIB * (i + 1) for i in range(9)]  # q k v o dout lse dq dk dv
    # B*H*N = 2^20 + 64 rows: larger than the static array
    assert pkg.attn_bwd_noalloc(*dense, 1, 1, CAPACITY + 64, 64, 0.125, 0, None) == pkg.ATTN_ERR_INVALID_ARG
    assert pkg.attn_bwd_noalloc(*dense, 0, 1, 128, 64, 0.125, 0, None) == pkg.ATTN_ERR_INVALID_ARG
    assert pkg.attn_bwd_noalloc(*dense, 1, 1, 128, 96, 0.125, 0, None) == pkg.ATTN_ERR_UNSUPPORTED


def _buffers(B, H, N, d, seed, causal):
    dev = torch.device("cuda:0")
    q, k, v = make_qkv(B, H, N, d, seed=seed)
    do = make_dout(B, H, N, d, seed=seed + 1)
    qd, kd, vd, dod = (x.to(dev) for x in (q, k, v, do))
    o, lse = pkg.forward(qd, kd, vd, causal=causal)
    dq = torch.empty((B, H, N, d), dtype=torch.float32, device=dev)
    dk, dv = torch.empty_like(qd), torch.empty_like(qd)
    return (q, k, v, do), (qd, kd, vd, o, dod, lse), (dq, dk, dv)


def _call(ins, outs, causal, stream=None):
    qd, kd, vd, o, dod, lse = ins
    dq, dk, dv = outs
    B, H, N, d = qd.shape
    handle = torch.cuda.current_stream().cuda_stream if stream is None else stream
    return pkg.attn_bwd_noalloc(qd.data_ptr(), kd.data_ptr(), vd.data_ptr(), o.data_ptr(), dod.data_ptr(),
                                lse.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), B, H, N, d,
                                1.0 / math.sqrt(d), causal, handle)


@pytest.mark.gpu
@pytest.mark.parametrize("causal", [False, True])
def test_noalloc_matches_oracle_and_attn_bwd(causal):
    B, H, N, d = 1, 2, 300, 64
    cpu, ins, outs = _buffers(B, H, N, d, 11, causal)
    assert _call(ins, outs, causal) == pkg.ATTN_OK
    assert pkg.attn_check_device_status() == pkg.ATTN_OK
    dq, dk, dv = (x.float().cpu().numpy() for x in outs)
    refs = oracle.attention_bwd_rows(*cpu, 1.0 / 8, causal)
    for g, r in zip((dq, dk, dv), refs):
        r = r.reshape(g.shape)
        assert np.abs(g - r).max() <= 2e-2 * np.abs(r).max()
    # the same kernels as attn_bwd with a caller workspace: dK, dV bit-equal
    qd, kd, vd, o, dod, lse = ins
    dq2, dk2, dv2 = pkg.backward(qd, kd, vd, o, lse, dod, causal=causal)
    assert torch.equal(dk2, outs[1]) and torch.equal(dv2, outs[2])
    np.testing.assert_allclose(dq2.cpu().numpy(), dq, rtol=0, atol=1e-5 * np.abs(dq).max())


@pytest.mark.gpu
def test_noalloc_allocates_nothing():
    B, H, N, d = 2, 4, 640, 64
    _, ins, outs = _buffers(B, H, N, d, 21, False)
    assert _call(ins, outs, False) == pkg.ATTN_OK  # resolves the array address
    torch.cuda.synchronize()
    base = torch.cuda.memory_allocated()
    torch.cuda.reset_peak_memory_stats()
    free0 = torch.cuda.mem_get_info()[0]
    for _ in range(3):
        assert _call(ins, outs, False) == pkg.ATTN_OK
    torch.cuda.synchronize()
    assert torch.cuda.max_memory_allocated() == base
    assert torch.cuda.mem_get_info()[0] == free0
    assert pkg.attn_check_device_status() == pkg.ATTN_OK


@pytest.mark.gpu
def test_noalloc_largest_size_matches_attn_bwd():
    # B*H*N = 2^20 exactly: the whole static array
    B, H, N, d = 64, 16, 1024, 64
    _, ins, outs = _buffers(B, H, N, d, 31, True)
    assert _call(ins, outs, True) == pkg.ATTN_OK
    qd, kd, vd, o, dod, lse = ins
    dq2, dk2, dv2 = pkg.backward(qd, kd, vd, o, lse, dod, causal=True)
    assert pkg.attn_check_device_status() == pkg.ATTN_OK
    assert torch.equal(dk2, outs[1]) and torch.equal(dv2, outs[2])
    assert torch.allclose(dq2, outs[0], rtol=0, atol=1e-5 * float(dq2.abs().max()))


@pytest.mark.gpu
def test_noalloc_inside_a_captured_graph():
    B, H, N, d = 1, 4, 512, 64
    _, ins, outs = _buffers(B, H, N, d, 41, False)
    assert _call(ins, outs, False) == pkg.ATTN_OK  # first call outside capture
    torch.cuda.synchronize()
    ref = [x.clone() for x in outs]
    for x in outs:
        x.zero_()
    stream = torch.cuda.Stream()
    graph = torch.cuda.CUDAGraph()
    stream.wait_stream(torch.cuda.current_stream())
    with torch.cuda.graph(graph, stream=stream):
        status = _call(ins, outs, False, stream=stream.cuda_stream)
    assert status == pkg.ATTN_OK
    graph.replay()
    torch.cuda.synchronize()
    assert pkg.attn_check_device_status() == pkg.ATTN_OK
    assert torch.equal(outs[1], ref[1]) and torch.equal(outs[2], ref[2])
    assert torch.allclose(outs[0], ref[0], rtol=0, atol=1e-5 * float(ref[0].abs().max()))
