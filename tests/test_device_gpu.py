"""Device-side behaviour that is not numerics: memory, argument checks with real
device pointers, and the bounded-wait failure path (no fault is provoked)."""
import numpy as np
import pytest
import torch

import exact_io_aware_102_b200 as pkg
from exact_io_aware_102_b200.inputs import make_qkv

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda:0")


def peak_extra_bytes(q, k, v, causal=False):
    """Peak device bytes one call asks the caching allocator for on top of
    what is already allocated, measured as the first page of the pages does it
    (a base, reset the peak, run, read the peak) on the allocator's
    requested-bytes counters.  Its allocated-bytes counters would also count
    the unsplit remainder of a cached block that an earlier test left behind
    (the allocator hands out a cached block whole when the rest would be
    small), which depends on the order of the tests, not on the call; the
    benchmark, in a fresh process, reports the allocated-bytes figure."""
    torch.cuda.synchronize()
    base = torch.cuda.memory_stats()["requested_bytes.all.current"]
    torch.cuda.reset_peak_memory_stats()
    o, lse = pkg.forward(q, k, v, causal=causal)
    torch.cuda.synchronize()
    extra = torch.cuda.memory_stats()["requested_bytes.all.peak"] - base
    del o, lse
    return extra


@pytest.mark.parametrize("N", [1944, 3952, 7776, 11616, 38400])
def test_peak_extra_memory_is_outputs_only(N):
    B, H, d = 1, 16, 64
    q, k, v = (x.to(DEV) for x in make_qkv(B, H, N, d, seed=0))
    pkg.forward(q, k, v)  # first call loads the module image
    torch.cuda.synchronize()
    torch.cuda.empty_cache()  # both device-wide readings without cached blocks
    free0, _ = torch.cuda.mem_get_info()
    extra = peak_extra_bytes(q, k, v)
    torch.cuda.empty_cache()
    free1, _ = torch.cuda.mem_get_info()
    out_bytes = B * H * N * d * 2 + B * H * N * 4
    assert extra <= 1.1 * out_bytes, (extra, out_bytes)
    # nothing allocated behind the caching allocator's back and kept (no N x N
    # anything): with the outputs freed, the device is back where it was
    assert abs(free0 - free1) < 2 * 1024 * 1024, (free0, free1)
    assert extra < B * H * N * N * 2 / 10  # far below one materialised score copy


def test_extra_memory_is_linear_in_n():
    ns = [1024, 2048, 3072, 4096]
    ex = []
    for n in ns:
        q, k, v = (x.to(DEV) for x in make_qkv(1, 16, n, 64, seed=0))
        ex.append(peak_extra_bytes(q, k, v))
    a, b, c = np.polyfit(np.array(ns, float), np.array(ex, float), 2)
    # quadratic coefficient ~0: a materialised table would give 16*2 = 32 bytes per N^2
    assert abs(a) < 1e-3, (a, b, c)


def test_host_pointers_rejected_and_outputs_untouched():
    q, k, v = (x.to(DEV) for x in make_qkv(1, 2, 64, 64, seed=1))
    o = torch.full_like(q, 7.0)
    lse = torch.full((1, 2, 64), 7.0, device=DEV)
    host = torch.zeros(1, 2, 64, 64, dtype=torch.bfloat16).pin_memory()
    st = pkg.attn_fwd(host.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                      1, 2, 64, 64, 0.125, 0, torch.cuda.current_stream().cuda_stream)
    assert st == pkg.ATTN_ERR_INVALID_ARG
    cpu = torch.zeros(1, 2, 64, 64, dtype=torch.bfloat16)
    st = pkg.attn_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), cpu.data_ptr(), lse.data_ptr(),
                      1, 2, 64, 64, 0.125, 0, torch.cuda.current_stream().cuda_stream)
    assert st == pkg.ATTN_ERR_INVALID_ARG
    torch.cuda.synchronize()
    assert (o.float() == 7.0).all() and (lse == 7.0).all()


def test_undersized_allocation_rejected():
    # q points 4 KB before the end of its allocation while the sizes describe
    # an 8 KB tensor: the host check against the driver's allocation range
    # refuses it, so nothing is launched.
    big = torch.empty(8 << 20, dtype=torch.uint8, device=DEV)
    seg = [s for s in torch.cuda.memory_snapshot()
           if s["address"] <= big.data_ptr() < s["address"] + s["total_size"]]
    assert len(seg) == 1
    end = seg[0]["address"] + seg[0]["total_size"]
    _, k, v = (x.to(DEV) for x in make_qkv(1, 1, 64, 64, seed=1))
    o = torch.empty_like(k)
    lse = torch.empty(1, 1, 64, device=DEV)
    st = pkg.attn_fwd(end - 4096, k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                      1, 1, 64, 64, 0.125, 0, torch.cuda.current_stream().cuda_stream)
    assert st == pkg.ATTN_ERR_INVALID_ARG
    st = pkg.attn_fwd(end - 8192, k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                      1, 1, 64, 64, 0.125, 0, torch.cuda.current_stream().cuda_stream)
    assert st == pkg.ATTN_OK  # exactly fits
    assert pkg.attn_check_device_status() == pkg.ATTN_OK


def test_bounded_wait_reports_timeout_and_context_survives():
    assert pkg.attn_check_device_status() == pkg.ATTN_OK
    assert pkg.attn_selftest_wait_timeout(2_000_000) == pkg.ATTN_OK  # 2 ms
    assert pkg.attn_check_device_status() == pkg.ATTN_ERR_TIMEOUT
    assert pkg.attn_check_device_status() == pkg.ATTN_OK  # cleared by the read
    q, k, v = (x.to(DEV) for x in make_qkv(1, 2, 200, 64, seed=2))
    o, lse = pkg.forward(q, k, v)
    assert pkg.attn_check_device_status() == pkg.ATTN_OK
    assert torch.isfinite(o.float()).all() and torch.isfinite(lse).all()
