"""The C ABI library: it loads, exports every declared entry point, and rejects
bad arguments on the host before touching a GPU (these run without one)."""
import ctypes
import os
import re

import pytest

import exact_io_aware_102_b200 as pkg

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    text = open(os.path.join(ROOT, "include", "attn.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?[A-Za-z_][\w\s\*]*?\b(attn_\w+)\s*\(", text, flags=re.M)))


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(pkg.LIB_PATH):
        from exact_io_aware_102_b200 import build
        build.build()
    return pkg.library()


def test_header_declares_the_boundary():
    names = declared_functions()
    assert {"attn_fwd", "attn_fwd_strided", "attn_fwd_block_sparse", "attn_bwd", "attn_status_string",
            "attn_check_device_status",
            "attn_selftest_wait_timeout", "attn_version"} <= set(names)


def test_library_exports_every_declared_symbol(lib):
    raw = ctypes.CDLL(pkg.LIB_PATH)
    for name in declared_functions():
        assert hasattr(raw, name), name


def test_status_strings(lib):
    assert pkg.attn_status_string(pkg.ATTN_OK) == "ok"
    for s in range(1, 5):
        assert pkg.attn_status_string(s) not in ("", "unknown status")
    assert pkg.attn_status_string(99) == "unknown status"
    assert pkg.attn_version() >= 100


FAKE = 0x10000  # an aligned address: never dereferenced, validation fails first


@pytest.mark.parametrize("B,H,N,d,scale,expect", [
    (1, 1, 128, 96, 0.125, pkg.ATTN_ERR_UNSUPPORTED),
    (1, 1, 128, 32, 0.125, pkg.ATTN_ERR_UNSUPPORTED),
    (0, 1, 128, 64, 0.125, pkg.ATTN_ERR_INVALID_ARG),
    (1, 0, 128, 64, 0.125, pkg.ATTN_ERR_INVALID_ARG),
    (1, 1, 0, 64, 0.125, pkg.ATTN_ERR_INVALID_ARG),
    (1, 1, -5, 64, 0.125, pkg.ATTN_ERR_INVALID_ARG),
    (1, 1, 128, 64, float("nan"), pkg.ATTN_ERR_INVALID_ARG),
    (1, 1, 128, 64, float("inf"), pkg.ATTN_ERR_INVALID_ARG),
    (1, 1, 128, 64, 0.0, pkg.ATTN_ERR_INVALID_ARG),
    (1, 1, 128, 64, -0.125, pkg.ATTN_ERR_INVALID_ARG),
    (65536, 65536, 128, 64, 0.125, pkg.ATTN_ERR_INVALID_ARG),
    (1, 1, 2**31 - 100, 64, 0.125, pkg.ATTN_ERR_INVALID_ARG),
])
def test_bad_sizes_rejected_on_host(lib, B, H, N, d, scale, expect):
    assert pkg.attn_fwd(FAKE, FAKE * 2, FAKE * 3, FAKE * 4, FAKE * 5, B, H, N, d, scale, 0, None) == expect


def test_null_and_misaligned_pointers_rejected(lib):
    ok = [FAKE, FAKE * 2, FAKE * 3, FAKE * 4, FAKE * 5]
    for i in range(5):
        ptrs = list(ok)
        ptrs[i] = None
        assert pkg.attn_fwd(*ptrs, 1, 1, 64, 64, 0.125, 0, None) == pkg.ATTN_ERR_INVALID_ARG
    for i in range(4):  # q, k, v, o need 16-byte alignment
        ptrs = list(ok)
        ptrs[i] += 8
        assert pkg.attn_fwd(*ptrs, 1, 1, 64, 64, 0.125, 0, None) == pkg.ATTN_ERR_INVALID_ARG
    ptrs = list(ok)
    ptrs[4] += 2  # lse needs 4-byte alignment
    assert pkg.attn_fwd(*ptrs, 1, 1, 64, 64, 0.125, 0, None) == pkg.ATTN_ERR_INVALID_ARG


def test_overlapping_outputs_rejected(lib):
    base = 1 << 20
    n_bytes = 1 * 2 * 64 * 64 * 2
    # o overlapping q
    assert pkg.attn_fwd(base, base + 2 * n_bytes, base + 4 * n_bytes, base + 16, base + 8 * n_bytes,
                        1, 2, 64, 64, 0.125, 0, None) == pkg.ATTN_ERR_INVALID_ARG
    # lse overlapping o
    assert pkg.attn_fwd(base, base + 2 * n_bytes, base + 4 * n_bytes, base + 6 * n_bytes,
                        base + 6 * n_bytes + 64, 1, 2, 64, 64, 0.125, 0, None) == pkg.ATTN_ERR_INVALID_ARG


@pytest.mark.parametrize("qkv,o", [
    ((8192, 64, 0), (8192, 64, 64)),       # zero row stride
    ((8192, 64, 60), (8192, 64, 64)),      # row stride below d
    ((8192, 64, 68), (8192, 64, 64)),      # not a multiple of 8 elements (16 bytes)
    ((8192, 4, 64), (8192, 64, 64)),       # head stride not a multiple of 8
    ((8192, 64, 64), (-8192, 64, 64)),     # negative stride
    ((8192, 64, 64), (8192, 64, 1 << 40)),  # beyond the tensor-map stride range
])
def test_bad_strides_rejected_on_host(lib, qkv, o):
    assert pkg.attn_fwd_strided(FAKE, FAKE * 2, FAKE * 3, FAKE * 4, FAKE * 5, 1, 2, 64, 64, qkv, o, 0.125, 0,
                                None) == pkg.ATTN_ERR_INVALID_ARG


@pytest.mark.parametrize("H,N,o", [
    (2, 64, (8192, 8, 64)),        # heads 8 elements apart: rows of head 0 and 1 share bytes
    (2, 64, (8192, 64, 64)),       # head stride = row stride: (h=1, n) is (h=0, n+1)
    (2, 64, (8192, 4096, 128)),    # head stride inside the span of one head's rows
    (3, 64, (65536, 64, 128)),     # interleaved heads, 3 heads in a 2-row stride
])
def test_aliasing_output_rows_rejected(lib, H, N, o):
    # two different (b, h, n) rows of O would overlap: rejected before any launch
    dense = (H * N * 64, N * 64, 64)
    assert pkg.attn_fwd_strided(GIB, 2 * GIB, 3 * GIB, 4 * GIB, 5 * GIB, 1, H, N, 64, dense, o, 0.125, 0,
                                None) == pkg.ATTN_ERR_INVALID_ARG


@pytest.mark.parametrize("H,N,o", [
    (2, 64, (8192, 4096, 64)),     # contiguous [B, H, N, d]
    (2, 64, (8192, 64, 128)),      # [B, N, H, d]: heads interleaved, rows nested
    (1, 64, (8192, 8, 64)),        # the stride of a size-1 dimension is never used
])
def test_nested_output_rows_accepted(lib, H, N, o):
    dense = (H * N * 64, N * 64, 64)
    # passes the host checks; with no GPU here it fails only at the driver
    assert pkg.attn_fwd_strided(GIB, 2 * GIB, 3 * GIB, 4 * GIB, 5 * GIB, 1, H, N, 64, dense, o, 0.125, 0,
                                None) not in (pkg.ATTN_ERR_INVALID_ARG, pkg.ATTN_OK)


def test_strided_overlap_uses_the_strided_span(lib):
    # O's span under its strides reaches into q's allocation range: rejected
    base = 1 << 24
    assert pkg.attn_fwd_strided(base, base + (1 << 22), base + (2 << 22), base - 4096, base + (3 << 22),
                                1, 2, 64, 64, (8192, 64, 128), (8192, 64, 128), 0.125, 0,
                                None) == pkg.ATTN_ERR_INVALID_ARG


GIB = 1 << 30  # spacing of fake buffers large enough for N = 65536


def _sparse(N, bm):
    dense = (2 * N * 64, N * 64, 64)
    return pkg.attn_fwd_block_sparse(GIB, 2 * GIB, 3 * GIB, 4 * GIB, 5 * GIB, 1, 2, N, 64, dense, dense, 0.125, 0,
                                     None, block_mask=bm)


def test_block_mask_checked_on_host(lib):
    # misaligned (the mask is read 16 bytes at a time)
    assert _sparse(1000, 6 * GIB + 8) == pkg.ATTN_ERR_INVALID_ARG
    # more than 512 x 512 blocks (N > 65536) does not fit the on-chip bit copy
    assert _sparse(65537, 6 * GIB) == pkg.ATTN_ERR_INVALID_ARG
    # the mask must not overlap O or LSE
    assert _sparse(1000, 4 * GIB + 64) == pkg.ATTN_ERR_INVALID_ARG
    assert _sparse(1000, 5 * GIB) == pkg.ATTN_ERR_INVALID_ARG
    # a well-formed call passes host validation (and, with no GPU here, fails
    # only when it reaches the CUDA driver)
    assert _sparse(65536, 6 * GIB) not in (pkg.ATTN_ERR_INVALID_ARG, pkg.ATTN_OK)
    # without a mask it is attn_fwd_strided
    assert _sparse(1000, None) not in (pkg.ATTN_ERR_INVALID_ARG, pkg.ATTN_OK)


def _bwd(ptrs, N=1000, d=64, scale=0.125, pad=None):
    return pkg.attn_bwd(*ptrs, 1, 2, N, d, scale, 0, None, key_padding_mask=pad)


def test_bwd_arguments_checked_on_host(lib):
    ok = [GIB * (i + 1) for i in range(10)]  # q k v o dout lse delta dq dk dv
    assert _bwd(ok) not in (pkg.ATTN_ERR_INVALID_ARG, pkg.ATTN_OK)  # reaches the driver
    assert _bwd(ok, d=96) == pkg.ATTN_ERR_UNSUPPORTED
    assert _bwd(ok, d=128) not in (pkg.ATTN_ERR_INVALID_ARG, pkg.ATTN_ERR_UNSUPPORTED, pkg.ATTN_OK)
    assert _bwd(ok, scale=0.0) == pkg.ATTN_ERR_INVALID_ARG
    for i in range(10):
        bad = list(ok)
        bad[i] = None
        assert _bwd(bad) == pkg.ATTN_ERR_INVALID_ARG
    bad = list(ok)
    bad[7] = ok[0] + 64           # dq overlapping q
    assert _bwd(bad) == pkg.ATTN_ERR_INVALID_ARG
    bad = list(ok)
    bad[9] = ok[8] + 128          # dv overlapping dk
    assert _bwd(bad) == pkg.ATTN_ERR_INVALID_ARG
    bad = list(ok)
    bad[8] += 8                   # dk misaligned
    assert _bwd(bad) == pkg.ATTN_ERR_INVALID_ARG
    assert _bwd(ok, pad=ok[7] + 16) == pkg.ATTN_ERR_INVALID_ARG   # mask overlapping dq
    assert _bwd(ok, pad=GIB * 11) not in (pkg.ATTN_ERR_INVALID_ARG, pkg.ATTN_OK)


def test_selftest_limit_validated(lib):
    assert pkg.attn_selftest_wait_timeout(10, 0) == pkg.ATTN_ERR_INVALID_ARG
    assert pkg.attn_selftest_wait_timeout(10**11, 0) == pkg.ATTN_ERR_INVALID_ARG


def test_forward_rejects_cpu_tensors(lib):
    import torch
    q = torch.zeros(1, 1, 8, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        pkg.forward(q, q, q)
    with pytest.raises(ValueError):
        pkg.forward(q.float(), q.float(), q.float())


def test_product_path_does_not_import_the_oracle():
    # The package and its sources never reference the oracle.
    pkg_dir = os.path.join(ROOT, "exact_io_aware_102_b200")
    for dirpath, _, files in os.walk(pkg_dir):
        for f in files:
            if f.endswith((".py", ".cu", ".h", ".cpp")):
                text = open(os.path.join(dirpath, f)).read()
                assert "import oracle" not in text and "from oracle" not in text, f
                assert "attn_oracle" not in text, f


def test_missing_library_fails_loudly():
    # no fallback: without libattn.so every entry point raises
    code = ("import exact_io_aware_102_b200 as p; p.LIB_PATH = '/nonexistent/libattn.so'\n"
            "try:\n    p.attn_version()\nexcept ImportError:\n    print('raised')\n")
    import subprocess
    import sys
    out = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, cwd=ROOT, timeout=120)
    assert out.stdout.strip() == "raised", out.stdout + out.stderr


def test_forward_host_and_backward_check_arguments_first(lib):
    import torch
    q = torch.zeros(1, 2, 8, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        pkg.forward_host(q, q, q[:, :1])                     # shapes differ
    with pytest.raises(ValueError):
        pkg.forward_host(q.float(), q.float(), q.float())    # not bf16
    with pytest.raises(ValueError):
        pkg.forward_host(q.transpose(2, 3), q.transpose(2, 3), q.transpose(2, 3))  # not contiguous
    lse = torch.zeros(1, 2, 8)
    with pytest.raises(ValueError):
        pkg.backward(q, q, q, q, lse, q)                     # host tensors are rejected
