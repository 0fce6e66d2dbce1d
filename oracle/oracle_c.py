"""ctypes loader and builder for the C oracle (test infrastructure only)."""
import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "attn_oracle.c")
_SRC_BWD = os.path.join(_HERE, "attn_bwd_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None


def library_path():
    return _LIB


def build(force=False):
    """Compile attn_oracle.c and attn_bwd_oracle.c with gcc -O2 -fopenmp into liboracle.so (in place)."""
    newest = max(os.path.getmtime(_SRC), os.path.getmtime(_SRC_BWD))
    if not force and os.path.exists(_LIB) and os.path.getmtime(_LIB) >= newest:
        return _LIB
    tmp = _LIB + ".tmp%d" % os.getpid()
    subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c99",
                           "-o", tmp, _SRC, _SRC_BWD, "-lm"])
    os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        ptr = ctypes.c_void_p
        for name in ("attn_oracle_f64", "attn_oracle_bf16"):
            fn = getattr(lib, name)
            fn.restype = ctypes.c_int
            fn.argtypes = [ptr, ptr, ptr, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                           ctypes.c_double, ctypes.c_int, ptr, ptr, ctypes.c_int, ctypes.c_int, ptr,
                           ctypes.c_int, ptr, ptr, ctypes.c_int]
        for name in ("attn_oracle_bwd_f64", "attn_oracle_bwd_bf16"):
            fn = getattr(lib, name)
            fn.restype = ctypes.c_int
            fn.argtypes = [ptr, ptr, ptr, ptr, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                           ctypes.c_double, ctypes.c_int, ptr, ptr, ctypes.c_int, ctypes.c_int, ptr, ctypes.c_int,
                           ptr, ctypes.c_int, ptr, ptr, ptr, ctypes.c_int]
        lib.attn_oracle_max_threads.restype = ctypes.c_int
        lib.attn_oracle_max_threads.argtypes = []
        _lib = lib
    return _lib


def max_threads():
    return _load().attn_oracle_max_threads()


def _bf16_bits(t):
    """Raw uint16 patterns of a bf16 torch tensor (CPU, contiguous)."""
    import torch
    assert t.dtype == torch.bfloat16
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def attention_rows(q, k, v, scale, causal=False, rows=None, n_threads=0, key_pad=None, block_mask=None,
                   block=(128, 128)):
    """Evaluate the oracle on selected query rows.

    q, k, v: [B, H, N, d], either bf16 torch tensors (widened exactly) or
    float64 arrays.  rows: None (all rows) or an int array [B*H, R] (or [R],
    shared by every head) of query indices.  key_pad: None or a [B, N] array,
    nonzero = padded key.  block_mask: None or a [ceil(N / Br), ceil(N / Bc)]
    array, (Br, Bc) = block, nonzero = that (query block, key block) pair is
    computed.  Returns (O [B*H, R, d], LSE [B*H, R]) as float64 numpy arrays;
    a row with no visible key has O = 0 and LSE = -inf.
    """
    lib = _load()
    try:
        import torch
        is_bf16 = isinstance(q, torch.Tensor) and q.dtype == torch.bfloat16
    except ImportError:  # pragma: no cover
        is_bf16 = False
    B, H, N, d = (int(x) for x in q.shape)
    if is_bf16:
        qa, ka, va = _bf16_bits(q), _bf16_bits(k), _bf16_bits(v)
        fn = lib.attn_oracle_bf16
    else:
        qa, ka, va = (np.ascontiguousarray(np.asarray(x, dtype=np.float64)) for x in (q, k, v))
        fn = lib.attn_oracle_f64
    if rows is None:
        n_rows, rows_a, rows_p = N, None, None
    else:
        rows_a = np.asarray(rows, dtype=np.int32)
        if rows_a.ndim == 1:
            rows_a = np.broadcast_to(rows_a, (B * H, rows_a.shape[0]))
        rows_a = np.ascontiguousarray(rows_a.reshape(B * H, -1))
        n_rows = rows_a.shape[1]
        rows_p = rows_a.ctypes.data
    pad_p = None
    if key_pad is not None:
        pad_a = np.ascontiguousarray(np.asarray(key_pad).astype(np.uint8).reshape(B, N))
        pad_p = pad_a.ctypes.data
    bm_p = None
    br, bc = (int(x) for x in block)
    if block_mask is not None:
        if br < 1 or bc < 1:
            raise ValueError("block sizes must be >= 1")
        tr, tc = (N + br - 1) // br, (N + bc - 1) // bc
        bm_a = np.ascontiguousarray(np.asarray(block_mask).astype(np.uint8).reshape(tr, tc))
        bm_p = bm_a.ctypes.data
    o = np.empty((B * H, n_rows, d), dtype=np.float64)
    lse = np.empty((B * H, n_rows), dtype=np.float64)
    rc = fn(qa.ctypes.data, ka.ctypes.data, va.ctypes.data, B, H, N, d, float(scale),
            int(bool(causal)), pad_p, bm_p, br, bc, rows_p, n_rows, o.ctypes.data, lse.ctypes.data,
            int(n_threads))
    if rc != 0:
        raise ValueError("oracle rejected its arguments (code %d)" % rc)
    return o, lse


def _select(rows, B, H, N):
    if rows is None:
        return N, None, None
    a = np.asarray(rows, dtype=np.int32)
    if a.ndim == 1:
        a = np.broadcast_to(a, (B * H, a.shape[0]))
    a = np.ascontiguousarray(a.reshape(B * H, -1))
    return a.shape[1], a, a.ctypes.data


def attention_bwd_rows(q, k, v, do, scale, causal=False, q_rows=None, k_rows=None, n_threads=0, key_pad=None,
                       block_mask=None, block=(128, 128)):
    """Exact gradients of O = softmax(scale Q K^T) V for the upstream gradient dO.

    q, k, v, do: [B, H, N, d], bf16 torch tensors (widened exactly) or float64
    arrays.  q_rows / k_rows: None (all rows) or int arrays [B*H, R] (or [R],
    shared by every head) of distinct rows: dQ is evaluated at q_rows, dK and
    dV at k_rows.  key_pad: None or a [B, N] array, nonzero = padded key.
    block_mask: None or a [ceil(N / Br), ceil(N / Bc)] array, (Br, Bc) = block.
    Returns (dQ [B*H, Rq, d], dK [B*H, Rk, d], dV [B*H, Rk, d]) as float64
    numpy arrays.
    """
    lib = _load()
    try:
        import torch
        is_bf16 = isinstance(q, torch.Tensor) and q.dtype == torch.bfloat16
    except ImportError:  # pragma: no cover
        is_bf16 = False
    B, H, N, d = (int(x) for x in q.shape)
    if is_bf16:
        arrs = [_bf16_bits(x) for x in (q, k, v, do)]
        fn = lib.attn_oracle_bwd_bf16
    else:
        arrs = [np.ascontiguousarray(np.asarray(x, dtype=np.float64)) for x in (q, k, v, do)]
        fn = lib.attn_oracle_bwd_f64
    n_q, qa, qp = _select(q_rows, B, H, N)
    n_k, ka, kp = _select(k_rows, B, H, N)
    for sel in (qa, ka):
        if sel is not None and any(len(set(r.tolist())) != len(r) for r in sel):
            raise ValueError("selected rows must be distinct within a head")
    pad_p = None
    if key_pad is not None:
        pad_a = np.ascontiguousarray(np.asarray(key_pad).astype(np.uint8).reshape(B, N))
        pad_p = pad_a.ctypes.data
    bm_p = None
    br, bc = (int(x) for x in block)
    if block_mask is not None:
        if br < 1 or bc < 1:
            raise ValueError("block sizes must be >= 1")
        bm_a = np.ascontiguousarray(np.asarray(block_mask).astype(np.uint8).reshape((N + br - 1) // br,
                                                                                     (N + bc - 1) // bc))
        bm_p = bm_a.ctypes.data
    dq = np.empty((B * H, n_q, d), dtype=np.float64)
    dk = np.empty((B * H, n_k, d), dtype=np.float64)
    dv = np.empty((B * H, n_k, d), dtype=np.float64)
    rc = fn(*(a.ctypes.data for a in arrs), B, H, N, d, float(scale), int(bool(causal)), pad_p, bm_p, br, bc, qp,
            n_q, kp, n_k,
            dq.ctypes.data, dk.ctypes.data, dv.ctypes.data, int(n_threads))
    if rc != 0:
        raise ValueError("oracle rejected its arguments (code %d)" % rc)
    return dq, dk, dv
