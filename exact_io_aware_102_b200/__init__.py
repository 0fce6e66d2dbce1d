"""Exact, IO-aware attention forward for B200 -- Python binding.

Argument marshalling only: every step of the attention runs in the CUDA
library ``libattn.so`` (built from ``csrc/attn_fwd.cu`` for sm_100a); PyTorch
supplies device memory and the current stream.  There is no fallback: if the
library is missing, every entry point raises.

The C entry points keep their names here (``attn_fwd``, ``attn_fwd_strided``,
``attn_fwd_block_sparse``, ``attn_bwd``, ``attn_bwd_noalloc``, ``attn_status_string``, ``attn_check_device_status``,
``attn_selftest_wait_timeout``, ``attn_selftest_ex2``, ``attn_version``); ``forward`` is the tensor
convenience wrapper, ``forward_host`` the same on host tensors with the
transfers overlapped with the kernel, and ``backward`` the gradient
counterpart.
"""
import ctypes
import math
import os

__all__ = [
    "AttnError", "LIB_PATH", "library", "attn_fwd", "attn_fwd_strided", "attn_fwd_block_sparse", "attn_bwd", "attn_bwd_noalloc", "attn_status_string", "attn_check_device_status",
    "attn_selftest_wait_timeout", "attn_selftest_ex2", "attn_version", "forward", "forward_host", "backward", "ATTN_OK", "ATTN_ERR_INVALID_ARG",
    "ATTN_ERR_UNSUPPORTED", "ATTN_ERR_CUDA", "ATTN_ERR_TIMEOUT",
]

ATTN_OK, ATTN_ERR_INVALID_ARG, ATTN_ERR_UNSUPPORTED, ATTN_ERR_CUDA, ATTN_ERR_TIMEOUT = 0, 1, 2, 3, 4

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libattn.so")
_lib = None


class AttnError(RuntimeError):
    """A library call returned a status other than ATTN_OK."""

    def __init__(self, status, what):
        self.status = status
        super().__init__("%s: %s (status %d)" % (what, attn_status_string(status), status))


def library():
    """The loaded ``libattn.so`` (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError("libattn.so is not built (expected at %s); run "
                              "`python -c 'import __graft_entry__ as g; g.build()'`" % LIB_PATH)
        lib = ctypes.CDLL(LIB_PATH)
        vp, i32 = ctypes.c_void_p, ctypes.c_int
        lib.attn_fwd.restype = i32
        lib.attn_fwd.argtypes = [vp, vp, vp, vp, vp, i32, i32, i32, i32, ctypes.c_float, i32, vp]
        i64 = ctypes.c_longlong
        lib.attn_fwd_strided.restype = i32
        lib.attn_fwd_strided.argtypes = [vp, vp, vp, vp, vp, i32, i32, i32, i32, i64, i64, i64, i64, i64, i64,
                                         vp, ctypes.c_float, i32, vp]
        lib.attn_fwd_block_sparse.restype = i32
        lib.attn_fwd_block_sparse.argtypes = [vp, vp, vp, vp, vp, i32, i32, i32, i32, i64, i64, i64, i64, i64,
                                              i64, vp, vp, ctypes.c_float, i32, vp]
        lib.attn_bwd.restype = i32
        lib.attn_bwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, ctypes.c_float,
                                 i32, vp]
        lib.attn_bwd_noalloc.restype = i32
        lib.attn_bwd_noalloc.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, i32, i32, i32, i32,
                                         ctypes.c_float, i32, vp]
        lib.attn_status_string.restype = ctypes.c_char_p
        lib.attn_status_string.argtypes = [i32]
        lib.attn_check_device_status.restype = i32
        lib.attn_check_device_status.argtypes = [vp]
        lib.attn_selftest_wait_timeout.restype = i32
        lib.attn_selftest_wait_timeout.argtypes = [ctypes.c_ulonglong, vp]
        lib.attn_selftest_ex2.restype = i32
        lib.attn_selftest_ex2.argtypes = [vp, vp, i32, vp]
        lib.attn_version.restype = i32
        lib.attn_version.argtypes = []
        _lib = lib
    return _lib


def attn_fwd(q, k, v, o, lse, B, H, N, d, scale, causal, stream):
    """Raw C call: pointers are ints (device addresses), stream an int handle; returns the status."""
    return library().attn_fwd(q, k, v, o, lse, int(B), int(H), int(N), int(d), float(scale),
                              int(bool(causal)), stream)


def attn_fwd_strided(q, k, v, o, lse, B, H, N, d, qkv_strides, o_strides, scale, causal, stream,
                     key_padding_mask=None):
    """Raw C call with (batch, head, row) element strides for Q/K/V and for O,
    and an optional device address of a [B, N] byte key-padding mask."""
    sb, sh, sn = (int(x) for x in qkv_strides)
    ob, oh, on = (int(x) for x in o_strides)
    return library().attn_fwd_strided(q, k, v, o, lse, int(B), int(H), int(N), int(d), sb, sh, sn, ob, oh, on,
                                      key_padding_mask, float(scale), int(bool(causal)), stream)


def attn_fwd_block_sparse(q, k, v, o, lse, B, H, N, d, qkv_strides, o_strides, scale, causal, stream,
                          key_padding_mask=None, block_mask=None):
    """Raw C call: attn_fwd_strided plus the device address of a
    [ceil(N/128), ceil(N/128)] byte block mask (nonzero = block computed)."""
    sb, sh, sn = (int(x) for x in qkv_strides)
    ob, oh, on = (int(x) for x in o_strides)
    return library().attn_fwd_block_sparse(q, k, v, o, lse, int(B), int(H), int(N), int(d), sb, sh, sn, ob, oh,
                                           on, key_padding_mask, block_mask, float(scale), int(bool(causal)),
                                           stream)


def attn_bwd(q, k, v, o, dout, lse, delta, dq, dk, dv, B, H, N, d, scale, causal, stream, key_padding_mask=None,
             block_mask=None):
    """Raw C call: device addresses as ints; returns the status."""
    return library().attn_bwd(q, k, v, o, dout, lse, key_padding_mask, block_mask, delta, dq, dk, dv, int(B), int(H),
                              int(N), int(d), float(scale), int(bool(causal)), stream)


def attn_bwd_noalloc(q, k, v, o, dout, lse, dq, dk, dv, B, H, N, d, scale, causal, stream, key_padding_mask=None,
                     block_mask=None):
    """Raw C call: attn_bwd with delta in the library's static device array (no allocation)."""
    return library().attn_bwd_noalloc(q, k, v, o, dout, lse, key_padding_mask, block_mask, dq, dk, dv, int(B), int(H),
                                      int(N), int(d), float(scale), int(bool(causal)), stream)


def attn_status_string(status):
    return library().attn_status_string(int(status)).decode()


def attn_check_device_status(stream=None):
    """Synchronise ``stream`` and return (and clear) the device status word."""
    return library().attn_check_device_status(_stream_handle(stream))


def attn_selftest_wait_timeout(limit_ns, stream=None):
    return library().attn_selftest_wait_timeout(int(limit_ns), _stream_handle(stream))


def attn_selftest_ex2(x, y, n, stream=None):
    """Raw C call: y[i] = the softmax's FMA-pipe 2^x[i] (device addresses as ints)."""
    return library().attn_selftest_ex2(x, y, int(n), _stream_handle(stream))


def attn_version():
    return library().attn_version()


def _stream_handle(stream):
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


BLOCK = 128  # query rows / keys per block of the block-sparse mask


def forward(q, k, v, scale=None, causal=False, out=None, lse=None, stream=None, key_padding_mask=None,
            block_mask=None):
    """Exact attention forward on bf16 CUDA tensors [B, H, N, d] (d = 64 or 128).

    q, k and v may be strided views (for example of one packed projection
    output) as long as their head dimension is contiguous and they share one
    set of strides; ``out`` may be a strided view too (default: a new
    contiguous tensor).  Returns (o, lse): o bf16 [B, H, N, d] and lse fp32
    [B, H, N] (natural-log log-sum-exp of each row's scaled scores).
    ``scale`` defaults to 1/sqrt(d).  ``key_padding_mask``: None or a bool /
    uint8 CUDA tensor [B, N], True (nonzero) = padded key, excluded from every
    query row of that batch; a row with no visible key gets O = 0 and LSE =
    -inf.  ``block_mask``: None or a bool / uint8 CUDA tensor [T, T], T =
    ceil(N / 128), contiguous and 16-byte aligned: entry (r, c) nonzero lets
    query rows [128 r, 128 r + 128) see keys [128 c, 128 c + 128), for every
    batch and head; only those blocks are computed.  The call is asynchronous
    on ``stream`` (default: the current stream).
    """
    import torch
    if q.dim() != 4 or q.shape != k.shape or q.shape != v.shape:
        raise ValueError("q, k, v must share one shape [B, H, N, d]")
    for name, t in (("q", q), ("k", k), ("v", v)):
        if t.dtype != torch.bfloat16 or not t.is_cuda or t.stride(3) != 1:
            raise ValueError("%s must be a bf16 CUDA tensor with a contiguous last dimension" % name)
    if k.stride() != q.stride() or v.stride() != q.stride():
        raise ValueError("q, k, v must share one set of strides")
    B, H, N, d = (int(x) for x in q.shape)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty((B, H, N, d), dtype=torch.bfloat16, device=q.device)
    if lse is None:
        lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    if out.shape != q.shape or out.dtype != torch.bfloat16 or out.stride(3) != 1:
        raise ValueError("out must be a bf16 tensor shaped like q with a contiguous last dimension")
    if lse.shape != (B, H, N) or lse.dtype != torch.float32 or not lse.is_contiguous():
        raise ValueError("lse must be a contiguous fp32 tensor [B, H, N]")
    pad_ptr = None
    if key_padding_mask is not None:
        if (key_padding_mask.shape != (B, N) or key_padding_mask.dtype not in (torch.bool, torch.uint8)
                or not key_padding_mask.is_cuda or not key_padding_mask.is_contiguous()):
            raise ValueError("key_padding_mask must be a contiguous bool/uint8 CUDA tensor [B, N]")
        pad_ptr = key_padding_mask.data_ptr()
    bm_ptr = None
    if block_mask is not None:
        T = (N + BLOCK - 1) // BLOCK
        if (block_mask.shape != (T, T) or block_mask.dtype not in (torch.bool, torch.uint8)
                or not block_mask.is_cuda or not block_mask.is_contiguous()):
            raise ValueError("block_mask must be a contiguous bool/uint8 CUDA tensor [ceil(N/128), ceil(N/128)]")
        bm_ptr = block_mask.data_ptr()
    # the stride of a size-1 dimension is never used: give it the contiguous value
    def strides(t):
        dense = (H * N * d, N * d, d)
        return [st if n > 1 else c for n, st, c in zip(t.shape[:3], t.stride()[:3], dense)]
    if bm_ptr is None:
        status = attn_fwd_strided(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(),
                                  B, H, N, d, strides(q), strides(out), scale, causal, _stream_handle(stream),
                                  key_padding_mask=pad_ptr)
        what = "attn_fwd_strided"
    else:
        status = attn_fwd_block_sparse(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(),
                                       B, H, N, d, strides(q), strides(out), scale, causal,
                                       _stream_handle(stream), key_padding_mask=pad_ptr, block_mask=bm_ptr)
        what = "attn_fwd_block_sparse"
    if status != ATTN_OK:
        raise AttnError(status, what)
    return out, lse


def backward(q, k, v, o, lse, dout, scale=None, causal=False, stream=None, key_padding_mask=None, block_mask=None):
    """Gradients of ``forward`` for the upstream gradient ``dout``.

    q, k, v, o, dout: contiguous bf16 CUDA tensors [B, H, N, d], d = 64 or 128 (o and lse
    from ``forward`` on the same q, k, v, scale, causal and
    ``key_padding_mask``, a bool / uint8 CUDA tensor [B, N] or None, and
    ``block_mask``, as in ``forward``).  Returns
    (dq fp32, dk bf16, dv bf16), each [B, H, N, d].  Asynchronous on
    ``stream`` (default: the current stream).
    """
    import torch
    for name, t in (("q", q), ("k", k), ("v", v), ("o", o), ("dout", dout)):
        if t.dtype != torch.bfloat16 or not t.is_cuda or not t.is_contiguous() or t.shape != q.shape:
            raise ValueError("%s must be a contiguous bf16 CUDA tensor shaped like q" % name)
    if q.dim() != 4:
        raise ValueError("q must be [B, H, N, d]")
    B, H, N, d = (int(x) for x in q.shape)
    if lse.shape != (B, H, N) or lse.dtype != torch.float32 or not lse.is_contiguous():
        raise ValueError("lse must be a contiguous fp32 tensor [B, H, N]")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    pad_ptr = None
    if key_padding_mask is not None:
        if (key_padding_mask.shape != (B, N) or key_padding_mask.dtype not in (torch.bool, torch.uint8)
                or not key_padding_mask.is_cuda or not key_padding_mask.is_contiguous()):
            raise ValueError("key_padding_mask must be a contiguous bool/uint8 CUDA tensor [B, N]")
        pad_ptr = key_padding_mask.data_ptr()
    bm_ptr = None
    if block_mask is not None:
        T = (N + BLOCK - 1) // BLOCK
        if (block_mask.shape != (T, T) or block_mask.dtype not in (torch.bool, torch.uint8)
                or not block_mask.is_cuda or not block_mask.is_contiguous()):
            raise ValueError("block_mask must be a contiguous bool/uint8 CUDA tensor [ceil(N/128), ceil(N/128)]")
        bm_ptr = block_mask.data_ptr()
    delta = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    dq = torch.empty((B, H, N, d), dtype=torch.float32, device=q.device)
    dk = torch.empty_like(q)
    dv = torch.empty_like(q)
    status = attn_bwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), dout.data_ptr(), lse.data_ptr(),
                      delta.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), B, H, N, d, scale, causal,
                      _stream_handle(stream), key_padding_mask=pad_ptr, block_mask=bm_ptr)
    if status != ATTN_OK:
        raise AttnError(status, "attn_bwd")
    return dq, dk, dv


def forward_host(q, k, v, scale=None, causal=False, chunks=4, out=None, lse=None, workspace=None,
                 device=None):
    """Attention on host tensors, with transfers overlapped with the kernel.

    q, k, v: contiguous bf16 CPU tensors [B, H, N, d] (pinned, for
    asynchronous copies).  The B*H heads are split into ``chunks`` groups;
    group c+1 is copied to the device while the kernel runs on group c and
    the outputs of group c-1 are copied back, on three CUDA streams.  Returns
    host tensors (o bf16 [B, H, N, d], lse fp32 [B, H, N]), written into
    ``out`` / ``lse`` when given (pinned host tensors).  ``workspace``: None
    or a tuple of device tensors (q, k, v, o, lse) shaped like the inputs and
    outputs, reused across calls.  On return every copy has been queued; the
    current stream of ``device`` is ordered after all of them (synchronize it
    before reading the outputs).
    """
    import torch
    if q.dim() != 4 or q.shape != k.shape or q.shape != v.shape:
        raise ValueError("q, k, v must share one shape [B, H, N, d]")
    for name, t in (("q", q), ("k", k), ("v", v)):
        if t.dtype != torch.bfloat16 or t.is_cuda or not t.is_contiguous():
            raise ValueError("%s must be a contiguous bf16 host tensor" % name)
    B, H, N, d = (int(x) for x in q.shape)
    BH = B * H
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    if out is None:
        out = torch.empty((B, H, N, d), dtype=torch.bfloat16).pin_memory()
    if lse is None:
        lse = torch.empty((B, H, N), dtype=torch.float32).pin_memory()
    if workspace is None:
        workspace = (torch.empty((B, H, N, d), dtype=torch.bfloat16, device=dev),
                     torch.empty((B, H, N, d), dtype=torch.bfloat16, device=dev),
                     torch.empty((B, H, N, d), dtype=torch.bfloat16, device=dev),
                     torch.empty((B, H, N, d), dtype=torch.bfloat16, device=dev),
                     torch.empty((B, H, N), dtype=torch.float32, device=dev))
    qd, kd, vd, od, ld = (w.view(BH, *w.shape[2:]) for w in workspace)
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    for w in workspace:  # used on the copy streams too: keep the allocator from reusing it early
        w.record_stream(s_in)
        w.record_stream(s_out)
    qh, kh, vh, oh, lh = (t.view(BH, *t.shape[2:]) for t in (q, k, v, out, lse))
    chunks = max(1, min(int(chunks), BH))
    bounds = [BH * c // chunks for c in range(chunks + 1)]
    compute = torch.cuda.current_stream(dev)
    s_in.wait_stream(compute)  # the workspace is free once earlier work on it is done
    s_out.wait_stream(compute)
    for c in range(chunks):
        h0, h1 = bounds[c], bounds[c + 1]
        if h1 == h0:
            continue
        with torch.cuda.stream(s_in):
            for dst, src in ((qd, qh), (kd, kh), (vd, vh)):
                dst[h0:h1].copy_(src[h0:h1], non_blocking=True)
        compute.wait_stream(s_in)
        view = lambda t: t[h0:h1].view(1, h1 - h0, *t.shape[1:])
        forward(view(qd), view(kd), view(vd), scale=scale, causal=causal, out=view(od), lse=view(ld),
                stream=compute)
        s_out.wait_stream(compute)
        with torch.cuda.stream(s_out):
            oh[h0:h1].copy_(od[h0:h1], non_blocking=True)
            lh[h0:h1].copy_(ld[h0:h1], non_blocking=True)
    compute.wait_stream(s_out)
    return out, lse
