"""ctypes binding of libfa_b200.so: the C ABI of ``include/fa.h`` with the same names.

Argument marshalling only.  Tensors are torch CUDA tensors (device memory and
streams come from PyTorch); every step of the attention path runs in the
library's kernels.  There is no fallback: if the library is missing the
import of a function raises.

Raw entry points (same argument order as the C ABI; tensors are passed as
torch tensors or None, the stream as a torch.cuda.Stream or None = current):
``fa_fwd``, ``fa_fwd_traced``, ``fa_bwd``, ``fa_bwd_traced``, ``fa_bwd_phase``,
``fa_bwd_deterministic``, ``fa_fwd_dropout``, ``fa_bwd_dropout``, ``fa_fwd_varlen``,
``fa_bwd_varlen``, ``fa_bwd_noalloc``, ``fa_bwd_workspace_size``,
``fa_selftest_wait_timeout``, ``fa_selftest_ex2``, ``fa_get_device_status``, ``fa_status_string``,
``fa_version``.

Convenience wrappers that allocate outputs: ``attention_forward`` and
``attention_backward`` (options ``dropout=(p, seed, offset)`` and, for the backward,
``deterministic=True``), ``attention_forward_varlen`` and ``attention_backward_varlen``
for packed batches.  They check what the raw pointers cannot carry (dtype, shape,
contiguity, one device for all tensors) and raise ValueError before any library call;
they launch on the current stream of q's device unless given a stream.
"""

from __future__ import annotations

import ctypes
import os
import threading

from . import build as _build

_lock = threading.Lock()
_lib = None

_vp = ctypes.c_void_p
_i = ctypes.c_int
_f = ctypes.c_float
_sz = ctypes.c_size_t
_u64 = ctypes.c_uint64
_u32 = ctypes.c_uint32

_SIGS = {
    "fa_fwd": (_i, [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _f, _i, _vp, _vp, _vp]),
    "fa_fwd_traced": (_i, [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _f, _i, _vp, _vp, _vp, _vp]),
    "fa_bwd_workspace_size": (_sz, [_i, _i, _i, _i]),
    "fa_bwd": (_i, [_vp] * 9 + [_i, _i, _i, _i, _f, _i, _vp, _vp, _vp, _sz, _vp]),
    "fa_bwd_traced": (_i, [_vp] * 9 + [_i, _i, _i, _i, _f, _i, _vp, _vp, _vp, _sz, _vp, _vp]),
    "fa_bwd_phase": (_i, [_i] + [_vp] * 9 + [_i, _i, _i, _i, _f, _i, _vp, _vp, _vp, _sz, _vp]),
    "fa_bwd_noalloc": (_i, [_vp] * 9 + [_i, _i, _i, _i, _f, _i, _vp, _vp, _vp]),
    "fa_bwd_deterministic": (_i, [_vp] * 9 + [_i, _i, _i, _i, _f, _i, _vp, _vp, _vp, _sz, _vp]),
    "fa_fwd_dropout": (_i, [_vp] * 5 + [_i, _i, _i, _i, _f, _i, _vp, _vp, _f, _u64, _u32, _vp]),
    "fa_bwd_dropout": (_i, [_vp] * 9 + [_i, _i, _i, _i, _f, _i, _vp, _vp, _f, _u64, _u32, _vp,
                                        _sz, _vp]),
    "fa_fwd_varlen": (_i, [_vp] * 6 + [_i, _i, _i, _i, _i, _f, _i, _f, _u64, _u32, _vp]),
    "fa_bwd_varlen": (_i, [_vp] * 10 + [_i, _i, _i, _i, _i, _f, _i, _f, _u64, _u32, _vp, _sz,
                                         _vp]),
    "fa_selftest_wait_timeout": (_i, [_i, ctypes.c_uint, _vp, _vp]),
    "fa_selftest_ex2": (_i, [_vp, _vp, _i, _i, _vp]),
    "fa_get_device_status": (_i, [_vp]),
    "fa_status_string": (ctypes.c_char_p, [_i]),
    "fa_version": (_i, []),
}

FA_OK = 0
STATUS_NAMES = {0: "FA_OK", -1: "FA_ERR_NULL", -2: "FA_ERR_ALIGN", -3: "FA_ERR_SHAPE",
                -4: "FA_ERR_UNSUPPORTED_D", -5: "FA_ERR_WORKSPACE", -6: "FA_ERR_CUDA",
                -7: "FA_ERR_TIMEOUT", -8: "FA_ERR_ARG", -9: "FA_ERR_SCRATCH_LIMIT"}

# size of the library's built-in scratch for fa_bwd_noalloc (FA_BWD_NOALLOC_SCRATCH_BYTES)
BWD_NOALLOC_SCRATCH_BYTES = 64 << 20


class FAError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: {STATUS_NAMES.get(status, status)} ({lib_status_string(status)})")
        self.status = status


def library_path() -> str:
    return _build.LIB


def load(build_if_missing: bool = True):
    """Load libfa_b200.so (building it first if it is missing or stale)."""
    global _lib
    with _lock:
        if _lib is None:
            if build_if_missing and _build.needs_build():
                _build.build()
            if not os.path.exists(_build.LIB):
                raise ImportError(f"{_build.LIB} is missing; run python -m exact_io_aware_63_b200.build")
            lib = ctypes.CDLL(_build.LIB)
            for name, (res, args) in _SIGS.items():
                fn = getattr(lib, name)
                fn.restype = res
                fn.argtypes = args
            _lib = lib
    return _lib


def lib_status_string(status: int) -> str:
    return load().fa_status_string(int(status)).decode()


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream, like=None):
    """The stream handle to pass: ``stream`` itself (a torch.cuda.Stream or a raw handle),
    else the current stream of the device that holds ``like`` (else of the current
    device)."""
    import torch
    if stream is None:
        dev = like.device if isinstance(like, torch.Tensor) and like.is_cuda else None
        stream = torch.cuda.current_stream(dev)
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


# ----------------------------------------------------------------------------
# raw C-ABI calls (same names and argument order)
# ----------------------------------------------------------------------------

def fa_fwd(q, k, v, o, lse, B, H, N, d, scale, causal, block_mask, kv_len, stream=None):
    return load().fa_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, H, N, d, float(scale),
                         int(bool(causal)), _ptr(block_mask), _ptr(kv_len), _stream(stream, q))


def fa_fwd_traced(q, k, v, o, lse, B, H, N, d, scale, causal, block_mask, kv_len, visited,
                  stream=None):
    return load().fa_fwd_traced(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, H, N, d,
                                float(scale), int(bool(causal)), _ptr(block_mask), _ptr(kv_len),
                                _ptr(visited), _stream(stream, q))


def fa_bwd_workspace_size(B, H, N, d):
    return load().fa_bwd_workspace_size(B, H, N, d)


def fa_bwd(q, k, v, o, lse, dout, dq, dk, dv, B, H, N, d, scale, causal, block_mask, kv_len,
           workspace, workspace_bytes, stream=None):
    return load().fa_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(dout), _ptr(dq),
                         _ptr(dk), _ptr(dv), B, H, N, d, float(scale), int(bool(causal)),
                         _ptr(block_mask), _ptr(kv_len), _ptr(workspace), int(workspace_bytes),
                         _stream(stream, q))


def fa_bwd_traced(q, k, v, o, lse, dout, dq, dk, dv, B, H, N, d, scale, causal, block_mask, kv_len,
                  workspace, workspace_bytes, visited, stream=None):
    return load().fa_bwd_traced(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(dout),
                                _ptr(dq), _ptr(dk), _ptr(dv), B, H, N, d, float(scale),
                                int(bool(causal)), _ptr(block_mask), _ptr(kv_len), _ptr(workspace),
                                int(workspace_bytes), _ptr(visited), _stream(stream, q))


def fa_bwd_phase(phase, q, k, v, o, lse, dout, dq, dk, dv, B, H, N, d, scale, causal, block_mask,
                 kv_len, workspace, workspace_bytes, stream=None):
    return load().fa_bwd_phase(int(phase), _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse),
                               _ptr(dout), _ptr(dq), _ptr(dk), _ptr(dv), B, H, N, d, float(scale),
                               int(bool(causal)), _ptr(block_mask), _ptr(kv_len), _ptr(workspace),
                               int(workspace_bytes), _stream(stream, q))


def fa_bwd_deterministic(q, k, v, o, lse, dout, dq, dk, dv, B, H, N, d, scale, causal,
                         block_mask, kv_len, workspace, workspace_bytes, stream=None):
    """fa_bwd with a bitwise-reproducible dQ (ordered per-query-tile kernel)."""
    return load().fa_bwd_deterministic(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(dout),
                                       _ptr(dq), _ptr(dk), _ptr(dv), B, H, N, d, float(scale),
                                       int(bool(causal)), _ptr(block_mask), _ptr(kv_len),
                                       _ptr(workspace), int(workspace_bytes), _stream(stream, q))


def fa_bwd_noalloc(q, k, v, o, lse, dout, dq, dk, dv, B, H, N, d, scale, causal, block_mask,
                   kv_len, stream=None):
    """fa_bwd without a workspace argument: the library's built-in static scratch is used
    (for callers that cannot allocate device memory; see include/fa.h)."""
    return load().fa_bwd_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(dout),
                                 _ptr(dq), _ptr(dk), _ptr(dv), B, H, N, d, float(scale),
                                 int(bool(causal)), _ptr(block_mask), _ptr(kv_len),
                                 _stream(stream, q))


def fa_fwd_dropout(q, k, v, o, lse, B, H, N, d, scale, causal, block_mask, kv_len, p_drop, seed,
                   offset, stream=None):
    """fa_fwd with dropout of probability p_drop on P (Philox keep mask, include/fa.h)."""
    return load().fa_fwd_dropout(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, H, N, d,
                                 float(scale), int(bool(causal)), _ptr(block_mask), _ptr(kv_len),
                                 float(p_drop), int(seed), int(offset), _stream(stream, q))


def fa_bwd_dropout(q, k, v, o, lse, dout, dq, dk, dv, B, H, N, d, scale, causal, block_mask,
                   kv_len, p_drop, seed, offset, workspace, workspace_bytes, stream=None):
    """fa_bwd for the output of fa_fwd_dropout with the same p_drop, seed and offset."""
    return load().fa_bwd_dropout(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(dout),
                                 _ptr(dq), _ptr(dk), _ptr(dv), B, H, N, d, float(scale),
                                 int(bool(causal)), _ptr(block_mask), _ptr(kv_len),
                                 float(p_drop), int(seed), int(offset), _ptr(workspace),
                                 int(workspace_bytes), _stream(stream, q))


def fa_fwd_varlen(q, k, v, o, lse, cu_seqlens, B, H, max_seqlen, total_tokens, d, scale, causal,
                  p_drop=0.0, seed=0, offset=0, stream=None):
    """Forward pass of a packed variable-length batch ([T, H, d] tensors, LSE [H, T])."""
    return load().fa_fwd_varlen(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(cu_seqlens),
                                B, H, max_seqlen, total_tokens, d, float(scale),
                                int(bool(causal)), float(p_drop), int(seed), int(offset),
                                _stream(stream, q))


def fa_bwd_varlen(q, k, v, o, lse, dout, dq, dk, dv, cu_seqlens, B, H, max_seqlen, total_tokens,
                  d, scale, causal, p_drop, seed, offset, workspace, workspace_bytes,
                  stream=None):
    """Backward pass of a packed variable-length batch; workspace of
    fa_bwd_workspace_size(B, H, max_seqlen, d) bytes."""
    return load().fa_bwd_varlen(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(dout),
                                _ptr(dq), _ptr(dk), _ptr(dv), _ptr(cu_seqlens), B, H, max_seqlen,
                                total_tokens, d, float(scale), int(bool(causal)), float(p_drop),
                                int(seed), int(offset), _ptr(workspace), int(workspace_bytes),
                                _stream(stream, q))


def fa_selftest_wait_timeout(arrive, limit_us, result, stream=None):
    """One warp waits on a barrier for at most limit_us; see include/fa.h."""
    return load().fa_selftest_wait_timeout(int(arrive), int(limit_us), _ptr(result),
                                           _stream(stream, result))


def fa_selftest_ex2(x, y, n, pair, stream=None):
    """y[i] = the kernels' FMA-pipe 2^x[i] for i < n (float32 device arrays); see
    include/fa.h."""
    return load().fa_selftest_ex2(_ptr(x), _ptr(y), int(n), int(bool(pair)), _stream(stream, x))


def fa_get_device_status(stream=None):
    return load().fa_get_device_status(_stream(stream))


def fa_status_string(status):
    return lib_status_string(status)


def fa_version():
    return load().fa_version()


# ----------------------------------------------------------------------------
# convenience wrappers (allocate outputs with torch, then call the C ABI)
# ----------------------------------------------------------------------------

def _check(rc, what):
    if rc != FA_OK:
        raise FAError(rc, what)


def _expect(t, name, dtype, shape, device):
    """Raise unless ``t`` is a contiguous tensor of ``dtype`` and ``shape`` on ``device``:
    the C ABI sees raw pointers and cannot tell a wrong layout from a right one."""
    import torch
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor, not {type(t).__name__}")
    if t.dtype != dtype:
        raise ValueError(f"{name}: dtype {t.dtype}, expected {dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: shape {tuple(t.shape)}, expected {tuple(shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device} (the device of q)")


def _expect_workspace(ws, device):
    import torch
    if not isinstance(ws, torch.Tensor) or not ws.is_contiguous() or ws.device != device:
        raise ValueError(f"workspace must be a contiguous tensor on {device}")


def _expect_visited(visited, B, H, N, device):
    import torch
    nt = (N + 127) // 128
    _expect(visited, "visited", torch.uint8, (B, H, nt, nt), device)


def _expect_cuda(q, stream):
    """Raise unless q is a CUDA tensor; return the stream to launch on (default: the current
    stream of q's device, not of the current device)."""
    import torch
    if q.device.type != "cuda":
        raise ValueError(f"the tensors must be CUDA tensors, q is on {q.device}")
    return torch.cuda.current_stream(q.device) if stream is None else stream


def _expect_dense(q, k, v, block_mask, kv_len, extra=()):
    """Checks of a [B, H, N, d] call: q, k, v and ``extra`` (name, tensor, dtype, shape)."""
    import torch
    if not isinstance(q, torch.Tensor) or q.dim() != 4:
        raise ValueError("q must be a 4-D tensor [B, H, N, d]")
    B, H, N, d = q.shape
    dev = q.device
    for name, t in (("q", q), ("k", k), ("v", v)):
        _expect(t, name, torch.bfloat16, (B, H, N, d), dev)
    for name, t, dtype, shape in extra:
        _expect(t, name, dtype, shape, dev)
    nt = (N + 127) // 128
    if block_mask is not None:
        _expect(block_mask, "block_mask", torch.uint8, (nt, nt), dev)
    if kv_len is not None:
        _expect(kv_len, "kv_len", torch.int32, (B,), dev)
    return B, H, N, d


def _expect_packed(q, k, v, cu_seqlens, extra=()):
    """Checks of a packed [T, H, d] call."""
    import torch
    if not isinstance(q, torch.Tensor) or q.dim() != 3:
        raise ValueError("q must be a 3-D tensor [T, H, d]")
    T, H, d = q.shape
    dev = q.device
    for name, t in (("q", q), ("k", k), ("v", v)):
        _expect(t, name, torch.bfloat16, (T, H, d), dev)
    if not isinstance(cu_seqlens, torch.Tensor) or cu_seqlens.dim() != 1 or cu_seqlens.numel() < 1:
        raise ValueError("cu_seqlens must be a 1-D tensor [B + 1]")
    _expect(cu_seqlens, "cu_seqlens", torch.int32, (cu_seqlens.numel(),), dev)
    for name, t, dtype, shape in extra:
        _expect(t, name, dtype, shape, dev)
    return T, H, d


def attention_forward(q, k, v, scale, causal=False, block_mask=None, kv_len=None, visited=None,
                      stream=None, dropout=None):
    """O, LSE for bf16 CUDA tensors q, k, v of shape [B, H, N, d].  ``dropout`` is None or
    (p_drop, seed, offset) and selects fa_fwd_dropout."""
    import torch
    B, H, N, d = _expect_dense(q, k, v, block_mask, kv_len)
    if visited is not None:
        _expect_visited(visited, B, H, N, q.device)
    stream = _expect_cuda(q, stream)
    o = torch.empty_like(q)
    lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    if dropout is not None:
        if visited is not None:
            raise ValueError("the dropout forward has no traced variant")
        p_drop, seed, offset = dropout
        rc = fa_fwd_dropout(q, k, v, o, lse, B, H, N, d, scale, causal, block_mask, kv_len,
                            p_drop, seed, offset, stream)
    elif visited is None:
        rc = fa_fwd(q, k, v, o, lse, B, H, N, d, scale, causal, block_mask, kv_len, stream)
    else:
        rc = fa_fwd_traced(q, k, v, o, lse, B, H, N, d, scale, causal, block_mask, kv_len,
                           visited, stream)
    _check(rc, "fa_fwd")
    return o, lse


def attention_backward(q, k, v, o, lse, dout, scale, causal=False, block_mask=None, kv_len=None,
                       workspace=None, visited=None, stream=None, deterministic=False,
                       dropout=None):
    """dQ, dK, dV for the forward that produced (o, lse).  ``deterministic`` selects
    fa_bwd_deterministic (bitwise-reproducible dQ); ``dropout`` = (p_drop, seed, offset),
    the forward's, selects fa_bwd_dropout."""
    import torch
    B, H, N, d = _expect_dense(q, k, v, block_mask, kv_len, extra=(
        ("o", o, torch.bfloat16, q.shape), ("dout", dout, torch.bfloat16, q.shape),
        ("lse", lse, torch.float32, q.shape[:3])))
    if visited is not None:
        _expect_visited(visited, B, H, N, q.device)
    stream = _expect_cuda(q, stream)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ws_bytes = fa_bwd_workspace_size(B, H, N, d)
    if workspace is None:
        workspace = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device=q.device)
    else:
        _expect_workspace(workspace, q.device)
    if dropout is not None:
        if visited is not None or deterministic:
            raise ValueError("the dropout backward has no traced or deterministic variant")
        p_drop, seed, offset = dropout
        rc = fa_bwd_dropout(q, k, v, o, lse, dout, dq, dk, dv, B, H, N, d, scale, causal,
                            block_mask, kv_len, p_drop, seed, offset, workspace,
                            workspace.nbytes, stream)
    elif deterministic:
        if visited is not None:
            raise ValueError("the deterministic backward has no traced variant")
        rc = fa_bwd_deterministic(q, k, v, o, lse, dout, dq, dk, dv, B, H, N, d, scale, causal,
                                  block_mask, kv_len, workspace, workspace.nbytes, stream)
    elif visited is None:
        rc = fa_bwd(q, k, v, o, lse, dout, dq, dk, dv, B, H, N, d, scale, causal, block_mask,
                    kv_len, workspace, workspace.nbytes, stream)
    else:
        rc = fa_bwd_traced(q, k, v, o, lse, dout, dq, dk, dv, B, H, N, d, scale, causal,
                           block_mask, kv_len, workspace, workspace.nbytes, visited, stream)
    _check(rc, "fa_bwd")
    return dq, dk, dv


def attention_forward_varlen(q, k, v, cu_seqlens, max_seqlen, scale, causal=False, dropout=None,
                             stream=None):
    """O [T, H, d] and LSE [H, T] for a packed batch: bf16 CUDA tensors [T, H, d] and
    int32 CUDA cu_seqlens [B + 1]; ``dropout`` = None or (p_drop, seed, offset)."""
    import torch
    T, H, d = _expect_packed(q, k, v, cu_seqlens)
    stream = _expect_cuda(q, stream)
    B = cu_seqlens.numel() - 1
    o = torch.empty_like(q)
    lse = torch.empty((H, T), dtype=torch.float32, device=q.device)
    p_drop, seed, offset = dropout if dropout is not None else (0.0, 0, 0)
    rc = fa_fwd_varlen(q, k, v, o, lse, cu_seqlens, B, H, max_seqlen, T, d, scale, causal, p_drop,
                       seed, offset, stream)
    _check(rc, "fa_fwd_varlen")
    return o, lse


def attention_backward_varlen(q, k, v, o, lse, dout, cu_seqlens, max_seqlen, scale, causal=False,
                              dropout=None, workspace=None, stream=None):
    """dQ, dK, dV [T, H, d] for the packed forward that produced (o, lse)."""
    import torch
    T, H, d = _expect_packed(q, k, v, cu_seqlens, extra=(
        ("o", o, torch.bfloat16, q.shape), ("dout", dout, torch.bfloat16, q.shape),
        ("lse", lse, torch.float32, (q.shape[1], q.shape[0]))))
    stream = _expect_cuda(q, stream)
    B = cu_seqlens.numel() - 1
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ws_bytes = fa_bwd_workspace_size(B, H, max_seqlen, d)
    if workspace is None:
        workspace = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device=q.device)
    else:
        _expect_workspace(workspace, q.device)
    p_drop, seed, offset = dropout if dropout is not None else (0.0, 0, 0)
    rc = fa_bwd_varlen(q, k, v, o, lse, dout, dq, dk, dv, cu_seqlens, B, H, max_seqlen, T, d,
                       scale, causal, p_drop, seed, offset, workspace, workspace.nbytes, stream)
    _check(rc, "fa_bwd_varlen")
    return dq, dk, dv
