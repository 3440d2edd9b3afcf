"""FP64 CPU oracle for exact softmax attention: test infrastructure only.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  It shares no code with the CUDA path
(``exact_io_aware_63_b200``) and never imports it.

The arithmetic lives in ``attention_oracle.c`` (plain C, double precision),
which states the definition it follows: standard attention, which the pages
("FlashAttention: Fast and Memory-Efficient Exact Attention with
IO-Awareness", opendecode.dev summary, "The key idea"; "FlashAttention,
Decoded", gloss of abstract sentence 4) say the tiled method reproduces
exactly.  This module only builds that file with gcc and marshals numpy
arrays to it.

Functions (all arrays contiguous, float64 unless stated):

* ``attention_forward(q, k, v, scale, causal, block_mask, kv_len)`` ->
  ``(o, lse)`` for q, k, v of shape [B, H, N, d].
* ``attention_backward(q, k, v, dout, scale, causal, block_mask, kv_len)`` ->
  ``(dq, dk, dv, delta)`` by the chain rule on sum(O * dO).
* ``attention_forward_band`` / ``attention_backward_band``: the same for query
  rows [r_begin, r_end) of every head (dK, dV then hold those rows' share);
  used to time bounded samples of large workloads.
* ``attention_forward_rows(q_rows, rows, k, v, scale, causal, block_mask,
  kv_len_b)`` -> ``(o_rows, lse_rows)`` for chosen query rows of one head.
* ``attention_backward_dq_rows(q_rows, dout_rows, rows, k, v, scale, causal,
  block_mask, kv_len_b)`` -> ``(dq_rows, delta_rows)``: the row-local part of
  the backward pass (dQ_r and D_r) for chosen query rows of one head.
* ``attention_backward_kv_cols(q, k, v, dout, cols, scale, causal, block_mask,
  kv_len_b)`` -> ``(dk_cols, dv_cols)``: dK and dV of chosen key columns of
  one head (a full pass over the head's rows).
* ``attention_forward_dropout`` / ``attention_backward_dropout`` (extra
  arguments ``p_drop, seed, offset``): the same with dropout on P; the mask is
  ``dropout_keep(BH, N, p_drop, seed, offset)``, cut from Philox-4x32-10 draws
  (``philox4x32_10(counter, key)``, checked word for word against cuRAND's
  host-side Philox-4x32-10 generator in the tests).
* ``attention_forward_varlen(q, k, v, cu_seqlens, scale, causal, dropout)`` /
  ``attention_backward_varlen(q, k, v, dout, cu_seqlens, scale, causal,
  dropout)``: packed variable-length batches (q, k, v, dout [T, H, d];
  sequence b = tokens cu_seqlens[b] .. cu_seqlens[b+1]-1), each sequence its
  own attention problem; computed through the functions above on the
  zero-padded [B, H, N, d] problem with key lengths kv_len = the sequence
  lengths, keeping each sequence's own rows.
* ``tile_visits(B, N, causal, block_mask, kv_len, T=128, i_begin=0,
  i_end=None)`` -> uint8 [B, i_end - i_begin, ceil(N / T)]: 1 where a
  (query tile, key tile) pair holds at least one allowed (row, key).
"""

from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "attention_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

_dp = ctypes.POINTER(ctypes.c_double)
_u8p = ctypes.POINTER(ctypes.c_uint8)
_i32p = ctypes.POINTER(ctypes.c_int32)
_i64p = ctypes.POINTER(ctypes.c_int64)


def build(force: bool = False) -> str:
    """Compile attention_oracle.c into liboracle.so next to it (gcc -O2)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-std=c11", "-Wall", "-shared", "-fPIC", "-o", tmp, _SRC,
             "-lpthread", "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            lib.oracle_attention_forward.argtypes = [
                _dp, _dp, _dp, _dp, _dp, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                ctypes.c_double, ctypes.c_int, _u8p, _i32p, ctypes.c_int]
            lib.oracle_attention_backward.argtypes = [
                _dp, _dp, _dp, _dp, _dp, _dp, _dp, _dp, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                ctypes.c_int, ctypes.c_double, ctypes.c_int, _u8p, _i32p, ctypes.c_int]
            lib.oracle_attention_forward_band.argtypes = [
                _dp, _dp, _dp, _dp, _dp, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                ctypes.c_double, ctypes.c_int, _u8p, _i32p, ctypes.c_int, ctypes.c_int,
                ctypes.c_int]
            lib.oracle_attention_backward_band.argtypes = [
                _dp, _dp, _dp, _dp, _dp, _dp, _dp, _dp, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                ctypes.c_int, ctypes.c_double, ctypes.c_int, _u8p, _i32p, ctypes.c_int,
                ctypes.c_int, ctypes.c_int]
            lib.oracle_attention_forward_rows.argtypes = [
                _dp, _i64p, ctypes.c_int, _dp, _dp, _dp, _dp, ctypes.c_int, ctypes.c_int,
                ctypes.c_double, ctypes.c_int, _u8p, ctypes.c_int, ctypes.c_int]
            lib.oracle_attention_backward_dq_rows.argtypes = [
                _dp, _dp, _i64p, ctypes.c_int, _dp, _dp, _dp, _dp, ctypes.c_int, ctypes.c_int,
                ctypes.c_double, ctypes.c_int, _u8p, ctypes.c_int, ctypes.c_int]
            lib.oracle_attention_backward_kv_cols.argtypes = [
                _dp, _dp, _dp, _dp, _i64p, ctypes.c_int, _dp, _dp, ctypes.c_int, ctypes.c_int,
                ctypes.c_double, ctypes.c_int, _u8p, ctypes.c_int, ctypes.c_int, ctypes.c_int]
            lib.oracle_tile_visits.argtypes = [
                _u8p, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, _u8p, _i32p,
                ctypes.c_int, ctypes.c_int]
            _f = ctypes.c_float
            lib.oracle_attention_forward_dropout.argtypes = [
                _dp, _dp, _dp, _dp, _dp, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                ctypes.c_double, ctypes.c_int, _u8p, _i32p, _f, ctypes.c_uint64, ctypes.c_uint32,
                ctypes.c_int]
            lib.oracle_attention_backward_dropout.argtypes = [
                _dp, _dp, _dp, _dp, _dp, _dp, _dp, _dp, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                ctypes.c_int, ctypes.c_double, ctypes.c_int, _u8p, _i32p, _f, ctypes.c_uint64,
                ctypes.c_uint32, ctypes.c_int]
            lib.oracle_dropout_keep.argtypes = [
                _u8p, ctypes.POINTER(ctypes.c_uint16), ctypes.c_int, ctypes.c_int, _f,
                ctypes.c_uint64, ctypes.c_uint32]
            lib.oracle_philox4x32_10.argtypes = [
                ctypes.POINTER(ctypes.c_uint32), ctypes.c_uint32, ctypes.c_uint32,
                ctypes.POINTER(ctypes.c_uint32)]
            lib.oracle_philox4x32_10.restype = None
            for fn in (lib.oracle_attention_forward_dropout, lib.oracle_attention_backward_dropout,
                       lib.oracle_dropout_keep):
                fn.restype = ctypes.c_int
            for fn in (lib.oracle_attention_forward, lib.oracle_attention_backward,
                       lib.oracle_attention_forward_rows, lib.oracle_tile_visits,
                       lib.oracle_attention_backward_dq_rows,
                       lib.oracle_attention_backward_kv_cols, lib.oracle_attention_forward_band,
                       lib.oracle_attention_backward_band):
                fn.restype = ctypes.c_int
            _lib = lib
    return _lib


def _f64(a):
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _ptr(a, typ):
    return a.ctypes.data_as(typ) if a is not None else None


def _mask_args(block_mask, kv_len):
    bm = None if block_mask is None else np.ascontiguousarray(np.asarray(block_mask, np.uint8))
    kl = None if kv_len is None else np.ascontiguousarray(np.asarray(kv_len, np.int32))
    return bm, kl


def _threads(nthreads):
    return int(nthreads) if nthreads else (os.cpu_count() or 1)


def attention_forward(q, k, v, scale, causal=False, block_mask=None, kv_len=None, nthreads=None):
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, H, N, d = q.shape
    assert k.shape == q.shape and v.shape == q.shape
    bm, kl = _mask_args(block_mask, kv_len)
    o = np.empty_like(q)
    lse = np.empty((B, H, N), np.float64)
    rc = _load().oracle_attention_forward(
        _ptr(q, _dp), _ptr(k, _dp), _ptr(v, _dp), _ptr(o, _dp), _ptr(lse, _dp), B, H, N, d,
        float(scale), int(bool(causal)), _ptr(bm, _u8p), _ptr(kl, _i32p), _threads(nthreads))
    if rc != 0:
        raise RuntimeError(f"oracle_attention_forward failed: {rc}")
    return o, lse


def attention_backward(q, k, v, dout, scale, causal=False, block_mask=None, kv_len=None,
                       nthreads=None):
    q, k, v, dout = _f64(q), _f64(k), _f64(v), _f64(dout)
    B, H, N, d = q.shape
    bm, kl = _mask_args(block_mask, kv_len)
    dq, dk, dv = np.empty_like(q), np.empty_like(q), np.empty_like(q)
    delta = np.empty((B, H, N), np.float64)
    rc = _load().oracle_attention_backward(
        _ptr(q, _dp), _ptr(k, _dp), _ptr(v, _dp), _ptr(dout, _dp), _ptr(dq, _dp), _ptr(dk, _dp),
        _ptr(dv, _dp), _ptr(delta, _dp), B, H, N, d, float(scale), int(bool(causal)),
        _ptr(bm, _u8p), _ptr(kl, _i32p), _threads(nthreads))
    if rc != 0:
        raise RuntimeError(f"oracle_attention_backward failed: {rc}")
    return dq, dk, dv, delta


def attention_forward_dropout(q, k, v, scale, p_drop, seed, offset=0, causal=False,
                              block_mask=None, kv_len=None, nthreads=None):
    """(o, lse) with dropout on P (keep mask from dropout_keep, kept entries scaled by
    65536 / (65536 - floor(p_drop * 65536)))."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, H, N, d = q.shape
    bm, kl = _mask_args(block_mask, kv_len)
    o = np.empty_like(q)
    lse = np.empty((B, H, N), np.float64)
    rc = _load().oracle_attention_forward_dropout(
        _ptr(q, _dp), _ptr(k, _dp), _ptr(v, _dp), _ptr(o, _dp), _ptr(lse, _dp), B, H, N, d,
        float(scale), int(bool(causal)), _ptr(bm, _u8p), _ptr(kl, _i32p), float(p_drop),
        int(seed), int(offset), _threads(nthreads))
    if rc != 0:
        raise RuntimeError(f"oracle_attention_forward_dropout failed: {rc}")
    return o, lse


def attention_backward_dropout(q, k, v, dout, scale, p_drop, seed, offset=0, causal=False,
                               block_mask=None, kv_len=None, nthreads=None):
    """(dq, dk, dv, delta) of sum(O * dO) for the dropout forward with the same mask."""
    q, k, v, dout = _f64(q), _f64(k), _f64(v), _f64(dout)
    B, H, N, d = q.shape
    bm, kl = _mask_args(block_mask, kv_len)
    dq, dk, dv = np.empty_like(q), np.empty_like(q), np.empty_like(q)
    delta = np.empty((B, H, N), np.float64)
    rc = _load().oracle_attention_backward_dropout(
        _ptr(q, _dp), _ptr(k, _dp), _ptr(v, _dp), _ptr(dout, _dp), _ptr(dq, _dp), _ptr(dk, _dp),
        _ptr(dv, _dp), _ptr(delta, _dp), B, H, N, d, float(scale), int(bool(causal)),
        _ptr(bm, _u8p), _ptr(kl, _i32p), float(p_drop), int(seed), int(offset),
        _threads(nthreads))
    if rc != 0:
        raise RuntimeError(f"oracle_attention_backward_dropout failed: {rc}")
    return dq, dk, dv, delta


def dropout_keep(BH, N, p_drop, seed, offset=0):
    """(keep uint8 [BH, N, N], draws uint16 [BH, N, N]): the dropout mask and the
    16-bit draws it is cut from."""
    keep = np.empty((BH, N, N), np.uint8)
    draws = np.empty((BH, N, N), np.uint16)
    rc = _load().oracle_dropout_keep(_ptr(keep, _u8p),
                                     draws.ctypes.data_as(ctypes.POINTER(ctypes.c_uint16)),
                                     BH, N, float(p_drop), int(seed), int(offset))
    if rc != 0:
        raise RuntimeError(f"oracle_dropout_keep failed: {rc}")
    return keep, draws


def philox4x32_10(counter, key):
    """The four 32-bit output words of Philox-4x32-10 for a counter of four words and a
    key of two."""
    ctr = (ctypes.c_uint32 * 4)(*[int(c) & 0xFFFFFFFF for c in counter])
    out = (ctypes.c_uint32 * 4)()
    _load().oracle_philox4x32_10(ctr, int(key[0]) & 0xFFFFFFFF, int(key[1]) & 0xFFFFFFFF, out)
    return [int(x) for x in out]


def attention_forward_band(q, k, v, scale, causal=False, block_mask=None, kv_len=None,
                           r_begin=0, r_end=None, nthreads=None):
    """O and LSE for query rows [r_begin, r_end) of every head (other rows are 0)."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, H, N, d = q.shape
    r_end = N if r_end is None else r_end
    bm, kl = _mask_args(block_mask, kv_len)
    o = np.zeros_like(q)
    lse = np.zeros((B, H, N), np.float64)
    rc = _load().oracle_attention_forward_band(
        _ptr(q, _dp), _ptr(k, _dp), _ptr(v, _dp), _ptr(o, _dp), _ptr(lse, _dp), B, H, N, d,
        float(scale), int(bool(causal)), _ptr(bm, _u8p), _ptr(kl, _i32p), int(r_begin),
        int(r_end), _threads(nthreads))
    if rc != 0:
        raise RuntimeError(f"oracle_attention_forward_band failed: {rc}")
    return o, lse


def attention_backward_band(q, k, v, dout, scale, causal=False, block_mask=None, kv_len=None,
                            r_begin=0, r_end=None, nthreads=None):
    """dQ rows [r_begin, r_end) and those rows' contributions to dK, dV, for every head."""
    q, k, v, dout = _f64(q), _f64(k), _f64(v), _f64(dout)
    B, H, N, d = q.shape
    r_end = N if r_end is None else r_end
    bm, kl = _mask_args(block_mask, kv_len)
    dq, dk, dv = np.zeros_like(q), np.zeros_like(q), np.zeros_like(q)
    delta = np.zeros((B, H, N), np.float64)
    rc = _load().oracle_attention_backward_band(
        _ptr(q, _dp), _ptr(k, _dp), _ptr(v, _dp), _ptr(dout, _dp), _ptr(dq, _dp), _ptr(dk, _dp),
        _ptr(dv, _dp), _ptr(delta, _dp), B, H, N, d, float(scale), int(bool(causal)),
        _ptr(bm, _u8p), _ptr(kl, _i32p), int(r_begin), int(r_end), _threads(nthreads))
    if rc != 0:
        raise RuntimeError(f"oracle_attention_backward_band failed: {rc}")
    return dq, dk, dv, delta


def attention_forward_rows(q_rows, rows, k, v, scale, causal=False, block_mask=None,
                           kv_len_b=None):
    """Forward for query rows ``rows`` (int array) of one head; q_rows is [R, d]."""
    q_rows, k, v = _f64(q_rows), _f64(k), _f64(v)
    rows = np.ascontiguousarray(np.asarray(rows, np.int64))
    R, d = q_rows.shape
    N = k.shape[0]
    bm, _ = _mask_args(block_mask, None)
    o = np.empty((R, d), np.float64)
    lse = np.empty((R,), np.float64)
    rc = _load().oracle_attention_forward_rows(
        _ptr(q_rows, _dp), _ptr(rows, _i64p), R, _ptr(k, _dp), _ptr(v, _dp), _ptr(o, _dp),
        _ptr(lse, _dp), N, d, float(scale), int(bool(causal)), _ptr(bm, _u8p),
        int(kv_len_b is not None), 0 if kv_len_b is None else int(kv_len_b))
    if rc != 0:
        raise RuntimeError(f"oracle_attention_forward_rows failed: {rc}")
    return o, lse


def attention_backward_dq_rows(q_rows, dout_rows, rows, k, v, scale, causal=False,
                               block_mask=None, kv_len_b=None):
    """dQ_r and D_r for query rows ``rows`` of one head; q_rows, dout_rows are [R, d]."""
    q_rows, dout_rows, k, v = _f64(q_rows), _f64(dout_rows), _f64(k), _f64(v)
    rows = np.ascontiguousarray(np.asarray(rows, np.int64))
    R, d = q_rows.shape
    N = k.shape[0]
    bm, _ = _mask_args(block_mask, None)
    dq = np.empty((R, d), np.float64)
    delta = np.empty((R,), np.float64)
    rc = _load().oracle_attention_backward_dq_rows(
        _ptr(q_rows, _dp), _ptr(dout_rows, _dp), _ptr(rows, _i64p), R, _ptr(k, _dp),
        _ptr(v, _dp), _ptr(dq, _dp), _ptr(delta, _dp), N, d, float(scale), int(bool(causal)),
        _ptr(bm, _u8p), int(kv_len_b is not None), 0 if kv_len_b is None else int(kv_len_b))
    if rc != 0:
        raise RuntimeError(f"oracle_attention_backward_dq_rows failed: {rc}")
    return dq, delta


def attention_backward_kv_cols(q, k, v, dout, cols, scale, causal=False, block_mask=None,
                               kv_len_b=None, nthreads=None):
    """dK_c and dV_c for key columns ``cols`` of one head; q, k, v, dout are [N, d]."""
    q, k, v, dout = _f64(q), _f64(k), _f64(v), _f64(dout)
    cols = np.ascontiguousarray(np.asarray(cols, np.int64))
    N, d = q.shape
    C = len(cols)
    bm, _ = _mask_args(block_mask, None)
    dk = np.empty((C, d), np.float64)
    dv = np.empty((C, d), np.float64)
    rc = _load().oracle_attention_backward_kv_cols(
        _ptr(q, _dp), _ptr(k, _dp), _ptr(v, _dp), _ptr(dout, _dp), _ptr(cols, _i64p), C,
        _ptr(dk, _dp), _ptr(dv, _dp), N, d, float(scale), int(bool(causal)), _ptr(bm, _u8p),
        int(kv_len_b is not None), 0 if kv_len_b is None else int(kv_len_b), _threads(nthreads))
    if rc != 0:
        raise RuntimeError(f"oracle_attention_backward_kv_cols failed: {rc}")
    return dk, dv


def tile_visits(B, N, causal=False, block_mask=None, kv_len=None, T=128, i_begin=0, i_end=None):
    nt = -(-N // T)  # ceil(N / T): a last, partial tile holds the remaining positions
    i_end = nt if i_end is None else i_end
    bm, kl = _mask_args(block_mask, kv_len)
    out = np.zeros((B, i_end - i_begin, nt), np.uint8)
    rc = _load().oracle_tile_visits(_ptr(out, _u8p), B, N, T, int(bool(causal)), _ptr(bm, _u8p),
                                    _ptr(kl, _i32p), i_begin, i_end)
    if rc != 0:
        raise RuntimeError(f"oracle_tile_visits failed: {rc}")
    return out


def _unpack_lengths(cu_seqlens):
    cu = [int(c) for c in np.asarray(cu_seqlens)]
    return cu, [cu[b + 1] - cu[b] for b in range(len(cu) - 1)]


def _pad(x, cu, lens, N):
    """[T, H, d] -> zero-padded [B, H, N, d]."""
    T, H, d = x.shape
    out = np.zeros((len(lens), H, N, d), np.float64)
    for b, n in enumerate(lens):
        out[b, :, :n] = np.transpose(x[cu[b]:cu[b] + n], (1, 0, 2))
    return out


def _unpad(x, cu, lens, T):
    """[B, H, N, d] -> [T, H, d] (each sequence's own rows)."""
    H, d = x.shape[1], x.shape[3]
    out = np.zeros((T, H, d), np.float64)
    for b, n in enumerate(lens):
        out[cu[b]:cu[b] + n] = np.transpose(x[b, :, :n], (1, 0, 2))
    return out


def attention_forward_varlen(q, k, v, cu_seqlens, scale, causal=False, dropout=None,
                             nthreads=None):
    """(o [T, H, d], lse [H, T]) of a packed variable-length batch.  Sequence b is the
    attention problem of its own tokens; as the zero-padded [B, H, N, d] problem with
    kv_len = lengths its rows are unchanged (padded keys are masked).  ``dropout`` is
    None or (p_drop, seed, offset); heads are numbered b*H + h, rows and keys within
    the sequence."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    T, H, d = q.shape
    cu, lens = _unpack_lengths(cu_seqlens)
    N = max(lens) if lens else 0
    kl = np.array(lens, np.int32)
    qp, kp, vp = (_pad(x, cu, lens, N) for x in (q, k, v))
    if dropout is None:
        o, lse = attention_forward(qp, kp, vp, scale, causal, None, kl, nthreads)
    else:
        o, lse = attention_forward_dropout(qp, kp, vp, scale, dropout[0], dropout[1], dropout[2],
                                           causal, None, kl, nthreads)
    lse_p = np.full((H, T), -np.inf)
    for b, n in enumerate(lens):
        lse_p[:, cu[b]:cu[b] + n] = lse[b, :, :n]
    return _unpad(o, cu, lens, T), lse_p


def attention_backward_varlen(q, k, v, dout, cu_seqlens, scale, causal=False, dropout=None,
                              nthreads=None):
    """(dq, dk, dv) [T, H, d] of sum(O * dO) for the packed batch.  In the padded
    problem the padded rows get dO = 0, so they add nothing to any gradient."""
    q, k, v, dout = _f64(q), _f64(k), _f64(v), _f64(dout)
    T, H, d = q.shape
    cu, lens = _unpack_lengths(cu_seqlens)
    N = max(lens) if lens else 0
    kl = np.array(lens, np.int32)
    qp, kp, vp, dp = (_pad(x, cu, lens, N) for x in (q, k, v, dout))
    if dropout is None:
        dq, dk, dv, _ = attention_backward(qp, kp, vp, dp, scale, causal, None, kl, nthreads)
    else:
        dq, dk, dv, _ = attention_backward_dropout(qp, kp, vp, dp, scale, dropout[0], dropout[1],
                                                   dropout[2], causal, None, kl, nthreads)
    return tuple(_unpad(x, cu, lens, T) for x in (dq, dk, dv))
