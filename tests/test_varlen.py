"""Packed variable-length batches (fa_fwd_varlen, fa_bwd_varlen) against the FP64 oracle,
with the tolerances of gpu_helpers; the equal-length case against the [B, H, N, d] kernels
bit for bit; and guard rows around every tensor that no call may touch."""

import numpy as np
import pytest
import torch

import oracle
from exact_io_aware_63_b200 import binding, inputs
from gpu_helpers import GRAD_TOL, LSE_TOL, O_TOL, rel_l2

pytestmark = pytest.mark.gpu

DEV = torch.device("cuda", 0)


def _status_ok():
    torch.cuda.synchronize()
    st = binding.fa_get_device_status()
    assert st == 0, binding.fa_status_string(st)


def _run(x, dropout=None):
    q, k, v, do = (t.to(DEV) for t in (x.q, x.k, x.v, x.dout))
    cu = x.cu_seqlens.to(DEV)
    o, lse = binding.attention_forward_varlen(q, k, v, cu, x.max_seqlen, x.scale, x.causal,
                                              dropout=dropout)
    dq, dk, dv = binding.attention_backward_varlen(q, k, v, o, lse, do, cu, x.max_seqlen,
                                                   x.scale, x.causal, dropout=dropout)
    _status_ok()
    return {n: t.double().cpu().numpy() for n, t in
            dict(o=o, lse=lse, dq=dq, dk=dk, dv=dv).items()}


def _f64(t):
    return t.double().numpy()


def _check(x, dropout=None):
    out = _run(x, dropout)
    q, k, v, do = (_f64(t) for t in (x.q, x.k, x.v, x.dout))
    o, lse = oracle.attention_forward_varlen(q, k, v, x.cu_seqlens.numpy(), x.scale, x.causal,
                                             dropout=dropout)
    fin = np.isfinite(lse)
    assert np.array_equal(np.isfinite(out["lse"]), fin)
    err = float(np.abs(out["o"] - o).max()) if o.size else 0.0
    if dropout is None:
        assert err <= O_TOL, err
    else:
        # the dropout weight lifts |O| above 2.56, where half a bf16 ulp exceeds O_TOL:
        # the element-wise bound of the kernel's two roundings (see test_dropout.py)
        pv, _ = oracle.attention_forward_varlen(q, k, np.abs(v), x.cu_seqlens.numpy(), x.scale,
                                                x.causal, dropout=dropout)
        u = 2.0 ** -8
        bound = np.maximum(O_TOL, u * pv + u * (1 + u) * np.abs(o) + 1e-5)
        assert np.all(np.abs(out["o"] - o) <= bound)
    if fin.any():
        assert float(np.abs(out["lse"][fin] - lse[fin]).max()) <= LSE_TOL
    g = oracle.attention_backward_varlen(q, k, v, do, x.cu_seqlens.numpy(), x.scale, x.causal,
                                         dropout=dropout)
    for name, ref in zip(("dq", "dk", "dv"), g):
        e = rel_l2(out[name], ref)
        assert e <= GRAD_TOL, (name, e)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
def test_mixed_lengths_against_oracle(cuda_device, d, causal):
    # a single token, one short of a tile, a tile, one past, several tiles with a
    # ragged tail, an empty sequence, and half a tile
    x = inputs.make_packed_inputs([1, 127, 128, 129, 300, 0, 64, 513], 2, d, causal=causal,
                                  seed=600 + d)
    _check(x)


def test_dropout_against_oracle(cuda_device):
    x = inputs.make_packed_inputs([200, 77, 384], 2, 64, causal=True, seed=610)
    _check(x, dropout=(0.2, 1234, 7))


def test_bert_shaped_batch_against_oracle(cuda_device):
    # the BERT-shaped workload as a packed batch: 16 sequences of 256..512 tokens
    lengths = inputs.draw_lengths(16, 256, 512, seed=1001)
    _check(inputs.make_packed_inputs(lengths, 16, 64, scale=1.0 / 8.0, seed=620))


@pytest.mark.parametrize("causal", [False, True])
def test_equal_lengths_match_the_dense_kernels_bit_for_bit(cuda_device, causal):
    B, H, N, d = 3, 2, 320, 64
    x = inputs.make_packed_inputs([N] * B, H, d, causal=causal, seed=630)
    packed = _run(x)
    dense = lambda t: t.reshape(B, N, H, d).permute(0, 2, 1, 3).contiguous().to(DEV)
    q, k, v, do = (dense(t) for t in (x.q, x.k, x.v, x.dout))
    o, lse = binding.attention_forward(q, k, v, x.scale, causal)
    dq, dk, dv = binding.attention_backward(q, k, v, o, lse, do, x.scale, causal)
    _status_ok()
    back = lambda t: t.permute(0, 2, 1, 3).reshape(B * N, H, d).double().cpu().numpy()
    assert np.array_equal(packed["o"], back(o))
    assert np.array_equal(packed["lse"], lse.permute(1, 0, 2).reshape(H, B * N).double().cpu().numpy())
    assert np.array_equal(packed["dk"], back(dk)) and np.array_equal(packed["dv"], back(dv))
    # dQ is summed with reduce-adds in a run-dependent order
    assert rel_l2(packed["dq"], back(dq)) < 1e-3


def test_guard_rows_untouched(cuda_device):
    # every tensor is a view into a larger buffer filled with a sentinel; the calls
    # may write only the [T, H, d] / [H, T] views
    x = inputs.make_packed_inputs([130, 5, 257], 2, 64, causal=True, seed=640)
    T, H, d = x.q.shape
    G = 300  # guard rows after each tensor
    sentinel = -12288.0  # exact in bfloat16 and float32

    def guarded(t=None, shape=(T, H, d), dtype=torch.bfloat16):
        buf = torch.full((shape[0] + G,) + tuple(shape[1:]), sentinel, dtype=dtype, device=DEV)
        if t is not None:
            buf[:shape[0]] = t.to(DEV)
        return buf, buf[:shape[0]]

    bufs = {}
    for name in ("q", "k", "v", "dout"):
        bufs[name] = guarded(getattr(x, name))
    for name in ("o", "dq", "dk", "dv"):
        bufs[name] = guarded()
    lse_buf = torch.full((H * T + G,), sentinel, dtype=torch.float32, device=DEV)
    lse = lse_buf[:H * T].view(H, T)
    cu = x.cu_seqlens.to(DEV)
    B = cu.numel() - 1
    rc = binding.fa_fwd_varlen(bufs["q"][1], bufs["k"][1], bufs["v"][1], bufs["o"][1], lse, cu,
                               B, H, x.max_seqlen, T, d, x.scale, True)
    assert rc == 0
    ws = torch.empty(binding.fa_bwd_workspace_size(B, H, x.max_seqlen, d), dtype=torch.uint8,
                     device=DEV)
    rc = binding.fa_bwd_varlen(bufs["q"][1], bufs["k"][1], bufs["v"][1], bufs["o"][1], lse,
                               bufs["dout"][1], bufs["dq"][1], bufs["dk"][1], bufs["dv"][1], cu,
                               B, H, x.max_seqlen, T, d, x.scale, True, 0.0, 0, 0, ws,
                               ws.numel())
    assert rc == 0
    _status_ok()
    for name, (buf, _) in bufs.items():
        assert bool((buf[T:].float() == sentinel).all()), name
    assert bool((lse_buf[H * T:] == sentinel).all())
    # and the values inside are right
    out_o = bufs["o"][1].double().cpu().numpy()
    o_ref, _ = oracle.attention_forward_varlen(*(t.double().numpy() for t in (x.q, x.k, x.v)),
                                               x.cu_seqlens.numpy(), x.scale, True)
    assert float(np.abs(out_o - o_ref).max()) <= O_TOL
