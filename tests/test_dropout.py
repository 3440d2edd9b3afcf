"""Dropout fused into the forward and backward kernels (fa_fwd_dropout, fa_bwd_dropout),
against the FP64 oracle with the same Philox-4x32-10 keep mask.

The keep pattern is compared bit for bit: with Q = 0 every allowed score is 0, so P is
the same positive value for every allowed key, and an output entry is zero exactly when
its key was dropped.  A block mask that gives each query tile a single key tile and
one-hot values (forward) or one-hot output gradients (backward) then expose every
(query, key) decision of the tile pairs the kernels visit.  Values are compared within
the tolerances of gpu_helpers."""

import numpy as np
import pytest
import torch

import oracle
from exact_io_aware_63_b200 import binding, inputs
from gpu_helpers import compare_forward, compare_grads, f64, to_dev

pytestmark = pytest.mark.gpu


def _status_ok():
    torch.cuda.synchronize()
    status = binding.fa_get_device_status()
    assert status == 0, binding.fa_status_string(status)


def _run(x, drop, backward=True):
    q, k, v, do, bm, kl = to_dev(x)
    o, lse = binding.attention_forward(q, k, v, x.scale, x.causal, bm, kl, dropout=drop)
    out = {"o": o, "lse": lse}
    if backward:
        out["dq"], out["dk"], out["dv"] = binding.attention_backward(
            q, k, v, o, lse, do, x.scale, x.causal, bm, kl, dropout=drop)
    _status_ok()
    return out


def _check(x, p_drop, seed, offset=0, heads=None):
    B, H = x.q.shape[:2]
    if heads is None:
        heads = [(b, h) for b in range(B) for h in range(H)]
    out = _run(x, (p_drop, seed, offset))
    pick = lambda t: np.stack([f64(t[b, h]) for b, h in heads])[:, None]
    # the oracle sees one head per batch entry, so its head index b*H+h must be
    # reproduced: run it on the whole problem and pick the heads afterwards
    q, k, v, do = (f64(t) for t in (x.q, x.k, x.v, x.dout))
    bm = None if x.block_mask is None else x.block_mask.numpy()
    kl = None if x.kv_len is None else x.kv_len.numpy()
    o_ref, lse_ref = oracle.attention_forward_dropout(q, k, v, x.scale, p_drop, seed, offset,
                                                      x.causal, bm, kl)
    dq, dk, dv, _ = oracle.attention_backward_dropout(q, k, v, do, x.scale, p_drop, seed, offset,
                                                      x.causal, bm, kl)
    ref = lambda t: np.stack([t[b, h] for b, h in heads])[:, None]
    compare_forward(pick(out["o"]), pick(out["lse"]), ref(o_ref), ref(lse_ref), "dropout forward")
    compare_grads({n: pick(out[n]) for n in ("dq", "dk", "dv")},
                  {"dq": ref(dq), "dk": ref(dk), "dv": ref(dv)}, "dropout backward")


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
def test_dense_against_oracle(cuda_device, d, causal):
    _check(inputs.make_inputs(2, 2, 384, d, causal=causal, seed=400 + d), 0.2, seed=7)


@pytest.mark.parametrize("d", [64, 128])
def test_partial_tile_and_key_padding(cuda_device, d):
    x = inputs.make_inputs(3, 1, 300, d, seed=410 + d,
                           kv_len=torch.tensor([1, 150, 300], dtype=torch.int32))
    _check(x, 0.1, seed=11, offset=5)


def test_block_mask_high_rate(cuda_device):
    x = inputs.make_inputs(1, 2, 640, 64, causal=True, seed=420, block_keep=0.5)
    _check(x, 0.5, seed=0x1234_5678_9ABC_DEF0)


def test_workload_first_batch_entry(cuda_device):
    # the GPT-2-shaped problem at its full size with dropout 0.1; batch entry 0 (heads
    # b*H+h = 0..H-1, the oracle's own numbering when it is given that entry alone)
    # is compared in full
    x = inputs.workload_inputs("gpt2")
    B, H, N, d = x.q.shape
    out = _run(x, (0.1, 99, 3))
    q, k, v, do = (f64(t[0:1]) for t in (x.q, x.k, x.v, x.dout))
    o_ref, lse_ref = oracle.attention_forward_dropout(q, k, v, x.scale, 0.1, 99, 3, x.causal)
    dq, dk, dv, _ = oracle.attention_backward_dropout(q, k, v, do, x.scale, 0.1, 99, 3, x.causal)
    first = lambda t: f64(t[0:1])
    compare_forward(first(out["o"]), first(out["lse"]), o_ref, lse_ref, "gpt2 dropout forward")
    compare_grads({n: first(out[n]) for n in ("dq", "dk", "dv")},
                  {"dq": dq, "dk": dk, "dv": dv}, "gpt2 dropout backward")


def _one_key_tile_per_query_tile(nt, shift):
    """Block mask in which query tile i sees key tile (i + shift) % nt only."""
    bm = torch.zeros((nt, nt), dtype=torch.uint8)
    for i in range(nt):
        bm[i, (i + shift) % nt] = 1
    return bm


@pytest.mark.parametrize("shift", [0, 1])
def test_keep_pattern_is_the_oracles_bit_for_bit(cuda_device, shift):
    B, H, N, d = 2, 3, 512, 128
    nt = N // 128
    p_drop, seed, offset = 0.3, 0xC0FFEE, 17
    dev = torch.device("cuda", 0)
    bm_h = _one_key_tile_per_query_tile(nt, shift)
    bm = bm_h.to(dev)
    q = torch.zeros((B, H, N, d), dtype=torch.bfloat16, device=dev)
    k = torch.randn((B, H, N, d), generator=torch.Generator().manual_seed(5)).to(
        torch.bfloat16).to(dev)
    one_hot = torch.eye(128, dtype=torch.bfloat16).repeat(nt, 1)  # row c = e_{c % 128}
    v = one_hot.expand(B, H, N, d).contiguous().to(dev)
    do = one_hot.expand(B, H, N, d).contiguous().to(dev)
    drop = (p_drop, seed, offset)
    o, lse = binding.attention_forward(q, k, v, 0.125, False, bm, None, dropout=drop)
    dq, dk, dv = binding.attention_backward(q, k, v, o, lse, do, 0.125, False, bm, None,
                                            dropout=drop)
    _status_ok()
    keep, _ = oracle.dropout_keep(B * H, N, p_drop, seed, offset)
    keep = keep.reshape(B, H, N, N)
    o = o.float().cpu().numpy()
    dv = dv.float().cpu().numpy()
    for i in range(nt):
        j = (i + shift) % nt
        rows, cols = slice(i * 128, (i + 1) * 128), slice(j * 128, (j + 1) * 128)
        want = keep[:, :, rows, cols].astype(bool)  # [B, H, query, key]
        # forward: O[r, x] = P * Z[r, j*128 + x]
        assert np.array_equal(o[:, :, rows, :] != 0, want), f"forward, query tile {i}"
        # backward: dV[c, x] = P * Z[i*128 + x, c]
        assert np.array_equal(dv[:, :, cols, :] != 0, want.transpose(0, 1, 3, 2)), \
            f"backward, key tile {j}"
    # the kept fraction is near 1 - p (65536 draws per head: several sigma wide)
    frac = float(keep.mean())
    assert abs(frac - (1 - p_drop)) < 0.01, frac


def test_probability_zero_is_the_plain_kernel(cuda_device):
    x = inputs.make_inputs(2, 2, 384, 64, causal=True, seed=430)
    q, k, v, do, bm, kl = to_dev(x)
    o0, lse0 = binding.attention_forward(q, k, v, x.scale, x.causal, bm, kl)
    o1, lse1 = binding.attention_forward(q, k, v, x.scale, x.causal, bm, kl,
                                         dropout=(0.0, 5, 0))
    g0 = binding.attention_backward(q, k, v, o0, lse0, do, x.scale, x.causal, bm, kl)
    g1 = binding.attention_backward(q, k, v, o1, lse1, do, x.scale, x.causal, bm, kl,
                                    dropout=(0.0, 5, 0))
    _status_ok()
    # keep everything, weight 1: the same products in the same order
    assert torch.equal(o0, o1) and torch.equal(lse0, lse1)
    assert torch.equal(g0[1], g1[1]) and torch.equal(g0[2], g1[2])
    # dQ is summed with reduce-adds in a run-dependent order
    rel = float((g0[0].float() - g1[0].float()).norm() / g0[0].float().norm())
    assert rel < 1e-3, rel


def test_same_counters_same_mask_new_offset_new_mask(cuda_device):
    x = inputs.make_inputs(1, 2, 256, 64, seed=440)
    q, k, v, _, _, _ = to_dev(x)
    a, _ = binding.attention_forward(q, k, v, x.scale, dropout=(0.25, 3, 0))
    b, _ = binding.attention_forward(q, k, v, x.scale, dropout=(0.25, 3, 0))
    c, _ = binding.attention_forward(q, k, v, x.scale, dropout=(0.25, 3, 1))
    e, _ = binding.attention_forward(q, k, v, x.scale, dropout=(0.25, 4, 0))
    _status_ok()
    assert torch.equal(a, b)
    assert not torch.equal(a, c) and not torch.equal(a, e)
