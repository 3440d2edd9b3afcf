"""Dropout fused into the forward and backward kernels (fa_fwd_dropout, fa_bwd_dropout),
against the FP64 oracle with the same Philox-4x32-10 keep mask.

The keep pattern is compared bit for bit: with Q = 0 every allowed score is 0, so P is
the same positive value for every allowed key, and an output entry is zero exactly when
its key was dropped.  A block mask that gives each query tile a single key tile and
one-hot values (forward) or one-hot output gradients (backward) then expose every
(query, key) decision of the tile pairs the kernels visit.  Gradients are compared
within GRAD_TOL of gpu_helpers.  O is compared element by element within the larger of
O_TOL and the bound that the kernel's two roundings give (gpu_helpers.BF16_U): the kept,
scaled P enters P V rounded to bfloat16, and O is rounded to bfloat16 once.  The scale
65536/(65536 - t) > 1 lifts entries of O above 2.56 in magnitude, where half a bfloat16
ulp already exceeds O_TOL; rows with a single allowed key show it (O = Z * V there)."""

import numpy as np
import pytest
import torch

import oracle
from exact_io_aware_63_b200 import binding, inputs
from gpu_helpers import (BF16_U, LSE_TOL, O_TOL, compare_grads, f64, report_beyond_o_tol,
                         to_dev)

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


def compare_forward(o_gpu, lse_gpu, o_ref, lse_ref, pv_abs, where):
    """pv_abs = sum_c P_rc Z_rc |V_cx|, the oracle's dropout output for values |V|."""
    empty = np.isneginf(lse_ref)
    assert np.array_equal(np.isneginf(lse_gpu), empty), f"{where}: -inf LSE rows differ"
    assert np.all(o_gpu[empty] == 0.0), f"{where}: rows with no key must be exactly 0"
    bound = np.maximum(O_TOL, BF16_U * pv_abs + BF16_U * (1 + BF16_U) * np.abs(o_ref) + 1e-5)
    err = np.abs(o_gpu - o_ref)
    if np.any(err > bound):
        idx = np.unravel_index(np.argmax(err - bound), err.shape)
        raise AssertionError(f"{where}: O error {err[idx]:.3e} > bound {bound[idx]:.3e} at "
                             f"{idx}: gpu {o_gpu[idx]:.6f} ref {o_ref[idx]:.6f}")
    report_beyond_o_tol(o_gpu, o_ref, where)
    fin = ~empty
    lerr = float(np.abs(lse_gpu[fin] - lse_ref[fin]).max()) if fin.any() else 0.0
    assert lerr <= LSE_TOL, f"{where}: LSE max-abs {lerr:.3e} > {LSE_TOL}"


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
    pv_abs, _ = oracle.attention_forward_dropout(q, k, np.abs(v), x.scale, p_drop, seed, offset,
                                                 x.causal, bm, kl)
    dq, dk, dv, _ = oracle.attention_backward_dropout(q, k, v, do, x.scale, p_drop, seed, offset,
                                                      x.causal, bm, kl)
    ref = lambda t: np.stack([t[b, h] for b, h in heads])[:, None]
    compare_forward(pick(out["o"]), pick(out["lse"]), ref(o_ref), ref(lse_ref), ref(pv_abs),
                    "dropout forward")
    compare_grads({n: pick(out[n]) for n in ("dq", "dk", "dv")},
                  {"dq": ref(dq), "dk": ref(dk), "dv": ref(dv)}, "dropout backward")


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
def test_dense_against_oracle(cuda_device, d, causal):
    _check(inputs.make_inputs(2, 2, 384, d, causal=causal, seed=400 + d), 0.2, seed=7)


@pytest.mark.parametrize("d", [64, 128])
def test_partial_tile_and_key_padding(cuda_device, d):
    x = inputs.make_inputs(2, 2, 300, d, seed=410 + d,
                           kv_len=torch.tensor([150, 300], dtype=torch.int32))
    _check(x, 0.1, seed=11, offset=5)


@pytest.mark.parametrize("d", [64, 128])
def test_single_key_rows(cuda_device, d):
    # kv_len = 1: every query sees key 0 alone, so P = 1 and the exact dS = P (Z dP - D)
    # is 0 (D = dO . O = Z dO . V_0 = Z dP): dQ and dK are exactly zero.  The kernel
    # takes D from the stored, bfloat16-rounded O = bf16(w V_0), so its dS is the
    # rounding residue Z dP - D, at most u * sum_x |dO_rx O_rx| (u = 2^-8) plus FP32
    # noise; dQ_r = scale * dS_r K_0 and dK_0 = scale * sum_r dS_r Q_r inherit it.
    # Without dropout O = V_0 is exact and the residue vanishes.
    x = inputs.make_inputs(1, 2, 300, d, seed=415 + d, kv_len=torch.tensor([1], dtype=torch.int32))
    out = _run(x, (0.1, 11, 5))
    q, k, v, do = (f64(t) for t in (x.q, x.k, x.v, x.dout))
    kl = x.kv_len.numpy()
    o_ref, lse_ref = oracle.attention_forward_dropout(q, k, v, x.scale, 0.1, 11, 5, False, None, kl)
    pv_abs, _ = oracle.attention_forward_dropout(q, k, np.abs(v), x.scale, 0.1, 11, 5, False,
                                                 None, kl)
    compare_forward(f64(out["o"]), f64(out["lse"]), o_ref, lse_ref, pv_abs, "single key forward")
    dq, dk, dv, _ = oracle.attention_backward_dropout(q, k, v, do, x.scale, 0.1, 11, 5, False,
                                                      None, kl)
    assert np.all(dq == 0) and np.all(dk == 0)
    assert np.linalg.norm(f64(out["dv"]) - dv) <= 1e-2 * np.linalg.norm(dv)
    ds_bound = 2 * BF16_U * np.sum(np.abs(do * o_ref), axis=-1) + 1e-5  # [B, H, N]
    dq_bound = x.scale * ds_bound[..., None] * np.abs(k[:, :, 0:1, :]) * (1 + BF16_U) + 1e-6
    assert np.all(np.abs(f64(out["dq"])) <= dq_bound)
    dk0_bound = x.scale * np.einsum("bhr,bhry->bhy", ds_bound, np.abs(q)) * (1 + BF16_U) + 1e-6
    assert np.all(np.abs(f64(out["dk"])[:, :, 0, :]) <= dk0_bound)
    assert np.all(f64(out["dk"])[:, :, 1:, :] == 0) and np.all(f64(out["dv"])[:, :, 1:, :] == 0)


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
    pv_abs, _ = oracle.attention_forward_dropout(q, k, np.abs(v), x.scale, 0.1, 99, 3, x.causal)
    dq, dk, dv, _ = oracle.attention_backward_dropout(q, k, v, do, x.scale, 0.1, 99, 3, x.causal)
    first = lambda t: f64(t[0:1])
    compare_forward(first(out["o"]), first(out["lse"]), o_ref, lse_ref, pv_abs,
                    "gpt2 dropout forward")
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
    # p = 0 keeps every entry with weight 1: the plain kernels' results.  The dropout
    # kernels take every exponential from the MUFU unit while the plain ones take a
    # share from a polynomial, so P (and what follows) may differ in its last bits.
    x = inputs.make_inputs(2, 2, 384, 64, causal=True, seed=430)
    q, k, v, do, bm, kl = to_dev(x)
    o0, lse0 = binding.attention_forward(q, k, v, x.scale, x.causal, bm, kl)
    o1, lse1 = binding.attention_forward(q, k, v, x.scale, x.causal, bm, kl,
                                         dropout=(0.0, 5, 0))
    g0 = binding.attention_backward(q, k, v, o0, lse0, do, x.scale, x.causal, bm, kl)
    g1 = binding.attention_backward(q, k, v, o0, lse0, do, x.scale, x.causal, bm, kl,
                                    dropout=(0.0, 5, 0))
    _status_ok()
    assert float((o0.float() - o1.float()).abs().max()) <= O_TOL
    assert float((lse0 - lse1).abs().max()) <= LSE_TOL
    for a, b in zip(g0, g1):
        rel = float((a.float() - b.float()).norm() / a.float().norm())
        assert rel < 2e-3, rel


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
