"""CUDA path vs the FP64 oracle, element by element, through the C ABI.

Small and medium shapes compare every output of every head; they span several
128-row tiles, an odd number of query tiles (a work unit with one tile),
partial key tiles from key padding, causal diagonals, block masks, rows with
no allowed key and batches with no key at all.  The workloads at full size
are covered in test_parity_full.py.
"""

import numpy as np
import pytest
import torch

import oracle
from exact_io_aware_63_b200 import inputs
from gpu_helpers import (LSE_TOL, check_all_heads, compare_grads, f64, forward_error_bound,
                         head_slices, report_beyond_o_tol, run_gpu)

pytestmark = pytest.mark.gpu


def test_tiny_workload(cuda_device):
    check_all_heads(inputs.workload_inputs("tiny"))


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N", [128, 384, 640])
def test_dense(cuda_device, d, causal, N):
    x = inputs.make_inputs(2, 2, N, d, causal=causal, seed=N + d + int(causal))
    check_all_heads(x)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
def test_key_padding(cuda_device, d, causal):
    # lengths inside a tile, on a tile edge, a single key and the full length
    x = inputs.make_inputs(4, 2, 512, d, causal=causal, seed=7 + d,
                           kv_len=torch.tensor([1, 130, 256, 512], dtype=torch.int32))
    check_all_heads(x)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
def test_block_sparse(cuda_device, d, causal):
    x = inputs.make_inputs(1, 3, 768, d, causal=causal, seed=11 + d, block_keep=0.3)
    check_all_heads(x)


@pytest.mark.parametrize("d", [64, 128])
def test_all_masks_combined(cuda_device, d):
    x = inputs.make_inputs(3, 2, 640, d, causal=True, seed=13 + d, block_keep=0.4,
                           kv_len=torch.tensor([77, 600, 640], dtype=torch.int32))
    check_all_heads(x)


@pytest.mark.parametrize("d", [64, 128])
def test_rows_without_keys(cuda_device, d):
    # query tile 0 keeps no key tile; causal + a masked diagonal empties query tile 2 too
    n_t = 4
    bm = torch.ones(n_t, n_t, dtype=torch.uint8)
    bm[0, :] = 0
    bm[2, 2] = 0
    bm[2, 0] = 0
    bm[2, 1] = 0
    x = inputs.make_inputs(2, 2, 512, d, causal=True, seed=17 + d, block_mask=bm,
                           kv_len=torch.tensor([0, 400], dtype=torch.int32))
    res, out = check_all_heads(x)
    o, lse = f64(out["o"]), f64(out["lse"])
    assert np.all(o[:, :, :128] == 0) and np.all(np.isneginf(lse[:, :, :128]))
    assert np.all(o[0] == 0) and np.all(np.isneginf(lse[0]))       # kv_len = 0
    for name in ("dq", "dk", "dv"):
        assert np.all(f64(out[name])[0] == 0), name
    assert np.all(f64(out["dq"])[:, :, :128] == 0)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
def test_key_lengths_outside_zero_to_n(cuda_device, d, causal):
    # kv_len values are taken clamped into [0, N]: -3 leaves batch 0 without keys,
    # N + 5 masks nothing in batch 1; the oracle follows the same contract
    N = 384
    x = inputs.make_inputs(2, 2, N, d, causal=causal, seed=31 + d + int(causal),
                           kv_len=torch.tensor([-3, N + 5], dtype=torch.int32))
    res, out = check_all_heads(x)
    assert np.all(f64(out["o"])[0] == 0) and np.all(np.isneginf(f64(out["lse"])[0]))
    for name in ("dq", "dk", "dv"):
        assert np.all(f64(out[name])[0] == 0), name


@pytest.mark.parametrize("d", [64, 128])
def test_padded_keys_get_zero_gradients(cuda_device, d):
    x = inputs.make_inputs(2, 2, 512, d, seed=19 + d,
                           kv_len=torch.tensor([200, 333], dtype=torch.int32))
    out = run_gpu(x)
    dk, dv = f64(out["dk"]), f64(out["dv"])
    for b, L in enumerate([200, 333]):
        assert np.all(dk[b, :, L:] == 0) and np.all(dv[b, :, L:] == 0)


def test_forward_is_deterministic(cuda_device):
    x = inputs.make_inputs(2, 4, 1024, 128, causal=True, seed=23)
    a, b = run_gpu(x, backward=True), run_gpu(x, backward=True)
    assert torch.equal(a["o"], b["o"]) and torch.equal(a["lse"], b["lse"])
    # dK and dV are accumulated in one CTA each: bitwise reproducible
    assert torch.equal(a["dk"], b["dk"]) and torch.equal(a["dv"], b["dv"])


@pytest.mark.parametrize("d", [64, 128, 256])
def test_large_scores(cuda_device, d):
    # scores of order 100: a peaked softmax whose row max grows across key tiles, which
    # exercises the online rescaling.  Peaked rows put most of the weight on a few keys,
    # so the bfloat16 rounding of P and of O is no longer averaged out; the check is the
    # element-wise bound that follows from those two roundings (forward_error_bound).
    # With the scale 1/sqrt(d) the scores' spread does not depend on d.
    x = inputs.make_inputs(1, 2, 1024, d, seed=29)
    ramp = torch.linspace(0.5, 6.0, 1024)[None, None, :, None]
    x.k = (x.k.float() * ramp).to(torch.bfloat16)
    x.q = (x.q.float() * 3.0).to(torch.bfloat16)
    heads = [(0, 0), (0, 1)]
    out = run_gpu(x)
    q, k, v, do, bm, kl = head_slices(x, heads)
    o_ref, lse_ref = oracle.attention_forward(q, k, v, x.scale, x.causal, bm, kl)
    o_gpu = np.stack([f64(out["o"][b, h]) for b, h in heads])[:, None]
    lse_gpu = np.stack([f64(out["lse"][b, h]) for b, h in heads])[:, None]
    bound = forward_error_bound(x, heads, o_ref)
    err = np.abs(o_gpu - o_ref)
    assert np.all(err <= bound), f"worst excess {float((err - bound).max()):.3e}"
    # elements above O_TOL (allowed by the bound) are reported with |O_ref| and their
    # error in bfloat16 ulps
    report_beyond_o_tol(o_gpu, o_ref, f"large scores d={d}")
    assert float(np.abs(lse_gpu - lse_ref).max()) <= LSE_TOL
    dq, dk, dv, _ = oracle.attention_backward(q, k, v, do, x.scale, x.causal, bm, kl)
    compare_grads({n: np.stack([f64(out[n][b, h]) for b, h in heads])[:, None]
                   for n in ("dq", "dk", "dv")}, {"dq": dq, "dk": dk, "dv": dv}, f"large scores d={d}")


# ---------------------------------------------------------------------------
# sequence lengths that 128 does not divide: a last, partial tile
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N", [1, 100, 200, 383])
def test_partial_last_tile(cuda_device, d, causal, N):
    # B * H > 1 so that a partial tile of one head sits next to the next head's rows
    x = inputs.make_inputs(2, 2, N, d, causal=causal, seed=500 + N + d + int(causal))
    check_all_heads(x)


@pytest.mark.parametrize("d", [64, 128])
def test_partial_last_tile_with_key_padding(cuda_device, d):
    x = inputs.make_inputs(3, 2, 300, d, causal=True, seed=540 + d,
                           kv_len=torch.tensor([300, 257, 129], dtype=torch.int32))
    check_all_heads(x)


def test_partial_last_tile_with_block_mask(cuda_device):
    bm = torch.tensor([[1, 0, 1], [0, 1, 0], [1, 1, 1]], dtype=torch.uint8)
    x = inputs.make_inputs(1, 3, 300, 64, seed=550, block_mask=bm)
    check_all_heads(x)
