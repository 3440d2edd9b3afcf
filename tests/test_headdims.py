"""Head dimensions other than 64 and 128, against the FP64 oracle.

32 and 96 run on the 64- and 128-column kernels with tensor maps that read the missing
columns as zeros and stores that stop at d.  256 has kernels of its own: a forward kernel
with one query tile per unit, and a backward pass in three passes (dQ, dK, dV), each
recomputing the score tile it needs."""

import numpy as np
import pytest
import torch

import oracle
from exact_io_aware_63_b200 import binding, inputs
from gpu_helpers import BF16_U, GRAD_TOL, LSE_TOL, O_TOL, check_all_heads, rel_l2

pytestmark = pytest.mark.gpu

DEV = torch.device("cuda", 0)


@pytest.mark.parametrize("d", [32, 96])
@pytest.mark.parametrize("causal", [False, True])
def test_dense_with_partial_tile_and_key_padding(cuda_device, d, causal):
    x = inputs.make_inputs(2, 2, 300, d, causal=causal, seed=800 + d,
                           kv_len=torch.tensor([300, 133], dtype=torch.int32))
    check_all_heads(x)


@pytest.mark.parametrize("d", [32, 96])
def test_block_mask(cuda_device, d):
    check_all_heads(inputs.make_inputs(1, 2, 640, d, seed=810 + d, block_keep=0.5))


@pytest.mark.parametrize("d", [32, 96])
def test_packed_batch(cuda_device, d):
    x = inputs.make_packed_inputs([1, 129, 300, 0, 64], 2, d, causal=True, seed=820 + d)
    q, k, v, do = (t.to(DEV) for t in (x.q, x.k, x.v, x.dout))
    cu = x.cu_seqlens.to(DEV)
    o, lse = binding.attention_forward_varlen(q, k, v, cu, x.max_seqlen, x.scale, True)
    dq, dk, dv = binding.attention_backward_varlen(q, k, v, o, lse, do, cu, x.max_seqlen,
                                                   x.scale, True)
    torch.cuda.synchronize()
    assert binding.fa_get_device_status() == 0
    f = lambda t: t.double().cpu().numpy()
    qd, kd, vd, dod = (f(t) for t in (x.q, x.k, x.v, x.dout))
    o_ref, lse_ref = oracle.attention_forward_varlen(qd, kd, vd, x.cu_seqlens.numpy(), x.scale,
                                                     True)
    assert float(np.abs(f(o) - o_ref).max()) <= O_TOL
    fin = np.isfinite(lse_ref)
    assert np.array_equal(np.isfinite(f(lse)), fin)
    assert float(np.abs(f(lse)[fin] - lse_ref[fin]).max()) <= LSE_TOL
    g = oracle.attention_backward_varlen(qd, kd, vd, dod, x.cu_seqlens.numpy(), x.scale, True)
    for name, got, ref in zip(("dq", "dk", "dv"), (dq, dk, dv), g):
        assert rel_l2(f(got), ref) <= GRAD_TOL, name


@pytest.mark.parametrize("d", [32, 96])
def test_dropout(cuda_device, d):
    x = inputs.make_inputs(1, 2, 384, d, causal=True, seed=830 + d)
    q, k, v, do = (t.to(DEV) for t in (x.q, x.k, x.v, x.dout))
    drop = (0.2, 5, 1)
    o, lse = binding.attention_forward(q, k, v, x.scale, True, dropout=drop)
    dq, dk, dv = binding.attention_backward(q, k, v, o, lse, do, x.scale, True, dropout=drop)
    torch.cuda.synchronize()
    assert binding.fa_get_device_status() == 0
    f = lambda t: t.double().cpu().numpy()
    qd, kd, vd, dod = (f(t) for t in (x.q, x.k, x.v, x.dout))
    o_ref, _ = oracle.attention_forward_dropout(qd, kd, vd, x.scale, *drop, causal=True)
    pv, _ = oracle.attention_forward_dropout(qd, kd, np.abs(vd), x.scale, *drop, causal=True)
    bound = np.maximum(O_TOL, BF16_U * pv + BF16_U * (1 + BF16_U) * np.abs(o_ref) + 1e-5)
    assert np.all(np.abs(f(o) - o_ref) <= bound)
    g = oracle.attention_backward_dropout(qd, kd, vd, dod, x.scale, *drop, causal=True)
    for name, got, ref in zip(("dq", "dk", "dv"), (dq, dk, dv), g[:3]):
        assert rel_l2(f(got), ref) <= GRAD_TOL, name


# ---------------------------------------------------------------------------
# head dimension 256
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N", [128, 384, 640])
def test_d256_dense(cuda_device, causal, N):
    check_all_heads(inputs.make_inputs(2, 2, N, 256, causal=causal, seed=900 + N + int(causal)))


@pytest.mark.parametrize("causal", [False, True])
def test_d256_partial_tile_and_key_padding(cuda_device, causal):
    # lengths inside a tile, on a tile edge, a single key, out of range
    x = inputs.make_inputs(4, 2, 300, 256, causal=causal, seed=910 + int(causal),
                           kv_len=torch.tensor([300, 128, 1, 77], dtype=torch.int32))
    check_all_heads(x)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N", [1, 100])
def test_d256_single_partial_tile(cuda_device, causal, N):
    # one query tile and one key tile, both partial; B * H > 1 so that the partial tile
    # of one head sits next to the next head's rows
    check_all_heads(inputs.make_inputs(2, 2, N, 256, causal=causal, seed=950 + N + int(causal)))


@pytest.mark.parametrize("causal", [False, True])
def test_d256_key_lengths_outside_zero_to_n(cuda_device, causal):
    # kv_len values are taken clamped into [0, N]: -3 leaves batch 0 without keys
    from gpu_helpers import f64
    N = 384
    x = inputs.make_inputs(2, 2, N, 256, causal=causal, seed=960 + int(causal),
                           kv_len=torch.tensor([-3, N + 5], dtype=torch.int32))
    res, out = check_all_heads(x)
    assert np.all(f64(out["o"])[0] == 0) and np.all(np.isneginf(f64(out["lse"])[0]))
    for name in ("dq", "dk", "dv"):
        assert np.all(f64(out[name])[0] == 0), name


def test_d256_block_mask_and_rows_without_keys(cuda_device):
    bm = inputs.draw_block_mask(5, 0.3, torch.Generator().manual_seed(920))
    bm[1, :] = 0  # query tile 1 sees no key tile
    x = inputs.make_inputs(2, 2, 600, 256, causal=True, seed=921, block_mask=bm,
                           kv_len=torch.tensor([600, 0], dtype=torch.int32))
    res, out = check_all_heads(x)
    from gpu_helpers import f64
    assert np.all(f64(out["o"])[:, :, 128:256] == 0)
    assert np.all(f64(out["o"])[1] == 0) and np.all(np.isneginf(f64(out["lse"])[1]))


def test_d256_tile_visits_match_the_mask(cuda_device):
    from gpu_helpers import run_gpu
    x = inputs.make_inputs(2, 1, 700, 256, causal=True, seed=930, block_keep=0.4,
                           kv_len=torch.tensor([700, 250], dtype=torch.int32))
    out = run_gpu(x, backward=True, traced=True)
    want = oracle.tile_visits(2, 700, True, x.block_mask.numpy(), x.kv_len.numpy())
    for name in ("vis_f", "vis_b"):
        got = out[name].cpu().numpy()[:, 0]
        assert np.array_equal(got, want), name


def test_d256_backward_is_bitwise_reproducible(cuda_device):
    # every gradient is summed in a fixed order on chip: fa_bwd repeats itself bit for
    # bit and equals fa_bwd_deterministic
    from gpu_helpers import to_dev
    x = inputs.make_inputs(1, 3, 512, 256, causal=True, seed=940)
    q, k, v, do, bm, kl = to_dev(x)
    o, lse = binding.attention_forward(q, k, v, x.scale, True)
    a = binding.attention_backward(q, k, v, o, lse, do, x.scale, True)
    b = binding.attention_backward(q, k, v, o, lse, do, x.scale, True)
    c = binding.attention_backward(q, k, v, o, lse, do, x.scale, True, deterministic=True)
    torch.cuda.synchronize()
    assert binding.fa_get_device_status() == 0
    for ta, tb, tc in zip(a, b, c):
        assert torch.equal(ta, tb) and torch.equal(ta, tc)
