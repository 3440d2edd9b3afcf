"""fa_bwd_deterministic: the ordered dQ kernel against the FP64 oracle, element by
element on every head, and bitwise reproducibility across repeated calls."""

import numpy as np
import pytest
import torch

import oracle
from exact_io_aware_63_b200 import binding, inputs
from gpu_helpers import GRAD_TOL, compare_grads, f64, head_slices, to_dev

pytestmark = pytest.mark.gpu


def _det_backward(x, runs=1):
    q, k, v, do, bm, kl = to_dev(x)
    o, lse = binding.attention_forward(q, k, v, x.scale, x.causal, bm, kl)
    outs = [binding.attention_backward(q, k, v, o, lse, do, x.scale, x.causal, bm, kl,
                                       deterministic=True) for _ in range(runs)]
    torch.cuda.synchronize()
    status = binding.fa_get_device_status()
    assert status == 0, binding.fa_status_string(status)
    return outs


def _check_against_oracle(x):
    (dq, dk, dv), = _det_backward(x)
    B, H = x.q.shape[:2]
    heads = [(b, h) for b in range(B) for h in range(H)]
    q, k, v, do, bm, kl = head_slices(x, heads)
    rq, rk, rv, _ = oracle.attention_backward(q, k, v, do, x.scale, x.causal, bm, kl)
    pick = lambda t: np.stack([f64(t[b, h]) for b, h in heads])[:, None]
    compare_grads({"dq": pick(dq), "dk": pick(dk), "dv": pick(dv)},
                  {"dq": rq, "dk": rk, "dv": rv}, "deterministic backward")


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
def test_dense_against_oracle(cuda_device, d, causal):
    _check_against_oracle(inputs.make_inputs(2, 2, 384, d, causal=causal, seed=300 + d))


@pytest.mark.parametrize("d", [64, 128])
def test_key_padding_against_oracle(cuda_device, d):
    # a single key, a length inside a tile, a tile edge, the full length, and no key
    x = inputs.make_inputs(5, 1, 512, d, seed=310 + d,
                           kv_len=torch.tensor([1, 200, 256, 512, 0], dtype=torch.int32))
    _check_against_oracle(x)


@pytest.mark.parametrize("d", [64, 128])
def test_partial_last_tile_against_oracle(cuda_device, d):
    _check_against_oracle(inputs.make_inputs(2, 2, 300, d, causal=True, seed=330 + d))


def test_block_mask_against_oracle(cuda_device):
    x = inputs.make_inputs(1, 2, 1024, 64, seed=320, block_keep=0.25)
    _check_against_oracle(x)


@pytest.mark.parametrize("name", ["bert", "gpt2"])
def test_bitwise_reproducible_on_workloads(cuda_device, name):
    x = inputs.workload_inputs(name)
    runs = _det_backward(x, runs=3)
    for r in runs[1:]:
        for a, b in zip(runs[0], r):
            assert torch.equal(a, b)


def test_agrees_with_the_atomic_backward(cuda_device):
    x = inputs.workload_inputs("gpt2")
    q, k, v, do, bm, kl = to_dev(x)
    o, lse = binding.attention_forward(q, k, v, x.scale, x.causal, bm, kl)
    det = binding.attention_backward(q, k, v, o, lse, do, x.scale, x.causal, bm, kl,
                                     deterministic=True)
    ato = binding.attention_backward(q, k, v, o, lse, do, x.scale, x.causal, bm, kl)
    # dK and dV come from the same kernel either way
    assert torch.equal(det[1], ato[1]) and torch.equal(det[2], ato[2])
    # each dQ is within GRAD_TOL (relative L2) of the exact one (the oracle tests
    # above and in test_parity.py), so by the triangle inequality they differ by
    # at most 2 * GRAD_TOL relative to the exact norm; the kernels round P and dS
    # to bf16 independently, so their difference is of the size of that rounding
    rel = float((det[0].float() - ato[0].float()).norm() / ato[0].float().norm())
    assert rel < 2 * GRAD_TOL, rel
