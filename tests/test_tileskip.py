"""The tiles the kernels compute are exactly the tiles holding an allowed entry.

The forward and backward kernels record every (query tile, key tile) pair
whose scores they form; the oracle derives the same set by brute force from
the mask definition.  The two must match bit for bit."""

import numpy as np
import pytest
import torch

import oracle
from exact_io_aware_63_b200 import inputs
from gpu_helpers import run_gpu

pytestmark = pytest.mark.gpu


def expected_visits(x, i_begin=0, i_end=None):
    B, H, N, _ = x.q.shape
    bm = None if x.block_mask is None else x.block_mask.numpy()
    kl = None if x.kv_len is None else x.kv_len.numpy()
    vis = oracle.tile_visits(B, N, x.causal, bm, kl, i_begin=i_begin, i_end=i_end)
    return np.repeat(vis[:, None], H, axis=1)


def check(x, band=None):
    out = run_gpu(x, backward=True, traced=True)
    vf, vb = out["vis_f"].cpu().numpy(), out["vis_b"].cpu().numpy()
    if band is None:
        exp = expected_visits(x)
    else:
        exp = expected_visits(x, *band)
        vf, vb = vf[:, :, band[0]:band[1]], vb[:, :, band[0]:band[1]]
    assert np.array_equal(vf, exp), f"forward visits differ at {np.argwhere(vf != exp)[:5]}"
    assert np.array_equal(vb, exp), f"backward visits differ at {np.argwhere(vb != exp)[:5]}"
    return exp


@pytest.mark.parametrize("causal", [False, True])
def test_masks_small(cuda_device, causal):
    x = inputs.make_inputs(3, 2, 896, 64, causal=causal, seed=31, block_keep=0.25,
                           kv_len=torch.tensor([1, 300, 896], dtype=torch.int32))
    check(x)


@pytest.mark.parametrize("causal", [False, True])
def test_masks_partial_last_tile(cuda_device, causal):
    # N = 700: five full tiles and a partial sixth
    x = inputs.make_inputs(3, 2, 700, 64, causal=causal, seed=33, block_keep=0.3,
                           kv_len=torch.tensor([1, 641, 700], dtype=torch.int32))
    check(x)


@pytest.mark.parametrize("name", ["bert", "gpt2"])
def test_workloads(cuda_device, name):
    check(inputs.workload_inputs(name))


def test_long_causal(cuda_device):
    x = inputs.workload_inputs("long16k_causal")
    exp = check(x)
    n_t = x.q.shape[2] // 128
    assert exp[0, 0].sum() == n_t * (n_t + 1) // 2


def test_block_sparse_64k(cuda_device):
    x = inputs.workload_inputs("sparse64k")
    check(x, band=(0, 24))
    check_tail = (488, 512)
    check(x, band=check_tail)
