"""CUDA path vs the FP64 oracle on the five workloads at full size, in the launch
configuration the benchmark times (one fa_fwd and one fa_bwd call over the whole
batch).

BERT- and GPT-2-shaped workloads: every output of a seeded sample of heads.
16K and 64K workloads (too large for the oracle's full backward): O and LSE on
sampled rows of every head, dQ on sampled rows of two heads, and dK, dV on
sampled key columns of one head.
"""

import numpy as np
import pytest

import oracle
from exact_io_aware_63_b200 import inputs
from gpu_helpers import GRAD_TOL, check_all_heads, compare_forward, f64, rel_l2, run_gpu

pytestmark = pytest.mark.gpu


def sample_heads(B, H, n, seed):
    rng = np.random.default_rng(seed)
    allh = [(b, h) for b in range(B) for h in range(H)]
    idx = rng.choice(len(allh), size=min(n, len(allh)), replace=False)
    return sorted(allh[i] for i in idx)


@pytest.mark.parametrize("name", ["tiny", "bert", "gpt2"])
def test_full_workload_sampled_heads(cuda_device, name):
    x = inputs.workload_inputs(name)
    B, H = x.q.shape[:2]
    check_all_heads(x, heads=sample_heads(B, H, 12, 5))


def sampled_rows(N, n, seed):
    rng = np.random.default_rng(seed)
    rows = rng.choice(N, size=n, replace=False)
    return np.sort(np.concatenate([rows, [0, 1, 127, 128, N - 1]]))


@pytest.mark.parametrize("name", ["long16k", "long16k_causal", "sparse64k"])
def test_long_workloads_sampled(cuda_device, name):
    x = inputs.workload_inputs(name)
    B, H, N, d = x.q.shape
    out = run_gpu(x)
    bm = None if x.block_mask is None else x.block_mask.numpy()
    o_gpu, lse_gpu = out["o"], out["lse"]
    # forward: sampled rows of every head
    for b in range(B):
        kl = None if x.kv_len is None else int(x.kv_len[b])
        for h in range(H):
            rows = sampled_rows(N, 24, 100 * b + h)
            k = f64(x.k[b, h]); v = f64(x.v[b, h])
            o_ref, lse_ref = oracle.attention_forward_rows(f64(x.q[b, h, rows]), rows, k, v,
                                                           x.scale, x.causal, bm, kl)
            compare_forward(f64(o_gpu[b, h, rows]), f64(lse_gpu[b, h, rows]), o_ref, lse_ref,
                            f"{name} head ({b},{h})")
    # backward: dQ and D on sampled rows of two heads
    dq_gpu = out["dq"]
    for (b, h) in [(0, 0), (B - 1, H - 1)]:
        rows = sampled_rows(N, 48, 7 + h)
        dq_ref, _ = oracle.attention_backward_dq_rows(
            f64(x.q[b, h, rows]), f64(x.dout[b, h, rows]), rows, f64(x.k[b, h]), f64(x.v[b, h]),
            x.scale, x.causal, bm, None)
        e = rel_l2(f64(dq_gpu[b, h, rows]), dq_ref)
        assert e <= GRAD_TOL, f"{name} dQ rows rel-L2 {e:.3e}"
    # backward: dK and dV on sampled key columns of the first head (a full pass over
    # its rows in the oracle)
    b, h = 0, 0
    cols = sampled_rows(N, 12, 11)
    dk_ref, dv_ref = oracle.attention_backward_kv_cols(
        f64(x.q[b, h]), f64(x.k[b, h]), f64(x.v[b, h]), f64(x.dout[b, h]), cols, x.scale,
        x.causal, bm, None)
    for nm, got, ref in (("dK", out["dk"], dk_ref), ("dV", out["dv"], dv_ref)):
        e = rel_l2(f64(got[b, h, cols]), ref)
        assert e <= GRAD_TOL, f"{name} {nm} columns rel-L2 {e:.3e}"
