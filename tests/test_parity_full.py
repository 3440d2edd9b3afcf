"""CUDA path vs the FP64 oracle on the five workloads at full size, in the launch
configuration the benchmark times (one fa_fwd and one fa_bwd call over the whole
batch).

BERT- and GPT-2-shaped workloads: every output of a seeded sample of heads.
16K and 64K workloads, and the 16K ones at head dimension 256 (too large for the
oracle's full backward): O and LSE on sampled rows of every head, dQ on sampled
rows of two heads, and dK, dV on sampled key columns of one head.
"""

import numpy as np
import pytest

import oracle
from exact_io_aware_63_b200 import inputs
from gpu_helpers import (GRAD_TOL, check_all_heads, compare_forward, dq_edge_bound, f64,
                         rel_l2, run_gpu)

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
    check_long_sampled(inputs.workload_inputs(name), name)


@pytest.mark.parametrize("name", ["long16k", "long16k_causal"])
def test_long_workloads_at_head_dimension_256_sampled(cuda_device, name):
    # the 16K workloads' kind of inputs at d = 256 (B=1 H=16 N=16384), the size the
    # benchmark times for head dimension 256
    w = inputs.WORKLOADS[name]
    x = inputs.make_inputs(1, 16, 16384, 256, causal=w.causal, seed=w.seed)
    check_long_sampled(x, f"{name} d=256")


def check_long_sampled(x, name):
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
    # backward: dQ on sampled rows of two heads.  The tolerance is a relative L2 error
    # of the whole tensor: random rows estimate it.  Rows at the edges (few keys under a
    # causal mask) are checked element by element against the bound that D taken from
    # the bf16 O implies (see dq_edge_bound).
    dq_gpu = out["dq"]
    for (b, h) in [(0, 0), (B - 1, H - 1)]:
        rows = np.sort(np.random.default_rng(7 + h).choice(N, size=48, replace=False))
        dq_ref, _ = oracle.attention_backward_dq_rows(
            f64(x.q[b, h, rows]), f64(x.dout[b, h, rows]), rows, f64(x.k[b, h]), f64(x.v[b, h]),
            x.scale, x.causal, bm, None)
        e = rel_l2(f64(dq_gpu[b, h, rows]), dq_ref)
        assert e <= GRAD_TOL, f"{name} dQ rows rel-L2 {e:.3e}"
        edge = np.array(sorted({0, 1, 127, 128, N - 1}))
        q_e, do_e = f64(x.q[b, h, edge]), f64(x.dout[b, h, edge])
        k, v = f64(x.k[b, h]), f64(x.v[b, h])
        dq_e, _ = oracle.attention_backward_dq_rows(q_e, do_e, edge, k, v, x.scale, x.causal, bm,
                                                    None)
        o_e, _ = oracle.attention_forward_rows(q_e, edge, k, v, x.scale, x.causal, bm, None)
        pk_abs, _ = oracle.attention_forward_rows(q_e, edge, k, np.abs(k), x.scale, x.causal, bm,
                                                  None)
        bound = dq_edge_bound(do_e, f64(o_gpu[b, h, edge]), o_e, pk_abs, dq_e, x.scale,
                              float(np.abs(v).max()))
        err = np.abs(f64(dq_gpu[b, h, edge]) - dq_e)
        if np.any(err > bound):
            i = np.unravel_index(np.argmax(err - bound), err.shape)
            raise AssertionError(f"{name} dQ row {edge[i[0]]}: error {err[i]:.3e} > bound "
                                 f"{bound[i]:.3e}")
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
