"""fa_bwd_noalloc: the backward pass for callers that cannot allocate device memory.

Such callers (for example a plugin whose host application hands it only its
input and output buffers, or a deployment that forbids device allocations
after start-up) cannot provide fa_bwd's workspace.  fa_bwd_noalloc uses a
fixed-size static buffer inside the library instead.  These tests check,
through the C ABI, that it returns what fa_bwd returns, on two calls in a
row (the second call finds the first call's data in the shared buffer), and
that shapes too large for the buffer are refused before anything runs.

This file is named to be collected last.
"""

import numpy as np
import pytest
import torch

import oracle
from exact_io_aware_63_b200 import binding, inputs
from gpu_helpers import compare_grads, f64, head_slices, rel_l2, to_dev

# dK and dV come from the same kernels on the same inputs, each row accumulated by one
# CTA in a fixed order: the same bits.  dQ is summed by reduce-adds whose order varies
# from run to run: equal up to float32 reordering, far inside this bound.
DQ_TOL = 2e-3


def test_refuses_shapes_beyond_the_static_buffer():
    # d = 128 needs 520 bytes of scratch per row: 2^18 rows is about 130 MiB > 64 MiB.
    # Fake, aligned pointers: the size check comes before any pointer is used.
    P = 1 << 40
    rc = binding.load().fa_bwd_noalloc(P, P, P, P, P, P, P, P, P, 1, 16, 16384, 128, 0.088, 0,
                                       None, None, None)
    assert rc == -9
    assert "FA_BWD_NOALLOC_SCRATCH_BYTES" in binding.fa_status_string(rc)
    assert binding.fa_bwd_workspace_size(1, 16, 16384, 128) > binding.BWD_NOALLOC_SCRATCH_BYTES


@pytest.mark.gpu
@pytest.mark.parametrize("name,shape,causal,pad", [
    ("bert", None, False, False),
    ("gpt2", None, True, False),
    ("small d128", (2, 3, 640, 128), True, True),
])
def test_matches_fa_bwd_on_two_calls_in_a_row(cuda_device, name, shape, causal, pad):
    if shape is None:
        x = inputs.workload_inputs(name)
    else:
        B, H, N, d = shape
        kv = torch.tensor([300, 640], dtype=torch.int32) if pad else None
        x = inputs.make_inputs(B, H, N, d, causal=causal, seed=77, kv_len=kv)
    q, k, v, do, bm, kl = to_dev(x)
    B, H, N, d = q.shape
    o, lse = binding.attention_forward(q, k, v, x.scale, x.causal, bm, kl)
    ref = binding.attention_backward(q, k, v, o, lse, do, x.scale, x.causal, bm, kl)
    for call in range(2):
        dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
        rc = binding.fa_bwd_noalloc(q, k, v, o, lse, do, dq, dk, dv, B, H, N, d, x.scale,
                                    x.causal, bm, kl)
        assert rc == 0, binding.fa_status_string(rc)
        torch.cuda.synchronize()
        assert binding.fa_get_device_status() == 0
        assert torch.equal(dk, ref[1]), f"{name} call {call}: dK differs from fa_bwd's"
        assert torch.equal(dv, ref[2]), f"{name} call {call}: dV differs from fa_bwd's"
        e = rel_l2(f64(dq), f64(ref[0]))
        assert e <= DQ_TOL, f"{name} call {call}: dQ rel-L2 {e:.3e} vs fa_bwd"
    if shape is not None:
        # the last call's gradients against the FP64 oracle, every head
        heads = [(b, h) for b in range(B) for h in range(H)]
        hq, hk, hv, hdo, hbm, hkl = head_slices(x, heads)
        rdq, rdk, rdv, _ = oracle.attention_backward(hq, hk, hv, hdo, x.scale, x.causal, hbm, hkl)
        pick = lambda t: np.stack([f64(t[b, h]) for b, h in heads])[:, None]
        compare_grads({"dq": pick(dq), "dk": pick(dk), "dv": pick(dv)},
                      {"dq": rdq, "dk": rdk, "dv": rdv}, f"{name} vs oracle")
