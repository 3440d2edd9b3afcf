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

import pytest
import torch

from exact_io_aware_63_b200 import binding, inputs
from gpu_helpers import GRAD_TOL, rel_l2, f64, to_dev


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
        for got, want, nm in zip((dq, dk, dv), ref, ("dq", "dk", "dv")):
            e = rel_l2(f64(got), f64(want))
            assert e <= GRAD_TOL, f"{name} call {call}: {nm} rel-L2 {e:.3e} vs fa_bwd"
