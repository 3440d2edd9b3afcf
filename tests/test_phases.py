"""fa_bwd_phase: the backward's launches one at a time, as callers that time or
schedule them separately use them (the benchmark does).

The header promises that phases 0, 1, 2 called in order on one stream with the
same arguments and workspace are exactly fa_bwd, and that 0, 1, 3 are exactly
fa_bwd_deterministic.  These tests hold the library to that through the C ABI:
dK and dV (one CTA owns each key tile and sums it in a fixed order) and the
ordered dQ must be the same bits; fa_bwd's dQ is summed by reduce-adds whose
order varies between runs, so it is compared within float32 reordering.
A workspace filled with garbage before each call checks that no phase relies
on what an earlier call left behind.
"""

import pytest
import torch

from exact_io_aware_63_b200 import binding, inputs
from gpu_helpers import f64, rel_l2, to_dev

DQ_TOL = 2e-3  # float32 reordering of the dQ reduce-adds, far inside this bound


def _case(shape, causal, kv, sparse):
    B, H, N, d = shape
    kvt = torch.tensor(kv, dtype=torch.int32) if kv is not None else None
    return inputs.make_inputs(B, H, N, d, causal=causal, seed=91, kv_len=kvt,
                              block_keep=0.5 if sparse else None)


def _garbage_workspace(nbytes, dev):
    ws = torch.empty(nbytes, dtype=torch.uint8, device=dev)
    ws.fill_(0xA5)  # neither zero nor a valid float pattern of interest
    return ws


@pytest.mark.gpu
@pytest.mark.parametrize("shape,causal,kv,sparse", [
    ((2, 3, 300, 64), False, [300, 170], False),  # key padding, partial last tile
    ((1, 4, 512, 64), True, None, True),          # causal and a block mask
    ((2, 2, 384, 128), True, [384, 200], False),
    ((1, 2, 256, 256), True, None, False),        # the three-pass d = 256 backward
])
def test_phases_in_order_are_the_whole_call(cuda_device, shape, causal, kv, sparse):
    x = _case(shape, causal, kv, sparse)
    q, k, v, do, bm, kl = to_dev(x)
    B, H, N, d = q.shape
    o, lse = binding.attention_forward(q, k, v, x.scale, x.causal, bm, kl)
    ws_bytes = binding.fa_bwd_workspace_size(B, H, N, d)
    for det in (False, True):
        whole = [torch.empty_like(t) for t in (q, k, v)]
        ws = _garbage_workspace(ws_bytes, q.device)
        fn = binding.fa_bwd_deterministic if det else binding.fa_bwd
        rc = fn(q, k, v, o, lse, do, *whole, B, H, N, d, x.scale, x.causal, bm, kl, ws, ws_bytes)
        assert rc == 0, binding.fa_status_string(rc)

        parts = [torch.empty_like(t) for t in (q, k, v)]
        ws = _garbage_workspace(ws_bytes, q.device)
        for ph in ((0, 1, 3) if det else (0, 1, 2)):
            rc = binding.fa_bwd_phase(ph, q, k, v, o, lse, do, *parts, B, H, N, d, x.scale,
                                      x.causal, bm, kl, ws, ws_bytes)
            assert rc == 0, f"phase {ph}: {binding.fa_status_string(rc)}"
        torch.cuda.synchronize()
        assert binding.fa_get_device_status() == 0
        label = f"{shape} {'ordered' if det else 'fa_bwd'}"
        assert torch.equal(parts[1], whole[1]), f"{label}: dK differs"
        assert torch.equal(parts[2], whole[2]), f"{label}: dV differs"
        if det or d == 256:
            # the ordered dQ (and the d = 256 dQ pass, summed on chip) is the same bits
            assert torch.equal(parts[0], whole[0]), f"{label}: dQ differs"
        else:
            e = rel_l2(f64(parts[0]), f64(whole[0]))
            assert e <= DQ_TOL, f"{label}: dQ rel-L2 {e:.3e}"
