"""CPU tests of bench.py's host-side helpers (no GPU)."""
import os
import sys

import torch

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))

import bench  # noqa: E402
from exact_io_aware_63_b200 import inputs  # noqa: E402


def _allowed_by_definition(x):
    """Element by element from the mask definition: causal (c <= r), key padding
    (c < kv_len[b]) and the 128 x 128 block mask, combined by AND."""
    B, H, N, d = x.q.shape
    out = torch.zeros((B, N, N), dtype=torch.bool)
    for b in range(B):
        for r in range(N):
            for c in range(N):
                ok = True
                if x.causal and c > r:
                    ok = False
                if x.kv_len is not None and c >= int(x.kv_len[b]):
                    ok = False
                if x.block_mask is not None and not bool(x.block_mask[r // 128, c // 128]):
                    ok = False
                out[b, r, c] = ok
    return out


def test_standard_attention_mask_matches_the_definition():
    x = inputs.make_inputs(2, 1, 256, 64, causal=True, seed=7, key_padding=(100, 256),
                           block_keep=0.5)
    got = bench.standard_allowed(x, torch.device("cpu"))
    want = _allowed_by_definition(x)
    assert torch.equal(got.expand(2, 1, 256, 256)[:, 0], want)


def test_standard_attention_mask_without_masks_is_all_true():
    x = inputs.make_inputs(1, 1, 128, 64, seed=3)
    got = bench.standard_allowed(x, torch.device("cpu"))
    assert bool(got.all())
