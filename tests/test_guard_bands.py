"""Every output (and the backward workspace) sits inside a larger buffer filled with a
sentinel; after a forward and a backward pass the bytes around each output must be
untouched.  Covers partial last tiles, key padding, causal masks, both head dimensions,
dropout and the deterministic backward."""

import pytest
import torch

from exact_io_aware_63_b200 import binding, inputs

pytestmark = pytest.mark.gpu

DEV = torch.device("cuda", 0)
GUARD = 4096  # elements before and after each output
SENTINEL = -12288.0  # exact in bfloat16 and float32


def _guarded(n, dtype):
    buf = torch.full((n + 2 * GUARD,), SENTINEL, dtype=dtype, device=DEV)
    return buf, buf[GUARD:GUARD + n]


def _untouched(buf, n):
    return bool((buf[:GUARD].float() == SENTINEL).all()) and \
        bool((buf[GUARD + n:].float() == SENTINEL).all())


@pytest.mark.parametrize("d", [32, 64, 96, 128])
@pytest.mark.parametrize("mode", ["plain", "dropout", "deterministic"])
def test_outputs_and_workspace_keep_their_bounds(cuda_device, d, mode):
    x = inputs.make_inputs(2, 2, 300, d, causal=True, seed=700 + d,
                           kv_len=torch.tensor([300, 171], dtype=torch.int32))
    B, H, N, _ = x.q.shape
    E, R = B * H * N * d, B * H * N
    q, k, v, do = (t.to(DEV).contiguous() for t in (x.q, x.k, x.v, x.dout))
    kl = x.kv_len.to(DEV)
    bufs = {n: _guarded(E, torch.bfloat16) for n in ("o", "dq", "dk", "dv")}
    lse_buf, lse = _guarded(R, torch.float32)
    ws_bytes = binding.fa_bwd_workspace_size(B, H, N, d)
    # the workspace view keeps 256-byte alignment: GUARD bytes before it
    ws_buf = torch.full((ws_bytes + 2 * GUARD,), 0x5A, dtype=torch.uint8, device=DEV)
    ws = ws_buf[GUARD:GUARD + ws_bytes]
    o, dq, dk, dv = (bufs[n][1] for n in ("o", "dq", "dk", "dv"))
    if mode == "dropout":
        rc = binding.fa_fwd_dropout(q, k, v, o, lse, B, H, N, d, x.scale, True, None, kl, 0.2,
                                    11, 3)
    else:
        rc = binding.fa_fwd(q, k, v, o, lse, B, H, N, d, x.scale, True, None, kl)
    assert rc == 0
    if mode == "dropout":
        rc = binding.fa_bwd_dropout(q, k, v, o, lse, do, dq, dk, dv, B, H, N, d, x.scale, True,
                                    None, kl, 0.2, 11, 3, ws, ws_bytes)
    elif mode == "deterministic":
        rc = binding.fa_bwd_deterministic(q, k, v, o, lse, do, dq, dk, dv, B, H, N, d, x.scale,
                                          True, None, kl, ws, ws_bytes)
        if d not in (64, 128):
            assert rc == -4  # the ordered dQ takes 64 and 128 only; nothing was launched
            torch.cuda.synchronize()
            for name in ("o",):
                assert _untouched(bufs[name][0], E), name
            return
    else:
        rc = binding.fa_bwd(q, k, v, o, lse, do, dq, dk, dv, B, H, N, d, x.scale, True, None, kl,
                            ws, ws_bytes)
    assert rc == 0
    torch.cuda.synchronize()
    assert binding.fa_get_device_status() == 0
    for name, (buf, _) in bufs.items():
        assert _untouched(buf, E), name
    assert _untouched(lse_buf, R), "lse"
    assert bool((ws_buf[:GUARD] == 0x5A).all()) and bool((ws_buf[GUARD + ws_bytes:] == 0x5A).all())
    # and every output element was written (no sentinel left inside)
    for name, (_, view) in bufs.items():
        assert not bool((view.float() == SENTINEL).any()), name
