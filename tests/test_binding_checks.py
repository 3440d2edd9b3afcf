"""CPU tests of the binding's argument checks: the convenience wrappers refuse tensors whose
dtype, shape, layout or device the C ABI could not detect from raw pointers, before any
library call (so these run without a GPU)."""

import pytest
import torch

from exact_io_aware_63_b200 import binding

B, H, N, d = 2, 3, 300, 64
NT = 3  # ceil(300 / 128)


def _bf16(*shape):
    return torch.zeros(shape, dtype=torch.bfloat16)


def _dense():
    q, k, v = _bf16(B, H, N, d), _bf16(B, H, N, d), _bf16(B, H, N, d)
    return q, k, v


def _bwd_args():
    q, k, v = _dense()
    return dict(q=q, k=k, v=v, o=_bf16(B, H, N, d), lse=torch.zeros(B, H, N),
                dout=_bf16(B, H, N, d), scale=0.125)


def test_well_formed_host_tensors_reach_the_device_check():
    q, k, v = _dense()
    with pytest.raises(ValueError, match="CUDA"):
        binding.attention_forward(q, k, v, 0.125, block_mask=torch.ones(NT, NT, dtype=torch.uint8),
                                  kv_len=torch.full((B,), N, dtype=torch.int32))
    with pytest.raises(ValueError, match="CUDA"):
        binding.attention_backward(**_bwd_args())


@pytest.mark.parametrize("bad", ["dtype", "shape", "layout", "rank"])
def test_forward_refuses_malformed_q_k_v(bad):
    q, k, v = _dense()
    if bad == "dtype":
        k = k.half()
    elif bad == "shape":
        v = _bf16(B, H, N + 1, d)
    elif bad == "layout":
        k = _bf16(B, N, H, d).transpose(1, 2)  # right shape, not contiguous
    else:
        q = _bf16(B * H, N, d)
    with pytest.raises(ValueError) as e:
        binding.attention_forward(q, k, v, 0.125)
    assert "CUDA" not in str(e.value)


@pytest.mark.parametrize("name,value", [
    ("block_mask", torch.ones(NT, NT, dtype=torch.bool)),       # not uint8
    ("block_mask", torch.ones(N // 128, N // 128, dtype=torch.uint8)),  # floor, not ceil
    ("kv_len", torch.full((B,), N, dtype=torch.int64)),         # not int32
    ("kv_len", torch.full((B + 1,), N, dtype=torch.int32)),     # not [B]
])
def test_forward_refuses_malformed_masks(name, value):
    q, k, v = _dense()
    with pytest.raises(ValueError, match=name):
        binding.attention_forward(q, k, v, 0.125, **{name: value})


@pytest.mark.parametrize("name,value", [
    ("lse", torch.zeros(B, H, N, dtype=torch.float64)),
    ("lse", torch.zeros(B * H * N)),
    ("o", torch.zeros(B, H, N, d)),                              # float32, not bf16
    ("dout", _bf16(B, H, N, d + 32)),
])
def test_backward_refuses_malformed_saved_tensors(name, value):
    args = _bwd_args()
    args[name] = value
    with pytest.raises(ValueError, match=name):
        binding.attention_backward(**args)


def test_traced_calls_check_the_visit_record():
    q, k, v = _dense()
    with pytest.raises(ValueError, match="visited"):
        binding.attention_forward(q, k, v, 0.125, visited=torch.zeros(B, H, NT, NT))
    with pytest.raises(ValueError, match="visited"):
        binding.attention_backward(**_bwd_args(),
                                   visited=torch.zeros(B, H, NT, NT - 1, dtype=torch.uint8))


def test_packed_wrappers_check_their_layout():
    T = 40
    q, k, v = _bf16(T, H, d), _bf16(T, H, d), _bf16(T, H, d)
    cu = torch.tensor([0, 15, 40], dtype=torch.int32)
    with pytest.raises(ValueError, match="CUDA"):
        binding.attention_forward_varlen(q, k, v, cu, 25, 0.125)
    with pytest.raises(ValueError, match="cu_seqlens"):
        binding.attention_forward_varlen(q, k, v, cu.long(), 25, 0.125)
    with pytest.raises(ValueError, match="3-D"):
        binding.attention_forward_varlen(q[None], k, v, cu, 25, 0.125)
    o, do = _bf16(T, H, d), _bf16(T, H, d)
    with pytest.raises(ValueError, match="CUDA"):
        binding.attention_backward_varlen(q, k, v, o, torch.zeros(H, T), do, cu, 25, 0.125)
    # LSE of a packed batch is [H, T], not [T, H]
    with pytest.raises(ValueError, match="lse"):
        binding.attention_backward_varlen(q, k, v, o, torch.zeros(T, H), do, cu, 25, 0.125)
