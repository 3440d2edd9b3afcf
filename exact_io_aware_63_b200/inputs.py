"""Seeded synthetic inputs shaped like the pages' attention workloads.

This module holds no attention arithmetic.  It only draws tensors and masks,
so that the CUDA path and the FP64 oracle can be fed the very same values.

Workloads ("FlashAttention, Decoded", abstract and its gloss: BERT-large at
sequence length 512, GPT-2 at 1K, Path-X at 16K and Path-256 at 64K with
block-sparse attention).  No dataset is used: every tensor is i.i.d. N(0, 1)
drawn in float32 from ``torch.Generator`` and rounded to bfloat16
(round-to-nearest-even), in the order q, k, v, dO; then the key lengths or the
block mask are drawn from the same generator.

* ``tiny``:            B=1  H=1  N=128   d=64,  scale 1/8, no mask.
* ``bert``:            B=16 H=16 N=512   d=64,  scale 1/8, key padding with
                       kv_len[b] uniform on the integers 256..512.
* ``gpt2``:            B=8  H=12 N=1024  d=64,  scale 1/8, causal.
* ``long16k``:         B=1  H=16 N=16384 d=128, scale 1/sqrt(128), no mask.
* ``long16k_causal``:  the same tensors, causal.
* ``sparse64k``:       B=1  H=8  N=65536 d=64,  scale 1/8, a 128x128 tile mask
                       shared by all heads: every diagonal tile kept plus
                       round(n_off/16) off-diagonal tiles chosen uniformly
                       without replacement (a seeded permutation).
"""

from __future__ import annotations

import dataclasses
import math
from typing import Optional

import torch

TILE = 128


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    N: int
    d: int
    scale: float
    causal: bool = False
    key_padding: bool = False
    block_sparse: bool = False
    seed: int = 1000
    description: str = ""


WORKLOADS = {
    w.name: w
    for w in [
        Workload("tiny", 1, 1, 128, 64, 1.0 / 8.0, seed=1000,
                 description="exact attention B=1 H=1 N=128 d=64, no mask"),
        Workload("bert", 16, 16, 512, 64, 1.0 / 8.0, key_padding=True, seed=1001,
                 description="BERT-large-shaped B=16 H=16 N=512 d=64, key padding "
                             "kv_len ~ U{256..512}"),
        Workload("gpt2", 8, 12, 1024, 64, 1.0 / 8.0, causal=True, seed=1002,
                 description="GPT-2-shaped causal B=8 H=12 N=1024 d=64"),
        Workload("long16k", 1, 16, 16384, 128, 1.0 / math.sqrt(128.0), seed=1003,
                 description="long context B=1 H=16 N=16384 d=128, no mask"),
        Workload("long16k_causal", 1, 16, 16384, 128, 1.0 / math.sqrt(128.0), causal=True,
                 seed=1003, description="long context B=1 H=16 N=16384 d=128, causal"),
        Workload("sparse64k", 1, 8, 65536, 64, 1.0 / 8.0, block_sparse=True, seed=1004,
                 description="block-sparse B=1 H=8 N=65536 d=64, 128x128 tile mask: "
                             "diagonal + 1/16 of off-diagonal tiles"),
    ]
}


@dataclasses.dataclass
class Inputs:
    """Host (CPU) tensors; q, k, v, dout are bfloat16 [B, H, N, d]."""
    q: torch.Tensor
    k: torch.Tensor
    v: torch.Tensor
    dout: torch.Tensor
    scale: float
    causal: bool
    kv_len: Optional[torch.Tensor]      # int32 [B] or None
    block_mask: Optional[torch.Tensor]  # uint8 [ceil(N/128), ceil(N/128)] or None

    @property
    def shape(self):
        return tuple(self.q.shape)


def draw_kv_len(B: int, N: int, lo: int, hi: int, gen: torch.Generator) -> torch.Tensor:
    """kv_len[b] uniform on the integers lo..hi (inclusive), clipped to N."""
    u = torch.rand(B, generator=gen, dtype=torch.float64)
    lens = lo + torch.floor(u * (hi - lo + 1)).to(torch.int64)
    return lens.clamp(1, N).to(torch.int32)


def draw_block_mask(n_t: int, keep_fraction: float, gen: torch.Generator) -> torch.Tensor:
    """Diagonal tiles kept; exactly round(keep_fraction * n_off) off-diagonal tiles kept."""
    mask = torch.zeros(n_t, n_t, dtype=torch.uint8)
    idx = torch.arange(n_t)
    mask[idx, idx] = 1
    n_off = n_t * n_t - n_t
    n_keep = int(round(keep_fraction * n_off))
    perm = torch.randperm(n_off, generator=gen)[:n_keep]
    # off-diagonal entries enumerated row by row, skipping the diagonal
    i = perm // (n_t - 1)
    jj = perm % (n_t - 1)
    j = jj + (jj >= i).to(jj.dtype)
    mask[i, j] = 1
    return mask


def make_inputs(B: int, H: int, N: int, d: int, *, scale: Optional[float] = None,
                causal: bool = False, seed: int = 0, kv_len=None, block_mask=None,
                key_padding: Optional[tuple] = None, block_keep: Optional[float] = None,
                with_dout: bool = True) -> Inputs:
    """Draw q, k, v, dO ~ N(0,1) (float32 -> bfloat16) and the masks, from ``seed``.

    ``key_padding=(lo, hi)`` draws kv_len uniform on lo..hi; ``block_keep=f``
    draws a tile mask with the diagonal plus a fraction f of the other tiles.
    Explicit ``kv_len`` / ``block_mask`` tensors are used as given.
    """
    gen = torch.Generator().manual_seed(int(seed))
    shape = (B, H, N, d)

    def draw():
        return torch.randn(shape, generator=gen, dtype=torch.float32).to(torch.bfloat16)

    q, k, v = draw(), draw(), draw()
    dout = draw() if with_dout else torch.zeros(shape, dtype=torch.bfloat16)
    if kv_len is None and key_padding is not None:
        kv_len = draw_kv_len(B, N, key_padding[0], key_padding[1], gen)
    if block_mask is None and block_keep is not None:
        block_mask = draw_block_mask(-(-N // TILE), block_keep, gen)  # ceil(N / 128) tiles
    if kv_len is not None:
        kv_len = torch.as_tensor(kv_len, dtype=torch.int32).contiguous()
    if block_mask is not None:
        block_mask = torch.as_tensor(block_mask, dtype=torch.uint8).contiguous()
    return Inputs(q, k, v, dout, float(scale if scale is not None else 1.0 / math.sqrt(d)),
                  bool(causal), kv_len, block_mask)


def workload_inputs(name: str) -> Inputs:
    w = WORKLOADS[name]
    return make_inputs(w.B, w.H, w.N, w.d, scale=w.scale, causal=w.causal, seed=w.seed,
                       key_padding=(256, 512) if w.key_padding else None,
                       block_keep=(1.0 / 16.0) if w.block_sparse else None)


@dataclasses.dataclass
class PackedInputs:
    """A packed variable-length batch on the host: q, k, v, dout bfloat16 [T, H, d];
    sequence b is tokens cu_seqlens[b] .. cu_seqlens[b+1]-1."""
    q: torch.Tensor
    k: torch.Tensor
    v: torch.Tensor
    dout: torch.Tensor
    cu_seqlens: torch.Tensor  # int32 [B + 1]
    max_seqlen: int
    scale: float
    causal: bool

    @property
    def lengths(self):
        return [int(self.cu_seqlens[b + 1] - self.cu_seqlens[b])
                for b in range(len(self.cu_seqlens) - 1)]


def make_packed_inputs(lengths, H: int, d: int, *, scale: Optional[float] = None,
                       causal: bool = False, seed: int = 0) -> PackedInputs:
    """q, k, v, dO ~ N(0,1) (float32 -> bfloat16) for sequences of the given lengths,
    packed token by token ([T, H, d], T = sum of lengths), drawn in the order q, k, v, dO."""
    lengths = [int(n) for n in lengths]
    cu = torch.zeros(len(lengths) + 1, dtype=torch.int32)
    if lengths:
        cu[1:] = torch.cumsum(torch.tensor(lengths, dtype=torch.int64), 0).to(torch.int32)
    T = int(cu[-1])
    gen = torch.Generator().manual_seed(int(seed))
    shape = (T, H, d)

    def draw():
        return torch.randn(shape, generator=gen, dtype=torch.float32).to(torch.bfloat16)

    q, k, v, dout = draw(), draw(), draw(), draw()
    return PackedInputs(q, k, v, dout, cu, max(lengths) if lengths else 0,
                        float(scale if scale is not None else 1.0 / math.sqrt(d)), bool(causal))


def draw_lengths(B: int, lo: int, hi: int, seed: int):
    """B sequence lengths uniform on the integers lo..hi (inclusive), from ``seed``."""
    gen = torch.Generator().manual_seed(int(seed))
    u = torch.rand(B, generator=gen, dtype=torch.float64)
    return [int(x) for x in (lo + torch.floor(u * (hi - lo + 1))).to(torch.int64)]
