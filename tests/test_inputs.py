"""CPU tests of the seeded input generators shared by the kernels' tests, the oracle and
bench.py: they draw what their docstrings and the workload table say, reproducibly."""

import math

import torch

from exact_io_aware_63_b200 import inputs


def test_same_seed_same_tensors_other_seed_other_tensors():
    a = inputs.make_inputs(1, 2, 256, 64, seed=1)
    b = inputs.make_inputs(1, 2, 256, 64, seed=1)
    c = inputs.make_inputs(1, 2, 256, 64, seed=2)
    for n in ("q", "k", "v", "dout"):
        assert torch.equal(getattr(a, n), getattr(b, n))
        assert not torch.equal(getattr(a, n), getattr(c, n))
        assert getattr(a, n).dtype == torch.bfloat16


def test_values_are_standard_normal_rounded_to_bf16():
    x = inputs.make_inputs(4, 4, 512, 64, seed=3)
    v = x.q.float()
    n = v.numel()
    assert abs(float(v.mean())) < 5 / math.sqrt(n)
    assert abs(float(v.std()) - 1.0) < 0.01
    # bf16 values: the low 16 bits of the float32 pattern are zero
    bits = v.view(torch.int32)
    assert bool(((bits & 0xFFFF) == 0).all())


def test_key_lengths_are_uniform_on_the_stated_integers():
    gen = torch.Generator().manual_seed(4)
    kl = inputs.draw_kv_len(20000, 512, 256, 512, gen)
    assert kl.dtype == torch.int32
    assert int(kl.min()) == 256 and int(kl.max()) == 512
    counts = torch.bincount(kl.long() - 256, minlength=257).double()
    e = 20000 / 257
    chi2 = float(((counts - e) ** 2 / e).sum())
    assert abs(chi2 - 256) < 5 * math.sqrt(2 * 256)


def test_block_mask_keeps_the_diagonal_and_the_stated_share():
    gen = torch.Generator().manual_seed(5)
    n_t = 64
    m = inputs.draw_block_mask(n_t, 1.0 / 16.0, gen)
    assert bool(torch.diagonal(m).bool().all())
    n_off = n_t * n_t - n_t
    assert int(m.sum()) - n_t == round(n_off / 16)


def test_sparse64k_workload_mask():
    # the block-sparse workload: 512 x 512 tiles, diagonal plus 1/16 of the rest
    x = inputs.workload_inputs("sparse64k")
    m = x.block_mask
    assert m.shape == (512, 512)
    assert bool(torch.diagonal(m).bool().all())
    assert int(m.sum()) == 16864


def test_bert_workload_key_lengths():
    x = inputs.workload_inputs("bert")
    assert x.kv_len.shape == (16,)
    assert int(x.kv_len.min()) >= 256 and int(x.kv_len.max()) <= 512


def test_packed_inputs_offsets_and_shapes():
    x = inputs.make_packed_inputs([5, 0, 130], 3, 32, seed=6, causal=True)
    assert x.cu_seqlens.tolist() == [0, 5, 5, 135]
    assert x.q.shape == (135, 3, 32) and x.dout.shape == (135, 3, 32)
    assert x.max_seqlen == 130 and x.lengths == [5, 0, 130]
    assert x.causal and abs(x.scale - 1 / math.sqrt(32)) < 1e-12
    assert inputs.draw_lengths(4, 10, 20, seed=7) == inputs.draw_lengths(4, 10, 20, seed=7)
    assert all(10 <= n <= 20 for n in inputs.draw_lengths(100, 10, 20, seed=8))


def test_workload_table_matches_the_stated_configurations():
    # (B, H, N, d), scale, causal, key padding, block-sparse for each named workload
    want = {
        "tiny": ((1, 1, 128, 64), 1 / 8, False, False, False),
        "bert": ((16, 16, 512, 64), 1 / 8, False, True, False),
        "gpt2": ((8, 12, 1024, 64), 1 / 8, True, False, False),
        "long16k": ((1, 16, 16384, 128), 1 / math.sqrt(128), False, False, False),
        "long16k_causal": ((1, 16, 16384, 128), 1 / math.sqrt(128), True, False, False),
        "sparse64k": ((1, 8, 65536, 64), 1 / 8, False, False, True),
    }
    assert set(inputs.WORKLOADS) == set(want)
    for name, (shape, scale, causal, padding, sparse) in want.items():
        w = inputs.WORKLOADS[name]
        assert (w.B, w.H, w.N, w.d) == shape, name
        assert abs(w.scale - scale) < 1e-15 and w.causal == causal, name
        assert w.key_padding == padding and w.block_sparse == sparse, name
    # the two 16K workloads draw the same tensors; the others each have their own seed
    assert inputs.WORKLOADS["long16k"].seed == inputs.WORKLOADS["long16k_causal"].seed
    seeds = [w.seed for n, w in inputs.WORKLOADS.items() if n != "long16k_causal"]
    assert len(set(seeds)) == len(seeds)


def test_tiny_workload_tensors():
    x = inputs.workload_inputs("tiny")
    assert x.q.shape == (1, 1, 128, 64) and x.q.dtype == torch.bfloat16
    assert x.kv_len is None and x.block_mask is None and not x.causal
    assert abs(x.scale - 0.125) < 1e-15
