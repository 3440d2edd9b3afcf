"""Pins the oracle's Philox-4x32-10 (the generator of the dropout keep mask) to an
independent implementation of the same published generator: cuRAND's host-side
CURAND_RNG_PSEUDO_PHILOX4_32_10, which runs on the CPU and needs no GPU.

cuRAND's host generator fills its output from 65536 streams: word j of the output is word
j % 4 of Philox-4x32-10(counter, key) with counter = (r mod 2^32, r div 2^32, t, 0),
r = j div 2^18, t = (j mod 2^18) div 4, and key = (low, high 32 bits of the seed).  A
generator offset of o starts the output at word o, so large offsets reach counter word 1.
Every output word checked below must equal the oracle's word for that counter and key:
counter words 0, 1, 2 and both key words take nonzero values.  Counter word 3 stays 0 in
every cuRAND stream; it enters the first round exactly as word 1 does (XORed with a high
product and a key word), and the dropout tests' offset checks cover it."""

import ctypes
import ctypes.util
import os

import numpy as np
import pytest

import oracle

PHILOX4_32_10 = 161  # curandRngType_t value of CURAND_RNG_PSEUDO_PHILOX4_32_10
STREAMS = 65536


def _curand():
    cands = [os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "lib64", "libcurand.so")]
    found = ctypes.util.find_library("curand")
    if found:
        cands.append(found)
    for path in cands:
        try:
            return ctypes.CDLL(path)
        except OSError:
            continue
    pytest.skip("cuRAND is not installed")


@pytest.fixture(scope="module")
def curand():
    lib = _curand()
    gen = ctypes.c_void_p()
    if lib.curandCreateGeneratorHost(ctypes.byref(gen), PHILOX4_32_10) != 0:
        pytest.skip("cuRAND host Philox generator unavailable")
    yield lib, gen
    lib.curandDestroyGenerator(gen)


def _draw(curand, seed, offset, n):
    lib, gen = curand
    assert lib.curandSetPseudoRandomGeneratorSeed(gen, ctypes.c_ulonglong(seed)) == 0
    assert lib.curandSetGeneratorOffset(gen, ctypes.c_ulonglong(offset)) == 0
    out = (ctypes.c_uint32 * n)()
    assert lib.curandGenerate(gen, out, ctypes.c_size_t(n)) == 0
    return np.frombuffer(out, dtype=np.uint32).copy()


def _oracle_word(seed, j):
    r, rem = divmod(j, 4 * STREAMS)
    t, w = divmod(rem, 4)
    key = (seed & 0xFFFFFFFF, seed >> 32)
    return oracle.philox4x32_10((r & 0xFFFFFFFF, r >> 32, t, 0), key)[w]


SEEDS = [0, 1, 0x5EED, 0xC0FFEE, 0x0F1E2D3C4B5A6978, 0xFFFFFFFFFFFFFFFF]


@pytest.mark.parametrize("seed", SEEDS)
def test_first_blocks_match_curand(curand, seed):
    # stream 0..63 of round 0: consecutive counters (0, 0, t, 0)
    a = _draw(curand, seed, 0, 256)
    got = [_oracle_word(seed, j) for j in range(256)]
    assert [int(v) for v in a] == got


@pytest.mark.parametrize("seed", SEEDS[2:])
def test_sampled_words_across_rounds_match_curand(curand, seed):
    # four rounds (counter word 0 = 0..3) and every stream, sampled
    n = 4 * 4 * STREAMS
    a = _draw(curand, seed, 0, n)
    for j in range(3, n, 997):
        assert int(a[j]) == _oracle_word(seed, j), j


@pytest.mark.parametrize("offset", [
    4 * STREAMS * 5 + 4 * 17 + 2,              # round 5, stream 17, from word 2
    1 << 40,                                    # round 2^22
    (1 << 50) + 12,                             # round 2^32: counter word 1 = 1
    (7 << 50) + (0xABCDE << 18) + 4 * 40000 + 1,  # word 1 = 7, word 0 = 0xABCDE
])
def test_offsets_reach_counter_words_0_and_1(curand, offset):
    seed = 0x0F1E2D3C4B5A6978
    a = _draw(curand, seed, offset, 64)
    assert [int(v) for v in a] == [_oracle_word(seed, offset + i) for i in range(64)]
