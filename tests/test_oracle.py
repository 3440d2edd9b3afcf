"""Pins for the FP64 oracle: closed forms, invariants, brute force and a hand-worked case.

None of these re-types the oracle's formula.  Each checks a fact that the
mathematics (or the pages' "exact attention" claim, opendecode.dev summary,
"The key idea") fixes, chosen so that a plausible slip in the oracle (a
dropped scale, a wrong sign, a transposed operand, an off-by-one in the mask,
a log base, a missing max-subtraction) fails at least one of them.
"""

import json
import math
import os

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


def allowed_count(N, r, causal, kv, bm):
    """Number of allowed keys of row r, counted one key at a time."""
    cnt = 0
    for c in range(N):
        ok = (not causal or c <= r) and (kv is None or c < kv)
        if bm is not None:
            ok = ok and bm[r // 128, c // 128] != 0
        cnt += int(ok)
    return cnt


# ---------------------------------------------------------------------------
# hand-worked example (tests/golden/two_key_attention.json)
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("case", ["noncausal", "causal"])
def test_golden_two_key(case):
    g = json.load(open(os.path.join(GOLDEN, "two_key_attention.json")))
    q = np.array(g["q"])[None, None]
    k = np.array(g["k"])[None, None]
    v = np.array(g["v"])[None, None]
    do = np.array(g["dout"])[None, None]
    causal = case == "causal"
    exp = g[case]
    o, lse = oracle.attention_forward(q, k, v, g["scale"], causal=causal)
    np.testing.assert_allclose(o[0, 0], exp["o"], rtol=0, atol=1e-14)
    np.testing.assert_allclose(lse[0, 0], exp["lse"], rtol=0, atol=1e-14)
    dq, dk, dv, delta = oracle.attention_backward(q, k, v, do, g["scale"], causal=causal)
    np.testing.assert_allclose(dq[0, 0], exp["dq"], rtol=0, atol=1e-14)
    np.testing.assert_allclose(dk[0, 0], exp["dk"], rtol=0, atol=1e-14)
    np.testing.assert_allclose(dv[0, 0], exp["dv"], rtol=0, atol=1e-14)
    np.testing.assert_allclose(delta[0, 0], exp["delta"], rtol=0, atol=1e-14)


# ---------------------------------------------------------------------------
# closed forms
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("causal,kv,use_bm", [(False, None, False), (True, None, False),
                                              (False, 300, False), (True, 200, True),
                                              (False, None, True)])
def test_zero_query_gives_mean_of_allowed_values(causal, kv, use_bm):
    B, H, N, d = 1, 2, 384, 16
    q = np.zeros((B, H, N, d))
    k, v = rand((B, H, N, d), 1), rand((B, H, N, d), 2)
    bm = None
    if use_bm:
        bm = np.array([[1, 0, 1], [1, 1, 0], [0, 1, 1]], np.uint8)
    kvl = None if kv is None else np.array([kv], np.int32)
    o, lse = oracle.attention_forward(q, k, v, 0.125, causal=causal, block_mask=bm, kv_len=kvl)
    for r in [0, 1, 127, 128, 200, 255, 256, 383]:
        keys = [c for c in range(N)
                if (not causal or c <= r) and (kv is None or c < kv)
                and (bm is None or bm[r // 128, c // 128])]
        cnt = allowed_count(N, r, causal, kv, bm)
        assert cnt == len(keys)
        for h in range(H):
            if cnt == 0:
                assert np.all(o[0, h, r] == 0) and lse[0, h, r] == -np.inf
                continue
            np.testing.assert_allclose(o[0, h, r], v[0, h, keys].mean(axis=0), atol=1e-13)
            assert abs(lse[0, h, r] - math.log(cnt)) < 1e-13


@pytest.mark.parametrize("causal,kv", [(False, None), (True, None), (False, 290), (True, 260)])
def test_zero_query_partial_last_tile(causal, kv):
    # N = 300: tiles 0..127, 128..255 and a partial tile 256..299; the block mask
    # has ceil(300 / 128) = 3 rows and columns, its last ones covering the rest
    B, H, N, d = 1, 1, 300, 8
    q = np.zeros((B, H, N, d))
    k, v = rand((B, H, N, d), 11), rand((B, H, N, d), 12)
    bm = np.array([[1, 0, 1], [0, 1, 0], [1, 1, 1]], np.uint8)
    kvl = None if kv is None else np.array([kv], np.int32)
    o, lse = oracle.attention_forward(q, k, v, 0.5, causal=causal, block_mask=bm, kv_len=kvl)
    for r in [0, 5, 127, 128, 255, 256, 270, 299]:
        keys = [c for c in range(N)
                if (not causal or c <= r) and (kv is None or c < kv) and bm[r // 128, c // 128]]
        if not keys:
            assert np.all(o[0, 0, r] == 0) and lse[0, 0, r] == -np.inf
            continue
        np.testing.assert_allclose(o[0, 0, r], v[0, 0, keys].mean(axis=0), atol=1e-13)
        assert abs(lse[0, 0, r] - math.log(len(keys))) < 1e-13


def test_dominant_score_selects_one_value_row():
    N, d = 64, 64
    rng = np.random.default_rng(3)
    # orthonormal key rows: each query aligned with one key gives score 50*scale*|k| for it,
    # and 0 for every other key
    basis, _ = np.linalg.qr(rng.standard_normal((d, d)))
    k = basis[:N]
    target = rng.permutation(N)
    q = 400.0 * k[target]          # score 400*scale = 50 for the target key, 0 elsewhere
    v = rng.standard_normal((N, d))
    o, lse = oracle.attention_forward(q[None, None], k[None, None], v[None, None], 0.125)
    np.testing.assert_allclose(o[0, 0], v[target], atol=1e-12 * 50)
    # LSE = 50 + ln(1 + (N-1) e^-50)
    np.testing.assert_allclose(lse[0, 0], 50.0 + np.log1p((N - 1) * np.exp(-50.0)), atol=1e-12)


def test_large_scores_do_not_overflow():
    # scores near 1000 overflow exp() unless the row max is subtracted first
    N, d = 8, 4
    q = np.zeros((N, d)); q[:, 0] = 1000.0
    k = np.zeros((N, d)); k[:, 0] = 1.0; k[3, 0] = 1.001
    v = rand((N, d), 4)
    o, lse = oracle.attention_forward(q[None, None], k[None, None], v[None, None], 1.0)
    w = np.exp(np.array([0.0] * 3 + [1.0] + [0.0] * 4))
    np.testing.assert_allclose(o[0, 0, 0], (w[:, None] * v).sum(0) / w.sum(), atol=1e-12)
    np.testing.assert_allclose(lse[0, 0, 0], 1000.0 + np.log(w.sum()), atol=1e-10)


def test_causal_row_zero():
    B, H, N, d = 2, 3, 256, 32
    q, k, v = rand((B, H, N, d), 5), rand((B, H, N, d), 6), rand((B, H, N, d), 7)
    s = 0.17
    o, lse = oracle.attention_forward(q, k, v, s, causal=True)
    assert np.array_equal(o[:, :, 0], v[:, :, 0])
    np.testing.assert_allclose(lse[:, :, 0], s * np.einsum("bhx,bhx->bh", q[:, :, 0], k[:, :, 0]),
                               atol=1e-13)


def test_single_key():
    q, k, v, do = (rand((1, 2, 1, 8), s) for s in range(4))
    o, lse = oracle.attention_forward(q, k, v, 0.3)
    assert np.array_equal(o, v)
    dq, dk, dv, _ = oracle.attention_backward(q, k, v, do, 0.3)
    assert np.all(dq == 0) and np.all(dk == 0)
    assert np.array_equal(dv, do)


def test_value_identity_gives_probability_rows():
    # with V = I (d = N) the output row is the probability row itself: rows sum to 1,
    # entries are non-negative and zero exactly on masked keys
    N = 256
    q, k = rand((1, 1, N, N), 8), rand((1, 1, N, N), 9)
    v = np.eye(N)[None, None]
    bm = np.array([[1, 0], [1, 1]], np.uint8)
    for causal, kv, m in [(False, None, None), (True, None, None), (False, 100, None),
                          (True, 200, bm)]:
        kvl = None if kv is None else np.array([kv], np.int32)
        p, _ = oracle.attention_forward(q, k, v, 0.05, causal=causal, block_mask=m, kv_len=kvl)
        p = p[0, 0]
        np.testing.assert_allclose(p.sum(axis=1), 1.0, atol=1e-14)
        assert np.all(p >= 0)
        for r in range(N):
            for c in range(N):
                ok = (not causal or c <= r) and (kv is None or c < kv) and \
                     (m is None or m[r // 128, c // 128])
                if not ok:
                    assert p[r, c] == 0.0


# ---------------------------------------------------------------------------
# invariants
# ---------------------------------------------------------------------------

def test_joint_key_value_permutation():
    B, H, N, d = 1, 2, 200, 16
    q, k, v, do = (rand((B, H, N, d), s) for s in (10, 11, 12, 13))
    perm = np.random.default_rng(14).permutation(N)
    o1, l1 = oracle.attention_forward(q, k, v, 0.25)
    o2, l2 = oracle.attention_forward(q, k[:, :, perm], v[:, :, perm], 0.25)
    np.testing.assert_allclose(o1, o2, atol=1e-12)
    np.testing.assert_allclose(l1, l2, atol=1e-12)
    _, dk1, dv1, _ = oracle.attention_backward(q, k, v, do, 0.25)
    _, dk2, dv2, _ = oracle.attention_backward(q, k[:, :, perm], v[:, :, perm], do, 0.25)
    np.testing.assert_allclose(dk1[:, :, perm], dk2, atol=1e-12)
    np.testing.assert_allclose(dv1[:, :, perm], dv2, atol=1e-12)


def test_key_shift_shifts_lse_only():
    B, H, N, d = 1, 1, 160, 8
    q, k, v = (rand((B, H, N, d), s) for s in (15, 16, 17))
    c = rand((d,), 18)
    s = 0.3
    o1, l1 = oracle.attention_forward(q, k, v, s, causal=True)
    o2, l2 = oracle.attention_forward(q, k + c, v, s, causal=True)
    np.testing.assert_allclose(o1, o2, atol=1e-12)
    np.testing.assert_allclose(l2 - l1, s * q @ c, atol=1e-12)


@pytest.mark.parametrize("causal,kv", [(False, None), (True, None), (False, 150)])
def test_gradient_sum_rules(causal, kv):
    B, H, N, d = 1, 2, 256, 16
    q, k, v, do = (rand((B, H, N, d), s) for s in (19, 20, 21, 22))
    kvl = None if kv is None else np.array([kv], np.int32)
    dq, dk, dv, delta = oracle.attention_backward(q, k, v, do, 0.2, causal=causal, kv_len=kvl)
    # P rows sum to 1, so the value gradients add up to the output gradients
    np.testing.assert_allclose(dv.sum(axis=2), do.sum(axis=2), atol=1e-11)
    # sum_c dS_rc = D_r - D_r = 0, so the key gradients add up to 0 per head
    np.testing.assert_allclose(dk.sum(axis=2), 0.0, atol=1e-11)
    if kv is not None:
        assert np.all(dk[:, :, kv:] == 0) and np.all(dv[:, :, kv:] == 0)
    # D_r = sum_c P dP equals rowsum(dO * O)
    o, _ = oracle.attention_forward(q, k, v, 0.2, causal=causal, kv_len=kvl)
    np.testing.assert_allclose(delta, (do * o).sum(axis=3), atol=1e-12)


def test_fully_masked_rows():
    # causal with the first diagonal tile masked out: rows 0..127 see no key
    B, H, N, d = 1, 1, 256, 8
    q, k, v, do = (rand((B, H, N, d), s) for s in (23, 24, 25, 26))
    bm = np.array([[0, 1], [1, 1]], np.uint8)
    o, lse = oracle.attention_forward(q, k, v, 0.5, causal=True, block_mask=bm)
    assert np.all(o[0, 0, :128] == 0) and np.all(np.isneginf(lse[0, 0, :128]))
    assert np.all(np.isfinite(lse[0, 0, 128:]))
    dq, dk, dv, _ = oracle.attention_backward(q, k, v, do, 0.5, causal=True, block_mask=bm)
    assert np.all(dq[0, 0, :128] == 0)
    assert np.all(np.isfinite(dk)) and np.all(np.isfinite(dv))


@pytest.mark.parametrize("causal", [False, True])
def test_key_lengths_outside_zero_to_n_are_clamped(causal):
    # The library's contract for kv_len: values are taken clamped into [0, N], so a
    # negative length (or 0) leaves a batch with no key at all, and a length above N
    # masks nothing.  Batch 0: kv_len = -3, batch 1: N + 5, batch 2: 0.
    B, H, N, d = 3, 2, 200, 8
    q, k, v, do = (rand((B, H, N, d), s) for s in (61, 62, 63, 64))
    kvl = np.array([-3, N + 5, 0], np.int32)
    o, lse = oracle.attention_forward(q, k, v, 0.3, causal=causal, kv_len=kvl)
    dq, dk, dv, _ = oracle.attention_backward(q, k, v, do, 0.3, causal=causal, kv_len=kvl)
    for b in (0, 2):  # no allowed key: the empty-row definition
        assert np.all(o[b] == 0) and np.all(np.isneginf(lse[b]))
        assert np.all(dq[b] == 0) and np.all(dk[b] == 0) and np.all(dv[b] == 0)
    # batch 1 sees every key: the same values as without key lengths (Q = 0 closed form
    # for the forward, and the unpadded call for the backward)
    o0, lse0 = oracle.attention_forward(np.zeros_like(q[1:2]), k[1:2], v[1:2], 0.3,
                                        causal=causal, kv_len=np.array([N + 5], np.int32))
    for r in (0, 57, 199):
        cnt = r + 1 if causal else N
        np.testing.assert_allclose(o0[0, :, r], v[1, :, :cnt].mean(axis=1), atol=1e-13)
        assert np.all(np.abs(lse0[0, :, r] - math.log(cnt)) < 1e-13)
    o1, lse1 = oracle.attention_forward(q[1:2], k[1:2], v[1:2], 0.3, causal=causal)
    dq1, dk1, dv1, _ = oracle.attention_backward(q[1:2], k[1:2], v[1:2], do[1:2], 0.3,
                                                 causal=causal)
    assert np.array_equal(o[1], o1[0]) and np.array_equal(lse[1], lse1[0])
    assert np.array_equal(dq[1], dq1[0]) and np.array_equal(dk[1], dk1[0])
    assert np.array_equal(dv[1], dv1[0])
    # the one-head row and column functions follow the same rule
    rows = np.array([0, 99, 199])
    for kv_b, b in ((-3, 0), (N + 5, 1), (0, 2)):
        orow, lrow = oracle.attention_forward_rows(q[b, 0, rows], rows, k[b, 0], v[b, 0], 0.3,
                                                   causal=causal, kv_len_b=kv_b)
        np.testing.assert_array_equal(orow, o[b, 0, rows])
        np.testing.assert_array_equal(lrow, lse[b, 0, rows])
        dqr, _ = oracle.attention_backward_dq_rows(q[b, 0, rows], do[b, 0, rows], rows, k[b, 0],
                                                   v[b, 0], 0.3, causal=causal, kv_len_b=kv_b)
        np.testing.assert_allclose(dqr, dq[b, 0, rows], rtol=0, atol=1e-12)
        dkc, dvc = oracle.attention_backward_kv_cols(q[b, 0], k[b, 0], v[b, 0], do[b, 0], rows,
                                                     0.3, causal=causal, kv_len_b=kv_b)
        np.testing.assert_allclose(dkc, dk[b, 0, rows], rtol=0, atol=1e-12)
        np.testing.assert_allclose(dvc, dv[b, 0, rows], rtol=0, atol=1e-12)


# ---------------------------------------------------------------------------
# brute force: finite differences of L = sum(O * dO)
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("causal,kv", [(False, None), (True, None), (False, 11)])
def test_finite_difference_gradients(causal, kv):
    N, d, s = 16, 8, 0.4
    q, k, v, do = (rand((1, 1, N, d), t) for t in (27, 28, 29, 30))
    kvl = None if kv is None else np.array([kv], np.int32)

    def loss(qq, kk, vv):
        o, _ = oracle.attention_forward(qq, kk, vv, s, causal=causal, kv_len=kvl, nthreads=1)
        return float((o * do).sum())

    dq, dk, dv, _ = oracle.attention_backward(q, k, v, do, s, causal=causal, kv_len=kvl)
    h = 1e-6
    for which, grad in ((0, dq), (1, dk), (2, dv)):
        num = np.zeros_like(grad)
        for r in range(N):
            for x in range(d):
                args_p = [q.copy(), k.copy(), v.copy()]
                args_m = [q.copy(), k.copy(), v.copy()]
                args_p[which][0, 0, r, x] += h
                args_m[which][0, 0, r, x] -= h
                num[0, 0, r, x] = (loss(*args_p) - loss(*args_m)) / (2 * h)
        err = np.linalg.norm(num - grad) / max(np.linalg.norm(grad), 1e-300)
        assert err < 1e-7, (which, err)


# ---------------------------------------------------------------------------
# the pages' mechanism: tiled online softmax reaches the same numbers
# ---------------------------------------------------------------------------

def online_softmax_tiled(q, k, v, scale, causal, Br=32, Bc=48):
    """Tiles of keys visited one at a time, keeping a running row max and row sum and
    rescaling the partial output whenever the max grows (opendecode.dev summary,
    'The key idea').  Test-only; unrelated to the oracle's code."""
    N, d = q.shape
    o = np.zeros((N, d))
    lse = np.zeros(N)
    for r0 in range(0, N, Br):
        qi = q[r0:r0 + Br]
        rows = np.arange(r0, min(r0 + Br, N))
        m = np.full(len(rows), -np.inf)
        l = np.zeros(len(rows))
        acc = np.zeros((len(rows), d))
        for c0 in range(0, N, Bc):
            cols = np.arange(c0, min(c0 + Bc, N))
            sc = scale * qi @ k[cols].T
            if causal:
                sc = np.where(cols[None, :] <= rows[:, None], sc, -np.inf)
            m_new = np.maximum(m, sc.max(axis=1))
            safe = np.where(np.isinf(m_new), 0.0, m_new)
            alpha = np.exp(m - safe)
            p = np.exp(sc - safe[:, None])
            l = alpha * l + p.sum(axis=1)
            acc = alpha[:, None] * acc + p @ v[cols]
            m = m_new
        o[rows] = acc / l[:, None]
        lse[rows] = m + np.log(l)
    return o, lse


@pytest.mark.parametrize("causal", [False, True])
def test_online_softmax_matches_oracle(causal):
    N, d = 230, 24
    q, k, v = (rand((N, d), t) * 2 for t in (31, 32, 33))
    o_t, l_t = online_softmax_tiled(q, k, v, 0.3, causal)
    o, l = oracle.attention_forward(q[None, None], k[None, None], v[None, None], 0.3,
                                    causal=causal)
    np.testing.assert_allclose(o[0, 0], o_t, atol=1e-12)
    np.testing.assert_allclose(l[0, 0], l_t, atol=1e-12)


# ---------------------------------------------------------------------------
# row-subset forward and tile visits
# ---------------------------------------------------------------------------

def test_forward_rows_match_full_forward():
    N, d = 512, 16
    q, k, v = (rand((1, 1, N, d), t) for t in (34, 35, 36))
    bm = np.array([[1, 0, 0, 1], [1, 1, 0, 0], [0, 0, 1, 0], [1, 0, 1, 1]], np.uint8)
    rows = np.array([0, 5, 130, 300, 511])
    for causal, kv in [(False, None), (True, 333)]:
        kvl = None if kv is None else np.array([kv], np.int32)
        o, l = oracle.attention_forward(q, k, v, 0.2, causal=causal, block_mask=bm, kv_len=kvl)
        orow, lrow = oracle.attention_forward_rows(q[0, 0, rows], rows, k[0, 0], v[0, 0], 0.2,
                                                   causal=causal, block_mask=bm, kv_len_b=kv)
        assert np.array_equal(orow, o[0, 0, rows]) and np.array_equal(lrow, l[0, 0, rows])


def test_tile_visits_hand_enumerated():
    # N = 512 -> 4 x 4 tiles.  Written out by hand from the mask definition.
    causal_only = oracle.tile_visits(1, 512, causal=True)[0]
    assert causal_only.tolist() == [[1, 0, 0, 0], [1, 1, 0, 0], [1, 1, 1, 0], [1, 1, 1, 1]]
    # keys < 200 live in key tiles 0 and 1 (tile 1 holds keys 128..255)
    kv = oracle.tile_visits(2, 512, kv_len=np.array([200, 512], np.int32))
    assert kv[0].tolist() == [[1, 1, 0, 0]] * 4
    assert kv[1].tolist() == [[1, 1, 1, 1]] * 4
    both = oracle.tile_visits(1, 512, causal=True, kv_len=np.array([129], np.int32))[0]
    assert both.tolist() == [[1, 0, 0, 0], [1, 1, 0, 0], [1, 1, 0, 0], [1, 1, 0, 0]]
    bm = np.array([[1, 1, 0, 0], [0, 1, 0, 1], [1, 0, 0, 0], [0, 0, 1, 1]], np.uint8)
    masked = oracle.tile_visits(1, 512, causal=True, block_mask=bm)[0]
    assert masked.tolist() == [[1, 0, 0, 0], [0, 1, 0, 0], [1, 0, 0, 0], [0, 0, 1, 1]]
    part = oracle.tile_visits(1, 512, causal=True, block_mask=bm, i_begin=2, i_end=4)[0]
    assert part.tolist() == masked[2:].tolist()


def test_tile_visits_partial_last_tile_hand_enumerated():
    # N = 300 -> tiles 0..127, 128..255, 256..299.  Written out by hand.
    assert oracle.tile_visits(1, 300, causal=True)[0].tolist() == [[1, 0, 0], [1, 1, 0],
                                                                    [1, 1, 1]]
    # keys < 256 end exactly at the second tile; keys < 257 reach the partial one
    kv = oracle.tile_visits(2, 300, kv_len=np.array([256, 257], np.int32))
    assert kv[0].tolist() == [[1, 1, 0]] * 3
    assert kv[1].tolist() == [[1, 1, 1]] * 3
    bm = np.array([[1, 0, 1], [0, 1, 0], [0, 1, 1]], np.uint8)
    assert oracle.tile_visits(1, 300, block_mask=bm)[0].tolist() == bm.tolist()
    # N = 100: a single partial tile
    assert oracle.tile_visits(1, 100, causal=True)[0].tolist() == [[1]]
    assert oracle.tile_visits(1, 100, kv_len=np.array([0], np.int32))[0].tolist() == [[0]]


def test_tile_visits_agree_with_value_identity_probabilities():
    # a tile pair is visited exactly when some probability inside it can be nonzero
    N = 384
    q, k = rand((1, 1, N, N), 37) * 0.01, rand((1, 1, N, N), 38) * 0.01
    v = np.eye(N)[None, None]
    bm = np.array([[1, 0, 1], [0, 1, 1], [1, 1, 0]], np.uint8)
    kvl = np.array([300], np.int32)
    p, _ = oracle.attention_forward(q, k, v, 1.0, causal=True, block_mask=bm, kv_len=kvl)
    vis = oracle.tile_visits(1, N, causal=True, block_mask=bm, kv_len=kvl)[0]
    for i in range(3):
        for j in range(3):
            blk = p[0, 0, i * 128:(i + 1) * 128, j * 128:(j + 1) * 128]
            assert bool(vis[i, j]) == bool(np.any(blk > 0)), (i, j)


def test_backward_dq_rows_match_full_backward():
    N, d = 384, 16
    q, k, v, do = (rand((1, 1, N, d), t) for t in (39, 40, 41, 42))
    bm = np.array([[1, 0, 1], [1, 1, 0], [0, 1, 1]], np.uint8)
    rows = np.array([0, 7, 128, 200, 383])
    for causal, kv in [(False, None), (True, 250)]:
        kvl = None if kv is None else np.array([kv], np.int32)
        dq, _, _, delta = oracle.attention_backward(q, k, v, do, 0.3, causal=causal,
                                                    block_mask=bm, kv_len=kvl)
        dqr, dr = oracle.attention_backward_dq_rows(q[0, 0, rows], do[0, 0, rows], rows, k[0, 0],
                                                    v[0, 0], 0.3, causal=causal, block_mask=bm,
                                                    kv_len_b=kv)
        np.testing.assert_allclose(dqr, dq[0, 0, rows], atol=1e-13)
        np.testing.assert_allclose(dr, delta[0, 0, rows], atol=1e-13)


def test_backward_kv_cols_match_full_backward():
    N, d = 640, 16
    q, k, v, do = (rand((1, 1, N, d), t) for t in (43, 44, 45, 46))
    bm = np.array([[1, 0, 1, 0, 1], [1, 1, 0, 0, 1], [0, 1, 1, 1, 0], [1, 0, 0, 1, 1],
                   [0, 1, 1, 0, 1]], np.uint8)
    cols = np.array([0, 5, 127, 128, 300, 511, 639])
    for causal, kv in [(False, None), (True, 500)]:
        kvl = None if kv is None else np.array([kv], np.int32)
        _, dk, dv, _ = oracle.attention_backward(q, k, v, do, 0.3, causal=causal, block_mask=bm,
                                                 kv_len=kvl)
        for nt in (1, 3):
            dkc, dvc = oracle.attention_backward_kv_cols(q[0, 0], k[0, 0], v[0, 0], do[0, 0], cols,
                                                         0.3, causal=causal, block_mask=bm,
                                                         kv_len_b=kv, nthreads=nt)
            np.testing.assert_allclose(dkc, dk[0, 0, cols], atol=1e-12)
            np.testing.assert_allclose(dvc, dv[0, 0, cols], atol=1e-12)


def test_row_bands_partition_the_full_result():
    N, d = 384, 8
    q, k, v, do = (rand((1, 2, N, d), t) for t in (47, 48, 49, 50))
    kvl = np.array([300], np.int32)
    o, l = oracle.attention_forward(q, k, v, 0.4, causal=True, kv_len=kvl)
    dq, dk, dv, _ = oracle.attention_backward(q, k, v, do, 0.4, causal=True, kv_len=kvl)
    o1, l1 = oracle.attention_forward_band(q, k, v, 0.4, True, None, kvl, 0, 150)
    o2, l2 = oracle.attention_forward_band(q, k, v, 0.4, True, None, kvl, 150, N)
    np.testing.assert_array_equal(o1[:, :, :150], o[:, :, :150])
    np.testing.assert_array_equal(o2[:, :, 150:], o[:, :, 150:])
    np.testing.assert_array_equal(l2[:, :, 150:], l[:, :, 150:])
    g1 = oracle.attention_backward_band(q, k, v, do, 0.4, True, None, kvl, 0, 150)
    g2 = oracle.attention_backward_band(q, k, v, do, 0.4, True, None, kvl, 150, N)
    np.testing.assert_array_equal(g1[0][:, :, :150], dq[:, :, :150])
    np.testing.assert_array_equal(g2[0][:, :, 150:], dq[:, :, 150:])
    np.testing.assert_allclose(g1[1] + g2[1], dk, atol=1e-13)
    np.testing.assert_allclose(g1[2] + g2[2], dv, atol=1e-13)


# ---------------------------------------------------------------------------
# dropout (the pages list dropout among the steps the fused kernel absorbs:
# [HF] "Standard Attention Algorithm"); the mask comes from Philox-4x32-10
# ---------------------------------------------------------------------------

def test_dropout_with_zero_probability_is_plain_attention():
    q, k, v, do = (rand((1, 2, 96, 8), t) for t in (60, 61, 62, 63))
    kvl = np.array([70], np.int32)
    o, l = oracle.attention_forward(q, k, v, 0.3, causal=True, kv_len=kvl)
    od, ld = oracle.attention_forward_dropout(q, k, v, 0.3, 0.0, seed=5, causal=True, kv_len=kvl)
    assert np.array_equal(o, od) and np.array_equal(l, ld)
    g = oracle.attention_backward(q, k, v, do, 0.3, causal=True, kv_len=kvl)
    gd = oracle.attention_backward_dropout(q, k, v, do, 0.3, 0.0, seed=5, causal=True, kv_len=kvl)
    for a, b in zip(g, gd):
        assert np.array_equal(a, b)


def test_philox_is_a_bijection_of_the_counter():
    # each round is invertible for a fixed key, so distinct counters never collide
    outs = {tuple(oracle.philox4x32_10([i, i >> 3, 7, 1], [11, 13])) for i in range(4096)}
    assert len(outs) == 4096


def test_dropout_draws_are_uniform_16_bit_values():
    _, u = oracle.dropout_keep(4, 256, 0.0, seed=0x1234567890ABCDEF, offset=3)
    x = u.astype(np.float64).ravel()
    n = x.size
    mu, sd = 32767.5, 65536 / math.sqrt(12)
    assert abs(x.mean() - mu) < 5 * sd / math.sqrt(n)
    assert abs(x.std() - sd) < 0.01 * sd
    # top bytes: chi-square with 255 degrees of freedom, far inside 5 standard deviations
    counts = np.bincount((u.ravel() >> 8).astype(np.int64), minlength=256)
    e = n / 256
    chi2 = float(((counts - e) ** 2 / e).sum())
    assert abs(chi2 - 255) < 5 * math.sqrt(2 * 255)
    # neighbours along keys and along queries are uncorrelated
    for a, b in ((u[:, :, :-1], u[:, :, 1:]), (u[:, :-1, :], u[:, 1:, :])):
        r = np.corrcoef(a.ravel().astype(np.float64), b.ravel().astype(np.float64))[0, 1]
        assert abs(r) < 5 / math.sqrt(a.size)


@pytest.mark.parametrize("p", [0.1, 0.5, 0.9])
def test_dropout_keep_fraction(p):
    keep, u = oracle.dropout_keep(2, 256, p, seed=99)
    t = int(np.float32(p) * np.float32(65536.0))
    assert np.array_equal(keep, (u >= t).astype(np.uint8))
    n = keep.size
    q_keep = 1 - t / 65536
    assert abs(keep.mean() - q_keep) < 5 * math.sqrt(q_keep * (1 - q_keep) / n)
    # another seed or offset draws another mask: disagreement 2 q (1 - q) on average
    k2, _ = oracle.dropout_keep(2, 256, p, seed=100)
    k3, _ = oracle.dropout_keep(2, 256, p, seed=99, offset=1)
    for other in (k2, k3):
        dis = (keep != other).mean()
        exp = 2 * q_keep * (1 - q_keep)
        assert abs(dis - exp) < 5 * math.sqrt(exp * (1 - exp) / n)


def test_dropout_zero_query_closed_form():
    # Q = 0: P is uniform over the allowed keys, so O_r = w / count * sum of kept V rows
    B, H, N, d, p = 1, 2, 200, 8, 0.3
    q = np.zeros((B, H, N, d))
    k, v = rand((B, H, N, d), 64), rand((B, H, N, d), 65)
    kvl = np.array([150], np.int32)
    o, l = oracle.attention_forward_dropout(q, k, v, 0.5, p, seed=21, offset=4, causal=True,
                                            kv_len=kvl)
    keep, _ = oracle.dropout_keep(B * H, N, p, seed=21, offset=4)
    t = int(np.float32(p) * np.float32(65536.0))
    w = 65536.0 / (65536.0 - t)
    for h in range(H):
        for r in [0, 1, 77, 149, 150, 199]:
            keys = [c for c in range(N) if c <= r and c < 150]
            kept = [c for c in keys if keep[h, r, c]]
            want = w * v[0, h, kept].sum(axis=0) / len(keys)
            np.testing.assert_allclose(o[0, h, r], want, atol=1e-13)
            assert abs(l[0, h, r] - math.log(len(keys))) < 1e-13


@pytest.mark.parametrize("causal,kv", [(False, None), (True, 11)])
def test_dropout_finite_difference_gradients(causal, kv):
    # the mask depends on (seed, offset, head, row, key) only, so L = sum(O * dO) is a
    # smooth function of q, k, v and its central differences give the gradients
    B, H, N, d, scale, p = 1, 1, 16, 8, 0.4, 0.35
    q, k, v, do = (rand((B, H, N, d), t) for t in (70, 71, 72, 73))
    kvl = None if kv is None else np.array([kv], np.int32)
    dq, dk, dv, _ = oracle.attention_backward_dropout(q, k, v, do, scale, p, seed=3,
                                                      causal=causal, kv_len=kvl)

    def loss(qq, kk, vv):
        o, _ = oracle.attention_forward_dropout(qq, kk, vv, scale, p, seed=3, causal=causal,
                                                kv_len=kvl)
        return float((o * do).sum())

    h = 1e-6
    for name, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        num = np.zeros_like(x)
        for idx in np.ndindex(x.shape):
            xp, xm = x.copy(), x.copy()
            xp[idx] += h
            xm[idx] -= h
            args = {"q": (q, k, v), "k": (q, k, v), "v": (q, k, v)}[name]
            a_p = [xp if n == name else t for n, t in zip("qkv", args)]
            a_m = [xm if n == name else t for n, t in zip("qkv", args)]
            num[idx] = (loss(*a_p) - loss(*a_m)) / (2 * h)
        err = np.linalg.norm(num - g) / np.linalg.norm(g)
        assert err < 1e-7, (name, err)


# ---------------------------------------------------------------------------
# packed variable-length batches: each sequence is its own attention problem
# ---------------------------------------------------------------------------

def _packed(lengths, H, d, seed):
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    T = int(cu[-1])
    q, k, v, do = (rand((T, H, d), seed + t) for t in range(4))
    return cu, q, k, v, do


@pytest.mark.parametrize("causal", [False, True])
def test_varlen_sequences_are_independent_problems(causal):
    lengths = [5, 1, 0, 13, 8]
    H, d, scale = 2, 4, 0.6
    cu, q, k, v, do = _packed(lengths, H, d, 80)
    o, lse = oracle.attention_forward_varlen(q, k, v, cu, scale, causal)
    dq, dk, dv = oracle.attention_backward_varlen(q, k, v, do, cu, scale, causal)
    for b, n in enumerate(lengths):
        if n == 0:
            continue
        sl = slice(cu[b], cu[b] + n)
        one = lambda x: np.transpose(x[sl], (1, 0, 2))[None]  # [1, H, n, d]
        o1, l1 = oracle.attention_forward(one(q), one(k), one(v), scale, causal)
        g1 = oracle.attention_backward(one(q), one(k), one(v), one(do), scale, causal)
        np.testing.assert_allclose(np.transpose(o[sl], (1, 0, 2)), o1[0], atol=1e-13)
        np.testing.assert_allclose(lse[:, sl], l1[0], atol=1e-13)
        for got, want in zip((dq, dk, dv), g1[:3]):
            np.testing.assert_allclose(np.transpose(got[sl], (1, 0, 2)), want[0], atol=1e-12)


def test_varlen_equal_lengths_is_the_batched_problem_with_dropout():
    B, H, N, d, scale = 3, 2, 24, 4, 0.5
    cu, q, k, v, do = _packed([N] * B, H, d, 90)
    dense = lambda x: np.transpose(x.reshape(B, N, H, d), (0, 2, 1, 3))
    drop = (0.3, 17, 2)
    o, lse = oracle.attention_forward_varlen(q, k, v, cu, scale, True, dropout=drop)
    od, ld = oracle.attention_forward_dropout(dense(q), dense(k), dense(v), scale, *drop,
                                              causal=True)
    np.testing.assert_allclose(dense(o), od, atol=1e-13)
    np.testing.assert_allclose(lse.reshape(H, B, N).transpose(1, 0, 2), ld, atol=1e-13)
    g = oracle.attention_backward_varlen(q, k, v, do, cu, scale, True, dropout=drop)
    gd = oracle.attention_backward_dropout(dense(q), dense(k), dense(v), dense(do), scale, *drop,
                                           causal=True)
    for got, want in zip(g, gd[:3]):
        np.testing.assert_allclose(dense(got), want, atol=1e-12)


# ---------------------------------------------------------------------------
# the backward against automatic differentiation at a multi-tile size
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("causal,kv,use_bm", [(False, None, False), (True, None, False),
                                              (False, (150, 300), True), (True, (100, 260), True)])
def test_backward_matches_automatic_differentiation(causal, kv, use_bm):
    # The finite-difference pins run at N = 16; this one runs at N = 300 (two full tiles and
    # a partial one), where the gradients come from torch's reverse-mode differentiation of
    # L = sum(O * dO) in float64 rather than from the oracle's hand-derived chain rule.
    import torch
    B, H, N, d, s = 2, 2, 300, 32, 0.17
    q, k, v, do = (rand((B, H, N, d), 900 + i) for i in range(4))
    kvl = None if kv is None else np.array(kv, np.int32)
    bm = None
    if use_bm:
        bm = np.zeros((3, 3), np.uint8)
        bm[np.arange(3), np.arange(3)] = 1
        bm[:, 0] = 1  # key 0 stays allowed, so no row is left without keys
        bm[0, 2] = 1
    dq, dk, dv, _ = oracle.attention_backward(q, k, v, do, s, causal, bm, kvl)

    r = np.arange(N)[:, None]
    c = np.arange(N)[None, :]
    allowed = np.ones((B, 1, N, N), bool)
    if causal:
        allowed &= (c <= r)[None, None]
    if kvl is not None:
        allowed &= (c[None, None] < kvl[:, None, None, None])
    if bm is not None:
        allowed &= bm[r // 128, c // 128].astype(bool)[None, None]
    tq, tk, tv = (torch.tensor(t, requires_grad=True) for t in (q, k, v))
    scores = s * tq @ tk.transpose(-1, -2)
    scores = scores.masked_fill(~torch.tensor(allowed), float("-inf"))
    out = torch.softmax(scores, dim=-1) @ tv
    (out * torch.tensor(do)).sum().backward()
    for name, mine, ref in (("dq", dq, tq.grad), ("dk", dk, tk.grad), ("dv", dv, tv.grad)):
        np.testing.assert_allclose(mine, ref.numpy(), rtol=0, atol=1e-11, err_msg=name)


@pytest.mark.parametrize("causal", [False, True])
def test_dropout_backward_matches_automatic_differentiation(causal):
    # dropout's keep mask is an input to the arithmetic (drawn by dropout_keep); given it,
    # O = w (P o Z) V and torch differentiates sum(O * dO) in float64 at N = 300
    import torch
    B, H, N, d, s = 1, 2, 300, 32, 0.2
    p_drop, seed, offset = 0.3, 77, 5
    q, k, v, do = (rand((B, H, N, d), 950 + i) for i in range(4))
    kvl = np.array([230], np.int32)
    dq, dk, dv, _ = oracle.attention_backward_dropout(q, k, v, do, s, p_drop, seed, offset,
                                                      causal=causal, kv_len=kvl)
    keep, _ = oracle.dropout_keep(B * H, N, p_drop, seed, offset)
    t = math.floor(p_drop * 65536)
    w = 65536.0 / (65536.0 - t)
    r = np.arange(N)[:, None]
    c = np.arange(N)[None, :]
    allowed = (c < kvl[0]) & ((c <= r) if causal else True)
    tq, tk, tv = (torch.tensor(x, requires_grad=True) for x in (q, k, v))
    scores = (s * tq @ tk.transpose(-1, -2)).masked_fill(~torch.tensor(allowed), float("-inf"))
    z = torch.tensor(keep.reshape(B, H, N, N).astype(np.float64))
    out = (torch.softmax(scores, dim=-1) * z * w) @ tv
    (out * torch.tensor(do)).sum().backward()
    for name, mine, ref in (("dq", dq, tq.grad), ("dk", dk, tk.grad), ("dv", dv, tv.grad)):
        np.testing.assert_allclose(mine, ref.numpy(), rtol=0, atol=1e-11, err_msg=name)


@pytest.mark.parametrize("causal,kv,use_bm", [(False, None, False), (True, None, False),
                                              (True, (120, 300), True)])
def test_forward_and_backward_match_torch_scaled_dot_product_attention(causal, kv, use_bm):
    # torch's own attention routine (its float64 CPU path), with the mask as a boolean
    # "may attend" matrix, is an independent implementation of the same definition
    import torch
    import torch.nn.functional as F
    B, H, N, d, s = 2, 3, 300, 32, 0.21
    q, k, v, do = (rand((B, H, N, d), 970 + i) for i in range(4))
    kvl = None if kv is None else np.array(kv, np.int32)
    bm = None
    if use_bm:
        bm = np.eye(3, dtype=np.uint8)
        bm[2, 1] = 1
        bm[:, 0] = 1  # key 0 stays allowed for every row
    o, _ = oracle.attention_forward(q, k, v, s, causal, bm, kvl)
    dq, dk, dv, _ = oracle.attention_backward(q, k, v, do, s, causal, bm, kvl)
    r = np.arange(N)[:, None]
    c = np.arange(N)[None, :]
    allowed = np.ones((B, 1, N, N), bool)
    if causal:
        allowed &= (c <= r)[None, None]
    if kvl is not None:
        allowed &= (c[None, None] < kvl[:, None, None, None])
    if bm is not None:
        allowed &= bm[r // 128, c // 128].astype(bool)[None, None]
    assert allowed.any(-1).all()  # every row keeps a key (the routine has no empty rows)
    tq, tk, tv = (torch.tensor(t, requires_grad=True) for t in (q, k, v))
    out = F.scaled_dot_product_attention(tq, tk, tv, attn_mask=torch.tensor(allowed), scale=s)
    (out * torch.tensor(do)).sum().backward()
    np.testing.assert_allclose(o, out.detach().numpy(), rtol=0, atol=1e-12)
    for name, mine, ref in (("dq", dq, tq.grad), ("dk", dk, tk.grad), ("dv", dv, tv.grad)):
        np.testing.assert_allclose(mine, ref.numpy(), rtol=0, atol=1e-11, err_msg=name)


def test_results_do_not_depend_on_the_thread_count():
    # each head runs on one thread, in one fixed order of additions
    q, k, v, do = (rand((2, 3, 200, 16), 990 + i) for i in range(4))
    kvl = np.array([150, 200], np.int32)
    outs = []
    for nt in (1, 2, 5):
        o, lse = oracle.attention_forward(q, k, v, 0.3, causal=True, kv_len=kvl, nthreads=nt)
        g = oracle.attention_backward(q, k, v, do, 0.3, causal=True, kv_len=kvl, nthreads=nt)
        outs.append((o, lse) + tuple(g))
    for other in outs[1:]:
        for a, b in zip(outs[0], other):
            assert np.array_equal(a, b)
