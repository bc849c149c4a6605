"""Pins of the dropout oracle (``oracle.dropout``): the Philox restatement
against numpy's Philox bit generator, the mask layout, the keep rate, the
unbiasedness of dropout, the p = 0 case, a closed form and finite differences
of the backward pass."""

import math
import os

import numpy as np
import pytest

import oracle
from oracle import dropout as dr


def test_philox_4x64_matches_numpy():
    """The same round function and key schedule with the 64-bit constants is
    numpy's Philox (4x64-10), which advances its counter before each block."""
    for key, ctr in [((3, 5), (7, 0, 0, 0)), ((0, 0), (0, 0, 0, 0)),
                     ((0xFFFFFFFFFFFFFFFF, 0x0123456789ABCDEF), (41, 0xFFFFFFFF, 2**63, 9))]:
        bg = np.random.Philox(key=np.array(key, dtype=np.uint64), counter=np.array(ctr, dtype=np.uint64))
        ref = [int(x) for x in bg.random_raw(4)]
        nxt = ((ctr[0] + 1) % 2**64,) + tuple(ctr[1:])
        assert dr.philox4(nxt, key, width=64) == ref


def _philox_kat():
    out = []
    with open(os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "philox4x32_10_kat.txt")) as f:
        for line in f:
            line = line.split("#", 1)[0].split()
            if line:
                words = [int(x, 16) for x in line[1:]]
                out.append((line[0], words[0:4], words[4:6], words[6:10]))
    return out


def test_philox_4x32_10_known_answers():
    """The 32-bit variant (the one the mask uses) against the published
    known-answer vectors of Philox-4x32-10: its multipliers, Weyl increments
    and round structure are pinned by values computed outside this code."""
    cases = _philox_kat()
    assert [c[0] for c in cases] == ["zeros", "ones", "pi"]
    for name, ctr, key, want in cases:
        assert dr.philox4(ctr, key, width=32) == want, name
        got = dr.philox4x32(*(np.array([c], dtype=np.uint64) for c in ctr), key[0], key[1])
        assert [int(w[0]) for w in got] == want, name


def test_philox_4x32_vectorised_equals_scalar():
    rng = np.random.default_rng(1)
    c = rng.integers(0, 2**32, size=(4, 50), dtype=np.uint64)
    k0, k1 = 0x9A3B1C2D, 0x01020304
    words = dr.philox4x32(c[0], c[1], c[2], c[3], k0, k1)
    for i in range(50):
        assert [int(w[i]) for w in words] == dr.philox4([int(x) for x in c[:, i]], (k0, k1), width=32)
    # changing any counter word or the key changes the block
    base = dr.philox4((1, 2, 3, 4), (5, 6))
    for j in range(4):
        ctr = [1, 2, 3, 4]
        ctr[j] += 1
        assert dr.philox4(ctr, (5, 6)) != base
    assert dr.philox4((1, 2, 3, 4), (5, 7)) != base


def test_mask_layout_is_the_4x4_block_rule():
    seed, offset, bh = 0x1234_5678_9ABC, 17, 5
    Z = dr.dropout_keep(seed, offset, bh, np.arange(9), np.arange(13), 0.4)
    t = dr.keep_threshold(0.4)
    for i in range(9):
        for j in range(13):
            w = dr.philox4((i >> 2, j >> 2, bh, offset), (seed & 0xFFFFFFFF, seed >> 32))[i & 3]
            assert Z[i, j] == (((w >> (8 * (j & 3))) & 0xFF) < t)
    # any sub-block of rows and columns is the same slice of the full mask
    Zs = dr.dropout_keep(seed, offset, bh, np.arange(3, 8), np.arange(6, 11), 0.4)
    np.testing.assert_array_equal(Zs, Z[3:8, 6:11])


def test_keep_rate_and_threshold():
    assert dr.keep_threshold(0.0) == 256 and dr.keep_threshold(0.5) == 128 and dr.keep_threshold(0.1) == 230
    with pytest.raises(ValueError):
        dr.keep_threshold(1.0)
    for p in (0.1, 0.5, 0.9):
        Z = dr.dropout_keep(99, 0, 3, np.arange(512), np.arange(512), p)
        q = dr.keep_threshold(p) / 256.0
        n = Z.size
        assert abs(Z.mean() - q) < 5 * math.sqrt(q * (1 - q) / n)
    # different seeds, offsets and heads give different masks
    a = dr.dropout_keep(1, 0, 0, np.arange(64), np.arange(64), 0.5)
    for args in ((2, 0, 0), (1, 1, 0), (1, 0, 1)):
        assert (dr.dropout_keep(*args, np.arange(64), np.arange(64), 0.5) != a).mean() > 0.3


def _inputs(B=1, T=24, Hq=2, Hkv=1, d=5, seed=0):
    rng = np.random.default_rng(seed)
    return [rng.standard_normal((B, T, H, d)) for H in (Hq, Hkv, Hkv, Hq)]


def test_no_dropout_equals_plain_attention():
    q, k, v, do = _inputs()
    O, L = dr.attention_forward_dropout(q, k, v, 0.4, True, 0.0, 7, 3)
    O0, L0 = oracle.attention_forward(q, k, v, 0.4, True)
    np.testing.assert_allclose(O, O0, rtol=1e-14, atol=1e-15)
    np.testing.assert_array_equal(L, L0)
    g = dr.attention_backward_dropout(q, k, v, do, 0.4, True, 0.0, 7, 3)
    g0 = oracle.attention_backward(q, k, v, do, 0.4, True)
    for a, b in zip(g, g0):
        np.testing.assert_allclose(a, b, rtol=1e-12, atol=1e-14)


def test_equal_scores_closed_form():
    """With equal scores every P_ij is 1/n: O_i = (256/t) / n * sum of the
    kept V_j, and LSE = ln n as without dropout."""
    n, d, p = 37, 3, 0.3
    q = np.zeros((1, n, 1, d))
    k = np.random.default_rng(2).standard_normal((1, n, 1, d))
    v = np.random.default_rng(3).standard_normal((1, n, 1, d))
    O, L = dr.attention_forward_dropout(q, k, v, 1.0, False, p, 11, 0)
    Z = dr.dropout_keep(11, 0, 0, np.arange(n), np.arange(n), p)
    t = dr.keep_threshold(p)
    for i in range(n):
        ref = sum(v[0, j, 0] for j in range(n) if Z[i, j]) * (256.0 / t) / n
        np.testing.assert_allclose(O[0, i, 0], ref, rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(L[0, 0], math.log(n), rtol=1e-15)


def test_dropout_is_unbiased():
    """The mean of O over many seeds approaches O without dropout (the
    1/(1-p) scale makes E[Z]/(1-p) = 1); the spread shrinks like 1/sqrt(N)."""
    q, k, v, _ = _inputs(T=16, Hq=1, Hkv=1, d=4, seed=5)
    O0, _ = oracle.attention_forward(q, k, v, 0.5, False)
    N = 400
    acc = np.zeros_like(O0)
    sq = np.zeros_like(O0)
    for s in range(N):
        O, _ = dr.attention_forward_dropout(q, k, v, 0.5, False, 0.25, 1000 + s, 0)
        acc += O
        sq += O ** 2
    mean = acc / N
    sd = np.sqrt(np.maximum(sq / N - mean ** 2, 0.0))
    assert (np.abs(mean - O0) <= 5 * sd / math.sqrt(N) + 1e-12).all()


@pytest.mark.parametrize("causal", [False, True])
def test_backward_finite_differences_with_fixed_mask(causal):
    """For a fixed (seed, offset) the dropped attention is a smooth function
    of q, k, v: central differences of L = sum(dO * O) match dq, dk, dv."""
    q, k, v, do = _inputs(T=10, Hq=2, Hkv=1, d=3, seed=9)
    args = (0.7, causal, 0.35, 123, 4)
    dq, dk, dv = dr.attention_backward_dropout(q, k, v, do, *args)

    def loss(q_, k_, v_):
        return float((dr.attention_forward_dropout(q_, k_, v_, *args)[0] * do).sum())

    h = 1e-6
    rng = np.random.default_rng(0)
    for grad, idx in ((dq, 0), (dk, 1), (dv, 2)):
        for _ in range(6):
            pos = tuple(int(rng.integers(0, s)) for s in grad.shape)
            xs = [q.copy(), k.copy(), v.copy()]
            xs[idx][pos] += h
            up = loss(*xs)
            xs[idx][pos] -= 2 * h
            dn = loss(*xs)
            fd = (up - dn) / (2 * h)
            assert abs(fd - grad[pos]) <= 1e-6 * max(1.0, abs(fd))
