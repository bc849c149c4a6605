"""Pins for the CPU oracle: values and properties fixed by the pages and by the
mathematics, chosen so that a dropped term, a wrong sign or index, or a
transposed operand in the oracle fails at least one of them."""

import math

import numpy as np
import pytest
import torch

import oracle
from conftest import read_golden

RNG = np.random.default_rng(12345)


def _rand(*shape):
    return RNG.standard_normal(shape)


# ---------------------------------------------------------------------------
# Worked examples printed on the pages
# ---------------------------------------------------------------------------

def test_two_tile_example_intermediates():
    g = read_golden("two_tile_example.txt")
    out, lse, hist = oracle.online_softmax_row(g["scores"], g["values"], int(g["tile"]))
    m1, l1, u1, _ = hist[0]
    nd = int(g["decimals"])
    assert m1 == g["after_tile1_m"]
    assert round(l1, nd) == g["after_tile1_l"]
    assert round(u1, nd) == g["after_tile1_u"]
    # The page's closed forms for the state after tile 2.
    l2 = math.exp(-1) * (1 + math.exp(-1)) + 1 + math.exp(-3)
    u2 = math.exp(-1) * (10 + 20 * math.exp(-1)) + 30 + 40 * math.exp(-3)
    m_final, l_final, u_final, _ = hist[1]
    assert m_final == 3.0
    assert math.isclose(l_final, l2, rel_tol=1e-14)
    assert math.isclose(u_final, u2, rel_tol=1e-14)
    # The page's assertion: the tiled result equals the full-row softmax, rel 1e-12.
    assert math.isclose(out, u2 / l2, rel_tol=1e-12)
    assert math.isclose(lse, 3.0 + math.log(l2), rel_tol=1e-14)


def test_two_tile_example_through_attention_definition():
    """The same row as a 1-query attention with d=1, q=1, keys=scores, scale=1."""
    g = read_golden("two_tile_example.txt")
    l2 = math.exp(-1) * (1 + math.exp(-1)) + 1 + math.exp(-3)
    u2 = math.exp(-1) * (10 + 20 * math.exp(-1)) + 30 + 40 * math.exp(-3)
    q = np.ones((1, 1, 1, 1))
    k = np.array(g["scores"]).reshape(1, 4, 1, 1)
    v = np.array(g["values"]).reshape(1, 4, 1, 1)
    O, LSE = oracle.attention_forward(q, k, v, 1.0, False)
    assert math.isclose(O[0, 0, 0, 0], u2 / l2, rel_tol=1e-12)
    assert math.isclose(O[0, 0, 0, 0], 24.71148648358232, rel_tol=1e-12)
    assert math.isclose(LSE[0, 0, 0], 3.0 + math.log(l2), rel_tol=1e-14)


def test_eight_key_example_every_tile_size():
    g = read_golden("eight_key_example.txt")
    nd = int(g["decimals"])
    out4, _, hist = oracle.online_softmax_row(g["scores"], g["values"], int(g["tile"]))
    assert hist[0][0] == g["after_tile1_max"]
    assert round(hist[0][3], nd) == g["after_tile1_output"]
    assert round(out4, nd) == g["final_output"]
    outs = []
    for tile in range(1, 9):
        o, lse, _ = oracle.online_softmax_row(g["scores"], g["values"], tile)
        assert round(o, nd) == g["final_output"]
        outs.append((o, lse))
    ref_o, ref_lse = oracle.brute_force_row(g["scores"], g["values"])
    for o, lse in outs:
        assert math.isclose(o, ref_o, rel_tol=1e-13)
        assert math.isclose(lse, ref_lse, rel_tol=1e-13)
    # and the attention definition agrees
    q = np.ones((1, 1, 1, 1))
    k = np.array(g["scores"]).reshape(1, 8, 1, 1)
    v = np.array(g["values"]).reshape(1, 8, 1, 1)
    O, LSE = oracle.attention_forward(q, k, v, 1.0, False)
    assert round(O[0, 0, 0, 0], nd) == g["final_output"]
    assert math.isclose(LSE[0, 0, 0], ref_lse, rel_tol=1e-14)


def test_online_softmax_vector_values_match_definition():
    s = _rand(37) * 3
    vals = _rand(37, 5)
    ref_w = np.exp(s - s.max())
    ref = (ref_w[:, None] * vals).sum(0) / ref_w.sum()
    for tile in (1, 3, 8, 37, 64):
        o, lse, _ = oracle.online_softmax_row(s, vals, tile)
        np.testing.assert_allclose(o, ref, rtol=1e-12, atol=1e-13)
        assert math.isclose(lse, s.max() + math.log(ref_w.sum()), rel_tol=1e-13)


# ---------------------------------------------------------------------------
# Brute force on tiny inputs (pure-Python loops), including the causal rule
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("Tq,Tk,causal", [(5, 5, False), (5, 5, True), (3, 6, True), (1, 4, True)])
def test_forward_matches_brute_force(Tq, Tk, causal):
    d = 3
    q, k, v = _rand(1, Tq, 1, d), _rand(1, Tk, 1, d), _rand(1, Tk, 1, d)
    s = 0.7
    O, LSE = oracle.attention_forward(q, k, v, s, causal)
    for i in range(Tq):
        keys = [j for j in range(Tk) if (not causal) or j <= i + Tk - Tq]
        scores = [s * sum(q[0, i, 0, c] * k[0, j, 0, c] for c in range(d)) for j in keys]
        for c in range(d):
            o, lse = oracle.brute_force_row(scores, [v[0, j, 0, c] for j in keys])
            assert math.isclose(O[0, i, 0, c], o, rel_tol=1e-12, abs_tol=1e-13)
        assert math.isclose(LSE[0, 0, i], lse, rel_tol=1e-13)


def test_causal_rule_position_three():
    """A query at position 3 uses columns 0..3 and ignores 4 and later."""
    assert [j for j in range(8) if oracle.causal_visible(3, j, 8, 8)] == [0, 1, 2, 3]
    # changing a future key/value must not change row 3
    q, k, v = _rand(1, 8, 1, 4), _rand(1, 8, 1, 4), _rand(1, 8, 1, 4)
    O1, L1 = oracle.attention_forward(q, k, v, 0.5, True)
    k2, v2 = k.copy(), v.copy()
    k2[0, 4:] += 10.0
    v2[0, 4:] -= 3.0
    O2, L2 = oracle.attention_forward(q, k2, v2, 0.5, True)
    np.testing.assert_array_equal(O1[0, :4], O2[0, :4])
    np.testing.assert_array_equal(L1[0, 0, :4], L2[0, 0, :4])
    assert not np.allclose(O1[0, 4:], O2[0, 4:])


# ---------------------------------------------------------------------------
# Invariants and degenerate cases
# ---------------------------------------------------------------------------

def test_probability_rows_sum_to_one_and_dv_sum():
    B, T, H, d = 2, 9, 2, 4
    q, k, v, do = _rand(B, T, H, d), _rand(B, T, H, d), _rand(B, T, H, d), _rand(B, T, H, d)
    for causal in (False, True):
        # P rows sum to 1: O of V = all-ones is all-ones
        O, _ = oracle.attention_forward(q, k, np.ones_like(v), 0.3, causal)
        np.testing.assert_allclose(O, 1.0, rtol=0, atol=1e-14)
        # sum_j dV_j = sum_i dO_i because P is row-stochastic
        _, _, dv = oracle.attention_backward(q, k, v, do, 0.3, causal)
        np.testing.assert_allclose(dv.sum(axis=1), do.sum(axis=1), rtol=1e-12, atol=1e-12)


def test_equal_scores_give_mean_of_values():
    T, d = 7, 3
    q = np.zeros((1, T, 1, d))
    k, v = _rand(1, T, 1, d), _rand(1, T, 1, d)
    O, LSE = oracle.attention_forward(q, k, v, 0.9, False)
    np.testing.assert_allclose(O[0, :, 0], np.broadcast_to(v[0, :, 0].mean(0), (T, d)), rtol=1e-13)
    np.testing.assert_allclose(LSE[0, 0], math.log(T), rtol=1e-14)
    O, LSE = oracle.attention_forward(q, k, v, 0.9, True)
    for i in range(T):
        np.testing.assert_allclose(O[0, i, 0], v[0, :i + 1, 0].mean(0), rtol=1e-12, atol=1e-14)
        assert math.isclose(LSE[0, 0, i], math.log(i + 1), rel_tol=1e-13, abs_tol=1e-15)


def test_single_key_and_first_causal_row():
    q, k, v = _rand(1, 1, 1, 4), _rand(1, 1, 1, 4), _rand(1, 1, 1, 4)
    O, LSE = oracle.attention_forward(q, k, v, 0.5, False)
    np.testing.assert_allclose(O[0, 0, 0], v[0, 0, 0], rtol=1e-15)
    assert math.isclose(LSE[0, 0, 0], 0.5 * float(q[0, 0, 0] @ k[0, 0, 0]), rel_tol=1e-14)
    q, k, v = _rand(1, 6, 1, 4), _rand(1, 6, 1, 4), _rand(1, 6, 1, 4)
    O, LSE = oracle.attention_forward(q, k, v, 0.5, True)
    np.testing.assert_allclose(O[0, 0, 0], v[0, 0, 0], rtol=1e-15)
    assert math.isclose(LSE[0, 0, 0], 0.5 * float(q[0, 0, 0] @ k[0, 0, 0]), rel_tol=1e-14)


def test_fully_masked_rows_are_zero():
    """Causal with Tq > Tk: the first Tq-Tk rows see no key -> O=0, LSE=-inf, zero grads."""
    Tq, Tk, d = 6, 3, 2
    q, k, v, do = _rand(1, Tq, 1, d), _rand(1, Tk, 1, d), _rand(1, Tk, 1, d), _rand(1, Tq, 1, d)
    O, LSE = oracle.attention_forward(q, k, v, 1.0, True)
    assert np.all(O[0, :Tq - Tk] == 0) and np.all(np.isneginf(LSE[0, 0, :Tq - Tk]))
    assert np.all(np.isfinite(LSE[0, 0, Tq - Tk:]))
    dq, dk, dv = oracle.attention_backward(q, k, v, do, 1.0, True)
    assert np.all(dq[0, :Tq - Tk] == 0)
    # Tk == 0
    O, LSE = oracle.attention_forward(q, k[:, :0], v[:, :0], 1.0, False)
    assert np.all(O == 0) and np.all(np.isneginf(LSE))


def test_key_permutation_and_shift_invariance():
    B, T, H, d = 1, 10, 1, 5
    q, k, v, do = _rand(B, T, H, d), _rand(B, T, H, d), _rand(B, T, H, d), _rand(B, T, H, d)
    s = 0.4
    O, LSE = oracle.attention_forward(q, k, v, s, False)
    dq, dk, dv = oracle.attention_backward(q, k, v, do, s, False)
    perm = RNG.permutation(T)
    O2, LSE2 = oracle.attention_forward(q, k[:, perm], v[:, perm], s, False)
    dq2, dk2, dv2 = oracle.attention_backward(q, k[:, perm], v[:, perm], do, s, False)
    np.testing.assert_allclose(O2, O, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(LSE2, LSE, rtol=1e-13)
    np.testing.assert_allclose(dq2, dq, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(dk2, dk[:, perm], rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(dv2, dv[:, perm], rtol=1e-11, atol=1e-12)
    # shift: K + w leaves O unchanged and shifts LSE_i by s q_i . w
    w = _rand(d)
    O3, LSE3 = oracle.attention_forward(q, k + w, v, s, False)
    np.testing.assert_allclose(O3, O, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(LSE3[0, 0], LSE[0, 0] + s * (q[0, :, 0] @ w), rtol=1e-12, atol=1e-12)


# ---------------------------------------------------------------------------
# Backward: finite differences, dK column sums, library cross-check, GQA
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("causal", [False, True])
def test_backward_finite_differences(causal):
    B, T, H, d = 1, 6, 1, 3
    q, k, v, do = _rand(B, T, H, d), _rand(B, T, H, d), _rand(B, T, H, d), _rand(B, T, H, d)
    s = 0.6

    def loss(q_, k_, v_):
        return float((oracle.attention_forward(q_, k_, v_, s, causal)[0] * do).sum())

    dq, dk, dv = oracle.attention_backward(q, k, v, do, s, causal)
    eps = 1e-5
    for name, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        num = np.zeros_like(x)
        for idx in np.ndindex(x.shape):
            xp, xm = x.copy(), x.copy()
            xp[idx] += eps
            xm[idx] -= eps
            args_p = {"q": q, "k": k, "v": v}
            args_m = dict(args_p)
            args_p[name], args_m[name] = xp, xm
            num[idx] = (loss(**{a + "_": b for a, b in args_p.items()})
                        - loss(**{a + "_": b for a, b in args_m.items()})) / (2 * eps)
        rel = np.linalg.norm(num - g) / np.linalg.norm(g)
        assert rel <= 1e-6, (name, rel)


def test_dk_columns_sum_to_zero():
    """Each dS row sums to zero, so sum_j dK_j = 0 for every KV head."""
    B, T, Hq, Hkv, d = 2, 8, 4, 2, 3
    q, do = _rand(B, T, Hq, d), _rand(B, T, Hq, d)
    k, v = _rand(B, T, Hkv, d), _rand(B, T, Hkv, d)
    for causal in (False, True):
        _, dk, _ = oracle.attention_backward(q, k, v, do, 0.5, causal)
        np.testing.assert_allclose(dk.sum(axis=1), 0.0, atol=1e-12)


@pytest.mark.parametrize("causal", [False, True])
def test_matches_torch_float64_sdpa(causal):
    """Library special case: PyTorch's math SDPA + autograd in float64."""
    B, T, H, d = 2, 7, 3, 4
    q, k, v, do = _rand(B, T, H, d), _rand(B, T, H, d), _rand(B, T, H, d), _rand(B, T, H, d)
    s = 0.45
    O, LSE = oracle.attention_forward(q, k, v, s, causal)
    dq, dk, dv = oracle.attention_backward(q, k, v, do, s, causal)
    tq, tk, tv = (torch.tensor(x.transpose(0, 2, 1, 3), requires_grad=True) for x in (q, k, v))
    to = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, is_causal=causal, scale=s)
    to.backward(torch.tensor(do.transpose(0, 2, 1, 3)))
    np.testing.assert_allclose(O, to.detach().numpy().transpose(0, 2, 1, 3), rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(dq, tq.grad.numpy().transpose(0, 2, 1, 3), rtol=1e-10, atol=1e-11)
    np.testing.assert_allclose(dk, tk.grad.numpy().transpose(0, 2, 1, 3), rtol=1e-10, atol=1e-11)
    np.testing.assert_allclose(dv, tv.grad.numpy().transpose(0, 2, 1, 3), rtol=1e-10, atol=1e-11)
    # LSE from the library's own logsumexp of the masked scaled scores
    S = torch.tensor(q.transpose(0, 2, 1, 3)) @ torch.tensor(k.transpose(0, 2, 3, 1)) * s
    if causal:
        S = S.masked_fill(torch.ones(T, T, dtype=torch.bool).triu(1), float("-inf"))
    np.testing.assert_allclose(LSE, torch.logsumexp(S, dim=-1).numpy(), rtol=1e-13)


def test_gqa_equals_repeated_heads():
    B, T, Hq, Hkv, d = 1, 6, 6, 2, 3
    G = Hq // Hkv
    q, do = _rand(B, T, Hq, d), _rand(B, T, Hq, d)
    k, v = _rand(B, T, Hkv, d), _rand(B, T, Hkv, d)
    krep, vrep = np.repeat(k, G, axis=2), np.repeat(v, G, axis=2)
    for causal in (False, True):
        O, LSE = oracle.attention_forward(q, k, v, 0.5, causal)
        Or, LSEr = oracle.attention_forward(q, krep, vrep, 0.5, causal)
        np.testing.assert_array_equal(O, Or)
        np.testing.assert_array_equal(LSE, LSEr)
        dq, dk, dv = oracle.attention_backward(q, k, v, do, 0.5, causal)
        dqr, dkr, dvr = oracle.attention_backward(q, krep, vrep, do, 0.5, causal)
        np.testing.assert_allclose(dq, dqr, rtol=1e-13, atol=1e-14)
        np.testing.assert_allclose(dk, dkr.reshape(B, T, Hkv, G, d).sum(3), rtol=1e-12, atol=1e-13)
        np.testing.assert_allclose(dv, dvr.reshape(B, T, Hkv, G, d).sum(3), rtol=1e-12, atol=1e-13)


# ---------------------------------------------------------------------------
# Decode and the split-KV combine
# ---------------------------------------------------------------------------

def test_split_kv_any_chunk_size():
    n, d = 300, 4
    q = _rand(d)
    kk, vv = _rand(n, d), _rand(n, d)
    s = 0.5
    o_ref, lse_ref = oracle.head_forward(q[None], kk, vv, s, False)
    for chunk in (1, 7, 256, n):
        parts_o, parts_l = [], []
        for c0 in range(0, n, chunk):
            o, l = oracle.head_forward(q[None], kk[c0:c0 + chunk], vv[c0:c0 + chunk], s, False)
            parts_o.append(o[0])
            parts_l.append(l[0])
        o, lse = oracle.combine_partials(parts_o, parts_l)
        np.testing.assert_allclose(o, o_ref[0], rtol=1e-12, atol=1e-13)
        assert math.isclose(lse, lse_ref[0], rel_tol=1e-13)


def test_combine_reproduces_two_tile_example():
    g = read_golden("two_tile_example.txt")
    sc, vals = g["scores"], g["values"]
    parts = [oracle.brute_force_row(sc[i:i + 2], vals[i:i + 2]) for i in (0, 2)]
    o, lse = oracle.combine_partials([[p[0]] for p in parts], [p[1] for p in parts])
    l2 = math.exp(-1) * (1 + math.exp(-1)) + 1 + math.exp(-3)
    u2 = math.exp(-1) * (10 + 20 * math.exp(-1)) + 30 + 40 * math.exp(-3)
    assert math.isclose(o[0], u2 / l2, rel_tol=1e-12)
    assert math.isclose(lse, 3.0 + math.log(l2), rel_tol=1e-14)


def test_decode_is_prefill_row_over_prefix():
    B, Hq, Hkv, d, Tmax = 3, 4, 2, 5, 40
    q = _rand(B, Hq, d)
    kc, vc = _rand(B, Tmax, Hkv, d), _rand(B, Tmax, Hkv, d)
    seqlens = [1, 17, 40]
    O, LSE = oracle.decode_forward(q, kc, vc, seqlens, 0.3)
    for b in range(B):
        n = seqlens[b]
        # garbage beyond the prefix must not matter
        kc2, vc2 = kc.copy(), vc.copy()
        kc2[b, n:] = 1e3
        vc2[b, n:] = -1e3
        O2, LSE2 = oracle.decode_forward(q, kc2, vc2, seqlens, 0.3)
        np.testing.assert_array_equal(O2[b], O[b])
        for h in range(Hq):
            g = h // (Hq // Hkv)
            Ob, Lb = oracle.attention_forward(q[b, h][None, None, None], kc[b, :n, g][None, :, None],
                                              vc[b, :n, g][None, :, None], 0.3, False)
            np.testing.assert_allclose(O[b, h], Ob[0, 0, 0], rtol=1e-13, atol=1e-14)
            assert math.isclose(LSE[b, h], Lb[0, 0, 0], rel_tol=1e-14)
    np.testing.assert_allclose(O[0], np.repeat(vc[0, 0], Hq // Hkv, axis=0), rtol=1e-15)


def test_merge_of_key_shares_is_full_decode():
    """Decoding disjoint shares of every sequence's keys (any split, empty
    shares included) and merging the shares' (O, LSE) by log-sum-exp gives
    the decode over all keys: the softmax over a union of key sets."""
    rng = np.random.default_rng(11)
    B, Hq, Hkv, d, Tmax, R = 3, 4, 2, 5, 50, 3
    q = rng.standard_normal((B, Hq, d))
    kc, vc = rng.standard_normal((B, Tmax, Hkv, d)), rng.standard_normal((B, Tmax, Hkv, d))
    seqlens = [1, 23, 50]
    O_ref, L_ref = oracle.decode_forward(q, kc, vc, seqlens, 0.4)
    for contiguous in (True, False):
        shares = [[] for _ in range(R)]
        for b, n in enumerate(seqlens):
            pos = np.arange(n) if contiguous else rng.permutation(n)
            cuts = sorted(rng.integers(0, n + 1, size=R - 1)) if not contiguous else [n // 3, 2 * n // 3]
            for r, part in enumerate(np.split(pos, cuts)):
                shares[r].append(part)
        o_parts, l_parts = [], []
        for r in range(R):
            ks, vs = np.zeros_like(kc), np.zeros_like(vc)
            sl = []
            for b in range(B):
                idx = shares[r][b]
                ks[b, :len(idx)], vs[b, :len(idx)] = kc[b, idx], vc[b, idx]
                sl.append(len(idx))
            o, l = oracle.decode_forward(q, ks, vs, sl, 0.4)
            o_parts.append(o)
            l_parts.append(l)
        assert any(len(shares[r][0]) == 0 for r in range(R))   # sequence 0 has empty shares
        O, L = oracle.merge_partials(np.stack(o_parts), np.stack(l_parts))
        np.testing.assert_allclose(O, O_ref, rtol=1e-12, atol=1e-13)
        np.testing.assert_allclose(L, L_ref, rtol=1e-13)


def test_merge_closed_forms():
    # weights e^{LSE_r}: LSE = (0, ln 3) puts 1/4 and 3/4 on the two partials
    O, L = oracle.merge_partials(np.array([[[1.0, 0.0]], [[0.0, 1.0]]]), np.array([[0.0], [math.log(3.0)]]))
    np.testing.assert_allclose(O[0], [0.25, 0.75], rtol=1e-15)
    assert math.isclose(L[0], math.log(4.0), rel_tol=1e-15)
    # two equal partials: the same output, LSE + ln 2
    o = np.array([[0.3, -1.2, 4.0]])
    O, L = oracle.merge_partials(np.stack([o, o]), np.array([[1.7], [1.7]]))
    np.testing.assert_allclose(O, o, rtol=1e-15)
    assert math.isclose(L[0], 1.7 + math.log(2.0), rel_tol=1e-15)
    # a partial that saw no key (LSE = -inf) changes nothing; all of them empty gives 0, -inf
    O, L = oracle.merge_partials(np.stack([o, np.zeros_like(o)]), np.array([[0.5], [-np.inf]]))
    np.testing.assert_allclose(O, o, rtol=1e-15)
    assert L[0] == 0.5
    O, L = oracle.merge_partials(np.zeros((3, 1, 3)), np.full((3, 1), -np.inf))
    assert (O == 0).all() and L[0] == -np.inf


def test_row_panels_do_not_change_results():
    """Rows are processed in panels; a long causal head must equal the
    brute-force row for rows in different panels."""
    T, d = 2100, 2
    q, k, v = _rand(T, d), _rand(T, d), _rand(T, d)
    O, LSE = oracle.head_forward(q, k, v, 0.5, True)
    for i in (0, 1, 2047, 2048, 2099):
        scores = list(0.5 * (k[:i + 1] @ q[i]))
        o0, l0 = oracle.brute_force_row(scores, list(v[:i + 1, 0]))
        assert math.isclose(O[i, 0], o0, rel_tol=1e-11, abs_tol=1e-12)
        assert math.isclose(LSE[i], l0, rel_tol=1e-12)
    Os, Ls = oracle.head_forward(q, k, v, 0.5, True, rows=[5, 2099, 3000 - 1000])
    np.testing.assert_array_equal(Os[1], O[2099])
    np.testing.assert_array_equal(Ls[2], LSE[2000])


# ---------------------------------------------------------------------------
# Sliding window (causal local window of W keys; reading of [FA "In practice"])
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("Tq,Tk,W", [(6, 6, 1), (6, 6, 3), (4, 7, 2), (5, 5, 5), (3, 8, 4)])
def test_window_matches_brute_force(Tq, Tk, W):
    """Each row is the softmax over exactly its W most recent visible keys,
    computed term by term in pure Python."""
    d = 3
    q, k, v = _rand(1, Tq, 1, d), _rand(1, Tk, 1, d), _rand(1, Tk, 1, d)
    s = 0.8
    O, LSE = oracle.attention_forward(q, k, v, s, True, window=W)
    off = Tk - Tq
    for i in range(Tq):
        keys = [j for j in range(Tk) if i + off - W < j <= i + off]
        if not keys:
            assert np.all(O[0, i, 0] == 0.0) and LSE[0, 0, i] == -np.inf
            continue
        scores = [s * sum(q[0, i, 0, c] * k[0, j, 0, c] for c in range(d)) for j in keys]
        for c in range(d):
            o, lse = oracle.brute_force_row(scores, [v[0, j, 0, c] for j in keys])
            assert math.isclose(O[0, i, 0, c], o, rel_tol=1e-12, abs_tol=1e-13)
        assert math.isclose(LSE[0, 0, i], lse, rel_tol=1e-13)


def test_window_of_one_key_is_the_diagonal():
    """W = 1: every row sees only its diagonal key, so O_i = V_{i+off},
    LSE_i is that single score, dQ = dK = 0 and dV_j = dO of the row that sees j."""
    Tq, Tk, d = 5, 7, 4
    q, k, v, do = _rand(1, Tq, 2, d), _rand(1, Tk, 2, d), _rand(1, Tk, 2, d), _rand(1, Tq, 2, d)
    s = 0.4
    O, LSE = oracle.attention_forward(q, k, v, s, True, window=1)
    off = Tk - Tq
    np.testing.assert_array_equal(O[0], v[0, off:])
    np.testing.assert_allclose(LSE[0], s * np.einsum("thd,thd->ht", q[0], k[0, off:]), rtol=1e-14)
    dq, dk, dv = oracle.attention_backward(q, k, v, do, s, True, window=1)
    assert np.abs(dq).max() == 0.0 and np.abs(dk).max() == 0.0
    np.testing.assert_array_equal(dv[0, off:], do[0])
    assert np.abs(dv[0, :off]).max() == 0.0


def test_window_covering_all_keys_is_causal():
    B, T, H, d = 2, 9, 2, 3
    q, k, v, do = _rand(B, T, H, d), _rand(B, T, H, d), _rand(B, T, H, d), _rand(B, T, H, d)
    a = oracle.attention_forward(q, k, v, 0.5, True)
    b = oracle.attention_forward(q, k, v, 0.5, True, window=T)
    np.testing.assert_array_equal(a[0], b[0])
    np.testing.assert_array_equal(a[1], b[1])
    ga = oracle.attention_backward(q, k, v, do, 0.5, True)
    gb = oracle.attention_backward(q, k, v, do, 0.5, True, window=T + 3)
    for x, y in zip(ga, gb):
        np.testing.assert_array_equal(x, y)


def test_window_row_equals_unmasked_attention_over_its_slice():
    """A windowed row is plain (unmasked) attention over the key slice
    [i + off - W + 1, i + off]."""
    Tq, Tk, d, W = 40, 50, 3, 7
    q, k, v = _rand(Tq, d), _rand(Tk, d), _rand(Tk, d)
    O, LSE = oracle.head_forward(q, k, v, 0.3, True, window=W)
    off = Tk - Tq
    for i in (0, 1, 13, 39):
        lo, hi = max(0, i + off - W + 1), i + off + 1
        Oi, Li = oracle.head_forward(q[i:i + 1], k[lo:hi], v[lo:hi], 0.3, False)
        np.testing.assert_allclose(O[i], Oi[0], rtol=1e-13, atol=1e-15)
        assert math.isclose(LSE[i], Li[0], rel_tol=1e-14)


def test_window_backward_finite_differences():
    B, T, H, d, W = 1, 7, 1, 3, 3
    q, k, v, do = _rand(B, T, H, d), _rand(B, T, H, d), _rand(B, T, H, d), _rand(B, T, H, d)
    s = 0.6

    def loss(q_, k_, v_):
        return float((oracle.attention_forward(q_, k_, v_, s, True, window=W)[0] * do).sum())

    dq, dk, dv = oracle.attention_backward(q, k, v, do, s, True, window=W)
    eps = 1e-5
    for name, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        num = np.zeros_like(x)
        for idx in np.ndindex(x.shape):
            args_p = {"q_": q, "k_": k, "v_": v}
            args_m = dict(args_p)
            xp, xm = x.copy(), x.copy()
            xp[idx] += eps
            xm[idx] -= eps
            args_p[name + "_"], args_m[name + "_"] = xp, xm
            num[idx] = (loss(**args_p) - loss(**args_m)) / (2 * eps)
        rel = np.linalg.norm(num - g) / np.linalg.norm(g)
        assert rel <= 1e-6, (name, rel)


def test_window_decode_is_last_prefill_row():
    """Decode with a window sees the last W keys of the sequence, i.e. the
    last row of a windowed prefill over the prefix."""
    B, Hq, Hkv, d, Tmax, W = 3, 4, 2, 3, 30, 5
    q = _rand(B, Hq, d)
    kc, vc = _rand(B, Tmax, Hkv, d), _rand(B, Tmax, Hkv, d)
    seqlens = [2, 11, 30]
    O, LSE = oracle.decode_forward(q, kc, vc, seqlens, 0.3, window=W)
    for b in range(B):
        n = seqlens[b]
        for h in range(Hq):
            g = h // (Hq // Hkv)
            lo = max(0, n - W)
            Ob, Lb = oracle.head_forward(q[b, h][None, :], kc[b, lo:n, g], vc[b, lo:n, g], 0.3, False)
            np.testing.assert_allclose(O[b, h], Ob[0], rtol=1e-13, atol=1e-15)
            assert math.isclose(LSE[b, h], Lb[0], rel_tol=1e-14)


# ---------------------------------------------------------------------------
# E4M3 decoding and the FP8 forward's reference
# ---------------------------------------------------------------------------

def test_e4m3_closed_forms():
    v = oracle.e4m3_value
    assert v(0x38) == 1.0 and v(0xB8) == -1.0          # E = 7, M = 0
    assert v(0x7E) == 448.0 and v(0xFE) == -448.0      # the largest finite value
    assert v(0x08) == 2.0 ** -6                        # the smallest normal
    assert v(0x01) == 2.0 ** -9 and v(0x07) == 7 * 2.0 ** -9   # subnormals
    assert v(0x00) == 0.0 and math.copysign(1.0, v(0x80)) == -1.0
    assert math.isnan(v(0x7F)) and math.isnan(v(0xFF))
    assert v(0x78) == 256.0 and v(0x3C) == 1.5 and v(0x40) == 2.0
    vals = [v(c) for c in range(0x7F)]
    assert all(a < b for a, b in zip(vals, vals[1:]))  # codes 0..126 increase


def test_e4m3_decode_matches_torch_conversion():
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    ours = oracle.e4m3_decode(codes.numpy())
    nan = np.isnan(ref)
    assert np.array_equal(nan, np.isnan(ours)) and nan.sum() == 2
    np.testing.assert_array_equal(ours[~nan], ref[~nan])


def test_e4m3_attention_descale_factors():
    """The factors act where the definition puts them: q and k scale the
    scores (doubling q's equals doubling the softmax scale), v scales O
    linearly and leaves LSE alone."""
    rng = np.random.default_rng(8)
    B, T, H, d = 1, 9, 2, 4
    q8, k8, v8 = (rng.integers(0, 0x7F, size=(B, T, H, d)) | (rng.integers(0, 2, size=(B, T, H, d)) << 7)
                  for _ in range(3))
    O, L = oracle.attention_forward_e4m3(q8, k8, v8, 0.01, 0.02, 0.5, 0.3, True)
    O2, L2 = oracle.attention_forward_e4m3(q8, k8, v8, 0.02, 0.02, 1.5, 0.3, True)
    O3, L3 = oracle.attention_forward_e4m3(q8, k8, v8, 0.01, 0.02, 1.5, 0.6, True)
    np.testing.assert_allclose(O2, O3, rtol=1e-13)
    np.testing.assert_allclose(L2, L3, rtol=1e-13)
    Ob, Lb = oracle.attention_forward_e4m3(q8, k8, v8, 0.01, 0.02, 1.5, 0.3, True)
    np.testing.assert_allclose(Ob, 3.0 * O, rtol=1e-13)
    np.testing.assert_array_equal(Lb, L)
    # first causal row sees key 0 only: O = that value row
    np.testing.assert_allclose(O[0, 0], oracle.e4m3_decode(v8[0, 0]) * 0.5, rtol=1e-15)
