"""Seeded random shapes: forward and backward (default and deterministic)
through the C ABI against the float64 oracle, on problem shapes drawn from a
fixed generator -- batch, query and KV heads (every GQA ratio that divides),
query and key lengths that are rarely multiples of the 128-row tile, head
size, causal or not, and sometimes a sliding window -- so that tile edges,
ragged tails and Tq != Tk meet every kernel in combinations the hand-picked
cases do not list."""

import random

import pytest
import torch

import oracle
from workloads import WORKLOADS, prefill_inputs, to_f64
from _parity import assert_grad_close, assert_lse_close, assert_o_close

pytestmark = pytest.mark.gpu

fa = pytest.importorskip("io_aware_exact_forward_b200")


def _draw(n, seed=20261203):
    rng = random.Random(seed)
    cases = []
    for i in range(n):
        hkv = rng.choice([1, 2, 3])
        g = rng.choice([1, 2, 4])
        tq = rng.randint(1, 520)
        tk = tq if rng.random() < 0.5 else rng.randint(1, 520)
        d = rng.choice([64, 128])
        causal = rng.random() < 0.6
        window = rng.choice([None, None, 1, 33, 128, 200]) if causal else None
        cases.append((i, rng.choice([1, 2]), hkv * g, hkv, tq, tk, d, causal, window))
    return cases


@pytest.mark.parametrize("i,B,Hq,Hkv,Tq,Tk,d,causal,window", _draw(24))
def test_random_shape(i, B, Hq, Hkv, Tq, Tk, d, causal, window):
    w = WORKLOADS[1].with_(B=B, Hq=Hq, Hkv=Hkv, d=d, causal=causal)
    inp = prefill_inputs(w, seed=1000 + i, Tq=Tq, Tk=Tk)
    q, k, v, do = (inp[n].cuda() for n in ("q", "k", "v", "do"))
    if window is None:
        o, lse = fa.forward(q, k, v, scale=w.scale, causal=causal)
    else:
        o, lse = fa.forward(q, k, v, scale=w.scale, window=window)
    grads = fa.backward(q, k, v, o, lse, do, scale=w.scale, causal=causal, window=window)
    det = fa.backward(q, k, v, o, lse, do, scale=w.scale, causal=causal, window=window, deterministic=True)
    torch.cuda.synchronize()
    assert fa.check() == 0
    f64 = {n: to_f64(inp[n]) for n in ("q", "k", "v", "do")}
    O, LSE = oracle.attention_forward(f64["q"], f64["k"], f64["v"], w.scale, causal, window=window)
    assert_o_close(to_f64(o), O)
    assert_lse_close(lse.cpu().numpy(), LSE)
    R = oracle.attention_backward(f64["q"], f64["k"], f64["v"], f64["do"], w.scale, causal, window=window)
    for name, x, y, r in zip(("dQ", "dK", "dV"), grads, det, R):
        assert_grad_close(to_f64(x), r, name)
        assert_grad_close(to_f64(y), r, name + " (deterministic)")
    # dK and dV are the same bits either way
    assert torch.equal(grads[1], det[1]) and torch.equal(grads[2], det[2])


def _draw_dropout(n, seed=977):
    rng = random.Random(seed)
    cases = []
    for i in range(n):
        hkv = rng.choice([1, 2])
        g = rng.choice([1, 2, 4])
        tq = rng.randint(1, 600)
        tk = tq if rng.random() < 0.5 else rng.randint(1, 600)
        cases.append((i, rng.choice([1, 2]), hkv * g, hkv, tq, tk, rng.choice([64, 128]), rng.random() < 0.5,
                      rng.choice([0.05, 0.1, 0.3, 0.6])))
    return cases


@pytest.mark.parametrize("i,B,Hq,Hkv,Tq,Tk,d,causal,p", _draw_dropout(12))
def test_random_shape_dropout(i, B, Hq, Hkv, Tq, Tk, d, causal, p):
    """fa_forward_dropout and fa_backward_dropout against the oracle's
    attention with the same Philox mask (O compared after undoing the
    256/t scale both sides apply)."""
    from oracle import dropout as dr
    w = WORKLOADS[1].with_(B=B, Hq=Hq, Hkv=Hkv, d=d, causal=causal)
    inp = prefill_inputs(w, seed=3000 + i, Tq=Tq, Tk=Tk)
    q, k, v, do = (inp[n].cuda() for n in ("q", "k", "v", "do"))
    seed, offset = 0x51DE_0000 + 17 * i, 5 + i
    o, lse = fa.forward_dropout(q, k, v, p, seed, offset, scale=w.scale, causal=causal)
    dq, dk, dv = fa.backward_dropout(q, k, v, o, lse, do, p, seed, offset, scale=w.scale, causal=causal)
    torch.cuda.synchronize()
    assert fa.check() == 0
    f64 = {n: to_f64(inp[n]) for n in ("q", "k", "v", "do")}
    O, LSE = dr.attention_forward_dropout(f64["q"], f64["k"], f64["v"], w.scale, causal, p, seed, offset)
    back = dr.keep_threshold(p) / 256.0
    assert_o_close(to_f64(o) * back, O * back)
    assert_lse_close(lse.cpu().numpy(), LSE)
    R = dr.attention_backward_dropout(f64["q"], f64["k"], f64["v"], f64["do"], w.scale, causal, p, seed, offset)
    for name, x, r in zip(("dQ", "dK", "dV"), (dq, dk, dv), R):
        assert_grad_close(to_f64(x), r, name)


def _draw_decode(n, seed=4242):
    rng = random.Random(seed)
    cases = []
    for i in range(n):
        hkv = rng.choice([1, 2, 4])
        g = rng.choice([1, 2, 4, 8])
        tk_max = rng.randint(1, 1500)
        b = rng.randint(1, 5)
        seqlens = [rng.choice([0, rng.randint(1, tk_max), tk_max]) for _ in range(b)]
        window = rng.choice([None, None, 1, 100, 700])
        cases.append((i, hkv * g, hkv, rng.choice([64, 128]), rng.choice([64, 128, 256, 512]), tk_max, seqlens,
                      window))
    return cases


@pytest.mark.parametrize("i,Hq,Hkv,d,chunk,Tk_max,seqlens,window", _draw_decode(12))
def test_random_shape_decode(i, Hq, Hkv, d, chunk, Tk_max, seqlens, window):
    """Split-KV decode (optionally windowed) against the oracle's one-token
    forward over each sequence's first seqlens[b] keys."""
    from workloads import decode_inputs
    w = WORKLOADS[5].with_(Hq=Hq, Hkv=Hkv, d=d)
    inp = decode_inputs(w, seed=5000 + i, B=len(seqlens), Tk_max=Tk_max, seqlens=seqlens)
    dev = {k: v.cuda() for k, v in inp.items()}
    o, lse = fa.decode_splitkv(dev["q"], dev["k_cache"], dev["v_cache"], dev["seqlens"], scale=w.scale,
                               chunk=chunk, window=window)
    torch.cuda.synchronize()
    assert fa.check() == 0
    O, LSE = oracle.decode_forward(to_f64(inp["q"]), to_f64(inp["k_cache"]), to_f64(inp["v_cache"]),
                                   inp["seqlens"].cpu().numpy(), w.scale, window=window)
    assert_o_close(to_f64(o), O)
    assert_lse_close(lse.cpu().numpy(), LSE)


def _draw_fp8(n, seed=808):
    rng = random.Random(seed)
    cases = []
    for i in range(n):
        hkv = rng.choice([1, 2])
        g = rng.choice([1, 2, 4])
        tq = rng.randint(1, 700)
        tk = tq if rng.random() < 0.5 else rng.randint(1, 700)
        cases.append((i, rng.choice([1, 2]), hkv * g, hkv, tq, tk, rng.random() < 0.6))
    return cases


@pytest.mark.parametrize("i,B,Hq,Hkv,Tq,Tk,causal", _draw_fp8(8))
def test_random_shape_fp8(i, B, Hq, Hkv, Tq, Tk, causal):
    """fa_forward_fp8 (d = 128) against the oracle on the dequantised inputs,
    each element under the bound E4M3 rounding of P allows."""
    from workloads import prefill_inputs_e4m3
    from test_parity_fp8 import _check_head
    w = WORKLOADS[3].with_(B=B, Hq=Hq, Hkv=Hkv, causal=causal)
    inp = prefill_inputs_e4m3(w, seed=7000 + i, Tq=Tq, Tk=Tk)
    dev = {n: (t.cuda() if torch.is_tensor(t) else t) for n, t in inp.items()}
    o, lse = fa.forward_fp8(dev["q"], dev["k"], dev["v"], inp["q_descale"], inp["k_descale"], inp["v_descale"],
                            scale=w.scale, causal=causal)
    torch.cuda.synchronize()
    assert fa.check() == 0
    for b in range(B):
        for h in range(Hq):
            _check_head(o, lse, inp, b, h, Hq // Hkv, w.scale, causal)
