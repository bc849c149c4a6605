"""Fused-dropout forward parity: fa_forward_dropout against the float64
oracle's attention with dropout on P (oracle.dropout), which draws the same
Philox-4x32-10 mask from the same (seed, offset).  The keep decisions are
integer and must agree exactly, so O agrees to the bf16 path's tolerances
(compared after undoing the 256/t scale, which both sides apply); LSE is
that of the undropped P."""

import numpy as np
import pytest
import torch

import oracle
from oracle import dropout as dr
from workloads import WORKLOADS, prefill_inputs, to_f64
from _parity import assert_grad_close, assert_lse_close, assert_o_close

pytestmark = pytest.mark.gpu

fa = pytest.importorskip("io_aware_exact_forward_b200")

CASES = [
    # B, Hq, Hkv, Tq, Tk, d, causal, p
    (1, 2, 2, 300, 300, 64, False, 0.1),
    (1, 2, 1, 517, 517, 128, True, 0.5),
    (2, 4, 2, 200, 450, 64, True, 0.3),
    (1, 2, 2, 450, 200, 128, True, 0.2),     # early rows see no key
    (1, 8, 1, 256, 256, 64, False, 0.9),     # G = 8, heavy dropout
    (1, 1, 1, 2048, 2048, 64, False, 0.25),  # long rows: many key tiles
]


@pytest.mark.parametrize("B,Hq,Hkv,Tq,Tk,d,causal,p", CASES)
def test_dropout_forward(B, Hq, Hkv, Tq, Tk, d, causal, p):
    w = WORKLOADS[2].with_(B=B, Hq=Hq, Hkv=Hkv, d=d, causal=causal)
    inp = prefill_inputs(w, seed=61 + Tq + 3 * Tk + d, Tq=Tq, Tk=Tk)
    q, k, v = (inp[n].cuda() for n in ("q", "k", "v"))
    seed, offset = 0x5EED_0000_1234 + Tq, 3 + Hq
    o, lse = fa.forward_dropout(q, k, v, p, seed, offset, scale=w.scale, causal=causal)
    assert fa.check() == 0
    O, LSE = dr.attention_forward_dropout(to_f64(inp["q"]), to_f64(inp["k"]), to_f64(inp["v"]), w.scale, causal,
                                          p, seed, offset)
    back = dr.keep_threshold(p) / 256.0
    assert_o_close(to_f64(o.cpu()) * back, O * back)
    assert_lse_close(lse.cpu().numpy(), LSE)


def test_dropout_zero_rate_is_the_plain_forward_and_masks_repeat():
    w = WORKLOADS[2].with_(B=1, Hq=2, Hkv=2, d=64, causal=True)
    inp = prefill_inputs(w, seed=5, Tq=384, Tk=384)
    q, k, v = (inp[n].cuda() for n in ("q", "k", "v"))
    o0, l0 = fa.forward(q, k, v, scale=w.scale, causal=True)
    o1, l1 = fa.forward_dropout(q, k, v, 0.0, 99, 0, scale=w.scale, causal=True)
    a, la = fa.forward_dropout(q, k, v, 0.4, 99, 0, scale=w.scale, causal=True)
    b, lb = fa.forward_dropout(q, k, v, 0.4, 99, 0, scale=w.scale, causal=True)
    c, _ = fa.forward_dropout(q, k, v, 0.4, 99, 1, scale=w.scale, causal=True)
    assert fa.check() == 0
    assert torch.equal(o0, o1) and torch.equal(l0, l1)
    assert torch.equal(a, b) and torch.equal(la, lb) and torch.equal(la, l0)
    assert not torch.equal(a, c)


BWD_CASES = [
    # B, Hq, Hkv, Tq, Tk, d, causal, p
    (1, 2, 2, 300, 300, 64, False, 0.1),
    (1, 2, 1, 517, 517, 128, True, 0.5),
    (2, 4, 2, 200, 450, 64, True, 0.3),      # GQA, Tq < Tk
    (1, 2, 2, 450, 200, 128, True, 0.2),     # Tq > Tk: early rows see no key
    (1, 8, 1, 256, 256, 64, False, 0.9),     # G = 8, heavy dropout
    (1, 2, 2, 1024, 1024, 64, False, 0.25),  # several key and query tiles
    (1, 4, 4, 640, 640, 128, False, 0.1),
]


@pytest.mark.parametrize("B,Hq,Hkv,Tq,Tk,d,causal,p", BWD_CASES)
def test_dropout_backward(B, Hq, Hkv, Tq, Tk, d, causal, p):
    """fa_backward_dropout after fa_forward_dropout with the same (p, seed,
    offset) against the oracle's backward with the same Philox mask."""
    w = WORKLOADS[2].with_(B=B, Hq=Hq, Hkv=Hkv, d=d, causal=causal)
    inp = prefill_inputs(w, seed=83 + Tq + 5 * Tk + d, Tq=Tq, Tk=Tk)
    q, k, v, do = (inp[n].cuda() for n in ("q", "k", "v", "do"))
    seed, offset = 0x0DD5_EED5_0000 + 7 * Tq, 11 + Hq
    o, lse = fa.forward_dropout(q, k, v, p, seed, offset, scale=w.scale, causal=causal)
    dq, dk, dv = fa.backward_dropout(q, k, v, o, lse, do, p, seed, offset, scale=w.scale, causal=causal)
    assert fa.check() == 0
    f64 = {n: to_f64(inp[n]) for n in ("q", "k", "v", "do")}
    rq, rk, rv = dr.attention_backward_dropout(f64["q"], f64["k"], f64["v"], f64["do"], w.scale, causal, p, seed,
                                               offset)
    for name, x, r in (("dQ", dq, rq), ("dK", dk, rk), ("dV", dv, rv)):
        assert_grad_close(to_f64(x.cpu()), r, name)


def test_dropout_backward_zero_rate_is_the_plain_backward():
    w = WORKLOADS[2].with_(B=1, Hq=2, Hkv=1, d=64, causal=True)
    inp = prefill_inputs(w, seed=9, Tq=384, Tk=384)
    q, k, v, do = (inp[n].cuda() for n in ("q", "k", "v", "do"))
    o, lse = fa.forward(q, k, v, scale=w.scale, causal=True)
    g0 = fa.backward(q, k, v, o, lse, do, scale=w.scale, causal=True)
    g1 = fa.backward_dropout(q, k, v, o, lse, do, 0.0, 1234, 5, scale=w.scale, causal=True)
    assert fa.check() == 0
    for a, b in zip(g0, g1):
        # dQ adds fp32 contributions in an unspecified order; dK and dV are exact
        assert torch.allclose(a.float(), b.float(), rtol=1e-2, atol=1e-3)
    assert torch.equal(g0[1], g1[1]) and torch.equal(g0[2], g1[2])


def test_dropout_persistent_items_d64():
    """d = 64 runs persistently (one CTA per SM walks several items), and its
    keep bits come from dedicated warps through double-buffered shared
    memory that carries over from one item to the next.  With 256 forward
    and 512 backward items on 148 SMs, the heads checked here are second or
    later items of their CTAs; each is compared with the oracle's per-head
    dropout forward and backward (same Philox mask, bh = b * Hq + h)."""
    B, H, T, d, p = 4, 16, 1024, 64, 0.1
    w = WORKLOADS[2].with_(B=B, Hq=H, Hkv=H, d=d, causal=False)
    inp = prefill_inputs(w, seed=1234, Tq=T, Tk=T)
    q, k, v, do = (inp[n].cuda() for n in ("q", "k", "v", "do"))
    seed, offset = 0x1234_5678_9ABC, 7
    o, lse = fa.forward_dropout(q, k, v, p, seed, offset, scale=w.scale, causal=False)
    dq, dk, dv = fa.backward_dropout(q, k, v, o, lse, do, p, seed, offset, scale=w.scale, causal=False)
    assert fa.check() == 0
    back = dr.keep_threshold(p) / 256.0
    for b, h in ((1, 4), (2, 8), (3, 15)):
        qh, kh, vh, doh = (to_f64(inp[n][b, :, h]) for n in ("q", "k", "v", "do"))
        O, LSE = dr.head_forward_dropout(qh, kh, vh, w.scale, False, p, seed, offset, b * H + h)
        assert_o_close(to_f64(o[b, :, h].cpu()) * back, O * back, f"O[{b},{h}]")
        assert_lse_close(lse[b, h].cpu().numpy(), LSE, f"LSE[{b},{h}]")
        rq, rk, rv = dr.head_backward_dropout(qh, kh, vh, doh, w.scale, False, p, seed, offset, b * H + h)
        for name, x, r in (("dQ", dq[b, :, h], rq), ("dK", dk[b, :, h], rk), ("dV", dv[b, :, h], rv)):
            assert_grad_close(to_f64(x.cpu()), r, f"{name}[{b},{h}]")
