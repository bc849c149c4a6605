"""Sliding-window parity: fa_forward_window / fa_backward_window (through the
C ABI) against the float64 oracle's windowed attention on the same seeded
bf16 inputs, with the forward and gradient tolerances of the other parity
tests.  The window is a causal local window of W keys: query i sees key j iff
i + (Tk - Tq) - W < j <= i + (Tk - Tq)."""

import numpy as np
import pytest

import oracle
from workloads import WORKLOADS, prefill_inputs, to_f64
from _parity import assert_grad_close, assert_lse_close, assert_o_close

pytestmark = pytest.mark.gpu

fa = pytest.importorskip("io_aware_exact_forward_b200")

CASES = [
    # B, Hq, Hkv, Tq, Tk, d, W
    (1, 2, 2, 300, 300, 64, 1),          # the diagonal key only
    (1, 2, 2, 300, 300, 64, 100),        # window inside one tile, ragged tail
    (1, 2, 1, 384, 384, 128, 128),       # window of exactly one tile, GQA 2
    (2, 4, 2, 517, 517, 128, 200),       # window straddling tile edges
    (1, 2, 2, 200, 450, 64, 130),        # Tq < Tk (bottom-right aligned)
    (1, 2, 2, 450, 200, 128, 64),        # Tq > Tk: early rows see no key
    (1, 4, 1, 640, 640, 64, 1000),       # window wider than the sequence = causal
    (1, 8, 1, 512, 512, 64, 257),        # G = 8
]


def _inputs(B, Hq, Hkv, Tq, Tk, d, W):
    w = WORKLOADS[1].with_(B=B, Hq=Hq, Hkv=Hkv, d=d, causal=True)
    return w, prefill_inputs(w, seed=31 + Tq + 3 * Tk + d + W, Tq=Tq, Tk=Tk)


@pytest.mark.parametrize("B,Hq,Hkv,Tq,Tk,d,W", CASES)
def test_window_forward(B, Hq, Hkv, Tq, Tk, d, W):
    w, inp = _inputs(B, Hq, Hkv, Tq, Tk, d, W)
    q, k, v = (inp[n].cuda() for n in ("q", "k", "v"))
    o, lse = fa.forward(q, k, v, scale=w.scale, window=W)
    assert fa.check() == 0
    O, LSE = oracle.attention_forward(to_f64(inp["q"]), to_f64(inp["k"]), to_f64(inp["v"]), w.scale, True,
                                      window=W)
    assert_o_close(to_f64(o.cpu()), O)
    assert_lse_close(lse.cpu().numpy(), LSE)


@pytest.mark.parametrize("B,Hq,Hkv,Tq,Tk,d,W", CASES)
def test_window_backward(B, Hq, Hkv, Tq, Tk, d, W):
    w, inp = _inputs(B, Hq, Hkv, Tq, Tk, d, W)
    q, k, v, do = (inp[n].cuda() for n in ("q", "k", "v", "do"))
    o, lse = fa.forward(q, k, v, scale=w.scale, window=W)
    dq, dk, dv = fa.backward(q, k, v, o, lse, do, scale=w.scale, window=W)
    assert fa.check() == 0
    rq, rk, rv = oracle.attention_backward(to_f64(inp["q"]), to_f64(inp["k"]), to_f64(inp["v"]),
                                           to_f64(inp["do"]), w.scale, True, window=W)
    assert_grad_close(to_f64(dq.cpu()), rq, "dQ")
    assert_grad_close(to_f64(dk.cpu()), rk, "dK")
    assert_grad_close(to_f64(dv.cpu()), rv, "dV")


def test_window_wider_than_sequence_matches_causal_path():
    """W >= Tk must give the causal kernel's result (same arithmetic, no
    tile skipped), bit for bit."""
    w, inp = _inputs(1, 2, 2, 384, 384, 128, 384)
    q, k, v, do = (inp[n].cuda() for n in ("q", "k", "v", "do"))
    o1, l1 = fa.forward(q, k, v, scale=w.scale, causal=True)
    o2, l2 = fa.forward(q, k, v, scale=w.scale, window=4096)
    assert fa.check() == 0
    assert (o1 == o2).all() and (l1 == l2).all()
    g1 = fa.backward(q, k, v, o1, l1, do, scale=w.scale, causal=True)
    g2 = fa.backward(q, k, v, o2, l2, do, scale=w.scale, window=4096)
    assert fa.check() == 0
    for a, b in zip(g1, g2):
        assert (a == b).all()


def test_window_long_sequence_sampled_rows():
    """T = 8192, d = 128, W = 1024: rows sampled along the sequence (tile
    edges, the first rows, the last rows) against the oracle row by row."""
    w = WORKLOADS[3].with_(B=1, Hq=2, Hkv=2)
    W = 1024
    inp = prefill_inputs(w, device="cuda")
    o, lse = fa.forward(inp["q"], inp["k"], inp["v"], scale=w.scale, window=W)
    assert fa.check() == 0
    o, lse = o.cpu(), lse.cpu()
    rows = np.array([0, 1, 127, 128, 1023, 1024, 1025, 4095, 4096, 8190, 8191])
    q64, k64, v64 = (to_f64(inp[n].cpu()) for n in ("q", "k", "v"))
    for h in range(2):
        O, LSE = oracle.head_forward(q64[0, :, h], k64[0, :, h], v64[0, :, h], w.scale, True, rows=rows, window=W)
        assert_o_close(to_f64(o[0, rows, h]), O)
        assert_lse_close(lse[0, h, rows].numpy(), LSE)


def test_window_persistent_items_sampled_rows():
    """Windowed forwards run persistently (one CTA per SM walks several
    items): with 16 heads of T = 8192 there are 512 items on 148 SMs, and
    heads 7 and 15 are second or later items of their CTAs.  Sampled rows
    against the oracle."""
    w = WORKLOADS[3].with_(B=1, Hq=16, Hkv=16)
    W = 1024
    inp = prefill_inputs(w, device="cuda")
    o, lse = fa.forward(inp["q"], inp["k"], inp["v"], scale=w.scale, window=W)
    assert fa.check() == 0
    o, lse = o.cpu(), lse.cpu()
    rows = np.array([0, 255, 256, 1023, 1024, 4097, 8191])
    for h in (7, 15):
        q64, k64, v64 = (to_f64(inp[n][0, :, h].cpu()) for n in ("q", "k", "v"))
        O, LSE = oracle.head_forward(q64, k64, v64, w.scale, True, rows=rows, window=W)
        assert_o_close(to_f64(o[0, rows, h]), O)
        assert_lse_close(lse[0, h, rows].numpy(), LSE)


@pytest.mark.parametrize("Hq,Hkv,d,chunk,W,seqlens", [
    (8, 2, 128, 256, 300, [1, 255, 256, 257, 1000]),   # window inside, across and beyond chunks
    (4, 4, 64, 256, 1, [1, 64, 65, 777]),              # the last key only
    (16, 2, 128, 512, 513, [3, 1000, 513, 514]),
    (2, 2, 64, 64, 5000, [1, 63, 64, 65, 500]),        # wider than every sequence
])
def test_window_decode(Hq, Hkv, d, chunk, W, seqlens):
    from workloads import decode_inputs
    w = WORKLOADS[5].with_(Hq=Hq, Hkv=Hkv, d=d)
    inp = decode_inputs(w, seed=77 + d + chunk + W, B=len(seqlens), Tk_max=1000, seqlens=seqlens)
    dev = {n: t.cuda() for n, t in inp.items()}
    o, lse = fa.decode_splitkv(dev["q"], dev["k_cache"], dev["v_cache"], dev["seqlens"], scale=w.scale,
                               chunk=chunk, window=W)
    assert fa.check() == 0
    O, LSE = oracle.decode_forward(to_f64(inp["q"]), to_f64(inp["k_cache"]), to_f64(inp["v_cache"]),
                                   inp["seqlens"].cpu().numpy(), w.scale, window=W)
    assert_o_close(to_f64(o.cpu()), O)
    assert_lse_close(lse.cpu().numpy(), LSE)
