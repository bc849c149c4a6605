"""Backward parity: dQ, dK, dV from the CUDA path (which recomputes S and P
from the forward's LSE) against the float64 oracle's gradients of
L = sum(dO * O), relative L2 error <= 2e-2 per tensor."""

import numpy as np
import pytest
import torch

import oracle
from workloads import WORKLOADS, prefill_inputs, to_f64
from _parity import assert_grad_close

pytestmark = pytest.mark.gpu

fa = pytest.importorskip("io_aware_exact_forward_b200")


def _gpu_fwd_bwd(inp, scale, causal):
    q, k, v, do = (inp[n] if inp[n].is_cuda else inp[n].cuda() for n in ("q", "k", "v", "do"))
    o, lse = fa.forward(q, k, v, scale=scale, causal=causal)
    dq, dk, dv = fa.backward(q, k, v, o, lse, do, scale=scale, causal=causal)
    assert fa.check() == 0
    return dq, dk, dv


def _full_check(inp, scale, causal):
    dq, dk, dv = _gpu_fwd_bwd(inp, scale, causal)
    rq, rk, rv = oracle.attention_backward(to_f64(inp["q"]), to_f64(inp["k"]), to_f64(inp["v"]),
                                           to_f64(inp["do"]), scale, causal)
    assert_grad_close(to_f64(dq), rq, "dQ")
    assert_grad_close(to_f64(dk), rk, "dK")
    assert_grad_close(to_f64(dv), rv, "dV")


def test_selfattn_b1_h1_t128_d64_backward():
    w = WORKLOADS[1]
    _full_check(prefill_inputs(w), w.scale, w.causal)


EDGE = [
    # B, Hq, Hkv, Tq, Tk, d, causal
    (1, 2, 2, 128, 128, 64, False),
    (1, 2, 2, 128, 128, 128, True),
    (2, 2, 1, 200, 200, 128, True),      # ragged tail, GQA 2
    (1, 1, 1, 1, 1, 64, True),
    (1, 4, 2, 77, 300, 128, True),       # Tq < Tk
    (1, 2, 2, 300, 77, 64, True),        # Tq > Tk: rows that see no key
    (1, 1, 1, 513, 1000, 128, False),
    (1, 8, 1, 256, 256, 64, True),       # G = 8: dK/dV summed over 8 heads
    (3, 3, 3, 129, 255, 64, False),
    (1, 4, 1, 384, 384, 128, False),
]


@pytest.mark.parametrize("B,Hq,Hkv,Tq,Tk,d,causal", EDGE)
def test_backward_edge_cases(B, Hq, Hkv, Tq, Tk, d, causal):
    w = WORKLOADS[1].with_(B=B, Hq=Hq, Hkv=Hkv, d=d, causal=causal)
    inp = prefill_inputs(w, seed=11 + Tq + Tk + d, Tq=Tq, Tk=Tk)
    _full_check(inp, w.scale, causal)


def test_backward_zero_length_keys_gives_zero_dq():
    w = WORKLOADS[1].with_(B=1, Hq=2, Hkv=2, d=64)
    inp = prefill_inputs(w, Tq=40, Tk=0)
    q, do = inp["q"].cuda(), inp["do"].cuda()
    k = torch.empty((1, 0, 2, 64), dtype=torch.bfloat16, device="cuda")
    o, lse = fa.forward(q, k, k)
    dq, dk, dv = fa.backward(q, k, k, o, lse, do)
    torch.cuda.synchronize()
    assert torch.all(dq == 0)


def _head_grads(inp, w, b, h):
    G = w.Hq // w.Hkv
    g = h // G
    return oracle.head_backward(to_f64(inp["q"][b, :, h]), to_f64(inp["k"][b, :, g]),
                                to_f64(inp["v"][b, :, g]), to_f64(inp["do"][b, :, h]), w.scale, w.causal)


def test_gpt2medium_b64_h16_t1024_d64_backward_sampled():
    w = WORKLOADS[2]
    inp = prefill_inputs(w, device="cuda")
    dq, dk, dv = _gpu_fwd_bwd(inp, w.scale, w.causal)
    for b, h in [(0, 0), (63, 15), (17, 5)]:
        rq, rk, rv = _head_grads(inp, w, b, h)
        assert_grad_close(to_f64(dq[b, :, h]), rq, f"dQ[{b},{h}]")
        assert_grad_close(to_f64(dk[b, :, h]), rk, f"dK[{b},{h}]")
        assert_grad_close(to_f64(dv[b, :, h]), rv, f"dV[{b},{h}]")


def test_causal_b4_h32_t8192_d128_backward_sampled():
    w = WORKLOADS[3]
    inp = prefill_inputs(w, device="cuda")
    dq, dk, dv = _gpu_fwd_bwd(inp, w.scale, w.causal)
    for b, h in [(0, 0), (3, 31)]:
        rq, rk, rv = _head_grads(inp, w, b, h)
        assert_grad_close(to_f64(dq[b, :, h]), rq, f"dQ[{b},{h}]")
        assert_grad_close(to_f64(dk[b, :, h]), rk, f"dK[{b},{h}]")
        assert_grad_close(to_f64(dv[b, :, h]), rv, f"dV[{b},{h}]")


def test_gqa_causal_t32768_outliers_backward_one_group():
    """One full GQA group (KV head 7 and its four query heads)."""
    w = WORKLOADS[4]
    inp = prefill_inputs(w, device="cuda")
    dq, dk, dv = _gpu_fwd_bwd(inp, w.scale, w.causal)
    g = 7
    G = w.Hq // w.Hkv
    sk = np.zeros((w.T, w.d))
    sv = np.zeros((w.T, w.d))
    for h in range(g * G, (g + 1) * G):
        rq, rk, rv = _head_grads(inp, w, 0, h)
        assert_grad_close(to_f64(dq[0, :, h]), rq, f"dQ[0,{h}]")
        sk += rk
        sv += rv
    assert_grad_close(to_f64(dk[0, :, g]), sk, f"dK[0,{g}]")
    assert_grad_close(to_f64(dv[0, :, g]), sv, f"dV[0,{g}]")
