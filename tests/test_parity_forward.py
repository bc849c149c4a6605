"""Forward parity: the CUDA path (through the C ABI) against the float64 CPU
oracle on the same seeded bf16 inputs."""

import numpy as np
import pytest
import torch

import oracle
from workloads import WORKLOADS, prefill_inputs, to_f64
from _parity import assert_lse_close, assert_o_close

pytestmark = pytest.mark.gpu

fa = pytest.importorskip("io_aware_exact_forward_b200")


def _run(inp, w, causal=None, scale=None):
    causal = w.causal if causal is None else causal
    scale = w.scale if scale is None else scale
    q, k, v = (inp[n].cuda() for n in ("q", "k", "v"))
    o, lse = fa.forward(q, k, v, scale=scale, causal=causal)
    assert fa.check() == 0
    return o.cpu(), lse.cpu()


def _full_oracle(inp, w, causal, scale):
    return oracle.attention_forward(to_f64(inp["q"]), to_f64(inp["k"]), to_f64(inp["v"]), scale, causal)


def test_selfattn_b1_h1_t128_d64_forward():
    w = WORKLOADS[1]
    inp = prefill_inputs(w)
    o, lse = _run(inp, w)
    O, LSE = _full_oracle(inp, w, w.causal, w.scale)
    assert_o_close(to_f64(o), O)
    assert_lse_close(lse.numpy(), LSE)


EDGE = [
    # B, Hq, Hkv, Tq, Tk, d, causal
    (1, 2, 2, 128, 128, 64, False),
    (1, 2, 2, 128, 128, 128, True),
    (2, 2, 1, 200, 200, 128, True),      # ragged tail, GQA 2
    (1, 1, 1, 1, 1, 64, True),           # single row, single key
    (1, 1, 1, 1, 1, 128, False),
    (1, 4, 2, 77, 300, 128, True),       # Tq < Tk, bottom-right causal
    (1, 2, 2, 300, 77, 64, True),        # Tq > Tk: fully masked rows
    (1, 1, 1, 513, 1000, 128, False),    # several tiles, ragged both ways
    (1, 8, 1, 256, 256, 64, True),       # G = 8
    (3, 3, 3, 129, 255, 64, False),
    (1, 2, 1, 640, 640, 128, True),      # several query blocks
]


@pytest.mark.parametrize("B,Hq,Hkv,Tq,Tk,d,causal", EDGE)
def test_forward_edge_cases(B, Hq, Hkv, Tq, Tk, d, causal):
    w = WORKLOADS[1].with_(B=B, Hq=Hq, Hkv=Hkv, d=d, causal=causal)
    inp = prefill_inputs(w, seed=7 + Tq + Tk + d, Tq=Tq, Tk=Tk)
    o, lse = _run(inp, w)
    O, LSE = _full_oracle(inp, w, causal, w.scale)
    assert_o_close(to_f64(o), O)
    assert_lse_close(lse.numpy(), LSE)


def test_forward_empty_keys():
    w = WORKLOADS[1].with_(B=1, Hq=2, Hkv=2, d=64)
    inp = prefill_inputs(w, Tq=70, Tk=0)
    q = inp["q"].cuda()
    k = torch.empty((1, 0, 2, 64), dtype=torch.bfloat16, device="cuda")
    o, lse = fa.forward(q, k, k, causal=False)
    torch.cuda.synchronize()
    assert torch.all(o == 0)
    assert torch.all(torch.isneginf(lse))


def test_forward_large_scores_stay_exact():
    """Scores far apart (scale 1, keys x4) exercise the lazy rescale and huge
    maxima.  Rows are nearly one-hot, so |O| reaches ~4.5."""
    w = WORKLOADS[1].with_(B=1, Hq=1, Hkv=1, d=64)
    inp = prefill_inputs(w, Tq=256, Tk=1024)
    inp["k"] = (inp["k"].float() * 4).to(torch.bfloat16)
    o, lse = _run(inp, w, scale=1.0)
    O, LSE = _full_oracle(inp, w, False, 1.0)
    assert_o_close(to_f64(o), O)
    assert_lse_close(lse.numpy(), LSE)


def _sampled_check(w, heads, rows_per_head=None):
    """Full-size run; the oracle evaluates the listed (b, h) heads (all rows,
    or the given rows)."""
    inp = prefill_inputs(w, device="cuda")
    o, lse = fa.forward(inp["q"], inp["k"], inp["v"], scale=w.scale, causal=w.causal)
    assert fa.check() == 0
    G = w.Hq // w.Hkv
    for b, h in heads:
        qh = to_f64(inp["q"][b, :, h])
        kh = to_f64(inp["k"][b, :, h // G])
        vh = to_f64(inp["v"][b, :, h // G])
        rows = rows_per_head
        O, LSE = oracle.head_forward(qh, kh, vh, w.scale, w.causal, rows=rows)
        sel = slice(None) if rows is None else torch.as_tensor(rows)
        assert_o_close(to_f64(o[b, sel, h]), O, what=f"O[b={b},h={h}]")
        assert_lse_close(lse[b, h, sel].cpu().numpy(), LSE, what=f"LSE[b={b},h={h}]")


def test_gpt2medium_b64_h16_t1024_d64_forward_sampled():
    w = WORKLOADS[2]
    _sampled_check(w, [(0, 0), (63, 15), (17, 5), (40, 11)])


def test_causal_b4_h32_t8192_d128_forward_sampled():
    w = WORKLOADS[3]
    rows = np.r_[0:130, 4000:4100, 8062:8192]
    _sampled_check(w, [(0, 0), (3, 31), (2, 17)], rows_per_head=rows)


def test_gqa_causal_t32768_outliers_forward_sampled():
    w = WORKLOADS[4]
    rows = np.r_[0:64, 16384:16448, 32704:32768]
    _sampled_check(w, [(0, 0), (0, 13), (0, 31)], rows_per_head=rows)
