"""FP8 forward parity: fa_forward_fp8 (E4M3 Q, K, V with per-tensor factors)
against the float64 oracle's exact attention on the dequantised inputs.

The kernel rounds P to E4M3 (3 mantissa bits) before P V, as the low-precision
forward of FlashAttention-3 does, so O cannot meet the bf16 path's bounds; each
element is held to the bound ``fp8_o_tolerance`` derives from that rounding
(and the mean to FP8_O_MEAN_ABS).  LSE sums the unrounded P and keeps the bf16
path's bound."""

import math

import numpy as np
import pytest
import torch

import oracle
from workloads import WORKLOADS, prefill_inputs_e4m3
from _parity import assert_fp8_o_close, assert_lse_close, fp8_o_tolerance

pytestmark = pytest.mark.gpu

fa = pytest.importorskip("io_aware_exact_forward_b200")


def _codes(t):
    return t.view(torch.uint8).cpu().numpy()


def _check_head(o, lse, inp, b, h, G, scale, causal, rows=None):
    """One (batch, head) against the oracle, with the per-element bound."""
    hk = h // G
    q = oracle.e4m3_decode(_codes(inp["q"][b, :, h])) * inp["q_descale"]
    k = oracle.e4m3_decode(_codes(inp["k"][b, :, hk])) * inp["k_descale"]
    v = oracle.e4m3_decode(_codes(inp["v"][b, :, hk])) * inp["v_descale"]
    Tq, Tk = q.shape[0], k.shape[0]
    rows = np.arange(Tq) if rows is None else np.asarray(rows)
    O, L = oracle.head_forward(q, k, v, scale, causal, rows=rows)
    S = scale * (q[rows] @ k.T)
    if causal:
        S = np.where(np.arange(Tk)[None, :] <= rows[:, None] + (Tk - Tq), S, -np.inf)
    tol = fp8_o_tolerance(S, v, O)
    og = o[b, rows, h].float().cpu().numpy()
    assert_fp8_o_close(og, O, tol, what=f"O[{b},:,{h}]")
    assert_lse_close(lse[b, h, rows].cpu().numpy(), L, what=f"LSE[{b},{h}]")


CASES = [
    # B, Hq, Hkv, Tq, Tk, causal
    (1, 2, 2, 128, 128, False),
    (1, 2, 2, 300, 300, True),       # ragged tail
    (2, 4, 2, 517, 517, True),       # GQA 2, several tiles
    (1, 2, 2, 200, 450, True),       # Tq < Tk
    (1, 2, 2, 450, 200, True),       # Tq > Tk: early rows see no key
    (1, 8, 1, 512, 512, False),      # G = 8
    (1, 1, 1, 1, 1, False),          # one key
    (1, 2, 2, 1000, 1000, False),
]


@pytest.mark.parametrize("B,Hq,Hkv,Tq,Tk,causal", CASES)
def test_fp8_forward(B, Hq, Hkv, Tq, Tk, causal):
    w = WORKLOADS[3].with_(B=B, Hq=Hq, Hkv=Hkv, causal=causal)
    inp = prefill_inputs_e4m3(w, seed=17 + Tq + 5 * Tk + Hq, Tq=Tq, Tk=Tk)
    dev = {n: (t.cuda() if torch.is_tensor(t) else t) for n, t in inp.items()}
    o, lse = fa.forward_fp8(dev["q"], dev["k"], dev["v"], inp["q_descale"], inp["k_descale"], inp["v_descale"],
                            scale=w.scale, causal=causal)
    assert fa.check() == 0
    for b in range(B):
        for h in range(Hq):
            _check_head(o, lse, inp, b, h, Hq // Hkv, w.scale, causal)


def test_fp8_forward_no_keys():
    w = WORKLOADS[3].with_(B=1, Hq=2, Hkv=2, causal=False)
    inp = prefill_inputs_e4m3(w, seed=3, Tq=130, Tk=0)
    q = inp["q"].cuda()
    kv = torch.empty((1, 0, 2, 128), dtype=torch.float8_e4m3fn, device="cuda")
    o, lse = fa.forward_fp8(q, kv, kv, inp["q_descale"], 1.0, 1.0, scale=w.scale)
    assert fa.check() == 0
    assert (o == 0).all() and torch.isneginf(lse).all()


def test_fp8_forward_rejects_head_dim_64():
    q = torch.zeros((1, 16, 1, 64), dtype=torch.float8_e4m3fn, device="cuda")
    with pytest.raises(fa.FAError) as e:
        fa.forward_fp8(q, q, q, 1.0, 1.0, 1.0)
    assert e.value.status == 2


def test_fp8_forward_gqa_long_context_sampled_rows():
    """The long-context GQA workload (B 1, Hq 32, Hkv 8, T 32768, d 128,
    causal, 1% of keys x4) in E4M3: rows sampled along the sequence for the
    first and last head of the first and last KV group."""
    w = WORKLOADS[4]
    inp = prefill_inputs_e4m3(w, device="cuda")
    o, lse = fa.forward_fp8(inp["q"], inp["k"], inp["v"], inp["q_descale"], inp["k_descale"], inp["v_descale"],
                            scale=w.scale, causal=True)
    assert fa.check() == 0
    rows = [0, 1, 2, 127, 128, 255, 4096, 16383, 16384, 32766, 32767]
    for h in (0, 3, 28, 31):
        _check_head(o, lse, inp, 0, h, w.Hq // w.Hkv, w.scale, True, rows=rows)


def test_fp8_forward_persistent_items_sampled_rows():
    """Non-causal E4M3 launches are persistent (one CTA per SM walks several
    items): B 2, Hq 32, Hkv 8, T 4096 gives 1024 items on 148 SMs, and the
    heads checked are later items of their CTAs.  Sampled rows."""
    w = WORKLOADS[3].with_(B=2, Hq=32, Hkv=8, causal=False)
    inp = prefill_inputs_e4m3(w, seed=29, Tq=4096, Tk=4096, device="cuda")
    o, lse = fa.forward_fp8(inp["q"], inp["k"], inp["v"], inp["q_descale"], inp["k_descale"], inp["v_descale"],
                            scale=w.scale, causal=False)
    assert fa.check() == 0
    rows = [0, 127, 128, 2047, 2048, 4095]
    for b, h in ((0, 15), (1, 31)):
        _check_head(o, lse, inp, b, h, w.Hq // w.Hkv, w.scale, False, rows=rows)
