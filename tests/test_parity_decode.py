"""Split-KV decode parity against the float64 oracle (one query token per
sequence over the first seqlens[b] cached keys)."""

import numpy as np
import pytest
import torch

import oracle
from workloads import WORKLOADS, decode_inputs, to_f64
from _parity import assert_lse_close, assert_o_close

pytestmark = pytest.mark.gpu

fa = pytest.importorskip("io_aware_exact_forward_b200")


def _oracle(inp, w, pairs=None):
    return oracle.decode_forward(to_f64(inp["q"]), to_f64(inp["k_cache"]), to_f64(inp["v_cache"]),
                                 inp["seqlens"].cpu().numpy(), w.scale, pairs=pairs)


@pytest.mark.parametrize("Hq,Hkv,d,chunk,seqlens", [
    (8, 2, 128, 256, [1, 255, 256, 257, 1000]),
    (4, 4, 64, 256, [0, 64, 65, 777]),
    (16, 2, 128, 512, [3, 1000, 513]),
    (2, 2, 64, 64, [1, 63, 64, 65, 500]),
])
def test_decode_edge_cases(Hq, Hkv, d, chunk, seqlens):
    w = WORKLOADS[5].with_(Hq=Hq, Hkv=Hkv, d=d)
    inp = decode_inputs(w, seed=99 + d + chunk, B=len(seqlens), Tk_max=1000, seqlens=seqlens)
    dev = {k: v.cuda() for k, v in inp.items()}
    o, lse = fa.decode_splitkv(dev["q"], dev["k_cache"], dev["v_cache"], dev["seqlens"],
                               scale=w.scale, chunk=chunk)
    assert fa.check() == 0
    O, LSE = _oracle(inp, w)
    assert_o_close(to_f64(o), O)
    assert_lse_close(lse.cpu().numpy(), LSE)


def test_decode_chunk_size_does_not_change_result_much():
    w = WORKLOADS[5].with_(Hq=8, Hkv=2, d=128)
    inp = decode_inputs(w, seed=5, B=2, Tk_max=3000, seqlens=[3000, 2049])
    dev = {k: v.cuda() for k, v in inp.items()}
    outs = [fa.decode_splitkv(dev["q"], dev["k_cache"], dev["v_cache"], dev["seqlens"], chunk=c)
            for c in (64, 256, 512)]
    O, LSE = _oracle(inp, w)
    for o, lse in outs:
        assert_o_close(to_f64(o), O)
        assert_lse_close(lse.cpu().numpy(), LSE)


def test_decode_splitkv_b64_hq32_hkv8_d128_sampled():
    w = WORKLOADS[5]
    inp = decode_inputs(w, device="cuda")
    o, lse = fa.decode_splitkv(inp["q"], inp["k_cache"], inp["v_cache"], inp["seqlens"],
                               scale=w.scale, chunk=w.chunk)
    assert fa.check() == 0
    sl = inp["seqlens"].cpu().numpy()
    assert sl.min() >= 1024 and sl.max() <= 32768
    pairs = [(0, 0), (63, 31), (int(np.argmax(sl)), 5), (int(np.argmin(sl)), 30), (31, 12), (7, 3)]
    for b, h in pairs:
        n = int(sl[b])
        g = h // (w.Hq // w.Hkv)
        Ob, Lb = oracle.head_forward(to_f64(inp["q"][b, h])[None], to_f64(inp["k_cache"][b, :n, g]),
                                     to_f64(inp["v_cache"][b, :n, g]), w.scale, False)
        assert_o_close(to_f64(o[b, h])[None], Ob, what=f"O[{b},{h}]")
        assert_lse_close(lse[b, h].cpu().numpy()[None], Lb, what=f"LSE[{b},{h}]")


def test_decode_lengths_outside_the_cache_are_clamped():
    """A seqlens entry above Tk_max reads as Tk_max and one below 0 as 0:
    the result equals the run with the clamped lengths (bit for bit, the same
    kernels on the same data), and no kernel reads past the partials its
    own call wrote."""
    w = WORKLOADS[5].with_(Hq=8, Hkv=2, d=128)
    inp = decode_inputs(w, seed=31, B=3, Tk_max=700, seqlens=[700, 300, 0])
    dev = {k: v.cuda() for k, v in inp.items()}
    bad = torch.tensor([700 + 5000, 300, -17], dtype=torch.int32, device="cuda")
    o_bad, lse_bad = fa.decode_splitkv(dev["q"], dev["k_cache"], dev["v_cache"], bad, scale=w.scale, chunk=256)
    o_ok, lse_ok = fa.decode_splitkv(dev["q"], dev["k_cache"], dev["v_cache"], dev["seqlens"], scale=w.scale,
                                     chunk=256)
    assert fa.check() == 0
    assert torch.equal(o_bad, o_ok)
    assert torch.equal(lse_bad, lse_ok)
    O, LSE = _oracle(inp, w)
    assert_o_close(to_f64(o_bad), O)
    assert_lse_close(lse_bad.cpu().numpy(), LSE)
