"""fa_decode_splitkv_noalloc: split-KV decode whose chunk partials live in a
device array inside the library, for callers that cannot allocate device
memory where they call (a serving engine's plug-in interface that passes
tensors but no allocator, or a decode loop that cannot take cudaMalloc's
implicit synchronisation).

The GPU test calls the entry point through the C ABI twice in a row, on
different inputs, and checks each result against fa_decode_splitkv with a
caller workspace and against the float64 oracle, within the decode
tolerances of the other parity tests.  This file is collected last so that a
stop-at-first-failure run has already run every other test."""

import ctypes

import pytest
import torch

import io_aware_exact_forward_b200 as fa
import oracle
from workloads import WORKLOADS, decode_inputs, to_f64
from _parity import assert_lse_close, assert_o_close

SCRATCH_BYTES = 32 << 20
FA_ERR_INVALID_ARG = 1
FA_ERR_WORKSPACE = 4


def test_noalloc_rejects_sizes_beyond_its_scratch():
    lib = fa.load_library()
    # 64 x 32 x 128 chunks x 129 floats is about 135 MB > 32 MiB
    assert lib.fa_decode_workspace_bytes(64, 32, 32768, 128, 256) > SCRATCH_BYTES
    st = lib.fa_decode_splitkv_noalloc(None, None, None, None, None, None, 64, 32, 8, 32768, 128, 0.1, 256, None)
    assert st == FA_ERR_WORKSPACE  # before any pointer is looked at


def test_noalloc_checks_arguments_like_the_workspace_entry_point_with_no_rows():
    """B = 0 with Hq not a multiple of Hkv (or a bad chunk) is rejected by
    both entry points alike, before any device work."""
    lib = fa.load_library()
    for Hq, Hkv, chunk in [(3, 2, 256), (4, 2, 100), (4, 2, 32)]:
        a = lib.fa_decode_splitkv(None, None, None, None, None, None, None, 0, 0, Hq, Hkv, 1024, 128, 0.1,
                                  chunk, None)
        b = lib.fa_decode_splitkv_noalloc(None, None, None, None, None, None, 0, Hq, Hkv, 1024, 128, 0.1,
                                          chunk, None)
        assert a == b == FA_ERR_INVALID_ARG, (Hq, Hkv, chunk, a, b)


@pytest.mark.gpu
def test_noalloc_matches_workspace_entry_point_twice():
    lib = fa.load_library()
    P = ctypes.c_void_p
    w = WORKLOADS[5].with_(Hq=16, Hkv=4)
    for call, (seed, seqlens) in enumerate([(21, [3000, 1, 2049, 256]), (22, [17, 4000, 1024, 777])]):
        inp = decode_inputs(w, seed=seed, B=4, Tk_max=4000, seqlens=seqlens)
        dev = {k: v.cuda() for k, v in inp.items()}
        B, Hq, d = dev["q"].shape
        Tk_max, Hkv = dev["k_cache"].shape[1], dev["k_cache"].shape[2]
        assert lib.fa_decode_workspace_bytes(B, Hq, Tk_max, d, 256) <= SCRATCH_BYTES
        o_ref, lse_ref = fa.decode_splitkv(dev["q"], dev["k_cache"], dev["v_cache"], dev["seqlens"],
                                           scale=w.scale, chunk=256)
        o = torch.empty_like(dev["q"])
        lse = torch.empty((B, Hq), dtype=torch.float32, device="cuda")
        stream = P(torch.cuda.current_stream().cuda_stream)
        st = lib.fa_decode_splitkv_noalloc(P(dev["q"].data_ptr()), P(dev["k_cache"].data_ptr()),
                                           P(dev["v_cache"].data_ptr()), P(dev["seqlens"].data_ptr()),
                                           P(o.data_ptr()), P(lse.data_ptr()), B, Hq, Hkv, Tk_max, d,
                                           w.scale, 256, stream)
        assert st == 0, f"call {call}: status {st}"
        assert lib.fa_check(stream) == 0
        assert_o_close(to_f64(o), to_f64(o_ref), what=f"O vs fa_decode_splitkv (call {call})")
        assert_lse_close(lse.cpu().numpy(), lse_ref.cpu().numpy(), what=f"LSE vs fa_decode_splitkv (call {call})")
        O, LSE = oracle.decode_forward(to_f64(inp["q"]), to_f64(inp["k_cache"]), to_f64(inp["v_cache"]),
                                       seqlens, w.scale)
        assert_o_close(to_f64(o), O, what=f"O vs oracle (call {call})")
        assert_lse_close(lse.cpu().numpy(), LSE, what=f"LSE vs oracle (call {call})")
