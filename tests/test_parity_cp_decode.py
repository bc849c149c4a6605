"""Context-parallel decode parity: the KV cache of every sequence is cut into
contiguous shares, each share decoded by fa_decode_splitkv_partial, the shares'
fp32 (O, LSE) merged by fa_decode_merge, and the result compared with the
float64 oracle's decode over the whole cache.  The ranks of a multi-GPU run
are emulated on one GPU as independent launches, one per share (no kernel
waits on another); the real all-gather is exercised by a one-rank NCCL group."""

import datetime
import os
import socket

import numpy as np
import pytest
import torch

import oracle
from workloads import WORKLOADS, decode_inputs, to_f64
from _parity import assert_lse_close, assert_o_close

pytestmark = pytest.mark.gpu

fa = pytest.importorskip("io_aware_exact_forward_b200")
cp = pytest.importorskip("io_aware_exact_forward_b200.context_parallel")


def _oracle(inp, w, pairs=None):
    return oracle.decode_forward(to_f64(inp["q"]), to_f64(inp["k_cache"]), to_f64(inp["v_cache"]),
                                 inp["seqlens"].cpu().numpy(), w.scale, pairs=pairs)


def _emulated_ranks(dev, w, R, shard_len, chunk):
    """Decode R contiguous shares into one packed buffer, as the all-gather
    would leave it, and merge."""
    B, Hq, d = dev["q"].shape
    n = cp.packed_block_floats(B, Hq, d)
    n_o = B * Hq * d
    blocks = torch.full((R, n), float("nan"), dtype=torch.float32, device="cuda")
    for r in range(R):
        lo = r * shard_len
        ks = dev["k_cache"][:, lo:lo + shard_len].contiguous()
        vs = dev["v_cache"][:, lo:lo + shard_len].contiguous()
        if ks.shape[1] == 0:   # past the cache: an empty share
            ks = vs = torch.zeros((B, 1) + tuple(dev["k_cache"].shape[2:]), dtype=torch.bfloat16, device="cuda")
        sl = cp.shard_seqlens(dev["seqlens"], r, shard_len)
        fa.decode_splitkv_partial(dev["q"], ks, vs, sl, scale=w.scale, chunk=chunk,
                                  out=blocks[r, :n_o].view(B, Hq, d), lse=blocks[r, n_o:n_o + B * Hq].view(B, Hq))
    o, lse = fa.decode_merge(blocks[:, :n_o].unflatten(1, (B, Hq, d)), blocks[:, n_o:n_o + B * Hq].unflatten(1, (B, Hq)))
    assert fa.check() == 0
    return o, lse, blocks


@pytest.mark.parametrize("Hq,Hkv,d,chunk,seqlens", [
    (8, 2, 128, 256, [1, 255, 256, 257, 1000]),
    (4, 4, 64, 256, [0, 64, 65, 777]),
    (16, 2, 128, 512, [3, 1000, 513]),
])
def test_partial_decode_fp32_output(Hq, Hkv, d, chunk, seqlens):
    w = WORKLOADS[5].with_(Hq=Hq, Hkv=Hkv, d=d)
    inp = decode_inputs(w, seed=41 + d + chunk, B=len(seqlens), Tk_max=1000, seqlens=seqlens)
    dev = {k: v.cuda() for k, v in inp.items()}
    o, lse = fa.decode_splitkv_partial(dev["q"], dev["k_cache"], dev["v_cache"], dev["seqlens"], scale=w.scale,
                                       chunk=chunk)
    assert fa.check() == 0
    assert o.dtype == torch.float32
    O, LSE = _oracle(inp, w)
    assert_o_close(o.cpu().double().numpy(), O)
    assert_lse_close(lse.cpu().numpy(), LSE)
    # the bf16 entry point rounds the same partial result
    ob, lb = fa.decode_splitkv(dev["q"], dev["k_cache"], dev["v_cache"], dev["seqlens"], scale=w.scale, chunk=chunk)
    assert fa.check() == 0
    assert torch.equal(ob, o.to(torch.bfloat16)) and torch.equal(lb, lse)


@pytest.mark.parametrize("R,shard_len,Hq,Hkv,d,chunk,seqlens", [
    (1, 1000, 8, 2, 128, 256, [1, 700, 1000]),
    (2, 500, 8, 2, 128, 256, [1, 499, 500, 501, 1000]),     # sequences ending in either share
    (3, 384, 4, 4, 64, 128, [0, 64, 383, 384, 385, 1000]),  # an empty sequence; ragged last share
    (8, 128, 32, 4, 128, 128, [1, 129, 1000, 640]),         # G = 8, most shares partly empty
    (5, 200, 2, 1, 64, 64, [17, 200, 999]),                 # share length not a multiple of 64
])
def test_emulated_ranks_match_whole_cache(R, shard_len, Hq, Hkv, d, chunk, seqlens):
    w = WORKLOADS[5].with_(Hq=Hq, Hkv=Hkv, d=d)
    inp = decode_inputs(w, seed=7 * R + d + shard_len, B=len(seqlens), Tk_max=1000, seqlens=seqlens)
    dev = {k: v.cuda() for k, v in inp.items()}
    o, lse, _ = _emulated_ranks(dev, w, R, shard_len, chunk)
    O, LSE = _oracle(inp, w)
    assert_o_close(to_f64(o), O)
    assert_lse_close(lse.cpu().numpy(), LSE)


@pytest.mark.parametrize("R,d", [(1, 64), (5, 128), (40, 64)])
def test_merge_kernel_against_oracle(R, d):
    """Random partials, some with LSE = -inf (a share with no key) and one row
    empty everywhere; R = 40 runs the lanes' loop over partials twice."""
    B, Hq = 3, 4
    g = torch.Generator().manual_seed(100 + R + d)
    o_parts = torch.randn((R, B, Hq, d), generator=g)
    lse_parts = 3.0 * torch.randn((R, B, Hq), generator=g)
    drop = torch.rand((R, B, Hq), generator=g) < 0.3
    lse_parts[drop] = float("-inf")
    o_parts[drop] = 0.0
    lse_parts[:, 1, 2] = float("-inf")
    o_parts[:, 1, 2] = 0.0
    o, lse = fa.decode_merge(o_parts.cuda(), lse_parts.cuda())
    assert fa.check() == 0
    O, LSE = oracle.merge_partials(o_parts.double().numpy(), lse_parts.double().numpy())
    assert_o_close(to_f64(o), O)
    assert_lse_close(lse.cpu().numpy(), LSE)
    assert (o[1, 2] == 0).all() and lse[1, 2].item() == float("-inf")


def test_emulated_eight_ranks_b64_hq32_hkv8_d128_sampled():
    """The decode workload (B 64, Hq 32, Hkv 8, d 128, Tk up to 32768) with
    every cache cut into 8 shares of 4096 keys; sampled (sequence, head)
    pairs against the oracle."""
    w = WORKLOADS[5]
    inp = decode_inputs(w, device="cuda")
    o, lse, _ = _emulated_ranks(inp, w, 8, 4096, w.chunk)
    sl = inp["seqlens"].cpu().numpy()
    pairs = [(0, 0), (63, 31), (int(np.argmax(sl)), 5), (int(np.argmin(sl)), 30), (31, 12)]
    for b, h in pairs:
        n = int(sl[b])
        g = h // (w.Hq // w.Hkv)
        Ob, Lb = oracle.head_forward(to_f64(inp["q"][b, h])[None], to_f64(inp["k_cache"][b, :n, g]),
                                     to_f64(inp["v_cache"][b, :n, g]), w.scale, False)
        assert_o_close(to_f64(o[b, h])[None], Ob, what=f"O[{b},{h}]")
        assert_lse_close(lse[b, h].cpu().numpy()[None], Lb, what=f"LSE[{b},{h}]")


def test_one_rank_nccl_group_end_to_end():
    """decode_splitkv_cp through a real NCCL all-gather (one rank) equals the
    plain decode, and the oracle."""
    import torch.distributed as dist
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    torch.cuda.set_device(0)
    dist.init_process_group("nccl", rank=0, world_size=1, timeout=datetime.timedelta(seconds=60),
                            device_id=torch.device("cuda", 0))
    try:
        w = WORKLOADS[5].with_(Hq=8, Hkv=2, d=128)
        inp = decode_inputs(w, seed=3, B=4, Tk_max=1000, seqlens=[1, 256, 999, 1000])
        dev = {k: v.cuda() for k, v in inp.items()}
        o, lse = fa.decode_splitkv_cp(dev["q"], dev["k_cache"], dev["v_cache"], dev["seqlens"], scale=w.scale)
        o2, l2 = fa.decode_splitkv(dev["q"], dev["k_cache"], dev["v_cache"], dev["seqlens"], scale=w.scale)
        assert fa.check() == 0
        O, LSE = _oracle(inp, w)
        assert_o_close(to_f64(o), O)
        assert_lse_close(lse.cpu().numpy(), LSE)
        assert (o.float() - o2.float()).abs().max().item() <= 2 ** -7
    finally:
        dist.destroy_process_group()
