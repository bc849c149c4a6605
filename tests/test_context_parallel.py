"""Host logic of the context-parallel decode on CPU: two gloo ranks, each
holding a contiguous share of every sequence's KV cache.  The per-rank decode
and the merge are stood in for by the float64 oracle (the kernels need a
GPU); what is checked is the library's own host path around them -- the
share lengths, the packed (O, LSE) block, the all-gather and the views the
merge receives -- against the oracle's decode over the whole cache."""

import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


B, HQ, HKV, D, TMAX, SCALE = 3, 4, 2, 64, 96, 0.125


def _inputs():
    from workloads import WORKLOADS, decode_inputs
    w = WORKLOADS[5].with_(Hq=HQ, Hkv=HKV, d=D)
    return decode_inputs(w, seed=5, B=B, Tk_max=TMAX, seqlens=[1, 50, 96])


def _worker(rank, world, port, shard_len, out):
    import datetime

    import torch.distributed as dist

    import oracle
    from io_aware_exact_forward_b200 import context_parallel as cp
    from workloads import to_f64

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        inp = _inputs()
        lo = rank * shard_len
        k_shard = inp["k_cache"][:, lo:lo + shard_len].contiguous()
        v_shard = inp["v_cache"][:, lo:lo + shard_len].contiguous()
        sl = cp.shard_seqlens(inp["seqlens"], rank, shard_len)
        seen = {}

        def partial(q, k, v, seqlens, scale, chunk, workspace, out, lse):
            assert out.dtype == torch.float32 and out.shape == (B, HQ, D)
            assert lse.shape == (B, HQ)
            O, L = oracle.decode_forward(to_f64(q), to_f64(k), to_f64(v), seqlens.numpy(), scale)
            out.copy_(torch.from_numpy(O))
            lse.copy_(torch.from_numpy(L))
            seen["sl"] = seqlens.tolist()

        def merge(o_parts, lse_parts):
            n = cp.packed_block_floats(B, HQ, D)
            assert o_parts.shape == (world, B, HQ, D) and lse_parts.shape == (world, B, HQ)
            assert o_parts.stride(0) == n and lse_parts.stride(0) == n and n % 4 == 0
            assert o_parts[0].is_contiguous() and lse_parts[0].is_contiguous()
            O, L = oracle.merge_partials(o_parts.double().numpy(), lse_parts.double().numpy())
            return torch.from_numpy(O), torch.from_numpy(L)

        O, L = cp._cp_decode(inp["q"], k_shard, v_shard, sl, SCALE, 256, None, None, partial, merge)
        out.put((rank, seen["sl"], O.numpy(), L.numpy()))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("shard_len", [48, 100])
def test_two_gloo_ranks_context_parallel_decode(shard_len):
    import oracle
    from workloads import to_f64

    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, shard_len, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted([q.get(timeout=180) for _ in range(2)], key=lambda x: x[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    inp = _inputs()
    O_ref, L_ref = oracle.decode_forward(to_f64(inp["q"]), to_f64(inp["k_cache"]), to_f64(inp["v_cache"]),
                                         inp["seqlens"].numpy(), SCALE)
    lens = [1, 50, 96]
    for rank, sl, O, L in res:
        assert sl == [min(max(n - rank * shard_len, 0), shard_len) for n in lens]
        # the partials travel in fp32: agreement to fp32 rounding
        np.testing.assert_allclose(O, O_ref, rtol=1e-5, atol=1e-6)
        np.testing.assert_allclose(L, L_ref, rtol=1e-6)
    if shard_len >= 96:
        assert res[1][1] == [0, 0, 0]      # rank 1 holds no key at all


def test_shard_seqlens_contiguous_split():
    from io_aware_exact_forward_b200.context_parallel import packed_block_floats, shard_seqlens
    sl = torch.tensor([0, 1, 255, 256, 257, 1000], dtype=torch.int32)
    parts = [shard_seqlens(sl, r, 256) for r in range(4)]
    assert all(p.dtype == torch.int32 for p in parts)
    assert (sum(parts) == sl.clamp(max=1024)).all()
    assert parts[1].tolist() == [0, 0, 0, 0, 1, 256]
    assert packed_block_floats(1, 1, 64) == 68 and packed_block_floats(2, 4, 128) == 1032
    with pytest.raises(ValueError):
        shard_seqlens(sl, 0, 0)


def _failing_worker(rank, world, port, out):
    import datetime
    import time

    import torch.distributed as dist

    from io_aware_exact_forward_b200 import context_parallel as cp

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=10))
    if rank == 1:
        out.put((rank, "failed before the exchange"))
        out.close()
        out.join_thread()        # the message is out before the process ends
        os._exit(3)              # the rank dies between steps, with nothing in flight
    inp = _inputs()

    def partial(q, k, v, seqlens, scale, chunk, workspace, out, lse):
        out.zero_()
        lse.fill_(float("-inf"))

    t0 = time.monotonic()
    try:
        cp._cp_decode(inp["q"], inp["k_cache"], inp["v_cache"], inp["seqlens"], SCALE, 256, None, None, partial,
                      lambda o, l: (o, l))
        out.put((rank, "no error"))
    except Exception as e:      # the exchange reports the lost peer instead of hanging
        out.put((rank, f"error after {time.monotonic() - t0:.1f} s: {type(e).__name__}"))


def test_lost_rank_fails_the_exchange_instead_of_hanging():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_failing_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=90) for _ in range(2))
    for p in procs:
        p.join(timeout=60)
        if p.is_alive():
            p.kill()
    assert res[1] == "failed before the exchange"
    assert res[0].startswith("error after"), res[0]
    assert float(res[0].split()[2]) < 60.0
    assert procs[1].exitcode == 3
