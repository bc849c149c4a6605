"""Context-parallel split-KV decode: one batch of sequences whose KV caches are
spread over several GPUs, one process per GPU.

FlashDecoding ("FlashAttention", interview track, section "In practice")
splits a long KV cache into chunks, decodes each chunk separately and merges
the chunk results by their log-sum-exp.  Here the same split runs across
devices: rank r holds a share of every sequence's keys and values, and

  1. fa_decode_splitkv_partial decodes the local share into a normalised fp32
     O_r [B,Hq,d] and LSE_r [B,Hq], written into one packed block per rank
     (O first, then LSE, padded to 16 bytes);
  2. one all-gather over the process group (NCCL over NVLink on B200) brings
     every rank's block to every rank: (d + 1) * 4 bytes per (sequence, head)
     per rank;
  3. fa_decode_merge combines the R blocks,
       LSE = log sum_r e^{LSE_r},  O = sum_r e^{LSE_r - LSE} O_r
     (the online-softmax rescale of "Flash Attention: Why Memory Traffic, Not
     Compute, Is the Bottleneck", section "Softmax Looks Like an Obstacle",
     applied to whole shares).

The exchange is a few hundred KB to a few MB per step and latency-bound, so a
plain NCCL all-gather is used; all arithmetic runs in the library's kernels.
Keys may be shared out in any way (the unmasked softmax does not depend on key
order).  ``shard_seqlens`` gives the contiguous split: rank r holds positions
[r * shard_len, (r + 1) * shard_len) of every sequence.
"""

from __future__ import annotations

import torch
import torch.distributed as dist

from ._binding import decode_merge, decode_splitkv_partial

__all__ = ["packed_block_floats", "shard_seqlens", "decode_splitkv_cp"]


def packed_block_floats(B: int, Hq: int, d: int) -> int:
    """Floats in one rank's packed (O, LSE) block: B*Hq*d + B*Hq, rounded up
    to a multiple of 4 so that every block starts 16-byte aligned."""
    n = B * Hq * d + B * Hq
    return (n + 3) // 4 * 4


def shard_seqlens(seqlens: torch.Tensor, rank: int, shard_len: int) -> torch.Tensor:
    """Keys of each sequence that rank ``rank`` holds under the contiguous
    split (positions [rank * shard_len, (rank + 1) * shard_len)), as int32."""
    if shard_len < 1 or rank < 0:
        raise ValueError("shard_len must be >= 1 and rank >= 0")
    return (seqlens.to(torch.int64) - rank * shard_len).clamp(0, shard_len).to(torch.int32)


def _cp_decode(q, k_shard, v_shard, seqlens_shard, scale, chunk, group, workspace, partial, merge):
    B, Hq, d = q.shape
    world = dist.get_world_size(group)
    n = packed_block_floats(B, Hq, d)
    n_o = B * Hq * d
    local = torch.empty(n, dtype=torch.float32, device=q.device)
    partial(q, k_shard, v_shard, seqlens_shard, scale=scale, chunk=chunk, workspace=workspace,
            out=local[:n_o].view(B, Hq, d), lse=local[n_o:n_o + B * Hq].view(B, Hq))
    gathered = torch.empty(world * n, dtype=torch.float32, device=q.device)
    dist.all_gather_into_tensor(gathered, local, group=group)
    blocks = gathered.view(world, n)
    o_parts = blocks[:, :n_o].unflatten(1, (B, Hq, d))
    lse_parts = blocks[:, n_o:n_o + B * Hq].unflatten(1, (B, Hq))
    return merge(o_parts, lse_parts)


def decode_splitkv_cp(q, k_shard, v_shard, seqlens_shard, scale=None, chunk=256, group=None, workspace=None):
    """Decode one query token per sequence against KV caches shared out over
    the ranks of ``group``.

    q             bf16 [B,Hq,d], the same on every rank
    k/v_shard     bf16 [B,Tk_shard,Hkv,d], this rank's share of each cache
    seqlens_shard int32 [B], keys of each sequence in this rank's share (0
                  allowed: that rank then contributes nothing to the sequence)

    Every rank returns the full result O bf16 [B,Hq,d] and LSE fp32 [B,Hq].
    Collective: every rank of ``group`` must call it, with the same B, Hq, d."""
    return _cp_decode(q, k_shard, v_shard, seqlens_shard, scale, chunk, group, workspace,
                      decode_splitkv_partial, decode_merge)
