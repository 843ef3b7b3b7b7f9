"""Context-parallel attention forward: keys and values sharded across GPUs.

Every rank holds all query rows and one contiguous shard of each sequence's
keys and values.  A rank computes the normalised fp32 partial (O_r, LSE_r) of
its shard on its own GPU, the ranks exchange the partials (one all-gather of
B*Sq*Hq*(D+1)*4 bytes per rank), and each rank merges them by LSE:

    LSE = log sum_r exp(LSE_r),   O = sum_r exp(LSE_r - LSE) * O_r

which is the exact result over all keys, because the rows' softmax
normaliser factors over any partition of the keys.  The pages state the
merge for a split over keys done outside the kernel through the returned LSE
("FlashAttention-4 backend for Blackwell #1235"; the split-KV combine of
"mgoin/tml-fa4"); here the split is across GPUs.  Masks and relative bias
use each key's position in the whole sequence: a shard passes, per
sequence, the number of keys after it (``k_after``), which moves every row's
diagonal that far to the right (bottom-right alignment).

The exchange is an NCCL all-gather over the process group (gloo for CPU
tensors), then the merge runs in this library's combine kernel.
"""
from __future__ import annotations

from typing import List, Optional, Sequence, Tuple

import torch

from . import fa_combine_partials, fa_fwd_shard_partial


def shard_bounds(k_len: int, world: int, rank: int, align: int = 128) -> Tuple[int, int, int]:
    """Contiguous key shard of `rank` among `world`: (start, length, after).

    Shards hold whole multiples of `align` keys (one key tile) except the
    last, differ in size by at most one multiple, cover [0, k_len) without
    overlap, and are in rank order; `after` is the number of keys that
    follow the shard.  A rank may get an empty shard when k_len is short."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("need 0 <= rank < world")
    if k_len < 0 or align < 1:
        raise ValueError("need k_len >= 0 and align >= 1")
    blocks = -(-k_len // align)
    base, extra = divmod(blocks, world)
    first = rank * base + min(rank, extra)
    count = base + (1 if rank < extra else 0)
    start = min(first * align, k_len)
    end = min((first + count) * align, k_len)
    return start, end - start, k_len - end


def shard_seqused(seqused_k: Sequence[int], start: int, length: int) -> Tuple[List[int], List[int]]:
    """Per-sequence valid keys of a shard [start, start + length) of padded
    sequences whose first seqused_k[b] keys are valid: (valid keys in the
    shard, valid keys after the shard), both per sequence."""
    used, after = [], []
    for n in seqused_k:
        n = max(int(n), 0)
        used.append(min(max(n - start, 0), length))
        after.append(max(n - (start + length), 0))
    return used, after


def gather_partials(o_part: torch.Tensor, lse_part: torch.Tensor,
                    group=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """All ranks' partials, stacked in rank order: ([world, rows, D],
    [world, rows]).  One all-gather per tensor (into one buffer on NCCL).
    Without an initialised process group there is one rank and no exchange."""
    import torch.distributed as dist
    if group is None and not (dist.is_available() and dist.is_initialized()):
        return o_part.unsqueeze(0), lse_part.unsqueeze(0)
    world = dist.get_world_size(group)
    rows, D = o_part.shape
    if dist.get_backend(group) == "nccl":
        o_all = torch.empty((world, rows, D), dtype=o_part.dtype, device=o_part.device)
        l_all = torch.empty((world, rows), dtype=lse_part.dtype, device=lse_part.device)
        dist.all_gather_into_tensor(o_all, o_part.contiguous(), group=group)
        dist.all_gather_into_tensor(l_all, lse_part.contiguous(), group=group)
        return o_all, l_all
    o_list = [torch.empty_like(o_part) for _ in range(world)]
    l_list = [torch.empty_like(lse_part) for _ in range(world)]
    dist.all_gather(o_list, o_part.contiguous(), group=group)
    dist.all_gather(l_list, lse_part.contiguous(), group=group)
    return torch.stack(o_list), torch.stack(l_list)


def fa_fwd_context_parallel(q: torch.Tensor, k_shard: torch.Tensor, v_shard: torch.Tensor, *,
                            k_after: Optional[torch.Tensor] = None,
                            seqused_k: Optional[torch.Tensor] = None,
                            causal: bool = False, softmax_scale: Optional[float] = None,
                            rel_bias: Optional[torch.Tensor] = None,
                            window: Optional[Tuple[int, int]] = None, softcap: float = 0.0,
                            num_splits: int = 0, group=None,
                            out: Optional[torch.Tensor] = None,
                            lse: Optional[torch.Tensor] = None
                            ) -> Tuple[torch.Tensor, torch.Tensor]:
    """Forward over keys sharded across the ranks of `group`.

    q [B,Sq,Hq,D] holds every query row on every rank; k_shard/v_shard
    [B,Sk_r,Hkv,D] hold this rank's keys; k_after (device int32 [B]) the
    number of each sequence's keys on later shards; seqused_k (device int32
    [B], optional) this shard's valid keys.  Every rank returns the full
    (out [B,Sq,Hq,D], lse [B,Hq,Sq])."""
    B, Sq, Hq, _ = q.shape
    o_part, lse_part = fa_fwd_shard_partial(
        q, k_shard, v_shard, k_after=k_after, causal=causal, softmax_scale=softmax_scale,
        seqused_k=seqused_k, rel_bias=rel_bias, window=window, softcap=softcap,
        num_splits=num_splits)
    o_all, l_all = gather_partials(o_part, lse_part, group)
    return fa_combine_partials(o_all, l_all, B, Sq, Hq, dtype=q.dtype, out=out, lse=lse)
