"""Sequence-sharded decode across the ranks of a torch.distributed group.

The cache of one sequence (length L, the query at position L - 1) is split
along L: each rank holds the contiguous rows [pos0, pos0 + L_shard) as its
own K and V.  The result (O, and the index set C_i with its count) is that
of a decode over the whole cache ("Condensate Theorem（冷凝定理）：注意力稀疏性的
拓扑本质", §2.1 Definition 1 for the last row, §2.2.3 Top-k, §5.2.2 select
then attend).  Every rank runs the same steps, in the same order:

1. its shard's best keys (condensate_attn_decode_shard_select);
2. an all-gather of those keys: P * k * 8 bytes per (batch, q-head);
3. the sequence's exact Top-k from them (the same on every rank), and the
   shard's softmax state over its members of C_i
   (condensate_attn_decode_shard_attend);
4. an all-gather of those states: P * (d + 2) * 4 bytes per (batch, q-head);
5. the combined output (condensate_attn_decode_shard_combine).

Every arithmetic step runs in the library's kernels; this module only moves
the two small exchanges through the process group (NCCL on GPUs).
"""
from typing import Optional, Tuple

import torch

from . import binding


def shard_bounds(L: int, P: int, rank: int) -> Tuple[int, int]:
    """(pos0, L_shard) of rank `rank` when L rows are split into P
    contiguous shards of nearly equal length (the first L % P one longer)."""
    if not 0 <= rank < P or L < P:
        raise ValueError(f"cannot split {L} rows over {P} ranks")
    base, extra = divmod(L, P)
    pos0 = rank * base + min(rank, extra)
    return pos0, base + (1 if rank < extra else 0)


def _all_gather(t: torch.Tensor, group, dist) -> torch.Tensor:
    """[P, *t.shape]: every rank's t in rank order."""
    P = dist.get_world_size(group)
    out = torch.empty((P,) + tuple(t.shape), dtype=t.dtype, device=t.device)
    if dist.get_backend(group) == "nccl":
        dist.all_gather_into_tensor(out, t.contiguous(), group=group)
    else:
        dist.all_gather(list(out.unbind(0)), t.contiguous(), group=group)
    return out


def decode_sharded(q: torch.Tensor, K: torch.Tensor, V: torch.Tensor,
                   pos0: int, L: int, W: int, k: int,
                   W_i: Optional[torch.Tensor] = None,
                   o_dtype: torch.dtype = torch.float32, group=None,
                   ops=None, dist=None):
    """Decode of q [B, Hq, d] against a cache of L rows of which this rank
    holds rows [pos0, pos0 + K.shape[2]) in K, V [B, Hkv, L_shard, d].

    Returns (O [B, Hq, d], idx [B, Hq, C_max], idx_count [B, Hq]), the same
    on every rank.  `ops` (the binding by default) provides the three
    per-rank steps; `dist` is torch.distributed unless given.
    """
    if dist is None:
        import torch.distributed as dist
    ops = binding if ops is None else ops
    keys = ops.condensate_attn_decode_shard_select(q, K, pos0, L, W, k,
                                                   W_i=W_i)
    keys_all = _all_gather(keys, group, dist)
    partial, idx, cnt = ops.condensate_attn_decode_shard_attend(
        q, K, V, pos0, L, W, k, keys_all, W_i=W_i)
    parts = _all_gather(partial, group, dist)
    O = ops.condensate_attn_decode_shard_combine(parts, o_dtype=o_dtype)
    return O, idx, cnt
