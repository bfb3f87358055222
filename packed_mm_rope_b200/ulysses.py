"""Head-sharded (Ulysses) packed attention across ranks.

The pages' deployment runs full attention with sequence parallelism on four
GPUs (news article on the open weights; model card, SGLang deployment with
--ulysses-degree 4): every rank holds a contiguous shard of the packed rows
for all heads; an all-to-all regroups the data so each rank holds ALL rows
for its share of the heads; attention (with the rotary embedding) runs
locally per head; a second all-to-all returns each rank's rows.

Heads and rows are split as evenly as possible (42 heads over 4 ranks:
11, 11, 10, 10).  The exchanges are torch.distributed all-to-alls (NCCL on
GPUs); the per-head work runs in the library's kernels.
"""
from __future__ import annotations

from typing import Callable, List, Optional, Sequence


def even_split(n: int, parts: int) -> List[int]:
    """n items over ``parts`` ranks, the first n % parts ranks taking one more."""
    if parts < 1 or n < 0:
        raise ValueError("bad split")
    base, extra = divmod(n, parts)
    return [base + (1 if r < extra else 0) for r in range(parts)]


def _offsets(sizes: Sequence[int]) -> List[int]:
    out, acc = [], 0
    for s in sizes:
        out.append(acc)
        acc += s
    return out + [acc]


def _all_to_all(send_blocks, recv_shapes, group):
    """Exchange one block per rank.  Bit copies: pairs of bf16 travel as int32
    (every block holds a multiple of 128 values, so the count is even)."""
    import torch
    import torch.distributed as dist
    send = torch.cat([b.contiguous().reshape(-1).view(torch.int32) for b in send_blocks])
    in_splits = [b.numel() // 2 for b in send_blocks]
    out_splits = [int(torch.Size(s).numel()) // 2 for s in recv_shapes]
    recv = torch.empty(sum(out_splits), dtype=torch.int32, device=send.device)
    dist.all_to_all_single(recv, send, out_splits, in_splits, group=group)
    blocks, o = [], 0
    for shape, n in zip(recv_shapes, out_splits):
        blocks.append(recv[o:o + n].view(torch.bfloat16).reshape(shape))
        o += n
    return blocks


def _library_attention(segments, perm, q, k, v, theta, sections, pair_layout):
    from . import packed_mmrope_attention
    return packed_mmrope_attention(segments, q, k, v, perm=perm, theta=theta, sections=sections,
                                   pair_layout=pair_layout)


def ulysses_packed_mmrope_attention(segments, q_shard, k_shard, v_shard, perm=None, group=None,
                                    theta: float = 10000.0, sections=(32, 48, 48), pair_layout: int = 0, *,
                                    local_attention: Optional[Callable] = None):
    """Packed MM-RoPE attention with rows sharded over the ranks of ``group``.

    q_shard, k_shard, v_shard: bf16 [n_r, H, 128], this rank's rows in the
    even split of the packed sequence (rank order = row order).  ``perm``:
    the packed-row permutation of the whole sequence (as for
    h3_build_coords) or None.  Returns this rank's output rows [n_r, H, 128].

    ``local_attention`` (keyword only) replaces the library's per-head step;
    it exists so the exchange logic can be tested on CPU processes, where
    the library's kernels cannot run.  Leave it unset.
    """
    import torch
    import torch.distributed as dist
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    n_total = sum(s.rows if hasattr(s, "rows") else 0 for s in segments)
    rows = even_split(n_total, world)
    if q_shard.shape[0] != rows[rank]:
        raise ValueError(f"rank {rank} holds {q_shard.shape[0]} rows, expected {rows[rank]}")
    H, D = q_shard.shape[1], q_shard.shape[2]
    heads = even_split(H, world)
    hoff = _offsets(heads)
    local_attention = local_attention or _library_attention

    # rows x all heads  ->  all rows x my heads  (Q, K, V stacked into one exchange)
    qkv = torch.stack([q_shard, k_shard, v_shard])                       # [3, n_r, H, D]
    send = [qkv[:, :, hoff[s]:hoff[s + 1]] for s in range(world)]
    recv_shapes = [(3, rows[r], heads[rank], D) for r in range(world)]
    got = _all_to_all(send, recv_shapes, group)
    full = torch.cat(got, dim=1)                                           # [3, N, h_me, D]
    if heads[rank] > 0:
        o_local = local_attention(segments, perm, full[0].contiguous(), full[1].contiguous(),
                                  full[2].contiguous(), theta, sections, pair_layout)   # [N, h_me, D]
    else:
        o_local = full[0]
    # all rows x my heads  ->  my rows x all heads
    roff = _offsets(rows)
    send = [o_local[roff[s]:roff[s + 1]] for s in range(world)]
    recv_shapes = [(rows[rank], heads[r], D) for r in range(world)]
    got = _all_to_all(send, recv_shapes, group)
    return torch.cat(got, dim=1)                                           # [n_r, H, D]
