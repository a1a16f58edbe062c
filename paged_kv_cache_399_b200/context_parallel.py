"""Decode of long sequences split over the GPUs of a process group (context parallelism).

Every rank holds the blocks of one contiguous range of table entries of every sequence
in its own pool; it computes the attention over that range as unnormalised pieces
(pa_decode_partial, its range cut into as many pieces as the decode heuristic would split
it) and combines them into one record per row (pa_combine_partials); the records are
all-gathered (world * B * q * H_q * (D + 2) floats); every rank then merges them by the
log-sum-exp rule of split softmax (pa_merge_partials; vLLM study notes, zihan-zhang.net,
§4.3.1).
The exchange is the only communication: each rank reads its own pool only.
"""

from __future__ import annotations

import torch
import torch.distributed as dist

from . import pa


def rank_block_range(max_blocks_per_seq: int, rank: int, world: int) -> tuple[int, int]:
    """Table entries [lo, hi) that `rank` of `world` holds: contiguous ranges of
    ceil(max_blocks_per_seq / world) entries, the last ones possibly shorter or empty."""
    if world <= 0 or not 0 <= rank < world:
        raise ValueError("rank outside the group")
    per = -(-max_blocks_per_seq // world)
    lo = min(max_blocks_per_seq, rank * per)
    return lo, min(max_blocks_per_seq, lo + per)


def gather_partials(part_o: torch.Tensor, part_ml: torch.Tensor, group=None) -> tuple[torch.Tensor, torch.Tensor]:
    """All-gather of every rank's pieces, part-major in rank order: ([world, *part_o.shape],
    [world, *part_ml.shape]). CUDA tensors go through one all_gather_into_tensor each (NCCL);
    CPU tensors (gloo) through all_gather."""
    world = dist.get_world_size(group)
    out_o = part_o.new_empty((world,) + tuple(part_o.shape))
    out_ml = part_ml.new_empty((world,) + tuple(part_ml.shape))
    if part_o.is_cuda:
        dist.all_gather_into_tensor(out_o, part_o.contiguous(), group=group)
        dist.all_gather_into_tensor(out_ml, part_ml.contiguous(), group=group)
    else:
        dist.all_gather(list(out_o.unbind(0)), part_o.contiguous(), group=group)
        dist.all_gather(list(out_ml.unbind(0)), part_ml.contiguous(), group=group)
    return out_o, out_ml


def context_parallel_decode(out: torch.Tensor, query: torch.Tensor, key_cache: torch.Tensor,
                            value_cache: torch.Tensor, block_tables: torch.Tensor, context_lens: torch.Tensor,
                            q_per_seq: int, scale: float, group=None) -> None:
    """pa_decode's result in `out` on every rank of `group`. This rank's block_tables entries
    in its range (rank_block_range) name blocks of its own key_cache / value_cache; query and
    context_lens are the same on every rank. Runs on torch's current stream, the one the
    collective is ordered against."""
    rank, world = dist.get_rank(group), dist.get_world_size(group)
    mb = block_tables.shape[1]
    lo, hi = rank_block_range(mb, rank, world)
    B, QS, HQ, D = query.shape
    S = partial_pieces(query, key_cache, mb, world)
    part_o = torch.empty((S, B, QS, HQ, D), dtype=torch.float32, device=query.device)
    part_ml = torch.empty((S, B, QS, HQ, 2), dtype=torch.float32, device=query.device)
    pa.pa_decode_partial(part_o, part_ml, query, key_cache, value_cache, block_tables, context_lens, q_per_seq,
                         scale, lo, hi)
    rec_o = torch.empty((B, QS, HQ, D), dtype=torch.float32, device=query.device)
    rec_ml = torch.empty((B, QS, HQ, 2), dtype=torch.float32, device=query.device)
    pa.pa_combine_partials(rec_o, rec_ml, part_o, part_ml)
    all_o, all_ml = gather_partials(rec_o, rec_ml, group)
    pa.pa_merge_partials(out, all_o, all_ml)


def partial_pieces(query: torch.Tensor, key_cache: torch.Tensor, max_blocks_per_seq: int, world: int) -> int:
    """Pieces per rank: the split count of the decode heuristic for a rank's range, the same on
    every rank of the group."""
    B, QS, HQ, D = query.shape
    per = -(-max_blocks_per_seq // world)
    S = pa.pa_decode_partial_pieces(B, QS, HQ, key_cache.shape[2], D, per)
    if S <= 0:
        raise ValueError("shapes outside the supported set")
    return S
