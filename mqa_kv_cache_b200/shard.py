"""Sequence-sharded decode and lightning indexer over torch.distributed (one
process per GPU).

A long cache is cut into contiguous slices of ``shard_len`` positions, slice r on
rank r; every rank runs ``attn_decode_gqa`` over its slice (its keys rotated at
their global positions, the query at the sequence's position), the ranks exchange
their (out, lse) once with an all-gather, and each merges them with
``attn_merge_lse`` -- the softmax over the union of the slices.  The exchange is
B * H * (d * 2 + 4) bytes per rank.

The lightning indexer shards the same way: rank r scores keys r * shard_len ..
(r + 1) * shard_len - 1 and keeps its own top-k (dsa_index_topk); the ranks
all-gather their selections as (score, global index) pairs -- B * k * 8 bytes per
rank -- and each takes the top-k of the union with dsa_topk_merge, which is the
selection the unsharded indexer makes.  Plumbing only: the arithmetic runs in the
library's kernels.
"""
import torch
import torch.distributed as dist


def shard_lengths(seq_lens: torch.Tensor, rank: int, shard_len: int) -> torch.Tensor:
    """Rows of each sequence that fall in slice `rank` (positions rank * shard_len ..
    (rank + 1) * shard_len - 1): clamp(len - rank * shard_len, 0, shard_len)."""
    return (seq_lens - rank * shard_len).clamp(min=0, max=shard_len).to(torch.int32)


def gather_parts(out: torch.Tensor, lse: torch.Tensor, group=None):
    """All-gather every rank's (out [B, H, d], lse [B, H]) -> (o_parts [n, B, H, d],
    lse_parts [n, B, H]) in rank order."""
    n = dist.get_world_size(group)
    outs = [torch.empty_like(out) for _ in range(n)]
    lses = [torch.empty_like(lse) for _ in range(n)]
    dist.all_gather(outs, out.contiguous(), group=group)
    dist.all_gather(lses, lse.contiguous(), group=group)
    return torch.stack(outs), torch.stack(lses)


def sharded_decode_merge(out: torch.Tensor, lse: torch.Tensor, group=None):
    """This rank's decode over its slice -> the decode over the whole cache (every rank
    gets the same result)."""
    from . import kvattn
    o_parts, lse_parts = gather_parts(out, lse, group)
    return kvattn.attn_merge_lse(o_parts, lse_parts)


def gather_candidates(cand_scores: torch.Tensor, cand_idx: torch.Tensor, group=None):
    """All-gather every rank's candidates ([B, k] scores and global indices) -> ([n, B, k],
    [n, B, k]) in rank order (= increasing slice order)."""
    n = dist.get_world_size(group)
    cs = [torch.empty_like(cand_scores) for _ in range(n)]
    ci = [torch.empty_like(cand_idx) for _ in range(n)]
    dist.all_gather(cs, cand_scores.contiguous(), group=group)
    dist.all_gather(ci, cand_idx.contiguous(), group=group)
    return torch.stack(cs), torch.stack(ci)


def sharded_index_topk(q_idx, w, k_slice, k, rank, shard_len, seq_lens=None, group=None):
    """This rank's keys k_slice [B, shard_len, 128] (global positions rank * shard_len ..)
    -> the top-k of the whole rows (every rank gets the same selection)."""
    from . import kvattn
    lens = None if seq_lens is None else shard_lengths(seq_lens, rank, shard_len)
    idx, scores = kvattn.dsa_index_topk(q_idx, w, k_slice, k, seq_lens=lens)
    cs, ci = kvattn.dsa_topk_candidates(scores, idx, rank * shard_len)
    cs_all, ci_all = gather_candidates(cs, ci, group)
    return kvattn.dsa_topk_merge(cs_all, ci_all)
