"""Context-parallel decode of one long sequence over G ranks (one process per GPU).

The pages describe CSA/HCA for a single device; at million-token contexts one
sequence's compressed caches can also be split over several GPUs.  This split
is exact (the same result as one GPU, up to rounding):

  * rank r holds the contiguous entry range [lo_r, lo_{r+1}) of each
    compressed cache (``shard_range``), lo ascending with r;
  * CSA: each rank scores its own entries and keeps its local top-k with their
    scores (``csa_indexer_topk_with_scores``, positions shifted by -lo_r * m so
    that visibility is unchanged); the ranks all-gather these (score, global
    index) candidates in rank order and every rank merges them into the global
    top-k (``csa_cp_topk_merge``) -- the top-k of the whole sequence is always
    among the local top-k's;
  * each rank attends over the selected entries it holds (indices outside its
    range fall outside [0, N_r) and are skipped by the kernel), rank 0 also over
    the sliding window (its range starts at entry 0, so no shift is needed);
    HCA: each rank attends densely over its own visible entries;
  * the partial (out, lse) are all-gathered and merged (``csa_cp_attn_merge``):
    one softmax over disjoint key sets is the lse-weighted merge of the parts.

Two exchanges per layer: k (score, index) pairs and H x 128 bf16 outputs plus
H lse values per query row and rank.  The compute steps are the library's
kernels (``KernelOps``); the exchange is ``torch.distributed.all_gather`` (NCCL
between GPUs).  The ops object is a parameter so that the host logic (ranges,
shifts, window ownership, exchange order) can also be driven on CPU ranks.
"""
from __future__ import annotations

import dataclasses

import torch


@dataclasses.dataclass(frozen=True)
class Shard:
    rank: int
    world: int
    lo: int      # first entry held
    hi: int      # one past the last entry held

    @property
    def n(self) -> int:
        return self.hi - self.lo


def shard_range(n_entries: int, world: int, rank: int) -> Shard:
    """Balanced contiguous entry range of `rank` (ranges ascend with the rank)."""
    if not 0 <= rank < world:
        raise ValueError("rank out of range")
    return Shard(rank, world, n_entries * rank // world, n_entries * (rank + 1) // world)


class KernelOps:
    """The library calls the context-parallel step is made of (CUDA tensors)."""

    def __init__(self):
        from . import _lib
        self.lib = _lib.load()

    def local_topk(self, qI, wI, kI_shard, m, k, q_pos0):
        from . import _check, _ptr, _stream, csa_indexer_topk_coded_workspace_size
        B, Tq = qI.shape[0], qI.shape[1]
        N = kI_shard.shape[1]
        idx = torch.empty(B, Tq, k, dtype=torch.int32, device=qI.device)
        sc = torch.empty(B, Tq, k, dtype=torch.float32, device=qI.device)
        ws = torch.empty(max(1, csa_indexer_topk_coded_workspace_size(B, Tq, N, k)), dtype=torch.uint8,
                         device=qI.device)
        st = self.lib.csa_indexer_topk_with_scores(_ptr(qI), _ptr(wI), _ptr(kI_shard), B, Tq, N, q_pos0, m, k,
                                                   _ptr(idx), _ptr(sc), _ptr(ws), ws.numel(), _stream(None))
        _check(st, "csa_indexer_topk_with_scores")
        return idx, sc

    def topk_merge(self, cand_scores, cand_idx, k):
        from . import _check, _ptr, _stream
        lead = cand_scores.shape[:-1]
        n = cand_scores.shape[-1]
        R = cand_scores.numel() // n
        idx = torch.empty(*lead, k, dtype=torch.int32, device=cand_scores.device)
        st = self.lib.csa_cp_topk_merge(_ptr(cand_scores.contiguous()), _ptr(cand_idx.contiguous()), R, n, k,
                                        _ptr(idx), _stream(None))
        _check(st, "csa_cp_topk_merge")
        return idx

    def sparse_mqa(self, q, cache, m, idx, win, scale, q_pos0):
        from . import csa_sparse_mqa
        return csa_sparse_mqa(q, cache, m, idx, win, scale, q_pos0=q_pos0)

    def dense_mqa(self, q, cache, m_prime, win, scale, q_pos0):
        from . import hca_dense_mqa
        return hca_dense_mqa(q, cache, m_prime, win, scale, q_pos0=q_pos0)

    def attn_merge(self, outs, lses):
        from . import _check, _ptr, _stream
        G = outs.shape[0]
        H = outs.shape[-2]
        R = outs[0].numel() // (H * 128)
        out = torch.empty(outs.shape[1:], dtype=torch.bfloat16, device=outs.device)
        lse = torch.empty(lses.shape[1:], dtype=torch.float32, device=lses.device)
        st = self.lib.csa_cp_attn_merge(_ptr(outs.contiguous()), _ptr(lses.contiguous()), G, R, H, _ptr(out),
                                        _ptr(lse), _stream(None))
        _check(st, "csa_cp_attn_merge")
        return out, lse


def empty_candidates(qI, k):
    B, Tq = qI.shape[0], qI.shape[1]
    return (torch.full((B, Tq, k), -1, dtype=torch.int32, device=qI.device),
            torch.full((B, Tq, k), float("-inf"), dtype=torch.float32, device=qI.device))


def local_candidates(ops, shard: Shard, qI, wI, kI_shard, m, k, t):
    """This rank's (scores, global indices) of its local top-k for queries at position t."""
    t_loc = t - shard.lo * m   # entry lo + j is visible at t iff (j + 1) m - 1 <= t_loc
    if t_loc < 0 or shard.n == 0:
        idx, sc = empty_candidates(qI, k)
        return sc, idx
    idx, sc = ops.local_topk(qI, wI, kI_shard, m, k, t_loc)
    gidx = torch.where(idx >= 0, idx + shard.lo, idx)
    return sc, gidx


def merge_candidates(ops, scores_by_rank, idx_by_rank, k):
    """Global top-k from the ranks' candidate lists (in rank order)."""
    return ops.topk_merge(torch.cat(list(scores_by_rank), dim=-1), torch.cat(list(idx_by_rank), dim=-1), k)


def _no_keys(q):
    B, Tq, H = q.shape[0], q.shape[1], q.shape[2]
    return (torch.zeros(B, Tq, H, 128, dtype=torch.bfloat16, device=q.device),
            torch.full((B, Tq, H), float("-inf"), dtype=torch.float32, device=q.device))


def local_sparse_attention(ops, shard: Shard, q, cache_shard, m, sel, win, scale, t):
    """This rank's part of the CSA attention: its selected entries (and, on rank 0, the window)."""
    t_loc = t - shard.lo * m
    w = win if shard.rank == 0 else None
    if t_loc < 0 or (shard.n == 0 and w is None):
        return _no_keys(q)
    idx_loc = torch.where(sel >= 0, sel - shard.lo, sel).to(torch.int32).contiguous()
    return ops.sparse_mqa(q, cache_shard, m, idx_loc, w, scale, t_loc)


def local_dense_attention(ops, shard: Shard, q, cache_shard, m_prime, win, scale, t):
    """This rank's part of the HCA attention: its own visible entries (and, on rank 0, the window)."""
    t_loc = t - shard.lo * m_prime
    w = win if shard.rank == 0 else None
    if t_loc < 0 or (shard.n == 0 and w is None):
        return _no_keys(q)
    return ops.dense_mqa(q, cache_shard, m_prime, w, scale, t_loc)


def _all_gather(t, group):
    import torch.distributed as dist
    parts = [torch.empty_like(t) for _ in range(dist.get_world_size(group))]
    dist.all_gather(parts, t.contiguous(), group=group)
    return parts


def csa_decode_step(ops, shard: Shard, q, qI, wI, kI_shard, cache_shard, m, k, win, scale, t, group=None):
    """One CSA decode step for queries at position t, over this rank's shard; returns (out, lse, selection) of
    the whole sequence on every rank.  Two all-gathers: the candidates, then the partial attentions."""
    sc, gidx = local_candidates(ops, shard, qI, wI, kI_shard, m, k, t)
    sel = merge_candidates(ops, _all_gather(sc, group), _all_gather(gidx, group), k)
    out, lse = local_sparse_attention(ops, shard, q, cache_shard, m, sel, win, scale, t)
    out, lse = ops.attn_merge(torch.stack(_all_gather(out, group)), torch.stack(_all_gather(lse, group)))
    return out, lse, sel


def hca_decode_step(ops, shard: Shard, q, cache_shard, m_prime, win, scale, t, group=None):
    """One HCA decode step over this rank's shard of the heavily compressed cache; one all-gather."""
    out, lse = local_dense_attention(ops, shard, q, cache_shard, m_prime, win, scale, t)
    return ops.attn_merge(torch.stack(_all_gather(out, group)), torch.stack(_all_gather(lse, group)))
