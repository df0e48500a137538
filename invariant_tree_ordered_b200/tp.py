"""Tensor parallelism across GPUs with the tree's shard level (one process per
GPU; torch.distributed carries the exchange).

The TBIK summary page ("Deterministic Inference across Tensor Parallel Sizes
That Eliminates Training-Inference Mismatch", 技术框架) orders the reduction
across GPUs by the same hierarchical binary tree as the reduction on each GPU.
Here each rank computes the root of its own subtree with the library's kernels,
an all-gather places the T shard results, in rank order, in every rank's own
memory, and every rank applies the top log2(T) levels of the tree locally
(tbik_tree_combine / tbik_logprob_combine).  A sum all-reduce is never used: its
internal order depends on the rank count, which is exactly the dependence the
method removes.  The results are bitwise those of the one-GPU calls for every T.

Argument marshalling and the collective only; every arithmetic step runs in
the library's CUDA kernels.
"""
from __future__ import annotations

from . import _binding as tbik


def _dist():
    import torch.distributed as dist
    return dist


def gather_shards(local, group=None):
    """All-gather of every rank's ``local`` tensor into a new tensor
    [T, *local.shape] in rank order, in this rank's own memory."""
    import torch
    dist = _dist()
    T = dist.get_world_size(group)
    local = local.contiguous()
    if local.dim() == 0:
        local = local.reshape(1)
    # concatenated along dim 0 (the form every backend accepts), then viewed as [T, ...]
    out = torch.empty((T * local.shape[0], *local.shape[1:]), dtype=local.dtype, device=local.device)
    dist.all_gather_into_tensor(out, local, group=group)
    return out.view(T, *local.shape)


def gemm_row_parallel(A_shard, B_shard, *, group=None, leaf: int = 256, tc: bool = True, noninv: bool = False,
                      b_nk: bool = False, out_bf16: bool = False, residual=None, stream=None):
    """C = A @ B with K split over the T ranks of ``group`` (row-parallel, as the
    distributed-training tutorial's figure 5 splits the second MLP layer).
    Rank t holds A[:, t*K/T:(t+1)*K/T] and the matching rows of B (columns with
    b_nk); K/T must be a whole number of leaves.  Each rank's fp32 subtree root
    is gathered and the shard level of the tree applied on every rank (with
    noninv, each rank's one chain and the left-to-right sum of the baseline).
    Returns C on every rank: fp32, or bf16 rounded once (out_bf16, or when a
    bf16 residual is added to the root first)."""
    q = tbik.gemm(A_shard, B_shard, T=1, leaf=leaf, tc=tc, noninv=noninv, b_nk=b_nk, stream=stream)
    parts = gather_shards(q, group)
    return tbik.tree_combine(parts, noninv=noninv, out_bf16=out_bf16, residual=residual, stream=stream)


def logprob_vocab_parallel(hidden, W_shard, targets, V: int, *, group=None, leaf: int = 256, tc: bool = True,
                           stream=None):
    """Target logprobs with the lm_head split over the vocabulary: rank t holds
    the rows of W_lm that ``vocab_shard(V, T, t)`` assigns it (possibly none).
    Each rank's per-row summary (m, s, z, owner) is gathered and the shard level
    of the vocabulary tree applied on every rank.  Returns fp32 [M]."""
    dist = _dist()
    T = dist.get_world_size(group)
    t = dist.get_rank(group)
    v0, vs, lvs = tbik.vocab_shard(V, T, t)
    if W_shard.shape[0] != vs:
        raise ValueError(f"rank {t} of {T} must hold {vs} vocabulary rows starting at {v0}")
    part = tbik.logprob_partial(hidden, W_shard, targets, v0=v0, Lvs=lvs, leaf=leaf, tc=tc, stream=stream)
    parts = gather_shards(part, group)
    return tbik.logprob_combine(parts, targets, V, stream=stream)
