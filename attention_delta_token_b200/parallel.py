"""Tensor-parallel (head-sharded) eviction.

In a tensor-parallel engine each rank holds a contiguous slice of the query
heads and of their kv heads.  I_j is a sum over heads ("What carries the
argument": the column-wise sum of the attention the block's queries pay token
j), so each rank computes the importance of its own heads for both layers with
focus_partial_importance, one all-reduce (sum, fp32, 2 x R x B values) combines
them, and every rank then runs focus_evict_from_importance (delta, MaxPool1D,
mask, top-K, compaction) on the same numbers, so all ranks keep the same tokens.

The all-reduce can also be fused into the library's kernels (PeerExchange):
the kernel that reduces a rank's column sums stores them into every rank's
exchange buffer over peer memory and raises a flag there; each rank's
selection kernel waits for all flags and sums the slots in rank order.

All arithmetic runs in the library's kernels; this module only slices the work,
sets up the buffers and issues the collective through torch.distributed (NCCL
on GPUs).
"""
from __future__ import annotations

import torch

from . import (Workspace, focus_evict_from_exchange, focus_evict_from_importance,
               focus_exchange_buffer_size, focus_partial_importance,
               focus_partial_importance_push, make_dims)


def shard_heads(Hq: int, Hkv: int, rank: int, world: int) -> tuple[slice, slice]:
    """The query-head and kv-head slices rank `rank` owns (kv heads split evenly, each
    with its G = Hq/Hkv query heads)."""
    if Hkv % world:
        raise ValueError(f"Hkv = {Hkv} does not split over {world} ranks")
    G = Hq // Hkv
    kv = Hkv // world
    return slice(rank * kv * G, (rank + 1) * kv * G), slice(rank * kv, (rank + 1) * kv)


def partial_importance(R, B, Hq_local, Hkv_local, d, q0, k0_prefix, k0_block, q1, k1_prefix,
                       k1_block, cu_prefix, softmax_scale, out=None, ws=None, stream=None, score=0):
    """[2, R, B] float32: this rank's share of I0 and I1 (its heads only), from one
    focus_partial_importance call (planner, attention over both layers, reduction)."""
    dims = make_dims(R, B, Hq_local, Hkv_local, d, 8, softmax_scale, score=score)
    if ws is None:
        ws = Workspace(dims, q1.device, stream)
    if out is None:
        out = torch.empty(2, R, B, dtype=torch.float32, device=q1.device)
    focus_partial_importance(dims, q0, k0_prefix, k0_block, q1, k1_prefix, k1_block, cu_prefix,
                             out, ws, stream)
    return out


def finish_from_importance(dims, importance, decoded, budget, hidden, kept_idx, cu_seqlens,
                           packed, ws=None, delta_out=None, stream=None):
    """Delta, MaxPool1D, mask, top-K and compaction from the summed [2, R, B] importance
    (focus_evict_from_importance).  Returns the workspace, whose status covers the call."""
    if ws is None:
        ws = Workspace(dims, importance.device, stream)
    focus_evict_from_importance(dims, importance, hidden, decoded, budget, kept_idx, cu_seqlens,
                                packed, ws, delta_out=delta_out, stream=stream)
    return ws


class PeerExchange:
    """The exchange buffers of one rank: its own buffer, the device array of every rank's
    buffer address, and the step counter (epoch) all ranks advance together."""

    def __init__(self, buffer: torch.Tensor, peer_ptrs: torch.Tensor, rank: int, world: int,
                 handle=None):
        self.buffer, self.peer_ptrs, self.rank, self.world = buffer, peer_ptrs, rank, world
        self.handle = handle  # keeps a symmetric-memory mapping alive
        self.epoch = 0
        self.push_ws = None   # workspace of the pushing calls (its block counter persists)

    @classmethod
    def local(cls, dims, device) -> "PeerExchange":
        """A group of one: the rank exchanges with itself (the single-GPU form)."""
        buf = torch.zeros(focus_exchange_buffer_size(dims, 1), dtype=torch.uint8, device=device)
        ptrs = torch.tensor([buf.data_ptr()], dtype=torch.int64, device=device)
        return cls(buf, ptrs, 0, 1)

    @classmethod
    def symmetric(cls, dims, group=None) -> "PeerExchange":
        """One buffer per rank in torch symmetric memory (peer-mapped over NVLink); every
        rank of `group` must call this together."""
        import torch.distributed as dist
        import torch.distributed._symmetric_memory as symm_mem
        group = group or dist.group.WORLD
        world, rank = dist.get_world_size(group), dist.get_rank(group)
        nbytes = focus_exchange_buffer_size(dims, world)
        buf = symm_mem.empty(nbytes, dtype=torch.uint8, device=torch.device("cuda"))
        buf.zero_()
        handle = symm_mem.rendezvous(buf, group)
        ptrs = torch.tensor(list(handle.buffer_ptrs), dtype=torch.int64, device=buf.device)
        torch.cuda.synchronize()
        dist.barrier(group)  # every buffer is zero before anyone pushes
        return cls(buf, ptrs, rank, world, handle)

    def next_epoch(self) -> int:
        self.epoch += 1
        return self.epoch


def evict_head_sharded(dims, rank, world, q0, k0_prefix, k0_block, q1, k1_prefix, k1_block,
                       cu_prefix, hidden, decoded, budget, kept_idx, cu_seqlens, packed,
                       group=None, delta_out=None, stream=None, exchange=None, ws=None):
    """The fused step on one rank of a head-sharded group.  `dims` holds the full head
    counts; q*/k* are this rank's slices (shard_heads); the other arguments are the
    full per-request tensors, identical on every rank.  One all-reduce, or with
    `exchange` (a PeerExchange) the sums travel inside the library's kernels.  Returns the
    workspace of the selection."""
    world_heads = dims.Hq // world, dims.Hkv // world
    if exchange is not None:
        if exchange.buffer.numel() < focus_exchange_buffer_size(dims, exchange.world):
            raise ValueError("exchange buffer too small for these dims")
        sdims = make_dims(dims.R, dims.B, world_heads[0], world_heads[1], dims.head_dim, 8,
                          dims.softmax_scale, score=dims.score)
        if exchange.push_ws is None or exchange.push_ws.nbytes < Workspace.size(sdims):
            exchange.push_ws = Workspace(sdims, q1.device, stream)
        epoch = exchange.next_epoch()
        focus_partial_importance_push(sdims, q0, k0_prefix, k0_block, q1, k1_prefix, k1_block,
                                      cu_prefix, exchange.peer_ptrs, exchange.rank,
                                      exchange.world, epoch, exchange.push_ws, stream)
        if ws is None:
            ws = Workspace(dims, q1.device, stream)
        focus_evict_from_exchange(dims, exchange.buffer, exchange.world, epoch, hidden, decoded,
                                  budget, kept_idx, cu_seqlens, packed, ws, delta_out=delta_out,
                                  stream=stream)
        return ws
    part = partial_importance(dims.R, dims.B, world_heads[0], world_heads[1], dims.head_dim, q0,
                              k0_prefix, k0_block, q1, k1_prefix, k1_block, cu_prefix,
                              dims.softmax_scale, stream=stream, score=dims.score)
    if world > 1:
        torch.distributed.all_reduce(part, op=torch.distributed.ReduceOp.SUM, group=group)
    return finish_from_importance(dims, part, decoded, budget, hidden, kept_idx, cu_seqlens,
                                  packed, delta_out=delta_out, stream=stream)
