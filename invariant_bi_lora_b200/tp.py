"""Tensor-parallel tree GEMM across ranks: the one exchange step of the path.

"Deterministic Inference across Tensor Parallel Sizes That Eliminates
Training-Inference Mismatch" (Abstract): the intra- and inter-GPU reductions
follow one hierarchical binary tree, so C = A . W^T has the same bits for
every TP size.  Row-parallel layout: rank q of `world` holds the contiguous
K range [q*K/world, (q+1)*K/world) of A and of W (whole 256-wide leaves).

A rank's partial is the canonical tree over its own leaves, which is the
subtree the single-GPU kernel computes for shard q (`bi_gemm_tree` with
shards=1 on the rank's slice).  The partials are gathered in rank order
(all-gather, never an all-reduce, whose order NCCL does not fix) and every
rank adds the top log2(world) levels with `bi_tree_combine`.  The result is
bitwise equal to `bi_gemm_tree(A, W, C, shards=world)` on one GPU, and to the
same call with any other power-of-two shard count.

A second exchange, `tree_gemm_tp_peers`, moves no data through NCCL: each
rank's partial lives in symmetric memory, and after a barrier one kernel
(`bi_tree_combine_peers`) on every rank reads all ranks' partials through
their peer pointers with plain loads (no multicast) and adds them by the
same tree; a second barrier keeps every partial alive until all ranks have
read it.  Same bits as the all-gather path.

The compute steps default to the library's kernels; `partial_fn`,
`combine_fn`, `combine_peers_fn` and `barrier_fn` exist so that the rank
logic can be exercised by CPU process groups.
"""
from __future__ import annotations

from typing import Callable, Optional

import torch
import torch.distributed as dist

LEAF = 256


def shard_k_range(K: int, world: int, rank: int, leaf: int = LEAF) -> tuple[int, int]:
    """K range [k0, k1) of `rank`: a contiguous block of whole leaves.
    world must be a power of two dividing the leaf count."""
    if K % leaf:
        raise ValueError(f"K={K} is not a multiple of the leaf width {leaf}")
    leaves = K // leaf
    if world < 1 or world & (world - 1) or leaves % world:
        raise ValueError(f"world={world} must be a power of two dividing {leaves} leaves")
    if not 0 <= rank < world:
        raise ValueError(f"rank {rank} outside [0, {world})")
    per = leaves // world
    return rank * per * leaf, (rank + 1) * per * leaf


def _gpu_partial(A_local, W_local, out):
    from invariant_bi_lora_b200 import bi
    bi.gemm_tree(A_local, W_local, out, shards=1)


def _gpu_combine(parts, out):
    from invariant_bi_lora_b200 import bi
    bi.tree_combine(parts, out)


def tree_gemm_tp(A_local: torch.Tensor, W_local: torch.Tensor, C: torch.Tensor,
                 group: Optional[dist.ProcessGroup] = None,
                 partial_fn: Optional[Callable] = None,
                 combine_fn: Optional[Callable] = None,
                 check_finite: bool = False) -> torch.Tensor:
    """C = sum over ranks of A_q . W_q^T, reduced by the canonical tree.

    A_local [M][K/world] and W_local [N][K/world] (bf16, K-contiguous) are
    this rank's slices; C [M][N] fp32 receives the full result on every
    rank.  Collective: every rank of `group` must call it with the same M, N
    and slice width.  A rank that fails or leaves before the gather makes
    the collective raise on the others (the process group's timeout bounds
    the wait).  With check_finite, every rank inspects the gathered partials
    before the combine and raises, naming the ranks, if any holds a NaN or an
    infinity; all ranks see the same partials, so all raise together."""
    partial_fn = partial_fn or _gpu_partial
    combine_fn = combine_fn or _gpu_combine
    world = dist.get_world_size(group) if dist.is_initialized() else 1
    if world & (world - 1):
        raise ValueError(f"world size {world} is not a power of two")
    M, N = C.shape
    if A_local.shape[0] != M or W_local.shape[0] != N or A_local.shape[1] != W_local.shape[1]:
        raise ValueError("slice shapes do not match C")
    if world == 1:
        partial_fn(A_local, W_local, C)
        return C
    partial = torch.empty(M, N, dtype=torch.float32, device=C.device)
    partial_fn(A_local, W_local, partial)
    parts = torch.empty(world * M, N, dtype=torch.float32, device=C.device)
    dist.all_gather_into_tensor(parts, partial, group=group)      # concatenated in rank order
    if check_finite:
        ok = torch.isfinite(parts.view(world, -1)).all(dim=1).tolist()
        bad = [q for q, good in enumerate(ok) if not good]
        if bad:
            raise RuntimeError(f"tree_gemm_tp: non-finite partial from rank(s) {bad}")
    combine_fn(parts.view(world, M, N), C)
    return C


class PeerPartials:
    """This rank's partial, fp32 [M][N], in symmetric memory, and the device
    pointers (ints) of every rank's partial as mapped into this process, in
    rank order.  Collective: every rank of `group` creates one with the same
    M and N; reuse it across calls of the same shape."""

    def __init__(self, M: int, N: int, group: Optional[dist.ProcessGroup] = None, device=None):
        import torch.distributed._symmetric_memory as symm_mem
        device = device or torch.device("cuda", torch.cuda.current_device())
        self.buf = symm_mem.empty(M, N, dtype=torch.float32, device=device)
        self.handle = symm_mem.rendezvous(self.buf, group or dist.group.WORLD)
        self.ptrs = [int(q) for q in self.handle.buffer_ptrs]


def _gpu_combine_peers(peers, out):
    from invariant_bi_lora_b200 import bi
    bi.tree_combine_peers(peers.ptrs, out)


def _device_barrier(group):
    # the partials' kernels (or the combine's reads) on this GPU end before
    # the ranks meet
    torch.cuda.current_stream().synchronize()
    dist.barrier(group=group)


def tree_gemm_tp_peers(A_local: torch.Tensor, W_local: torch.Tensor, C: torch.Tensor, peers,
                       group: Optional[dist.ProcessGroup] = None,
                       partial_fn: Optional[Callable] = None,
                       combine_peers_fn: Optional[Callable] = None,
                       barrier_fn: Optional[Callable] = None) -> torch.Tensor:
    """C = sum over ranks of A_q . W_q^T by the canonical tree, the exchange
    done by peer loads: this rank's partial into peers.buf, a barrier, one
    combine kernel reading every rank's peers.buf through peers.ptrs, a
    barrier.  Bitwise equal to `tree_gemm_tp` and to the one-GPU
    `bi_gemm_tree(shards=world)`.  `peers` is a PeerPartials of C's shape.
    A rank that fails or leaves makes the others' barrier raise (the process
    group's timeout bounds the wait)."""
    partial_fn = partial_fn or _gpu_partial
    combine_peers_fn = combine_peers_fn or _gpu_combine_peers
    barrier_fn = barrier_fn or _device_barrier
    world = dist.get_world_size(group) if dist.is_initialized() else 1
    if world & (world - 1):
        raise ValueError(f"world size {world} is not a power of two")
    M, N = C.shape
    if A_local.shape[0] != M or W_local.shape[0] != N or A_local.shape[1] != W_local.shape[1]:
        raise ValueError("slice shapes do not match C")
    if tuple(peers.buf.shape) != (M, N) or len(peers.ptrs) != world:
        raise ValueError("peers does not match C or the group")
    partial_fn(A_local, W_local, peers.buf)
    barrier_fn(group)                  # every partial is written before any rank reads it
    combine_peers_fn(peers, C)
    barrier_fn(group)                  # every rank has read before any partial is rewritten
    return C


def max_over_ranks(values, device="cpu", group: Optional[dist.ProcessGroup] = None) -> list[float]:
    """Elementwise maximum of `values` over the ranks of `group` (one
    all-reduce); the values themselves when no process group is running."""
    vals = [float(v) for v in values]
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size(group) == 1:
        return vals
    t = torch.tensor(vals, dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX, group=group)
    return [float(v) for v in t.tolist()]
