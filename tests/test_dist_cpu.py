"""Multi-rank host logic on CPU process groups (gloo, world sizes 2 and 4).

- max_over_ranks: the bench's device-time reduction (every rank gets the
  elementwise maximum).
- tree_gemm_tp and tree_gemm_tp_peers: the tensor-parallel exchange of the
  tree GEMM, by all-gather and by peer loads ("Deterministic
  Inference across Tensor Parallel Sizes That Eliminates Training-Inference
  Mismatch", Abstract).  Each rank computes the subtree over its own K range,
  the partials are gathered in rank order and the top levels are added.  The
  leaf and combine steps are the oracle's here (the GPU kernels need a GPU);
  what is checked is the rank plumbing: K ranges, gather order, and that the
  result is the oracle's canonical tree over all leaves, bit for bit.
"""
import datetime
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from invariant_bi_lora_b200 import synth
from invariant_bi_lora_b200.tp import LEAF, max_over_ranks, shard_k_range, tree_gemm_tp, tree_gemm_tp_peers

M, N, K = 24, 16, 2048          # 8 leaves of 256


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _leaf_values(a, w):
    """Stand-in leaf values: each 256-wide leaf's exact product rounded to
    fp32 (the GPU's leaves come from the tensor core)."""
    L = a.shape[1] // LEAF
    out = []
    for l in range(L):
        sl = slice(l * LEAF, (l + 1) * LEAF)
        exact, _ = oracle.gemm_exact(np.ascontiguousarray(a[:, sl]), np.ascontiguousarray(w[:, sl]))
        out.append(exact.astype(np.float32))
    return np.stack(out)


def _bits(t):
    return torch.as_tensor(t).contiguous().view(torch.int32).numpy()


def _worker(rank, world, port, result_dir):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        got = max_over_ranks([rank, 10 - rank, 0.5 * rank])
        assert got == [world - 1, 10.0, 0.5 * (world - 1)], got

        a, w = synth.gemm_inputs(M, N, K, seed=7)
        k0, k1 = shard_k_range(K, world, rank)
        a_loc = torch.from_numpy(np.ascontiguousarray(a[:, k0:k1]).view(np.int16))
        w_loc = torch.from_numpy(np.ascontiguousarray(w[:, k0:k1]).view(np.int16))

        def partial_fn(A_local, W_local, out):
            leaves = _leaf_values(A_local.numpy().view(np.uint16), W_local.numpy().view(np.uint16))
            out.copy_(torch.from_numpy(oracle.tree_combine(leaves)))

        def combine_fn(parts, out):
            out.copy_(torch.from_numpy(oracle.tree_combine(parts.numpy())))

        C = torch.empty(M, N, dtype=torch.float32)
        tree_gemm_tp(a_loc, w_loc, C, partial_fn=partial_fn, combine_fn=combine_fn)
        np.save(os.path.join(result_dir, f"c{rank}.npy"), _bits(C))

        # the peer-load exchange: the partial goes into this rank's shared
        # buffer; "peer loads" are stood in for by gathering the buffers
        # (on CPU there is no peer memory), after the first barrier
        class Peers:
            buf = torch.full((M, N), 7.0, dtype=torch.float32)
            ptrs = list(range(world))
        events = []

        def combine_peers_fn(peers, out):
            got = [torch.empty_like(peers.buf) for _ in range(world)]
            dist.all_gather(got, peers.buf)
            events.append("combine")
            out.copy_(torch.from_numpy(oracle.tree_combine(torch.stack(got).numpy())))

        def barrier_fn(group):
            events.append("barrier")
            dist.barrier(group=group)

        C2 = torch.empty(M, N, dtype=torch.float32)
        tree_gemm_tp_peers(a_loc, w_loc, C2, Peers(), partial_fn=partial_fn, combine_peers_fn=combine_peers_fn,
                           barrier_fn=barrier_fn)
        assert events == ["barrier", "combine", "barrier"], events
        np.save(os.path.join(result_dir, f"p{rank}.npy"), _bits(C2))
    finally:
        dist.destroy_process_group()


def _fault_worker(rank, world, port, result_dir, kind):
    """Host-side failures: a rank whose partial is NaN (kind 'nan'), or a
    rank that leaves before the collective (kind 'leave')."""
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=10))
    try:
        if kind == "leave" and rank == world - 1:
            return
        a, w = synth.gemm_inputs(M, N, K, seed=3)
        k0, k1 = shard_k_range(K, world, rank)
        a_loc = torch.from_numpy(np.ascontiguousarray(a[:, k0:k1]).view(np.int16))
        w_loc = torch.from_numpy(np.ascontiguousarray(w[:, k0:k1]).view(np.int16))

        def partial_fn(A_local, W_local, out):
            out.copy_(torch.from_numpy(oracle.tree_combine(
                _leaf_values(A_local.numpy().view(np.uint16), W_local.numpy().view(np.uint16)))))
            if kind == "nan" and rank == 1:
                out[3, 5] = float("nan")

        def combine_fn(parts, out):
            out.copy_(torch.from_numpy(oracle.tree_combine(parts.numpy())))

        C = torch.empty(M, N, dtype=torch.float32)
        try:
            tree_gemm_tp(a_loc, w_loc, C, partial_fn=partial_fn, combine_fn=combine_fn, check_finite=True)
            msg = "no error"
        except RuntimeError as e:
            msg = str(e)
        with open(os.path.join(result_dir, f"r{rank}.txt"), "w") as f:
            f.write(msg)
    finally:
        if not (kind == "leave" and rank == world - 1):
            try:
                dist.destroy_process_group()
            except Exception:
                pass


@pytest.mark.parametrize("kind", ["nan", "leave"])
def test_tp_failures_are_reported(tmp_path, kind):
    oracle.tree_sum(np.zeros(1, np.float32))
    world = 2
    mp.start_processes(_fault_worker, args=(world, _free_port(), str(tmp_path), kind), nprocs=world,
                       join=True, start_method="spawn")
    if kind == "nan":
        for r in range(world):
            assert "non-finite partial from rank(s) [1]" in (tmp_path / f"r{r}.txt").read_text(), r
    else:
        msg = (tmp_path / "r0.txt").read_text()
        assert msg != "no error", msg           # the survivor's collective failed, it did not hang


def test_shard_k_range():
    assert shard_k_range(4096, 4, 0) == (0, 1024)
    assert shard_k_range(4096, 4, 3) == (3072, 4096)
    assert shard_k_range(256, 1, 0) == (0, 256)
    for bad in [(4096, 3, 0), (4096, 32, 0), (1000, 1, 0), (4096, 2, 2)]:
        with pytest.raises(ValueError):
            shard_k_range(*bad)


def test_max_over_ranks_without_group():
    assert max_over_ranks([1, 2.5]) == [1.0, 2.5]


@pytest.mark.parametrize("world", [2, 4])
def test_tp_tree_gemm_ranks(tmp_path, world):
    oracle.tree_sum(np.zeros(1, np.float32))        # build the oracle library before forking ranks
    mp.start_processes(_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world,
                       join=True, start_method="spawn")
    a, w = synth.gemm_inputs(M, N, K, seed=7)
    want = _bits(torch.from_numpy(oracle.tree_combine(_leaf_values(a, w))))
    for r in range(world):
        got = np.load(tmp_path / f"c{r}.npy")
        assert np.array_equal(got, want), r
        assert np.array_equal(np.load(tmp_path / f"p{r}.npy"), want), r
