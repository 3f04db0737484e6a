"""TP-invariant tree GEMM against the oracle.  (b) bit-exact: the output is
the oracle's canonical fp32 tree over the kernel's own 256-wide leaves (each
leaf measured by a K=256 call on that slice), and bi_tree_combine over the
per-shard partials is the oracle's tree over them; (c) invariance: the same
bits for 1, 2, 4, 8 (and 16) emulated shards; (a) tolerance against fp64.
Source: "Deterministic Inference across Tensor Parallel Sizes That
Eliminates Training-Inference Mismatch", Abstract."""
import numpy as np
import pytest
import torch

import oracle
from helpers import assert_tol, dev_bf16, host_bits
from invariant_bi_lora_b200 import bi, synth

pytestmark = pytest.mark.gpu


def tree(A, W, shards):
    M, N = A.shape[0], W.shape[0]
    C = torch.empty(M, N, dtype=torch.float32, device="cuda")
    bi.gemm_tree(A, W, C, shards=shards)
    torch.cuda.synchronize()
    return C


@pytest.mark.parametrize("M", [1, 128, 2048])
def test_shard_invariance_cfg5(M):
    """K=16384, N=4096, shards 1/2/4/8 bitwise equal (K split into 64 leaves)."""
    a, w = synth.gemm_inputs(M, 4096, 16384, seed=M)
    A, W = dev_bf16(a), dev_bf16(w)
    ref = host_bits(tree(A, W, 1))
    for s in (2, 4, 8, 16):
        assert np.array_equal(host_bits(tree(A, W, s)), ref), s
    rows = np.unique([0, M // 2, M - 1])
    exact, bound = oracle.gemm_exact(a, w, rows=rows)
    assert_tol(ref.view(np.float32)[rows], exact, bound, what=f"M={M}")


@pytest.mark.parametrize("K,shards", [(16384, 8), (1280, 1), (1536, 2), (4096, 4)])
def test_leaves_and_combine_bit_exact(K, shards):
    M, N = 130, 128
    a, w = synth.gemm_inputs(M, N, K, seed=K)
    A, W = dev_bf16(a), dev_bf16(w)
    L = K // 256
    leaves = np.stack([tree(dev_bf16(np.ascontiguousarray(a[:, 256 * l:256 * l + 256])),
                            dev_bf16(np.ascontiguousarray(w[:, 256 * l:256 * l + 256])), 1).cpu().numpy()
                       for l in range(L)])
    want = oracle.tree_combine(leaves)
    got = tree(A, W, shards).cpu().numpy()
    assert np.array_equal(got.view(np.uint32), want.view(np.uint32))
    parts = torch.empty(shards, M, N, dtype=torch.float32, device="cuda")
    bi.gemm_tree_partials(A, W, parts, shards)
    ph = parts.cpu().numpy()
    for s in range(shards):
        sub = leaves[s * L // shards:(s + 1) * L // shards]
        assert np.array_equal(ph[s].view(np.uint32), oracle.tree_combine(sub).view(np.uint32)), s
    assert np.array_equal(oracle.tree_combine(ph).view(np.uint32), want.view(np.uint32))
    exact, bound = oracle.gemm_exact(a, w)
    assert_tol(got, exact, bound)


def test_tree_gemm_rejects():
    a = dev_bf16(synth.normal_bf16((4, 512), 1.0, seed=1))
    w = dev_bf16(synth.normal_bf16((64, 512), 1.0, seed=1))
    C = torch.empty(4, 64, dtype=torch.float32, device="cuda")
    with pytest.raises(bi.BiError):
        bi.gemm_tree(a, w, C, shards=4)                  # 2 leaves cannot make 4 shards
    with pytest.raises(bi.BiError):
        bi.gemm_tree(a, w, C, shards=3)
    assert bi.get_device_status() == 0


@pytest.mark.parametrize("M,N,seed", [(300, 512, 1), (2048, 1024, 2)])
def test_leaf_bits_independent_of_mma_width(M, N, seed):
    """One 256-wide leaf: the batch-invariant GEMM (N=256 instructions) and
    the tree GEMM (N=64 instructions) accumulate the same K order per output
    element, so their bits agree; the tree GEMM's leaves rely on it."""
    a, w = synth.gemm_inputs(M, N, 256, seed=seed)
    A, W = dev_bf16(a), dev_bf16(w)
    C1 = torch.empty(M, N, dtype=torch.float32, device="cuda")
    bi.gemm(A, W, C1)
    C2 = tree(A, W, 1)
    assert np.array_equal(host_bits(C1), host_bits(C2))
