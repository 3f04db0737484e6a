"""The tensor-parallel contract of the tree GEMM on one GPU: a rank that
holds only its K slice and runs the tree GEMM on it (shards=1) produces
exactly the partial of shard q of the single-GPU kernel, so gathering the
ranks' partials in order and adding them with bi_tree_combine reproduces
bi_gemm_tree(shards=world) bit for bit.  The ranks are emulated in one
process (the gather is a stack); the collective itself is covered by the CPU
process-group test.  Source: "Deterministic Inference across Tensor Parallel
Sizes That Eliminates Training-Inference Mismatch", Abstract."""
import numpy as np
import pytest
import torch

from helpers import dev_bf16, host_bits
from invariant_bi_lora_b200 import bi, synth
from invariant_bi_lora_b200.tp import shard_k_range

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("M,N,K,world", [(200, 256, 4096, 2), (130, 128, 8192, 4), (64, 512, 16384, 8)])
def test_rank_slices_reproduce_the_emulated_shards(M, N, K, world):
    a, w = synth.gemm_inputs(M, N, K, seed=world)
    A, W = dev_bf16(a), dev_bf16(w)
    ref = torch.empty(M, N, dtype=torch.float32, device="cuda")
    bi.gemm_tree(A, W, ref, shards=world)
    parts = torch.empty(world, M, N, dtype=torch.float32, device="cuda")
    for q in range(world):
        k0, k1 = shard_k_range(K, world, q)
        bi.gemm_tree(dev_bf16(np.ascontiguousarray(a[:, k0:k1])), dev_bf16(np.ascontiguousarray(w[:, k0:k1])),
                     parts[q], shards=1)
    C = torch.empty(M, N, dtype=torch.float32, device="cuda")
    bi.tree_combine(parts, C)
    torch.cuda.synchronize()
    assert np.array_equal(host_bits(C), host_bits(ref))
    one = torch.empty(M, N, dtype=torch.float32, device="cuda")
    bi.gemm_tree(A, W, one, shards=1)
    torch.cuda.synchronize()
    assert np.array_equal(host_bits(one), host_bits(ref))
    assert bi.get_device_status() == 0
