"""Batch-invariant tcgen05 GEMM against the oracle: tolerance (a) against
the fp64 exact product, exactness on integer-valued operands, and batch
invariance (c): rows of the M=1 result are bitwise the same rows computed at
every larger M, at any position inside the 128-row tile.  Sources: "The
biggest Mystery of LLMs have just been solved" (Batch-Variant vs.
Batch-Invariant: locked kernel policy); "Batch Invariant Ops" (torch.mm)."""
import numpy as np
import pytest
import torch

import oracle
from helpers import assert_tol, bf16_ulp, dev_bf16, host_bits
from invariant_bi_lora_b200 import bi, synth

pytestmark = pytest.mark.gpu


def run_gemm(a, w, bf16_out=False):
    M, N = a.shape[0], w.shape[0]
    C = torch.empty(M, N, dtype=torch.bfloat16 if bf16_out else torch.float32, device="cuda")
    bi.gemm(a, w, C)
    torch.cuda.synchronize()
    return C


@pytest.mark.parametrize("M,N,K", [(1, 4096, 4096), (16, 4096, 4096), (64, 512, 4096), (130, 272, 64),
                                   (256, 4096, 192), (1024, 4096, 4096), (129, 16, 128), (300, 1040, 1024),
                                   (2200, 512, 1024), (4096, 256, 256)])
def test_gemm_tolerance(M, N, K):
    a, w = synth.gemm_inputs(M, N, K, seed=M + N + K)
    C = run_gemm(dev_bf16(a), dev_bf16(w)).cpu().numpy()
    rows = np.unique(np.concatenate([np.arange(min(M, 40)), np.arange(max(0, M - 40), M)]))
    exact, bound = oracle.gemm_exact(a, w, rows=rows)
    assert_tol(C[rows], exact, bound, what=f"{M}x{N}x{K}")


def test_gemm_integer_exact():
    a = synth.integer_bf16((200, 1024), -3, 3, seed=1, tag=1)
    w = synth.integer_bf16((512, 1024), -3, 3, seed=1, tag=2)
    C = run_gemm(dev_bf16(a), dev_bf16(w)).cpu().numpy()
    exact, _ = oracle.gemm_exact(a, w)
    assert np.array_equal(C.astype(np.float64), exact)


def test_gemm_bf16_output():
    a, w = synth.gemm_inputs(256, 1024, 4096, seed=3)
    A, W = dev_bf16(a), dev_bf16(w)
    C32 = run_gemm(A, W)
    C16 = run_gemm(A, W, bf16_out=True)
    # the bf16 output is the round-to-nearest-even of the fp32 accumulator
    assert np.array_equal(host_bits(C16), host_bits(C32.to(torch.bfloat16)))
    # within one bf16 ulp of the bf16 rounding of the exact value; where
    # cancellation leaves a result smaller than the fp32 accumulation error,
    # the tolerance (a) term is added to that ulp
    exact, bound = oracle.gemm_exact(a, w, rows=np.arange(64))
    exact_bf16 = oracle.bf16_to_f32(oracle.f32_to_bf16(exact.astype(np.float32))).astype(np.float64)
    got = oracle.bf16_to_f32(host_bits(C16)[:64]).astype(np.float64)
    err = np.abs(got - exact_bf16)
    ulp = bf16_ulp(exact_bf16)
    assert np.all(err <= ulp + 1e-3 * bound)
    assert np.mean(err <= ulp) > 0.999


@pytest.mark.parametrize("N", [4096, 14336])
def test_gemm_batch_invariance(N):
    """Rows of the M=1 result == the same rows at M = 16 ... 4096 (K=4096),
    wherever they sit in a tile; the M values cross the tile-width changes
    (128 x 32 up to M = 128, 128 x 64 up to 512, 128 x 256 above) and end
    with ragged last tiles."""
    K = 4096
    big_a, w = synth.gemm_inputs(4096, N, K, seed=7)
    W = dev_bf16(w)
    probe = big_a[:8]
    ref = np.stack([host_bits(run_gemm(dev_bf16(probe[i:i + 1]), W))[0] for i in range(8)])
    for M in (16, 64, 128, 129, 256, 512, 513, 1024, 2047, 2048, 2200, 4096):
        a = big_a[:M].copy()
        positions = sorted({0, M - 1, min(127, M - 1), min(128, M - 1), min(255, M - 1), min(256, M - 1), M // 2,
                            max(0, M - 8), max(0, M - 130)})
        for j, pos in enumerate(positions):
            a[pos] = probe[j % 8]
        C = host_bits(run_gemm(dev_bf16(a), W))
        for j, pos in enumerate(positions):
            assert np.array_equal(C[pos], ref[j % 8]), (M, pos)


def test_gemm_full_size_sampled():
    """M=4096, N=14336, K=4096 (the largest GEMM shape), sampled rows."""
    a, w = synth.gemm_inputs(4096, 14336, 4096, seed=11)
    C = run_gemm(dev_bf16(a), dev_bf16(w))
    rows = np.random.default_rng(0).choice(4096, 24, replace=False)
    rows = np.union1d(rows, [0, 127, 128, 4095])
    exact, bound = oracle.gemm_exact(a, w, rows=rows)
    assert_tol(C.cpu().numpy()[rows], exact, bound, what="4096x14336x4096")
    assert bi.get_device_status() == 0


def test_gemm_rejects():
    a = dev_bf16(synth.normal_bf16((4, 100), 1.0, seed=1))
    w = dev_bf16(synth.normal_bf16((16, 100), 1.0, seed=1))
    with pytest.raises(bi.BiError):
        run_gemm(a, w)                                   # K not a multiple of 64
    C = torch.empty(0, 16, dtype=torch.float32, device="cuda")
    bi.gemm(torch.empty(0, 64, dtype=torch.bfloat16, device="cuda"),
            dev_bf16(synth.normal_bf16((16, 64), 1.0, seed=1)), C)


@pytest.mark.parametrize("M,N,K", [(1, 4096, 4096), (64, 512, 1024), (300, 1040, 1024), (1024, 4096, 4096),
                                   (2200, 1024, 512)])
def test_addmm(M, N, K):
    """torch.addmm ("Batch Invariant Ops", Highlighted Details): within
    tolerance of the oracle's exact bias + A.W^T, and bitwise the GEMM's fp32
    result plus the bias in one IEEE addition (bf16 output: its RNE)."""
    a, w = synth.gemm_inputs(M, N, K, seed=M + 5)
    bias = synth.normal_bf16((N,), 1.0, seed=M, tag=9)
    A, W, Bv = dev_bf16(a), dev_bf16(w), dev_bf16(bias)
    C = torch.empty(M, N, dtype=torch.float32, device="cuda")
    bi.addmm(Bv, A, W, C)
    G = run_gemm(A, W)
    assert torch.equal(C.view(torch.int32), (G + Bv.float()[None, :]).view(torch.int32))
    C16 = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    bi.addmm(Bv, A, W, C16)
    assert torch.equal(C16.view(torch.int16), C.to(torch.bfloat16).view(torch.int16))
    rows = np.unique(np.concatenate([np.arange(min(M, 24)), np.arange(max(0, M - 24), M)]))
    exact, bound = oracle.addmm_exact(bias, a, w, rows=rows)
    assert_tol(C.cpu().numpy()[rows], exact, bound, what=f"addmm {M}x{N}x{K}")
    # batch invariance carries over: row 0 alone gives the same bits
    C1 = torch.empty(1, N, dtype=torch.float32, device="cuda")
    bi.addmm(Bv, A[:1], W, C1)
    assert torch.equal(C1.view(torch.int32), C[:1].view(torch.int32))
