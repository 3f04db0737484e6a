"""The segmented shrink entry point that allocates nothing.

Callers such as a plugin inside a host application that owns all device
memory, or a latency-critical loop that must not hit the allocator, cannot
allocate the token plan the regular path needs.  bi_lora_shrink_segmented_noalloc
builds that plan in a fixed device array of the library instead.  Here it is
called through the C ABI twice in a row and checked against the regular
entry points (bi_lora_plan + bi_lora_shrink_segmented): the same tolerance
against the exact product that the shrink parity tests use, and, since the
plan is the same, the same bits.  The file sorts last so that a run that stops
at the first failure has run every other test first; it also passes alone
in a fresh process (the first call does the per-device set-up)."""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from helpers import assert_tol, dev, dev_bf16, host_bits
from invariant_bi_lora_b200 import bi, synth

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("mode,splits", [("tree", 8), ("unsplit", 1), ("atomic", 8)])
def test_noalloc_matches_regular_path(mode, splits):
    M, K, r, n_ad = 4096, 4096, 16, 8
    d = synth.lora_inputs(M, K, r, n_adapters=n_ad, seed=0)
    ids = d["ids"].copy()
    ids[::31] = -1                               # some tokens without an adapter
    X, A, I = dev_bf16(d["x"]), dev_bf16(d["at"]), dev(ids)

    plan = bi.lora_plan(I, n_ad)
    ref = torch.empty(M, r, dtype=torch.float32, device="cuda")
    bi.lora_shrink_segmented(X, A, plan, ref, splits=splits, mode=mode)
    refh = ref.cpu().numpy()

    rows = np.random.default_rng(1).choice(M, 256, replace=False)
    exact, bound = oracle.shrink_exact(d["x"][rows], d["at"], ids[rows])
    for call in range(2):
        y = torch.full((M, r), float("nan"), dtype=torch.float32, device="cuda")
        bi.lora_shrink_segmented_noalloc(X, A, I, y, splits=splits, mode=mode)
        yh = y.cpu().numpy()
        assert_tol(yh[rows], exact, bound, what=f"noalloc {mode} call {call}")
        assert np.all(yh[::31] == 0.0)
        if mode != "atomic":
            assert np.array_equal(yh.view(np.uint32), refh.view(np.uint32)), call
        else:
            assert_tol(yh[rows], refh[rows].astype(np.float64), bound * 2, what="atomic vs regular")
    assert bi.get_device_status() == 0


def test_noalloc_smaller_batch_after_larger():
    """The shared array keeps the previous call's plan; a smaller call that
    follows must not see it."""
    K, r, n_ad = 1024, 16, 3
    big = synth.lora_inputs(3000, K, r, n_adapters=n_ad, seed=5)
    small = synth.lora_inputs(37, K, r, n_adapters=n_ad, seed=6)
    A = dev_bf16(big["at"])
    y = torch.empty(3000, r, dtype=torch.float32, device="cuda")
    bi.lora_shrink_segmented_noalloc(dev_bf16(big["x"]), A, dev(big["ids"]), y, splits=8)
    ys = torch.empty(37, r, dtype=torch.float32, device="cuda")
    bi.lora_shrink_segmented_noalloc(dev_bf16(small["x"]), A, dev(small["ids"]), ys, splits=8)
    exact, bound = oracle.shrink_exact(small["x"], big["at"], small["ids"])
    assert_tol(ys.cpu().numpy(), exact, bound, what="small after large")


def test_noalloc_rejects_oversize():
    lib = bi.lib()
    fake = ctypes.c_void_p(0x10000)                # never touched: rejected first
    st = lib.bi_lora_shrink_segmented_noalloc(fake, fake, fake, 8, fake, bi.NOALLOC_MAX_TOKENS + 1,
                                              4096, 16, 8, 2, None)
    assert st == 2                                 # BI_ERR_UNSUPPORTED_SHAPE
    st = lib.bi_lora_shrink_segmented_noalloc(fake, fake, fake, 257, fake, 16, 4096, 16, 8, 2, None)
    assert st == 2
