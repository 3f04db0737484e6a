"""Failure reporting of the real GEMM pipeline, without a GPU fault.

The host-set fault BI_FAULT_SKIP_STAGE makes the TMA producer of the GEMM's
first CTA leave one stage unloaded, so the MMA issuer's bounded wait on that
stage runs out.  The kernel must record BI_ERR_TIMEOUT, wait (bounded) for
every load and MMA it did issue, free its tensor memory and return; the same
context must then compute a clean GEMM correctly."""
import numpy as np
import pytest
import torch

import oracle
from helpers import assert_tol, dev_bf16
from invariant_bi_lora_b200 import bi, synth

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("M", [64, 256, 1024])          # the three tile widths
def test_gemm_timeout_is_reported_and_the_context_survives(M):
    N, K = 512, 1024
    a, w = synth.gemm_inputs(M, N, K, seed=M)
    A, W = dev_bf16(a), dev_bf16(w)
    C = torch.empty(M, N, dtype=torch.float32, device="cuda")
    assert bi.get_device_status() == 0
    bi.debug_set_fault(bi.FAULT_SKIP_STAGE)
    try:
        bi.gemm(A, W, C)
        st = bi.get_device_status()
    finally:
        bi.debug_set_fault(bi.FAULT_NONE)
    assert st == 5, bi.status_string(st)                 # BI_ERR_TIMEOUT
    C2 = torch.empty_like(C)
    bi.gemm(A, W, C2)
    torch.cuda.synchronize()
    assert bi.get_device_status() == 0
    rows = np.arange(0, M, 7)
    exact, bound = oracle.gemm_exact(a, w, rows=rows)
    assert_tol(C2.cpu().numpy()[rows], exact, bound, what="clean gemm after the timeout")
