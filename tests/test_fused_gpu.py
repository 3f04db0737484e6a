"""Fused segmented LoRA (shrink then expand in one launch, y kept on chip)
against the two separate calls and the oracle.  Source: "Reproducible LoRA
Inference Through Deterministic Split-K Reduction", Q&A (LoRA is two
low-rank products: the shrink reduces over the hidden size, the expand over
the rank).

(b) bitwise: out and y equal bi_lora_shrink_segmented (tree, same splits)
    followed by bi_lora_expand_segmented;
(a) tolerance: y against the oracle's exact shrink, out against the
    oracle's exact expand of that y;
(c) the split count does not change the bits; no-adapter tokens follow the
    expand's rule (zero when writing, untouched when accumulating)."""
import numpy as np
import pytest
import torch

import oracle
from helpers import assert_tol, dev, dev_bf16, host_bits
from invariant_bi_lora_b200 import bi, synth

pytestmark = pytest.mark.gpu


def two_calls(X, A, B, plan, M, r, N, splits, prev=None):
    y = torch.empty(M, r, dtype=torch.float32, device="cuda")
    bi.lora_shrink_segmented(X, A, plan, y, splits, "tree" if splits > 1 else "unsplit")
    out = torch.zeros(M, N, dtype=torch.float32, device="cuda") if prev is None else prev.clone()
    bi.lora_expand_segmented(y, B, plan, out, accumulate=prev is not None)
    torch.cuda.synchronize()
    return y, out


@pytest.mark.parametrize("M,K,r,N,n_ad", [(4096, 4096, 16, 4096, 8), (300, 1024, 8, 1040, 3),
                                          (513, 2048, 64, 512, 5), (16, 4096, 16, 4096, 1)])
def test_fused_matches_two_calls(M, K, r, N, n_ad):
    d = synth.lora_inputs(M, K, r, n_adapters=n_ad, N=N, seed=M + r)
    ids = d["ids"].copy()
    ids[::41] = -1                                   # tokens without an adapter
    X, A, B = dev_bf16(d["x"]), dev_bf16(d["at"]), dev_bf16(d["bt"])
    plan = bi.lora_plan(dev(ids), n_ad)
    ref_y, ref_out = two_calls(X, A, B, plan, M, r, N, 8)
    for splits in (8, 4, 1):
        y = torch.full((M, r), float("nan"), dtype=torch.float32, device="cuda")
        out = torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
        bi.lora_fused(X, A, B, plan, out, y=y, splits=splits)
        torch.cuda.synchronize()
        assert np.array_equal(host_bits(y), host_bits(ref_y)), splits
        assert np.array_equal(host_bits(out), host_bits(ref_out)), splits
    assert np.all(host_bits(out)[::41] == 0)
    # tolerance against the oracle on sampled tokens
    rows = np.random.default_rng(1).choice(M, min(M, 96), replace=False)
    yh = y.cpu().numpy()
    ex_y, b_y = oracle.shrink_exact(d["x"][rows], d["at"], ids[rows])
    assert_tol(yh[rows], ex_y, b_y, what="fused y")
    ex_o, b_o = oracle.expand_exact(yh[rows], d["bt"], ids[rows])
    assert_tol(out.cpu().numpy()[rows], ex_o, b_o, what="fused out")


def test_fused_accumulate_and_no_y():
    M, K, r, N, n_ad = 1000, 1024, 16, 768, 4
    d = synth.lora_inputs(M, K, r, n_adapters=n_ad, N=N, seed=3)
    ids = d["ids"].copy()
    ids[::13] = 7                                    # out of range: no adapter
    X, A, B = dev_bf16(d["x"]), dev_bf16(d["at"]), dev_bf16(d["bt"])
    plan = bi.lora_plan(dev(ids), n_ad)
    prev = torch.from_numpy(np.random.default_rng(2).standard_normal((M, N)).astype(np.float32)).cuda()
    _, ref_out = two_calls(X, A, B, plan, M, r, N, 8, prev=prev)
    out = prev.clone()
    bi.lora_fused(X, A, B, plan, out, y=None, splits=8, accumulate=True)
    torch.cuda.synchronize()
    assert np.array_equal(host_bits(out), host_bits(ref_out))
    assert np.array_equal(host_bits(out)[::13], host_bits(prev)[::13])   # untouched
    assert bi.get_device_status() == 0


def test_fused_rejects_atomic_shapes():
    M, K, r, N = 32, 1024, 16, 100                   # N not a multiple of 8
    d = synth.lora_inputs(M, K, r, n_adapters=2, N=104, seed=4)
    X, A = dev_bf16(d["x"]), dev_bf16(d["at"])
    B = torch.zeros(2, N, r, dtype=torch.bfloat16, device="cuda")
    plan = bi.lora_plan(dev(d["ids"]), 2)
    out = torch.empty(M, N, dtype=torch.float32, device="cuda")
    with pytest.raises(bi.BiError):
        bi.lora_fused(X, A, B, plan, out, splits=8)
