"""LoRA expand on the GPU against the oracle: out (+)= bf16(y) . B^T.
K = r is a single tensor-core chain per output, so parity is the tolerance
test (a) against the fp64 exact product of the bf16-rounded y, plus
batch invariance (c).  Source: "Reproducible LoRA Inference Through
Deterministic Split-K Reduction" (Q&A: the two low-rank products)."""
import numpy as np
import pytest
import torch

import oracle
from helpers import assert_tol, dev, dev_bf16, host_bits
from invariant_bi_lora_b200 import bi, synth

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("r,N,M", [(16, 4096, 64), (8, 512, 37), (64, 1024, 130), (24, 136, 17),
                                   (128, 256, 16)])
def test_expand_single(r, N, M):
    y = synth.normal_f32((M, r), 1.0, seed=r, tag=1)
    bt = synth.normal_bf16((N, r), 1.0 / np.sqrt(r), seed=r, tag=3)
    out = torch.empty(M, N, dtype=torch.float32, device="cuda")
    bi.lora_expand(dev(y), dev_bf16(bt), out)
    exact, bound = oracle.expand_exact(y, bt)
    assert_tol(out.cpu().numpy(), exact, bound, what=f"r={r}")
    # accumulate onto a previous output
    prev = synth.normal_f32((M, N), 1.0, seed=r, tag=4)
    o2 = dev(prev.copy())
    bi.lora_expand(dev(y), dev_bf16(bt), o2, accumulate=True)
    exact2, bound2 = oracle.expand_exact(y, bt, prev=prev)
    assert_tol(o2.cpu().numpy(), exact2, bound2, what="accumulate")
    # accumulate = fl(prev + e) with e the written value, bit for bit
    e = out.cpu().numpy()
    assert np.array_equal(o2.cpu().numpy().view(np.uint32), (prev + e).astype(np.float32).view(np.uint32))


def test_expand_batch_invariance():
    r, N = 16, 4096
    y = synth.normal_f32((4096, r), 1.0, seed=2, tag=1)
    bt = dev_bf16(synth.normal_bf16((N, r), 0.25, seed=2, tag=3))
    full = torch.empty(4096, N, dtype=torch.float32, device="cuda")
    bi.lora_expand(dev(y), bt, full)
    fb = host_bits(full)
    for M, pos in ((1, 0), (7, 3), (64, 60), (513, 200)):
        part = torch.empty(M, N, dtype=torch.float32, device="cuda")
        bi.lora_expand(dev(y[pos:pos + M]), bt, part)
        assert np.array_equal(host_bits(part), fb[pos:pos + M]), (M, pos)


@pytest.mark.parametrize("r", [8, 16, 64])
def test_expand_segmented(r):
    d = synth.lora_inputs(4096, 256, r, n_adapters=8, N=4096, seed=0)
    ids = d["ids"].copy()
    ids[::53] = -1
    y = synth.normal_f32((4096, r), 1.0, seed=r, tag=9)
    plan = bi.lora_plan(dev(ids), 8)
    B = dev_bf16(d["bt"])
    out = torch.empty(4096, 4096, dtype=torch.float32, device="cuda")
    bi.lora_expand_segmented(dev(y), B, plan, out)
    rows = np.random.default_rng(r).choice(4096, 128, replace=False)
    rows = np.union1d(rows, np.arange(0, 4096, 53)[:8])
    exact, bound = oracle.expand_exact(y[rows], d["bt"], ids[rows])
    oh = out.cpu().numpy()
    assert_tol(oh[rows], exact, bound, what="segmented")
    assert np.all(oh[::53] == 0.0)
    # same bits as the single-adapter kernel on each adapter's rows
    for a in range(8):
        sel = np.nonzero(ids == a)[0][:20]
        o1 = torch.empty(len(sel), 4096, dtype=torch.float32, device="cuda")
        bi.lora_expand(dev(y[sel]), dev_bf16(d["bt"][a]), o1)
        assert np.array_equal(host_bits(o1), oh[sel].view(np.uint32)), a
    # accumulate leaves rows without an adapter untouched
    prev = synth.normal_f32((4096, 4096), 1.0, seed=5, tag=5)
    o2 = dev(prev.copy())
    bi.lora_expand_segmented(dev(y), B, plan, o2, accumulate=True)
    o2h = o2.cpu().numpy()
    assert np.array_equal(o2h[::53], prev[::53])
    exact2, bound2 = oracle.expand_exact(y[rows], d["bt"], ids[rows], prev=prev[rows])
    assert_tol(o2h[rows], exact2, bound2, what="segmented accumulate")
