"""Out-of-bounds writes on ragged shapes: every output buffer sits inside a
larger allocation whose margins hold a sentinel bit pattern, and the margins
must be intact after the call (the stand-in for a memory checker, which this
pool does not run).  Shapes are ragged on purpose: M not a multiple of the
row tile, rows and columns with tails, segments of uneven length."""
import numpy as np
import pytest
import torch

from helpers import dev_bf16
from invariant_bi_lora_b200 import bi, synth

pytestmark = pytest.mark.gpu

PAD = 64                      # elements of margin on each side (256 B for 4-byte types)
SENT32 = 0x7FC0DEAD
SENT16 = 0x7FAD


def padded(shape, dtype):
    n = int(np.prod(shape))
    if dtype == torch.bfloat16:
        buf = torch.full((n + 2 * PAD,), SENT16, dtype=torch.int16, device="cuda").view(torch.bfloat16)
    elif dtype == torch.int32:
        buf = torch.full((n + 2 * PAD,), SENT32, dtype=torch.int32, device="cuda")
    else:
        buf = torch.full((n + 2 * PAD,), SENT32, dtype=torch.int32, device="cuda").view(torch.float32)
    return buf, buf[PAD:PAD + n].view(shape)


def margins_intact(buf):
    torch.cuda.synchronize()
    if buf.dtype == torch.bfloat16:
        raw = buf.view(torch.int16).cpu().numpy().astype(np.int64) & 0xFFFF
        sent = SENT16
    else:
        raw = buf.view(torch.int32).cpu().numpy().astype(np.int64) & 0xFFFFFFFF
        sent = SENT32
    return bool(np.all(raw[:PAD] == sent) and np.all(raw[-PAD:] == sent))


@pytest.mark.parametrize("M,mode,splits", [(37, "tree", 8), (37, "atomic", 8), (37, "unsplit", 1), (1, "tree", 16)])
def test_shrink_margins(M, mode, splits):
    d = synth.lora_inputs(M, 4096, 16, seed=M)
    buf, y = padded((M, 16), torch.float32)
    bi.lora_shrink(dev_bf16(d["x"]), dev_bf16(d["at"][0]), y, splits, mode)
    assert margins_intact(buf)


@pytest.mark.parametrize("r", [8, 16, 64])
def test_segmented_margins(r):
    M, n_ad, N = 301, 5, 520
    d = synth.lora_inputs(M, 2048, r, n_adapters=n_ad, N=N, seed=r)
    ids = torch.from_numpy(d["ids"]).cuda()
    pbuf, plan = padded((bi.lora_plan_bytes(M, n_ad) // 4,), torch.int32)
    bi.lora_plan(ids, n_ad, plan)
    assert margins_intact(pbuf)
    for mode, splits in (("tree", 8), ("atomic", 4), ("unsplit", 1)):
        ybuf, y = padded((M, r), torch.float32)
        bi.lora_shrink_segmented(dev_bf16(d["x"]), dev_bf16(d["at"]), plan, y, splits, mode)
        assert margins_intact(ybuf), mode
    obuf, out = padded((M, N), torch.float32)
    bi.lora_expand_segmented(y, dev_bf16(d["bt"]), plan, out)
    assert margins_intact(obuf)


def test_row_op_margins():
    x, w = synth.rmsnorm_inputs(7, 4104, seed=3)
    ybuf, y = padded((7, 4104), torch.bfloat16)
    bi.rmsnorm(dev_bf16(x), dev_bf16(w), y)
    assert margins_intact(ybuf)
    lg = synth.logits_inputs(3, 151940, seed=4)
    obuf, out = padded((3, 151940), torch.float32)
    bi.log_softmax(torch.from_numpy(lg).cuda(), out)
    assert margins_intact(obuf)
    mbuf, m = padded((3,), torch.float32)
    bi.mean(torch.from_numpy(lg).cuda(), m)
    assert margins_intact(mbuf)


@pytest.mark.parametrize("M,shards", [(130, 1), (130, 4), (1, 8)])
def test_gemm_margins(M, shards):
    a, w = synth.gemm_inputs(M, 384, 4096, seed=M + shards)
    A, W = dev_bf16(a), dev_bf16(w)
    cbuf, C = padded((M, 384), torch.float32)
    bi.gemm(A, W, C)
    assert margins_intact(cbuf)
    tbuf, T = padded((M, 384), torch.float32)
    bi.gemm_tree(A, W, T, shards=shards)
    assert margins_intact(tbuf)
    assert bi.get_device_status() == 0
