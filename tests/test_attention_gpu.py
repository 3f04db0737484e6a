"""Batch-invariant decode attention with a fixed-size KV split on the GPU.
Source: "Restoring AI Reproducibility: Thinking Machines Lab's Challenge to
Overcome Nondeterminism", 2-3 (attention is one of the three operations
whose reduction order must not depend on the batch) and 3-2 (split the KV
cache by a fixed size, not by a count chosen from the batch).

(b) bit-exact against the oracle's canonical fp32 order (256-slot chunk
    frames, perfect trees, the written exp);
(a) within tolerance of the fp64 exact attention;
(c) a sequence's rows are the same bits alone, in any batch, at any
    position and under any Lmax padding; the hand-derived frame cases."""
import math

import numpy as np
import pytest
import torch

import oracle
from helpers import dev, host_bits
from invariant_bi_lora_b200 import bi

pytestmark = pytest.mark.gpu


def bf(x):
    return torch.from_numpy(np.ascontiguousarray(x, np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def dbf(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def inputs(B, Hq, Hkv, D, Lmax, seed):
    g = np.random.default_rng(seed)
    return (bf(g.standard_normal((B, Hq, D))), bf(g.standard_normal((B, Hkv, Lmax, D))),
            bf(g.standard_normal((B, Hkv, Lmax, D))))


def run(q, k, v, lens, scale):
    B, Hq, D = q.shape
    out = torch.full((B, Hq, D), float("nan"), dtype=torch.float32, device="cuda")
    bi.attn_decode(dbf(q), dbf(k), dbf(v), dev(np.asarray(lens, np.int32)), out, scale=scale)
    torch.cuda.synchronize()
    return out.cpu().numpy()


@pytest.mark.parametrize("B,Hq,Hkv,D,lens", [
    (3, 8, 2, 128, [1, 300, 1100]),
    (4, 4, 4, 64, [256, 257, 0, 512]),
    (2, 8, 2, 256, [700, 33]),
    (2, 16, 2, 128, [4096, 1]),
    (3, 8, 2, 128, [256, 0, 17]),          # one chunk at most: kernel 1 writes the output itself
    (1, 4, 1, 64, [5]),
])
def test_attention_bit_exact(B, Hq, Hkv, D, lens):
    Lmax = max(lens) if max(lens) > 0 else 1
    q, k, v = inputs(B, Hq, Hkv, D, Lmax, seed=B * D + Hq)
    scale = 1.0 / math.sqrt(D)
    got = run(q, k, v, lens, scale)
    want = oracle.attn_decode_canon(q, k, v, np.array(lens, np.int32), scale)
    assert np.array_equal(got.view(np.uint32), want.view(np.uint32))
    ex = oracle.attn_decode_exact(q, k, v, np.array(lens, np.int32), scale)
    assert np.max(np.abs(got - ex)) <= 1e-5 * max(1.0, np.max(np.abs(ex)))


def test_attention_batch_and_layout_invariance():
    """One sequence (L = 999) alone, then in batches of 7 at every position,
    then with a larger Lmax (more padding after its keys)."""
    Hq, Hkv, D, L = 8, 2, 128, 999
    q1, k1, v1 = inputs(1, Hq, Hkv, D, L, seed=5)
    ref = run(q1, k1, v1, [L], 0.088)
    qb, kb, vb = inputs(7, Hq, Hkv, D, 1600, seed=6)
    for pos in range(7):
        q, k, v = qb.copy(), kb.copy(), vb.copy()
        q[pos] = q1[0]
        k[pos, :, :L] = k1[0]
        v[pos, :, :L] = v1[0]
        lens = [1600, 3, 999, 257, 0, 1500, 64]
        lens[pos] = L
        got = run(q, k, v, lens, 0.088)
        assert np.array_equal(got[pos].view(np.uint32), ref[0].view(np.uint32)), pos


def test_attention_frame_cases():
    """The oracle's hand-derived frame pins, on the kernel: p = 1 everywhere
    (zero keys) and value column [2^24, 0, 1, 1, 0] inside one chunk, or the
    same chunk sums over five chunks: out = fl((2^24 + 2) / L)."""
    D = 64
    for L, col in ((5, [2.0 ** 24, 0.0, 1.0, 1.0, 0.0]),
                   (1280, np.repeat([2.0 ** 16, 0.0, 2.0 ** -8, 2.0 ** -8, 0.0], 256))):
        vf = np.zeros((1, 1, L, D), np.float32)
        vf[0, 0, :, 0] = col
        out = run(np.zeros((1, 1, D), np.uint16), np.zeros((1, 1, L, D), np.uint16), bf(vf), [L], 1.0)
        want = np.float32(np.float32(2.0 ** 24 + 2) / np.float32(L))
        assert out[0, 0, 0].view(np.uint32) == want.view(np.uint32), L


def test_attention_rejects():
    q = torch.zeros(1, 3, 128, dtype=torch.bfloat16, device="cuda")
    k = torch.zeros(1, 2, 16, 128, dtype=torch.bfloat16, device="cuda")
    out = torch.empty(1, 3, 128, dtype=torch.float32, device="cuda")
    with pytest.raises(bi.BiError):                  # 3 query heads over 2 kv heads
        bi.attn_decode(q, k, k, dev(np.array([16], np.int32)), out)
    q = torch.zeros(1, 2, 96, dtype=torch.bfloat16, device="cuda")
    k = torch.zeros(1, 2, 16, 96, dtype=torch.bfloat16, device="cuda")
    out = torch.empty(1, 2, 96, dtype=torch.float32, device="cuda")
    with pytest.raises(bi.BiError):                  # D not in {64, 128, 256}
        bi.attn_decode(q, k, k, dev(np.array([16], np.int32)), out)
    assert bi.get_device_status() == 0
