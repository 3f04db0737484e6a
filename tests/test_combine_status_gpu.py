"""Cross-shard tree combine (bit-exact against the oracle's canonical tree)
and the bounded-wait failure path of the device status word.  Source of the
tree combine: "Deterministic Inference across Tensor Parallel Sizes That
Eliminates Training-Inference Mismatch", Abstract."""
import numpy as np
import pytest
import torch

import oracle
from helpers import dev, host_bits
from invariant_bi_lora_b200 import bi, synth

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("s,count", [(1, 16), (2, 4096), (3, 1000), (4, 4100), (5, 4), (8, 1 << 20), (16, 65540), (64, 4096), (6, 0)])
def test_tree_combine(s, count):
    g = np.random.default_rng(s)
    parts = (g.standard_normal((s, count)) * g.choice([1e8, 1.0, 1e-3, 3.5], size=(s, count))).astype(np.float32)
    out = torch.empty(count, dtype=torch.float32, device="cuda")
    bi.tree_combine(dev(parts), out)
    if count:
        assert np.array_equal(host_bits(out), oracle.tree_combine(parts).view(np.uint32))


@pytest.mark.parametrize("s", [1, 2, 3, 4, 5, 8, 16, 64])
def test_tree_combine_peers(s):
    """The cross-GPU combine reads each partial through its own pointer
    (here s separate allocations of this GPU stand in for the ranks'
    buffers): bitwise the oracle's tree and the contiguous combine, for the
    whole range and for per-rank shares written into one output."""
    count = 4 * 1031
    g = np.random.default_rng(100 + s)
    parts = (g.standard_normal((s, count)) * g.choice([1e8, 1.0, 1e-3, 3.5], size=(s, count))).astype(np.float32)
    bufs = [dev(np.ascontiguousarray(parts[j])) for j in range(s)]
    ptrs = [b.data_ptr() for b in bufs]
    want = oracle.tree_combine(parts).view(np.uint32)
    out = torch.full((count,), 7.0, dtype=torch.float32, device="cuda")
    bi.tree_combine_peers(ptrs, out)
    assert np.array_equal(host_bits(out), want)
    contiguous = torch.empty(count, dtype=torch.float32, device="cuda")
    bi.tree_combine(dev(parts), contiguous)
    assert np.array_equal(host_bits(out), host_bits(contiguous))
    # reduce-scatter shape: "rank" q combines its share [q*share, (q+1)*share)
    out2 = torch.full((count,), 7.0, dtype=torch.float32, device="cuda")
    world = 4
    share = (count // world) // 4 * 4
    for q in range(world):
        begin = q * share
        n = share if q < world - 1 else count - begin
        bi.tree_combine_peers(ptrs, out2, begin, n)
    assert np.array_equal(host_bits(out2), want)


def test_bounded_wait_reports_timeout():
    assert bi.get_device_status() == 0
    bi.selftest_bounded_wait(200)
    assert bi.get_device_status() == 5          # BI_ERR_TIMEOUT, context still usable
    assert bi.get_device_status() == 0          # read-and-clear
    x = torch.ones(4, 64, device="cuda")
    out = torch.empty(4, device="cuda")
    bi.mean(x, out)
    assert torch.all(out == 1.0)
