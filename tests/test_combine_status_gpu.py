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


def test_bounded_wait_reports_timeout():
    assert bi.get_device_status() == 0
    bi.selftest_bounded_wait(200)
    assert bi.get_device_status() == 5          # BI_ERR_TIMEOUT, context still usable
    assert bi.get_device_status() == 0          # read-and-clear
    x = torch.ones(4, 64, device="cuda")
    out = torch.empty(4, device="cuda")
    bi.mean(x, out)
    assert torch.all(out == 1.0)
