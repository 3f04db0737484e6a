"""Every entry point can be captured in a CUDA graph and the replay gives
the same bits as the eager call (the benchmark times graph replays)."""
import numpy as np
import pytest
import torch

from helpers import dev, dev_bf16, host_bits
from invariant_bi_lora_b200 import bi, synth

pytestmark = pytest.mark.gpu


def eager_and_graph(fn, out):
    fn()
    torch.cuda.synchronize()
    want = host_bits(out).copy()
    out.fill_(0)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        fn()
    torch.cuda.synchronize()
    out.fill_(0)
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    return want, host_bits(out)


@pytest.fixture(scope="module")
def data():
    d = synth.lora_inputs(1000, 4096, 16, n_adapters=4, N=1024, seed=3)
    return {"X": dev_bf16(d["x"]), "A": dev_bf16(d["at"]), "B": dev_bf16(d["bt"]),
            "ids": dev(d["ids"]), "A0": dev_bf16(d["at"][0])}


@pytest.mark.parametrize("mode,splits", [("tree", 8), ("atomic", 8), ("unsplit", 1)])
def test_shrink_in_graph(data, mode, splits):
    plan = bi.lora_plan(data["ids"], 4)
    y = torch.empty(1000, 16, dtype=torch.float32, device="cuda")
    want, got = eager_and_graph(lambda: bi.lora_shrink_segmented(data["X"], data["A"], plan, y, splits, mode), y)
    if mode == "atomic":
        np.testing.assert_allclose(got.view(np.float32), want.view(np.float32), rtol=1e-5, atol=1e-6)
    else:
        assert np.array_equal(got, want)
    y16 = torch.empty(1000, 16, dtype=torch.float32, device="cuda")
    want, got = eager_and_graph(lambda: bi.lora_shrink(data["X"], data["A0"], y16, splits, mode), y16)
    if mode != "atomic":
        assert np.array_equal(got, want)


def test_plan_expand_in_graph(data):
    plan = torch.empty(bi.lora_plan_bytes(1000, 4) // 4, dtype=torch.int32, device="cuda")
    want, got = eager_and_graph(lambda: bi.lora_plan(data["ids"], 4, plan), plan)
    assert np.array_equal(got, want)
    y = torch.randn(1000, 16, device="cuda")
    out = torch.empty(1000, 1024, dtype=torch.float32, device="cuda")
    want, got = eager_and_graph(lambda: bi.lora_expand_segmented(y, data["B"], plan, out), out)
    assert np.array_equal(got, want)


def test_gemms_and_rowops_in_graph():
    a, w = synth.gemm_inputs(300, 512, 1024, seed=2)
    A, W = dev_bf16(a), dev_bf16(w)
    C = torch.empty(300, 512, dtype=torch.float32, device="cuda")
    want, got = eager_and_graph(lambda: bi.gemm(A, W, C), C)
    assert np.array_equal(got, want)
    ws = torch.empty(bi.gemm_tree_ws_bytes(300, 512, 4), dtype=torch.uint8, device="cuda")
    want, got = eager_and_graph(lambda: bi.gemm_tree(A, W, C, 4, ws), C)
    assert np.array_equal(got, want)
    x, wn = synth.rmsnorm_inputs(64, 4096, seed=1)
    X, WN = dev_bf16(x), dev_bf16(wn)
    Y = torch.empty_like(X)
    want, got = eager_and_graph(lambda: bi.rmsnorm(X, WN, Y), Y)
    assert np.array_equal(got, want)
    L = dev(synth.logits_inputs(8, 151936, seed=1))
    O = torch.empty_like(L)
    want, got = eager_and_graph(lambda: bi.log_softmax(L, O), O)
    assert np.array_equal(got, want)
    m = torch.empty(8, dtype=torch.float32, device="cuda")
    want, got = eager_and_graph(lambda: bi.mean(L, m), m)
    assert np.array_equal(got, want)
