"""Batch-invariant RMSNorm, log_softmax and mean on the GPU: bit-exact
against the oracle's canonical fp32 order (test b), within tolerance of the
fp64 exact value, and row i identical at every row count (test c).
Sources: "Restoring AI Reproducibility" 2-3 / 3-1 (RMSNorm, one core per
row, consistent order); "Batch Invariant Ops", Highlighted Details
(log_softmax, mean)."""
import math

import numpy as np
import pytest
import torch

import oracle
from helpers import bf16_ulp, dev, dev_bf16, host_bits
from invariant_bi_lora_b200 import bi, synth

pytestmark = pytest.mark.gpu

ROWS = (1, 7, 64, 513, 4096)


def rms(x_bits, w_bits, eps=1e-6):
    x = dev_bf16(x_bits)
    y = torch.empty_like(x)
    bi.rmsnorm(x, dev_bf16(w_bits), y, eps)
    return host_bits(y)


@pytest.fixture(scope="module")
def norm_inputs():
    return synth.rmsnorm_inputs(4096, 4096, seed=0)


def test_rmsnorm_bit_exact_and_invariant(norm_inputs):
    x, w = norm_inputs
    full = rms(x, w)
    sample = np.random.default_rng(0).choice(4096, 96, replace=False)
    want = oracle.rmsnorm_canon(x[sample], w)
    assert np.array_equal(full[sample], want)
    ex = oracle.rmsnorm_exact(x[sample], w)
    got = oracle.bf16_to_f32(full[sample]).astype(np.float64)
    assert np.all(np.abs(got - ex) <= bf16_ulp(ex))
    for R in ROWS[:-1]:
        assert np.array_equal(rms(x[:R], w), full[:R]), R
        assert np.array_equal(rms(x[4096 - R:], w), full[4096 - R:]), R


@pytest.mark.parametrize("n", [8, 104, 4096, 5120, 8192, 14336, 32768])
def test_rmsnorm_shapes(n):
    x, w = synth.rmsnorm_inputs(9, n, seed=n)
    assert np.array_equal(rms(x, w), oracle.rmsnorm_canon(x, w))


def test_rmsnorm_closed_form():
    w = synth.normal_bf16((4096,), 0.1, mean=1.0, seed=7, tag=5)
    ones = np.full((3, 4096), 0x3F80, np.uint16)
    assert np.array_equal(rms(ones, w, eps=0.0), np.tile(w, (3, 1)))


def test_rmsnorm_product_order_rows():
    """The rows of the oracle's product-order pin (x = k/16, |k| <= 63, so
    the sum of squares is exact in any order): some outputs change if the
    two final products are taken in another order, and the kernel must
    give the oracle's bits on all of them."""
    g = np.random.default_rng(2)
    k = g.integers(-63, 64, size=(512, 4096))
    x = torch.from_numpy((k / 16.0).astype(np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    w = torch.from_numpy((g.standard_normal(4096) * 0.1 + 1.0).astype(np.float32)).to(torch.bfloat16)
    wb = w.view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(rms(x, wb), oracle.rmsnorm_canon(x, wb))


@pytest.fixture(scope="module")
def logits():
    return synth.logits_inputs(4096, 151936, seed=0)


def lsm(x):
    X = dev(x)
    out = torch.empty_like(X)
    bi.log_softmax(X, out)
    return host_bits(out)


def test_log_softmax_bit_exact_and_invariant(logits):
    full = lsm(logits)
    sample = np.random.default_rng(1).choice(4096, 24, replace=False)
    want = oracle.log_softmax_canon(logits[sample])
    assert np.array_equal(full[sample], want.view(np.uint32))
    ex = oracle.log_softmax_exact(logits[sample])
    got = full[sample].view(np.float32).astype(np.float64)
    assert np.all(np.abs(got - ex) <= 1e-5 * np.maximum(1.0, np.abs(ex)))
    for R in ROWS[:-1]:
        assert np.array_equal(lsm(logits[:R]), full[:R]), R
        assert np.array_equal(lsm(logits[4096 - R:]), full[4096 - R:]), R


@pytest.mark.parametrize("n", [4, 1000, 4096, 4100, 32000, 128000, 262144])
def test_log_softmax_shapes(n):
    x = synth.logits_inputs(5, n, seed=n)
    assert np.array_equal(lsm(x), oracle.log_softmax_canon(x).view(np.uint32))


@pytest.mark.parametrize("R", [7, 160])
def test_log_softmax_wide_range_rows(R):
    """Logits spread over hundreds: many vectors take the general exp path
    (x - max < -87, down to the flush to zero below -103), in a few rows
    and in enough rows for several waves of clusters."""
    x = synth.normal_f32((R, 151936), 60.0, seed=77)
    x[3, ::5] = -1e4
    x[R - 1, 7::3] = -1e4
    assert np.array_equal(lsm(x), oracle.log_softmax_canon(x).view(np.uint32))


def test_log_softmax_shift_invariance():
    """Integer logits and the same logits + 2^20 give the same bits: every
    x - max is exact in both, and the output is (x - max) - L."""
    g = np.random.default_rng(11)
    x = g.integers(-40, 1, size=(5, 151936)).astype(np.float32)
    assert np.array_equal(lsm(x), lsm(x + np.float32(2.0 ** 20)))


def test_exp_shortcut_matches_exp():
    """The log_softmax exp shortcut gives bi_exp's bits on [-87, 88]."""
    xs = np.concatenate([np.linspace(-87, 88, 1 << 20), -np.abs(np.random.default_rng(4).standard_normal(1 << 18) * 30)])
    xs = xs[(xs >= -87) & (xs <= 88)].astype(np.float32)
    a = torch.empty(xs.size, dtype=torch.float32, device="cuda")
    b = torch.empty_like(a)
    bi.math_spec(dev(xs), a, "exp")
    bi.math_spec(dev(xs), b, "exp_fast")
    assert np.array_equal(host_bits(a), host_bits(b))
    c = torch.empty_like(a)
    bi.math_spec(dev(xs), c, "exp_fast2")              # packed pairs, both lanes
    assert np.array_equal(host_bits(a), host_bits(c))
    bi.math_spec(dev(xs[1:]), c[:-1], "exp_fast2")     # the other pairing
    assert np.array_equal(host_bits(a)[1:], host_bits(c[:-1]))


def test_log_softmax_closed_form():
    x = np.full((2, 151936), 1.5, np.float32)
    out = lsm(x).view(np.float32)
    assert np.all(out == out[0, 0])
    assert abs(float(out[0, 0]) + math.log(151936)) <= float(np.spacing(np.float32(11.93)))


def mean_gpu(x):
    X = dev(x)
    out = torch.empty(x.shape[0], dtype=torch.float32, device="cuda")
    bi.mean(X, out)
    return host_bits(out)


@pytest.mark.parametrize("n", [4096, 151936, 4, 1028, 100000])
def test_mean_bit_exact_and_invariant(n, logits):
    x = logits[:, :n] if n == 151936 else synth.normal_f32((513, n), 1.0, seed=n)
    x = np.ascontiguousarray(x)
    full = mean_gpu(x)
    sample = np.random.default_rng(2).choice(x.shape[0], min(64, x.shape[0]), replace=False)
    assert np.array_equal(full[sample], oracle.mean_canon(x[sample]).view(np.uint32))
    ex = oracle.mean_exact(x[sample])
    assert np.all(np.abs(full[sample].view(np.float32) - ex) <= 1e-6 * np.abs(x[sample]).mean(axis=1) * 4)
    for R in (1, 7, 64):
        assert np.array_equal(mean_gpu(x[:R]), full[:R])


@pytest.mark.parametrize("n", [4, 100, 4096, 4100, 33000])
def test_mean_few_rows_cluster_path(n):
    """Up to 128 rows the mean runs one 16-CTA cluster per row (each CTA a
    block of 64 lanes, a subtree): bitwise the oracle's canonical mean at
    widths where some lanes hold no vector, one vector or many, and bitwise
    the many-row kernel's rows."""
    x = np.ascontiguousarray(synth.normal_f32((200, n), 1.0, seed=n + 1))
    many = mean_gpu(x)                                  # 200 rows: one CTA per row
    for R in (1, 3, 128):
        few = mean_gpu(x[:R])
        assert np.array_equal(few, oracle.mean_canon(x[:R]).view(np.uint32)), R
        assert np.array_equal(few, many[:R]), R


def test_mean_order_case():
    x = np.zeros((1, 8192), np.float32)
    x[0, 0], x[0, 4096], x[0, 4] = 1e8, 1.0, -1e8
    assert mean_gpu(x)[0] == 0


def test_math_spec_matches_oracle():
    g = np.random.default_rng(3)
    xe = np.concatenate([-np.abs(g.standard_normal(1 << 20) * 20), g.uniform(-104, 88, 1 << 20),
                         np.array([0.0, -103.0, -103.5, -87.5, -88.0, -100.0])]).astype(np.float32)
    ye = torch.empty(xe.size, dtype=torch.float32, device="cuda")
    bi.math_spec(dev(xe), ye, "exp")
    want = np.array([oracle.exp_spec(v) for v in xe[:20000]], np.float32)
    want = np.concatenate([want, np.array([oracle.exp_spec(v) for v in xe[-6:]], np.float32)])
    got = ye.cpu().numpy()
    got = np.concatenate([got[:20000], got[-6:]])
    assert np.array_equal(got.view(np.uint32), want.view(np.uint32))
    xl = np.concatenate([g.uniform(1.0, 151936.0, 20000), np.geomspace(1e-30, 1e30, 5000)]).astype(np.float32)
    yl = torch.empty(xl.size, dtype=torch.float32, device="cuda")
    bi.math_spec(dev(xl), yl, "log")
    want = np.array([oracle.log_spec(v) for v in xl], np.float32)
    assert np.array_equal(yl.cpu().numpy().view(np.uint32), want.view(np.uint32))
