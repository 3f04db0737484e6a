"""Pins for the CPU oracle: each function is checked against something other
than itself -- the pages' worked example (corrected), hand-derived trees and
sums under tests/golden/, closed forms, special cases that reduce to a
textbook or library routine (numpy / torch in float64), and brute force on
tiny inputs.  CPU only."""
import math

import numpy as np
import pytest
import torch

from conftest import read_golden
from invariant_bi_lora_b200 import synth

F32 = np.float32


def f32bits(x):
    return np.asarray(x, dtype=np.float32).view(np.uint32)


def ulp32(x):
    """Spacing of fp32 numbers at |x| (float64 result)."""
    x = np.abs(np.asarray(x, dtype=np.float64)).astype(np.float32)
    return np.spacing(x).astype(np.float64)


# ------------------------------------------------------------- worked example

def _eval_expr(expr, env, dtype):
    return eval(expr, {"__builtins__": {}}, {k: dtype(v) for k, v in env.items()})


def test_fp32_worked_example(oracle_mod):
    rows = read_golden("fp32_order_example.txt")
    n_tree = 0
    for row in rows:
        if row[0] == "tree4":
            leaves = np.array([float(v) for v in row[1].split()], dtype=np.float32)
            assert oracle_mod.tree_sum(leaves) == F32(row[2]), row
            # fp64 sum of the same multiset is 1 whatever the order
            assert math.fsum(leaves.astype(np.float64)) == 1.0
            n_tree += 1
            continue
        name, expr, vals, want32, want64 = row
        a, b, c = (float(v) for v in vals.split())
        env = {"a": a, "b": b, "c": c}
        got32 = _eval_expr(expr, env, np.float32)
        got64 = _eval_expr(expr, env, np.float64)
        assert isinstance(got32, np.float32)
        assert got32 == F32(want32), name
        assert got64 == float(want64), name
    assert n_tree == 2


# ------------------------------------------------------------ canonical tree

DISCRIMINATING = np.array([1e8, -1e8, 1.0, -3.5, 2.0 ** 25, -(2.0 ** 25), 0.75, 3.0, 1e-3, 7.0],
                          dtype=np.float32)


def test_tree_shapes_golden(oracle_mod):
    g = np.random.default_rng(11)
    for n_str, expr in read_golden("tree_shapes.txt"):
        n = int(n_str)
        py = expr
        for i in reversed(range(n)):       # leaf index i -> v[i]
            py = py.replace(str(i), f"v[{i}]")
        for _ in range(300):
            v = [F32(x) for x in g.choice(DISCRIMINATING, size=n)]
            want = eval(py, {"__builtins__": {}}, {"v": v})
            got = oracle_mod.tree_sum(np.array(v, np.float32))
            assert f32bits(got) == f32bits(want), (n, v)


def test_tree_is_not_sequential(oracle_mod):
    # the golden shapes must be able to tell tree from left-to-right order
    v = np.array([1e8, 1, -1e8, 1], np.float32)
    seq = F32(0)
    for x in v:
        seq = F32(seq + x)
    assert oracle_mod.tree_sum(v) != seq or v.size < 4


@pytest.mark.parametrize("n", [8, 64, 80, 96, 6])
def test_tree_split_into_subtrees(oracle_mod, n):
    """For every power-of-two s dividing n, the tree over the s block
    subtrees equals the full tree: the property that makes split counts and
    shard counts bitwise irrelevant."""
    g = np.random.default_rng(n)
    for _ in range(50):
        v = g.choice(DISCRIMINATING, size=n) * g.standard_normal(n).astype(np.float32)
        v = v.astype(np.float32)
        full = oracle_mod.tree_sum(v)
        s = 1
        while n % s == 0:
            blocks = np.array([oracle_mod.tree_sum(b) for b in v.reshape(s, n // s)], np.float32)
            assert f32bits(oracle_mod.tree_sum(blocks)) == f32bits(full), (n, s)
            s *= 2


def test_tree_combine_axis0(oracle_mod):
    g = np.random.default_rng(3)
    parts = (g.choice(DISCRIMINATING, size=(8, 37)) * g.standard_normal((8, 37))).astype(np.float32)
    out = oracle_mod.tree_combine(parts)
    for i in range(37):
        assert f32bits(out[i]) == f32bits(oracle_mod.tree_sum(parts[:, i]))
    # s = 1 is the identity
    assert np.array_equal(oracle_mod.tree_combine(parts[:1]).view(np.uint32), parts[0].view(np.uint32))


# ---------------------------------------------------------- canonical row sum

def test_canon_sum_golden(oracle_mod):
    for T, V, vals, want in read_golden("canon_sum_cases.txt"):
        v = np.array([float(x) for x in vals.split()], np.float32)
        got = oracle_mod.canon_sum(v, int(T), int(V))
        assert got == F32(want), (T, V, vals)


def test_canon_sum_special_cases(oracle_mod):
    g = np.random.default_rng(5)
    v = (g.standard_normal(256) * g.choice(DISCRIMINATING, 256)).astype(np.float32)
    seq = np.add.accumulate(v, dtype=np.float32)[-1]          # left-to-right
    # one lane, any vector width: a single sequential chain
    assert f32bits(oracle_mod.canon_sum(v, 1, 1)) == f32bits(seq)
    assert f32bits(oracle_mod.canon_sum(v, 1, 256)) == f32bits(seq)
    # one element per lane: the plain tree
    assert f32bits(oracle_mod.canon_sum(v, 256, 1)) == f32bits(oracle_mod.tree_sum(v))
    # more lanes than vectors: empty lanes are +0 and change nothing
    assert f32bits(oracle_mod.canon_sum(v, 512, 1)) == f32bits(oracle_mod.tree_sum(v))
    # all-ones rows: every partial is an integer below 2^24, so exact
    for n, T, V in [(4096, 512, 8), (151936, 1024, 4), (4096, 1024, 4), (8, 1024, 4)]:
        assert oracle_mod.canon_sum(np.ones(n, np.float32), T, V) == F32(n)


# ---------------------------------------------------------------------- bf16

def test_bf16_roundtrip_all_patterns(oracle_mod):
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    f = oracle_mod.bf16_to_f32(bits)
    finite = np.isfinite(f)
    back = oracle_mod.f32_to_bf16(f[finite])
    assert np.array_equal(back, bits[finite])


def test_bf16_rne_matches_torch(oracle_mod):
    g = np.random.default_rng(9)
    raw = g.integers(0, 2 ** 32, size=200000, dtype=np.uint64).astype(np.uint32)
    raw[:1000] = (raw[:1000] & 0xFFFF0000) | 0x8000          # exact ties
    f = raw.view(np.float32)
    f = f[np.isfinite(f)]
    want = torch.from_numpy(f.copy()).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(oracle_mod.f32_to_bf16(f), want)
    # ties go to even: 1 + 2^-8 -> 1.0 ; 1 + 3*2^-8 -> 1 + 2^-6
    assert oracle_mod.f32_to_bf16(np.array([1.0 + 2 ** -8], np.float32))[0] == 0x3F80
    assert oracle_mod.f32_to_bf16(np.array([1.0 + 3 * 2 ** -8], np.float32))[0] == 0x3F82


# ------------------------------------------------------------------ exp / log

def test_exp_spec_accuracy(oracle_mod):
    xs = np.concatenate([np.linspace(-103, 0, 40001), np.linspace(0, 88, 8001),
                         -np.abs(np.random.default_rng(1).standard_normal(20000) * 10)]).astype(np.float32)
    got = np.array([oracle_mod.exp_spec(x) for x in xs], np.float64)
    ref = np.exp(xs.astype(np.float64))
    err = np.abs(got - ref) / ulp32(ref)
    normal = ref > 2.0 ** -126
    assert err[normal].max() <= 2.0, float(err[normal].max())
    # subnormal range: within one subnormal spacing of a correct rounding
    assert np.all(np.abs(got[~normal] - ref[~normal]) <= 2.0 ** -149 * 2)
    assert oracle_mod.exp_spec(0.0) == 1.0
    assert oracle_mod.exp_spec(-103.5) == 0.0
    assert oracle_mod.exp_spec(-200.0) == 0.0


def test_log_spec_accuracy(oracle_mod):
    g = np.random.default_rng(2)
    xs = np.concatenate([np.geomspace(1.0, 2.0 ** 24, 30001), np.geomspace(2.0 ** -20, 1.0, 10001),
                         g.uniform(1.0, 151936.0, 20000), np.linspace(0.7, 1.45, 5001)]).astype(np.float32)
    got = np.array([oracle_mod.log_spec(x) for x in xs], np.float64)
    ref = np.log(xs.astype(np.float64))
    nz = ref != 0
    err = np.abs(got[nz] - ref[nz]) / ulp32(ref[nz])
    assert err.max() <= 2.0, float(err.max())
    assert oracle_mod.log_spec(1.0) == 0.0
    for k in range(-20, 25):
        want = F32(k * math.log(2.0))
        assert abs(float(oracle_mod.log_spec(2.0 ** k)) - float(want)) <= float(ulp32(want)), k


# ------------------------------------------------------------- LoRA shrink

def test_shrink_exact_vs_numpy(oracle_mod):
    M, K, r = 19, 320, 12
    x = synth.normal_bf16((M, K), 1.0, seed=1, tag=1)
    at = synth.normal_bf16((r, K), 0.05, seed=1, tag=2)
    y, b = oracle_mod.shrink_exact(x, at)
    xf = oracle_mod.bf16_to_f32(x).astype(np.float64)
    af = oracle_mod.bf16_to_f32(at).astype(np.float64)
    np.testing.assert_allclose(y, xf @ af.T, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(b, np.abs(xf) @ np.abs(af).T, rtol=1e-12, atol=0)


def test_shrink_exact_integers(oracle_mod):
    M, K, r = 7, 256, 16
    x = synth.integer_bf16((M, K), -4, 4, seed=2, tag=1)
    at = synth.integer_bf16((r, K), -4, 4, seed=2, tag=2)
    y, _ = oracle_mod.shrink_exact(x, at)
    xi = oracle_mod.bf16_to_f32(x).astype(np.int64)
    ai = oracle_mod.bf16_to_f32(at).astype(np.int64)
    assert np.array_equal(y, (xi @ ai.T).astype(np.float64))


def test_shrink_exact_segmented(oracle_mod):
    M, K, r, n_ad = 33, 128, 8, 3
    x = synth.normal_bf16((M, K), 1.0, seed=3, tag=1)
    at = synth.normal_bf16((n_ad, r, K), 0.1, seed=3, tag=2)
    ids = synth.adapter_ids(M, n_ad, seed=3)
    ids[5] = -1
    ids[6] = n_ad                      # invalid ids -> zero rows
    y, b = oracle_mod.shrink_exact(x, at, ids)
    xf = oracle_mod.bf16_to_f32(x).astype(np.float64)
    af = oracle_mod.bf16_to_f32(at).astype(np.float64)
    for m in range(M):
        if 0 <= ids[m] < n_ad:
            np.testing.assert_allclose(y[m], af[ids[m]] @ xf[m], rtol=1e-12, atol=1e-12)
        else:
            assert np.all(y[m] == 0) and np.all(b[m] == 0)


def test_expand_exact(oracle_mod):
    M, r, N, n_ad = 11, 16, 40, 2
    y = synth.normal_f32((M, r), 1.0, seed=4, tag=1)
    bt = synth.normal_bf16((n_ad, N, r), 0.25, seed=4, tag=2)
    ids = synth.adapter_ids(M, n_ad, seed=4)
    prev = synth.normal_f32((M, N), 1.0, seed=4, tag=3)
    out, b = oracle_mod.expand_exact(y, bt, ids, prev=prev)
    yb = torch.from_numpy(y).to(torch.bfloat16).to(torch.float64).numpy()   # bf16 input
    bf = oracle_mod.bf16_to_f32(bt).astype(np.float64)
    for m in range(M):
        want = prev[m].astype(np.float64) + bf[ids[m]] @ yb[m]
        np.testing.assert_allclose(out[m], want, rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(b[m], np.abs(prev[m]) + np.abs(bf[ids[m]]) @ np.abs(yb[m]), rtol=1e-12)
    out0, _ = oracle_mod.expand_exact(y, bt[0])
    np.testing.assert_allclose(out0, yb @ bf[0].T, rtol=1e-12, atol=1e-12)


def test_segment_stable_sort(oracle_mod):
    for M, n_ad in [(4096, 8), (1, 1), (100, 7), (0, 3)]:
        ids = synth.adapter_ids(M, n_ad, seed=M)
        perm, offs = oracle_mod.segment(ids, n_ad)
        want = np.argsort(ids, kind="stable")
        assert np.array_equal(perm, want)
        assert np.array_equal(offs, np.concatenate([[0], np.cumsum(np.bincount(ids, minlength=n_ad))]))
    ids = np.array([2, -1, 0, 5, 2, 0], np.int32)
    perm, offs = oracle_mod.segment(ids, 3)
    assert perm.tolist() == [2, 5, 0, 4] and offs.tolist() == [0, 2, 2, 4]


# ------------------------------------------------------------------ GEMM

def test_gemm_exact(oracle_mod):
    M, N, K = 9, 23, 200
    a, w = synth.gemm_inputs(M, N, K, seed=5)
    C, b = oracle_mod.gemm_exact(a, w)
    af = oracle_mod.bf16_to_f32(a).astype(np.float64)
    wf = oracle_mod.bf16_to_f32(w).astype(np.float64)
    np.testing.assert_allclose(C, af @ wf.T, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(b, np.abs(af) @ np.abs(wf).T, rtol=1e-12)
    rows = np.array([8, 0, 3])
    Cr, br = oracle_mod.gemm_exact(a, w, rows=rows)
    assert np.array_equal(Cr, C[rows]) and np.array_equal(br, b[rows])

def test_addmm_exact_pins(oracle_mod):
    """torch.addmm's value, exact: bias + a @ w.T.  Pinned by numpy float64,
    integer brute force, and two special cases (zero bias reduces to the
    GEMM; zero operands give the bias)."""
    M, N, K = 7, 48, 192
    a, w = synth.gemm_inputs(M, N, K, seed=11)
    bias = synth.normal_bf16((N,), 1.0, seed=11, tag=9)
    C, bound = oracle_mod.addmm_exact(bias, a, w)
    af, wf, bf = (oracle_mod.bf16_to_f32(v).astype(np.float64) for v in (a, w, bias))
    np.testing.assert_allclose(C, bf[None, :] + af @ wf.T, rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(bound, np.abs(bf)[None, :] + np.abs(af) @ np.abs(wf).T, rtol=1e-13)
    zero = np.zeros(N, np.uint16)
    C0, _ = oracle_mod.addmm_exact(zero, a, w)
    G, _ = oracle_mod.gemm_exact(a, w)
    assert np.array_equal(C0, G)
    Cz, _ = oracle_mod.addmm_exact(bias, np.zeros_like(a), w)
    assert np.array_equal(Cz, np.tile(bf, (M, 1)))
    ai = synth.integer_bf16((5, 64), -4, 4, seed=2, tag=1)
    wi = synth.integer_bf16((16, 64), -4, 4, seed=2, tag=2)
    bi_ = synth.integer_bf16((16,), -100, 100, seed=2, tag=3)
    Ci, _ = oracle_mod.addmm_exact(bi_, ai, wi)
    A_i = oracle_mod.bf16_to_f32(ai).astype(np.int64)
    W_i = oracle_mod.bf16_to_f32(wi).astype(np.int64)
    want = oracle_mod.bf16_to_f32(bi_).astype(np.int64)[None, :] + np.array(
        [[sum(int(A_i[m, k]) * int(W_i[n, k]) for k in range(64)) for n in range(16)] for m in range(5)])
    assert np.array_equal(Ci, want.astype(np.float64))
    rows = np.array([6, 0, 3])
    Cr, _ = oracle_mod.addmm_exact(bias, a, w, rows=rows)
    assert np.array_equal(Cr, C[rows])



# ---------------------------------------------------------------- RMSNorm

def test_rmsnorm_exact_vs_torch(oracle_mod):
    x, w = synth.rmsnorm_inputs(5, 512, seed=6)
    y = oracle_mod.rmsnorm_exact(x, w, 1e-6)
    xt = torch.from_numpy(oracle_mod.bf16_to_f32(x).astype(np.float64))
    wt = torch.from_numpy(oracle_mod.bf16_to_f32(w).astype(np.float64))
    want = torch.nn.functional.rms_norm(xt, (512,), wt, eps=1e-6).numpy()
    np.testing.assert_allclose(y, want, rtol=1e-12, atol=1e-12)


def test_rmsnorm_canon_closed_forms(oracle_mod):
    n = 4096
    w = synth.normal_bf16((n,), 0.1, mean=1.0, seed=7, tag=5)
    ones = np.full((1, n), 0x3F80, np.uint16)                   # x = 1.0
    # eps = 0: S = n exactly, ms = 1, inv = 1, so y = w bit for bit
    assert np.array_equal(oracle_mod.rmsnorm_canon(ones, w, eps=0.0)[0], w)
    # x = 2: S = 4n, ms = 4, inv = 1/2 exactly, y = w bit for bit again
    twos = np.full((1, n), 0x4000, np.uint16)
    assert np.array_equal(oracle_mod.rmsnorm_canon(twos, w, eps=0.0)[0], w)
    # x = 1, eps = 1e-6: every output is bf16(w * 1/sqrt(1+1e-6)) within rounding
    y = oracle_mod.bf16_to_f32(oracle_mod.rmsnorm_canon(ones, w, eps=1e-6)[0]).astype(np.float64)
    want = oracle_mod.bf16_to_f32(w).astype(np.float64) / math.sqrt(1.0 + 1e-6)
    assert np.all(np.abs(y - want) <= np.spacing(want.astype(np.float32)).astype(np.float64) * 2 ** 16)


def test_rmsnorm_canon_sum_order(oracle_mod):
    """x = [2^12, 1, 1, ...] (n = 4096, T = 512 lanes of V = 8): lane 0
    (elements 0..7) absorbs its seven 1's into 2^24 (fp32 spacing 2 there),
    the other 511 lanes hold 8 each, and the tree adds these even numbers
    exactly: S = 2^24 + 4088 (exact sum 2^24 + 4095; a left-to-right fp32
    sum gives 2^24; lanes of V = 4 would give 2^24 + 4092)."""
    n = 4096
    x = np.full(n, 0x3F80, np.uint16)
    x[0] = 0x4580                                              # 4096.0 = 2^12
    for eps in (0.0, 1e-6):
        S = F32(2.0 ** 24 + 4088)
        want = F32(F32(1.0) / np.sqrt(F32(F32(S / F32(n)) + F32(eps)), dtype=np.float32))
        assert f32bits(oracle_mod.rmsnorm_inv_canon(x, eps)) == f32bits(want)
    # constant row: S = n exactly
    ones = np.full(n, 0x3F80, np.uint16)
    want = F32(F32(1.0) / np.sqrt(F32(F32(1.0) + F32(1e-6)), dtype=np.float32))
    assert f32bits(oracle_mod.rmsnorm_inv_canon(ones, 1e-6)) == f32bits(want)


def test_rmsnorm_canon_product_order(oracle_mod):
    """Rows x = k/16 with integer |k| <= 63, n = 4096: every x^2 is a
    multiple of 1/256 and the whole sum stays below 2^16, so every partial
    sum is exact and S = sum(k^2)/256 in any order.  inv = fl(1/fl(sqrt(
    fl(fl(S/n) + eps)))) is then a closed form, and the reading of the RMSNorm
    output is y = bf16(fl(fl(x * inv) * w)).  On these 512 rows (seed 2)
    some outputs change under either other order of the two products,
    x * (inv * w) or (x * w) * inv, so the pin tells the orders apart."""
    R, n = 512, 4096
    g = np.random.default_rng(2)
    k = g.integers(-63, 64, size=(R, n))
    x = (k / 16.0).astype(np.float32)
    xb = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(oracle_mod.bf16_to_f32(xb), x)                  # x is exact in bf16
    w = torch.from_numpy((g.standard_normal(n) * 0.1 + 1.0).astype(np.float32)).to(torch.bfloat16)
    wb = w.view(torch.int16).numpy().view(np.uint16)
    wf = w.float().numpy()
    m = (k.astype(np.int64) ** 2).sum(axis=1)
    assert np.all(m < 2 ** 24)
    S = (m / 256.0).astype(np.float32)
    assert np.all(S.astype(np.float64) == m / 256.0)
    eps = F32(1e-6)
    inv = (F32(1.0) / np.sqrt((S / F32(n)).astype(np.float32) + eps).astype(np.float32)).astype(np.float32)
    inv = inv[:, None]

    def bf16(v):
        return torch.from_numpy(np.ascontiguousarray(v, np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)

    want = bf16((x * inv).astype(np.float32) * wf)
    other1 = bf16(x * (inv * wf).astype(np.float32))
    other2 = bf16((x * wf).astype(np.float32) * inv)
    assert np.sum(want != other1) > 0 and np.sum(want != other2) > 0     # the pin discriminates
    got = oracle_mod.rmsnorm_canon(xb, wb, eps=1e-6)
    assert np.array_equal(got, want)


def test_rmsnorm_canon_vs_exact(oracle_mod):
    x, w = synth.rmsnorm_inputs(16, 4096, seed=8)
    yc = oracle_mod.bf16_to_f32(oracle_mod.rmsnorm_canon(x, w)).astype(np.float64)
    ye = oracle_mod.rmsnorm_exact(x, w)
    ulp = np.spacing(np.abs(ye).astype(np.float32)).astype(np.float64) * 2 ** 16   # bf16 ulp
    assert np.all(np.abs(yc - ye) <= ulp)


# ------------------------------------------------------------- log_softmax

def test_log_softmax_exact_vs_torch(oracle_mod):
    x = synth.logits_inputs(3, 1000, seed=9)
    got = oracle_mod.log_softmax_exact(x)
    want = torch.log_softmax(torch.from_numpy(x.astype(np.float64)), dim=-1).numpy()
    np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-12)


def test_log_softmax_canon_closed_forms(oracle_mod):
    n = 151936
    # equal logits: every term is exp(0) = 1, S = n exactly, out = -log(n)
    x = np.full((1, n), 0.37, np.float32)
    out = oracle_mod.log_softmax_canon(x)[0]
    want = -math.log(n)
    assert np.all(out == out[0])
    assert abs(float(out[0]) - want) <= float(ulp32(want))
    # one logit far above the rest: S = 1, L = 0, out = x - max exactly
    x = np.full((1, 1024), -200.0, np.float32)
    x[0, 17] = 5.0
    out = oracle_mod.log_softmax_canon(x)[0]
    assert out[17] == 0.0 and np.all(out[np.arange(1024) != 17] == F32(-205.0))


def test_log_softmax_canon_sum_order(oracle_mod):
    """n = 8192, T = 4096 lanes of V = 4.  x[0] = 0 is the max (term 1),
    x[4..7] = -17 (term eps = exp(-17) ~ 4.1e-8, below half an ulp of 1),
    every other logit -200 (term 0).  Lane 0 holds elements 0..3: 1.
    Lane 1 holds elements 4..7: c = ((eps + eps) + eps) + eps ~ 1.7e-7.
    The tree gives S = fl(1 + c) = 1 + 2^-23, so L = log(S) != 0; a
    left-to-right sum would absorb every eps into 1 and give L = 0."""
    n = 8192
    x = np.full((1, n), -200.0, np.float32)
    x[0, 0] = 0.0
    x[0, 4:8] = -17.0
    eps = oracle_mod.exp_spec(-17.0)
    assert eps < 2.0 ** -24
    c = F32(F32(F32(F32(F32(0) + eps) + eps) + eps) + eps)
    S = F32(F32(1.0) + c)
    assert S == F32(1.0 + 2.0 ** -23)
    L = oracle_mod.log_spec(S)
    out = oracle_mod.log_softmax_canon(x)[0]
    assert f32bits(out[0]) == f32bits(F32(F32(0.0) - L))
    assert f32bits(out[5]) == f32bits(F32(F32(-17.0) - L))
    assert f32bits(out[9]) == f32bits(F32(F32(-200.0) - L))


def test_log_softmax_canon_lane_count(oracle_mod):
    """Pins T = 4096: n = 8192, x[0] = 0 (term 1), x[4096..4099] = -17
    (vector 1024, terms eps), rest -200 (terms 0).  With 4096 lanes vector
    1024 is lane 1024, its own chain: c = four eps, S = fl(1 + c) = 1 + 2^-23,
    L != 0 and out[0] = -L.  With 1024 lanes it would be lane 0 again and be
    absorbed into 1 (L = 0, out[0] = 0)."""
    n = 8192
    x = np.full((1, n), -200.0, np.float32)
    x[0, 0] = 0.0
    x[0, 4096:4100] = -17.0
    eps = oracle_mod.exp_spec(-17.0)
    c = F32(F32(F32(F32(F32(0) + eps) + eps) + eps) + eps)
    L = oracle_mod.log_spec(F32(F32(1.0) + c))
    assert L != 0
    out = oracle_mod.log_softmax_canon(x)[0]
    assert f32bits(out[0]) == f32bits(F32(F32(0.0) - L))
    assert f32bits(out[4097]) == f32bits(F32(F32(-17.0) - L))


def test_log_softmax_canon_shift_invariance(oracle_mod):
    """log_softmax(x + c) = log_softmax(x) exactly when every x - max is
    exact in both: integer logits in [-40, 0] shifted by c = 2^20 (all
    exactly representable, their differences exact).  This pins the order
    of the output step: (x - max) - L; x - (max + L) would round max + L at
    the scale of 2^20."""
    g = np.random.default_rng(11)
    x = g.integers(-40, 1, size=(3, 8192)).astype(np.float32)
    a = oracle_mod.log_softmax_canon(x)
    b = oracle_mod.log_softmax_canon(x + np.float32(2.0 ** 20))
    assert np.array_equal(f32bits(a), f32bits(b))
    assert not np.all(a == np.round(a))               # L is not an integer: the case is not trivial


def test_log_softmax_canon_vs_exact(oracle_mod):
    x = synth.logits_inputs(4, 151936, seed=10)
    c = oracle_mod.log_softmax_canon(x).astype(np.float64)
    e = oracle_mod.log_softmax_exact(x)
    assert np.all(np.abs(c - e) <= 4 * ulp32(e) + 4 * ulp32(12.0))


# ------------------------------------------------------------------- mean

def test_mean_exact_and_canon(oracle_mod):
    x = synth.normal_f32((6, 4096), 1.0, seed=11)
    np.testing.assert_allclose(oracle_mod.mean_exact(x), x.astype(np.float64).mean(axis=1), rtol=1e-12)
    c = oracle_mod.mean_canon(x).astype(np.float64)
    assert np.all(np.abs(c - oracle_mod.mean_exact(x)) <= 1e-6)
    # constant rows and integer rows are exact
    assert np.all(oracle_mod.mean_canon(np.full((3, 151936), 0.25, np.float32)) == F32(0.25))
    xi = synth.integer_f32((4, 8192), -50, 50, seed=12)
    assert np.array_equal(oracle_mod.mean_canon(xi),
                          (xi.astype(np.int64).sum(axis=1) / 8192).astype(np.float32))


def test_mean_canon_order(oracle_mod):
    """n = 8192, V = 4, T = 1024: lane 0 holds vectors 0 and 1024 (elements
    0..3 and 4096..4099), lane 1 holds vector 1 (elements 4..7).  x[0] = 1e8,
    x[4096] = 1 land in lane 0 (1e8 + 1 -> 1e8), x[4] = -1e8 in lane 1; the
    tree then cancels them: canonical mean 0 (sequential fp32: 1/8192)."""
    x = np.zeros((1, 8192), np.float32)
    x[0, 0], x[0, 4096], x[0, 4] = 1e8, 1.0, -1e8
    assert oracle_mod.mean_canon(x)[0] == 0.0
    assert oracle_mod.mean_exact(x)[0] == 1.0 / 8192


# ------------------------------------------------------- decode attention
# "Restoring AI Reproducibility", 2-3 (attention) and 3-2 (a fixed-size
# split of the KV cache, so the order depends on nothing but the sequence).

def _bf(x):
    return torch.from_numpy(np.ascontiguousarray(x, np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def test_attn_exact_vs_torch(oracle_mod):
    g = np.random.default_rng(21)
    B, Hq, Hkv, D, Lmax = 3, 4, 2, 64, 300
    q = _bf(g.standard_normal((B, Hq, D)))
    k = _bf(g.standard_normal((B, Hkv, Lmax, D)))
    v = _bf(g.standard_normal((B, Hkv, Lmax, D)))
    lens = np.array([300, 1, 129], np.int32)
    scale = 1.0 / math.sqrt(D)
    got = oracle_mod.attn_decode_exact(q, k, v, lens, scale)
    qf, kf, vf = (torch.from_numpy(oracle_mod.bf16_to_f32(a).astype(np.float64)) for a in (q, k, v))
    for b in range(B):
        for h in range(Hq):
            hk = h // (Hq // Hkv)
            L = int(lens[b])
            w = torch.softmax(scale * (kf[b, hk, :L] @ qf[b, h]), dim=0)
            np.testing.assert_allclose(got[b, h], (w @ vf[b, hk, :L]).numpy(), rtol=1e-12, atol=1e-12)
    # a sequence of length 0 gives 0
    z = oracle_mod.attn_decode_exact(q, k, v, np.array([0, 5, 0], np.int32), scale)
    assert np.all(z[0] == 0) and np.all(z[2] == 0)


def test_attn_canon_vs_exact(oracle_mod):
    g = np.random.default_rng(22)
    B, Hq, Hkv, D, Lmax = 2, 8, 2, 128, 1100
    q = _bf(g.standard_normal((B, Hq, D)))
    k = _bf(g.standard_normal((B, Hkv, Lmax, D)))
    v = _bf(g.standard_normal((B, Hkv, Lmax, D)))
    lens = np.array([1100, 517], np.int32)
    scale = 1.0 / math.sqrt(D)
    c = oracle_mod.attn_decode_canon(q, k, v, lens, scale).astype(np.float64)
    e = oracle_mod.attn_decode_exact(q, k, v, lens, scale)
    assert np.max(np.abs(c - e)) <= 1e-5 * np.max(np.abs(e)) + 1e-6


def test_attn_canon_closed_forms(oracle_mod):
    D, Lmax = 128, 1300
    q = _bf(np.random.default_rng(23).standard_normal((1, 1, D)))
    zero_k = np.zeros((1, 1, Lmax, D), np.uint16)                  # every score 0, every p = 1
    # constant value rows: out = that row exactly, at any length
    vrow = _bf(np.linspace(-3, 3, D))
    v = np.tile(vrow, (1, 1, Lmax, 1))
    for L in (1, 5, 255, 256, 257, 1280, 1300):
        out = oracle_mod.attn_decode_canon(q, zero_k, v, np.array([L], np.int32), 0.125)
        assert np.array_equal(out[0, 0], oracle_mod.bf16_to_f32(vrow)), L
    # one dominant key (score > 103 above the rest): out = its value row
    k = np.zeros((1, 1, Lmax, D), np.uint16)
    qd = np.zeros((1, 1, D), np.float32)
    qd[0, 0, 0] = 16.0
    kd = np.zeros((1, 1, Lmax, D), np.float32)
    kd[0, 0, 700, 0] = 64.0                                        # score 1024 * 0.125 = 128
    vals = _bf(np.random.default_rng(24).standard_normal((1, 1, Lmax, D)))
    out = oracle_mod.attn_decode_canon(_bf(qd), _bf(kd), vals, np.array([1300], np.int32), 0.125)
    assert np.array_equal(out[0, 0], oracle_mod.bf16_to_f32(vals[0, 0, 700]))


def test_attn_canon_frame_order(oracle_mod):
    """The two frames of the reading.  Inside a chunk, L = 5 keys with p = 1
    and values [2^24, 0, 1, 1, 0]: the padded 256-slot perfect tree pairs
    (2^24 + 0) and (1 + 1) and gives 2^24 + 2 exactly (a halving tree over 5
    or a running sum loses both 1's: 2^24).  Across chunks, 5 full chunks
    whose sums are [2^24, 0, 1, 1, 0] (values 2^16, 0, 2^-8, 2^-8, 0): the
    chunk count padded to 8 gives the same pairing.  out = fl((2^24+2)/L)."""
    D = 32
    q = np.zeros((1, 1, D), np.uint16)
    for L, col in ((5, [2.0 ** 24, 0.0, 1.0, 1.0, 0.0]),
                   (1280, np.repeat([2.0 ** 16, 0.0, 2.0 ** -8, 2.0 ** -8, 0.0], 256))):
        vf = np.zeros((1, 1, L, D), np.float32)
        vf[0, 0, :, 0] = col
        out = oracle_mod.attn_decode_canon(q, np.zeros((1, 1, L, D), np.uint16), _bf(vf), np.array([L], np.int32), 1.0)
        want = F32(F32(2.0 ** 24 + 2) / F32(L))
        assert f32bits(out[0, 0, 0]) == f32bits(want), L
        assert f32bits(want) != f32bits(F32(F32(2.0 ** 24) / F32(L)))
