"""LoRA shrink on the GPU against the oracle.

(a) every mode within |gpu - exact| <= 1e-3 * sum|x*a| of the fp64 exact
    product; integer-valued inputs (every partial exact) give the exact value;
(b) the fixed-order combine is bit-exact: the kernel's output equals the
    oracle's canonical fp32 tree over the kernel's own 64-wide leaves (each
    leaf measured by a K = 64 call on that slice);
(c) invariance: bitwise the same for every split count, for UNSPLIT vs TREE,
    for every M and row position, for every replay; ATOMIC is allowed to vary.
Source: "Reproducible LoRA Inference Through Deterministic Split-K Reduction"
(Highlights, Q&A)."""
import numpy as np
import pytest
import torch

import oracle
from helpers import assert_tol, check_plan_table, dev, dev_bf16, host_bits
from invariant_bi_lora_b200 import bi, synth

pytestmark = pytest.mark.gpu


def run_shrink(x, at, splits, mode, M=None):
    M = x.shape[0]
    y = torch.empty(M, at.shape[0], dtype=torch.float32, device="cuda")
    bi.lora_shrink(x, at, y, splits=splits, mode=mode)
    torch.cuda.synchronize()
    return y


@pytest.fixture(scope="module")
def cfg1():
    """Config of the split-K study: M=16, K=4096, r=16; x ~ N(0,1),
    A ~ N(0, 1/sqrt(K)); seed 0."""
    d = synth.lora_inputs(16, 4096, 16, seed=0)
    return d["x"], d["at"][0]


@pytest.mark.parametrize("mode,splits", [("unsplit", 1), ("tree", 8), ("atomic", 8), ("tree", 1),
                                         ("tree", 16), ("atomic", 2)])
def test_cfg1_tolerance(cfg1, mode, splits):
    x, at = cfg1
    y = run_shrink(dev_bf16(x), dev_bf16(at), splits, mode).cpu().numpy()
    exact, bound = oracle.shrink_exact(x, at)
    assert_tol(y, exact, bound, what=f"{mode} s={splits}")


def test_cfg1_split_and_mode_invariance(cfg1):
    x, at = (dev_bf16(a) for a in cfg1)
    ref = host_bits(run_shrink(x, at, 1, "unsplit"))
    for s in (1, 2, 4, 8, 16):
        assert np.array_equal(host_bits(run_shrink(x, at, s, "tree")), ref), s


def test_cfg1_replay_100(cfg1):
    """100 identical-input replays: TREE never varies; ATOMIC is measured
    (the variation rate of the atomic mode is what the study reports)."""
    x, at = (dev_bf16(a) for a in cfg1)
    first = host_bits(run_shrink(x, at, 8, "tree"))
    outs_atomic = []
    for _ in range(100):
        assert np.array_equal(host_bits(run_shrink(x, at, 8, "tree")), first)
        outs_atomic.append(host_bits(run_shrink(x, at, 8, "atomic")))
    exact, bound = oracle.shrink_exact(*cfg1)
    for o in outs_atomic:
        assert_tol(o.view(np.float32), exact, bound, what="atomic replay")


def test_atomic_varies_where_tree_does_not(cfg1):
    """The nondeterminism the split-K study measures ("Reproducible LoRA
    Inference ...", Highlights): identical-input replays of the atomic
    split-K shrink give more than one bit pattern, while the tree combine
    gives one.  Up to 10,000 replays, stopping at the first change."""
    x, at = (dev_bf16(a) for a in cfg1)
    first_tree = host_bits(run_shrink(x, at, 8, "tree"))
    first_atomic = host_bits(run_shrink(x, at, 8, "atomic"))
    varied = 0
    for i in range(10000):
        if not np.array_equal(host_bits(run_shrink(x, at, 8, "atomic")), first_atomic):
            varied = i + 1
            break
        if i % 50 == 0:
            assert np.array_equal(host_bits(run_shrink(x, at, 8, "tree")), first_tree)
    assert varied, "10,000 atomic replays all gave the same bits"
    for _ in range(20):
        assert np.array_equal(host_bits(run_shrink(x, at, 8, "tree")), first_tree)


def test_leaf_tree_bit_exact(cfg1):
    """The output is exactly the canonical fp32 tree over the 64 leaves,
    each leaf = the kernel's value for that 64-wide K slice alone."""
    x, at = cfg1
    K = x.shape[1]
    L = K // 64
    leaves = np.empty((L, x.shape[0], at.shape[0]), np.float32)
    for l in range(L):
        xs = dev_bf16(np.ascontiguousarray(x[:, 64 * l:64 * l + 64]))
        as_ = dev_bf16(np.ascontiguousarray(at[:, 64 * l:64 * l + 64]))
        leaves[l] = run_shrink(xs, as_, 1, "unsplit").cpu().numpy()
    want = oracle.tree_combine(leaves)
    for mode, s in (("unsplit", 1), ("tree", 8), ("tree", 2)):
        got = run_shrink(dev_bf16(x), dev_bf16(at), s, mode).cpu().numpy()
        assert np.array_equal(got.view(np.uint32), want.view(np.uint32)), (mode, s)


@pytest.mark.parametrize("K", [192, 320, 5120])
def test_leaf_tree_non_power_of_two(K):
    """Leaf counts 3, 5, 80: the halving tree with ceil(n/2) on the left."""
    d = synth.lora_inputs(9, K, 8, seed=K)
    x, at = d["x"], d["at"][0]
    L = K // 64
    leaves = np.stack([run_shrink(dev_bf16(np.ascontiguousarray(x[:, 64 * l:64 * l + 64])),
                                  dev_bf16(np.ascontiguousarray(at[:, 64 * l:64 * l + 64])),
                                  1, "unsplit").cpu().numpy() for l in range(L)])
    want = oracle.tree_combine(leaves)
    got = run_shrink(dev_bf16(x), dev_bf16(at), 1, "unsplit").cpu().numpy()
    assert np.array_equal(got.view(np.uint32), want.view(np.uint32))
    s = 1
    while L % (2 * s) == 0 and 2 * s <= 16:
        s *= 2
        g2 = run_shrink(dev_bf16(x), dev_bf16(at), s, "tree").cpu().numpy()
        assert np.array_equal(g2.view(np.uint32), want.view(np.uint32)), s
    exact, bound = oracle.shrink_exact(x, at)
    assert_tol(got, exact, bound)


def test_integer_inputs_exact():
    """x, A in {-4..4}: every partial sum is an integer below 2^24, so any
    order is exact and the result must equal the exact product."""
    x = synth.integer_bf16((37, 4096), -4, 4, seed=3, tag=1)
    at = synth.integer_bf16((16, 4096), -4, 4, seed=3, tag=2)
    exact, _ = oracle.shrink_exact(x, at)
    for mode, s in (("unsplit", 1), ("tree", 8), ("atomic", 8)):
        got = run_shrink(dev_bf16(x), dev_bf16(at), s, mode).cpu().numpy()
        assert np.array_equal(got.astype(np.float64), exact), mode


@pytest.mark.parametrize("r", [8, 16, 32, 64, 128])
def test_ranks_and_ragged_rows(r):
    M, K = 37, 1024
    d = synth.lora_inputs(M, K, r, seed=r)
    x, at = d["x"], d["at"][0]
    exact, bound = oracle.shrink_exact(x, at)
    ref = None
    for mode, s in (("unsplit", 1), ("tree", 4), ("tree", 16), ("atomic", 4)):
        got = run_shrink(dev_bf16(x), dev_bf16(at), s, mode).cpu().numpy()
        assert_tol(got, exact, bound, what=f"r={r} {mode}")
        if mode != "atomic":
            ref = got if ref is None else ref
            assert np.array_equal(got.view(np.uint32), ref.view(np.uint32)), (r, mode, s)


def test_batch_invariance_rows_and_positions(cfg1):
    """Row i of the M=16 result is bitwise the same when the row sits at
    any position of a larger batch (M = 1, 7, 64, 513, 4096)."""
    x, at = cfg1
    A = dev_bf16(at)
    ref = host_bits(run_shrink(dev_bf16(x), A, 8, "tree"))
    filler = synth.normal_bf16((4096, 4096), 1.0, seed=99, tag=1)
    for M in (1, 7, 64, 513, 4096):
        for pos in sorted({0, M // 2, M - 1, max(0, M - 16)}):
            rows = min(16, M - pos)
            xb = filler[:M].copy()
            xb[pos:pos + rows] = x[:rows]
            got = host_bits(run_shrink(dev_bf16(xb), A, 8, "tree"))
            assert np.array_equal(got[pos:pos + rows], ref[:rows]), (M, pos)
            got1 = host_bits(run_shrink(dev_bf16(xb), A, 1, "unsplit"))
            assert np.array_equal(got1[pos:pos + rows], ref[:rows]), (M, pos)


def test_empty_batch():
    A = dev_bf16(synth.normal_bf16((16, 4096), 0.02, seed=1))
    x = torch.empty(0, 4096, dtype=torch.bfloat16, device="cuda")
    y = torch.empty(0, 16, dtype=torch.float32, device="cuda")
    bi.lora_shrink(x, A, y, splits=8, mode="tree")
    torch.cuda.synchronize()


def test_rejects_bad_split():
    A = dev_bf16(synth.normal_bf16((16, 4096), 0.02, seed=1))
    x = dev_bf16(synth.normal_bf16((4, 4096), 1.0, seed=1))
    y = torch.empty(4, 16, dtype=torch.float32, device="cuda")
    with pytest.raises(bi.BiError):
        bi.lora_shrink(x, A, y, splits=3, mode="tree")


# ------------------------------------------------------------- segmented

@pytest.fixture(scope="module")
def cfg4():
    """Segmented multi-adapter config: M=4096 tokens, 8 adapters (uniform
    random id per token), K=4096, r=16."""
    return synth.lora_inputs(4096, 4096, 16, n_adapters=8, N=4096, seed=0)


def test_plan_matches_oracle(cfg4):
    ids = cfg4["ids"].copy()
    ids[::97] = -1                       # some tokens without an adapter
    ids[5] = 8
    plan = bi.lora_plan(dev(ids), 8).cpu().numpy()
    M = ids.size
    perm, offs = plan[:M], plan[M:]
    want_perm, want_offs = oracle.segment(ids, 8)
    assert np.array_equal(offs[:9], want_offs)
    assert offs[9] == M
    assert np.array_equal(perm[:offs[8]], want_perm)
    invalid = np.nonzero((ids < 0) | (ids >= 8))[0]
    assert np.array_equal(perm[offs[8]:], invalid)
    check_plan_table(plan, np.concatenate([want_perm, invalid]).astype(np.int32), offs, 8)


@pytest.mark.parametrize("M,n_ad,bad", [(1, 1, 0), (5, 3, 0), (1000, 8, 0), (4096, 8, 0), (3000, 256, 0),
                                        (0, 4, 0), (4097, 2, 0), (12289, 8, 0), (65536, 256, 0), (4096, 31, 1),
                                        (4096, 32, 1), (513, 64, 1), (20000, 31, 1), (100003, 5, 1),
                                        (70001, 200, 1)])
def test_plan_shapes(M, n_ad, bad):
    """Every size path of the plan kernel (one chunk per warp or several,
    at most 32 classes or more), with tokens outside every adapter where
    `bad` is set (id -1 and id >= n_ad go to the last class)."""
    ids = synth.adapter_ids(M, n_ad, seed=M + n_ad)
    if bad:
        ids[::13] = -1
        ids[7::29] = n_ad + 3
    plan = bi.lora_plan(dev(ids), n_ad).cpu().numpy() if M else None
    if M == 0:
        return
    want_perm, want_offs = oracle.segment(ids, n_ad)
    invalid = np.nonzero((ids < 0) | (ids >= n_ad))[0]
    full = np.concatenate([want_perm, invalid]).astype(np.int32)
    assert np.array_equal(plan[M:M + n_ad + 1], want_offs)
    assert np.array_equal(plan[:M], full)
    assert plan[M + n_ad + 1] == M
    check_plan_table(plan, full, plan[M:M + n_ad + 2], n_ad)


@pytest.mark.parametrize("r", [8, 16, 64])
def test_segmented_shrink(cfg4, r):
    d = cfg4 if r == 16 else synth.lora_inputs(4096, 4096, r, n_adapters=8, seed=0)
    x, at, ids = d["x"], d["at"], d["ids"]
    X, A = dev_bf16(x), dev_bf16(at)
    plan = bi.lora_plan(dev(ids), 8)
    outs = {}
    for mode, s in (("tree", 8), ("unsplit", 1), ("atomic", 8), ("tree", 2)):
        y = torch.empty(4096, r, dtype=torch.float32, device="cuda")
        bi.lora_shrink_segmented(X, A, plan, y, splits=s, mode=mode)
        outs[(mode, s)] = host_bits(y)
    assert np.array_equal(outs[("tree", 8)], outs[("unsplit", 1)])
    assert np.array_equal(outs[("tree", 8)], outs[("tree", 2)])
    # sampled rows against the exact product
    rows = np.random.default_rng(r).choice(4096, 256, replace=False)
    exact, bound = oracle.shrink_exact(x[rows], at, ids[rows])
    for key, o in outs.items():
        assert_tol(o.view(np.float32)[rows], exact, bound, what=str(key))
    # each row equals the single-adapter kernel on that row alone (bitwise)
    for a in range(8):
        sel = np.nonzero(ids == a)[0][:40]
        y1 = host_bits(run_shrink(dev_bf16(x[sel]), dev_bf16(at[a]), 8, "tree"))
        assert np.array_equal(outs[("tree", 8)][sel], y1), a


def test_segmented_no_adapter_rows_are_zero(cfg4):
    x, at, ids = cfg4["x"][:300], cfg4["at"], cfg4["ids"][:300].copy()
    ids[::7] = -1
    plan = bi.lora_plan(dev(ids), 8)
    for mode, s in (("tree", 8), ("unsplit", 1), ("atomic", 8)):
        y = torch.full((300, 16), 7.0, dtype=torch.float32, device="cuda")
        bi.lora_shrink_segmented(dev_bf16(x), dev_bf16(at), plan, y, splits=s, mode=mode)
        yh = y.cpu().numpy()
        assert np.all(yh[::7] == 0.0), mode
        exact, bound = oracle.shrink_exact(x, at, ids)
        assert_tol(yh, exact, bound, what=mode)


def test_status_clean_after_shrink(cfg1):
    x, at = (dev_bf16(a) for a in cfg1)
    run_shrink(x, at, 8, "tree")
    assert bi.get_device_status() == 0


@pytest.mark.parametrize("K,r", [(4096, 16), (2048, 16), (4096, 8), (2048, 8)])
def test_large_ragged_batch(K, r):
    """A batch of 4099 tokens (several waves of row tiles, a ragged last
    tile, rows without an adapter): in modes TREE and UNSPLIT every row
    must equal, bit for bit, the same row computed in a small batch, rows
    without an adapter must be zero, and a ragged plain batch must match
    too."""
    M = 4099
    d = synth.lora_inputs(M, K, r, n_adapters=5, seed=K + r)
    x, at, ids = d["x"], d["at"], d["ids"].copy()
    ids[::11] = -1
    ids[3::17] = 9                         # out of range: no adapter
    X, A = dev_bf16(x), dev_bf16(at)
    plan = bi.lora_plan(dev(ids), 5)
    got = {}
    for mode, s in (("tree", 8), ("unsplit", 1), ("tree", 4)):
        y = torch.full((M, r), 7.0, dtype=torch.float32, device="cuda")
        bi.lora_shrink_segmented(X, A, plan, y, splits=s, mode=mode)
        got[(mode, s)] = host_bits(y)
    ref = got[("tree", 8)]
    for k, v in got.items():
        assert np.array_equal(v, ref), k
    none = (ids < 0) | (ids >= 5)
    assert np.all(ref.view(np.float32)[none] == 0.0)
    for a in range(5):
        sel = np.nonzero(ids == a)[0]
        sel = np.concatenate([sel[:24], sel[-24:]])
        y1 = host_bits(run_shrink(dev_bf16(x[sel]), dev_bf16(at[a]), 8, "tree"))
        assert np.array_equal(ref[sel], y1), a
    # plain (single adapter) batch with a ragged last tile
    y = host_bits(run_shrink(X, dev_bf16(at[0]), 8, "tree"))
    tail = np.arange(M - 21, M)
    y1 = host_bits(run_shrink(dev_bf16(x[tail]), dev_bf16(at[0]), 8, "tree"))
    assert np.array_equal(y[tail], y1)
    exact, bound = oracle.shrink_exact(x[tail], at[0])
    assert_tol(y[tail].view(np.float32), exact, bound)
    assert bi.get_device_status() == 0
