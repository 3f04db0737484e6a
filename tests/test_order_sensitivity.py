"""Why the atomic combine varies, as a CPU fact that does not depend on GPU
timing ("Reproducible LoRA Inference Through Deterministic Split-K
Reduction", Highlights: fp32 atomics add the split-K partials in arrival
order).  For the split-K study's configuration (M = 16, K = 4096, r = 16,
split-K 8), the eight split partials of every output element are added one
after another from 0 -- what atomicAdd does -- in all 8! = 40,320 orders.
Most elements take several different bit patterns; the canonical tree over
the same partials is one fixed value.  The partials are stand-ins for the
kernel's: each 64-wide leaf is the oracle's exact product rounded to fp32,
and each split's value is the oracle's canonical tree over its 8 leaves."""
import itertools

import numpy as np

import oracle
from invariant_bi_lora_b200 import synth


def test_split_partials_in_all_orders():
    d = synth.lora_inputs(16, 4096, 16, seed=0)
    x, at = d["x"], d["at"][0]
    L = 64
    leaves = np.stack([oracle.shrink_exact(np.ascontiguousarray(x[:, 64 * l:64 * l + 64]),
                                           np.ascontiguousarray(at[:, 64 * l:64 * l + 64]))[0]
                       for l in range(L)]).astype(np.float32)                  # [64, 16, 16]
    splits = np.stack([oracle.tree_combine(leaves[8 * s:8 * s + 8]) for s in range(8)])   # [8, 16, 16]
    P = splits.reshape(8, -1)                                                   # [8, 256]
    perms = np.array(list(itertools.permutations(range(8))), np.int64)         # [40320, 8]
    acc = np.zeros((perms.shape[0], P.shape[1]), np.float32)
    for step in range(8):
        acc = (acc + P[perms[:, step]]).astype(np.float32)
    bits = acc.view(np.uint32)
    distinct = np.array([np.unique(bits[:, e]).size for e in range(bits.shape[1])])
    varying = float(np.mean(distinct > 1))
    assert varying > 0.9, varying                 # nearly every element depends on the order
    assert distinct.max() >= 4
    # the canonical tree over the same partials is one value, equal to the
    # tree over all 64 leaves (the splits are its subtrees)
    tree = oracle.tree_combine(splits).reshape(-1)
    assert np.array_equal(tree.view(np.uint32), oracle.tree_combine(leaves).reshape(-1).view(np.uint32))
    # and the sequential orders scatter around it
    assert np.any(bits != tree.view(np.uint32)[None, :])
