"""CPU checks of the bench's work accounting: the algorithmic FLOPs behind
the reported TFLOP/s and the roofline, and the achieved sparsity.

The bench counts 4*d FLOPs per (query, key) pair of the listed blocks (two
products of d multiply-adds each), a full 64 x 64 block holding 4096 pairs
and the diagonal block the 64*65/2 causally visible ones.  Here the pairs are
counted instead by enumerating token positions, so a wrong diagonal test, a
wrong pair count or an off-by-one in the list lengths fails.
"""
import numpy as np
import torch

import bench
import oracle
from learned_block_sparse_seer_b200 import synth


def _pairs_by_enumeration(counts, indices):
    """Visible (query, key) token pairs of the listed blocks, by positions."""
    q = np.arange(64)[:, None]
    k = np.arange(64)[None, :]
    total = 0
    B, H, nb = counts.shape
    for b in range(B):
        for h in range(H):
            for i in range(nb):
                for j in indices[b, h, i, :counts[b, h, i]]:
                    # absolute positions 64 i + q (query) and 64 j + k (key)
                    total += int(np.count_nonzero(64 * int(j) + k <= 64 * i + q))
    return total


def _lists(mode, seed, **kw):
    w = synth.Workload("t", 2, 4, 2, 64 * 13, 64, 64, "fp32", "tiny", 0)
    s = synth.make_scores_like(w, seed=seed)
    c, ix, _ = oracle.select(s, mode, **kw)
    return w, c, ix


def _check(w, c, ix):
    flops, blocks, diag, sparsity = bench.attn_flops(torch.from_numpy(c), torch.from_numpy(ix), w.d)
    pairs = _pairs_by_enumeration(c, ix)
    assert flops == 4.0 * w.d * pairs
    assert blocks == int(c.sum())
    causal = w.B * w.Hq * w.nb * (w.nb + 1) // 2
    assert abs(sparsity - (1.0 - blocks / causal)) < 1e-12
    # the diagonal count is the number of rows whose list holds block i
    nd = sum(int(i in ix[b, h, i, :c[b, h, i]]) for b in range(w.B) for h in range(w.Hq) for i in range(w.nb))
    assert diag == nd


def test_flops_topk_density_lists():
    w, c, ix = _lists(oracle.MODE_TOPK_DENSITY, seed=5, density=0.3)
    _check(w, c, ix)


def test_flops_threshold_lists_without_diagonal():
    # threshold lists often leave out the diagonal block, and some rows are empty
    w, c, ix = _lists(oracle.MODE_THRESHOLD, seed=6, T=0.2)
    assert (c == 0).any() and any(
        c[0, 0, i] > 0 and i not in ix[0, 0, i, :c[0, 0, i]] for i in range(w.nb))
    _check(w, c, ix)


def test_flops_all_ones_mask_is_dense_causal():
    w = synth.Workload("t", 1, 2, 1, 64 * 9, 64, 64, "fp32", "tiny", 0)
    c, ix = oracle.dense_lists(w.B, w.Hq, w.nb)
    flops, blocks, diag, sparsity = bench.attn_flops(torch.from_numpy(c), torch.from_numpy(ix), w.d)
    n = w.n
    # every causal token pair of every head: n (n + 1) / 2 per head
    assert flops == 4.0 * w.d * w.B * w.Hq * n * (n + 1) // 2
    assert diag == w.B * w.Hq * w.nb and sparsity == 0.0
