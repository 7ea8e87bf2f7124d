"""Pins for the fp64 oracle: library routines, closed forms, invariants and the
values the SeerAttention pages print.  CPU only.

Each test checks the oracle against something other than itself, so that a
dropped term, wrong sign, wrong index or transposed operand in any oracle
function fails at least one of them.
"""
import json
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from learned_block_sparse_seer_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "pages_examples.json")
BLK = 64


def _rand(shape, seed, scale=1.0):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(*shape, generator=g) * scale).contiguous()


# ------------------------------------------------------------------ pooling --
def test_pool_q_is_avg_pool1d():
    Q = _rand((2, 3, 256, 16), 1)
    ref = F.avg_pool1d(Q.double().reshape(-1, 256, 16).transpose(1, 2), BLK, BLK)
    ref = ref.transpose(1, 2).reshape(2, 3, 4, 16).numpy()
    np.testing.assert_allclose(oracle.pool_q(Q), ref, rtol=0, atol=1e-14)


def test_pool_k_is_max_min_avg_in_that_order():
    K = _rand((1, 2, 192, 8), 2)
    x = K.double().reshape(-1, 192, 8).transpose(1, 2)
    mx = F.max_pool1d(x, BLK, BLK)
    mn = -F.max_pool1d(-x, BLK, BLK)
    av = F.avg_pool1d(x, BLK, BLK)
    ref = torch.cat([mx, mn, av], dim=1).transpose(1, 2).reshape(1, 2, 3, 24).numpy()
    got = oracle.pool_k(K)
    np.testing.assert_array_equal(got[..., :16], ref[..., :16])  # max/min exact
    np.testing.assert_allclose(got, ref, rtol=0, atol=1e-14)


def test_pool_constant_block_and_ordering():
    K = torch.zeros(1, 1, 128, 4)
    K[0, 0, :64] = torch.tensor([1.5, -2.0, 0.25, 7.0])
    kb = oracle.pool_k(K)
    np.testing.assert_array_equal(kb[0, 0, 0], np.tile([1.5, -2.0, 0.25, 7.0], 3))
    R = _rand((1, 2, 512, 8), 3)
    kb = oracle.pool_k(R)
    d = 8
    assert np.all(kb[..., :d] >= kb[..., 2 * d:]) and np.all(kb[..., 2 * d:] >= kb[..., d:2 * d])


# --------------------------------------------------------------- projection --
def test_project_matches_matmul_and_selects_rows():
    x = _rand((2, 3, 5, 12), 4).double()
    W = _rand((3, 7, 12), 5)
    ref = torch.einsum("hrc,bhic->bhir", W.double(), x).numpy()
    np.testing.assert_allclose(oracle.project(x, W), ref, rtol=1e-13, atol=1e-13)
    # a selector matrix picks the first 4 features (catches transposed W)
    sel = torch.zeros(3, 4, 12)
    sel[:, torch.arange(4), torch.arange(4)] = 1.0
    np.testing.assert_array_equal(oracle.project(x, sel), x[..., :4].numpy())


# ---------------------------------------------------------------- gate (Eq.1)
def _gate_inputs(seed=6, B=2, Hq=4, Hkv=2, nb=9, h=8):
    qt = _rand((B, Hq, nb, h), seed).double()
    kt = _rand((B, Hkv, nb, h), seed + 1).double()
    return qt, kt


def test_gate_scores_match_masked_softmax():
    qt, kt = _gate_inputs()
    d = 64
    G = qt.shape[1] // kt.shape[1]
    z = torch.einsum("bhic,bhjc->bhij", qt, kt.repeat_interleave(G, dim=1)) / math.sqrt(d)
    nb = qt.shape[2]
    mask = torch.tril(torch.ones(nb, nb, dtype=torch.bool))
    ref = torch.softmax(z.masked_fill(~mask, float("-inf")), dim=-1).numpy()
    got = oracle.gate_scores(qt, kt, d)
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-15)


def test_gate_rows_sum_to_one_and_upper_triangle_zero():
    qt, kt = _gate_inputs(seed=9)
    s = oracle.gate_scores(qt, kt, 128)
    np.testing.assert_allclose(s.sum(-1), 1.0, rtol=0, atol=1e-13)
    nb = s.shape[-1]
    assert np.all(s[..., np.triu_indices(nb, 1)[0], np.triu_indices(nb, 1)[1]] == 0)


def test_gate_uniform_when_query_weights_zero():
    w = synth.custom("g", 1, 2, 1, 512, 16, 8, "fp32", "tiny", 3)
    Q, K, _ = synth.make_qkv(w)
    Wq = torch.zeros(2, 8, 16)
    _, Wk = synth.make_gate_weights(w)
    s = oracle.gate(Q, K, Wq, Wk)
    nb = w.nb
    ref = np.tril(1.0 / np.arange(1, nb + 1)[:, None] * np.ones((nb, nb)))
    np.testing.assert_allclose(s[0, 0], ref, rtol=1e-14, atol=0)


def test_gate_two_blocks_is_sigmoid():
    qt, kt = _gate_inputs(seed=12, B=1, Hq=1, Hkv=1, nb=2, h=4)
    d = 16
    z10 = float(qt[0, 0, 1] @ kt[0, 0, 0]) / 4.0
    z11 = float(qt[0, 0, 1] @ kt[0, 0, 1]) / 4.0
    s = oracle.gate_scores(qt, kt, d)
    assert s[0, 0, 0, 0] == 1.0 and s[0, 0, 0, 1] == 0.0
    assert abs(s[0, 0, 1, 0] - 1.0 / (1.0 + math.exp(z11 - z10))) < 1e-15
    assert abs(s[0, 0, 1, 1] - 1.0 / (1.0 + math.exp(z10 - z11))) < 1e-15


def test_gate_gqa_uses_kv_head_of_group():
    # query heads 0,1 -> kv head 0; 2,3 -> kv head 1.  Swapping kv heads must
    # swap the score maps of the two groups.
    qt, kt = _gate_inputs(seed=21)
    s = oracle.gate_scores(qt, kt, 64)
    s_sw = oracle.gate_scores(qt[:, [2, 3, 0, 1]], kt[:, [1, 0]], 64)
    np.testing.assert_array_equal(s[:, [2, 3, 0, 1]], s_sw)


def test_gate_end_to_end_against_torch_pipeline():
    w = synth.custom("g2", 1, 4, 2, 640, 32, 16, "bf16", "layer", 4)
    Q, K, _ = synth.make_qkv(w)
    Wq, Wk = synth.make_gate_weights(w)
    x = Q.double().reshape(-1, w.n, w.d).transpose(1, 2)
    qb = F.avg_pool1d(x, BLK, BLK).transpose(1, 2).reshape(1, 4, w.nb, w.d)
    y = K.double().reshape(-1, w.n, w.d).transpose(1, 2)
    kb = torch.cat([F.max_pool1d(y, BLK, BLK), -F.max_pool1d(-y, BLK, BLK),
                    F.avg_pool1d(y, BLK, BLK)], 1).transpose(1, 2).reshape(1, 2, w.nb, 3 * w.d)
    qt = torch.einsum("hrc,bhic->bhir", Wq.double(), qb)
    kt = torch.einsum("hrc,bhic->bhir", Wk.double(), kb).repeat_interleave(2, dim=1)
    z = qt @ kt.transpose(-1, -2) / math.sqrt(w.d)
    mask = torch.tril(torch.ones(w.nb, w.nb, dtype=torch.bool))
    ref = torch.softmax(z.masked_fill(~mask, float("-inf")), -1).numpy()
    np.testing.assert_allclose(oracle.gate(Q, K, Wq, Wk), ref, rtol=1e-11, atol=1e-16)


# ------------------------------------------------------------- block RoPE --
def test_block_rope_rotation_structure():
    """Rotation keeps norms, rotates pair 0 by exactly the block index, and
    makes the dot product depend only on the block offset.  (The base reading
    theta/B itself is parity unpinned.)"""
    nb, h = 12, 8
    x = _rand((1, 1, nb, h), 30).double()
    y = oracle.block_rope(x, 10000.0)
    np.testing.assert_allclose(np.linalg.norm(y, axis=-1), np.linalg.norm(x.numpy(), axis=-1),
                               rtol=1e-13)
    for i in range(nb):
        a, b = x[0, 0, i, 0].item(), x[0, 0, i, h // 2].item()
        assert abs(y[0, 0, i, 0] - (a * math.cos(i) - b * math.sin(i))) < 1e-12
    # relative position: same vectors placed at (i, j) and (i+3, j+3)
    q = _rand((1, 1, 1, h), 31).double()
    k = _rand((1, 1, 1, h), 32).double()
    qs = oracle.block_rope(q.expand(1, 1, nb, h).contiguous(), 500000.0)[0, 0]
    ks = oracle.block_rope(k.expand(1, 1, nb, h).contiguous(), 500000.0)[0, 0]
    assert abs(qs[7] @ ks[2] - qs[10] @ ks[5]) < 1e-12
    assert abs(qs[7] @ ks[2] - qs[8] @ ks[2]) > 1e-6


# --------------------------------------------------------------- selection --
def test_threshold_is_strict_and_causal():
    w = synth.custom("s", 1, 2, 1, 64 * 40, 16, 8, "fp32")
    s = synth.make_scores_like(w, seed=3)
    T = 0.03
    counts, idx, worst = oracle.select(s, oracle.MODE_THRESHOLD, T=T)
    s64 = s.double().numpy()
    for h in range(2):
        for i in range(w.nb):
            ref = [j for j in range(i + 1) if s64[0, h, i, j] > np.float32(T)]
            assert counts[0, h, i] == len(ref)
            assert list(idx[0, h, i, :len(ref)]) == ref
    # a score exactly equal to T is not selected (strict '>')
    s2 = torch.zeros(1, 1, 2, 2)
    s2[0, 0, 0, 0] = 1.0
    s2[0, 0, 1] = torch.tensor([np.float32(0.25), np.float32(0.75)])
    c, ix, _ = oracle.select(s2, oracle.MODE_THRESHOLD, T=0.25)
    assert c[0, 0, 1] == 1 and ix[0, 0, 1, 0] == 1


def test_topk_matches_stable_argsort_with_ties():
    w = synth.custom("s", 1, 3, 1, 64 * 33, 16, 8, "fp32")
    for ties in (False, True):
        s = synth.make_scores_like(w, seed=5, ties=ties)
        s64 = s.double().numpy()
        for mode, k, rho in ((oracle.MODE_TOPK_K, 5, 0.0), (oracle.MODE_TOPK_DENSITY, 0, 0.3)):
            counts, idx, _ = oracle.select(s, mode, k=k, density=rho)
            for h in range(3):
                for i in range(w.nb):
                    row = s64[0, h, i, :i + 1]
                    order = np.argsort(-row, kind="stable")  # ties: lower j first
                    if mode == oracle.MODE_TOPK_K:
                        ki = min(k, i + 1)
                    else:
                        ki = min(max(math.ceil(float(np.float32(np.float32(rho) * np.float32(i + 1)))), 1), i + 1)
                    ref = sorted(order[:ki].tolist())
                    assert counts[0, h, i] == ki
                    assert idx[0, h, i, :ki].tolist() == ref
                    sel = set(ref)
                    if 0 < ki < i + 1:
                        lo = min(row[j] for j in sel)
                        hi = max(row[j] for j in range(i + 1) if j not in sel)
                        assert lo >= hi


def test_topk_row_zero_always_selects_block_zero():
    w = synth.custom("s", 1, 1, 1, 64 * 8, 16, 8, "fp32")
    s = synth.make_scores_like(w)
    for mode, k, rho in ((1, 1, 0.0), (2, 0, 0.01)):
        c, ix, _ = oracle.select(s, mode, k=k, density=rho)
        assert c[0, 0, 0] == 1 and ix[0, 0, 0, 0] == 0


def test_select_capacity_reports_worst_count():
    w = synth.custom("s", 1, 1, 1, 64 * 16, 16, 8, "fp32")
    s = synth.make_scores_like(w)
    c, ix, worst = oracle.select(s, oracle.MODE_TOPK_K, k=10, cap=4)
    assert worst == 10 and c.max() == 4


def test_pages_topk_sparsity_example():
    g = json.load(open(GOLDEN))["topk_sparsity"]
    nb, k = g["nb"], g["k"]
    # the last causal row has all nb blocks as candidates
    assert oracle.topk_count(nb - 1, oracle.MODE_TOPK_K, k) == k
    assert abs((1 - k / nb) - g["sparsity"]) < 1e-12
    # and the density form gives the same count on that row
    assert oracle.topk_count(nb - 1, oracle.MODE_TOPK_DENSITY, density=1 - g["sparsity"]) == k


def test_pages_gate_size_ratio_and_threshold_example():
    g = json.load(open(GOLDEN))
    B = g["gate_size_ratio"]["block"]
    assert (1.0 / B) ** 2 == g["gate_size_ratio"]["ratio"]
    # a uniform row of length L has scores 1/L; with T = 0.002 rows longer than
    # 500 blocks select nothing and shorter ones select everything.
    T = g["threshold_example"]["T_longbench"]
    nb = 520
    s = torch.tril(torch.ones(nb, nb, dtype=torch.float64))
    s = (s / s.sum(-1, keepdim=True)).float()[None, None]
    c, _, _ = oracle.select(s, oracle.MODE_THRESHOLD, T=T)
    L = np.arange(1, nb + 1)
    expect = np.where(np.float32(1.0) / L.astype(np.float32) > np.float32(T), L, 0)
    # 1/L as fp32 vs T as fp32: the strict comparison of the stored fp32 scores
    sf = s[0, 0].numpy()
    expect = np.array([(i + 1) if sf[i, 0] > np.float32(T) else 0 for i in range(nb)])
    np.testing.assert_array_equal(c[0, 0], expect)
    assert c[0, 0, 498] == 499 and c[0, 0, 500] == 0


# --------------------------------------------------------------- attention --
def _attn_case(B=1, Hq=4, Hkv=2, n=320, d=32, seed=40):
    g = torch.Generator().manual_seed(seed)
    Q = torch.randn(B, Hq, n, d, generator=g)
    K = torch.randn(B, Hkv, n, d, generator=g)
    V = torch.randn(B, Hkv, n, d, generator=g)
    return Q, K, V


def _sdpa(Q, K, V, mask=None, causal=False):
    G = Q.shape[1] // K.shape[1]
    Kr = K.double().repeat_interleave(G, 1)
    Vr = V.double().repeat_interleave(G, 1)
    return F.scaled_dot_product_attention(Q.double(), Kr, Vr, attn_mask=mask, is_causal=causal)


def test_all_ones_mask_equals_dense_causal_sdpa():
    Q, K, V = _attn_case()
    B, Hq, n, d = Q.shape
    counts, idx = oracle.dense_lists(B, Hq, n // BLK)
    O, lse = oracle.sparse_attn(Q, K, V, counts, idx)
    ref = _sdpa(Q, K, V, causal=True).numpy()
    np.testing.assert_allclose(O, ref, rtol=0, atol=1e-12)
    G = Hq // K.shape[1]
    z = Q.double() @ K.double().repeat_interleave(G, 1).transpose(-1, -2) / math.sqrt(d)
    z = z.masked_fill(~torch.tril(torch.ones(n, n, dtype=torch.bool)), float("-inf"))
    np.testing.assert_allclose(lse, torch.logsumexp(z, -1).numpy(), rtol=0, atol=1e-12)


def test_sparse_mask_equals_sdpa_with_block_mask():
    Q, K, V = _attn_case(seed=41)
    B, Hq, n, d = Q.shape
    nb = n // BLK
    w = synth.custom("a", B, Hq, 2, n, d, 8, "fp32")
    s = synth.make_scores_like(w, seed=9)
    counts, idx, _ = oracle.select(s, oracle.MODE_TOPK_DENSITY, density=0.4)
    blockmask = torch.zeros(B, Hq, nb, nb, dtype=torch.bool)
    for h in range(Hq):
        for i in range(nb):
            blockmask[0, h, i, idx[0, h, i, :counts[0, h, i]]] = True
    m = blockmask.repeat_interleave(BLK, 2).repeat_interleave(BLK, 3)
    m &= torch.tril(torch.ones(n, n, dtype=torch.bool))
    O, lse = oracle.sparse_attn(Q, K, V, counts, idx)
    ref = _sdpa(Q, K, V, mask=m).numpy()
    np.testing.assert_allclose(O, ref, rtol=0, atol=1e-12)


def test_dropped_blocks_contribute_nothing():
    Q, K, V = _attn_case(seed=42)
    B, Hq, n, d = Q.shape
    nb = n // BLK
    counts = np.zeros((B, Hq, nb), np.int32)
    idx = np.full((B, Hq, nb, nb), -1, np.int32)
    for i in range(nb):
        lst = [j for j in range(i + 1) if (i + j) % 2 == 0]  # keeps even blocks of even rows...
        counts[0, :, i] = len(lst)
        idx[0, :, i, :len(lst)] = lst
    O1, l1 = oracle.sparse_attn(Q, K, V, counts, idx)
    # every query head of kv head 0 only uses blocks listed for it; poison all
    # blocks of kv heads that no list of that row uses.  Use row 4 only.
    i = 4
    used = set(idx[0, 0, i, :counts[0, 0, i]].tolist())
    K2, V2 = K.clone(), V.clone()
    for j in range(nb):
        if j not in used:
            K2[:, :, j * BLK:(j + 1) * BLK] = float("nan")
            V2[:, :, j * BLK:(j + 1) * BLK] = 1e30
    units = [(0 * Hq + h) * nb + i for h in range(Hq)]
    O2, l2 = oracle.sparse_attn_units(Q, K2, V2, counts, idx, units)
    for u, h in enumerate(range(Hq)):
        np.testing.assert_array_equal(O2[u], O1[0, h, i * BLK:(i + 1) * BLK])
        np.testing.assert_array_equal(l2[u], l1[0, h, i * BLK:(i + 1) * BLK])


def test_single_block_list_and_empty_row():
    Q, K, V = _attn_case(B=1, Hq=1, Hkv=1, n=256, d=16, seed=43)
    nb = 4
    counts = np.array([[[0, 1, 1, 1]]], np.int32)
    idx = np.array([[[[-1], [0], [2], [3]]]], np.int32)
    O, lse = oracle.sparse_attn(Q, K, V, counts, idx)
    assert np.all(O[0, 0, :64] == 0) and np.all(np.isneginf(lse[0, 0, :64]))
    # row 1 attends block 0 only: plain (non-causal) attention over those keys
    ref = F.scaled_dot_product_attention(Q[:, :, 64:128].double(), K[:, :, :64].double(),
                                         V[:, :, :64].double())
    np.testing.assert_allclose(O[0, 0, 64:128], ref[0, 0].numpy(), rtol=0, atol=1e-12)
    # row 3 attends its own block only: causal attention inside the block
    ref = F.scaled_dot_product_attention(Q[:, :, 192:].double(), K[:, :, 192:].double(),
                                         V[:, :, 192:].double(), is_causal=True)
    np.testing.assert_allclose(O[0, 0, 192:], ref[0, 0].numpy(), rtol=0, atol=1e-12)
    assert abs(lse[0, 0, 192] - float(Q[0, 0, 192].double() @ K[0, 0, 192].double()) / 4.0) < 1e-12


def test_lse_merge_of_split_lists():
    Q, K, V = _attn_case(seed=44)
    B, Hq, n, d = Q.shape
    nb = n // BLK
    cA, iA = oracle.dense_lists(B, Hq, nb)
    OA, lA = oracle.sparse_attn(Q, K, V, cA, iA)
    # split every row's list into even and odd blocks
    cE = np.zeros_like(cA); iE = np.full_like(iA, -1)
    cO = np.zeros_like(cA); iO = np.full_like(iA, -1)
    for i in range(nb):
        ev = [j for j in range(i + 1) if j % 2 == 0]
        od = [j for j in range(i + 1) if j % 2 == 1]
        cE[..., i] = len(ev); iE[..., i, :len(ev)] = ev
        cO[..., i] = len(od); iO[..., i, :len(od)] = od
    OE, lE = oracle.sparse_attn(Q, K, V, cE, iE)
    OO, lO = oracle.sparse_attn(Q, K, V, cO, iO)
    lm = np.logaddexp(lE, lO)
    wE = np.exp(lE - lm)[..., None]
    wO = np.exp(lO - lm)[..., None]
    np.testing.assert_allclose(lm, lA, rtol=0, atol=1e-12)
    np.testing.assert_allclose(wE * OE + np.nan_to_num(wO) * OO, OA, rtol=0, atol=1e-12)


def test_gqa_head_mapping():
    Q, K, V = _attn_case(Hq=4, Hkv=2, seed=45)
    counts, idx = oracle.dense_lists(1, 4, Q.shape[2] // BLK)
    O, _ = oracle.sparse_attn(Q, K, V, counts, idx)
    # heads 2,3 must use kv head 1: recompute with kv heads swapped and heads permuted
    O2, _ = oracle.sparse_attn(Q[:, [2, 3, 0, 1]], K[:, [1, 0]], V[:, [1, 0]], counts, idx)
    np.testing.assert_array_equal(O[:, [2, 3, 0, 1]], O2)


# ----------------------------------------------------------------- blockmax --
def test_blockmax_is_maxpool2d_of_causal_softmax():
    Q, K, _ = _attn_case(B=2, Hq=4, Hkv=2, n=320, d=32, seed=50)
    B, Hq, n, d = Q.shape
    gt, lse = oracle.blockmax(Q, K)
    z = Q.double() @ K.double().repeat_interleave(2, 1).transpose(-1, -2) / math.sqrt(d)
    z = z.masked_fill(~torch.tril(torch.ones(n, n, dtype=torch.bool)), float("-inf"))
    P = torch.softmax(z, -1)
    ref = F.max_pool2d(P.reshape(B * Hq, 1, n, n), BLK, BLK).reshape(B, Hq, n // BLK, n // BLK)
    np.testing.assert_allclose(gt, ref.numpy(), rtol=0, atol=1e-15)
    np.testing.assert_allclose(lse, torch.logsumexp(z, -1).numpy(), rtol=0, atol=1e-12)


def test_blockmax_invariants():
    w = synth.custom("b", 1, 2, 1, 512, 32, 8, "bf16", "layer", 8)
    Q, K, _ = synth.make_qkv(w)
    gt, _ = oracle.blockmax(Q, K)
    nb = w.nb
    assert np.all(gt[..., 0, 0] == 1.0)  # token 0 attends only to itself
    assert np.all(gt <= 1.0 + 1e-15) and np.all(gt >= 0)
    iu = np.triu_indices(nb, 1)
    assert np.all(gt[..., iu[0], iu[1]] == 0)
    rowmax = gt.max(-1)
    for i in range(nb):
        assert np.all(rowmax[..., i] >= 1.0 / (64 * i + 1) - 1e-15)
    # units API agrees with the full map
    units = [0 * nb + 3, 1 * nb + 7]
    gu, lu = oracle.blockmax_units(Q, K, units)
    np.testing.assert_array_equal(gu[0], gt[0, 0, 3])
    np.testing.assert_array_equal(gu[1], gt[0, 1, 7])


def test_blockmax_lse_matches_dense_attention_lse():
    Q, K, V = _attn_case(B=1, Hq=2, Hkv=1, n=256, d=16, seed=51)
    _, lse_b = oracle.blockmax(Q, K)
    c, ix = oracle.dense_lists(1, 2, 4)
    _, lse_a = oracle.sparse_attn(Q, K, V, c, ix)
    np.testing.assert_allclose(lse_b, lse_a, rtol=0, atol=1e-12)


# ------------------------------------------------------------ input recipe --
def test_synth_is_deterministic_and_shaped():
    w = synth.WORKLOADS["tiny"]
    a = synth.make_qkv(w)
    b = synth.make_qkv(w)
    for x, y in zip(a, b):
        assert torch.equal(x, y)
    assert a[0].shape == (1, 2, 512, 64) and a[1].shape == (1, 1, 512, 64)
    assert a[0].dtype == torch.float32
    Wq, Wk = synth.make_gate_weights(w)
    assert Wq.shape == (2, 64, 64) and Wk.shape == (1, 64, 192)
    assert abs(Wq.std().item() - 0.02) < 0.002
    w8 = synth.custom("l", 1, 4, 2, 1024, 32, 16, "bf16", "layer", 1)
    Q, K, V = synth.make_qkv(w8)
    assert Q.dtype == torch.bfloat16 and K.shape == (1, 2, 1024, 32)
    # the sink block carries the planted shift: its mean key norm is larger
    kb = K.float().view(1, 2, 16, 64, 32).mean(3).norm(dim=-1)
    assert torch.all(kb[:, :, 0] > 2.0)


def test_unit_subset_entry_points_agree_with_full_ones():
    qt, kt = _gate_inputs(seed=60, B=2, Hq=4, Hkv=2, nb=11, h=8)
    full = oracle.gate_scores(qt, kt, 64)
    units = [0, 5, 11 + 10, 3 * 11 + 7, 8 * 11 - 1]
    rows = oracle.gate_scores_units(qt, kt, 64, units)
    np.testing.assert_array_equal(rows, full.reshape(-1, 11)[units])
    row_i = np.array([u % 11 for u in units])
    for mode, kw in ((oracle.MODE_THRESHOLD, dict(T=0.09)), (oracle.MODE_TOPK_K, dict(k=3)),
                     (oracle.MODE_TOPK_DENSITY, dict(density=0.4))):
        c, ix, _ = oracle.select(full, mode, **kw)
        cr, ir = oracle.select_rows(rows, row_i, mode, **kw)
        np.testing.assert_array_equal(cr, c.reshape(-1)[units])
        for r, u in enumerate(units):
            np.testing.assert_array_equal(ir[r, :cr[r]], ix.reshape(-1, 11)[u, :cr[r]])


# ------------------------------------------- gate distillation (KL) -------
def _gate_torch_chain(Q, K, Wq, Wk):
    """The gate forward as torch fp64 ops (library pooling and softmax), with
    Wq and Wk as leaf tensors for autograd."""
    q = Q.double()
    k = K.double()
    B, Hq, n, d = q.shape
    Hkv = k.shape[1]
    nb = n // 64
    qb = F.avg_pool1d(q.reshape(-1, n, d).transpose(1, 2), 64).transpose(1, 2).reshape(B, Hq, nb, d)
    kt_ = k.reshape(-1, n, d).transpose(1, 2)
    kb = torch.cat([F.max_pool1d(kt_, 64), -F.max_pool1d(-kt_, 64), F.avg_pool1d(kt_, 64)], dim=1)
    kb = kb.transpose(1, 2).reshape(B, Hkv, nb, 3 * d)
    wq = Wq.double().clone().requires_grad_(True)
    wk = Wk.double().clone().requires_grad_(True)
    qt = torch.einsum("hcd,bhid->bhic", wq, qb)
    ktil = torch.einsum("hcd,bhid->bhic", wk, kb)
    ktil = ktil.repeat_interleave(Hq // Hkv, dim=1)
    z = torch.matmul(qt, ktil.transpose(-1, -2)) / math.sqrt(d)
    mask = torch.tril(torch.ones(nb, nb, dtype=torch.bool))
    logp = torch.log_softmax(z.masked_fill(~mask, float("-inf")), dim=-1)
    return logp, mask, wq, wk


def test_gate_kl_gradients_match_autograd():
    """Hand-derived chain rule (oracle) against torch autograd through the
    whole gate on the same inputs, in fp64."""
    w = synth.custom("kl", 2, 4, 2, 8 * 64, 32, 16, "fp32", "layer", 11)
    Q, K, _ = synth.make_qkv(w)
    Wq, Wk = synth.make_gate_weights(w)
    gt, _ = oracle.blockmax(Q, K)
    loss, dWq, dWk = oracle.gate_kl_backward(Q, K, Wq, Wk, gt)
    logp, mask, wq, wk = _gate_torch_chain(Q, K, Wq, Wk)
    g = torch.from_numpy(gt).masked_fill(~mask, 0.0)
    g = g / g.sum(dim=-1, keepdim=True)
    terms = torch.where(g > 0, g * (torch.log(g) - logp.masked_fill(~mask, 0.0)), torch.zeros_like(g))
    tl = terms.sum() / (g.shape[0] * g.shape[1] * g.shape[2])
    tl.backward()
    assert abs(tl.item() - loss) <= 1e-12 * max(1.0, abs(loss))
    np.testing.assert_allclose(dWq, wq.grad.numpy(), rtol=1e-9, atol=1e-15)
    np.testing.assert_allclose(dWk, wk.grad.numpy(), rtol=1e-9, atol=1e-15)


def test_gate_kl_gradient_by_finite_differences():
    """Central differences of the oracle's own loss on a tiny gate."""
    w = synth.custom("klfd", 1, 2, 1, 4 * 64, 16, 8, "fp32", "layer", 13)
    Q, K, _ = synth.make_qkv(w)
    Wq, Wk = synth.make_gate_weights(w)
    Wq = Wq * 20.0   # larger logits so that the loss is not flat
    Wk = Wk * 20.0
    gt, _ = oracle.blockmax(Q, K)
    _, dWq, dWk = oracle.gate_kl_backward(Q, K, Wq, Wk, gt)
    rng = np.random.default_rng(5)
    for W, dW, which in ((Wq, dWq, "q"), (Wk, dWk, "k")):
        for _ in range(6):
            idx = tuple(int(rng.integers(0, s)) for s in W.shape)
            h = 1e-3
            Wp, Wm = W.clone().double(), W.clone().double()
            Wp[idx] += h
            Wm[idx] -= h
            if which == "q":
                lp = oracle.gate_kl_backward(Q, K, Wp, Wk, gt)[0]
                lm = oracle.gate_kl_backward(Q, K, Wm, Wk, gt)[0]
            else:
                lp = oracle.gate_kl_backward(Q, K, Wq, Wp, gt)[0]
                lm = oracle.gate_kl_backward(Q, K, Wq, Wm, gt)[0]
            fd = (lp - lm) / (2 * h)
            # central differences carry an O(h^2) truncation error (~1e-5 relative here)
            assert abs(fd - dW[idx]) <= 1e-4 * max(1e-3, abs(dW[idx])) + 1e-9, (which, idx, fd, dW[idx])


def test_gate_kl_zero_at_match_and_nonnegative():
    w = synth.custom("kl0", 1, 2, 1, 6 * 64, 16, 8, "fp32", "layer", 17)
    Q, K, _ = synth.make_qkv(w)
    Wq, Wk = synth.make_gate_weights(w)
    s = oracle.gate(Q, K, Wq, Wk)
    # gt equal to the score (up to a per-row factor): zero loss, zero gradient
    loss, dz = oracle.gate_kl(s * 3.0, s)
    loss, dz = oracle.gate_kl(s, s * 3.0)
    assert abs(loss) < 1e-14 and np.abs(dz).max() < 1e-15
    gt, _ = oracle.blockmax(Q, K)
    loss, dz = oracle.gate_kl(s, gt)
    assert loss > 0
    # each causal row of dz sums to zero (both rows are distributions)
    assert np.abs(dz.sum(axis=-1)).max() < 1e-15


def test_gate_kl_two_block_closed_form():
    """nb = 2: row 0 has one candidate (loss 0); row 1 is a two-way softmax
    s = (sigmoid(z0 - z1), sigmoid(z1 - z0)) against g = gt / sum(gt)."""
    s = np.zeros((1, 1, 2, 2))
    z0, z1 = 0.3, -0.4
    s[0, 0, 0, 0] = 1.0
    s[0, 0, 1, 0] = 1.0 / (1.0 + math.exp(z1 - z0))
    s[0, 0, 1, 1] = 1.0 / (1.0 + math.exp(z0 - z1))
    gt = np.array([[[[0.7, 0.0], [0.2, 0.6]]]])
    loss, dz = oracle.gate_kl(s, gt)
    g0, g1 = 0.2 / 0.8, 0.6 / 0.8
    row1 = g0 * math.log(g0 / s[0, 0, 1, 0]) + g1 * math.log(g1 / s[0, 0, 1, 1])
    assert abs(loss - row1 / 2) < 1e-15
    assert abs(dz[0, 0, 1, 0] - (s[0, 0, 1, 0] - g0) / 2) < 1e-16
    assert dz[0, 0, 0, 0] == 0.0 and dz[0, 0, 0, 1] == 0.0


# ----------------------------------------------------------- decode stage --
def _decode_inputs(B=2, Hq=4, Hkv=2, n=5 * 64 + 17, d=32, seed=23):
    g = torch.Generator("cpu").manual_seed(seed)
    q = torch.randn(B, Hq, d, generator=g)
    K = torch.randn(B, Hkv, n, d, generator=g)
    V = torch.randn(B, Hkv, n, d, generator=g)
    return q, K, V


def test_decode_attn_all_blocks_is_last_row_of_prefill_attention():
    """Every candidate selected: the token attends to all n keys, which is the
    prefill oracle's causal attention at query position n - 1."""
    B, Hq, Hkv, d, nblk = 2, 4, 2, 32, 6
    n = nblk * 64
    q, K, V = _decode_inputs(B, Hq, Hkv, n, d, 29)
    c = (n - 1) // 64
    counts = np.full((B, Hq), c, np.int32)
    idx = np.tile(np.arange(c, dtype=np.int32), (B, Hq, 1))
    O, lse = oracle.decode_attn(q, K, V, n, counts, idx)
    Qf = torch.zeros(B, Hq, n, d)
    Qf[:, :, n - 1] = q
    cl, il = oracle.dense_lists(B, Hq, nblk)
    Of, lf = oracle.sparse_attn(Qf, K, V, cl, il)
    np.testing.assert_allclose(O, Of[:, :, n - 1], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(lse, lf[:, :, n - 1], rtol=1e-12, atol=1e-12)


def test_decode_attn_subset_matches_sdpa_with_key_mask():
    B, Hq, Hkv, d = 2, 4, 2, 32
    n = 7 * 64 + 9
    q, K, V = _decode_inputs(B, Hq, Hkv, n, d, 31)
    c = (n - 1) // 64
    rng = np.random.default_rng(1)
    counts = np.zeros((B, Hq), np.int32)
    idx = np.full((B, Hq, c), -1, np.int32)
    for b in range(B):
        for h in range(Hq):
            sel = np.sort(rng.choice(c, size=int(rng.integers(0, c + 1)), replace=False))
            counts[b, h] = len(sel)
            idx[b, h, :len(sel)] = sel
    O, _ = oracle.decode_attn(q, K, V, n, counts, idx)
    G = Hq // Hkv
    for b in range(B):
        for h in range(Hq):
            mask = torch.zeros(n, dtype=torch.bool)
            for j in idx[b, h, :counts[b, h]]:
                mask[j * 64:(j + 1) * 64] = True
            mask[c * 64:n] = True
            ref = F.scaled_dot_product_attention(q[b, h].double().view(1, 1, 1, d),
                                                 K[b, h // G].double().view(1, 1, n, d),
                                                 V[b, h // G].double().view(1, 1, n, d),
                                                 attn_mask=mask.view(1, 1, 1, n))
            np.testing.assert_allclose(O[b, h], ref.view(d).numpy(), rtol=1e-12, atol=1e-12)


def test_decode_blockmax_is_maxpool1d_of_softmax():
    B, Hq, Hkv, d = 2, 4, 2, 32
    n = 4 * 64 + 33
    q, K, _ = _decode_inputs(B, Hq, Hkv, n, d, 37)
    gt, lse = oracle.decode_blockmax(q, K, n)
    G = Hq // Hkv
    for b in range(B):
        for h in range(Hq):
            z = (K[b, h // G].double() @ q[b, h].double()) / math.sqrt(d)
            p = torch.softmax(z, dim=0)
            ref = F.max_pool1d(p.view(1, 1, n), 64, ceil_mode=True).view(-1)
            np.testing.assert_allclose(gt[b, h], ref.numpy(), rtol=1e-12, atol=1e-15)
            assert abs(lse[b, h] - torch.logsumexp(z, 0).item()) < 1e-12
    # the block holding the row maximum has the largest entry; every entry <= 1
    assert np.all(gt <= 1.0) and np.all(gt.max(-1) >= 1.0 / n)


def test_decode_gate_is_softmax_over_compressed_cache():
    B, Hq, Hkv, d = 2, 4, 2, 32
    n = 6 * 64 + 5
    q, K, _ = _decode_inputs(B, Hq, Hkv, n, d, 41)
    g = torch.Generator("cpu").manual_seed(43)
    Wk = torch.randn(Hkv, d, 3 * d, generator=g) * 0.05
    c = (n - 1) // 64
    kt = oracle.decode_kcache(K, Wk, c)
    assert kt.shape == (B, Hkv, c, d)
    # the compressed entry of a block is Wk applied to its [max | min | avg]
    blk = K[1, 1, 2 * 64:3 * 64].double()
    feat = torch.cat([blk.max(0).values, blk.min(0).values, blk.mean(0)])
    np.testing.assert_allclose(kt[1, 1, 2], (Wk[1].double() @ feat).numpy(), rtol=1e-12, atol=1e-12)
    s = oracle.decode_gate(q, kt, d)
    G = Hq // Hkv
    for b in range(B):
        for h in range(Hq):
            ref = torch.softmax(torch.from_numpy(kt[b, h // G]) @ q[b, h].double() / math.sqrt(d), 0)
            np.testing.assert_allclose(s[b, h], ref.numpy(), rtol=1e-12, atol=1e-15)
    cnt, ix = oracle.decode_select(s, oracle.MODE_TOPK_DENSITY, density=0.5)
    assert np.all(cnt == math.ceil(0.5 * c))
    cnt, ix = oracle.decode_select(s, oracle.MODE_TOPK_K, k=2)
    for b in range(B):
        for h in range(Hq):
            top = np.argsort(-s[b, h], kind="stable")[:2]
            assert sorted(top.tolist()) == ix[b, h, :2].tolist()


# ------------------------------------------------------- force diagonal ---
def test_force_diagonal_threshold_keeps_only_diagonal_above_all_scores():
    """T above every score: the forced lists are exactly [i]."""
    w = synth.custom("fd", 1, 3, 1, 64 * 10, 32, 8, "fp32")
    s = synth.make_scores_like(w, seed=31)
    cnt, idx, _ = oracle.select(s, oracle.MODE_THRESHOLD, T=2.0, force_diag=True)
    assert np.all(cnt == 1)
    assert np.array_equal(idx[..., 0], np.broadcast_to(np.arange(10), (1, 3, 10)))
    cnt0, _, _ = oracle.select(s, oracle.MODE_THRESHOLD, T=2.0)
    assert np.all(cnt0 == 0)


@pytest.mark.parametrize("mode,kw", [(oracle.MODE_THRESHOLD, dict(T=0.08)), (oracle.MODE_TOPK_K, dict(k=3)),
                                     (oracle.MODE_TOPK_DENSITY, dict(density=0.3))])
def test_force_diagonal_is_selection_plus_diagonal(mode, kw):
    """Forced lists = the mode's own lists (an independent call) with i
    added where it was missing; the worst count follows."""
    w = synth.custom("fd", 2, 2, 1, 64 * 12, 32, 8, "fp32")
    s = synth.make_scores_like(w, seed=32, ties=True)
    c0, i0, _ = oracle.select(s, mode, **kw)
    c1, i1, worst = oracle.select(s, mode, force_diag=True, **kw)
    for r in np.ndindex(c0.shape):
        base = set(i0[r][:c0[r]].tolist())
        forced = i1[r][:c1[r]].tolist()
        assert forced == sorted(base | {r[-1]})
    assert worst == int(c1.max())


# -------------------------------------------------------- varlen packing ---
def test_varlen_single_full_sequence_is_the_plain_gate():
    Q, K = _rand((1, 4, 64 * 7, 16), 71), _rand((1, 2, 64 * 7, 16), 72)
    Wq, Wk = _rand((4, 8, 16), 73, 0.3), _rand((2, 8, 48), 74, 0.3)
    ref = oracle.gate(Q, K, Wq, Wk)
    got = oracle.gate_varlen(Q, K, Wq, Wk, [0], [64 * 7])
    np.testing.assert_allclose(got, ref, rtol=0, atol=1e-13)


def test_varlen_partial_block_pooling_is_ceil_mode_pooling():
    """A sequence of 150 tokens: the last block pools its 22 tokens only,
    as avg/max pooling with ceil_mode on the unpadded sequence does."""
    X = _rand((1, 2, 64 * 5, 8), 75)
    a, l = 128, 150
    x = X[:, :, a:a + l].double().reshape(2, l, 8).transpose(1, 2)
    av = F.avg_pool1d(x, BLK, BLK, ceil_mode=True).transpose(1, 2).reshape(1, 2, 3, 8).numpy()
    mx = F.max_pool1d(x, BLK, BLK, ceil_mode=True).transpose(1, 2).reshape(1, 2, 3, 8).numpy()
    mn = -F.max_pool1d(-x, BLK, BLK, ceil_mode=True).transpose(1, 2).reshape(1, 2, 3, 8).numpy()
    np.testing.assert_allclose(oracle.pool_varlen(X, a, l, False), av, rtol=0, atol=1e-14)
    kp = oracle.pool_varlen(X, a, l, True)
    np.testing.assert_array_equal(kp[..., :8], mx)
    np.testing.assert_array_equal(kp[..., 8:16], mn)
    np.testing.assert_allclose(kp[..., 16:], av, rtol=0, atol=1e-14)


def test_varlen_packed_sequence_equals_the_gate_on_it_alone():
    """Two sequences with a gap: the second one's block of the packed scores
    equals the plain gate run on that sequence cut out of the buffer, and
    nothing crosses between sequences."""
    starts, n = synth.varlen_layout([200, 256], [0, 1])
    Q, K = _rand((1, 4, n, 16), 76), _rand((1, 2, n, 16), 77)
    Wq, Wk = _rand((4, 8, 16), 78, 0.3), _rand((2, 8, 48), 79, 0.3)
    s = oracle.gate_varlen(Q, K, Wq, Wk, starts, [200, 256])
    a = starts[1]
    alone = oracle.gate(Q[:, :, a:a + 256].contiguous(), K[:, :, a:a + 256].contiguous(), Wq, Wk)
    f = a // BLK
    np.testing.assert_allclose(s[:, :, f:f + 4, f:f + 4], alone, rtol=0, atol=1e-13)
    assert np.all(s[:, :, f:, :f] == 0) and np.all(s[:, :, :f, f:] == 0)
    assert np.all(s[:, :, 4, :] == 0)  # the gap block
    # the first sequence's rows sum to one over its own blocks
    np.testing.assert_allclose(s[:, :, :4, :4].sum(-1), 1.0, rtol=0, atol=1e-12)


def test_varlen_rope_depends_on_block_distance_only():
    """Block RoPE scores at packed (global) positions equal those at the
    sequence's own positions: the rotation leaves q~_i . k~_j a function of
    i - j.  (The CUDA gate rotates at global positions.)"""
    h = 8
    q = _rand((1, 1, 12, h), 80)
    k = _rand((1, 1, 12, h), 81)
    g_q, g_k = oracle.block_rope(q, 5000.0), oracle.block_rope(k, 5000.0)
    l_q, l_k = oracle.block_rope(q[:, :, 5:].contiguous(), 5000.0), oracle.block_rope(k[:, :, 5:].contiguous(), 5000.0)
    np.testing.assert_allclose(g_q[0, 0, 5:] @ g_k[0, 0, 5:].T, l_q[0, 0] @ l_k[0, 0].T, rtol=0, atol=1e-12)


def test_varlen_attention_is_causal_sdpa_per_sequence():
    """Every block listed: each packed sequence (lengths 150 and 64, a gap
    between them) gets causal attention over its own tokens only."""
    lens = [150, 64]
    starts, n = synth.varlen_layout(lens, [0, 1])
    Q, K, V = _attn_case(n=n, d=16, seed=82)
    nb = n // BLK
    s = np.zeros((1, 4, nb, nb))
    for a, l in zip(starts, lens):
        f, nbs = a // BLK, (l + BLK - 1) // BLK
        s[:, :, f:f + nbs, f:f + nbs] = np.tril(np.ones((nbs, nbs)))
    cnt, idx = oracle.select_varlen(s, starts, lens, oracle.MODE_THRESHOLD, T=0.5)
    O, lse = oracle.sparse_attn_varlen(Q, K, V, cnt, idx, starts, lens)
    for a, l in zip(starts, lens):
        ref = _sdpa(Q[:, :, a:a + l], K[:, :, a:a + l], V[:, :, a:a + l], causal=True).numpy()
        np.testing.assert_allclose(O[:, :, a:a + l], ref, rtol=0, atol=1e-12)
    assert np.isnan(O[:, :, 150:192]).all()  # padding and gap are not defined
