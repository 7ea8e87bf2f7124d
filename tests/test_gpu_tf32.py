"""GPU parity of the tf32 attention path (seer_sparse_attn_tf32: fp32 Q/K/V
read by the tensor cores as tf32) against the fp64 oracle on the unrounded
fp32 inputs, through the C ABI.

Tolerances, derived per case from the inputs.  The tensor core keeps 10
mantissa bits of each fp32 operand (relative error below 2^-10 per operand,
against 2^-8 for the bf16 path's rounding), so a logit moves by at most
delta = 2^-9 * scale * max_(t,s) sum_c |q_tc k_sc|.  The LSE is 1-Lipschitz
in the logits: |dLSE| <= delta (+ fp32 summation, far smaller).  O moves by
at most about (2 delta + 2^-9) * max|v| (the probabilities' relative change,
then P and V each rounded to tf32).  Mean O error: a tenth of its bound.
Each case also runs the bf16 path on the same inputs and requires the tf32
path's error to be the smaller one.
"""
import numpy as np
import pytest
import torch

import learned_block_sparse_seer_b200 as seer
import oracle
from learned_block_sparse_seer_b200 import synth

pytestmark = pytest.mark.gpu



def _bounds(Q, K, V):
    """(O max, O mean, LSE max) tolerances of the tf32 path for these inputs."""
    q, k, v = Q.double(), K.double(), V.double()
    G = q.shape[1] // k.shape[1]
    kr = k.abs().repeat_interleave(G, 1)
    worst = (q.abs() @ kr.transpose(-1, -2)).max().item()
    delta = 2.0 ** -9 * worst / np.sqrt(q.shape[-1])
    vmax = v.abs().max().item()
    o_max = (2 * delta + 2.0 ** -9) * vmax
    return o_max, o_max / 10, delta * 1.01 + 1e-6


def _lists(w, mode="density", density=0.4, seed=3):
    s = synth.make_scores_like(w, seed=seed)
    if mode == "dense":
        return oracle.dense_lists(w.B, w.Hq, w.nb)
    c, ix, _ = oracle.select(s, oracle.MODE_TOPK_DENSITY, density=density)
    return c, ix


def _run_both(Q, K, V, c, ix):
    cd = torch.from_numpy(np.ascontiguousarray(c)).cuda()
    idd = torch.from_numpy(np.ascontiguousarray(ix)).cuda()
    Qd, Kd, Vd = Q.cuda(), K.cuda(), V.cuda()
    B, Hq, n, d = Q.shape
    ws = torch.empty(seer.sparse_attn_tf32_workspace_size(B, Hq, K.shape[1], n, d), dtype=torch.uint8, device="cuda")
    O, lse = seer.seer_sparse_attn_tf32(Qd, Kd, Vd, cd, idd, workspace=ws)
    assert seer.seer_workspace_status(ws) == 0
    Ob, lseb = seer.seer_sparse_attn(Qd, Kd, Vd, cd, idd)  # fp32 in, bf16 tensor cores
    return O.cpu().double().numpy(), lse.cpu().double().numpy(), Ob.cpu().double().numpy(), lseb.cpu().double().numpy()


def _check(Q, K, V, c, ix):
    O_MAX, O_MEAN, LSE_MAX = _bounds(Q, K, V)
    O, lse, Ob, lseb = _run_both(Q, K, V, c, ix)
    O_ref, lse_ref = oracle.sparse_attn(Q, K, V, c, ix)
    fin = np.isfinite(lse_ref)
    assert np.array_equal(np.isfinite(lse), fin)
    eo, el = np.abs(O - O_ref), np.abs(lse[fin] - lse_ref[fin])
    assert eo.max() <= O_MAX and eo.mean() <= O_MEAN, (eo.max(), eo.mean(), O_MAX)
    assert el.max() <= LSE_MAX, (el.max(), LSE_MAX)
    # more precise than the bf16 path on the same inputs
    assert eo.mean() < np.abs(Ob - O_ref).mean()
    assert el.max() < np.abs(lseb[fin] - lse_ref[fin]).max()
    return eo, el


def test_tiny_threshold_lists():
    """The tiny workload (fp32) with the oracle gate's threshold lists."""
    w = synth.WORKLOADS["tiny"]
    Q, K, V = synth.make_qkv(w)
    Wq, Wk = synth.make_gate_weights(w)
    c, ix, _ = oracle.select(oracle.gate(Q, K, Wq, Wk), oracle.MODE_THRESHOLD, T=5e-4)
    _check(Q, K, V, c, ix)


@pytest.mark.parametrize("B,Hq,Hkv,nb,d,mode", [(2, 4, 2, 5, 128, "density"), (1, 4, 1, 7, 64, "density"),
                                                 (1, 2, 2, 16, 128, "dense"), (1, 6, 2, 9, 64, "dense")])
def test_shapes(B, Hq, Hkv, nb, d, mode):
    w = synth.custom("tf", B, Hq, Hkv, 64 * nb, d, 16, "fp32", "layer", 17)
    Q, K, V = synth.make_qkv(w)
    c, ix = _lists(w, mode)
    _check(Q, K, V, c, ix)


def test_rescale_path():
    """A key block far above the first one forces the lazy rescale of O^T
    (the running maximum rises by more than 2^8)."""
    w = synth.custom("tf", 1, 2, 1, 64 * 6, 64, 16, "fp32", "layer", 19)
    Q, K, V = synth.make_qkv(w)
    K = K.clone()
    K[:, :, 64 * 4:64 * 5] *= 12.0  # block 4: scores up to ~100x larger
    c, ix = oracle.dense_lists(1, 2, 6)
    _check(Q, K, V, c, ix)


def test_empty_rows_and_bad_entry():
    w = synth.custom("tf", 1, 2, 1, 64 * 4, 64, 16, "fp32", "layer", 21)
    Q, K, V = synth.make_qkv(w)
    c = np.array([[[1, 0, 2, 0], [0, 1, 1, 3]]], dtype=np.int32)
    ix = np.array([[[[0, -1, -1], [-1, -1, -1], [0, 2, -1], [-1, -1, -1]],
                    [[-1, -1, -1], [1, -1, -1], [2, -1, -1], [0, 1, 3]]]], dtype=np.int32)
    O_MAX, _, LSE_MAX = _bounds(Q, K, V)
    O, lse, _, _ = _run_both(Q, K, V, c, ix)
    O_ref, lse_ref = oracle.sparse_attn(Q, K, V, c, ix)
    assert np.all(O[0, 0, 64:128] == 0) and np.all(lse[0, 0, 64:128] == -np.inf)
    fin = np.isfinite(lse_ref)
    assert np.abs(O - O_ref).max() <= O_MAX
    assert np.abs(lse[fin] - lse_ref[fin]).max() <= LSE_MAX
    # an entry past the diagonal is recorded as a device check
    ix2 = ix.copy()
    ix2[0, 0, 2, 1] = 3
    ws = torch.empty(seer.sparse_attn_tf32_workspace_size(1, 2, 1, 256, 64), dtype=torch.uint8, device="cuda")
    seer.seer_sparse_attn_tf32(Q.cuda(), K.cuda(), V.cuda(), torch.from_numpy(c).cuda(), torch.from_numpy(ix2).cuda(),
                               workspace=ws)
    assert seer.seer_workspace_status(ws) == 6


def test_layer8k_sampled():
    """The 8k layer (bf16 values held in fp32, so only P and the arithmetic
    round): sampled units against the oracle, density-0.1 lists."""
    w = synth.WORKLOADS["layer8k"]
    Q, K, V = (t.float() for t in synth.make_qkv(w))
    c, ix = _lists(w, "density", density=0.1, seed=8)
    cd = torch.from_numpy(c).cuda()
    idd = torch.from_numpy(ix).cuda()
    O, lse = seer.seer_sparse_attn_tf32(Q.cuda(), K.cuda(), V.cuda(), cd, idd)
    units = np.array([0, 127, 128 * 5 + 64, 128 * 17 + 127, 128 * 31 + 100], dtype=np.int64)
    O_u, lse_u = oracle.sparse_attn_units(Q, K, V, c, ix, units)
    Of = O.cpu().double().numpy().reshape(-1, 64, w.d)
    lf = lse.cpu().double().numpy().reshape(-1, 64)
    for k, u in enumerate(units):
        hq, i = divmod(int(u), w.nb)
        g = hq // w.G
        # this unit's bounds: its 64 query rows against every key of its KV head
        O_MAX, _, LSE_MAX = _bounds(Q[:, hq:hq + 1, 64 * i:64 * (i + 1)], K[:, g:g + 1], V[:, g:g + 1])
        assert np.abs(Of[u] - O_u[k]).max() <= O_MAX
        assert np.abs(lf[u] - lse_u[k]).max() <= LSE_MAX


def _unit_bounds(Q, K, V, b, hq, g, i, keys):
    """Per-unit tolerances over the keys the unit attends (the bound of
    _bounds restricted to those keys)."""
    q = Q[b, hq, 64 * i:64 * (i + 1)].double()
    k = K[b, g, keys].double()
    v = V[b, g, keys].double()
    worst = (q.abs() @ k.abs().T).max().item()
    delta = 2.0 ** -9 * worst / np.sqrt(q.shape[-1])
    o_max = (2 * delta + 2.0 ** -9) * v.abs().max().item()
    return o_max, delta * 1.01 + 1e-6


def test_layer128k_sampled_bench_config():
    """The 128k layer as the bench times it: the gate's density-0.1 lists of
    the bf16 layer, the layer's values held in fp32, one full-size launch;
    sampled units (first and last query blocks of the first and last heads,
    plus seeded random ones) against the oracle."""
    from gpu_common import inputs, sample_units, to_dev
    w, Q, K, V, Wq, Wk = inputs("layer128k")
    Qd, Kd, Wqd, Wkd = to_dev(Q, K, Wq, Wk)
    cd, idd = seer.seer_gate(Qd, Kd, Wqd, Wkd, "density", density=0.1)
    del Qd, Kd
    c, ix = cd.cpu().numpy(), idd.cpu().numpy()
    Qf, Kf, Vf = Q.float(), K.float(), V.float()
    ws = torch.empty(seer.sparse_attn_tf32_workspace_size(w.B, w.Hq, w.Hkv, w.n, w.d), dtype=torch.uint8,
                     device="cuda")
    O, lse = seer.seer_sparse_attn_tf32(Qf.cuda(), Kf.cuda(), Vf.cuda(), cd, idd, workspace=ws)
    assert seer.seer_workspace_status(ws) == 0
    units = sample_units(w.B, w.Hq, w.nb, 12, seed=128)
    O_u, lse_u = oracle.sparse_attn_units(Qf, Kf, Vf, c, ix, units)
    Of = O.cpu().double().numpy().reshape(-1, 64, w.d)
    lf = lse.cpu().double().numpy().reshape(-1, 64)
    cf = c.reshape(-1)
    ixf = ix.reshape(-1, ix.shape[-1])
    for k, u in enumerate(units):
        bh, i = divmod(int(u), w.nb)
        b, hq = divmod(bh, w.Hq)
        blocks = ixf[u, :cf[u]]
        keys = torch.from_numpy((blocks[:, None] * 64 + np.arange(64)[None, :]).reshape(-1))
        O_MAX, LSE_MAX = _unit_bounds(Qf, Kf, Vf, b, hq, hq // w.G, i, keys)
        assert np.abs(Of[u] - O_u[k]).max() <= O_MAX, (u, np.abs(Of[u] - O_u[k]).max(), O_MAX)
        assert np.abs(lf[u] - lse_u[k]).max() <= LSE_MAX, (u, np.abs(lf[u] - lse_u[k]).max(), LSE_MAX)
