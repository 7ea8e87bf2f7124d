"""GPU parity of the decode stage (compressed K cache, token gate, block-sparse
decode attention, 1D ground truth) against the fp64 oracle, through the C ABI.

Tolerances (all fp32 arithmetic on the GPU, no tensor cores):
  * k~ cache: 1e-5 of the largest |k~| (fp32 pooling and a 3d-term dot).
  * scores: SCORE_RTOL of the row's largest score; index lists bit-exact when
    the oracle's selection is fed the GPU's fp32 scores.
  * O and LSE: the bf16 I/O bounds of the prefill path (O is rounded to the
    cache dtype on output); fp32 caches get 1e-4 on LSE.
  * gt: BMAX_TOL absolute.
"""
import numpy as np
import pytest
import torch

import learned_block_sparse_seer_b200 as seer
import oracle
from learned_block_sparse_seer_b200 import synth

from gpu_common import BMAX_TOL, LSE_TOL, SCORE_RTOL, check_o

pytestmark = pytest.mark.gpu

MODES = [(seer.SELECT_THRESHOLD, dict(T=0.02)), (seer.SELECT_TOPK_K, dict(k=3)),
         (seer.SELECT_TOPK_DENSITY, dict(density=0.3))]


def _case(B, Hq, Hkv, nb, d, dtype, seq_len, seed=5):
    w = synth.custom("dec", B, Hq, Hkv, 64 * nb, d, d, dtype, "decode", seed)
    q, Kc, Vc = synth.make_decode(w, seq_len)
    _, Wk = synth.make_gate_weights(w)
    return w, q, Kc, Vc, Wk


def _kt(Kc, Wk, c):
    kt = seer.seer_decode_kcache_update(Kc.cuda(), Wk.cuda(), 0, c)
    return kt


@pytest.mark.parametrize("dtype,d", [("fp32", 64), ("bf16", 128), ("bf16", 64)])
def test_kcache(dtype, d):
    w, q, Kc, Vc, Wk = _case(2, 4, 2, 9, d, dtype, 64 * 7 + 5)
    c = 7
    kt = _kt(Kc, Wk, c).cpu().double().numpy()
    ref = oracle.decode_kcache(Kc, Wk, c)
    tol = 1e-5 * np.abs(ref).max()
    assert np.abs(kt[:, :, :c] - ref).max() <= tol
    assert np.all(kt[:, :, c:] == 0), "blocks outside the range were written"
    # incremental updates give the same cache
    Kd, Wd = Kc.cuda(), Wk.cuda()
    kt2 = torch.zeros(2, 2, 9, d, dtype=torch.float32, device="cuda")
    for a, b in ((0, 3), (3, 3), (3, 7)):
        seer.seer_decode_kcache_update(Kd, Wd, a, b, kt2)
    assert torch.equal(kt2.cpu(), torch.from_numpy(kt).float())


def test_kcache_rejects():
    w, q, Kc, Vc, Wk = _case(1, 2, 1, 4, 64, "fp32", 200)
    with pytest.raises(seer.SeerError):
        seer.seer_decode_kcache_update(Kc.cuda(), Wk.cuda(), 2, 5)  # past the capacity
    with pytest.raises(seer.SeerError):  # h != d
        seer.seer_decode_kcache_update(Kc.cuda(), Wk[:, :32].contiguous().cuda(), 0, 1)


@pytest.mark.parametrize("mode,kw", MODES)
@pytest.mark.parametrize("dtype,d,nb,seq_len,Hq,Hkv", [("fp32", 64, 12, 64 * 11 + 1, 8, 2), ("bf16", 128, 20, 64 * 20, 8, 2),
                                                        ("bf16", 128, 40, 64 * 33 + 17, 8, 2),
                                                        ("bf16", 64, 300, 64 * 290 + 3, 6, 2),
                                                        ("fp32", 128, 50, 64 * 45, 4, 2)])
def test_gate(mode, kw, dtype, d, nb, seq_len, Hq, Hkv):
    w, q, Kc, Vc, Wk = _case(2, Hq, Hkv, nb, d, dtype, seq_len)
    c = (seq_len - 1) // 64
    kt = _kt(Kc, Wk, c)
    counts, idx, scores = seer.seer_decode_gate(q.cuda(), kt, w.n, seq_len, mode, return_scores=True, **kw)
    s = scores.cpu().double().numpy()
    s_ref = oracle.decode_gate(q, oracle.decode_kcache(Kc, Wk, c), d)
    err = np.abs(s - s_ref).max(axis=-1) / s_ref.max(axis=-1)
    assert err.max() <= SCORE_RTOL
    # bit-exact lists on the GPU's own scores
    cnt_ref, idx_ref = oracle.decode_select(scores.cpu(), mode, **kw)
    cnt = counts.cpu().numpy()
    ix = idx.cpu().numpy()
    assert np.array_equal(cnt, cnt_ref)
    for r in np.ndindex(cnt.shape):
        assert np.array_equal(ix[r][:cnt[r]], idx_ref[r][:cnt[r]])


@pytest.mark.parametrize("seq_len", [1, 40, 64])
def test_gate_no_candidates(seq_len):
    """The token's own block is the only one: every count is 0."""
    w, q, Kc, Vc, Wk = _case(1, 4, 2, 2, 64, "bf16", seq_len)
    kt = torch.zeros(1, 2, 2, 64, dtype=torch.float32, device="cuda")
    counts, idx = seer.seer_decode_gate(q.cuda(), kt, w.n, seq_len, seer.SELECT_TOPK_K, k=4)
    assert counts.cpu().eq(0).all()


def _attn_ref(q, Kc, Vc, seq_len, counts, idx):
    return oracle.decode_attn(q, Kc, Vc, seq_len, counts.cpu().numpy(), idx.cpu().numpy())


@pytest.mark.parametrize("dtype,d,nb,seq_len", [("fp32", 64, 10, 64 * 9 + 3), ("bf16", 128, 24, 64 * 24),
                                                ("bf16", 64, 30, 64 * 17 + 63), ("bf16", 128, 3, 5)])
def test_attn_selected(dtype, d, nb, seq_len):
    w, q, Kc, Vc, Wk = _case(2, 8, 2, nb, d, dtype, seq_len)
    c = (seq_len - 1) // 64
    kt = _kt(Kc, Wk, c)
    counts, idx = seer.seer_decode_gate(q.cuda(), kt, w.n, seq_len, seer.SELECT_TOPK_DENSITY, density=0.4)
    ws = torch.empty(seer.sparse_decode_attn_workspace_size(2, 8, 2, w.n, d), dtype=torch.uint8, device="cuda")
    O, lse = seer.seer_sparse_decode_attn(q.cuda(), Kc.cuda(), Vc.cuda(), seq_len, counts, idx, workspace=ws)
    assert seer.seer_workspace_status(ws) == 0
    O_ref, lse_ref = _attn_ref(q, Kc, Vc, seq_len, counts, idx)
    check_o(O.cpu().double().numpy(), O_ref)
    tol = 1e-4 if dtype == "fp32" else LSE_TOL
    assert np.abs(lse.cpu().double().numpy() - lse_ref).max() <= tol


def test_attn_repeat_same_workspace():
    """Back-to-back calls on one workspace give identical results (the
    per-row merge tickets are left at zero)."""
    w, q, Kc, Vc, Wk = _case(2, 8, 2, 40, 128, "bf16", 64 * 39 + 11)
    seq_len = 64 * 39 + 11
    kt = _kt(Kc, Wk, 39)
    counts, idx = seer.seer_decode_gate(q.cuda(), kt, w.n, seq_len, seer.SELECT_TOPK_K, k=9)
    ws = torch.empty(seer.sparse_decode_attn_workspace_size(2, 8, 2, w.n, 128), dtype=torch.uint8, device="cuda")
    qd, Kd, Vd = q.cuda(), Kc.cuda(), Vc.cuda()
    O1, l1 = seer.seer_sparse_decode_attn(qd, Kd, Vd, seq_len, counts, idx, workspace=ws)
    O2, l2 = seer.seer_sparse_decode_attn(qd, Kd, Vd, seq_len, counts, idx, workspace=ws)
    assert torch.equal(O1, O2) and torch.equal(l1, l2)
    gws = torch.empty(seer.decode_blockmax_workspace_size(2, 8, 2, w.n, 128), dtype=torch.uint8, device="cuda")
    g1, _ = seer.seer_decode_blockmax(qd, Kd, seq_len, workspace=gws)
    g2, _ = seer.seer_decode_blockmax(qd, Kd, seq_len, workspace=gws)
    assert torch.equal(g1, g2)


def test_attn_all_candidates_is_dense():
    """Every complete block listed: the result is the token's full causal
    attention (blockmax's LSE is the same row statistic)."""
    w, q, Kc, Vc, Wk = _case(1, 4, 1, 16, 128, "bf16", 64 * 15 + 9)
    seq_len = 64 * 15 + 9
    c = 15
    counts = torch.full((1, 4), c, dtype=torch.int32, device="cuda")
    idx = torch.arange(c, dtype=torch.int32, device="cuda").repeat(1, 4, 1).contiguous()
    O, lse = seer.seer_sparse_decode_attn(q.cuda(), Kc.cuda(), Vc.cuda(), seq_len, counts, idx)
    O_ref, lse_ref = _attn_ref(q, Kc, Vc, seq_len, counts, idx)
    check_o(O.cpu().double().numpy(), O_ref)
    _, lse_full = oracle.decode_blockmax(q, Kc, seq_len)
    assert np.abs(lse.cpu().double().numpy() - lse_full).max() <= LSE_TOL


def test_attn_empty_lists():
    """Counts 0: only the token's own block is attended."""
    w, q, Kc, Vc, Wk = _case(2, 4, 2, 8, 64, "fp32", 64 * 6 + 10)
    seq_len = 64 * 6 + 10
    counts = torch.zeros(2, 4, dtype=torch.int32, device="cuda")
    idx = torch.zeros(2, 4, 1, dtype=torch.int32, device="cuda")
    O, lse = seer.seer_sparse_decode_attn(q.cuda(), Kc.cuda(), Vc.cuda(), seq_len, counts, idx)
    O_ref, lse_ref = _attn_ref(q, Kc, Vc, seq_len, counts, idx)
    check_o(O.cpu().double().numpy(), O_ref)
    assert np.abs(lse.cpu().double().numpy() - lse_ref).max() <= 1e-4


def test_attn_bad_list_recorded():
    """A count above the capacity and an entry at the token's own block are
    clamped by the kernel's checks and reported in the workspace status."""
    w, q, Kc, Vc, Wk = _case(1, 2, 1, 8, 64, "bf16", 64 * 7 + 1)
    seq_len = 64 * 7 + 1
    counts = torch.tensor([[9, 1]], dtype=torch.int32, device="cuda")
    idx = torch.tensor([[[0, 1, 2, 3], [7, 0, 0, 0]]], dtype=torch.int32, device="cuda")
    ws = torch.empty(seer.sparse_decode_attn_workspace_size(1, 2, 1, w.n, 64), dtype=torch.uint8, device="cuda")
    seer.seer_sparse_decode_attn(q.cuda(), Kc.cuda(), Vc.cuda(), seq_len, counts, idx, workspace=ws)
    assert seer.seer_workspace_status(ws) == 6  # SEER_ERR_DEVICE_CHECK


@pytest.mark.parametrize("dtype,d,nb,seq_len,Hq,Hkv", [("fp32", 64, 6, 64 * 5 + 7, 8, 4), ("bf16", 128, 20, 64 * 20, 8, 2),
                                                        ("bf16", 64, 9, 33, 8, 4), ("bf16", 128, 70, 64 * 67 + 5, 6, 2),
                                                        ("fp32", 128, 12, 64 * 11 + 30, 3, 3)])
def test_blockmax(dtype, d, nb, seq_len, Hq, Hkv):
    w, q, Kc, Vc, Wk = _case(2, Hq, Hkv, nb, d, dtype, seq_len)
    gt, lse = seer.seer_decode_blockmax(q.cuda(), Kc.cuda(), seq_len)
    gt_ref, lse_ref = oracle.decode_blockmax(q, Kc, seq_len)
    assert gt.shape[-1] == (seq_len - 1) // 64 + 1
    assert np.abs(gt.cpu().double().numpy() - gt_ref).max() <= BMAX_TOL
    assert np.abs(lse.cpu().double().numpy() - lse_ref).max() <= LSE_TOL


def test_decode128k_sampled():
    """The 128k-token cache of the layer's heads, in the launch configuration
    the bench times: the full k~ cache, the density-0.1 gate, the sparse
    attention and the ground truth, each checked on sampled KV heads."""
    w = synth.WORKLOADS["decode128k"]
    seq_len = synth.decode_seq_len(w)
    q, Kc, Vc = synth.make_decode(w, seq_len)
    _, Wk = synth.make_gate_weights(w)
    c = (seq_len - 1) // 64
    qd, Kd, Vd = q.cuda(), Kc.cuda(), Vc.cuda()
    kt = seer.seer_decode_kcache_update(Kd, Wk.cuda(), 0, c)
    counts, idx, scores = seer.seer_decode_gate(qd, kt, w.n, seq_len, seer.SELECT_TOPK_DENSITY, density=0.1,
                                                return_scores=True)
    O, lse = seer.seer_sparse_decode_attn(qd, Kd, Vd, seq_len, counts, idx)
    gt, glse = seer.seer_decode_blockmax(qd, Kd, seq_len)
    torch.cuda.synchronize()
    G = w.G
    for g in (0, w.Hkv - 1):
        heads = slice(g * G, (g + 1) * G)
        kt_ref = oracle.decode_kcache(Kc[:, g:g + 1], Wk[g:g + 1], c)
        kt_g = kt[:, g:g + 1, :c].cpu().double().numpy()
        assert np.abs(kt_g - kt_ref).max() <= 1e-5 * np.abs(kt_ref).max()
        s_ref = oracle.decode_gate(q[:, heads], kt_ref, w.d)
        s = scores[:, heads].cpu().double().numpy()
        assert (np.abs(s - s_ref).max(axis=-1) / s_ref.max(axis=-1)).max() <= SCORE_RTOL
        cnt_ref, idx_ref = oracle.decode_select(scores[:, heads].cpu(), seer.SELECT_TOPK_DENSITY, density=0.1)
        cnt = counts[:, heads].cpu().numpy()
        ix = idx[:, heads].cpu().numpy()
        assert np.array_equal(cnt, cnt_ref)
        for r in np.ndindex(cnt.shape):
            assert np.array_equal(ix[r][:cnt[r]], idx_ref[r][:cnt[r]])
        O_ref, lse_ref = oracle.decode_attn(q[:, heads], Kc[:, g:g + 1], Vc[:, g:g + 1], seq_len, cnt, ix)
        check_o(O[:, heads].cpu().double().numpy(), O_ref)
        assert np.abs(lse[:, heads].cpu().double().numpy() - lse_ref).max() <= LSE_TOL
        gt_ref, glse_ref = oracle.decode_blockmax(q[:, heads], Kc[:, g:g + 1], seq_len)
        assert np.abs(gt[:, heads].cpu().double().numpy() - gt_ref).max() <= BMAX_TOL
        assert np.abs(glse[:, heads].cpu().double().numpy() - glse_ref).max() <= LSE_TOL
