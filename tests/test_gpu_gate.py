"""GPU parity of seer_gate / seer_gate_select against the fp64 oracle, called
through the C ABI (via the ctypes binding)."""
import math

import numpy as np
import pytest
import torch

import learned_block_sparse_seer_b200 as seer
import oracle
from learned_block_sparse_seer_b200 import synth

from gpu_common import SCORE_RTOL, inputs, lists_equal, to_dev

pytestmark = pytest.mark.gpu


def _gate_case(name, mode, **sel):
    w, Q, K, V, Wq, Wk = inputs(name)
    Qd, Kd, Wqd, Wkd = to_dev(Q, K, Wq, Wk)
    counts, idx, scores = seer.seer_gate(Qd, Kd, Wqd, Wkd, mode, return_scores=True, **sel)
    torch.cuda.synchronize()
    return w, Q, K, Wq, Wk, counts.cpu().numpy(), idx.cpu().numpy(), scores.cpu()


def _check_scores(scores_gpu, s_ref):
    sg = scores_gpu.double().numpy()
    rowmax = s_ref.max(-1, keepdims=True)
    err = np.abs(sg - s_ref) / np.maximum(rowmax, 1e-300)
    assert err.max() <= SCORE_RTOL, f"score error {err.max():.2e}"
    nb = s_ref.shape[-1]
    iu = np.triu_indices(nb, 1)
    assert np.all(sg[..., iu[0], iu[1]] == 0.0)


def _check_threshold_vs_fp64(c_gpu, i_gpu, s_ref, T):
    """GPU decisions (fp32 scores) may differ from the fp64 oracle's only where
    the score lies within 1e-3 relative of T."""
    B, H, nb, _ = s_ref.shape
    for b, h, i in np.ndindex(B, H, nb):
        sel = set(i_gpu[b, h, i, :c_gpu[b, h, i]].tolist())
        ref = set(np.nonzero(s_ref[b, h, i, :i + 1] > T)[0].tolist())
        for j in sel ^ ref:
            assert abs(s_ref[b, h, i, j] - T) <= 1e-3 * T, (b, h, i, j, s_ref[b, h, i, j])


@pytest.mark.parametrize("name", ["tiny", "layer8k"])
def test_gate_threshold_matches_oracle(name):
    T = 5e-4
    w, Q, K, Wq, Wk, c, ix, sc = _gate_case(name, "threshold", T=T)
    s_ref = oracle.gate(Q, K, Wq, Wk)
    _check_scores(sc, s_ref)
    # bit-exact against the oracle's selection on the same fp32 scores
    c_ref, i_ref, _ = oracle.select(sc, oracle.MODE_THRESHOLD, T=T)
    lists_equal(c, ix, c_ref, i_ref)
    _check_threshold_vs_fp64(c, ix, s_ref, T)


def test_gate_topk_density_32k():
    w, Q, K, Wq, Wk, c, ix, sc = _gate_case("layer32k", "density", density=0.1)
    s_ref = oracle.gate(Q, K, Wq, Wk)
    _check_scores(sc, s_ref)
    c_ref, i_ref, _ = oracle.select(sc, oracle.MODE_TOPK_DENSITY, density=0.1, cap=ix.shape[-1])
    lists_equal(c, ix, c_ref, i_ref)
    # against the fp64 scores: any differing choice is a near-tie at the k-th score
    B, H, nb, _ = s_ref.shape
    rng = np.random.default_rng(1)
    for h, i in zip(rng.integers(0, H, 200), rng.integers(0, nb, 200)):
        row = s_ref[0, h, i, :i + 1]
        ki = c[0, h, i]
        order = np.argsort(-row, kind="stable")
        ref = set(order[:ki].tolist())
        got = set(ix[0, h, i, :ki].tolist())
        if ref != got and ki < i + 1:
            kth, nxt = row[order[ki - 1]], row[order[ki]]
            assert abs(kth - nxt) <= 1e-3 * kth


def test_gate_128k_density_properties():
    """Full-size gate: exact counts, ascending lists, and bit-exact selection
    on the GPU's own fp32 scores (oracle select on the same scores)."""
    w, Q, K, Wq, Wk, c, ix, sc = _gate_case("layer128k", "density", density=0.1)
    nb = w.nb
    ki = np.array([oracle.topk_count(i, oracle.MODE_TOPK_DENSITY, density=0.1) for i in range(nb)])
    assert np.array_equal(c, np.broadcast_to(ki, c.shape))
    sums = sc.double().sum(-1).numpy()
    np.testing.assert_allclose(sums, 1.0, atol=1e-4)
    # selection parity on sampled heads (oracle select on the GPU fp32 scores)
    for h in (0, 13, 31):
        sub = sc[:, h:h + 1].contiguous()
        c_ref, i_ref, _ = oracle.select(sub, oracle.MODE_TOPK_DENSITY, density=0.1,
                                        cap=ix.shape[-1])
        lists_equal(c[:, h:h + 1], ix[:, h:h + 1], c_ref, i_ref)


@pytest.mark.parametrize("ties", [False, True])
@pytest.mark.parametrize("nb", [1, 37, 130])
def test_gate_select_bitexact(nb, ties):
    w = synth.custom("sel", 2, 3, 1, 64 * nb, 64, 16, "fp32")
    s = synth.make_scores_like(w, seed=nb, ties=ties)
    sd = s.cuda()
    for mode, kw in (("threshold", dict(T=1.0 / (nb + 1))), ("topk", dict(k=5)),
                     ("density", dict(density=0.3)), ("density", dict(density=1.0))):
        c, ix = seer.seer_gate_select(sd, mode, **kw)
        torch.cuda.synchronize()
        mc = seer._lib.mode_code(mode)
        c_ref, i_ref, _ = oracle.select(s, mc, T=kw.get("T", 0.0), k=kw.get("k", 0),
                                        density=kw.get("density", 0.0), cap=ix.shape[-1])
        lists_equal(c.cpu().numpy(), ix.cpu().numpy(), c_ref, i_ref)


@pytest.mark.parametrize("ties", [False, True])
@pytest.mark.parametrize("B,Hq,nb", [(2, 16, 40), (1, 12, 130), (1, 1, 2048), (1, 1, 2049)])
def test_gate_select_bitexact_many_rows(B, Hq, nb, ties):
    """Enough rows for the warp-per-row selection (rows of up to 2048
    candidates), and a row length one past it (the CTA-per-row kernel), with
    and without the forced diagonal."""
    w = synth.custom("sel", B, Hq, 1, 64 * nb, 64, 16, "fp32")
    s = synth.make_scores_like(w, seed=nb + 7, ties=ties)
    sd = s.cuda()
    for fd in (False, True):
        for mode, kw in (("threshold", dict(T=1.0 / (nb + 1))), ("topk", dict(k=5)),
                         ("density", dict(density=0.3)), ("density", dict(density=1.0))):
            c, ix = seer.seer_gate_select(sd, mode, force_diagonal=fd, **kw)
            torch.cuda.synchronize()
            mc = seer._lib.mode_code(mode)
            c_ref, i_ref, _ = oracle.select(s, mc, T=kw.get("T", 0.0), k=kw.get("k", 0),
                                            density=kw.get("density", 0.0), cap=ix.shape[-1], force_diag=fd)
            lists_equal(c.cpu().numpy(), ix.cpu().numpy(), c_ref, i_ref)


def test_gate_force_diagonal_layer8k():
    """The whole gate (softmax of the logits, then selection) on 4096 rows with
    the forced diagonal: bit-exact against the oracle's selection of the GPU's
    scores, every row holding its diagonal block."""
    for mode, kw in (("threshold", dict(T=0.02)), ("density", dict(density=0.05))):
        w, Q, K, Wq, Wk, c, ix, sc = _gate_case("layer8k", mode, force_diagonal=True, **kw)
        mc = seer._lib.mode_code(mode)
        c_ref, i_ref, _ = oracle.select(sc, mc, T=kw.get("T", 0.0), density=kw.get("density", 0.0),
                                        cap=ix.shape[-1], force_diag=True)
        lists_equal(c, ix, c_ref, i_ref)
        # ascending lists: the diagonal block is each row's last entry
        last = np.take_along_axis(ix[0], (c[0] - 1)[..., None].astype(np.int64), axis=-1)[..., 0]
        assert np.array_equal(last, np.broadcast_to(np.arange(w.nb), last.shape))


def test_gate_select_threshold_empty_rows():
    w = synth.custom("sel", 1, 2, 1, 64 * 600, 64, 16, "fp32")
    # uniform rows: 1/(i+1) > 2e-3 only for rows shorter than 500 blocks
    nb = w.nb
    s = torch.tril(torch.ones(nb, nb, dtype=torch.float64))
    s = (s / s.sum(-1, keepdim=True)).float().expand(1, 2, nb, nb).contiguous()
    c, ix = seer.seer_gate_select(s.cuda(), "threshold", T=2e-3)
    c = c.cpu().numpy()
    c_ref, i_ref, _ = oracle.select(s, oracle.MODE_THRESHOLD, T=2e-3, cap=ix.shape[-1])
    lists_equal(c, ix.cpu().numpy(), c_ref, i_ref)
    assert c[0, 0, nb - 1] == 0 and c[0, 0, 0] == 1


def test_gate_rope_matches_oracle():
    """Block RoPE path (off in the workloads; base reading theta/64 unpinned)."""
    w = synth.custom("rope", 1, 4, 2, 64 * 24, 64, 32, "bf16", "layer", 9)
    Q, K, _ = synth.make_qkv(w)
    Wq, Wk = synth.make_gate_weights(w)
    Qd, Kd, Wqd, Wkd = to_dev(Q, K, Wq, Wk)
    c, ix, sc = seer.seer_gate(Qd, Kd, Wqd, Wkd, "topk", k=4, rope_theta=500000.0,
                               return_scores=True)
    s_ref = oracle.gate(Q, K, Wq, Wk, rope_theta=500000.0)
    _check_scores(sc.cpu(), s_ref)
    c_ref, i_ref, _ = oracle.select(sc.cpu(), oracle.MODE_TOPK_K, k=4, cap=ix.shape[-1])
    lists_equal(c.cpu().numpy(), ix.cpu().numpy(), c_ref, i_ref)


def test_gate_rejects_bad_arguments():
    w, Q, K, V, Wq, Wk = inputs("tiny")
    Qd, Kd, Wqd, Wkd = to_dev(Q, K, Wq, Wk)
    with pytest.raises(seer.SeerError) as e:
        seer.seer_gate(Qd, Kd, Wqd, Wkd, "threshold", T=0.0)
    assert e.value.status == 1
    with pytest.raises(seer.SeerError) as e:
        seer.seer_gate(Qd, Kd, Wqd, Wkd, "topk", k=4, cap=2)
    assert e.value.status == 3
