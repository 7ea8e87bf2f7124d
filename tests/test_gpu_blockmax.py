"""GPU parity of seer_attn_blockmax (the gate's max-pooled ground truth)
against the fp64 oracle's direct definition, through the C ABI."""
import numpy as np
import pytest
import torch

import learned_block_sparse_seer_b200 as seer
import oracle
from learned_block_sparse_seer_b200 import synth

from gpu_common import BMAX_TOL, LSE_TOL, LSE_TOL_FP32_INPUT, inputs, sample_units, to_dev

pytestmark = pytest.mark.gpu


def _run(Q, K):
    Qd, Kd = to_dev(Q, K)
    ws = torch.empty(seer.blockmax_workspace_size(*Q.shape[:2], K.shape[1], *Q.shape[2:],
                                                  0 if Q.dtype == torch.bfloat16 else 1),
                     dtype=torch.uint8, device="cuda")
    M, lse = seer.seer_attn_blockmax(Qd, Kd, workspace=ws)
    assert seer.seer_workspace_status(ws) == 0
    return M.cpu().double().numpy(), lse.cpu().double().numpy()


def _check_rows(M, lse, Q, K, units, nb, lse_tol=LSE_TOL):
    gt_ref, lse_ref = oracle.blockmax_units(Q, K, units)
    got = M.reshape(-1, nb)[units]
    err = np.abs(got - gt_ref).max()
    assert err <= BMAX_TOL, f"blockmax error {err:.3e}"
    n = nb * 64
    lflat = lse.reshape(-1, n)
    lrows = np.stack([lflat[u // nb, (u % nb) * 64:(u % nb + 1) * 64] for u in units])
    assert np.abs(lrows - lse_ref).max() <= lse_tol


def test_tiny_full():
    w, Q, K, V, Wq, Wk = inputs("tiny")
    M, lse = _run(Q, K)
    gt_ref, lse_ref = oracle.blockmax(Q, K)
    assert np.abs(M - gt_ref).max() <= BMAX_TOL
    assert np.abs(lse - lse_ref).max() <= LSE_TOL_FP32_INPUT


@pytest.mark.parametrize("name,nrand", [("bmax4k", 48), ("bmax32k", 12)])
def test_workloads_sampled(name, nrand):
    w, Q, K, V, Wq, Wk = inputs(name)
    M, lse = _run(Q, K)
    nb = w.nb
    # structure that holds at any size: causal zeros, row 0 is exactly 1
    iu = np.triu_indices(nb, 1)
    assert np.all(M[..., iu[0], iu[1]] == 0)
    assert np.allclose(M[..., 0, 0], 1.0, atol=1e-6)
    assert np.all(M <= 1.0 + 1e-6)
    rowmax = M.max(-1)
    assert np.all(rowmax >= 1.0 / (64 * np.arange(nb) + 1) - 1e-6)
    units = sample_units(w.B, w.Hq, nb, nrand, seed=3)
    _check_rows(M, lse, Q, K, units, nb)


@pytest.mark.parametrize("B,Hq,Hkv,nb,d", [(2, 3, 3, 7, 128), (1, 2, 1, 1, 64), (1, 4, 2, 2, 64)])
def test_shapes(B, Hq, Hkv, nb, d):
    """Odd block counts (a half-empty last tile pair), MHA, d = 64, n = 64."""
    w = synth.custom("bm", B, Hq, Hkv, 64 * nb, d, 16, "bf16", "layer", 40 + nb)
    Q, K, _ = synth.make_qkv(w)
    M, lse = _run(Q, K)
    gt_ref, lse_ref = oracle.blockmax(Q, K)
    assert np.abs(M - gt_ref).max() <= BMAX_TOL
    assert np.abs(lse - lse_ref).max() <= LSE_TOL
