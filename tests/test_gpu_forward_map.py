"""GPU parity of seer_attn_forward_map (the training forward: dense causal O
and LSE plus the 2D-max-pooled map in one call) against the fp64 oracle,
through the C ABI."""
import numpy as np
import pytest
import torch

import learned_block_sparse_seer_b200 as seer
import oracle
from learned_block_sparse_seer_b200 import synth

from gpu_common import (BMAX_TOL, LSE_TOL, LSE_TOL_FP32_INPUT, check_lse, check_o, inputs, sample_units, to_dev,
                        unit_rows)

pytestmark = pytest.mark.gpu


def _run(Q, K, V):
    Qd, Kd, Vd = to_dev(Q, K, V)
    B, Hq, n, d = Q.shape
    ws = torch.empty(seer.attn_forward_map_workspace_size(B, Hq, K.shape[1], n, d,
                                                          0 if Q.dtype == torch.bfloat16 else 1),
                     dtype=torch.uint8, device="cuda")
    O, lse, M = seer.seer_attn_forward_map(Qd, Kd, Vd, workspace=ws)
    assert seer.seer_workspace_status(ws) == 0
    return O.cpu(), lse.cpu().double().numpy(), M.cpu().double().numpy()


def test_tiny_full():
    """fp32 tiny workload: O and LSE equal dense causal attention (the oracle
    with every causal block listed), the map equals the oracle's."""
    w, Q, K, V, Wq, Wk = inputs("tiny")
    O, lse, M = _run(Q, K, V)
    counts, idx = oracle.dense_lists(w.B, w.Hq, w.nb)
    # the tensor cores see bf16-rounded fp32 inputs
    Qr, Kr, Vr = (t.to(torch.bfloat16) for t in (Q, K, V))
    O_ref, lse_ref = oracle.sparse_attn(Qr, Kr, Vr, counts, idx)
    check_o(O.double().numpy(), O_ref)
    check_lse(lse, lse_ref, LSE_TOL_FP32_INPUT)
    gt_ref, _ = oracle.blockmax(Q, K)
    assert np.abs(M - gt_ref).max() <= BMAX_TOL


@pytest.mark.parametrize("B,Hq,Hkv,nb,d", [(2, 4, 2, 5, 128), (1, 4, 1, 7, 64)])
def test_shapes_bf16(B, Hq, Hkv, nb, d):
    wl = synth.custom("fm", B, Hq, Hkv, 64 * nb, d, 16, "bf16", "layer", 41)
    Q, K, V = synth.make_qkv(wl)
    O, lse, M = _run(Q, K, V)
    counts, idx = oracle.dense_lists(B, Hq, nb)
    O_ref, lse_ref = oracle.sparse_attn(Q, K, V, counts, idx)
    check_o(O.double().numpy(), O_ref)
    check_lse(lse, lse_ref, LSE_TOL)
    gt_ref, _ = oracle.blockmax(Q, K)
    assert np.abs(M - gt_ref).max() <= BMAX_TOL


def test_layer8k_sampled():
    """The 8k layer, checked on sampled units: O rows, LSE and map rows."""
    w, Q, K, V, Wq, Wk = inputs("layer8k")
    O, lse, M = _run(Q, K, V)
    nb = w.nb
    units = sample_units(w.B, w.Hq, nb, 16, seed=7)
    counts, idx = oracle.dense_lists(w.B, w.Hq, nb)
    O_ref, lse_ref = oracle.sparse_attn_units(Q, K, V, counts, idx, units)
    check_o(unit_rows(O, units, nb).double().numpy(), O_ref)
    gt_ref, _ = oracle.blockmax_units(Q, K, units)
    assert np.abs(M.reshape(-1, nb)[units] - gt_ref).max() <= BMAX_TOL
    iu = np.triu_indices(nb, 1)
    assert np.all(M[..., iu[0], iu[1]] == 0)


def test_fallback_units_keep_an_exact_map():
    """A key block far above the first step's maximum (scores more than 2^64
    above it) sends its units to the exact fallback, which also rewrites their
    map rows."""
    wl = synth.custom("fm", 1, 2, 1, 64 * 6, 64, 16, "bf16", "layer", 43)
    Q, K, V = synth.make_qkv(wl)
    K = K.float()
    K[:, :, 64 * 4:64 * 5] *= 40.0
    K = K.to(torch.bfloat16).contiguous()
    O, lse, M = _run(Q, K, V)
    counts, idx = oracle.dense_lists(1, 2, 6)
    O_ref, lse_ref = oracle.sparse_attn(Q, K, V, counts, idx)
    check_o(O.double().numpy(), O_ref)
    check_lse(lse, lse_ref, LSE_TOL)
    gt_ref, _ = oracle.blockmax(Q, K)
    assert np.abs(M - gt_ref).max() <= BMAX_TOL
