"""GPU parity of seer_gate_kl_backward (the AttnGate's distillation step:
KL(gt || score) and the gradients of the gate's two linear layers) against
the fp64 oracle, called through the C ABI (via the ctypes binding)."""
import numpy as np
import pytest
import torch

import learned_block_sparse_seer_b200 as seer
import oracle
from learned_block_sparse_seer_b200 import synth

from gpu_common import inputs, to_dev

pytestmark = pytest.mark.gpu

# fp32 sums over O(nb) terms per entry: relative to the largest entry
GRAD_RTOL = 2e-4
LOSS_RTOL = 1e-4


def _check(loss_gpu, dWq_gpu, dWk_gpu, loss_ref, dWq_ref, dWk_ref):
    lg = float(loss_gpu.item())
    assert abs(lg - loss_ref) <= LOSS_RTOL * abs(loss_ref), (lg, loss_ref)
    for name, g, r in (("dWq", dWq_gpu, dWq_ref), ("dWk", dWk_gpu, dWk_ref)):
        gg = g.double().cpu().numpy()
        err = np.abs(gg - r).max() / np.abs(r).max()
        assert err <= GRAD_RTOL, f"{name}: relative error {err:.2e}"


def _random_gt(B, Hq, nb, seed):
    g = torch.Generator("cpu").manual_seed(seed)
    gt = torch.rand(B, Hq, nb, nb, generator=g, dtype=torch.float32) ** 4 + 1e-3
    return torch.tril(gt)


def test_tiny_with_oracle_ground_truth():
    """Tiny workload (fp32 inputs); gt is the oracle's own max-pooled map."""
    w, Q, K, V, Wq, Wk = inputs("tiny")
    gt, _ = oracle.blockmax(Q, K)
    gt32 = torch.from_numpy(gt).float()
    loss_ref, dWq_ref, dWk_ref = oracle.gate_kl_backward(Q, K, Wq, Wk, gt32.double().numpy())
    Qd, Kd, Wqd, Wkd, gtd = to_dev(Q, K, Wq, Wk, gt32)
    loss, dWq, dWk = seer.seer_gate_kl_backward(Qd, Kd, Wqd, Wkd, gtd)
    torch.cuda.synchronize()
    _check(loss, dWq, dWk, loss_ref, dWq_ref, dWk_ref)


@pytest.mark.parametrize("B,Hq,Hkv,nb,d,h", [(2, 4, 2, 9, 64, 32), (1, 8, 2, 33, 128, 64)])
def test_shapes_bf16(B, Hq, Hkv, nb, d, h):
    """Ragged block counts (not multiples of the 64-wide GEMM tiles), GQA
    groups of 2 and 4, both head sizes; bf16 inputs."""
    wl = synth.custom("kls", B, Hq, Hkv, 64 * nb, d, h, "bf16", "layer", 21)
    Q, K, _ = synth.make_qkv(wl)
    Wq, Wk = synth.make_gate_weights(wl)
    Wq, Wk = Wq * 10.0, Wk * 10.0
    gt = _random_gt(B, Hq, nb, 5)
    loss_ref, dWq_ref, dWk_ref = oracle.gate_kl_backward(Q, K, Wq, Wk, gt.double().numpy())
    Qd, Kd, Wqd, Wkd, gtd = to_dev(Q, K, Wq, Wk, gt)
    loss, dWq, dWk = seer.seer_gate_kl_backward(Qd, Kd, Wqd, Wkd, gtd)
    torch.cuda.synchronize()
    _check(loss, dWq, dWk, loss_ref, dWq_ref, dWk_ref)


def test_layer8k_and_repeatable():
    """The 8k layer (32/8 heads, d = h = 128); two calls give bit-identical
    loss and gradients (fixed summation orders throughout)."""
    w, Q, K, V, Wq, Wk = inputs("layer8k")
    gt = _random_gt(w.B, w.Hq, w.nb, 9)
    loss_ref, dWq_ref, dWk_ref = oracle.gate_kl_backward(Q, K, Wq, Wk, gt.double().numpy())
    Qd, Kd, Wqd, Wkd, gtd = to_dev(Q, K, Wq, Wk, gt)
    loss, dWq, dWk = seer.seer_gate_kl_backward(Qd, Kd, Wqd, Wkd, gtd)
    loss2, dWq2, dWk2 = seer.seer_gate_kl_backward(Qd, Kd, Wqd, Wkd, gtd)
    torch.cuda.synchronize()
    _check(loss, dWq, dWk, loss_ref, dWq_ref, dWk_ref)
    assert torch.equal(loss, loss2) and torch.equal(dWq, dWq2) and torch.equal(dWk, dWk2)


def test_rejects_bad_arguments():
    w, Q, K, V, Wq, Wk = inputs("tiny")
    Qd, Kd, Wqd, Wkd = to_dev(Q, K, Wq, Wk)
    gt = torch.ones(1, 2, 8, 8, device="cuda")
    with pytest.raises(TypeError):
        seer.seer_gate_kl_backward(Qd, Kd, Wqd, Wkd, gt.double())
    with pytest.raises(seer.SeerError):
        seer.seer_gate_kl_backward(Qd[..., :48].contiguous(), Kd[..., :48].contiguous(), Wqd[..., :48].contiguous(),
                                   Wkd[..., :144].contiguous(), gt)
