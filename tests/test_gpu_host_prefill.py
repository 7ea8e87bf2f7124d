"""GPU checks of seer_prefill_host (gate + sparse attention for inputs and
outputs in host memory, one KV head's group of query heads at a time, the
copies overlapped with the compute) through the C ABI.

Every step of the path is per head and per query block, so the results must
be bit-identical to seer_gate + seer_sparse_attn run on the whole layer on
the device (which the other GPU tests hold against the fp64 oracle); one
case is also checked against the oracle directly."""
import numpy as np
import pytest
import torch

import learned_block_sparse_seer_b200 as seer
import oracle
from learned_block_sparse_seer_b200 import synth

from gpu_common import check_lse, check_o, LSE_TOL

pytestmark = pytest.mark.gpu


def _device_path(Q, K, V, Wq, Wk, mode, kw, fd=False):
    Qd, Kd, Vd, Wqd, Wkd = (t.cuda() for t in (Q, K, V, Wq, Wk))
    c, ix = seer.seer_gate(Qd, Kd, Wqd, Wkd, mode, force_diagonal=fd, **kw)
    O, lse = seer.seer_sparse_attn(Qd, Kd, Vd, c, ix)
    return O.cpu(), lse.cpu()


def _host_path(Q, K, V, Wq, Wk, mode, kw, fd=False, pinned=True, return_lse=True):
    hQ, hK, hV = (t.contiguous() for t in (Q, K, V))
    if pinned:
        hQ, hK, hV = (t.pin_memory() for t in (hQ, hK, hV))
    O, lse = seer.seer_prefill_host(hQ, hK, hV, Wq.cuda(), Wk.cuda(), mode, force_diagonal=fd,
                                    return_lse=return_lse, **kw)
    return O, lse


@pytest.mark.parametrize("B,Hq,Hkv,nb,d,dtype", [(2, 8, 2, 40, 128, "bf16"), (1, 4, 4, 37, 64, "bf16"),
                                                 (1, 6, 2, 24, 128, "fp32"), (3, 2, 1, 9, 64, "bf16"),
                                                 (2, 1, 1, 1, 64, "bf16"), (1, 3, 1, 130, 128, "bf16")])
@pytest.mark.parametrize("mode,kw", [("density", dict(density=0.2)), ("threshold", dict(T=0.02)),
                                     ("topk", dict(k=3))])
def test_matches_device_path_bit_exact(B, Hq, Hkv, nb, d, dtype, mode, kw):
    w = synth.custom("hp", B, Hq, Hkv, 64 * nb, d, 64, dtype, "layer", 31)
    Q, K, V = synth.make_qkv(w)
    Wq, Wk = synth.make_gate_weights(w)
    O_ref, lse_ref = _device_path(Q, K, V, Wq, Wk, mode, kw)
    O, lse = _host_path(Q, K, V, Wq, Wk, mode, kw)
    assert not O.is_cuda and not lse.is_cuda
    assert torch.equal(O, O_ref)
    assert torch.equal(lse, lse_ref)


def test_forced_diagonal_pageable_and_no_lse():
    w = synth.custom("hp", 2, 4, 2, 64 * 20, 128, 32, "bf16", "layer", 33)
    Q, K, V = synth.make_qkv(w)
    Wq, Wk = synth.make_gate_weights(w)
    kw = dict(T=0.5)
    O_ref, _ = _device_path(Q, K, V, Wq, Wk, "threshold", kw, fd=True)
    O, lse = _host_path(Q, K, V, Wq, Wk, "threshold", kw, fd=True, pinned=False, return_lse=False)
    assert lse is None
    assert torch.equal(O, O_ref)


def test_against_oracle_tiny():
    """The tiny workload (fp32) end to end from host memory against the fp64
    oracle (gate, selection on the GPU's own scores, attention)."""
    w = synth.WORKLOADS["tiny"]
    Q, K, V = synth.make_qkv(w)
    Wq, Wk = synth.make_gate_weights(w)
    O, lse = _host_path(Q, K, V, Wq, Wk, "threshold", dict(T=5e-4))
    _, _, sc = seer.seer_gate(Q.cuda(), K.cuda(), Wq.cuda(), Wk.cuda(), "threshold", T=5e-4, return_scores=True)
    c_ref, i_ref, _ = oracle.select(sc.cpu(), oracle.MODE_THRESHOLD, T=5e-4)
    O_ref, lse_ref = oracle.sparse_attn(Q, K, V, c_ref, i_ref)
    check_o(O.double().numpy(), O_ref)
    # fp32 inputs are rounded to bf16 for the tensor cores (see the smoke check)
    check_lse(lse.double().numpy(), lse_ref, 1e-2)


def test_buffer_too_small_is_rejected():
    w = synth.custom("hp", 1, 4, 2, 64 * 8, 64, 32, "bf16", "layer", 35)
    Q, K, V = synth.make_qkv(w)
    Wq, Wk = synth.make_gate_weights(w)
    need = seer.prefill_host_buffer_size(1, 4, 2, 64 * 8, 64, 32, "topk", k=2)
    assert need > 0
    small = torch.empty(need - 256, dtype=torch.uint8, device="cuda")
    with pytest.raises(ValueError):
        seer.seer_prefill_host(Q, K, V, Wq.cuda(), Wk.cuda(), "topk", k=2, buffer=small)
