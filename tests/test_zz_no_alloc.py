"""seer_gate_noalloc: the gate for callers that cannot allocate device memory
(a plugin inside a framework that owns all device allocations and hands out
only its own tensors, or a runtime that forbids device allocation after
start-up).  Its scratch is a fixed buffer inside the library.

This file is collected last on purpose.  The test calls the entry point
through the C ABI and checks it against seer_gate (which uses a caller
workspace) on two calls in a row; it must pass alone in a fresh process (the
first call resolves the buffer's address) and after the other tests.
"""
import ctypes

import numpy as np
import pytest
import torch

import learned_block_sparse_seer_b200 as seer
from learned_block_sparse_seer_b200 import _lib, synth

from gpu_common import SCORE_RTOL, inputs

pytestmark = pytest.mark.gpu


def _noalloc_c_abi(Q, K, Wq, Wk, mode, T=0.0, k=0, density=0.0, with_scores=True):
    L = _lib.lib()
    B, Hq, n, d = Q.shape
    Hkv, h, nb = K.shape[1], Wq.shape[1], n // 64
    dims = _lib._dims(B, Hq, Hkv, n, d)
    mc = _lib.mode_code(mode)
    cap = L.seer_gate_required_cap(ctypes.byref(dims), mc, k, density)
    counts = torch.full((B, Hq, nb), -7, dtype=torch.int32, device="cuda")
    idx = torch.full((B, Hq, nb, cap), -7, dtype=torch.int32, device="cuda")
    scores = torch.full((B, Hq, nb, nb), float("nan"), dtype=torch.float32, device="cuda")
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    # without scores_out the block logits stay in the library's own buffer
    sp = p(scores) if with_scores else None
    st = L.seer_gate_noalloc(ctypes.byref(dims), p(Q), p(K), _lib._dtype_code(Q), p(Wq), p(Wk), h,
                             0.0, mc, T, k, density, sp, p(counts), p(idx), cap,
                             ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    torch.cuda.synchronize()
    return st, counts.cpu().numpy(), idx.cpu().numpy(), scores.cpu().double().numpy()


@pytest.mark.parametrize("name,mode,kw", [("tiny", "threshold", {"T": 5e-4}),
                                          ("layer8k", "density", {"density": 0.1})])
def test_noalloc_matches_workspace_gate_on_two_calls(name, mode, kw):
    w, Q, K, V, Wq, Wk = inputs(name)
    Qd, Kd, Wqd, Wkd = (t.cuda() for t in (Q, K, Wq, Wk))
    c_ref, i_ref, s_ref = seer.seer_gate(Qd, Kd, Wqd, Wkd, mode, return_scores=True, **kw)
    c_ref, i_ref = c_ref.cpu().numpy(), i_ref.cpu().numpy()
    s_ref = s_ref.cpu().double().numpy()
    # two calls in a row with the logits going to the caller's tensor, then two
    # that keep them in the library's buffer (scores_out = NULL)
    for with_scores in (True, True, False, False):
        st, c, ix, sc = _noalloc_c_abi(Qd, Kd, Wqd, Wkd, mode, with_scores=with_scores, **kw)
        assert st == 0, _lib.STATUS_NAMES.get(st, st)
        np.testing.assert_array_equal(c, c_ref)
        for r in zip(*np.nonzero(c_ref)):
            np.testing.assert_array_equal(ix[r][:c_ref[r]], i_ref[r][:c_ref[r]])
        if with_scores:
            rowmax = np.maximum(s_ref.max(-1, keepdims=True), 1e-300)
            assert np.max(np.abs(sc - s_ref) / rowmax) <= SCORE_RTOL
        else:
            assert np.isnan(sc).all()  # nothing was written to the unused tensor


def test_noalloc_rejects_problems_above_its_buffer():
    # 32k tokens x 32 heads needs more scratch than the fixed buffer holds;
    # the call is refused before anything is touched or launched
    L = _lib.lib()
    dims = _lib._dims(1, 32, 8, 32768, 128)
    need = L.seer_gate_workspace_size(ctypes.byref(dims), 128)
    assert need > (32 << 20)
    dummy = ctypes.c_void_p(256)
    st = L.seer_gate_noalloc(ctypes.byref(dims), dummy, dummy, 0, dummy, dummy, 128, 0.0, 2, 0.0, 0,
                             0.1, None, dummy, dummy, 205, None)
    assert st == 7  # SEER_ERR_WORKSPACE
