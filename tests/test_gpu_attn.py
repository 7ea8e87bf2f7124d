"""GPU parity of seer_sparse_attn against the fp64 oracle (through the C ABI)."""
import numpy as np
import pytest
import torch

import learned_block_sparse_seer_b200 as seer
import oracle
from learned_block_sparse_seer_b200 import synth

from gpu_common import (LSE_TOL, LSE_TOL_FP32_INPUT, check_lse, check_o, inputs, sample_units, to_dev,
                        unit_rows)

pytestmark = pytest.mark.gpu


def _run(Q, K, V, counts, idx, **kw):
    Qd, Kd, Vd = to_dev(Q, K, V)
    cd = torch.as_tensor(counts, dtype=torch.int32).cuda()
    idd = torch.as_tensor(idx, dtype=torch.int32).cuda()
    ws = torch.empty(seer.sparse_attn_workspace_size(*Q.shape[:2], K.shape[1], *Q.shape[2:],
                                                     0 if Q.dtype == torch.bfloat16 else 1),
                     dtype=torch.uint8, device="cuda")
    O, lse = seer.seer_sparse_attn(Qd, Kd, Vd, cd, idd, workspace=ws, **kw)
    assert seer.seer_workspace_status(ws) == 0
    return O.cpu(), lse.cpu()


def _oracle_lists(w, mode, **sel):
    _, Q, K, V, Wq, Wk = inputs(w.name)
    s = oracle.gate(Q, K, Wq, Wk)
    c, ix, _ = oracle.select(s, mode, **sel)
    return c, ix


def test_tiny_fp32_threshold():
    w, Q, K, V, Wq, Wk = inputs("tiny")
    c, ix = _oracle_lists(w, oracle.MODE_THRESHOLD, T=5e-4)
    O, lse = _run(Q, K, V, c, ix)
    O_ref, lse_ref = oracle.sparse_attn(Q, K, V, c, ix)
    check_o(O.double().numpy(), O_ref)
    check_lse(lse.double().numpy(), lse_ref, LSE_TOL_FP32_INPUT)


def test_tiny_bf16_topk():
    w, Q, K, V, Wq, Wk = inputs("tiny")
    Qb, Kb, Vb = (t.to(torch.bfloat16) for t in (Q, K, V))
    s = oracle.gate(Qb, Kb, Wq, Wk)
    for k in (1, 2, 3, 8):
        c, ix, _ = oracle.select(s, oracle.MODE_TOPK_K, k=k)
        O, lse = _run(Qb, Kb, Vb, c, ix)
        O_ref, lse_ref = oracle.sparse_attn(Qb, Kb, Vb, c, ix)
        check_o(O.double().numpy(), O_ref)
        check_lse(lse.double().numpy(), lse_ref)


def test_layer8k_threshold_sampled():
    w, Q, K, V, Wq, Wk = inputs("layer8k")
    Qd, Kd, Wqd, Wkd = to_dev(Q, K, Wq, Wk)
    cd, idd = seer.seer_gate(Qd, Kd, Wqd, Wkd, "threshold", T=5e-4)
    c, ix = cd.cpu().numpy(), idd.cpu().numpy()
    O, lse = _run(Q, K, V, c, ix)
    units = sample_units(w.B, w.Hq, w.nb, 40, seed=8)
    O_ref, lse_ref = oracle.sparse_attn_units(Q, K, V, c, ix, units)
    check_o(unit_rows(O, units, w.nb).double().numpy(), O_ref)
    check_lse(unit_rows(lse, units, w.nb).double().numpy(), lse_ref)


@pytest.mark.parametrize("name,rho", [("layer32k", 0.1), ("layer128k", 0.1), ("layer128k", 0.5)])
def test_full_size_density_sampled(name, rho):
    w, Q, K, V, Wq, Wk = inputs(name)
    Qd, Kd, Wqd, Wkd = to_dev(Q, K, Wq, Wk)
    cd, idd = seer.seer_gate(Qd, Kd, Wqd, Wkd, "density", density=rho)
    c, ix = cd.cpu().numpy(), idd.cpu().numpy()
    O, lse = _run(Q, K, V, c, ix)
    assert torch.isfinite(lse).all() and torch.isfinite(O.float()).all()
    units = sample_units(w.B, w.Hq, w.nb, 24, seed=int(rho * 100))
    O_ref, lse_ref = oracle.sparse_attn_units(Q, K, V, c, ix, units)
    check_o(unit_rows(O, units, w.nb).double().numpy(), O_ref)
    check_lse(unit_rows(lse, units, w.nb).double().numpy(), lse_ref)


@pytest.mark.parametrize("B,Hq,Hkv,nb,d", [(2, 4, 2, 9, 64), (1, 2, 1, 1, 128), (1, 4, 4, 3, 128)])
def test_all_ones_mask_dense_path_shapes(B, Hq, Hkv, nb, d):
    """All-ones lists take the dense 128-row kernel (bf16 inputs): odd block
    counts (a last tile with one valid query block), a single block, MHA,
    d = 64 and B > 1 against the oracle; one row off the all-ones mask sends
    the same call to the sparse kernel, with the same result."""
    w = synth.custom("dense_shapes", B, Hq, Hkv, 64 * nb, d, 16, "bf16", "layer", 40 + nb)
    Q, K, V = synth.make_qkv(w)
    c, ix = oracle.dense_lists(B, Hq, nb)
    O, lse = _run(Q, K, V, c, ix)
    O_ref, lse_ref = oracle.sparse_attn(Q, K, V, c, ix)
    check_o(O.double().numpy(), O_ref)
    check_lse(lse.double().numpy(), lse_ref)
    if nb > 1:
        # drop block 0 from the last row of the last head: no longer all-ones
        c2, ix2 = c.copy(), ix.copy()
        c2[B - 1, Hq - 1, nb - 1] = nb - 1
        ix2[B - 1, Hq - 1, nb - 1, :nb - 1] = np.arange(1, nb)
        ix2[B - 1, Hq - 1, nb - 1, nb - 1:] = -1
        O2, lse2 = _run(Q, K, V, c2, ix2)
        O2_ref, lse2_ref = oracle.sparse_attn(Q, K, V, c2, ix2)
        check_o(O2.double().numpy(), O2_ref)
        check_lse(lse2.double().numpy(), lse2_ref)


def test_all_ones_mask_equals_dense():
    w = synth.custom("dense", 1, 8, 2, 64 * 40, 128, 128, "bf16", "layer", 12)
    Q, K, V = synth.make_qkv(w)
    c, ix = oracle.dense_lists(w.B, w.Hq, w.nb)
    O, lse = _run(Q, K, V, c, ix)
    O_ref, lse_ref = oracle.sparse_attn(Q, K, V, c, ix)
    check_o(O.double().numpy(), O_ref)
    check_lse(lse.double().numpy(), lse_ref)
    # cross-check with the library SDPA of the same device
    G = w.Hq // w.Hkv
    ref = torch.nn.functional.scaled_dot_product_attention(
        Q.cuda(), K.cuda().repeat_interleave(G, 1), V.cuda().repeat_interleave(G, 1), is_causal=True)
    assert (ref.float().cpu() - O.float()).abs().max() < 2e-2


@pytest.mark.parametrize("B,Hq,Hkv,nb,d", [(2, 4, 4, 5, 128), (1, 2, 1, 1, 128), (3, 6, 2, 9, 64),
                                            (1, 4, 1, 33, 128)])
def test_edge_cases(B, Hq, Hkv, nb, d):
    """Empty rows, diagonal-only rows, single-block lists, odd counts, full
    rows, batch > 1, MHA, d = 64, a single 64-token sequence."""
    w = synth.custom("edge", B, Hq, Hkv, 64 * nb, d, 16, "bf16", "layer", 20 + nb)
    Q, K, V = synth.make_qkv(w)
    rng = np.random.default_rng(nb)
    cap = nb + 3
    counts = np.zeros((B, Hq, nb), np.int32)
    idx = np.full((B, Hq, nb, cap), -1, np.int32)
    for b, h, i in np.ndindex(B, Hq, nb):
        kind = (b + h + i) % 5
        if kind == 0:
            lst = []                               # empty row
        elif kind == 1:
            lst = [i]                              # diagonal only
        elif kind == 2:
            lst = list(range(i + 1))               # full causal row
        elif kind == 3:
            lst = [0]                              # sink only
        else:
            m = rng.integers(1, i + 2)
            lst = sorted(rng.choice(i + 1, size=m, replace=False).tolist())
        counts[b, h, i] = len(lst)
        idx[b, h, i, :len(lst)] = lst
    O, lse = _run(Q, K, V, counts, idx)
    O_ref, lse_ref = oracle.sparse_attn(Q, K, V, counts, idx)
    check_o(O.double().numpy(), O_ref)
    check_lse(lse.double().numpy(), lse_ref)
    empty = counts == 0
    assert torch.all(O.view(B, Hq, nb, 64, d)[torch.as_tensor(empty)] == 0)


@pytest.mark.parametrize("d,dtype", [(128, torch.bfloat16), (64, torch.bfloat16), (128, torch.float32)])
@pytest.mark.parametrize("kval,overflows", [(4.0, False), (6.0, True)])
def test_score_far_above_first_step(d, dtype, kval, overflows):
    """The attention kernel keeps each unit's running maximum at its first
    step's column maximum.  A later key whose score is far above it (a
    shifted query block against one large key in a later block) must still
    give the exact softmax.  Up to about 2^128 in probability (kval = 4:
    about 2^90 .. 2^130 across the two head sizes) the kernel's own arithmetic
    stays finite; beyond it (kval = 6) P, the column sums or O overflow, the
    kernel flags the unit and the fallback kernel recomputes it exactly."""
    nb = 7
    w = synth.custom("spike", 1, 2, 1, 64 * nb, d, 16, "bf16", "layer", 31)
    Q, K, V = synth.make_qkv(w)
    Q = Q.float()
    K = K.float()
    Q[:, :, 64 * 3:, :] += 2.0
    K[:, :, 64 * 3 + 8, :] = kval
    Q, K, V = Q.to(dtype), K.to(dtype), V.to(dtype)
    counts, idx = oracle.dense_lists(1, 2, nb)
    Qd, Kd, Vd = to_dev(Q, K, V)
    ws = torch.empty(seer.sparse_attn_workspace_size(1, 2, 1, 64 * nb, d,
                                                     0 if dtype == torch.bfloat16 else 1),
                     dtype=torch.uint8, device="cuda")
    O, lse = seer.seer_sparse_attn(Qd, Kd, Vd, torch.as_tensor(counts).cuda(),
                                   torch.as_tensor(idx).cuda(), workspace=ws)
    assert seer.seer_workspace_status(ws) == 0
    # the header's second work counter holds the number of flagged units
    flagged = int(ws[12:16].view(torch.int32).item())
    if overflows:
        assert flagged > 0
    # fp32 inputs are converted to bf16 before the tensor-core pass; with
    # logits near 100 that rounding alone moves the LSE by up to ~0.4, so the
    # oracle is given the same bf16 values
    Qr, Kr, Vr = (t.to(torch.bfloat16) for t in (Q, K, V))
    O_ref, lse_ref = oracle.sparse_attn(Qr, Kr, Vr, counts, idx)
    assert np.isfinite(O_ref).all()
    check_o(O.double().cpu().numpy(), O_ref)
    check_lse(lse.double().cpu().numpy(), lse_ref, LSE_TOL)


def test_bad_lists_are_flagged_not_followed():
    """Out-of-range counts and indices are clamped by the kernel and reported
    as SEER_ERR_DEVICE_CHECK; nothing outside the tensors is read."""
    w = synth.custom("bad", 1, 2, 1, 64 * 4, 64, 16, "bf16", "layer", 3)
    Q, K, V = synth.make_qkv(w)
    cap = 4
    counts = np.array([[[1, 2, 3, 9], [1, 1, 1, 1]]], np.int32)       # 9 > cap
    idx = np.zeros((1, 2, 4, cap), np.int32)
    idx[0, 0, 1, :2] = [0, 1]
    idx[0, 0, 2, :3] = [0, 2, 1]                                       # not ascending
    idx[0, 1, 0, 0] = 3                                                # j > i
    Qd, Kd, Vd = to_dev(Q, K, V)
    ws = torch.empty(seer.sparse_attn_workspace_size(1, 2, 1, 256, 64), dtype=torch.uint8,
                     device="cuda")
    seer.seer_sparse_attn(Qd, Kd, Vd, torch.as_tensor(counts).cuda(), torch.as_tensor(idx).cuda(),
                          workspace=ws)
    assert seer.seer_workspace_status(ws) == 6  # SEER_ERR_DEVICE_CHECK


def test_repeat_runs_bitwise_identical():
    w, Q, K, V, Wq, Wk = inputs("layer8k")
    c, ix = _oracle_lists(w, oracle.MODE_TOPK_DENSITY, density=0.2)
    O1, l1 = _run(Q, K, V, c, ix)
    O2, l2 = _run(Q, K, V, c, ix)
    assert torch.equal(O1, O2) and torch.equal(l1, l2)


def test_rejects_bad_arguments():
    import ctypes
    w, Q, K, V, Wq, Wk = inputs("tiny")
    Qd, Kd, Vd = to_dev(Q, K, V)
    c = torch.ones(1, 2, 8, dtype=torch.int32, device="cuda")
    ix = torch.zeros(1, 2, 8, 1, dtype=torch.int32, device="cuda")
    small = torch.empty(8, dtype=torch.uint8, device="cuda")
    with pytest.raises(ValueError):
        seer.seer_sparse_attn(Qd, Kd, Vd, c, ix, workspace=small)
    # the C entry point itself refuses a too-small workspace before launching
    L = seer.lib()
    dims = seer._lib._dims(1, 2, 1, 512, 64)
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    O = torch.empty_like(Qd)
    st = L.seer_sparse_attn(ctypes.byref(dims), p(Qd), p(Kd), p(Vd), 1, p(c), p(ix), 1, 0.0, p(O),
                            None, p(small), 8, None)
    assert st == 7  # SEER_ERR_WORKSPACE
    with pytest.raises(seer.SeerError) as e:
        seer.seer_sparse_attn(Qd, Kd, Vd, c, ix, scale=-1.0)
    assert e.value.status == 1


def test_bounded_wait_gives_up_and_the_device_stays_usable():
    """The failure path of the kernel's bounded waits, without faulting the GPU:
    the library's test hook leaves out the completion signal of every CTA's
    first QK step, so the waits that depend on it give up after 20 ms.  The
    call must report SEER_ERR_TIMEOUT through the workspace status word (its
    kernel unwinds, draining its bulk copies), and the next call on the same
    device and workspace must match the oracle."""
    from learned_block_sparse_seer_b200 import _lib
    L = _lib.lib()
    w, Q, K, V, Wq, Wk = inputs("tiny")
    Qb, Kb, Vb = (t.to(torch.bfloat16) for t in (Q, K, V))
    # k = 4 of 8 blocks: not the all-ones mask, which seer_sparse_attn hands
    # to the dense 128-row kernel instead of the sparse one
    c, ix, _ = oracle.select(oracle.gate(Qb, Kb, Wq, Wk), oracle.MODE_TOPK_K, k=4)
    Qd, Kd, Vd = to_dev(Qb, Kb, Vb)
    cd = torch.as_tensor(c, dtype=torch.int32).cuda()
    idd = torch.as_tensor(ix, dtype=torch.int32).cuda()
    ws = torch.empty(seer.sparse_attn_workspace_size(w.B, w.Hq, w.Hkv, w.n, w.d), dtype=torch.uint8, device="cuda")
    try:
        L.seer_testing_attn_wait_fault(0, 20_000_000)
        seer.seer_sparse_attn(Qd, Kd, Vd, cd, idd, workspace=ws)
        assert seer.seer_workspace_status(ws) == 5  # SEER_ERR_TIMEOUT
    finally:
        L.seer_testing_attn_wait_fault(-1, 0)
    for _ in range(2):
        O, lse = seer.seer_sparse_attn(Qd, Kd, Vd, cd, idd, workspace=ws)
        assert seer.seer_workspace_status(ws) == 0
        O_ref, lse_ref = oracle.sparse_attn(Qb, Kb, Vb, c, ix)
        check_o(O.cpu().double().numpy(), O_ref)
        check_lse(lse.cpu().double().numpy(), lse_ref)
