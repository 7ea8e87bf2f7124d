"""GPU parity of the forced-diagonal selection and of variable-length
sequences packed along the token axis (seer_gate_varlen, then
seer_sparse_attn on the packed buffer), against the fp64 oracle through the
C ABI.  Tolerances as the prefill gate and attention (gpu_common)."""
import numpy as np
import pytest
import torch

import learned_block_sparse_seer_b200 as seer
import oracle
from learned_block_sparse_seer_b200 import synth

from gpu_common import LSE_TOL, LSE_TOL_FP32_INPUT, SCORE_RTOL, check_lse, check_o

pytestmark = pytest.mark.gpu

MODES = [(seer.SELECT_THRESHOLD, dict(T=0.06)), (seer.SELECT_TOPK_K, dict(k=3)),
         (seer.SELECT_TOPK_DENSITY, dict(density=0.3))]


def _lists_equal(cnt, ix, cnt_ref, idx_ref):
    assert np.array_equal(cnt, cnt_ref)
    for r in np.ndindex(cnt.shape):
        assert np.array_equal(ix[r][:cnt[r]], idx_ref[r][:cnt[r]]), r


# ------------------------------------------------------------ force diagonal --
@pytest.mark.parametrize("mode,kw", MODES)
def test_force_diagonal_select_bit_exact(mode, kw):
    w = synth.custom("fd", 2, 4, 2, 64 * 40, 64, 16, "fp32")
    s = synth.make_scores_like(w, seed=5, ties=True)
    c, ix = seer.seer_gate_select(s.cuda(), mode, force_diagonal=True, **kw)
    c_ref, i_ref, _ = oracle.select(s, mode, force_diag=True, **kw)
    _lists_equal(c.cpu().numpy(), ix.cpu().numpy(), c_ref, i_ref)
    assert np.all(c.cpu().numpy() >= 1)


def test_force_diagonal_gate_no_empty_rows():
    """Threshold 1 (no score exceeds it): without the flag every row is empty,
    with it every row is exactly its diagonal block."""
    w = synth.custom("fd", 1, 4, 2, 64 * 16, 64, 64, "bf16", "layer", 3)
    Q, K, V = synth.make_qkv(w)
    Wq, Wk = synth.make_gate_weights(w)
    Qd, Kd, Wqd, Wkd = (t.cuda() for t in (Q, K, Wq, Wk))
    c0, _ = seer.seer_gate(Qd, Kd, Wqd, Wkd, "threshold", T=1.0)
    c1, i1 = seer.seer_gate(Qd, Kd, Wqd, Wkd, "threshold", T=1.0, force_diagonal=True)
    assert c0.cpu().eq(0).all()
    assert c1.cpu().eq(1).all()
    assert torch.equal(i1[..., 0].cpu(), torch.arange(16, dtype=torch.int32).expand(1, 4, 16))


# ------------------------------------------------------------------ varlen --
LAYOUTS = [([300, 64, 1, 517], [0, 1, 0, 2]), ([1024], [0]), ([65, 127, 128, 3], [2, 0, 1, 1])]


def _varlen_case(lens, gaps, dtype="bf16", d=128, Hq=8, Hkv=2, pad="nan", seed=11):
    starts, n = synth.varlen_layout(lens, gaps)
    n += 64  # a trailing empty block
    w = synth.custom("vl", 1, Hq, Hkv, n, d, d, dtype, "layer", seed)
    Q, K, V = synth.make_varlen(w, starts, lens, pad=pad)
    Wq, Wk = synth.make_gate_weights(w)
    return w, starts, n, Q, K, V, Wq, Wk


@pytest.mark.parametrize("lens,gaps", LAYOUTS)
@pytest.mark.parametrize("mode,kw", MODES)
@pytest.mark.parametrize("fd", [False, True])
def test_gate_varlen(lens, gaps, mode, kw, fd):
    """Scores against the per-sequence oracle gate; lists bit-exact against
    the oracle's per-sequence selection of the GPU's scores.  Padding is NaN:
    the gate must not read it."""
    w, starts, n, Q, K, V, Wq, Wk = _varlen_case(lens, gaps, pad="nan")
    st = torch.tensor(starts, dtype=torch.int32, device="cuda")
    ln = torch.tensor(lens, dtype=torch.int32, device="cuda")
    c, ix, sc = seer.seer_gate_varlen(Q.cuda(), K.cuda(), Wq.cuda(), Wk.cuda(), st, ln, mode, return_scores=True,
                                      force_diagonal=fd, **kw)
    s = sc.cpu().double().numpy()
    assert np.isfinite(s).all()
    s_ref = oracle.gate_varlen(Q, K, Wq, Wk, starts, lens)
    rowmax = np.maximum(s_ref.max(-1, keepdims=True), 1e-30)
    assert (np.abs(s - s_ref) / rowmax).max() <= SCORE_RTOL
    c_ref, i_ref = oracle.select_varlen(sc.cpu(), starts, lens, mode, force_diag=fd, cap=ix.shape[-1], **kw)
    _lists_equal(c.cpu().numpy(), ix.cpu().numpy(), c_ref, i_ref)


@pytest.mark.parametrize("mode,kw", MODES)
@pytest.mark.parametrize("fd", [False, True])
def test_gate_varlen_many_rows(mode, kw, fd):
    """32 query heads over about 40 blocks: enough rows for the warp-per-row
    selection, with its varlen windows."""
    lens, gaps = [1000, 700, 65, 300], [0, 2, 1, 0]
    w, starts, n, Q, K, V, Wq, Wk = _varlen_case(lens, gaps, pad="nan", Hq=32, Hkv=8, d=64)
    st = torch.tensor(starts, dtype=torch.int32, device="cuda")
    ln = torch.tensor(lens, dtype=torch.int32, device="cuda")
    c, ix, sc = seer.seer_gate_varlen(Q.cuda(), K.cuda(), Wq.cuda(), Wk.cuda(), st, ln, mode, return_scores=True,
                                      force_diagonal=fd, **kw)
    assert 32 * w.nb >= 8 * 148
    s = sc.cpu().double().numpy()
    s_ref = oracle.gate_varlen(Q, K, Wq, Wk, starts, lens)
    rowmax = np.maximum(s_ref.max(-1, keepdims=True), 1e-30)
    assert (np.abs(s - s_ref) / rowmax).max() <= SCORE_RTOL
    c_ref, i_ref = oracle.select_varlen(sc.cpu(), starts, lens, mode, force_diag=fd, cap=ix.shape[-1], **kw)
    _lists_equal(c.cpu().numpy(), ix.cpu().numpy(), c_ref, i_ref)


@pytest.mark.parametrize("dtype,d", [("fp32", 64), ("bf16", 64)])
def test_gate_varlen_rope_and_dtypes(dtype, d):
    """Block RoPE at packed positions equals the per-sequence oracle's local
    positions (RoPE scores depend on i - j only)."""
    lens, gaps = [200, 700, 64], [1, 0, 3]
    w, starts, n, Q, K, V, Wq, Wk = _varlen_case(lens, gaps, dtype=dtype, d=d, pad="zero")
    st = torch.tensor(starts, dtype=torch.int32, device="cuda")
    ln = torch.tensor(lens, dtype=torch.int32, device="cuda")
    c, ix, sc = seer.seer_gate_varlen(Q.cuda(), K.cuda(), Wq.cuda(), Wk.cuda(), st, ln, "topk", k=4,
                                      rope_theta=500000.0, return_scores=True)
    s_ref = oracle.gate_varlen(Q, K, Wq, Wk, starts, lens, rope_theta=500000.0)
    rowmax = np.maximum(s_ref.max(-1, keepdims=True), 1e-30)
    assert (np.abs(sc.cpu().double().numpy() - s_ref) / rowmax).max() <= SCORE_RTOL
    c_ref, i_ref = oracle.select_varlen(sc.cpu(), starts, lens, oracle.MODE_TOPK_K, k=4, cap=ix.shape[-1])
    _lists_equal(c.cpu().numpy(), ix.cpu().numpy(), c_ref, i_ref)


@pytest.mark.parametrize("lens,gaps", LAYOUTS)
def test_sparse_attn_on_packed_sequences(lens, gaps):
    """The varlen lists drive the unchanged sparse attention on the packed
    buffer: every sequence's rows match per-sequence attention; blocks of no
    sequence get O = 0 and LSE = -inf; finite noise in the padding changes
    nothing."""
    w, starts, n, Q, K, V, Wq, Wk = _varlen_case(lens, gaps, pad="zero", Hq=4, Hkv=2)
    st = torch.tensor(starts, dtype=torch.int32, device="cuda")
    ln = torch.tensor(lens, dtype=torch.int32, device="cuda")
    c, ix = seer.seer_gate_varlen(Q.cuda(), K.cuda(), Wq.cuda(), Wk.cuda(), st, ln, "density", density=0.5,
                                  force_diagonal=True)
    O, lse = seer.seer_sparse_attn(Q.cuda(), K.cuda(), V.cuda(), c, ix)
    O_ref, lse_ref = oracle.sparse_attn_varlen(Q, K, V, c.cpu().numpy(), ix.cpu().numpy(), starts, lens)
    inside = ~np.isnan(lse_ref[0, 0])
    check_o(O.cpu().double().numpy()[:, :, inside], O_ref[:, :, inside])
    check_lse(lse.cpu().double().numpy()[:, :, inside], lse_ref[:, :, inside], LSE_TOL)
    # blocks of no sequence: empty rows
    cn = c.cpu().numpy()[0, 0]
    for b in np.nonzero(cn == 0)[0]:
        assert torch.all(O[:, :, 64 * b:64 * (b + 1)] == 0)
        assert torch.all(lse[:, :, 64 * b:64 * (b + 1)] == float("-inf"))
    # padding holding noise: the sequences' rows are bit-identical
    _, _, _, Qn, Kn, Vn, _, _ = _varlen_case(lens, gaps, pad="noise", Hq=4, Hkv=2)
    On, lsen = seer.seer_sparse_attn(Qn.cuda(), Kn.cuda(), Vn.cuda(), c, ix)
    assert torch.equal(On[:, :, torch.from_numpy(inside).cuda()], O[:, :, torch.from_numpy(inside).cuda()])


def test_gate_varlen_fp32_attention():
    lens, gaps = [100, 250], [0, 1]
    w, starts, n, Q, K, V, Wq, Wk = _varlen_case(lens, gaps, dtype="fp32", d=64, Hq=4, Hkv=1, pad="zero")
    st = torch.tensor(starts, dtype=torch.int32, device="cuda")
    ln = torch.tensor(lens, dtype=torch.int32, device="cuda")
    c, ix = seer.seer_gate_varlen(Q.cuda(), K.cuda(), Wq.cuda(), Wk.cuda(), st, ln, "threshold", T=0.1,
                                  force_diagonal=True)
    O, lse = seer.seer_sparse_attn(Q.cuda(), K.cuda(), V.cuda(), c, ix)
    Qr, Kr, Vr = (t.to(torch.bfloat16) for t in (Q, K, V))
    O_ref, lse_ref = oracle.sparse_attn_varlen(Qr, Kr, Vr, c.cpu().numpy(), ix.cpu().numpy(), starts, lens)
    inside = ~np.isnan(lse_ref[0, 0])
    check_o(O.cpu().double().numpy()[:, :, inside], O_ref[:, :, inside])
    check_lse(lse.cpu().double().numpy()[:, :, inside], lse_ref[:, :, inside], LSE_TOL_FP32_INPUT)


@pytest.mark.parametrize("start,length", [(32, 40), (0, 0), (0, 10000)])
def test_gate_varlen_bad_table_is_reported(start, length):
    """A start off the 64-token grid, an empty sequence, or one past the
    buffer: recorded as SEER_ERR_DEVICE_CHECK, its blocks left empty."""
    w, starts, n, Q, K, V, Wq, Wk = _varlen_case([200], [0], pad="zero", Hq=4, Hkv=2)
    st = torch.tensor([start], dtype=torch.int32, device="cuda")
    ln = torch.tensor([length], dtype=torch.int32, device="cuda")
    ws = torch.empty(seer.gate_varlen_workspace_size(4, 2, n, 128, 128), dtype=torch.uint8, device="cuda")
    c, ix = seer.seer_gate_varlen(Q.cuda(), K.cuda(), Wq.cuda(), Wk.cuda(), st, ln, "topk", k=2, workspace=ws)
    assert seer.seer_workspace_status(ws) == 6
    assert c.cpu().eq(0).all()


def test_gate_varlen_rejects_batched_dims():
    w = synth.custom("vl", 2, 4, 2, 256, 64, 64, "bf16")
    Q, K, V = synth.make_qkv(w)
    Wq, Wk = synth.make_gate_weights(w)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    ln = torch.full((1,), 256, dtype=torch.int32, device="cuda")
    with pytest.raises(ValueError):
        seer.seer_gate_varlen(Q.cuda(), K.cuda(), Wq.cuda(), Wk.cuda(), st, ln, "topk", k=2)
