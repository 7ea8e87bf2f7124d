"""fp64 CPU oracle for the SeerAttention prefill path (test infrastructure).

Only the tests, the package smoke check and the benchmark's CPU-baseline leg
may import this package.  The product path (the CUDA library and its Python
binding) never does, and this package never imports the product.

The arithmetic lives in ``seer_oracle.c`` (plain C, fp64, OpenMP); this module
compiles it with gcc and marshals numpy arrays.  Every entry point names the
passage of "SeerAttention: Learning Intrinsic Sparse Attention in Your LLMs"
it follows (paper-graph summary page, section 3.4; OpenReview rebuttal,
section 3.3).

Parity status: block RoPE's base reading (theta' = theta / B) is "parity
unpinned"; every other function is pinned by the CPU tests.
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "seer_oracle.c")
_LIB = os.path.join(_HERE, "libseer_oracle.so")
BLOCK = 64

_lib = None


def build(force: bool = False) -> str:
    """Compile the C oracle into oracle/libseer_oracle.so (gcc, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        P = ctypes.c_void_p
        I = ctypes.c_int64
        D = ctypes.c_double
        F = ctypes.c_float
        lib.orc_pool_q.argtypes = [P, I, I, I, I, P]
        lib.orc_pool_k.argtypes = [P, I, I, I, I, P]
        lib.orc_project.argtypes = [P, P, I, I, I, I, I, P]
        lib.orc_block_rope.argtypes = [P, I, I, I, D, I]
        lib.orc_gate_scores.argtypes = [P, P, I, I, I, I, I, D, P]
        lib.orc_select_threshold.argtypes = [P, I, I, F, P, P, I, P, ctypes.c_int]
        lib.orc_select_threshold.restype = I
        lib.orc_select_topk.argtypes = [P, I, I, ctypes.c_int, I, F, P, P, I, P, ctypes.c_int]
        lib.orc_gate_scores_units.argtypes = [P, P, I, I, I, I, I, D, P, I, P]
        lib.orc_select_topk.restype = I
        lib.orc_topk_count.argtypes = [I, ctypes.c_int, I, F]
        lib.orc_topk_count.restype = I
        lib.orc_sparse_attn_units.argtypes = [P, P, P, I, I, I, I, I, I, P, P, I, D, P, I, P, P]
        lib.orc_sparse_attn.argtypes = [P, P, P, I, I, I, I, I, I, P, P, I, D, P, P]
        lib.orc_blockmax_units.argtypes = [P, P, I, I, I, I, I, I, D, P, I, P, P]
        lib.orc_blockmax.argtypes = [P, P, I, I, I, I, I, I, D, P, P]
        lib.orc_num_threads.restype = ctypes.c_int
        _lib = lib
    return _lib


def _f32(x) -> np.ndarray:
    """Contiguous fp32 numpy view of a tensor/array (bf16 is upcast exactly)."""
    try:
        import torch
        if isinstance(x, torch.Tensor):
            x = x.detach().to("cpu")
            if x.dtype != torch.float32:
                x = x.to(torch.float32)
            return np.ascontiguousarray(x.numpy())
    except ImportError:  # pragma: no cover
        pass
    return np.ascontiguousarray(np.asarray(x, dtype=np.float32))


def _f64(x) -> np.ndarray:
    try:
        import torch
        if isinstance(x, torch.Tensor):
            x = x.detach().to("cpu").to(torch.float64)
            return np.ascontiguousarray(x.numpy())
    except ImportError:  # pragma: no cover
        pass
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _p(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def num_threads() -> int:
    return int(_load().orc_num_threads())


# ---------------------------------------------------------------- gate ---
def pool_q(Q) -> np.ndarray:
    """Average pooling of Q per 64-token block (summary page, section 3.4,
    "Input and pooling").  Q [B,H,n,d] -> [B,H,nb,d] fp64."""
    q = _f32(Q)
    B, H, n, d = q.shape
    out = np.empty((B, H, n // BLOCK, d), np.float64)
    _load().orc_pool_q(_p(q), B * H, n, d, BLOCK, _p(out))
    return out


def pool_k(K) -> np.ndarray:
    """Max, min and average pooling of K concatenated as [max|min|avg]
    (summary page, section 3.4, "Pooling Method Selection").
    K [B,H,n,d] -> [B,H,nb,3d] fp64."""
    k = _f32(K)
    B, H, n, d = k.shape
    out = np.empty((B, H, n // BLOCK, 3 * d), np.float64)
    _load().orc_pool_k(_p(k), B * H, n, d, BLOCK, _p(out))
    return out


def project(x, W) -> np.ndarray:
    """Gate linear layer, no bias (summary page, section 3.4, "Linear
    transformation"): y[b,hh,i] = W[hh] @ x[b,hh,i].  W is [H, h, din]."""
    xv = _f64(x)
    w = _f32(W)
    B, H, nb, din = xv.shape
    h = w.shape[1]
    assert w.shape == (H, h, din)
    out = np.empty((B, H, nb, h), np.float64)
    _load().orc_project(_p(xv), _p(w), B, H, nb, din, h, _p(out))
    return out


def block_rope(x, theta: float) -> np.ndarray:
    """Block-level RoPE with base theta / 64 at block positions (summary page,
    section 3.4, "Block-Level RoPE").  Parity unpinned for the base reading."""
    xv = _f64(x).copy()
    B, H, nb, h = xv.shape
    _load().orc_block_rope(_p(xv), B * H, nb, h, float(theta), BLOCK)
    return xv


def gate_scores(qt, kt, d: int) -> np.ndarray:
    """Eq. 1 (summary page, section 3.4): causal row softmax of
    q~ k~^T / sqrt(d) over key blocks j <= i; 0 above the diagonal."""
    q = _f64(qt)
    k = _f64(kt)
    B, Hq, nb, h = q.shape
    Hkv = k.shape[1]
    out = np.empty((B, Hq, nb, nb), np.float64)
    _load().orc_gate_scores(_p(q), _p(k), B, Hq, Hkv, nb, h, 1.0 / math.sqrt(d), _p(out))
    return out


def gate(Q, K, Wq, Wk, rope_theta: float = 0.0) -> np.ndarray:
    """The whole AttnGate (pool, project, optional block RoPE, Eq. 1)."""
    d = Q.shape[-1]
    qt = project(pool_q(Q), Wq)
    kt = project(pool_k(K), Wk)
    if rope_theta > 0:
        qt = block_rope(qt, rope_theta)
        kt = block_rope(kt, rope_theta)
    return gate_scores(qt, kt, d)


# ----------------------------------------------------------- selection ---
MODE_THRESHOLD, MODE_TOPK_K, MODE_TOPK_DENSITY = 0, 1, 2


def select(scores, mode: int, T: float = 0.0, k: int = 0, density: float = 0.0,
           cap: int | None = None, force_diag: bool = False):
    """Binary block mask as ascending index lists (summary page, section 3.4,
    "Generating the binary block mask"; rebuttal section 3.3).  With
    force_diag the diagonal block joins every row's list (an option the
    pages do not use).  Returns (counts [B,Hq,nb] int32, idx [B,Hq,nb,cap]
    int32 padded with -1, worst) where worst is the largest per-row count
    before truncation."""
    s = _f64(scores)
    B, Hq, nb, _ = s.shape
    cap = nb if cap is None else cap
    rows = B * Hq * nb
    counts = np.zeros((B, Hq, nb), np.int32)
    idx = np.full((B, Hq, nb, cap), -1, np.int32)
    lib = _load()
    fd = 1 if force_diag else 0
    if mode == MODE_THRESHOLD:
        worst = lib.orc_select_threshold(_p(s), rows, nb, float(T), _p(counts), _p(idx), cap, None, fd)
    else:
        worst = lib.orc_select_topk(_p(s), rows, nb, int(mode), int(k), float(density),
                                    _p(counts), _p(idx), cap, None, fd)
    return counts, idx, int(worst)


def select_rows(rows_scores, row_i, mode: int, T: float = 0.0, k: int = 0, density: float = 0.0,
                cap: int | None = None, force_diag: bool = False):
    """As select, for a stack of score rows [R, nb] whose query blocks are
    given by row_i [R].  Returns (counts [R], idx [R, cap])."""
    s = _f64(rows_scores)
    R, nb = s.shape
    ri = np.ascontiguousarray(row_i, dtype=np.int64)
    cap = nb if cap is None else cap
    counts = np.zeros(R, np.int32)
    idx = np.full((R, cap), -1, np.int32)
    lib = _load()
    fd = 1 if force_diag else 0
    if mode == MODE_THRESHOLD:
        lib.orc_select_threshold(_p(s), R, nb, float(T), _p(counts), _p(idx), cap, _p(ri), fd)
    else:
        lib.orc_select_topk(_p(s), R, nb, int(mode), int(k), float(density), _p(counts), _p(idx),
                            cap, _p(ri), fd)
    return counts, idx


def gate_scores_units(qt, kt, d: int, units) -> np.ndarray:
    """Eq. 1 for the listed rows u = (b*Hq + hq)*nb + i: [len(units), nb]."""
    q = _f64(qt)
    k = _f64(kt)
    B, Hq, nb, h = q.shape
    Hkv = k.shape[1]
    u = np.ascontiguousarray(units, dtype=np.int64)
    out = np.empty((len(u), nb), np.float64)
    _load().orc_gate_scores_units(_p(q), _p(k), B, Hq, Hkv, nb, h, 1.0 / math.sqrt(d), _p(u),
                                  len(u), _p(out))
    return out


def topk_count(i: int, mode: int, k: int = 0, density: float = 0.0) -> int:
    return int(_load().orc_topk_count(i, mode, k, density))


# ----------------------------------------------------------- attention ---
def sparse_attn(Q, K, V, counts, idx, scale: float | None = None):
    """Block-sparse causal attention (summary page, section 3.4,
    "Block-sparse FlashAttention kernel").  Returns (O [B,Hq,n,d], lse
    [B,Hq,n]) in fp64; rows with no admissible key get O = 0, lse = -inf."""
    q, k, v = _f32(Q), _f32(K), _f32(V)
    B, Hq, n, d = q.shape
    Hkv = k.shape[1]
    c = np.ascontiguousarray(counts, dtype=np.int32)
    ix = np.ascontiguousarray(idx, dtype=np.int32)
    cap = ix.shape[-1]
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    O = np.empty((B, Hq, n, d), np.float64)
    lse = np.empty((B, Hq, n), np.float64)
    _load().orc_sparse_attn(_p(q), _p(k), _p(v), B, Hq, Hkv, n, d, BLOCK, _p(c), _p(ix), cap,
                            scale, _p(O), _p(lse))
    return O, lse


def sparse_attn_units(Q, K, V, counts, idx, units, scale: float | None = None):
    """As sparse_attn, for the listed units u = (b*Hq + hq)*nb + i only.
    Returns (O [len(units), 64, d], lse [len(units), 64])."""
    q, k, v = _f32(Q), _f32(K), _f32(V)
    B, Hq, n, d = q.shape
    Hkv = k.shape[1]
    c = np.ascontiguousarray(counts, dtype=np.int32)
    ix = np.ascontiguousarray(idx, dtype=np.int32)
    cap = ix.shape[-1]
    u = np.ascontiguousarray(units, dtype=np.int64)
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    O = np.empty((len(u), BLOCK, d), np.float64)
    lse = np.empty((len(u), BLOCK), np.float64)
    _load().orc_sparse_attn_units(_p(q), _p(k), _p(v), B, Hq, Hkv, n, d, BLOCK, _p(c), _p(ix),
                                  cap, scale, _p(u), len(u), _p(O), _p(lse))
    return O, lse


def dense_lists(B: int, Hq: int, nb: int):
    """All-ones causal mask as lists: row i lists 0..i."""
    counts = np.broadcast_to(np.arange(1, nb + 1, dtype=np.int32), (B, Hq, nb)).copy()
    idx = np.broadcast_to(np.arange(nb, dtype=np.int32), (B, Hq, nb, nb)).copy()
    return counts, idx


def blockmax(Q, K, scale: float | None = None):
    """2D max-pooled causal attention probabilities (summary page, section
    3.4, "Ground truth generation").  Returns (gt [B,Hq,nb,nb], lse)."""
    q, k = _f32(Q), _f32(K)
    B, Hq, n, d = q.shape
    Hkv = k.shape[1]
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    gt = np.empty((B, Hq, n // BLOCK, n // BLOCK), np.float64)
    lse = np.empty((B, Hq, n), np.float64)
    _load().orc_blockmax(_p(q), _p(k), B, Hq, Hkv, n, d, BLOCK, scale, _p(gt), _p(lse))
    return gt, lse


def blockmax_units(Q, K, units, scale: float | None = None):
    """As blockmax for the listed units: (gt rows [len, nb], lse [len, 64])."""
    q, k = _f32(Q), _f32(K)
    B, Hq, n, d = q.shape
    Hkv = k.shape[1]
    u = np.ascontiguousarray(units, dtype=np.int64)
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    gt = np.empty((len(u), n // BLOCK), np.float64)
    lse = np.empty((len(u), BLOCK), np.float64)
    _load().orc_blockmax_units(_p(q), _p(k), B, Hq, Hkv, n, d, BLOCK, scale, _p(u), len(u),
                               _p(gt), _p(lse))
    return gt, lse


# ------------------------------------------------ gate distillation loss ---
def gate_kl(scores, gt):
    """KL(gt || score) per query-block row and its gradient with respect to
    the gate's logits (summary page, section 3.4, "Loss function:
    KL-divergence"; Eq. 1 for the score).

    Reading: the page treats both maps as row distributions, so each gt row
    is divided by its sum over the causal blocks j <= i before the
    divergence; the loss is the mean over all rows (batch x query head x
    query block).  With g the normalised row and s the score row,
    loss_row = sum_j g_j (log g_j - log s_j), terms with g_j = 0 being 0, and
    d loss / d z_ij = (s_ij - g_ij) / rows, since s = softmax(z) over j <= i
    and sum_j g_j = 1.  Returns (loss, dz [B,Hq,nb,nb], 0 above the diagonal).
    """
    s = _f64(scores)
    g = _f64(gt)
    B, Hq, nb, _ = s.shape
    causal = np.tril(np.ones((nb, nb), dtype=bool))
    g = np.where(causal, g, 0.0)
    gn = g / g.sum(axis=-1, keepdims=True)
    with np.errstate(divide="ignore", invalid="ignore"):
        terms = np.where(gn > 0, gn * (np.log(gn) - np.log(np.where(causal, s, 1.0))), 0.0)
    rows = B * Hq * nb
    loss = terms.sum() / rows
    dz = np.where(causal, (s - gn) / rows, 0.0)
    return loss, dz


def gate_kl_backward(Q, K, Wq, Wk, gt):
    """The AttnGate's distillation step without RoPE: forward (pooling,
    projection, Eq. 1), KL(gt || score) and the gradients of the loss with
    respect to Wq [Hq,h,d] and Wk [Hkv,h,3d] (summary page, section 3.4:
    only the gate's linear layers are trained).  Chain rule through
    z_ij = q~_i . k~_j / sqrt(d), q~ = Wq qbar, k~ = Wk kbar:
      dq~_i = sum_j dz_ij k~_j / sqrt(d),  dk~_j = sum_{heads of g} sum_i dz_ij q~_i / sqrt(d),
      dWq[hq] = sum_{b,i} dq~_i qbar_i^T,  dWk[g] = sum_{b,j} dk~_j kbar_j^T.
    Returns (loss, dWq, dWk) in fp64."""
    d = Q.shape[-1]
    qb, kb = pool_q(Q), pool_k(K)
    qt, kt = project(qb, Wq), project(kb, Wk)
    s = gate_scores(qt, kt, d)
    loss, dz = gate_kl(s, gt)
    B, Hq, nb, h = qt.shape
    Hkv = kt.shape[1]
    G = Hq // Hkv
    kt_q = np.repeat(kt, G, axis=1)                      # KV head of each query head
    dqt = np.matmul(dz, kt_q) / math.sqrt(d)             # [B,Hq,nb,h]
    dkt_q = np.matmul(np.swapaxes(dz, -1, -2), qt) / math.sqrt(d)
    dkt = dkt_q.reshape(B, Hkv, G, nb, h).sum(axis=2)    # [B,Hkv,nb,h]
    dWq = np.einsum("bhic,bhie->hce", dqt, qb)
    dWk = np.einsum("bgjc,bgje->gce", dkt, kb)
    return loss, dWq, dWk


# --------------------------------------------------------- decode stage ---
# Rebuttal, "decode-stage evaluation": the decode gate drops the Q branch's
# pooling and projection (each token's own Q scores the blocks) and keeps a
# small compressed K cache (pooled after RoPE) for gating; its ground truth is
# the 1D max-pooling of the token's attention row along the sequence.
# Readings: the compressed cache holds k~_j = Wk [max | min | avg](K block j)
# for the complete blocks j < c, where c = (n - 1) // 64 is the block of the
# current token (position n - 1); the current block is always attended and is
# not a selection candidate; no further RoPE is applied (K and Q arrive
# rotated); h = d so that q . k~ is defined; the row softmax and the selection
# rules are the prefill ones over the c candidates.

def decode_kcache(K, Wk, nblocks: int) -> np.ndarray:
    """k~ [B, Hkv, nblocks, h] for key blocks 0 .. nblocks-1 of K."""
    k = _f32(K)
    kb = pool_k(k[:, :, :nblocks * BLOCK])
    return project(kb, Wk)


def decode_gate(q, kt, d: int) -> np.ndarray:
    """Scores [B, Hq, c] = softmax_j(q . k~_j / sqrt(d)) over the c candidate
    blocks (q [B, Hq, d] is the current token's query)."""
    qv = _f64(q)
    kv = _f64(kt)
    B, Hq, _ = qv.shape
    Hkv, c = kv.shape[1], kv.shape[2]
    out = np.zeros((B, Hq, c), np.float64)
    for b in range(B):
        for hq in range(Hq):
            g = hq // (Hq // Hkv)
            z = kv[b, g] @ qv[b, hq] / math.sqrt(d)
            e = np.exp(z - z.max())
            out[b, hq] = e / e.sum()
    return out


def decode_select(scores, mode: int, T: float = 0.0, k: int = 0, density: float = 0.0):
    """Per (b, hq) row, the selected candidate blocks (ascending), by the
    prefill rules applied to a row with c candidates."""
    s = _f64(scores)
    B, Hq, c = s.shape
    rows = s.reshape(B * Hq, c)
    cnt, idx = select_rows(rows, np.full(B * Hq, c - 1, dtype=np.int64), mode, T=T, k=k, density=density)
    return cnt.reshape(B, Hq), idx.reshape(B, Hq, -1)


def decode_attn(q, K, V, n: int, counts, idx, scale: float | None = None):
    """O [B, Hq, d] and LSE [B, Hq] of the current token (position n - 1)
    over the keys of its selected complete blocks and of its own block
    c = (n - 1) // 64 (positions 64c .. n-1)."""
    qv, kv, vv = _f64(q), _f64(K), _f64(V)
    B, Hq, d = qv.shape
    Hkv = kv.shape[1]
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    c = (n - 1) // BLOCK
    O = np.zeros((B, Hq, d), np.float64)
    lse = np.zeros((B, Hq), np.float64)
    for b in range(B):
        for hq in range(Hq):
            g = hq // (Hq // Hkv)
            keys = [np.arange(j * BLOCK, (j + 1) * BLOCK) for j in idx[b, hq, :counts[b, hq]]]
            keys.append(np.arange(c * BLOCK, n))
            ks = np.concatenate(keys)
            z = kv[b, g, ks] @ qv[b, hq] * scale
            m = z.max()
            e = np.exp(z - m)
            O[b, hq] = e @ vv[b, g, ks] / e.sum()
            lse[b, hq] = m + math.log(e.sum())
    return O, lse


def decode_blockmax(q, K, n: int, scale: float | None = None):
    """1D ground truth: gt [B, Hq, c + 1], the maximum of the token's causal
    attention probabilities over each key block (the last block partial),
    and the row's LSE [B, Hq]."""
    qv, kv = _f64(q), _f64(K)
    B, Hq, d = qv.shape
    Hkv = kv.shape[1]
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    c = (n - 1) // BLOCK
    gt = np.zeros((B, Hq, c + 1), np.float64)
    lse = np.zeros((B, Hq), np.float64)
    for b in range(B):
        for hq in range(Hq):
            g = hq // (Hq // Hkv)
            z = kv[b, g, :n] @ qv[b, hq] * scale
            m = z.max()
            l = np.exp(z - m).sum()
            p = np.exp(z - m) / l
            for j in range(c + 1):
                gt[b, hq, j] = p[j * BLOCK:min((j + 1) * BLOCK, n)].max()
            lse[b, hq] = m + math.log(l)
    return gt, lse


# ------------------------------------------------------- varlen packing ---
# Rebuttal (batching): variable-length prefill inputs are packed along the
# sequence axis.  Reading: sequence s occupies tokens start[s] .. start[s] +
# len[s] - 1 of the packed buffer, start[s] a multiple of 64, so every block
# belongs to one sequence.  Each sequence is then its own prefill problem; the
# functions below run the plain definitions on each sequence alone (local
# positions) and place the results at the sequence's blocks.
def _seq_blocks(a: int, l: int):
    return a // BLOCK, (l + BLOCK - 1) // BLOCK


def pool_varlen(X, a: int, l: int, is_k: bool) -> np.ndarray:
    """Pooling over the blocks of one packed sequence; its last block pools
    only the sequence's own tokens.  Q: mean; K: [max | min | mean]."""
    x = _f64(X)[:, :, a:a + l]
    f, nbs = _seq_blocks(a, l)
    outs = []
    for b in range(nbs):
        blk = x[:, :, BLOCK * b:min(BLOCK * (b + 1), l)]
        if is_k:
            outs.append(np.concatenate([blk.max(axis=2), blk.min(axis=2), blk.mean(axis=2)], axis=-1))
        else:
            outs.append(blk.mean(axis=2))
    return np.stack(outs, axis=2)


def gate_varlen(Q, K, Wq, Wk, starts, lens, rope_theta: float = 0.0) -> np.ndarray:
    """The AttnGate per packed sequence: scores [1, Hq, nb, nb] with row i's
    Eq. 1 softmax over its own sequence's blocks f .. i; 0 elsewhere (rows
    of no sequence are all 0)."""
    d = Q.shape[-1]
    nb = Q.shape[2] // BLOCK
    out = np.zeros((1, Q.shape[1], nb, nb), np.float64)
    for a, l in zip(starts, lens):
        f, nbs = _seq_blocks(int(a), int(l))
        qt = project(pool_varlen(Q, int(a), int(l), False), Wq)
        kt = project(pool_varlen(K, int(a), int(l), True), Wk)
        if rope_theta > 0:
            qt = block_rope(qt, rope_theta)
            kt = block_rope(kt, rope_theta)
        out[:, :, f:f + nbs, f:f + nbs] = gate_scores(qt, kt, d)
    return out


def select_varlen(scores, starts, lens, mode: int, T: float = 0.0, k: int = 0, density: float = 0.0,
                  force_diag: bool = False, cap: int | None = None):
    """Selection per packed sequence at local rows; lists hold global block
    indices.  Returns (counts [1,Hq,nb], idx [1,Hq,nb,cap] padded with -1)."""
    s = _f64(scores)
    _, Hq, nb, _ = s.shape
    cap = nb if cap is None else cap
    counts = np.zeros((1, Hq, nb), np.int32)
    idx = np.full((1, Hq, nb, cap), -1, np.int32)
    for a, l in zip(starts, lens):
        f, nbs = _seq_blocks(int(a), int(l))
        c, ix, _ = select(np.ascontiguousarray(s[:, :, f:f + nbs, f:f + nbs]), mode, T=T, k=k, density=density,
                          cap=cap, force_diag=force_diag)
        counts[:, :, f:f + nbs] = c
        idx[:, :, f:f + nbs] = np.where(ix >= 0, ix + f, -1)
    return counts, idx


def sparse_attn_varlen(Q, K, V, counts, idx, starts, lens, scale: float | None = None):
    """Block-sparse attention per packed sequence, each on its own tokens
    (the keys of its listed blocks, causal, none past the sequence's end).
    Returns (O [1,Hq,n,d], lse [1,Hq,n]) fp64; positions of no sequence are
    NaN (not defined)."""
    q, k, v = _f64(Q), _f64(K), _f64(V)
    _, Hq, n, d = q.shape
    O = np.full((1, Hq, n, d), np.nan)
    lse = np.full((1, Hq, n), np.nan)
    cn = np.asarray(counts)
    ix = np.asarray(idx)
    for a, l in zip(starts, lens):
        a, l = int(a), int(l)
        f, nbs = _seq_blocks(a, l)
        # the sequence alone, its last block filled out with zeros: keys past
        # its end come after every one of its queries, so the causal rule
        # already leaves them out
        pad = nbs * BLOCK - l
        def seq(x):
            t = x[:, :, a:a + l]
            return np.concatenate([t, np.zeros((1, x.shape[1], pad, d))], axis=2) if pad else t
        loc = np.where(ix[:, :, f:f + nbs] >= 0, ix[:, :, f:f + nbs] - f, -1).astype(np.int32)
        o, ls = sparse_attn(seq(q), seq(k), seq(v), np.ascontiguousarray(cn[:, :, f:f + nbs]),
                            np.ascontiguousarray(loc), scale)
        O[:, :, a:a + l] = o[:, :, :l]
        lse[:, :, a:a + l] = ls[:, :, :l]
    return O, lse
