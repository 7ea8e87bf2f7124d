"""CPU check of the numerical claim behind the gate's tensor-core logits:
splitting each fp32 operand into a tf32 part (rounded to nearest, 10
mantissa bits) and its fp32 remainder, and forming hi*hi + hi*lo + lo*hi on
a tf32 multiplier (which reads the top 19 bits of each operand, truncated or
rounded), keeps the dot products within about 2^-20 of sum|a b| -- the
fp32-level accuracy the gate's 1e-4 score tolerance needs.  Plain numpy, no
GPU; it checks the arithmetic, not the kernel (the GPU tests do that)."""
import numpy as np
import pytest


def _tf32_round(x):
    """Round fp32 to the nearest tf32 value (ties away from zero)."""
    b = x.astype(np.float32).view(np.uint32).astype(np.uint64)
    b = (b + 0x1000) & 0xFFFFE000
    return b.astype(np.uint32).view(np.float32)


def _tf32_trunc(x):
    b = x.astype(np.float32).view(np.uint32) & np.uint32(0xFFFFE000)
    return b.view(np.float32)


@pytest.mark.parametrize("read", [_tf32_trunc, _tf32_round])
def test_three_product_split_keeps_fp32_accuracy(read):
    rng = np.random.default_rng(0)
    a = rng.standard_normal((512, 128)).astype(np.float32) * rng.uniform(0.01, 10, (512, 1)).astype(np.float32)
    b = rng.standard_normal((512, 128)).astype(np.float32)
    ah = _tf32_round(a)
    al = (a - ah).astype(np.float32)
    bh = _tf32_round(b)
    bl = (b - bh).astype(np.float32)
    # the remainders are exact in fp32 and small
    assert np.all(np.abs(al) <= np.abs(a) * 2.0 ** -11 + 1e-45)
    A, Al, B, Bl = (read(x).astype(np.float64) for x in (ah, al, bh, bl))
    assert np.array_equal(A, ah.astype(np.float64))  # the tf32 parts pass unchanged
    approx = A @ B.T + A @ Bl.T + Al @ B.T  # products exact in fp64; accumulation order aside
    exact = a.astype(np.float64) @ b.astype(np.float64).T
    scale = np.abs(a).astype(np.float64) @ np.abs(b).astype(np.float64).T
    rel = np.abs(approx - exact) / scale
    assert rel.max() <= 2.0 ** -20
    # one tf32 product alone is about three orders of magnitude worse
    one = A @ B.T
    assert (np.abs(one - exact) / scale).max() > 2.0 ** -14


def test_tf32_attention_tolerance_covers_tf32_arithmetic():
    """The tolerances of the tf32 attention parity tests (tests/test_gpu_tf32.py,
    _bounds) against the arithmetic they describe: Q, K, V and the
    probabilities P read as tf32 (truncated to 10 mantissa bits), every
    product and sum exact (fp64), compared with exact fp64 causal attention.
    The row sums use P before the tensor core reads it, as the kernel's
    softmax threads do."""
    import torch
    from test_gpu_tf32 import _bounds

    rng = np.random.default_rng(3)
    B, H, n, d = 1, 2, 256, 128
    Q = rng.standard_normal((B, H, n, d)).astype(np.float32)
    K = rng.standard_normal((B, H, n, d)).astype(np.float32)
    V = rng.standard_normal((B, H, n, d)).astype(np.float32)
    K[:, :, 64:72] *= 3.0  # a few keys well above the rest: peaked rows
    scale = 1.0 / np.sqrt(d)
    causal = np.tril(np.ones((n, n), dtype=bool))

    def attn(q, k, v, read_p):
        s = np.where(causal, (q @ np.swapaxes(k, -1, -2)) * scale, -np.inf)
        m = s.max(-1, keepdims=True)
        p = np.exp(s - m)
        lsum = p.sum(-1, keepdims=True)
        o = (read_p(p) @ v) / lsum
        return o, (m + np.log(lsum))[..., 0]

    def t(x):
        return _tf32_trunc(x.astype(np.float32)).astype(np.float64)

    f64 = [x.astype(np.float64) for x in (Q, K, V)]
    O_ex, L_ex = attn(*f64, lambda p: p)
    O_tf, L_tf = attn(t(Q), t(K), t(V), t)
    O_MAX, O_MEAN, LSE_MAX = _bounds(torch.from_numpy(Q), torch.from_numpy(K), torch.from_numpy(V))
    eo, el = np.abs(O_tf - O_ex), np.abs(L_tf - L_ex)
    assert eo.max() <= O_MAX and eo.mean() <= O_MEAN, (eo.max(), eo.mean(), O_MAX)
    assert el.max() <= LSE_MAX, (el.max(), LSE_MAX)
    # and the arithmetic does move the result: the bound is not vacuous
    assert eo.max() > O_MAX / 1000


def test_bf16_attention_tolerance_covers_bf16_rounding():
    """The fixed O tolerances of the bf16 attention parity tests
    (tests/gpu_common.py) against the rounding the path adds on bf16 inputs:
    P rounded to bf16 for the PV product, the row sums taken before that
    rounding, O rounded to bf16 on output; a layer-structured bf16 case with
    the oracle gate's density-0.3 lists, against the fp64 oracle."""
    import torch
    import oracle
    from gpu_common import O_MAX, O_MEAN
    from learned_block_sparse_seer_b200 import synth

    w = synth.Workload("t", 1, 4, 1, 2048, 128, 128, "bf16", "layer", 7)
    Q, K, V = synth.make_qkv(w)
    Wq, Wk = synth.make_gate_weights(w)
    c, ix, _ = oracle.select(oracle.gate(Q, K, Wq, Wk), oracle.MODE_TOPK_DENSITY, density=0.3)
    O_ref, _ = oracle.sparse_attn(Q, K, V, c, ix)

    def bf16(x):
        return torch.from_numpy(np.ascontiguousarray(x)).float().to(torch.bfloat16).double().numpy()

    q, k, v = (t.double().numpy() for t in (Q, K, V))
    O = np.empty_like(O_ref)
    for h in range(w.Hq):
        g = h // w.G
        for i in range(w.nb):
            keys = (ix[0, h, i, :c[0, h, i]][:, None] * 64 + np.arange(64)[None, :]).reshape(-1)
            s = (q[0, h, 64 * i:64 * i + 64] @ k[0, g, keys].T) / np.sqrt(w.d)
            s = np.where(keys[None, :] <= 64 * i + np.arange(64)[:, None], s, -np.inf)
            p = np.exp(s - s.max(-1, keepdims=True))
            O[0, h, 64 * i:64 * i + 64] = bf16((bf16(p) @ v[0, g, keys]) / p.sum(-1, keepdims=True))
    e = np.abs(O - O_ref)
    assert e.max() <= O_MAX and e.mean() <= O_MEAN, (e.max(), e.mean())
    assert e.max() > O_MAX / 100  # the rounding is visible against the bound
