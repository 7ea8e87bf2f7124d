"""Shared helpers of the GPU parity tests: cached seeded inputs, unit
sampling, and the tolerances (written here once, used by every test).

Tolerances
  * gate scores: relative 1e-4 of the row's largest score (fp32 pooling,
    projection and softmax against fp64).
  * index lists: bit-exact when the same fp32 scores are supplied; against the
    oracle's own fp64 scores a threshold decision may differ only where
    |s - T| <= 1e-3 T, a top-k decision only where the k_i-th and (k_i+1)-th
    oracle scores are within 1e-3 relative.
  * O: max abs <= 2e-2, mean abs <= 2e-3 (bf16 I/O); LSE: abs <= 1e-3.
  * blockmax map: abs <= 1e-3.
  * fp32 inputs are rounded to bf16 for the tensor cores; that rounding
    (relative 2^-9 per operand) moves a logit by up to 2^-8 * scale *
    sum_c |q_c k_c|, about 4e-3 on the tiny case, so LSE gets 1e-2 there.
"""
from __future__ import annotations

import functools

import numpy as np
import torch

from learned_block_sparse_seer_b200 import synth

SCORE_RTOL = 1e-4
O_MAX, O_MEAN = 2e-2, 2e-3
LSE_TOL = 1e-3
LSE_TOL_FP32_INPUT = 1e-2
BMAX_TOL = 1e-3
BLK = 64


@functools.lru_cache(maxsize=4)
def inputs(name: str):
    w = synth.WORKLOADS[name]
    Q, K, V = synth.make_qkv(w)
    Wq, Wk = synth.make_gate_weights(w)
    return w, Q, K, V, Wq, Wk


def to_dev(*ts):
    return tuple(t.to("cuda:0") for t in ts)


def sample_units(B: int, Hq: int, nb: int, n_random: int, seed: int = 0) -> np.ndarray:
    """First and last query block of every head plus seeded random units."""
    rng = np.random.default_rng(seed)
    units = set()
    for b in range(B):
        for h in (0, Hq - 1):
            base = (b * Hq + h) * nb
            units.update((base, base + nb - 1))
    total = B * Hq * nb
    units.update(int(u) for u in rng.choice(total, size=min(n_random, total), replace=False))
    return np.array(sorted(units), dtype=np.int64)


def unit_rows(O: torch.Tensor, units: np.ndarray, nb: int):
    """Gather the 64 rows of each unit from [B, H, n, ...] into [U, 64, ...]."""
    B, H, n = O.shape[:3]
    flat = O.reshape(B * H, n, *O.shape[3:])
    out = []
    for u in units:
        bh, i = divmod(int(u), nb)
        out.append(flat[bh, i * BLK:(i + 1) * BLK])
    return torch.stack(out)


def check_o(O_gpu: np.ndarray, O_ref: np.ndarray, what: str = "O"):
    err = np.abs(O_gpu.astype(np.float64) - O_ref)
    assert err.max() <= O_MAX, f"{what}: max abs error {err.max():.3e} > {O_MAX}"
    assert err.mean() <= O_MEAN, f"{what}: mean abs error {err.mean():.3e} > {O_MEAN}"
    return err


def check_lse(l_gpu: np.ndarray, l_ref: np.ndarray, tol: float = LSE_TOL):
    fin = np.isfinite(l_ref)
    assert np.array_equal(np.isfinite(l_gpu), fin), "LSE finiteness differs (empty rows)"
    assert np.all(l_gpu[~fin] == -np.inf)
    if fin.any():
        e = np.abs(l_gpu[fin].astype(np.float64) - l_ref[fin]).max()
        assert e <= tol, f"LSE abs error {e:.3e} > {tol}"


def lists_equal(c_gpu, i_gpu, c_ref, i_ref):
    c_gpu = np.asarray(c_gpu)
    assert np.array_equal(c_gpu, c_ref), "counts differ"
    for r in zip(*np.nonzero(c_ref)):
        k = c_ref[r]
        assert np.array_equal(i_gpu[r][:k], i_ref[r][:k]), f"lists differ at row {r}"
