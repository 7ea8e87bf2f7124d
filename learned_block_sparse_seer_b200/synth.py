"""Seeded synthetic inputs for the SeerAttention prefill path.

This module is the only code shared by the CUDA path and the fp64 oracle: it
draws random tensors and plants block structure in them.  It holds none of the
method's arithmetic (no pooling, scoring, selection or attention).

Shapes follow the Llama-3.1-8B attention layer that SeerAttention is evaluated
on (SeerAttention, section 3.4 "Input and pooling": per-head dimension 128,
32 query heads sharing 8 KV heads).  The pages evaluate on PG19 / RULER /
LongBench prompts through that model; those are not available here, so these
tensors stand in for them, with the structures the pages describe attention as
having (SeerAttention, section 4, Figure 8: attention sinks / A-shapes, local
diagonals and vertical stripes).

Layout of every tensor is [B, H, n, d], contiguous, row-major.

Recipe (all draws from ``torch.Generator('cpu').manual_seed(seed)``, fp32):
  * Q, K, V ~ N(0, 1), drawn in that order.
  * ``tiny`` structure: u = one random unit vector; for the single KV head the
    key rows of block 0 and of 2 distinct random blocks in 1..nb-1 get +3u.
  * ``layer`` structure (per KV head g, for every batch entry):
      - sink:   K[g, block 0] += 3u, and every query row of g's query heads
                gets +0.5u;
      - local band of 4 blocks: e_m (m = 0..nb+2) random unit vectors shared
                by all heads; Q[block i] += 2 e_i for every query head and
                K[g, block j] += 2 (e_j + e_{j+1} + e_{j+2} + e_{j+3}), so q.k
                is raised for key blocks j in [i-3, i];
      - vertical stripes: ceil(0.05 nb) random key blocks in 1..nb-1 get
                K += 3 w_g (w_g a unit vector per KV head) and g's query heads
                get +0.5 w_g on every row.
  * bf16 configurations round Q, K, V once; the oracle consumes the rounded
    values (upcast exactly to fp32).
  * Gate weights Wq [Hq, h, d] and Wk [Hkv, h, 3d] ~ N(0, 0.02), fp32, from a
    second generator seeded with seed + 100.
  * ``decode`` structure (one new token per (batch, query head) against a KV
    cache of capacity n holding seq_len tokens; make_decode): K, V ~ N(0, 1)
    [B, Hkv, n, d] and q ~ N(0, 1) [B, Hq, d], drawn in that order; per KV
    head g the layer's sink (K block 0 += 3u, q += 0.5u) and vertical stripes
    (ceil(0.05 nb) random blocks += 3 w_g, q += 0.5 w_g), and for the token's
    local window the key blocks c-3 .. c (c = (seq_len-1) // 64) get
    += 2 e_g with q += 2 e_g; cache rows at positions >= seq_len are set to
    NaN, so any read past the token shows up in the result.
"""
from __future__ import annotations

import dataclasses
import math

import torch

BLOCK = 64


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    Hq: int
    Hkv: int
    n: int
    d: int
    h: int
    dtype: str  # "fp32" or "bf16"
    structure: str  # "tiny" or "layer"
    seed: int

    @property
    def nb(self) -> int:
        return self.n // BLOCK

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv


# The workloads: a tiny parity case, the Llama-3.1-8B-shaped layer at 8k, 32k
# and 128k tokens, and the ground-truth (blockmax) cases.
WORKLOADS = {
    "tiny": Workload("tiny", 1, 2, 1, 512, 64, 64, "fp32", "tiny", 0),
    "layer8k": Workload("layer8k", 1, 32, 8, 8192, 128, 128, "bf16", "layer", 1),
    "layer32k": Workload("layer32k", 1, 32, 8, 32768, 128, 128, "bf16", "layer", 2),
    "layer128k": Workload("layer128k", 1, 32, 8, 131072, 128, 128, "bf16", "layer", 3),
    "bmax4k": Workload("bmax4k", 4, 32, 8, 4096, 128, 128, "bf16", "layer", 4),
    "bmax32k": Workload("bmax32k", 1, 32, 8, 32768, 128, 128, "bf16", "layer", 5),
    # decode: the layer's heads against a 128k-token KV cache
    "decode128k": Workload("decode128k", 1, 32, 8, 131072, 128, 128, "bf16", "decode", 6),
}

# Tokens in the decode cache by default: 37 short of capacity, so the token's
# own block is partial.
DECODE_TAIL = 37


def custom(name: str, B: int, Hq: int, Hkv: int, n: int, d: int, h: int,
           dtype: str = "bf16", structure: str = "layer", seed: int = 7) -> Workload:
    """A workload with arbitrary shapes (used for edge-case tests)."""
    assert n % BLOCK == 0 and Hq % Hkv == 0
    return Workload(name, B, Hq, Hkv, n, d, h, dtype, structure, seed)


def _unit(g: torch.Generator, *shape: int) -> torch.Tensor:
    v = torch.randn(*shape, generator=g)
    return v / v.norm(dim=-1, keepdim=True)


def make_qkv(w: Workload):
    """Return (Q, K, V) as CPU tensors of w.dtype, shape [B, H, n, d]."""
    g = torch.Generator("cpu").manual_seed(w.seed)
    Q = torch.randn(w.B, w.Hq, w.n, w.d, generator=g)
    K = torch.randn(w.B, w.Hkv, w.n, w.d, generator=g)
    V = torch.randn(w.B, w.Hkv, w.n, w.d, generator=g)
    nb, G = w.nb, w.G
    u = _unit(g, w.d)
    Qb = Q.view(w.B, w.Hq, nb, BLOCK, w.d)
    Kb = K.view(w.B, w.Hkv, nb, BLOCK, w.d)
    if w.structure == "tiny":
        for kv in range(w.Hkv):
            extra = torch.randperm(nb - 1, generator=g)[:2] + 1 if nb > 1 else torch.empty(0, dtype=torch.long)
            blocks = [0] + [int(b) for b in extra]
            for j in blocks:
                Kb[:, kv, j] += 3.0 * u
    elif w.structure == "layer":
        e = _unit(g, nb + 3, w.d)
        band = e[0:nb] + e[1:nb + 1] + e[2:nb + 2] + e[3:nb + 3]
        n_stripes = math.ceil(0.05 * nb)
        for kv in range(w.Hkv):
            heads = slice(kv * G, (kv + 1) * G)
            # sink
            Kb[:, kv, 0] += 3.0 * u
            Q[:, heads] += 0.5 * u
            # vertical stripes
            wv = _unit(g, w.d)
            if nb > 1:
                stripes = torch.randperm(nb - 1, generator=g)[:n_stripes] + 1
                Kb[:, kv, stripes] += 3.0 * wv
            Q[:, heads] += 0.5 * wv
            # local band
            Kb[:, kv] += 2.0 * band[:, None, :]
        Qb += 2.0 * e[0:nb][None, None, :, None, :]
    else:
        raise ValueError(w.structure)
    if w.dtype == "bf16":
        Q, K, V = (t.to(torch.bfloat16) for t in (Q, K, V))
    return Q.contiguous(), K.contiguous(), V.contiguous()


def make_gate_weights(w: Workload):
    """Return (Wq [Hq, h, d], Wk [Hkv, h, 3d]) fp32 CPU tensors ~ N(0, 0.02)."""
    g = torch.Generator("cpu").manual_seed(w.seed + 100)
    Wq = torch.randn(w.Hq, w.h, w.d, generator=g) * 0.02
    Wk = torch.randn(w.Hkv, w.h, 3 * w.d, generator=g) * 0.02
    return Wq.contiguous(), Wk.contiguous()


def make_scores_like(w: Workload, seed: int = 11, ties: bool = False):
    """Random fp32 arrays shaped like gate scores [B, Hq, nb, nb].

    Used to drive the selection step directly.  Each causal row is a random
    positive vector normalised to sum to 1 over j <= i (entries above the
    diagonal are 0).  With ``ties`` the values are quantised to a few levels
    so that equal scores occur.
    """
    g = torch.Generator("cpu").manual_seed(seed)
    x = torch.rand(w.B, w.Hq, w.nb, w.nb, generator=g, dtype=torch.float64)
    if ties:
        x = torch.floor(x * 4) + 1
    tri = torch.tril(torch.ones(w.nb, w.nb, dtype=torch.float64))
    x = x * tri
    x = x / x.sum(-1, keepdim=True)
    return x.to(torch.float32).contiguous()


def decode_seq_len(w: Workload) -> int:
    return w.n - DECODE_TAIL


def make_decode(w: Workload, seq_len: int | None = None):
    """Return (q [B, Hq, d], Kc, Vc [B, Hkv, n, d]) CPU tensors of w.dtype for
    a token at position seq_len - 1 (default n - 37)."""
    seq_len = decode_seq_len(w) if seq_len is None else seq_len
    assert 1 <= seq_len <= w.n
    g = torch.Generator("cpu").manual_seed(w.seed)
    K = torch.randn(w.B, w.Hkv, w.n, w.d, generator=g)
    V = torch.randn(w.B, w.Hkv, w.n, w.d, generator=g)
    q = torch.randn(w.B, w.Hq, w.d, generator=g)
    nb, G = w.nb, w.G
    c = (seq_len - 1) // BLOCK
    Kb = K.view(w.B, w.Hkv, nb, BLOCK, w.d)
    u = _unit(g, w.d)
    n_stripes = math.ceil(0.05 * nb)
    for kv in range(w.Hkv):
        heads = slice(kv * G, (kv + 1) * G)
        Kb[:, kv, 0] += 3.0 * u
        q[:, heads] += 0.5 * u
        wv = _unit(g, w.d)
        if nb > 1:
            stripes = torch.randperm(nb - 1, generator=g)[:n_stripes] + 1
            Kb[:, kv, stripes] += 3.0 * wv
        q[:, heads] += 0.5 * wv
        e = _unit(g, w.d)
        Kb[:, kv, max(0, c - 3):c + 1] += 2.0 * e
        q[:, heads] += 2.0 * e
    K[:, :, seq_len:] = float("nan")
    V[:, :, seq_len:] = float("nan")
    if w.dtype == "bf16":
        q, K, V = (t.to(torch.bfloat16) for t in (q, K, V))
    return q.contiguous(), K.contiguous(), V.contiguous()


def varlen_layout(lens, gap_blocks=None):
    """Packed variable-length layout: sequence s starts at the first 64-token
    boundary after sequence s - 1 plus gap_blocks[s] empty blocks.  Returns
    (starts, n) with n the packed length (a multiple of 64)."""
    gap_blocks = [0] * len(lens) if gap_blocks is None else gap_blocks
    starts, pos = [], 0
    for l, gb in zip(lens, gap_blocks):
        pos += gb * BLOCK
        starts.append(pos)
        pos += ((l + BLOCK - 1) // BLOCK) * BLOCK
    return starts, pos


def make_varlen(w: Workload, starts, lens, pad: str = "zero"):
    """(Q, K, V) [1, H, w.n, d] for a packed layout: w's recipe over the whole
    buffer, then every token outside the sequences set by `pad`: "zero",
    "nan", or "noise" (fresh N(0, 1) draws from seed + 200)."""
    assert w.B == 1
    Q, K, V = (t.float() for t in make_qkv(Workload(w.name, 1, w.Hq, w.Hkv, w.n, w.d, w.h, "fp32",
                                                     w.structure, w.seed)))
    inside = torch.zeros(w.n, dtype=torch.bool)
    for a, l in zip(starts, lens):
        inside[a:a + l] = True
    out = []
    g = torch.Generator("cpu").manual_seed(w.seed + 200)
    for t in (Q, K, V):
        t = t.clone()
        if pad == "zero":
            t[:, :, ~inside] = 0.0
        elif pad == "nan":
            t[:, :, ~inside] = float("nan")
        elif pad == "noise":
            t[:, :, ~inside] = torch.randn(t.shape[0], t.shape[1], int((~inside).sum()), t.shape[3], generator=g)
        else:
            raise ValueError(pad)
        out.append(t.to(torch.bfloat16) if w.dtype == "bf16" else t)
    return tuple(o.contiguous() for o in out)
