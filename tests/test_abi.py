"""CPU checks of the C-ABI library: it loads, exports every function that
include/seer.h declares, and its host-side queries and argument validation
work without a GPU (no kernel is launched)."""
import ctypes
import os
import re
import subprocess

import pytest

import learned_block_sparse_seer_b200 as seer
from learned_block_sparse_seer_b200 import _lib
from learned_block_sparse_seer_b200 import build as seer_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "seer.h")


@pytest.fixture(scope="module")
def L():
    seer_build.build()
    return _lib.lib()


def declared_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"SEER_API\s+[\w\s\*]+?\b(seer_\w+)\s*\(", text)))


def test_header_declares_the_four_calls():
    names = declared_functions()
    for fn in ("seer_gate", "seer_gate_select", "seer_sparse_attn", "seer_attn_blockmax"):
        assert fn in names
    assert len(names) >= 12


def test_library_exports_every_declared_symbol(L):
    out = subprocess.check_output(["nm", "-D", "--defined-only", _lib.LIB_PATH]).decode()
    exported = set(re.findall(r"\bT (seer_\w+)", out))
    missing = [f for f in declared_functions() if f not in exported]
    assert not missing, missing
    for f in declared_functions():
        assert hasattr(L, f)


def test_version_and_status_strings(L):
    assert L.seer_version().decode().count(".") == 2
    for code, name in _lib.STATUS_NAMES.items():
        assert L.seer_status_string(code).decode() == name


def test_required_cap():
    nb = 2048
    assert seer.gate_required_cap(1, 32, 8, 64 * nb, 128, "threshold") == nb
    assert seer.gate_required_cap(1, 32, 8, 64 * nb, 128, "topk", k=200) == 200
    assert seer.gate_required_cap(1, 32, 8, 64 * nb, 128, "topk", k=5000) == nb
    assert seer.gate_required_cap(1, 32, 8, 64 * nb, 128, "density", density=0.1) == 205
    assert seer.gate_required_cap(1, 32, 8, 64 * nb, 128, "density", density=1.5) == -1
    assert seer.gate_required_cap(1, 32, 8, 100, 128, "topk", k=3) == -1  # n % 64 != 0


def test_workspace_sizes_cover_their_buffers():
    B, Hq, Hkv, n, d, h = 1, 32, 8, 8192, 128, 128
    nb = n // 64
    g = seer.gate_workspace_size(B, Hq, Hkv, n, d, h)
    need = 4 * (B * Hq * nb * d + B * Hkv * nb * 3 * d + B * Hq * nb * h + B * Hkv * nb * h
                + B * Hq * nb * nb)
    assert g >= need + 256 and g % 256 == 0
    # bf16: header + the K^T block records (d rows x 64 keys per 64-key block;
    # V is read in place) + the list of units flagged for the exact fallback
    # (one int32 per unit)
    redo = -(-(4 * B * Hq * nb) // 256) * 256
    assert seer.sparse_attn_workspace_size(B, Hq, Hkv, n, d, 0) == 256 + 2 * B * Hkv * n * d + redo
    # fp32: also bf16 copies of Q and V
    f32 = seer.sparse_attn_workspace_size(B, Hq, Hkv, n, d, 1)
    assert f32 >= 256 + 2 * n * d * (Hq + 2 * Hkv)
    assert seer.blockmax_workspace_size(B, Hq, Hkv, n, d, 0) >= 256 + 4 * 128 * nb


def test_prefill_host_buffer_size():
    """The host-memory call's device buffer: two chunk slots (half a KV-head
    group of Q, O, LSE and lists each), two KV slots, a gate and an attention
    workspace for one chunk; 0 for invalid arguments."""
    B, Hq, Hkv, n, d, h = 1, 32, 8, 8192, 128, 128
    nb, C = n // 64, 2  # chunk: half of the 4 query heads of a KV head
    size = seer.prefill_host_buffer_size(B, Hq, Hkv, n, d, h, "density", density=0.1)
    cap = seer.gate_required_cap(1, C, 1, n, d, "density", density=0.1)
    slot = 2 * C * n * d * 2 + C * n * 4 + C * nb * 4 + C * nb * cap * 4
    kv = 2 * n * d * 2
    ws = seer.gate_workspace_size(1, C, 1, n, d, h) + seer.sparse_attn_workspace_size(1, C, 1, n, d)
    assert size >= 2 * slot + 2 * kv + ws
    assert size <= 2 * slot + 2 * kv + ws + 64 * 256 + 4 * B * Hkv * 2 * 2
    # fp32 inputs need more; the size does not depend on the batch
    assert seer.prefill_host_buffer_size(B, Hq, Hkv, n, d, h, "density", density=0.1, dtype_code=1) > size
    assert seer.prefill_host_buffer_size(4, Hq, Hkv, n, d, h, "density", density=0.1) >= size
    # odd groups are not split
    odd = seer.prefill_host_buffer_size(1, 3, 1, n, d, h, "topk", k=4)
    assert odd >= 2 * (2 * 3 * n * d * 2)
    # invalid: Hq not a multiple of Hkv, a density above 1, a non-positive h
    assert seer.prefill_host_buffer_size(1, 3, 2, n, d, h, "topk", k=4) == 0
    assert seer.prefill_host_buffer_size(1, 4, 2, n, d, h, "density", density=1.5) == 0
    assert seer.prefill_host_buffer_size(1, 4, 2, n, d, 0, "topk", k=4) == 0


def test_invalid_arguments_rejected_before_any_launch(L):
    bad = _lib.Dims(1, 3, 2, 512, 128, 64)        # Hq not a multiple of Hkv
    st = L.seer_sparse_attn(ctypes.byref(bad), None, None, None, 0, None, None, 1, 0.0, None,
                            None, None, 0, None)
    assert st == 1
    ok = _lib.Dims(1, 4, 2, 512, 128, 32)         # block != 64
    st = L.seer_gate_select(ctypes.byref(ok), ctypes.c_void_p(16), 0, 1e-3, 0, 0.0,
                            ctypes.c_void_p(16), ctypes.c_void_p(16), 8, None)
    assert st == 2
    d96 = _lib.Dims(1, 4, 2, 512, 96, 64)         # unsupported head dim
    p = ctypes.c_void_p(256)
    st = L.seer_attn_blockmax(ctypes.byref(d96), p, p, 0, 0.0, p, None, p, 1 << 20, None)
    assert st == 2
    assert L.seer_workspace_status(None, None) == 7


def test_binding_fails_loudly_without_library(monkeypatch):
    monkeypatch.setattr(_lib, "_lib", None)
    monkeypatch.setattr(_lib, "LIB_PATH", "/nonexistent/libseer.so")
    with pytest.raises(RuntimeError, match="no CPU fallback"):
        _lib.lib()
