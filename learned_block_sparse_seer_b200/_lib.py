"""Thin ctypes binding of libseer.so (include/seer.h): argument marshalling only.

Every computation runs in the CUDA library; this module only checks tensor
properties, allocates caller-owned outputs and workspaces with torch, and
passes raw device pointers and the current CUDA stream.  If the library is
missing it raises: there is no fallback.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libseer.so")

SEER_OK = 0
STATUS_NAMES = {
    0: "SEER_OK", 1: "SEER_ERR_INVALID_ARG", 2: "SEER_ERR_UNSUPPORTED", 3: "SEER_ERR_CAPACITY",
    4: "SEER_ERR_CUDA", 5: "SEER_ERR_TIMEOUT", 6: "SEER_ERR_DEVICE_CHECK", 7: "SEER_ERR_WORKSPACE",
}
SEER_BF16, SEER_FP32 = 0, 1
SELECT_THRESHOLD, SELECT_TOPK_K, SELECT_TOPK_DENSITY = 0, 1, 2
SELECT_FORCE_DIAGONAL = 0x100  # flag OR-ed into a mode: the diagonal block joins every list


class SeerError(RuntimeError):
    def __init__(self, func: str, status: int, cuda_err: int = 0):
        name = STATUS_NAMES.get(status, str(status))
        msg = f"{func} returned {name}"
        if status == 4:
            msg += f" (cudaError {cuda_err})"
        super().__init__(msg)
        self.status = status


class Dims(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int32), ("Hq", ctypes.c_int32), ("Hkv", ctypes.c_int32),
                ("n", ctypes.c_int32), ("d", ctypes.c_int32), ("block", ctypes.c_int32)]


_lib = None


def lib() -> ctypes.CDLL:
    """The loaded library; raises if libseer.so has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing: build it with "
                "`python -m learned_block_sparse_seer_b200.build` (no CPU fallback exists)")
        L = ctypes.CDLL(LIB_PATH)
        P, I32, F, SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_float, ctypes.c_size_t
        DP = ctypes.POINTER(Dims)
        L.seer_gate.argtypes = [DP, P, P, I32, P, P, I32, F, I32, F, I32, F, P, P, P, I32, P, SZ, P]
        L.seer_gate.restype = I32
        L.seer_gate_workspace_size.argtypes = [DP, I32]
        L.seer_gate_varlen.argtypes = [DP, P, P, I32, P, P, I32, F, P, P, I32, I32, F, I32, F, P, P, P, I32, P, SZ, P]
        L.seer_gate_varlen.restype = I32
        L.seer_gate_varlen_workspace_size.argtypes = [DP, I32]
        L.seer_gate_varlen_workspace_size.restype = SZ
        L.seer_gate_workspace_size.restype = SZ
        L.seer_gate_required_cap.argtypes = [DP, I32, I32, F]
        L.seer_gate_required_cap.restype = I32
        L.seer_gate_noalloc.argtypes = [DP, P, P, I32, P, P, I32, F, I32, F, I32, F, P, P, P, I32, P]
        L.seer_gate_noalloc.restype = I32
        L.seer_gate_select.argtypes = [DP, P, I32, F, I32, F, P, P, I32, P]
        L.seer_gate_select.restype = I32
        L.seer_gate_kl_backward.argtypes = [DP, P, P, I32, P, P, I32, P, P, P, P, P, SZ, P]
        L.seer_gate_kl_backward.restype = I32
        L.seer_gate_kl_backward_workspace_size.argtypes = [DP, I32]
        L.seer_gate_kl_backward_workspace_size.restype = SZ
        L.seer_sparse_attn.argtypes = [DP, P, P, P, I32, P, P, I32, F, P, P, P, SZ, P]
        L.seer_sparse_attn.restype = I32
        L.seer_prefill_host.argtypes = [DP, P, P, P, I32, P, P, I32, F, I32, F, I32, F, F, P, P, P, SZ, P]
        L.seer_prefill_host.restype = I32
        L.seer_prefill_host_buffer_size.argtypes = [DP, I32, I32, I32, I32, F]
        L.seer_prefill_host_buffer_size.restype = SZ
        L.seer_sparse_attn_workspace_size.argtypes = [DP, I32]
        L.seer_sparse_attn_workspace_size.restype = SZ
        L.seer_attn_blockmax.argtypes = [DP, P, P, I32, F, P, P, P, SZ, P]
        L.seer_attn_blockmax.restype = I32
        L.seer_attn_forward_map.argtypes = [DP, P, P, P, I32, F, P, P, P, P, SZ, P]
        L.seer_attn_forward_map.restype = I32
        L.seer_attn_forward_map_workspace_size.argtypes = [DP, I32]
        L.seer_attn_forward_map_workspace_size.restype = SZ
        L.seer_blockmax_workspace_size.argtypes = [DP, I32]
        L.seer_blockmax_workspace_size.restype = SZ
        L.seer_decode_kcache_update.argtypes = [DP, P, I32, P, I32, I32, I32, P, P]
        L.seer_decode_kcache_update.restype = I32
        L.seer_decode_gate.argtypes = [DP, P, I32, P, I32, I32, F, I32, F, P, P, P, I32, P, SZ, P]
        L.seer_decode_gate.restype = I32
        L.seer_decode_gate_workspace_size.argtypes = [DP]
        L.seer_decode_gate_workspace_size.restype = SZ
        L.seer_decode_gate_required_cap.argtypes = [DP, I32, I32, I32, F]
        L.seer_decode_gate_required_cap.restype = I32
        L.seer_sparse_decode_attn.argtypes = [DP, P, P, P, I32, I32, P, P, I32, F, P, P, P, SZ, P]
        L.seer_sparse_decode_attn.restype = I32
        L.seer_sparse_decode_attn_workspace_size.argtypes = [DP]
        L.seer_sparse_decode_attn_workspace_size.restype = SZ
        L.seer_decode_blockmax.argtypes = [DP, P, P, I32, I32, F, P, P, P, SZ, P]
        L.seer_decode_blockmax_workspace_size.argtypes = [DP]
        L.seer_decode_blockmax_workspace_size.restype = SZ
        L.seer_decode_blockmax.restype = I32
        L.seer_sparse_attn_tf32.argtypes = [DP, P, P, P, P, P, I32, F, P, P, P, SZ, P]
        L.seer_sparse_attn_tf32.restype = I32
        L.seer_sparse_attn_tf32_workspace_size.argtypes = [DP]
        L.seer_sparse_attn_tf32_workspace_size.restype = SZ
        L.seer_workspace_status.argtypes = [P, P]
        L.seer_workspace_status.restype = I32
        L.seer_status_string.argtypes = [I32]
        L.seer_status_string.restype = ctypes.c_char_p
        L.seer_last_cuda_error.restype = I32
        L.seer_version.restype = ctypes.c_char_p
        L.seer_testing_attn_wait_fault.argtypes = [I32, ctypes.c_uint64]
        L.seer_testing_attn_wait_fault.restype = None
        _lib = L
    return _lib


def _check(func: str, status: int):
    if status != SEER_OK:
        raise SeerError(func, status, lib().seer_last_cuda_error())


def _dims(B, Hq, Hkv, n, d) -> Dims:
    return Dims(int(B), int(Hq), int(Hkv), int(n), int(d), 64)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return SEER_BF16
    if t.dtype == torch.float32:
        return SEER_FP32
    raise TypeError(f"unsupported dtype {t.dtype}: bf16 or fp32")


def _dev(*ts: torch.Tensor):
    dev = ts[0].device
    for t in ts:
        if t.device.type != "cuda" or t.device != dev:
            raise ValueError("all tensors must be on the same CUDA device")
        if not t.is_contiguous():
            raise ValueError("tensors must be contiguous [B, H, n, d]")
    return dev


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else None


def _stream(dev) -> ctypes.c_void_p:
    return ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream)


def _workspace(nbytes: int, dev, ws: torch.Tensor | None) -> torch.Tensor:
    if ws is not None:
        if ws.numel() * ws.element_size() < nbytes:
            raise ValueError(f"workspace too small: need {nbytes} bytes")
        return ws
    return torch.empty(max(nbytes, 256), dtype=torch.uint8, device=dev)


def mode_code(mode, force_diagonal: bool = False) -> int:
    if not isinstance(mode, int):
        mode = {"threshold": SELECT_THRESHOLD, "topk": SELECT_TOPK_K, "topk_k": SELECT_TOPK_K,
                "density": SELECT_TOPK_DENSITY, "topk_density": SELECT_TOPK_DENSITY}[mode]
    return mode | (SELECT_FORCE_DIAGONAL if force_diagonal else 0)


# --------------------------------------------------------------------- gate --
def gate_workspace_size(B, Hq, Hkv, n, d, h) -> int:
    return int(lib().seer_gate_workspace_size(ctypes.byref(_dims(B, Hq, Hkv, n, d)), int(h)))


def gate_required_cap(B, Hq, Hkv, n, d, mode, k=0, density=0.0) -> int:
    return int(lib().seer_gate_required_cap(ctypes.byref(_dims(B, Hq, Hkv, n, d)), mode_code(mode),
                                            int(k), float(density)))


def seer_gate(Q, K, Wq, Wk, mode, T=0.0, k=0, density=0.0, rope_theta=0.0, return_scores=False,
              cap=None, workspace=None, out=None, force_diagonal=False):
    """AttnGate + mask generation.  Returns (counts, indices[, scores])."""
    dev = _dev(Q, K, Wq, Wk)
    B, Hq, n, d = Q.shape
    Hkv = K.shape[1]
    if Wq.dtype != torch.float32 or Wk.dtype != torch.float32:
        raise TypeError("gate weights must be fp32")
    h = Wq.shape[1]
    nb = n // 64
    mc = mode_code(mode, force_diagonal)
    dims = _dims(B, Hq, Hkv, n, d)
    if cap is None:
        cap = max(1, lib().seer_gate_required_cap(ctypes.byref(dims), mc, int(k), float(density)))
    if out is None:
        counts = torch.empty(B, Hq, nb, dtype=torch.int32, device=dev)
        indices = torch.empty(B, Hq, nb, cap, dtype=torch.int32, device=dev)
        scores = torch.empty(B, Hq, nb, nb, dtype=torch.float32, device=dev) if return_scores else None
    else:
        counts, indices, scores = out
    ws = _workspace(gate_workspace_size(B, Hq, Hkv, n, d, h), dev, workspace)
    st = lib().seer_gate(ctypes.byref(dims), _ptr(Q), _ptr(K), _dtype_code(Q), _ptr(Wq), _ptr(Wk),
                         int(h), float(rope_theta), mc, float(T), int(k), float(density),
                         _ptr(scores), _ptr(counts), _ptr(indices), int(cap), _ptr(ws),
                         ws.numel(), _stream(dev))
    _check("seer_gate", st)
    return (counts, indices, scores) if return_scores else (counts, indices)


def gate_kl_backward_workspace_size(B, Hq, Hkv, n, d, h) -> int:
    return int(lib().seer_gate_kl_backward_workspace_size(ctypes.byref(_dims(B, Hq, Hkv, n, d)), int(h)))


def seer_gate_kl_backward(Q, K, Wq, Wk, gt, workspace=None, out=None):
    """One AttnGate distillation step: (loss [1] fp32, dWq [Hq,h,d], dWk
    [Hkv,h,3d]) for KL(gt || score), gt the max-pooled map [B,Hq,nb,nb]."""
    dev = _dev(Q, K, Wq, Wk, gt)
    B, Hq, n, d = Q.shape
    Hkv = K.shape[1]
    if Wq.dtype != torch.float32 or Wk.dtype != torch.float32 or gt.dtype != torch.float32:
        raise TypeError("gate weights and gt must be fp32")
    h = Wq.shape[1]
    if out is None:
        loss = torch.empty(1, dtype=torch.float32, device=dev)
        dWq = torch.empty_like(Wq)
        dWk = torch.empty_like(Wk)
    else:
        loss, dWq, dWk = out
    dims = _dims(B, Hq, Hkv, n, d)
    ws = _workspace(gate_kl_backward_workspace_size(B, Hq, Hkv, n, d, h), dev, workspace)
    st = lib().seer_gate_kl_backward(ctypes.byref(dims), _ptr(Q), _ptr(K), _dtype_code(Q), _ptr(Wq), _ptr(Wk),
                                     int(h), _ptr(gt), _ptr(loss), _ptr(dWq), _ptr(dWk), _ptr(ws), ws.numel(),
                                     _stream(dev))
    _check("seer_gate_kl_backward", st)
    return loss, dWq, dWk


def seer_gate_noalloc(Q, K, Wq, Wk, mode, T=0.0, k=0, density=0.0, rope_theta=0.0,
                      return_scores=False, cap=None, out=None):
    """seer_gate without a workspace, for callers that cannot allocate device
    memory (their scratch lives in a fixed buffer inside the library; see
    seer_gate_noalloc in include/seer.h for its size limit and sharing rules).
    Outputs are still passed in (`out`) or allocated here for convenience.
    Every count is -1 if a bounded wait on the device gave up."""
    dev = _dev(Q, K, Wq, Wk)
    B, Hq, n, d = Q.shape
    Hkv = K.shape[1]
    h = Wq.shape[1]
    nb = n // 64
    mc = mode_code(mode)
    dims = _dims(B, Hq, Hkv, n, d)
    if cap is None:
        cap = max(1, lib().seer_gate_required_cap(ctypes.byref(dims), mc, int(k), float(density)))
    if out is None:
        counts = torch.empty(B, Hq, nb, dtype=torch.int32, device=dev)
        indices = torch.empty(B, Hq, nb, cap, dtype=torch.int32, device=dev)
        scores = torch.empty(B, Hq, nb, nb, dtype=torch.float32, device=dev) if return_scores else None
    else:
        counts, indices, scores = out
    # the library's buffer is the current device's: make the tensors' device current
    with torch.cuda.device(dev):
        st = lib().seer_gate_noalloc(ctypes.byref(dims), _ptr(Q), _ptr(K), _dtype_code(Q), _ptr(Wq),
                                     _ptr(Wk), int(h), float(rope_theta), mc, float(T), int(k),
                                     float(density), _ptr(scores), _ptr(counts), _ptr(indices),
                                     int(cap), _stream(dev))
    _check("seer_gate_noalloc", st)
    return (counts, indices, scores) if return_scores else (counts, indices)


def seer_gate_select(scores, mode, T=0.0, k=0, density=0.0, cap=None, out=None, force_diagonal=False):
    """Mask generation on supplied fp32 scores [B, Hq, nb, nb]."""
    dev = _dev(scores)
    if scores.dtype != torch.float32:
        raise TypeError("scores must be fp32")
    B, Hq, nb, _ = scores.shape
    mc = mode_code(mode, force_diagonal)
    dims = _dims(B, Hq, 1, nb * 64, 64)
    if cap is None:
        cap = max(1, lib().seer_gate_required_cap(ctypes.byref(dims), mc, int(k), float(density)))
    if out is None:
        counts = torch.empty(B, Hq, nb, dtype=torch.int32, device=dev)
        indices = torch.empty(B, Hq, nb, cap, dtype=torch.int32, device=dev)
    else:
        counts, indices = out
    st = lib().seer_gate_select(ctypes.byref(dims), _ptr(scores), mc, float(T), int(k),
                                float(density), _ptr(counts), _ptr(indices), int(cap), _stream(dev))
    _check("seer_gate_select", st)
    return counts, indices


# ---------------------------------------------------------------- attention --
def sparse_attn_workspace_size(B, Hq, Hkv, n, d, dtype_code=SEER_BF16) -> int:
    return int(lib().seer_sparse_attn_workspace_size(ctypes.byref(_dims(B, Hq, Hkv, n, d)),
                                                     int(dtype_code)))


def seer_sparse_attn(Q, K, V, counts, indices, scale=0.0, workspace=None, out=None,
                     return_lse=True):
    """Block-sparse causal attention over the listed key blocks.
    Returns (O, lse)."""
    dev = _dev(Q, K, V, counts, indices)
    B, Hq, n, d = Q.shape
    Hkv = K.shape[1]
    dt = _dtype_code(Q)
    if counts.dtype != torch.int32 or indices.dtype != torch.int32:
        raise TypeError("counts/indices must be int32")
    cap = indices.shape[-1]
    if out is None:
        O = torch.empty_like(Q)
        lse = torch.empty(B, Hq, n, dtype=torch.float32, device=dev) if return_lse else None
    else:
        O, lse = out
    ws = _workspace(sparse_attn_workspace_size(B, Hq, Hkv, n, d, dt), dev, workspace)
    st = lib().seer_sparse_attn(ctypes.byref(_dims(B, Hq, Hkv, n, d)), _ptr(Q), _ptr(K), _ptr(V),
                                dt, _ptr(counts), _ptr(indices), int(cap), float(scale), _ptr(O),
                                _ptr(lse), _ptr(ws), ws.numel(), _stream(dev))
    _check("seer_sparse_attn", st)
    return O, lse


def prefill_host_buffer_size(B, Hq, Hkv, n, d, h, mode, T=0.0, k=0, density=0.0, dtype_code=SEER_BF16,
                             force_diagonal=False) -> int:
    return int(lib().seer_prefill_host_buffer_size(ctypes.byref(_dims(B, Hq, Hkv, n, d)), int(dtype_code), int(h),
                                                   mode_code(mode, force_diagonal), int(k), float(density)))


def seer_prefill_host(Q, K, V, Wq, Wk, mode, T=0.0, k=0, density=0.0, rope_theta=0.0, scale=0.0, out=None,
                      return_lse=True, buffer=None, force_diagonal=False):
    """seer_gate + seer_sparse_attn for Q/K/V in host memory (page-locked
    for the copy/compute overlap), the weights on the device.  Returns
    (O, lse) in host memory once they are there.  Without `out`, page-locked
    outputs are allocated per call (pinning is slow for large tensors: pass
    `out` and `buffer` when calling repeatedly)."""
    for t in (Q, K, V):
        if t.is_cuda or not t.is_contiguous():
            raise ValueError("Q, K, V must be contiguous host tensors")
    dev = _dev(Wq, Wk)
    B, Hq, n, d = Q.shape
    Hkv = K.shape[1]
    h = Wq.shape[1]
    dt = _dtype_code(Q)
    mc = mode_code(mode, force_diagonal)
    if out is None:
        O = torch.empty(Q.shape, dtype=Q.dtype, pin_memory=True)
        lse = torch.empty(B, Hq, n, dtype=torch.float32, pin_memory=True) if return_lse else None
    else:
        O, lse = out
    nbytes = prefill_host_buffer_size(B, Hq, Hkv, n, d, h, mode, T, k, density, dt, force_diagonal)
    if nbytes == 0:
        raise ValueError("invalid arguments for seer_prefill_host")
    buf = _workspace(nbytes, dev, buffer)
    st = lib().seer_prefill_host(ctypes.byref(_dims(B, Hq, Hkv, n, d)), _ptr(Q), _ptr(K), _ptr(V), dt, _ptr(Wq),
                                 _ptr(Wk), int(h), float(rope_theta), mc, float(T), int(k), float(density),
                                 float(scale), _ptr(O), _ptr(lse), _ptr(buf), buf.numel(), _stream(dev))
    _check("seer_prefill_host", st)
    return O, lse


def blockmax_workspace_size(B, Hq, Hkv, n, d, dtype_code=SEER_BF16) -> int:
    return int(lib().seer_blockmax_workspace_size(ctypes.byref(_dims(B, Hq, Hkv, n, d)),
                                                  int(dtype_code)))


def seer_attn_blockmax(Q, K, scale=0.0, workspace=None, out=None, return_lse=True):
    """2D max-pooled causal attention probabilities.  Returns (map, lse)."""
    dev = _dev(Q, K)
    B, Hq, n, d = Q.shape
    Hkv = K.shape[1]
    dt = _dtype_code(Q)
    nb = n // 64
    if out is None:
        M = torch.empty(B, Hq, nb, nb, dtype=torch.float32, device=dev)
        lse = torch.empty(B, Hq, n, dtype=torch.float32, device=dev) if return_lse else None
    else:
        M, lse = out
    ws = _workspace(blockmax_workspace_size(B, Hq, Hkv, n, d, dt), dev, workspace)
    st = lib().seer_attn_blockmax(ctypes.byref(_dims(B, Hq, Hkv, n, d)), _ptr(Q), _ptr(K), dt,
                                  float(scale), _ptr(M), _ptr(lse), _ptr(ws), ws.numel(),
                                  _stream(dev))
    _check("seer_attn_blockmax", st)
    return M, lse


def seer_workspace_status(workspace: torch.Tensor) -> int:
    """Synchronises the current stream and returns the device status code."""
    return int(lib().seer_workspace_status(_ptr(workspace), _stream(workspace.device)))


def attn_forward_map_workspace_size(B, Hq, Hkv, n, d, dtype_code=SEER_BF16) -> int:
    return int(lib().seer_attn_forward_map_workspace_size(ctypes.byref(_dims(B, Hq, Hkv, n, d)), int(dtype_code)))


def seer_attn_forward_map(Q, K, V, scale=0.0, workspace=None, out=None):
    """Training forward: (O [B,Hq,n,d], lse [B,Hq,n] fp32, map [B,Hq,nb,nb]
    fp32) -- dense causal attention and the 2D-max-pooled probability map."""
    dev = _dev(Q, K, V)
    B, Hq, n, d = Q.shape
    Hkv = K.shape[1]
    nb = n // 64
    dc = _dtype_code(Q)
    if out is None:
        O = torch.empty_like(Q)
        lse = torch.empty(B, Hq, n, dtype=torch.float32, device=dev)
        M = torch.empty(B, Hq, nb, nb, dtype=torch.float32, device=dev)
    else:
        O, lse, M = out
    dims = _dims(B, Hq, Hkv, n, d)
    ws = _workspace(attn_forward_map_workspace_size(B, Hq, Hkv, n, d, dc), dev, workspace)
    st = lib().seer_attn_forward_map(ctypes.byref(dims), _ptr(Q), _ptr(K), _ptr(V), dc, float(scale), _ptr(O),
                                     _ptr(lse), _ptr(M), _ptr(ws), ws.numel(), _stream(dev))
    _check("seer_attn_forward_map", st)
    return O, lse, M


# ------------------------------------------------------------------ decode --
# The KV cache is [B, Hkv, n, d] with n its capacity in tokens; the current
# token (query q [B, Hq, d]) sits at position seq_len - 1, in block
# c = (seq_len - 1) // 64.  Candidates are the complete blocks j < c.
def _cache_dims(q, Kc):
    B, Hq, d = q.shape
    _, Hkv, n, dk = Kc.shape
    if dk != d:
        raise ValueError("q and the cache disagree on d")
    return _dims(B, Hq, Hkv, n, d)


def seer_decode_kcache_update(Kc, Wk, block_begin, block_end, kt_cache=None):
    """k~ of key blocks [block_begin, block_end) of the cache into kt_cache
    [B, Hkv, n/64, d] fp32 (allocated when None); returns kt_cache."""
    dev = _dev(Kc, Wk)
    B, Hkv, n, d = Kc.shape
    if Wk.dtype != torch.float32:
        raise TypeError("gate weights must be fp32")
    h = Wk.shape[1]
    if kt_cache is None:
        kt_cache = torch.zeros(B, Hkv, n // 64, h, dtype=torch.float32, device=dev)
    dims = _dims(B, Hkv, Hkv, n, d)
    st = lib().seer_decode_kcache_update(ctypes.byref(dims), _ptr(Kc), _dtype_code(Kc), _ptr(Wk), int(h),
                                         int(block_begin), int(block_end), _ptr(kt_cache), _stream(dev))
    _check("seer_decode_kcache_update", st)
    return kt_cache


def decode_gate_required_cap(B, Hq, Hkv, n, d, seq_len, mode, k=0, density=0.0) -> int:
    return int(lib().seer_decode_gate_required_cap(ctypes.byref(_dims(B, Hq, Hkv, n, d)), int(seq_len),
                                                   mode_code(mode), int(k), float(density)))


def decode_gate_workspace_size(B, Hq, Hkv, n, d) -> int:
    return int(lib().seer_decode_gate_workspace_size(ctypes.byref(_dims(B, Hq, Hkv, n, d))))


def seer_decode_gate(q, kt_cache, n, seq_len, mode, T=0.0, k=0, density=0.0, return_scores=False, cap=None,
                     workspace=None, out=None):
    """Decode-stage gate: (counts [B,Hq], indices [B,Hq,cap][, scores
    [B,Hq,c]]) for the token at seq_len - 1 of a cache of n tokens."""
    dev = _dev(q, kt_cache)
    B, Hq, d = q.shape
    Hkv = kt_cache.shape[1]
    dims = _dims(B, Hq, Hkv, n, d)
    mc = mode_code(mode)
    c = (int(seq_len) - 1) // 64
    if cap is None:
        cap = max(1, lib().seer_decode_gate_required_cap(ctypes.byref(dims), int(seq_len), mc, int(k),
                                                         float(density)))
    if out is None:
        counts = torch.empty(B, Hq, dtype=torch.int32, device=dev)
        indices = torch.empty(B, Hq, cap, dtype=torch.int32, device=dev)
        scores = torch.empty(B, Hq, c, dtype=torch.float32, device=dev) if return_scores else None
    else:
        counts, indices, scores = out
    ws = _workspace(decode_gate_workspace_size(B, Hq, Hkv, n, d), dev, workspace)
    st = lib().seer_decode_gate(ctypes.byref(dims), _ptr(q), _dtype_code(q), _ptr(kt_cache), int(seq_len), mc,
                                float(T), int(k), float(density), _ptr(scores), _ptr(counts), _ptr(indices),
                                int(cap), _ptr(ws), ws.numel(), _stream(dev))
    _check("seer_decode_gate", st)
    return (counts, indices, scores) if return_scores else (counts, indices)


def sparse_decode_attn_workspace_size(B, Hq, Hkv, n, d) -> int:
    return int(lib().seer_sparse_decode_attn_workspace_size(ctypes.byref(_dims(B, Hq, Hkv, n, d))))


def seer_sparse_decode_attn(q, Kc, Vc, seq_len, counts, indices, scale=0.0, workspace=None, out=None):
    """Block-sparse decode attention: (O [B,Hq,d], lse [B,Hq] fp32)."""
    dev = _dev(q, Kc, Vc, counts, indices)
    dims = _cache_dims(q, Kc)
    B, Hq, d = q.shape
    if out is None:
        O = torch.empty_like(q)
        lse = torch.empty(B, Hq, dtype=torch.float32, device=dev)
    else:
        O, lse = out
    ws = _workspace(sparse_decode_attn_workspace_size(B, Hq, Kc.shape[1], Kc.shape[2], d), dev, workspace)
    st = lib().seer_sparse_decode_attn(ctypes.byref(dims), _ptr(q), _ptr(Kc), _ptr(Vc), _dtype_code(q),
                                       int(seq_len), _ptr(counts), _ptr(indices), int(indices.shape[-1]),
                                       float(scale), _ptr(O), _ptr(lse), _ptr(ws), ws.numel(), _stream(dev))
    _check("seer_sparse_decode_attn", st)
    return O, lse


def decode_blockmax_workspace_size(B, Hq, Hkv, n, d) -> int:
    return int(lib().seer_decode_blockmax_workspace_size(ctypes.byref(_dims(B, Hq, Hkv, n, d))))


def seer_decode_blockmax(q, Kc, seq_len, scale=0.0, workspace=None, out=None):
    """1D ground truth of the token's attention row: (gt [B,Hq,c+1], lse
    [B,Hq]) fp32."""
    dev = _dev(q, Kc)
    dims = _cache_dims(q, Kc)
    B, Hq, d = q.shape
    c = (int(seq_len) - 1) // 64
    if out is None:
        gt = torch.empty(B, Hq, c + 1, dtype=torch.float32, device=dev)
        lse = torch.empty(B, Hq, dtype=torch.float32, device=dev)
    else:
        gt, lse = out
    ws = _workspace(decode_blockmax_workspace_size(B, Hq, Kc.shape[1], Kc.shape[2], d), dev, workspace)
    st = lib().seer_decode_blockmax(ctypes.byref(dims), _ptr(q), _ptr(Kc), _dtype_code(q), int(seq_len),
                                    float(scale), _ptr(gt), _ptr(lse), _ptr(ws), ws.numel(), _stream(dev))
    _check("seer_decode_blockmax", st)
    return gt, lse


# ------------------------------------------------------------------ varlen --
def gate_varlen_workspace_size(Hq, Hkv, n, d, h) -> int:
    return int(lib().seer_gate_varlen_workspace_size(ctypes.byref(_dims(1, Hq, Hkv, n, d)), int(h)))


def seer_gate_varlen(Q, K, Wq, Wk, seq_start, seq_len, mode, T=0.0, k=0, density=0.0, rope_theta=0.0,
                     return_scores=False, cap=None, workspace=None, out=None, force_diagonal=False):
    """AttnGate + mask generation over sequences packed along the token axis
    (Q [1,Hq,n,d], K [1,Hkv,n,d]; seq_start / seq_len int32 CUDA tensors).
    Returns (counts, indices[, scores]) with global block indices."""
    dev = _dev(Q, K, Wq, Wk, seq_start, seq_len)
    B, Hq, n, d = Q.shape
    Hkv = K.shape[1]
    if B != 1:
        raise ValueError("packed sequences: B must be 1")
    if seq_start.dtype != torch.int32 or seq_len.dtype != torch.int32:
        raise TypeError("seq_start and seq_len must be int32")
    if Wq.dtype != torch.float32 or Wk.dtype != torch.float32:
        raise TypeError("gate weights must be fp32")
    h = Wq.shape[1]
    nb = n // 64
    mc = mode_code(mode, force_diagonal)
    dims = _dims(1, Hq, Hkv, n, d)
    if cap is None:
        cap = max(1, lib().seer_gate_required_cap(ctypes.byref(dims), mc, int(k), float(density)))
    if out is None:
        counts = torch.empty(1, Hq, nb, dtype=torch.int32, device=dev)
        indices = torch.empty(1, Hq, nb, cap, dtype=torch.int32, device=dev)
        scores = torch.empty(1, Hq, nb, nb, dtype=torch.float32, device=dev) if return_scores else None
    else:
        counts, indices, scores = out
    ws = _workspace(gate_varlen_workspace_size(Hq, Hkv, n, d, h), dev, workspace)
    st = lib().seer_gate_varlen(ctypes.byref(dims), _ptr(Q), _ptr(K), _dtype_code(Q), _ptr(Wq), _ptr(Wk), int(h),
                                float(rope_theta), _ptr(seq_start), _ptr(seq_len), int(seq_start.numel()), mc,
                                float(T), int(k), float(density), _ptr(scores), _ptr(counts), _ptr(indices),
                                int(cap), _ptr(ws), ws.numel(), _stream(dev))
    _check("seer_gate_varlen", st)
    return (counts, indices, scores) if return_scores else (counts, indices)


# -------------------------------------------------------------- tf32 attn --
def sparse_attn_tf32_workspace_size(B, Hq, Hkv, n, d) -> int:
    return int(lib().seer_sparse_attn_tf32_workspace_size(ctypes.byref(_dims(B, Hq, Hkv, n, d))))


def seer_sparse_attn_tf32(Q, K, V, counts, indices, scale=0.0, workspace=None, out=None):
    """Block-sparse attention for fp32 Q/K/V on the tf32 tensor cores:
    (O [B,Hq,n,d] fp32, lse [B,Hq,n] fp32)."""
    dev = _dev(Q, K, V, counts, indices)
    for t in (Q, K, V):
        if t.dtype != torch.float32:
            raise TypeError("the tf32 path takes fp32 Q, K, V")
    B, Hq, n, d = Q.shape
    Hkv = K.shape[1]
    if out is None:
        O = torch.empty_like(Q)
        lse = torch.empty(B, Hq, n, dtype=torch.float32, device=dev)
    else:
        O, lse = out
    dims = _dims(B, Hq, Hkv, n, d)
    ws = _workspace(sparse_attn_tf32_workspace_size(B, Hq, Hkv, n, d), dev, workspace)
    st = lib().seer_sparse_attn_tf32(ctypes.byref(dims), _ptr(Q), _ptr(K), _ptr(V), _ptr(counts), _ptr(indices),
                                     int(indices.shape[-1]), float(scale), _ptr(O), _ptr(lse), _ptr(ws), ws.numel(),
                                     _stream(dev))
    _check("seer_sparse_attn_tf32", st)
    return O, lse
