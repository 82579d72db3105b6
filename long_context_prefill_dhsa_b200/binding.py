"""ctypes binding of libdhsa (the C ABI in include/dhsa.h).

Argument marshalling only: torch tensors are checked for dtype, shape,
contiguity and device, then their data pointers and the current CUDA stream
are handed to the library. Every step of the path runs in the library's CUDA
kernels; there is no fallback. If the library is missing, loading fails
loudly (build it with `python -m long_context_prefill_dhsa_b200.build`).
"""
from __future__ import annotations

import ctypes
import math
import os
import re
from typing import Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libdhsa.so")
HEADER_PATH = os.path.join(os.path.dirname(_PKG), "include", "dhsa.h")

DHSA_OK = 0
STATUS_NAMES = {0: "DHSA_OK", 1: "DHSA_ERR_INVALID_ARG", 2: "DHSA_ERR_UNSUPPORTED", 3: "DHSA_ERR_CUDA",
                4: "DHSA_ERR_DEVICE", 5: "DHSA_ERR_WORKSPACE"}
DEVFLAG_WAIT_TIMEOUT, DEVFLAG_BAD_OFFSETS, DEVFLAG_BAD_SELECTION = 0x1, 0x2, 0x4


class DHSAError(RuntimeError):
    def __init__(self, status: int, where: str, cuda_error: int = 0, flags: int = 0):
        self.status, self.where, self.cuda_error, self.flags = status, where, cuda_error, flags
        msg = f"{where}: {STATUS_NAMES.get(status, status)}"
        if cuda_error:
            msg += f" (cudaError {cuda_error})"
        if flags:
            msg += f" (device flags 0x{flags:x})"
        super().__init__(msg)


_c = ctypes
_P, _I, _F, _SZ = _c.c_void_p, _c.c_int, _c.c_float, _c.c_size_t
_SIGNATURES = {
    "dhsa_status_string": (_c.c_char_p, [_I]),
    "dhsa_last_cuda_error": (_I, []),
    "dhsa_version": (_I, []),
    "dhsa_check_device_status": (_I, [_P, _c.POINTER(_c.c_uint32)]),
    "dhsa_validate_offsets": (_I, [_P, _P, _I, _I, _I, _P]),
    "dhsa_chunk_pool": (_I, [_P, _I, _I, _I, _I, _P, _P, _I, _P, _P]),
    "dhsa_chunk_pool_qk": (_I, [_P, _P, _I, _I, _I, _I, _I, _P, _P, _I, _P, _P, _P]),
    "dhsa_sel_stride": (_I, [_I, _I]),
    "dhsa_score_topk_workspace_size": (_SZ, [_I, _I, _I]),
    "dhsa_chunk_score_topk": (_I, [_P, _P, _I, _I, _I, _I, _P, _I, _P, _P, _P, _SZ, _P]),
    "dhsa_chunk_score_topk_csr": (_I, [_P, _P, _I, _I, _I, _I, _P, _P, _I, _P, _P, _P, _P, _P, _P, _SZ, _P]),
    "dhsa_budget_max_chunks": (_I, []),
    "dhsa_chunk_score_select_budget": (_I, [_P, _P, _I, _I, _I, _I, _P, _P, _I, _P, _I, _I, _P, _P, _P, _SZ, _P]),
    "dhsa_route_fused_workspace_size": (_SZ, [_I, _I, _I]),
    "dhsa_route_fused": (_I, [_P, _P, _I, _I, _I, _I, _I, _P, _P, _I, _I, _P, _P, _P, _P, _P, _SZ, _P]),
    "dhsa_route_topk_csr": (_I, [_P, _P, _I, _I, _I, _I, _I, _P, _P, _I, _I, _P, _P, _P, _P, _P, _P, _P, _P, _SZ,
                                 _P]),
    "dhsa_csr_nnz_upper": (_SZ, [_I, _I, _I, _I]),
    "dhsa_build_block_csr": (_I, [_P, _P, _I, _I, _I, _I, _P, _P, _P, _P, _P, _P]),
    "dhsa_sparse_attn_workspace_size": (_SZ, [_I, _I, _I, _I]),
    "dhsa_sparse_attn_fwd": (_I, [_P, _P, _P, _I, _I, _I, _I, _I, _P, _P, _I, _P, _P, _P, _F, _P, _P, _SZ, _P]),
    "dhsa_sparse_attn_fwd_noalloc": (_I, [_P, _P, _P, _I, _I, _I, _I, _I, _P, _P, _I, _P, _P, _F, _P, _P]),
    "dhsa_sparse_attn_tiles_workspace_size": (_SZ, [_I, _I, _I, _I, _I]),
    "dhsa_sparse_attn_fwd_tiles": (_I, [_P, _P, _P, _I, _I, _I, _I, _I, _P, _P, _I, _P, _P, _F, _I, _P, _P, _SZ,
                                        _P]),
    "dhsa_debug_arm_wait_timeout": (_I, [_I, _c.c_uint64]),
}

_lib: Optional[ctypes.CDLL] = None


def load() -> ctypes.CDLL:
    """Load libdhsa.so (once). Raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m long_context_prefill_dhsa_b200.build`")
        lib = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGNATURES.items():
            fn = getattr(lib, name)
            fn.restype, fn.argtypes = res, args
        _lib = lib
    return _lib


def header_functions() -> list[str]:
    """Names of the functions include/dhsa.h declares."""
    text = open(HEADER_PATH).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(dhsa_[a-z0-9_]+)\s*\(", text)))


def _check(status: int, where: str):
    if status != DHSA_OK:
        raise DHSAError(status, where, load().dhsa_last_cuda_error() if status == 3 else 0)


def _stream_ptr() -> int:
    return torch.cuda.current_stream().cuda_stream


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else t.data_ptr()


def _need(t: torch.Tensor, dtype, shape, name):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name}: expected a torch.Tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name}: dtype {t.dtype}, expected {dtype}")
    if not t.is_cuda:
        raise ValueError(f"{name}: must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name}: must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: shape {tuple(t.shape)}, expected {tuple(shape)}")


# ----------------------------------------------------------------- stage calls
def check_device_status() -> int:
    flags = ctypes.c_uint32(0)
    st = load().dhsa_check_device_status(_stream_ptr(), ctypes.byref(flags))
    if st != DHSA_OK:
        raise DHSAError(st, "dhsa_check_device_status", load().dhsa_last_cuda_error() if st == 3 else 0,
                        flags.value)
    return flags.value


def debug_arm_wait_timeout(mode: int, limit_ns: int = 0):
    """Test hook of the bounded device waits (include/dhsa.h, 5): mode 1 makes
    the next attention launch's first waits run out after limit_ns, mode 2
    the next fused-routing launch's first grid barrier; 0 disarms."""
    _check(load().dhsa_debug_arm_wait_timeout(mode, limit_ns), "dhsa_debug_arm_wait_timeout")


def validate_offsets(off: torch.Tensor, n_chunks: torch.Tensor, L: int):
    B, n1 = off.shape
    _need(off, torch.int32, None, "off")
    _need(n_chunks, torch.int32, (B,), "n_chunks")
    _check(load().dhsa_validate_offsets(_ptr(off), _ptr(n_chunks), B, n1 - 1, L, _stream_ptr()),
           "dhsa_validate_offsets")


def chunk_pool(X: torch.Tensor, off: torch.Tensor, n_chunks: torch.Tensor, out: Optional[torch.Tensor] = None):
    """Xp[b,h,c] = sum of chunk c's rows / sqrt(n_c), fp32 [B,H,Nmax,128]."""
    B, H, L, d = X.shape
    nmax = off.shape[1] - 1
    _need(X, torch.bfloat16, None, "X")
    _need(off, torch.int32, (B, nmax + 1), "off")
    _need(n_chunks, torch.int32, (B,), "n_chunks")
    if out is None:
        out = torch.empty((B, H, nmax, d), dtype=torch.float32, device=X.device)
    _need(out, torch.float32, (B, H, nmax, d), "out")
    _check(load().dhsa_chunk_pool(_ptr(X), B, H, L, d, _ptr(off), _ptr(n_chunks), nmax, _ptr(out), _stream_ptr()),
           "dhsa_chunk_pool")
    return out


def chunk_pool_qk(Q: torch.Tensor, K: torch.Tensor, off: torch.Tensor, n_chunks: torch.Tensor,
                  Qp: Optional[torch.Tensor] = None, Kp: Optional[torch.Tensor] = None):
    """Both poolings in one launch; same values as chunk_pool(Q) and chunk_pool(K)."""
    B, Hq, L, d = Q.shape
    Hkv = K.shape[1]
    nmax = off.shape[1] - 1
    _need(Q, torch.bfloat16, None, "Q")
    _need(K, torch.bfloat16, (B, Hkv, L, d), "K")
    _need(off, torch.int32, (B, nmax + 1), "off")
    _need(n_chunks, torch.int32, (B,), "n_chunks")
    if Qp is None:
        Qp = torch.empty((B, Hq, nmax, d), dtype=torch.float32, device=Q.device)
    if Kp is None:
        Kp = torch.empty((B, Hkv, nmax, d), dtype=torch.float32, device=Q.device)
    _need(Qp, torch.float32, (B, Hq, nmax, d), "Qp")
    _need(Kp, torch.float32, (B, Hkv, nmax, d), "Kp")
    _check(load().dhsa_chunk_pool_qk(_ptr(Q), _ptr(K), B, Hq, Hkv, L, d, _ptr(off), _ptr(n_chunks), nmax, _ptr(Qp),
                                     _ptr(Kp), _stream_ptr()), "dhsa_chunk_pool_qk")
    return Qp, Kp


def sel_stride(k: int, nmax: int) -> int:
    return load().dhsa_sel_stride(k, nmax)


def chunk_score_topk_csr(Qp: torch.Tensor, Kp: torch.Tensor, off: torch.Tensor, n_chunks: torch.Tensor, k: int,
                         sel: torch.Tensor, n_sel: torch.Tensor, row_ptr: torch.Tensor, col_idx: torch.Tensor,
                         cost: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None):
    """Top-k selection that also writes the block CSR (include/dhsa.h, 2b):
    the results of chunk_score_topk followed by build_block_csr."""
    B, Hq, nmax, d = Qp.shape
    Hkv = Kp.shape[1]
    _need(Qp, torch.float32, None, "Qp")
    _need(Kp, torch.float32, (B, Hkv, nmax, d), "Kp")
    _need(off, torch.int32, (B, nmax + 1), "off")
    _need(n_chunks, torch.int32, (B,), "n_chunks")
    lib = load()
    stride = lib.dhsa_sel_stride(k, nmax)
    _need(sel, torch.int32, (B, Hq, nmax, stride), "sel")
    _need(n_sel, torch.int32, (B, Hq, nmax), "n_sel")
    _need(row_ptr, torch.int32, (B * Hq * nmax + 1,), "row_ptr")
    _need(col_idx, torch.int32, None, "col_idx")
    if col_idx.numel() < lib.dhsa_csr_nnz_upper(B, Hq, nmax, k):
        raise ValueError("col_idx: smaller than dhsa_csr_nnz_upper")
    if cost is not None:
        _need(cost, torch.int64, (B * Hq * nmax,), "cost")
    if workspace is None:
        workspace = torch.empty(lib.dhsa_score_topk_workspace_size(B, Hq, nmax), dtype=torch.uint8, device=Qp.device)
    _check(lib.dhsa_chunk_score_topk_csr(_ptr(Qp), _ptr(Kp), B, Hq, Hkv, nmax, _ptr(off), _ptr(n_chunks), k,
                                         _ptr(sel), _ptr(n_sel), _ptr(row_ptr), _ptr(col_idx), _ptr(cost),
                                         _ptr(workspace), workspace.numel() * workspace.element_size(),
                                         _stream_ptr()), "dhsa_chunk_score_topk_csr")
    return sel, n_sel


def chunk_score_topk(Qp: torch.Tensor, Kp: torch.Tensor, n_chunks: torch.Tensor, k: int,
                     sel: Optional[torch.Tensor] = None, n_sel: Optional[torch.Tensor] = None,
                     workspace: Optional[torch.Tensor] = None):
    """sel [B,Hq,Nmax,stride] (ascending, diagonal last, -1 padded) and n_sel [B,Hq,Nmax]."""
    B, Hq, nmax, d = Qp.shape
    Hkv = Kp.shape[1]
    _need(Qp, torch.float32, None, "Qp")
    _need(Kp, torch.float32, (B, Hkv, nmax, d), "Kp")
    _need(n_chunks, torch.int32, (B,), "n_chunks")
    lib = load()
    stride = lib.dhsa_sel_stride(k, nmax)
    if sel is None:
        sel = torch.empty((B, Hq, nmax, stride), dtype=torch.int32, device=Qp.device)
    if n_sel is None:
        n_sel = torch.empty((B, Hq, nmax), dtype=torch.int32, device=Qp.device)
    _need(sel, torch.int32, (B, Hq, nmax, stride), "sel")
    _need(n_sel, torch.int32, (B, Hq, nmax), "n_sel")
    ws_bytes = lib.dhsa_score_topk_workspace_size(B, Hq, nmax)
    if ws_bytes and workspace is None:
        workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=Qp.device)
    ws_ptr = _ptr(workspace) if ws_bytes else None
    ws_len = workspace.numel() * workspace.element_size() if (ws_bytes and workspace is not None) else 0
    _check(lib.dhsa_chunk_score_topk(_ptr(Qp), _ptr(Kp), B, Hq, Hkv, nmax, _ptr(n_chunks), k, _ptr(sel),
                                     _ptr(n_sel), ws_ptr, ws_len, _stream_ptr()), "dhsa_chunk_score_topk")
    return sel, n_sel


def route_fused(Q: torch.Tensor, K: torch.Tensor, off: torch.Tensor, n_chunks: torch.Tensor, k: int,
                Qp: Optional[torch.Tensor] = None, Kp: Optional[torch.Tensor] = None,
                sel: Optional[torch.Tensor] = None, n_sel: Optional[torch.Tensor] = None,
                workspace: Optional[torch.Tensor] = None, row_ptr: Optional[torch.Tensor] = None,
                col_idx: Optional[torch.Tensor] = None, cost: Optional[torch.Tensor] = None):
    """Pooling of Q and K plus the top-k selection in one launch (include/dhsa.h,
    2c); the same results as chunk_pool_qk followed by chunk_score_topk. With
    row_ptr and col_idx given, the launch also writes the block CSR (2d), as
    build_block_csr would. Returns (Qp, Kp, sel, n_sel)."""
    B, Hq, L, d = Q.shape
    Hkv = K.shape[1]
    nmax = off.shape[1] - 1
    _need(Q, torch.bfloat16, None, "Q")
    _need(K, torch.bfloat16, (B, Hkv, L, d), "K")
    _need(off, torch.int32, (B, nmax + 1), "off")
    _need(n_chunks, torch.int32, (B,), "n_chunks")
    lib = load()
    stride = lib.dhsa_sel_stride(k, nmax)
    if Qp is None:
        Qp = torch.empty((B, Hq, nmax, d), dtype=torch.float32, device=Q.device)
    if Kp is None:
        Kp = torch.empty((B, Hkv, nmax, d), dtype=torch.float32, device=Q.device)
    if sel is None:
        sel = torch.empty((B, Hq, nmax, stride), dtype=torch.int32, device=Q.device)
    if n_sel is None:
        n_sel = torch.empty((B, Hq, nmax), dtype=torch.int32, device=Q.device)
    _need(Qp, torch.float32, (B, Hq, nmax, d), "Qp")
    _need(Kp, torch.float32, (B, Hkv, nmax, d), "Kp")
    _need(sel, torch.int32, (B, Hq, nmax, stride), "sel")
    _need(n_sel, torch.int32, (B, Hq, nmax), "n_sel")
    ws_bytes = lib.dhsa_route_fused_workspace_size(B, Hq, nmax)
    if workspace is None:
        workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=Q.device)
    if row_ptr is None:
        _check(lib.dhsa_route_fused(_ptr(Q), _ptr(K), B, Hq, Hkv, L, d, _ptr(off), _ptr(n_chunks), nmax, k,
                                    _ptr(Qp), _ptr(Kp), _ptr(sel), _ptr(n_sel), _ptr(workspace),
                                    workspace.numel() * workspace.element_size(), _stream_ptr()), "dhsa_route_fused")
    else:
        _need(row_ptr, torch.int32, (B * Hq * nmax + 1,), "row_ptr")
        _need(col_idx, torch.int32, None, "col_idx")
        if col_idx.numel() < lib.dhsa_csr_nnz_upper(B, Hq, nmax, k):
            raise ValueError("col_idx: smaller than dhsa_csr_nnz_upper")
        if cost is not None:
            _need(cost, torch.int64, (B * Hq * nmax,), "cost")
        _check(lib.dhsa_route_topk_csr(_ptr(Q), _ptr(K), B, Hq, Hkv, L, d, _ptr(off), _ptr(n_chunks), nmax, k,
                                       _ptr(Qp), _ptr(Kp), _ptr(sel), _ptr(n_sel), _ptr(row_ptr), _ptr(col_idx),
                                       _ptr(cost), _ptr(workspace), workspace.numel() * workspace.element_size(),
                                       _stream_ptr()), "dhsa_route_topk_csr")
    return Qp, Kp, sel, n_sel


def chunk_score_select_budget(Qp: torch.Tensor, Kp: torch.Tensor, off: torch.Tensor, n_chunks: torch.Tensor,
                              budget, recent: int, k_max: int, sel: Optional[torch.Tensor] = None,
                              n_sel: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None):
    """Selection under a token budget per row (see include/dhsa.h, 2').

    `budget` is an int (every row) or an int32 CUDA tensor [B, Hq, Nmax] of
    per-row budgets. Returns sel [B,Hq,Nmax,stride(k_max)] and n_sel."""
    B, Hq, nmax, d = Qp.shape
    Hkv = Kp.shape[1]
    _need(Qp, torch.float32, None, "Qp")
    _need(Kp, torch.float32, (B, Hkv, nmax, d), "Kp")
    _need(off, torch.int32, (B, nmax + 1), "off")
    _need(n_chunks, torch.int32, (B,), "n_chunks")
    budgets = None
    if isinstance(budget, torch.Tensor):
        _need(budget, torch.int32, (B, Hq, nmax), "budget")
        budgets, budget = budget, 0
    lib = load()
    stride = lib.dhsa_sel_stride(k_max, nmax)
    if sel is None:
        sel = torch.empty((B, Hq, nmax, stride), dtype=torch.int32, device=Qp.device)
    if n_sel is None:
        n_sel = torch.empty((B, Hq, nmax), dtype=torch.int32, device=Qp.device)
    _need(sel, torch.int32, (B, Hq, nmax, stride), "sel")
    _need(n_sel, torch.int32, (B, Hq, nmax), "n_sel")
    ws_bytes = lib.dhsa_score_topk_workspace_size(B, Hq, nmax)
    if ws_bytes and workspace is None:
        workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=Qp.device)
    ws_ptr = _ptr(workspace) if ws_bytes else None
    ws_len = workspace.numel() * workspace.element_size() if (ws_bytes and workspace is not None) else 0
    _check(lib.dhsa_chunk_score_select_budget(_ptr(Qp), _ptr(Kp), B, Hq, Hkv, nmax, _ptr(off), _ptr(n_chunks),
                                              int(budget), _ptr(budgets), recent, k_max, _ptr(sel), _ptr(n_sel),
                                              ws_ptr, ws_len, _stream_ptr()), "dhsa_chunk_score_select_budget")
    return sel, n_sel


def build_block_csr(sel: torch.Tensor, n_sel: torch.Tensor, k: int, off: torch.Tensor, n_chunks: torch.Tensor,
                    row_ptr=None, col_idx=None, cost=None, want_cost: bool = True):
    B, Hq, nmax, stride = sel.shape
    lib = load()
    _need(sel, torch.int32, None, "sel")
    _need(n_sel, torch.int32, (B, Hq, nmax), "n_sel")
    if row_ptr is None:
        row_ptr = torch.empty(B * Hq * nmax + 1, dtype=torch.int32, device=sel.device)
    if col_idx is None:
        col_idx = torch.empty(lib.dhsa_csr_nnz_upper(B, Hq, nmax, k), dtype=torch.int32, device=sel.device)
    if cost is None and want_cost:
        cost = torch.empty(B * Hq * nmax, dtype=torch.int64, device=sel.device)
    _check(lib.dhsa_build_block_csr(_ptr(sel), _ptr(n_sel), B, Hq, nmax, k, _ptr(off), _ptr(n_chunks),
                                    _ptr(row_ptr), _ptr(col_idx), _ptr(cost), _stream_ptr()),
           "dhsa_build_block_csr")
    return row_ptr, col_idx, cost


def sparse_attn_fwd(Q: torch.Tensor, K: torch.Tensor, V: torch.Tensor, off: torch.Tensor, n_chunks: torch.Tensor,
                    row_ptr: torch.Tensor, col_idx: torch.Tensor, cost: Optional[torch.Tensor] = None,
                    softmax_scale: Optional[float] = None, out: Optional[torch.Tensor] = None,
                    workspace: Optional[torch.Tensor] = None, short_tiles: int = 0):
    """Attention over the kept chunk pairs. short_tiles != 0 calls the
    tile-policy entry (include/dhsa.h, 4c): 1 sends chunk tails of at most 64
    rows, 2 every row, to the 64-row kernel."""
    B, Hq, L, d = Q.shape
    Hkv = K.shape[1]
    nmax = off.shape[1] - 1
    _need(Q, torch.bfloat16, None, "Q")
    _need(K, torch.bfloat16, (B, Hkv, L, d), "K")
    _need(V, torch.bfloat16, (B, Hkv, L, d), "V")
    lib = load()
    if out is None:
        out = torch.empty_like(Q)
    _need(out, torch.bfloat16, (B, Hq, L, d), "out")
    ws_bytes = lib.dhsa_sparse_attn_tiles_workspace_size(B, Hq, L, nmax, short_tiles)
    if workspace is None:
        workspace = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device=Q.device)
    scale = 1.0 / math.sqrt(d) if softmax_scale is None else float(softmax_scale)
    if short_tiles == 0:
        _check(lib.dhsa_sparse_attn_fwd(_ptr(Q), _ptr(K), _ptr(V), B, Hq, Hkv, L, d, _ptr(off), _ptr(n_chunks),
                                        nmax, _ptr(row_ptr), _ptr(col_idx), _ptr(cost), scale, _ptr(out),
                                        _ptr(workspace), workspace.numel(), _stream_ptr()), "dhsa_sparse_attn_fwd")
    else:
        _check(lib.dhsa_sparse_attn_fwd_tiles(_ptr(Q), _ptr(K), _ptr(V), B, Hq, Hkv, L, d, _ptr(off),
                                              _ptr(n_chunks), nmax, _ptr(row_ptr), _ptr(col_idx), scale,
                                              int(short_tiles), _ptr(out), _ptr(workspace), workspace.numel(),
                                              _stream_ptr()), "dhsa_sparse_attn_fwd_tiles")
    return out


def sparse_attn_fwd_noalloc(Q: torch.Tensor, K: torch.Tensor, V: torch.Tensor, off: torch.Tensor,
                            n_chunks: torch.Tensor, row_ptr: torch.Tensor, col_idx: torch.Tensor,
                            softmax_scale: Optional[float] = None, out: Optional[torch.Tensor] = None):
    """sparse_attn_fwd with the library's static scratch instead of a caller
    workspace (for callers that cannot allocate; see include/dhsa.h, 4b).
    `out` should be preallocated by such callers."""
    B, Hq, L, d = Q.shape
    Hkv = K.shape[1]
    nmax = off.shape[1] - 1
    _need(Q, torch.bfloat16, None, "Q")
    _need(K, torch.bfloat16, (B, Hkv, L, d), "K")
    _need(V, torch.bfloat16, (B, Hkv, L, d), "V")
    if out is None:
        out = torch.empty_like(Q)
    _need(out, torch.bfloat16, (B, Hq, L, d), "out")
    scale = 1.0 / math.sqrt(d) if softmax_scale is None else float(softmax_scale)
    _check(load().dhsa_sparse_attn_fwd_noalloc(_ptr(Q), _ptr(K), _ptr(V), B, Hq, Hkv, L, d, _ptr(off),
                                               _ptr(n_chunks), nmax, _ptr(row_ptr), _ptr(col_idx), scale,
                                               _ptr(out), _stream_ptr()), "dhsa_sparse_attn_fwd_noalloc")
    return out


# ----------------------------------------------------------------- whole layer
class DHSAPrefill:
    """The five calls of one DHSA prefill layer with buffers allocated once.

    run(Q, K, V) does pool(Q), pool(K), score + selection, CSR build and
    sparse attention on the current stream and returns O (bf16, like Q).
    Selection is the top-k rule, or, when `budget` is given (an int, or an
    int32 tensor [B, Hq, Nmax] of per-row budgets), the token-budget rule with
    a window of `recent` chunks and at most k earlier chunks per row.
    `short_tiles` picks the query-tile policy of the attention (0: 128-row
    tiles only, the fast default; 1 and 2: see sparse_attn_fwd).
    `fused_routing` runs pooling, the top-k selection and the CSR as one
    launch (route_fused; top-k rule only). Under the top-k rule the selection
    writes the CSR itself (chunk_score_topk_csr); `csr_from_selection=False`
    runs the separate CSR build instead (the same results).
    """

    def __init__(self, B: int, Hq: int, Hkv: int, L: int, off: torch.Tensor, n_chunks: torch.Tensor, k: int,
                 device="cuda", softmax_scale: Optional[float] = None, budget=None, recent: int = 0,
                 short_tiles: int = 0, fused_routing: bool = False, csr_from_selection: bool = True):
        lib = load()
        self.B, self.Hq, self.Hkv, self.L, self.k = B, Hq, Hkv, L, k
        self.short_tiles = short_tiles
        if fused_routing and budget is not None:
            raise ValueError("fused_routing supports the top-k rule only")
        self.fused_routing = fused_routing
        self.csr_from_selection = csr_from_selection
        self.budget, self.recent = budget, recent
        self.off, self.n_chunks = off, n_chunks
        self.nmax = off.shape[1] - 1
        nmax = self.nmax
        dev = torch.device(device)
        self.scale = 1.0 / math.sqrt(128) if softmax_scale is None else softmax_scale
        self.Qp = torch.empty((B, Hq, nmax, 128), dtype=torch.float32, device=dev)
        self.Kp = torch.empty((B, Hkv, nmax, 128), dtype=torch.float32, device=dev)
        self.stride = lib.dhsa_sel_stride(k, nmax)
        self.sel = torch.empty((B, Hq, nmax, self.stride), dtype=torch.int32, device=dev)
        self.n_sel = torch.empty((B, Hq, nmax), dtype=torch.int32, device=dev)
        ws1 = lib.dhsa_score_topk_workspace_size(B, Hq, nmax)
        self.ws_topk = torch.empty(max(ws1, 1), dtype=torch.uint8, device=dev) if ws1 else None
        self.row_ptr = torch.empty(B * Hq * nmax + 1, dtype=torch.int32, device=dev)
        self.col_idx = torch.empty(lib.dhsa_csr_nnz_upper(B, Hq, nmax, k), dtype=torch.int32, device=dev)
        self.cost = torch.empty(B * Hq * nmax, dtype=torch.int64, device=dev)
        self.ws_attn = torch.empty(max(lib.dhsa_sparse_attn_tiles_workspace_size(B, Hq, L, nmax, short_tiles), 1),
                                   dtype=torch.uint8, device=dev)
        self.O = torch.empty((B, Hq, L, 128), dtype=torch.bfloat16, device=dev)

    def routing(self, Q, K):
        if self.fused_routing:
            route_fused(Q, K, self.off, self.n_chunks, self.k, Qp=self.Qp, Kp=self.Kp, sel=self.sel,
                        n_sel=self.n_sel, workspace=self.ws_topk, row_ptr=self.row_ptr, col_idx=self.col_idx,
                        cost=self.cost)
            return
        chunk_pool_qk(Q, K, self.off, self.n_chunks, Qp=self.Qp, Kp=self.Kp)
        if self.budget is None and self.csr_from_selection:
            chunk_score_topk_csr(self.Qp, self.Kp, self.off, self.n_chunks, self.k, self.sel, self.n_sel,
                                 self.row_ptr, self.col_idx, cost=self.cost, workspace=self.ws_topk)
            return
        if self.budget is None:
            chunk_score_topk(self.Qp, self.Kp, self.n_chunks, self.k, sel=self.sel, n_sel=self.n_sel,
                             workspace=self.ws_topk)
        else:
            chunk_score_select_budget(self.Qp, self.Kp, self.off, self.n_chunks, self.budget, self.recent, self.k,
                                      sel=self.sel, n_sel=self.n_sel, workspace=self.ws_topk)
        build_block_csr(self.sel, self.n_sel, self.k, self.off, self.n_chunks, row_ptr=self.row_ptr,
                        col_idx=self.col_idx, cost=self.cost)

    def attention(self, Q, K, V):
        return sparse_attn_fwd(Q, K, V, self.off, self.n_chunks, self.row_ptr, self.col_idx, self.cost,
                               self.scale, out=self.O, workspace=self.ws_attn, short_tiles=self.short_tiles)

    def run(self, Q, K, V):
        self.routing(Q, K)
        return self.attention(Q, K, V)


class HostStreamedPrefill:
    """Layers whose Q, K, V arrive in pinned host memory and whose O goes back
    to host memory, one call per layer, with the copies overlapped.

    submit(Qh, Kh, Vh, Oh) enqueues: the host-to-device copy of the layer's
    inputs on a copy-in stream, routing + attention on a compute stream, and
    the device-to-host copy of O on a copy-out stream, chained by events.
    Inputs and outputs are double-buffered on the device, so the copy-in of
    layer s+1 and the copy-out of layer s-1 run while layer s computes (the
    two copy directions use the two PCIe directions). Returns at once;
    synchronize() waits for every submitted layer. Host buffers must stay
    untouched until then.
    """

    def __init__(self, layer: DHSAPrefill):
        self.layer = layer
        dev = layer.O.device
        B, Hq, Hkv, L = layer.B, layer.Hq, layer.Hkv, layer.L
        self.Qd = [torch.empty((B, Hq, L, 128), dtype=torch.bfloat16, device=dev) for _ in range(2)]
        self.Kd = [torch.empty((B, Hkv, L, 128), dtype=torch.bfloat16, device=dev) for _ in range(2)]
        self.Vd = [torch.empty((B, Hkv, L, 128), dtype=torch.bfloat16, device=dev) for _ in range(2)]
        self.Od = [layer.O, torch.empty_like(layer.O)]
        self.s_in, self.s_comp, self.s_out = (torch.cuda.Stream(dev) for _ in range(3))
        self.e_in = [torch.cuda.Event() for _ in range(2)]
        self.e_comp = [torch.cuda.Event() for _ in range(2)]
        self.e_out = [torch.cuda.Event() for _ in range(2)]
        self.n = 0

    def submit(self, Qh: torch.Tensor, Kh: torch.Tensor, Vh: torch.Tensor, Oh: torch.Tensor):
        b = self.n & 1
        lay = self.layer
        if self.n >= 2:
            self.s_in.wait_event(self.e_comp[b])       # layer n-2 has read this input set
        with torch.cuda.stream(self.s_in):
            self.Qd[b].copy_(Qh, non_blocking=True)
            self.Kd[b].copy_(Kh, non_blocking=True)
            self.Vd[b].copy_(Vh, non_blocking=True)
            self.e_in[b].record(self.s_in)
        self.s_comp.wait_event(self.e_in[b])
        if self.n >= 2:
            self.s_comp.wait_event(self.e_out[b])      # layer n-2's O has left this buffer
        with torch.cuda.stream(self.s_comp):
            lay.routing(self.Qd[b], self.Kd[b])
            sparse_attn_fwd(self.Qd[b], self.Kd[b], self.Vd[b], lay.off, lay.n_chunks, lay.row_ptr, lay.col_idx,
                            lay.cost, lay.scale, out=self.Od[b], workspace=lay.ws_attn)
            self.e_comp[b].record(self.s_comp)
        self.s_out.wait_event(self.e_comp[b])
        with torch.cuda.stream(self.s_out):
            Oh.copy_(self.Od[b], non_blocking=True)
            self.e_out[b].record(self.s_out)
        self.n += 1

    def synchronize(self):
        for s in (self.s_in, self.s_comp, self.s_out):
            s.synchronize()


class GraphedPrefill:
    """One DHSA layer captured as a CUDA graph: the eight launches of
    DHSAPrefill.run replayed with one graph launch.

    Q, K, V are the device tensors the graph reads; refill them in place and
    call replay(), which returns the layer's O tensor (the same buffer each
    time). The chunk offsets and the selection settings are those of `layer`
    at capture time.
    """

    def __init__(self, layer: DHSAPrefill, Q: torch.Tensor, K: torch.Tensor, V: torch.Tensor):
        self.layer, self.Q, self.K, self.V = layer, Q, K, V
        s = torch.cuda.Stream(Q.device)
        s.wait_stream(torch.cuda.current_stream(Q.device))
        with torch.cuda.stream(s):              # one eager run first (module load, function attributes)
            layer.run(Q, K, V)
        torch.cuda.current_stream(Q.device).wait_stream(s)
        torch.cuda.synchronize(Q.device)
        self.graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.graph):
            self.O = layer.run(Q, K, V)

    def replay(self) -> torch.Tensor:
        self.graph.replay()
        return self.O
