"""ctypes binding of libress.so: the C entry points of include/ress.h under the same names.

Argument marshalling only: shapes and parameters are packed into the C structs, torch
tensors are passed as raw device pointers, and a non-OK status raises RessError.  Every
step of the computation runs in the library's CUDA kernels.  If libress.so has not been
built, the first call raises RessError (there is no fallback implementation).
"""
from __future__ import annotations

import ctypes
import os
import threading
from typing import Optional, Sequence

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libress.so")

RESS_OK = 0
STATUS_NAMES = {0: "RESS_OK", 1: "RESS_ERR_INVALID_ARG", 2: "RESS_ERR_UNSUPPORTED",
                3: "RESS_ERR_CUDA", 4: "RESS_ERR_DEVICE_BOUNDS", 5: "RESS_ERR_DEVICE_TIMEOUT"}
SELECT_MASS, SELECT_DRIFT, SELECT_RANDOM, SELECT_CDF = 0, 1, 2, 3
DRIFT_MINIMISE, DRIFT_MAXIMISE_SWAPS, DRIFT_MAXIMISE_FULL = 0, 1, 2
HEAD_DIM, BLOCK = 64, 128


class RessError(RuntimeError):
    def __init__(self, fn: str, status: int):
        super().__init__(f"{fn} failed: {STATUS_NAMES.get(status, status)}")
        self.status = status


class ress_shape(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int32), ("heads", ctypes.c_int32), ("seq_len", ctypes.c_int32),
                ("head_dim", ctypes.c_int32), ("block", ctypes.c_int32),
                ("key_block", ctypes.c_int32)]


class ress_select_params(ctypes.Structure):
    _fields_ = [("method", ctypes.c_int32), ("budgets", ctypes.POINTER(ctypes.c_int32)),
                ("keep_k", ctypes.c_void_p), ("dense_q", ctypes.c_void_p),
                ("rounds", ctypes.c_int32), ("rho", ctypes.c_float), ("eps", ctypes.c_float),
                ("seed", ctypes.c_uint64), ("objective", ctypes.c_int32), ("top_p", ctypes.c_float),
                ("drift", ctypes.c_void_p)]


_lib = None
_lock = threading.Lock()
_VP, _I32, _SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_size_t
_SIGS = {
    "ress_abi_version": (_I32, []),
    "ress_status_string": (ctypes.c_char_p, [_I32]),
    "ress_head_gram": (_I32, [ctypes.POINTER(ress_shape), _I32, _VP, _VP, _VP]),
    "ress_token_gather": (_I32, [ctypes.POINTER(ress_shape), _I32, _I32, _I32, _VP, _VP, _VP]),
    "ress_pool_blocks": (_I32, [ctypes.POINTER(ress_shape), _VP, _VP, _VP, _VP, _VP, _VP, _VP]),
    "ress_block_scores": (_I32, [ctypes.POINTER(ress_shape), _VP, _VP, _VP, ctypes.c_float, _VP,
                                 _VP, _VP]),
    "ress_drift_workspace_bytes": (_SZ, [ctypes.POINTER(ress_shape)]),
    "ress_drift_scores": (_I32, [ctypes.POINTER(ress_shape), _VP, _VP, _VP, _VP, _VP, _VP, _SZ,
                                 _VP]),
    "ress_drift_scores_static": (_I32, [ctypes.POINTER(ress_shape), _VP, _VP, _VP, _VP, _VP, _VP]),
    "ress_select_blocks": (_I32, [ctypes.POINTER(ress_shape), ctypes.POINTER(ress_select_params),
                                  _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP]),
    "ress_scores_select": (_I32, [ctypes.POINTER(ress_shape), ctypes.POINTER(ress_select_params),
                                  _VP, _VP, _VP, ctypes.c_float, _VP, _VP, _VP, _VP, _VP, _VP,
                                  _VP]),
    "ress_drift_select_workspace_bytes": (_SZ, [ctypes.POINTER(ress_shape)]),
    "ress_drift_select": (_I32, [ctypes.POINTER(ress_shape), ctypes.POINTER(ress_select_params),
                                 _VP, _VP, _VP, _VP, ctypes.c_float, _VP, _VP, _VP, _VP, _VP,
                                 _VP, _VP, _VP, _SZ, _VP]),
    "ress_attn_schedule": (_I32, [ctypes.POINTER(ress_shape), _VP, _VP, _VP]),
    "ress_block_sparse_attn": (_I32, [ctypes.POINTER(ress_shape), _VP, _VP, _VP, _VP, _VP, _VP,
                                      ctypes.c_float, _VP, _VP, _VP, _VP]),
    "ress_debug_attn_forced_timeout": (_I32, [ctypes.POINTER(ress_shape), _VP, _VP, _VP, _VP,
                                              _VP, ctypes.c_float, _VP, _VP, ctypes.c_int64,
                                              _VP]),
}


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """Loads libress.so (once).  Raises RessError-compatible RuntimeError if missing."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(path):
                raise RuntimeError(f"libress.so not built at {path}; run "
                                   "`python -m block_sparse_global_b200.build`")
            lib = ctypes.CDLL(path)
            for name, (res, args) in _SIGS.items():
                fn = getattr(lib, name)
                fn.restype = res
                fn.argtypes = args
            _lib = lib
        return _lib


def _check(fn: str, status: int):
    if status != RESS_OK:
        raise RessError(fn, status)


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not isinstance(t, torch.Tensor):
        raise TypeError("expected a torch.Tensor or None")
    if not t.is_contiguous():
        raise ValueError("tensors passed to libress must be contiguous")
    return t.data_ptr() or None


def _stream(stream) -> Optional[int]:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream if torch.cuda.is_available() else None
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def make_shape(batch: int, heads: int, seq_len: int, head_dim: int = HEAD_DIM,
               block: int = BLOCK, key_block: int = 0) -> ress_shape:
    """key_block 0 means key blocks of the query block's size (128); 64 is the grid of
    ReSS Supp. F (128-token query blocks, 64-token key blocks)."""
    return ress_shape(batch, heads, seq_len, head_dim, block, key_block)


def grid(seq_len: int, key_block: int = 0):
    """(nq, nk): query blocks of 128 tokens and key blocks of key_block tokens."""
    kb = key_block or BLOCK
    return (seq_len + BLOCK - 1) // BLOCK, (seq_len + kb - 1) // kb


def _shape(shape) -> ress_shape:
    if isinstance(shape, ress_shape):
        return shape
    return make_shape(*shape)


def ress_abi_version() -> int:
    return load().ress_abi_version()


def ress_status_string(status: int) -> str:
    return load().ress_status_string(status).decode()


def ress_head_gram(shape, w_o: torch.Tensor, gram: torch.Tensor, stream=None):
    st = load().ress_head_gram(ctypes.byref(_shape(shape)), int(w_o.shape[0]), _ptr(w_o),
                               _ptr(gram), _stream(stream))
    _check("ress_head_gram", st)


def ress_pool_blocks(shape, q, k, v, q_pool, k_pool, v_pool, stream=None):
    st = load().ress_pool_blocks(ctypes.byref(_shape(shape)), _ptr(q), _ptr(k), _ptr(v),
                                 _ptr(q_pool), _ptr(k_pool), _ptr(v_pool), _stream(stream))
    _check("ress_pool_blocks", st)


def ress_block_scores(shape, q_pool, k_pool, v_pool, scale: float, P, v_bar, stream=None):
    st = load().ress_block_scores(ctypes.byref(_shape(shape)), _ptr(q_pool), _ptr(k_pool),
                                  _ptr(v_pool), float(scale), _ptr(P), _ptr(v_bar), _stream(stream))
    _check("ress_block_scores", st)


def ress_drift_workspace_bytes(shape) -> int:
    return int(load().ress_drift_workspace_bytes(ctypes.byref(_shape(shape))))


def ress_drift_scores(shape, P, v_pool, v_bar, gram, s, workspace: torch.Tensor, stream=None):
    nbytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    st = load().ress_drift_scores(ctypes.byref(_shape(shape)), _ptr(P), _ptr(v_pool), _ptr(v_bar),
                                  _ptr(gram), _ptr(s), _ptr(workspace), nbytes, _stream(stream))
    _check("ress_drift_scores", st)


def ress_drift_scores_static(shape, P, v_pool, v_bar, gram, s, stream=None):
    """Drift score with the library's fixed static scratch (no workspace argument), for
    callers that cannot allocate device memory; see include/ress.h."""
    st = load().ress_drift_scores_static(ctypes.byref(_shape(shape)), _ptr(P), _ptr(v_pool),
                                         _ptr(v_bar), _ptr(gram), _ptr(s), _stream(stream))
    _check("ress_drift_scores_static", st)


def select_params(method: int, budgets: Sequence[int], keep_k=None, dense_q=None, rounds: int = 0,
                  rho: float = 0.5, eps: float = 1e-4, seed: int = 0, objective: int = 0,
                  drift=None, top_p: float = 1.0):
    """Packs ress_select_params (`drift`: optional fp32 [B,H,nb] device tensor for the
    realized J per row).  Returns (struct, host budget array that must stay alive)."""
    arr = (ctypes.c_int32 * len(budgets))(*[int(b) for b in budgets])
    p = ress_select_params(int(method), ctypes.cast(arr, ctypes.POINTER(ctypes.c_int32)),
                           _ptr(keep_k), _ptr(dense_q), int(rounds), float(rho), float(eps),
                           int(seed) & ((1 << 64) - 1), int(objective), float(top_p), _ptr(drift))
    return p, arr


def ress_select_blocks(shape, params, P, s, v_pool, v_bar, gram, kv_idx, kv_cnt, mask=None,
                       dev_err=None, stream=None):
    """params: a ress_select_params, or the (struct, budgets) pair of select_params()."""
    keep = None
    if isinstance(params, tuple):
        params, keep = params
    st = load().ress_select_blocks(ctypes.byref(_shape(shape)), ctypes.byref(params), _ptr(P),
                                   _ptr(s), _ptr(v_pool), _ptr(v_bar), _ptr(gram), _ptr(kv_idx),
                                   _ptr(kv_cnt), _ptr(mask), _ptr(dev_err), _stream(stream))
    del keep
    _check("ress_select_blocks", st)


def ress_scores_select(shape, params, q_pool, k_pool, v_pool, scale: float, P, v_bar, kv_idx,
                       kv_cnt, mask=None, dev_err=None, stream=None):
    """Block map fused with MASS / RANDOM selection; P and v_bar may be None."""
    keep = None
    if isinstance(params, tuple):
        params, keep = params
    st = load().ress_scores_select(ctypes.byref(_shape(shape)), ctypes.byref(params), _ptr(q_pool),
                                   _ptr(k_pool), _ptr(v_pool), float(scale), _ptr(P), _ptr(v_bar),
                                   _ptr(kv_idx), _ptr(kv_cnt), _ptr(mask), _ptr(dev_err),
                                   _stream(stream))
    del keep
    _check("ress_scores_select", st)


def ress_drift_select_workspace_bytes(shape) -> int:
    return int(load().ress_drift_select_workspace_bytes(ctypes.byref(_shape(shape))))


def ress_drift_select(shape, params, q_pool, k_pool, v_pool, gram, scale: float, P, v_bar, s,
                      kv_idx, kv_cnt, workspace: torch.Tensor, mask=None, dev_err=None,
                      stream=None):
    """Block map, drift score and DRIFT selection in one kernel; P, v_bar, s may be None."""
    keep = None
    if isinstance(params, tuple):
        params, keep = params
    st = load().ress_drift_select(ctypes.byref(_shape(shape)), ctypes.byref(params), _ptr(q_pool),
                                  _ptr(k_pool), _ptr(v_pool), _ptr(gram), float(scale), _ptr(P),
                                  _ptr(v_bar), _ptr(s), _ptr(kv_idx), _ptr(kv_cnt), _ptr(mask),
                                  _ptr(dev_err), _ptr(workspace),
                                  workspace.numel() * workspace.element_size(), _stream(stream))
    del keep
    _check("ress_drift_select", st)


def ress_token_gather(shape, views: int, specials: int, inverse: bool, src, dst, stream=None):
    """Moves every view's special tokens to the tail (inverse=False) or back."""
    st = load().ress_token_gather(ctypes.byref(_shape(shape)), int(views), int(specials),
                                  1 if inverse else 0, _ptr(src), _ptr(dst), _stream(stream))
    _check("ress_token_gather", st)


def ress_attn_schedule(shape, kv_cnt, work_order, stream=None):
    st = load().ress_attn_schedule(ctypes.byref(_shape(shape)), _ptr(kv_cnt), _ptr(work_order),
                                   _stream(stream))
    _check("ress_attn_schedule", st)


def ress_block_sparse_attn(shape, q, k, v, kv_idx, kv_cnt, work_order, scale: float, out,
                           lse=None, dev_err=None, stream=None):
    st = load().ress_block_sparse_attn(ctypes.byref(_shape(shape)), _ptr(q), _ptr(k), _ptr(v),
                                       _ptr(kv_idx), _ptr(kv_cnt), _ptr(work_order), float(scale),
                                       _ptr(out), _ptr(lse), _ptr(dev_err), _stream(stream))
    _check("ress_block_sparse_attn", st)


def ress_debug_attn_forced_timeout(shape, q, k, v, kv_idx, kv_cnt, scale: float, out, dev_err,
                                   limit_cycles: int, stream=None):
    """Diagnostics of the device error path (see include/ress.h): the attention kernel with
    every CTA's softmax stalled on a barrier that nothing completes, so that each takes its
    bounded-wait timeout path and writes RESS_ERR_DEVICE_TIMEOUT to dev_err."""
    st = load().ress_debug_attn_forced_timeout(ctypes.byref(_shape(shape)), _ptr(q), _ptr(k),
                                               _ptr(v), _ptr(kv_idx), _ptr(kv_cnt), float(scale),
                                               _ptr(out), _ptr(dev_err), int(limit_cycles),
                                               _stream(stream))
    _check("ress_debug_attn_forced_timeout", st)
