"""Python binding of liblowram.so: the C entry points of include/lowram.h under the same
names, with torch CUDA tensors in place of device pointers.

This layer only marshals arguments: every step of the compressed-cache path runs
in the library's CUDA kernels. A missing library raises at import of the first
call; there is no other implementation to fall back to.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "liblowram.so")

LR_OK, LR_ERR_INVALID_ARG, LR_ERR_UNSUPPORTED, LR_ERR_WORKSPACE, LR_ERR_CUDA, LR_ERR_DEVICE_CHECK = range(6)
LR_F32, LR_BF16 = 0, 1
LR_BLOCK_TOKENS = 64
LR_MAX_TAIL = 4096
LR_DEVERR_BLOCK_RANGE, LR_DEVERR_BLOCK_ORDER, LR_DEVERR_RES_RANGE, LR_DEVERR_RES_ORDER, LR_DEVERR_PTR = 1, 2, 4, 8, 16
LR_DEVERR_TIMEOUT, LR_DEVERR_LAUNCH = 32, 64

_DT = {torch.float32: LR_F32, torch.bfloat16: LR_BF16}


class LowRAMError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{message} (status {status})")
        self.status = status


class lr_cache_shape(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int32), ("T", ctypes.c_int32), ("n_layers", ctypes.c_int32),
                ("n_kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32), ("rank", ctypes.c_int32),
                ("hidden", ctypes.c_int32), ("dtype", ctypes.c_int32)]


class lr_predictor(ctypes.Structure):
    _fields_ = [("W_lin", ctypes.c_void_p), ("W1", ctypes.c_void_p), ("b1", ctypes.c_void_p),
                ("W2", ctypes.c_void_p), ("b2", ctypes.c_void_p), ("per_sequence", ctypes.c_int32)]


class lr_predictor_f32(ctypes.Structure):
    _fields_ = [("W_lin", ctypes.c_void_p), ("W1", ctypes.c_void_p), ("b1", ctypes.c_void_p),
                ("W2", ctypes.c_void_p), ("b2", ctypes.c_void_p), ("per_sequence", ctypes.c_int32)]


class lr_predictor_out(ctypes.Structure):
    _fields_ = [("W_lin", ctypes.c_void_p), ("W1", ctypes.c_void_p), ("b1", ctypes.c_void_p),
                ("W2", ctypes.c_void_p), ("b2", ctypes.c_void_p)]


_lib = None
_P = ctypes.c_void_p
_I = ctypes.c_int32
_Z = ctypes.c_size_t


def library() -> ctypes.CDLL:
    """Load liblowram.so (built in-tree); raises if it is missing."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m long_context_decode_lr_b200.build`")
        lib = ctypes.CDLL(LIB_PATH)
        S, Pr = ctypes.POINTER(lr_cache_shape), ctypes.POINTER(lr_predictor)
        sig = {
            "lr_pack_workspace_bytes": (_Z, [S, _I]),
            "lr_pack_prefill": (_I, [S, _P, _P, _P, Pr, _I, _P, _P, _P, _P, _P, _P, _Z, _P]),
            "lr_decode_workspace_bytes": (_Z, [S, _I, _I]),
            "lr_decode_attn": (_I, [S, _I, _I, _P, _P, _P, Pr, _P, _P, _P, _I, _P, _I, ctypes.c_float,
                                    _P, _P, _Z, _P]),
            "lr_decode_attn_noalloc": (_I, [S, _I, _I, _P, _P, _P, Pr, _P, _P, _P, _I, _P, _I, ctypes.c_float,
                                            _P, _P]),
            "lr_decode_attn_tail": (_I, [S, _I, _I, _P, _P, _P, Pr, _P, _P, _P, _I, _P, _I, _P, _P, _I,
                                         ctypes.c_float, _P, _P, _Z, _P]),
            "lr_select_workspace_bytes": (_Z, [S, _I]),
            "lr_block_means": (_I, [S, _P, _P, _P]),
            "lr_fit_workspace_bytes": (_Z, [S, _I]),
            "lr_fit_predictor": (_I, [S, _P, _P, _P, ctypes.POINTER(lr_predictor_f32), _I, ctypes.c_float,
                                      ctypes.POINTER(lr_predictor_out), _P, _Z, _P]),
            "lr_quantize_residuals": (_I, [S, ctypes.c_int64, _P, _P, _P, _P, _P]),
            "lr_decode_attn_q2": (_I, [S, _I, _I, _P, _P, _P, Pr, _P, _P, _P, _P, _P, _I, _P, _I, ctypes.c_float,
                                       _P, _P, _Z, _P]),
            "lr_select_blocks": (_I, [S, _I, _I, _P, _P, _P, _I, ctypes.c_float, _P, _P, _P, _Z, _P]),
            "lr_topk_workspace_bytes": (_Z, [_I, _I, _I]),
            "lr_topk_tokens": (_I, [_P, _I, _I, _I, _P, _P, _Z, _P]),
            "lr_residual_block_ptr": (_I, [_P, _I, _I, _I, _P, _P]),
            "lr_get_device_error": (_I, [_P, _P, ctypes.POINTER(_I)]),
            "lr_status_string": (ctypes.c_char_p, [_I]),
            "lr_last_error": (ctypes.c_char_p, []),
            "lr_abi_version": (_I, []),
        }
        for name, (res, args) in sig.items():
            f = getattr(lib, name)
            f.restype, f.argtypes = res, args
        _lib = lib
    return _lib


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    if t is None:
        return None
    if not isinstance(t, torch.Tensor):
        raise TypeError("expected a torch.Tensor or None")
    if not t.is_cuda:
        raise ValueError("tensor must live on a CUDA device")
    if not t.is_contiguous():
        raise ValueError("tensor must be contiguous")
    return t.data_ptr() or None


def _stream(stream) -> Optional[int]:
    if stream is None:
        stream = torch.cuda.current_stream()
    return getattr(stream, "cuda_stream", stream) or None


def _check(status: int) -> None:
    if status != LR_OK:
        lib = library()
        raise LowRAMError(status, lib.lr_last_error().decode() or lib.lr_status_string(status).decode())


def cache_shape(batch: int, T: int, n_layers: int, n_kv_heads: int, head_dim: int, rank: int,
                hidden: int, dtype) -> lr_cache_shape:
    dt = _DT[dtype] if isinstance(dtype, torch.dtype) else int(dtype)
    return lr_cache_shape(batch, T, n_layers, n_kv_heads, head_dim, rank, hidden, dt)


class Predictor:
    """Holds the predictor tensors alive and exposes the C struct."""

    def __init__(self, W_lin, W1, b1, W2, b2=None, per_sequence: bool = True):
        self.tensors = (W_lin, W1, b1, W2, b2)
        self.c = lr_predictor(_ptr(W_lin), _ptr(W1), _ptr(b1), _ptr(W2), _ptr(b2), int(per_sequence))


def lr_abi_version() -> int:
    return library().lr_abi_version()


def lr_pack_workspace_bytes(shape: lr_cache_shape, k: int) -> int:
    return library().lr_pack_workspace_bytes(ctypes.byref(shape), k)


def lr_pack_prefill(shape, K_group, V, Bt, predictor: Predictor, k, A, res_idx, res_val,
                    res_blk_ptr=None, err_out=None, ws=None, stream=None) -> None:
    _check(library().lr_pack_prefill(
        ctypes.byref(shape), _ptr(K_group), _ptr(V), _ptr(Bt), ctypes.byref(predictor.c), k, _ptr(A),
        _ptr(res_idx), _ptr(res_val), _ptr(res_blk_ptr), _ptr(err_out), _ptr(ws),
        0 if ws is None else ws.numel() * ws.element_size(), _stream(stream)))


def lr_decode_workspace_bytes(shape: lr_cache_shape, n_q_heads: int, n_sel: int = 0) -> int:
    return library().lr_decode_workspace_bytes(ctypes.byref(shape), n_q_heads, n_sel)


def lr_decode_attn(shape, layer, n_q_heads, q, A, Bt, predictor: Predictor, res_idx, res_val,
                   res_blk_ptr, k, block_list, n_sel, scale, o, ws, stream=None) -> None:
    _check(library().lr_decode_attn(
        ctypes.byref(shape), layer, n_q_heads, _ptr(q), _ptr(A), _ptr(Bt), ctypes.byref(predictor.c),
        _ptr(res_idx), _ptr(res_val), _ptr(res_blk_ptr), k, _ptr(block_list), n_sel, float(scale),
        _ptr(o), _ptr(ws), 0 if ws is None else ws.numel() * ws.element_size(), _stream(stream)))


def lr_fit_workspace_bytes(shape: lr_cache_shape, per_sequence: bool = True) -> int:
    return library().lr_fit_workspace_bytes(ctypes.byref(shape), int(per_sequence))


def lr_fit_predictor(shape, A, Bt, V, params, n_steps, lr, ws, out=None, per_sequence=True, stream=None) -> None:
    """Fit the predictor to the context: params = (W_lin, W1, b1, W2, b2 or None), fp32 tensors
    updated in place; out = the same five in the cache dtype (written after the last step) or None."""
    p = lr_predictor_f32(*[_ptr(t) for t in params], int(per_sequence))
    o = None if out is None else ctypes.byref(lr_predictor_out(*[_ptr(t) for t in out]))
    _check(library().lr_fit_predictor(ctypes.byref(shape), _ptr(A), _ptr(Bt), _ptr(V), ctypes.byref(p), int(n_steps),
                                      float(lr), o, _ptr(ws), 0 if ws is None else ws.numel() * ws.element_size(),
                                      _stream(stream)))


def lr_quantize_residuals(shape, n_rows, res_val, res_codes, res_lo, res_step, stream=None) -> None:
    """2-bit codes [n_rows, hd / 4] uint8 plus row minimum and step (fp32) of residual rows."""
    _check(library().lr_quantize_residuals(ctypes.byref(shape), int(n_rows), _ptr(res_val), _ptr(res_codes),
                                           _ptr(res_lo), _ptr(res_step), _stream(stream)))


def lr_decode_attn_q2(shape, layer, n_q_heads, q, A, Bt, predictor: Predictor, res_idx, res_codes, res_lo,
                      res_step, res_blk_ptr, k, block_list, n_sel, scale, o, ws, stream=None) -> None:
    """lr_decode_attn with 2-bit residual rows (codes, row minimum, step)."""
    _check(library().lr_decode_attn_q2(
        ctypes.byref(shape), layer, n_q_heads, _ptr(q), _ptr(A), _ptr(Bt), ctypes.byref(predictor.c),
        _ptr(res_idx), _ptr(res_codes), _ptr(res_lo), _ptr(res_step), _ptr(res_blk_ptr), k, _ptr(block_list),
        n_sel, float(scale), _ptr(o), _ptr(ws), 0 if ws is None else ws.numel() * ws.element_size(),
        _stream(stream)))


def lr_decode_attn_noalloc(shape, layer, n_q_heads, q, A, Bt, predictor: Predictor, res_idx, res_val,
                           res_blk_ptr, k, block_list, n_sel, scale, o, stream=None) -> None:
    """lr_decode_attn on the library's static scratch area (no workspace, no allocation)."""
    _check(library().lr_decode_attn_noalloc(
        ctypes.byref(shape), layer, n_q_heads, _ptr(q), _ptr(A), _ptr(Bt), ctypes.byref(predictor.c),
        _ptr(res_idx), _ptr(res_val), _ptr(res_blk_ptr), k, _ptr(block_list), n_sel, float(scale),
        _ptr(o), _stream(stream)))


def lr_decode_attn_tail(shape, layer, n_q_heads, q, A, Bt, predictor: Predictor, res_idx, res_val,
                        res_blk_ptr, k, block_list, n_sel, tail_K, tail_V, n_tail, scale, o, ws,
                        stream=None) -> None:
    """lr_decode_attn plus an exact recent-token tail tail_K / tail_V [B, Hkv, n_tail, hd]."""
    _check(library().lr_decode_attn_tail(
        ctypes.byref(shape), layer, n_q_heads, _ptr(q), _ptr(A), _ptr(Bt), ctypes.byref(predictor.c),
        _ptr(res_idx), _ptr(res_val), _ptr(res_blk_ptr), k, _ptr(block_list), n_sel, _ptr(tail_K),
        _ptr(tail_V), n_tail, float(scale), _ptr(o), _ptr(ws), 0 if ws is None else ws.numel() * ws.element_size(),
        _stream(stream)))


def lr_select_workspace_bytes(shape: lr_cache_shape, n_q_heads: int) -> int:
    return library().lr_select_workspace_bytes(ctypes.byref(shape), n_q_heads)


def lr_block_means(shape, A, Abar, stream=None) -> None:
    """Abar [B, nblk, r] fp32: the mean A row of every 64-token block (query-independent)."""
    _check(library().lr_block_means(ctypes.byref(shape), _ptr(A), _ptr(Abar), _stream(stream)))


def lr_select_blocks(shape, layer, n_q_heads, q, Abar, Bt, n_sel, scale, block_list, ws, scores_out=None,
                     stream=None) -> None:
    """The n_sel blocks per (sequence, KV head) whose mean rebuilt key best matches the query;
    scores_out [B, Hkv, nblk] fp32 (optional) receives the scores the list was taken from."""
    _check(library().lr_select_blocks(
        ctypes.byref(shape), layer, n_q_heads, _ptr(q), _ptr(Abar), _ptr(Bt), n_sel, float(scale),
        _ptr(block_list), _ptr(scores_out), _ptr(ws), 0 if ws is None else ws.numel() * ws.element_size(),
        _stream(stream)))


def lr_topk_workspace_bytes(n_segments: int, T: int, k: int) -> int:
    return library().lr_topk_workspace_bytes(n_segments, T, k)


def lr_topk_tokens(err, n_segments, T, k, idx_out, ws, stream=None) -> None:
    _check(library().lr_topk_tokens(_ptr(err), n_segments, T, k, _ptr(idx_out), _ptr(ws),
                                    0 if ws is None else ws.numel() * ws.element_size(), _stream(stream)))


def lr_residual_block_ptr(idx, n_segments, k, T, ptr_out, stream=None) -> None:
    _check(library().lr_residual_block_ptr(_ptr(idx), n_segments, k, T, _ptr(ptr_out), _stream(stream)))


def lr_get_device_error(ws, stream=None) -> int:
    code = ctypes.c_int32(0)
    st = library().lr_get_device_error(_ptr(ws), _stream(stream), ctypes.byref(code))
    if st not in (LR_OK, LR_ERR_DEVICE_CHECK):
        _check(st)
    return code.value


def workspace(nbytes: int, device=None) -> torch.Tensor:
    """A caller-owned workspace tensor (256-byte aligned by the caching allocator)."""
    return torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device or "cuda")
