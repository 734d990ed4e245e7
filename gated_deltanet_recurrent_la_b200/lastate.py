"""Thin Python binding of liblastate.so (C ABI declared in include/la_state.h).

Argument marshalling only: every function takes torch tensors, passes their device
pointers and sizes to the C entry point of the same name, and returns its la_status.
All arithmetic happens in the library's CUDA kernels; there is no fallback path.  If
the shared library is missing, loading raises instead of degrading.

    pool = Pool(tensor, n_qk_heads)          # tensor [n_slots, H_v, d_k, d_v], fp32 / bf16, CUDA
    st = la_state_step("gated_delta", pool, read_slot, pool, write_slot, q, k, v, g, beta, 1.0, o, err)
    check(st)                                # raises LAError unless LA_OK
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "liblastate.so")

RULES = {"linear": 0, "gated": 1, "delta": 2, "gated_delta": 3, "kda": 4}
LA_F32, LA_BF16, LA_Q8 = 0, 1, 2
STATUS = {0: "LA_OK", 1: "LA_ERR_NULL", 2: "LA_ERR_SHAPE", 3: "LA_ERR_UNSUPPORTED", 4: "LA_ERR_ALIGN",
          5: "LA_ERR_ALIAS", 6: "LA_ERR_CUDA"}
LA_OK, LA_ERR_NULL, LA_ERR_SHAPE, LA_ERR_UNSUPPORTED, LA_ERR_ALIGN, LA_ERR_ALIAS, LA_ERR_CUDA = range(7)
DEVERR_READ_SLOT, DEVERR_WRITE_SLOT, DEVERR_CU_SEQLENS, DEVERR_TIMEOUT, DEVERR_Q8_MASK = 1, 2, 4, 8, 16

EXPORTS = ("la_state_bytes", "la_shape_supported", "la_state_step", "la_state_scan", "la_state_scan_chunked",
           "la_state_scan_checkpointed", "la_state_scan_chunked_checkpointed", "la_state_step_qgroups",
           "la_state_scan_qgroups", "la_state_scan_chunked_qgroups",
           "la_pool_slot_bytes", "la_state_pool_encode", "la_state_pool_decode", "la_state_step_conv",
           "la_state_scan_conv", "la_state_scan_chunked_conv", "la_state_scan_chunked_conv_ws",
           "la_scan_chunked_conv_workspace_bytes", "la_scan_chunked_workspace_bytes", "la_scan_chunked_workspace_bytes_rule",
           "la_state_scan_chunked_ws",
           "la_state_scan_chunked_noalloc",
           "la_state_pool_copy",
           "la_state_pool_gather", "la_state_pool_scatter", "la_state_pool_zero", "la_state_check_slots",
           "la_status_str", "la_last_cuda_error", "la_abi_version", "la_debug_set_wait_limit_us",
           "la_debug_withhold_step_tile")


class LAError(RuntimeError):
    def __init__(self, status: int):
        self.status = status
        msg = lib().la_status_str(status).decode() if status in STATUS else f"status {status}"
        if status == LA_ERR_CUDA:
            msg += f" (cudaError {lib().la_last_cuda_error()})"
        super().__init__(msg)


class la_shape(ctypes.Structure):
    _fields_ = [("n_qk_heads", ctypes.c_int32), ("n_v_heads", ctypes.c_int32), ("d_k", ctypes.c_int32),
                ("d_v", ctypes.c_int32)]


class la_pool(ctypes.Structure):
    _fields_ = [("data", ctypes.c_void_p), ("dtype", ctypes.c_int32), ("n_slots", ctypes.c_int32),
                ("shape", la_shape), ("n_hp", ctypes.c_int32), ("hp_mask", ctypes.c_void_p)]


class la_conv(ctypes.Structure):
    _fields_ = [("width", ctypes.c_int32), ("activation", ctypes.c_int32), ("qk_l2norm", ctypes.c_int32),
                ("w_q", ctypes.c_void_p), ("w_k", ctypes.c_void_p), ("w_v", ctypes.c_void_p),
                ("hist_src", ctypes.c_void_p), ("hist_dst", ctypes.c_void_p)]


_lib = None


def lib():
    """The loaded liblastate.so.  Raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m gated_deltanet_recurrent_la_b200.build` (there is no fallback)")
        L = ctypes.CDLL(LIB_PATH)
        P, I32, F = ctypes.c_void_p, ctypes.c_int32, ctypes.c_float
        PP = ctypes.POINTER(la_pool)
        L.la_state_bytes.argtypes = [ctypes.POINTER(la_shape), I32]
        L.la_state_bytes.restype = ctypes.c_size_t
        L.la_shape_supported.argtypes = [I32, I32]
        L.la_shape_supported.restype = ctypes.c_int
        L.la_state_step.argtypes = [I32, PP, P, PP, P, I32, P, P, P, I32, P, P, F, P, P, P]
        L.la_state_step.restype = I32
        L.la_state_scan.argtypes = [I32, PP, P, PP, P, I32, P, I32, P, P, P, P, I32, P, P, F, P, P, P]
        L.la_state_scan.restype = I32
        L.la_state_scan_chunked.argtypes = L.la_state_scan.argtypes
        L.la_state_scan_chunked.restype = I32
        L.la_state_scan_checkpointed.argtypes = L.la_state_scan.argtypes[:-2] + [I32, P, P, P, P]
        L.la_state_scan_checkpointed.restype = I32
        L.la_state_scan_chunked_checkpointed.argtypes = L.la_state_scan_checkpointed.argtypes
        L.la_state_scan_chunked_checkpointed.restype = I32
        L.la_state_step_qgroups.argtypes = L.la_state_step.argtypes[:6] + [I32] + L.la_state_step.argtypes[6:]
        L.la_state_step_qgroups.restype = I32
        L.la_state_scan_qgroups.argtypes = L.la_state_scan.argtypes[:9] + [I32] + L.la_state_scan.argtypes[9:]
        L.la_state_scan_qgroups.restype = I32
        L.la_state_scan_chunked_qgroups.argtypes = L.la_state_scan_qgroups.argtypes
        L.la_state_scan_chunked_qgroups.restype = I32
        L.la_state_pool_copy.argtypes = [PP, I32, P, P, P, P]
        L.la_state_pool_gather.argtypes = [PP, I32, P, P, P, P]
        L.la_state_pool_scatter.argtypes = [PP, I32, P, P, P, P]
        L.la_state_pool_zero.argtypes = [PP, I32, P, P, P]
        for f in (L.la_state_pool_copy, L.la_state_pool_gather, L.la_state_pool_scatter, L.la_state_pool_zero):
            f.restype = I32
        L.la_state_step_conv.argtypes = L.la_state_step.argtypes[:6] + [ctypes.POINTER(la_conv)] + \
            L.la_state_step.argtypes[6:]
        L.la_state_step_conv.restype = I32
        L.la_state_scan_conv.argtypes = L.la_state_scan.argtypes[:9] + [ctypes.POINTER(la_conv)] + \
            L.la_state_scan.argtypes[9:]
        L.la_state_scan_conv.restype = I32
        L.la_state_scan_chunked_conv.argtypes = L.la_state_scan_conv.argtypes
        L.la_state_scan_chunked_conv.restype = I32
        L.la_state_scan_chunked_conv_ws.argtypes = L.la_state_scan_conv.argtypes[:-2] + [ctypes.c_void_p, ctypes.c_size_t] + \
            L.la_state_scan_conv.argtypes[-2:]
        L.la_state_scan_chunked_conv_ws.restype = I32
        L.la_scan_chunked_conv_workspace_bytes.argtypes = [I32, I32]
        L.la_scan_chunked_conv_workspace_bytes.restype = ctypes.c_size_t
        L.la_scan_chunked_workspace_bytes.argtypes = [I32, I32, I32]
        L.la_scan_chunked_workspace_bytes.restype = ctypes.c_size_t
        L.la_scan_chunked_workspace_bytes_rule.argtypes = [ctypes.c_int, I32, I32, I32]
        L.la_scan_chunked_workspace_bytes_rule.restype = ctypes.c_size_t
        L.la_state_scan_chunked_ws.argtypes = L.la_state_scan.argtypes[:-2] + [P, ctypes.c_size_t, P, P]
        L.la_state_scan_chunked_ws.restype = I32
        L.la_state_scan_chunked_noalloc.argtypes = L.la_state_scan.argtypes
        L.la_state_scan_chunked_noalloc.restype = I32
        L.la_pool_slot_bytes.argtypes = [PP]
        L.la_pool_slot_bytes.restype = ctypes.c_size_t
        L.la_state_pool_encode.argtypes = [PP, I32, P, P, P, P]
        L.la_state_pool_encode.restype = I32
        L.la_state_pool_decode.argtypes = [PP, I32, P, P, P, P]
        L.la_state_pool_decode.restype = I32
        L.la_state_check_slots.argtypes = [I32, P, P, I32]
        L.la_state_check_slots.restype = I32
        L.la_status_str.argtypes = [I32]
        L.la_status_str.restype = ctypes.c_char_p
        L.la_last_cuda_error.restype = I32
        L.la_abi_version.restype = I32
        L.la_debug_set_wait_limit_us.argtypes = [ctypes.c_uint32]
        L.la_debug_set_wait_limit_us.restype = None
        L.la_debug_withhold_step_tile.argtypes = [I32]
        L.la_debug_withhold_step_tile.restype = None
        _lib = L
    return _lib


def check(status: int) -> None:
    if status != LA_OK:
        raise LAError(status)


def dtype_code(dt: torch.dtype) -> int:
    if dt == torch.float32:
        return LA_F32
    if dt == torch.bfloat16:
        return LA_BF16
    raise ValueError(f"unsupported dtype {dt}")


def _ptr(t: Optional[torch.Tensor], dtype=None):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("tensor must live on a CUDA device")
    if not t.is_contiguous():
        raise ValueError("tensor must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"expected {dtype}, got {t.dtype}")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


class Pool:
    """A slot pool: tensor [n_slots, H_v, d_k, d_v] (float32 or bfloat16) plus H_qk; or, for
    the mixed INT8 / BF16 storage, Pool.q8(...)."""

    def __init__(self, tensor: torch.Tensor, n_qk_heads: int):
        if tensor.dim() != 4:
            raise ValueError("pool tensor must be [n_slots, H_v, d_k, d_v]")
        self.tensor = tensor
        self.mask = None
        n, hv, dk, dv = tensor.shape
        self.struct = la_pool(_ptr(tensor), dtype_code(tensor.dtype), n,
                              la_shape(int(n_qk_heads), hv, dk, dv), 0, None)

    @classmethod
    def q8(cls, tensor: torch.Tensor, n_qk_heads: int, d_k: int, d_v: int, n_hp: int, mask: torch.Tensor):
        """A q8 pool: tensor uint8 [n_slots, H_v, tile bytes], mask int32 [H_v, d_k / 32]
        holding the uint32 channel-mask words (bit i set: channel i kept in BF16)."""
        if tensor.dim() != 3 or tensor.dtype != torch.uint8:
            raise ValueError("q8 pool tensor must be uint8 [n_slots, H_v, tile bytes]")
        self = cls.__new__(cls)
        self.tensor = tensor
        self.mask = mask
        n, hv, _ = tensor.shape
        self.struct = la_pool(_ptr(tensor), LA_Q8, n, la_shape(int(n_qk_heads), hv, int(d_k), int(d_v)), int(n_hp),
                              _ptr(mask, torch.int32))
        return self

    @property
    def ref(self):
        return ctypes.byref(self.struct)


def la_state_bytes(n_qk_heads: int, n_v_heads: int, d_k: int, d_v: int, dtype: torch.dtype) -> int:
    s = la_shape(n_qk_heads, n_v_heads, d_k, d_v)
    return lib().la_state_bytes(ctypes.byref(s), dtype_code(dtype))


def la_shape_supported(d_k: int, d_v: int) -> bool:
    return bool(lib().la_shape_supported(d_k, d_v))


def la_state_step(rule, src: Pool, read_slot, dst: Pool, write_slot, q, k, v, g, beta, scale, o, err_word,
                  stream=None) -> int:
    io = dtype_code(q.dtype)
    return lib().la_state_step(RULES[rule] if isinstance(rule, str) else int(rule), src.ref,
                               _ptr(read_slot, torch.int32), dst.ref, _ptr(write_slot, torch.int32),
                               int(q.shape[0]), _ptr(q), _ptr(k, q.dtype), _ptr(v, q.dtype), io,
                               _ptr(g, torch.float32), _ptr(beta, torch.float32), float(scale), _ptr(o, q.dtype),
                               _ptr(err_word, torch.int32), _stream(stream))


def la_state_scan(rule, src: Optional[Pool], read_slot, dst: Pool, write_slot, cu_seqlens, q, k, v, g, beta,
                  scale, o, err_word, seq_order=None, stream=None) -> int:
    io = dtype_code(q.dtype)
    return lib().la_state_scan(RULES[rule] if isinstance(rule, str) else int(rule),
                               None if src is None else src.ref, _ptr(read_slot, torch.int32), dst.ref,
                               _ptr(write_slot, torch.int32), int(cu_seqlens.numel() - 1),
                               _ptr(cu_seqlens, torch.int32), int(q.shape[0]), _ptr(seq_order, torch.int32),
                               _ptr(q), _ptr(k, q.dtype), _ptr(v, q.dtype), io, _ptr(g, torch.float32),
                               _ptr(beta, torch.float32), float(scale), _ptr(o, q.dtype),
                               _ptr(err_word, torch.int32), _stream(stream))


def la_state_scan_chunked(rule, src: Optional[Pool], read_slot, dst: Pool, write_slot, cu_seqlens, q, k, v, g, beta,
                          scale, o, err_word, seq_order=None, stream=None) -> int:
    io = dtype_code(q.dtype)
    return lib().la_state_scan_chunked(RULES[rule] if isinstance(rule, str) else int(rule),
                                       None if src is None else src.ref, _ptr(read_slot, torch.int32), dst.ref,
                                       _ptr(write_slot, torch.int32), int(cu_seqlens.numel() - 1),
                                       _ptr(cu_seqlens, torch.int32), int(q.shape[0]), _ptr(seq_order, torch.int32),
                                       _ptr(q), _ptr(k, q.dtype), _ptr(v, q.dtype), io, _ptr(g, torch.float32),
                                       _ptr(beta, torch.float32), float(scale), _ptr(o, q.dtype),
                                       _ptr(err_word, torch.int32), _stream(stream))


def la_scan_chunked_workspace_bytes(total_tokens: int, n_seqs: int, n_v_heads: int) -> int:
    return lib().la_scan_chunked_workspace_bytes(int(total_tokens), int(n_seqs), int(n_v_heads))


def la_scan_chunked_workspace_bytes_rule(rule, total_tokens: int, n_seqs: int, n_v_heads: int) -> int:
    return lib().la_scan_chunked_workspace_bytes_rule(RULES[rule] if isinstance(rule, str) else int(rule),
                                                      int(total_tokens), int(n_seqs), int(n_v_heads))


def la_state_scan_chunked_ws(rule, src: Optional[Pool], read_slot, dst: Pool, write_slot, cu_seqlens, q, k, v, g,
                             beta, scale, o, workspace, err_word, seq_order=None, stream=None) -> int:
    """la_state_scan_chunked in two launches; workspace: a uint8 device tensor of at least
    la_scan_chunked_workspace_bytes_rule(rule, ...) bytes."""
    io = dtype_code(q.dtype)
    return lib().la_state_scan_chunked_ws(
        RULES[rule] if isinstance(rule, str) else int(rule), None if src is None else src.ref,
        _ptr(read_slot, torch.int32), dst.ref, _ptr(write_slot, torch.int32), int(cu_seqlens.numel() - 1),
        _ptr(cu_seqlens, torch.int32), int(q.shape[0]), _ptr(seq_order, torch.int32), _ptr(q), _ptr(k, q.dtype),
        _ptr(v, q.dtype), io, _ptr(g, torch.float32), _ptr(beta, torch.float32), float(scale), _ptr(o, q.dtype),
        _ptr(workspace), int(workspace.numel() * workspace.element_size()), _ptr(err_word, torch.int32),
        _stream(stream))


def la_state_scan_chunked_noalloc(rule, src: Optional[Pool], read_slot, dst: Pool, write_slot, cu_seqlens, q, k, v,
                                  g, beta, scale, o, err_word, seq_order=None, stream=None) -> int:
    """la_state_scan_chunked_ws with the library's own fixed workspace (no scratch argument)."""
    io = dtype_code(q.dtype)
    return lib().la_state_scan_chunked_noalloc(
        RULES[rule] if isinstance(rule, str) else int(rule), None if src is None else src.ref,
        _ptr(read_slot, torch.int32), dst.ref, _ptr(write_slot, torch.int32), int(cu_seqlens.numel() - 1),
        _ptr(cu_seqlens, torch.int32), int(q.shape[0]), _ptr(seq_order, torch.int32), _ptr(q), _ptr(k, q.dtype),
        _ptr(v, q.dtype), io, _ptr(g, torch.float32), _ptr(beta, torch.float32), float(scale), _ptr(o, q.dtype),
        _ptr(err_word, torch.int32), _stream(stream))


def la_state_scan_checkpointed(rule, src: Optional[Pool], read_slot, dst: Pool, write_slot, cu_seqlens, q, k, v, g,
                               beta, scale, o, ckpt_every, ckpt_cu, ckpt_slots, err_word, seq_order=None,
                               stream=None) -> int:
    io = dtype_code(q.dtype)
    return lib().la_state_scan_checkpointed(
        RULES[rule] if isinstance(rule, str) else int(rule), None if src is None else src.ref,
        _ptr(read_slot, torch.int32), dst.ref, _ptr(write_slot, torch.int32), int(cu_seqlens.numel() - 1),
        _ptr(cu_seqlens, torch.int32), int(q.shape[0]), _ptr(seq_order, torch.int32), _ptr(q), _ptr(k, q.dtype),
        _ptr(v, q.dtype), io, _ptr(g, torch.float32), _ptr(beta, torch.float32), float(scale), _ptr(o, q.dtype),
        int(ckpt_every), _ptr(ckpt_cu, torch.int32), _ptr(ckpt_slots, torch.int32), _ptr(err_word, torch.int32),
        _stream(stream))


def la_state_scan_chunked_checkpointed(rule, src: Optional[Pool], read_slot, dst: Pool, write_slot, cu_seqlens, q, k,
                                       v, g, beta, scale, o, ckpt_every, ckpt_cu, ckpt_slots, err_word,
                                       seq_order=None, stream=None) -> int:
    """la_state_scan_checkpointed by the one-launch chunked prefill (ckpt_every a multiple of 64)."""
    io = dtype_code(q.dtype)
    return lib().la_state_scan_chunked_checkpointed(
        RULES[rule] if isinstance(rule, str) else int(rule), None if src is None else src.ref,
        _ptr(read_slot, torch.int32), dst.ref, _ptr(write_slot, torch.int32), int(cu_seqlens.numel() - 1),
        _ptr(cu_seqlens, torch.int32), int(q.shape[0]), _ptr(seq_order, torch.int32), _ptr(q), _ptr(k, q.dtype),
        _ptr(v, q.dtype), io, _ptr(g, torch.float32), _ptr(beta, torch.float32), float(scale), _ptr(o, q.dtype),
        int(ckpt_every), _ptr(ckpt_cu, torch.int32), _ptr(ckpt_slots, torch.int32), _ptr(err_word, torch.int32),
        _stream(stream))


class Conv:
    """The short causal convolution ahead of the step: weights (float32 [heads, channels,
    W] on the device) and the history pools (io dtype [n_slots, H_v, 2 d_k + d_v, W - 1])."""

    def __init__(self, w_q, w_k, w_v, hist_src, hist_dst=None, activation=0, qk_l2norm=0):
        self.keep = (w_q, w_k, w_v, hist_src, hist_dst)
        hist_dst = hist_src if hist_dst is None else hist_dst
        self.struct = la_conv(int(w_q.shape[2]), int(activation), int(qk_l2norm), _ptr(w_q, torch.float32),
                              _ptr(w_k, torch.float32), _ptr(w_v, torch.float32), _ptr(hist_src), _ptr(hist_dst))

    @property
    def ref(self):
        return ctypes.byref(self.struct)


def la_state_step_conv(rule, src: Pool, read_slot, dst: Pool, write_slot, conv: Conv, xq, xk, xv, g, beta, scale, o,
                       err_word, stream=None) -> int:
    io = dtype_code(xq.dtype)
    return lib().la_state_step_conv(RULES[rule] if isinstance(rule, str) else int(rule), src.ref,
                                    _ptr(read_slot, torch.int32), dst.ref, _ptr(write_slot, torch.int32),
                                    int(xq.shape[0]), conv.ref, _ptr(xq), _ptr(xk, xq.dtype), _ptr(xv, xq.dtype), io,
                                    _ptr(g, torch.float32), _ptr(beta, torch.float32), float(scale),
                                    _ptr(o, xq.dtype), _ptr(err_word, torch.int32), _stream(stream))


def la_state_scan_conv(rule, src: Optional[Pool], read_slot, dst: Pool, write_slot, cu_seqlens, conv: Conv, xq, xk,
                       xv, g, beta, scale, o, err_word, seq_order=None, stream=None) -> int:
    io = dtype_code(xq.dtype)
    return lib().la_state_scan_conv(RULES[rule] if isinstance(rule, str) else int(rule),
                                    None if src is None else src.ref, _ptr(read_slot, torch.int32), dst.ref,
                                    _ptr(write_slot, torch.int32), int(cu_seqlens.numel() - 1),
                                    _ptr(cu_seqlens, torch.int32), int(xq.shape[0]), _ptr(seq_order, torch.int32),
                                    conv.ref, _ptr(xq), _ptr(xk, xq.dtype), _ptr(xv, xq.dtype), io,
                                    _ptr(g, torch.float32), _ptr(beta, torch.float32), float(scale),
                                    _ptr(o, xq.dtype), _ptr(err_word, torch.int32), _stream(stream))


def la_state_scan_chunked_conv(rule, src: Optional[Pool], read_slot, dst: Pool, write_slot, cu_seqlens, conv: Conv,
                               xq, xk, xv, g, beta, scale, o, err_word, seq_order=None, stream=None) -> int:
    io = dtype_code(xq.dtype)
    return lib().la_state_scan_chunked_conv(RULES[rule] if isinstance(rule, str) else int(rule),
                                            None if src is None else src.ref, _ptr(read_slot, torch.int32), dst.ref,
                                            _ptr(write_slot, torch.int32), int(cu_seqlens.numel() - 1),
                                            _ptr(cu_seqlens, torch.int32), int(xq.shape[0]),
                                            _ptr(seq_order, torch.int32), conv.ref, _ptr(xq), _ptr(xk, xq.dtype),
                                            _ptr(xv, xq.dtype), io, _ptr(g, torch.float32),
                                            _ptr(beta, torch.float32), float(scale), _ptr(o, xq.dtype),
                                            _ptr(err_word, torch.int32), _stream(stream))


def la_scan_chunked_conv_workspace_bytes(total_tokens: int, n_v_heads: int) -> int:
    return lib().la_scan_chunked_conv_workspace_bytes(int(total_tokens), int(n_v_heads))


def la_state_scan_chunked_conv_ws(rule, src: Optional[Pool], read_slot, dst: Pool, write_slot, cu_seqlens,
                                  conv: Conv, xq, xk, xv, g, beta, scale, o, workspace, err_word, seq_order=None,
                                  stream=None) -> int:
    """la_state_scan_chunked_conv in two launches; workspace: a uint8 device tensor of at
    least la_scan_chunked_conv_workspace_bytes(...) bytes."""
    io = dtype_code(xq.dtype)
    return lib().la_state_scan_chunked_conv_ws(RULES[rule] if isinstance(rule, str) else int(rule),
                                               None if src is None else src.ref, _ptr(read_slot, torch.int32),
                                               dst.ref, _ptr(write_slot, torch.int32), int(cu_seqlens.numel() - 1),
                                               _ptr(cu_seqlens, torch.int32), int(xq.shape[0]),
                                               _ptr(seq_order, torch.int32), conv.ref, _ptr(xq), _ptr(xk, xq.dtype),
                                               _ptr(xv, xq.dtype), io, _ptr(g, torch.float32),
                                               _ptr(beta, torch.float32), float(scale), _ptr(o, xq.dtype),
                                               _ptr(workspace), int(workspace.numel() * workspace.element_size()),
                                               _ptr(err_word, torch.int32), _stream(stream))


def q8_tile_bytes(d_k: int, d_v: int, n_hp: int) -> int:
    """Bytes of one (slot, head) tile of a q8 pool (the layout of la_state.h)."""
    return (d_k - n_hp) * d_v + (d_k - n_hp) * (d_v // 32) * 4 + n_hp * d_v * 2


def la_pool_slot_bytes(pool: Pool) -> int:
    return lib().la_pool_slot_bytes(pool.ref)


def la_state_pool_encode(pool: Pool, slots, dense, err_word, stream=None) -> int:
    return lib().la_state_pool_encode(pool.ref, int(slots.numel()), _ptr(slots, torch.int32),
                                      _ptr(dense, torch.float32), _ptr(err_word, torch.int32), _stream(stream))


def la_state_pool_decode(pool: Pool, slots, dense, err_word, stream=None) -> int:
    return lib().la_state_pool_decode(pool.ref, int(slots.numel()), _ptr(slots, torch.int32),
                                      _ptr(dense, torch.float32), _ptr(err_word, torch.int32), _stream(stream))


def la_state_step_qgroups(rule, src: Pool, read_slot, dst: Pool, write_slot, q, k, v, g, beta, scale, o, err_word,
                          stream=None) -> int:
    """Query-group direction: k [B, H_v, d_k], q [B, n_q_heads, d_k], o [B, n_q_heads, d_v]."""
    io = dtype_code(q.dtype)
    return lib().la_state_step_qgroups(RULES[rule] if isinstance(rule, str) else int(rule), src.ref,
                                       _ptr(read_slot, torch.int32), dst.ref, _ptr(write_slot, torch.int32),
                                       int(q.shape[0]), int(q.shape[1]), _ptr(q), _ptr(k, q.dtype), _ptr(v, q.dtype),
                                       io, _ptr(g, torch.float32), _ptr(beta, torch.float32), float(scale),
                                       _ptr(o, q.dtype), _ptr(err_word, torch.int32), _stream(stream))


def la_state_scan_qgroups(rule, src: Optional[Pool], read_slot, dst: Pool, write_slot, cu_seqlens, q, k, v, g, beta,
                          scale, o, err_word, seq_order=None, stream=None) -> int:
    """Query-group direction of la_state_scan: k [T, H_v, d_k], q [T, n_q_heads, d_k]."""
    io = dtype_code(q.dtype)
    return lib().la_state_scan_qgroups(RULES[rule] if isinstance(rule, str) else int(rule),
                                       None if src is None else src.ref, _ptr(read_slot, torch.int32), dst.ref,
                                       _ptr(write_slot, torch.int32), int(cu_seqlens.numel() - 1),
                                       _ptr(cu_seqlens, torch.int32), int(q.shape[0]), _ptr(seq_order, torch.int32),
                                       int(q.shape[1]), _ptr(q), _ptr(k, q.dtype), _ptr(v, q.dtype), io,
                                       _ptr(g, torch.float32), _ptr(beta, torch.float32), float(scale),
                                       _ptr(o, q.dtype), _ptr(err_word, torch.int32), _stream(stream))


def la_state_scan_chunked_qgroups(rule, src: Optional[Pool], read_slot, dst: Pool, write_slot, cu_seqlens, q, k, v, g,
                                  beta, scale, o, err_word, seq_order=None, stream=None) -> int:
    """Query-group direction of la_state_scan_chunked: k [T, H_v, 128], q [T, n_q_heads, 128]."""
    io = dtype_code(q.dtype)
    return lib().la_state_scan_chunked_qgroups(RULES[rule] if isinstance(rule, str) else int(rule),
                                               None if src is None else src.ref, _ptr(read_slot, torch.int32),
                                               dst.ref, _ptr(write_slot, torch.int32), int(cu_seqlens.numel() - 1),
                                               _ptr(cu_seqlens, torch.int32), int(q.shape[0]),
                                               _ptr(seq_order, torch.int32), int(q.shape[1]), _ptr(q),
                                               _ptr(k, q.dtype), _ptr(v, q.dtype), io, _ptr(g, torch.float32),
                                               _ptr(beta, torch.float32), float(scale), _ptr(o, q.dtype),
                                               _ptr(err_word, torch.int32), _stream(stream))


def la_state_pool_copy(pool: Pool, src_slots, dst_slots, err_word, stream=None) -> int:
    return lib().la_state_pool_copy(pool.ref, int(src_slots.numel()), _ptr(src_slots, torch.int32),
                                    _ptr(dst_slots, torch.int32), _ptr(err_word, torch.int32), _stream(stream))


def la_state_pool_gather(pool: Pool, slots, dense, err_word, stream=None) -> int:
    return lib().la_state_pool_gather(pool.ref, int(slots.numel()), _ptr(slots, torch.int32),
                                      _ptr(dense, pool.tensor.dtype), _ptr(err_word, torch.int32), _stream(stream))


def la_state_pool_scatter(pool: Pool, slots, dense, err_word, stream=None) -> int:
    return lib().la_state_pool_scatter(pool.ref, int(slots.numel()), _ptr(slots, torch.int32),
                                       _ptr(dense, pool.tensor.dtype), _ptr(err_word, torch.int32), _stream(stream))


def la_state_pool_zero(pool: Pool, slots, err_word, stream=None) -> int:
    return lib().la_state_pool_zero(pool.ref, int(slots.numel()), _ptr(slots, torch.int32),
                                    _ptr(err_word, torch.int32), _stream(stream))


def la_state_check_slots(read_slot_host, write_slot_host, n_slots: int, B: Optional[int] = None) -> int:
    """Host-side slot precondition check on CPU int32 tensors (or None = identity)."""
    def hp(t):
        if t is None:
            return None
        t = t.to(torch.int32).contiguous().cpu()
        hp.keep.append(t)
        return ctypes.c_void_p(t.data_ptr())
    hp.keep = []
    if B is None:
        B = int((read_slot_host if read_slot_host is not None else write_slot_host).numel())
    return lib().la_state_check_slots(int(B), hp(read_slot_host), hp(write_slot_host), int(n_slots))


def la_abi_version() -> int:
    return lib().la_abi_version()


def la_debug_set_wait_limit_us(us: int) -> None:
    """Test hook: the decode step's pipeline wait limit on this thread (0: the default 1 s)."""
    lib().la_debug_set_wait_limit_us(int(us))


def la_debug_withhold_step_tile(tile: int) -> None:
    """Test hook: the next decode step on this thread withholds one tile's arrival, so its
    waits run out and LA_DEVERR_TIMEOUT is reported (nothing is left in flight)."""
    lib().la_debug_withhold_step_tile(int(tile))
