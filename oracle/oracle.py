"""ctypes binding of the CPU oracle.  TEST INFRASTRUCTURE ONLY.

Only tests/, the smoke check and the benchmark's CPU-baseline leg may import this.
Arrays are numpy float64 (values already rounded to their storage / io type by the
caller, which is exact in float64) and int32 slot / cu_seqlens arrays.  What each
function computes, and which passage of the pages it follows, is in la_oracle.c.
"""
import ctypes
import os

import numpy as np

from . import build as _build

RULES = {"linear": 0, "gated": 1, "delta": 2, "gated_delta": 3, "kda": 4}
DTYPES = {"f64": 0, "f32": 1, "bf16": 2}

_lib = None


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        _lib = ctypes.CDLL(path)
        d, i, p = ctypes.c_double, ctypes.c_int, ctypes.c_void_p
        sz = ctypes.c_size_t
        _lib.lao_round_bf16.argtypes = [d]
        _lib.lao_round_bf16.restype = d
        _lib.lao_round_to.argtypes = [d, i]
        _lib.lao_round_to.restype = d
        _lib.lao_step.argtypes = [i, i, i, i, i, p, i, p, i, i, p, p, i, p, p, p, i, p, p, d, p]
        _lib.lao_step.restype = i
        _lib.lao_readout_rearranged.argtypes = [i, i, i, i, i, p, i, p, p, p, p, p, d, p]
        _lib.lao_readout_rearranged.restype = None
        _lib.lao_scan.argtypes = [i, i, i, i, i, p, i, p, p, i, i, p, i, p, i, p, p, p, i, p, p, d, p]
        _lib.lao_scan.restype = i
        _lib.lao_scan_ckpt.argtypes = _lib.lao_scan.argtypes + [i, p, p]
        _lib.lao_scan_ckpt.restype = i
        _lib.lao_q8_tile_bytes.argtypes = [i, i, i]
        _lib.lao_q8_tile_bytes.restype = sz
        _lib.lao_q8_encode.argtypes = [p, i, i, i, i, i, p, p]
        _lib.lao_q8_encode.restype = i
        _lib.lao_q8_decode.argtypes = [p, i, i, i, i, i, p, p]
        _lib.lao_q8_decode.restype = i
        _lib.lao_step_q8.argtypes = [i, i, i, i, i, p, i, p, i, p, p, i, p, p, p, i, p, p, d, p, p]
        _lib.lao_step_q8.restype = i
        _lib.lao_scan_q8.argtypes = [i, i, i, i, i, p, i, p, p, i, p, i, p, i, p, p, p, i, p, p, d, p, i, p, p, p]
        _lib.lao_scan_q8.restype = i
        _lib.lao_conv.argtypes = [i, i, i, i, i, i, i, i, p, p, p, p, p, p, p, p, p, p, p]
        _lib.lao_conv.restype = None
        _lib.lao_step_conv.argtypes = [i, i, i, i, i, p, i, p, i, i, p, p, i, p, p, p, i, p, p, d, p,
                                       i, i, i, p, p, p, p, p]
        _lib.lao_step_conv.restype = i
        _lib.lao_scan_conv.argtypes = _lib.lao_scan.argtypes + [i, i, i, p, p, p, p, p]
        _lib.lao_scan_conv.restype = i
        _lib.lao_step_qgroups.argtypes = _lib.lao_step.argtypes
        _lib.lao_step_qgroups.restype = i
        _lib.lao_scan_qgroups.argtypes = _lib.lao_scan.argtypes
        _lib.lao_scan_qgroups.restype = i
        _lib.lao_pool_copy.argtypes = [p, sz, i, i, p, p]
        _lib.lao_pool_gather.argtypes = [p, sz, i, i, p, p]
        _lib.lao_pool_scatter.argtypes = [p, sz, i, i, p, p]
        _lib.lao_pool_zero.argtypes = [p, sz, i, i, p]
        for f in (_lib.lao_pool_copy, _lib.lao_pool_gather, _lib.lao_pool_scatter, _lib.lao_pool_zero):
            f.restype = i
        _lib.lao_num_threads.restype = i
        _lib.lao_set_threads.argtypes = [i]
    return _lib


def use_library(path):
    """Load the oracle from another shared object (used by the tests that plant a
    mistake in a copy of the oracle and check the pins catch it).  Returns the previous
    handle; pass it to restore_library() to switch back."""
    global _lib
    prev = lib()
    _lib = None
    saved = _build.LIB
    _build.LIB = path
    try:
        _build.build = (lambda force=False, _p=path: _p)  # type: ignore[assignment]
        lib()
    finally:
        _build.LIB = saved
        _build.build = _BUILD
    return prev


def restore_library(handle):
    global _lib
    _lib = handle


_BUILD = _build.build


def _f64(a):
    return np.ascontiguousarray(a, dtype=np.float64)


def _i32(a):
    return None if a is None else np.ascontiguousarray(a, dtype=np.int32)


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def round_bf16(x):
    """Round each element of a float64 array to the nearest bfloat16 (ties to even)."""
    f = lib().lao_round_bf16
    x = _f64(x)
    return np.array([f(float(e)) for e in x.ravel()], dtype=np.float64).reshape(x.shape)


def round_to(x, dtype):
    f = lib().lao_round_to
    x = _f64(x)
    code = DTYPES[dtype]
    return np.array([f(float(e), code) for e in x.ravel()], dtype=np.float64).reshape(x.shape)


def step(rule, n_qk_heads, src_pool, q, k, v, g=None, beta=None, scale=1.0, *,
         dst_pool=None, dst_dtype="f64", io_dtype="f64", read_slot=None, write_slot=None):
    """One decode step.  src_pool [n_src, H_v, d_k, d_v]; dst_pool (updated in place and
    returned; defaults to a copy of src_pool).  Returns (dst_pool, o, err_bits)."""
    src = _f64(src_pool)
    dst = src.copy() if dst_pool is None else dst_pool
    assert dst.dtype == np.float64 and dst.flags.c_contiguous
    n_src, hv, dk, dv = src.shape
    q, k, v = _f64(q), _f64(k), _f64(v)
    B = q.shape[0]
    g = None if g is None else _f64(g)
    beta = None if beta is None else _f64(beta)
    rs, ws = _i32(read_slot), _i32(write_slot)
    o = np.zeros((B, hv, dv), dtype=np.float64)
    err = lib().lao_step(RULES[rule], n_qk_heads, hv, dk, dv, _ptr(src), n_src,
                         _ptr(dst), dst.shape[0], DTYPES[dst_dtype], _ptr(rs), _ptr(ws), B,
                         _ptr(q), _ptr(k), _ptr(v), DTYPES[io_dtype], _ptr(g), _ptr(beta),
                         float(scale), _ptr(o))
    return dst, o, err


def step_qgroups(rule, n_q_heads, src_pool, q, k, v, g=None, beta=None, scale=1.0, *,
                 dst_pool=None, dst_dtype="f64", io_dtype="f64", read_slot=None, write_slot=None):
    """One decode step in the query-group direction of the ONNX operator: k [B, H_v, d_k]
    (one key per state head), q [B, n_q_heads, d_k], o [B, n_q_heads, d_v]; query head i
    reads state head i / (n_q_heads / H_v).  Returns (dst_pool, o, err_bits)."""
    src = _f64(src_pool)
    dst = src.copy() if dst_pool is None else dst_pool
    assert dst.dtype == np.float64 and dst.flags.c_contiguous
    n_src, hv, dk, dv = src.shape
    q, k, v = _f64(q), _f64(k), _f64(v)
    B = q.shape[0]
    g = None if g is None else _f64(g)
    beta = None if beta is None else _f64(beta)
    rs, ws = _i32(read_slot), _i32(write_slot)
    o = np.zeros((B, n_q_heads, dv), dtype=np.float64)
    err = lib().lao_step_qgroups(RULES[rule], n_q_heads, hv, dk, dv, _ptr(src), n_src,
                                 _ptr(dst), dst.shape[0], DTYPES[dst_dtype], _ptr(rs), _ptr(ws), B,
                                 _ptr(q), _ptr(k), _ptr(v), DTYPES[io_dtype], _ptr(g), _ptr(beta),
                                 float(scale), _ptr(o))
    return dst, o, err


def scan_qgroups(rule, n_q_heads, cu_seqlens, q, k, v, g=None, beta=None, scale=1.0, *,
                 src_pool=None, read_slot=None, dst_pool=None, dst_dtype="f64", write_slot=None,
                 io_dtype="f64"):
    """Token-serial scan in the query-group direction (layouts as step_qgroups with T
    rows).  Returns (dst_pool, o, err_bits)."""
    cu = _i32(cu_seqlens)
    n_seqs = cu.shape[0] - 1
    q, k, v = _f64(q), _f64(k), _f64(v)
    T, hv, dk = k.shape
    dv = v.shape[2]
    if dst_pool is None:
        dst_pool = np.zeros((n_seqs, hv, dk, dv), dtype=np.float64)
    assert dst_pool.dtype == np.float64 and dst_pool.flags.c_contiguous
    src = None if src_pool is None else _f64(src_pool)
    n_src = 0 if src is None else src.shape[0]
    g = None if g is None else _f64(g)
    beta = None if beta is None else _f64(beta)
    o = np.zeros((T, n_q_heads, dv), dtype=np.float64)
    err = lib().lao_scan_qgroups(RULES[rule], n_q_heads, hv, dk, dv, _ptr(src), n_src, _ptr(_i32(read_slot)),
                                 _ptr(dst_pool), dst_pool.shape[0], DTYPES[dst_dtype], _ptr(_i32(write_slot)),
                                 n_seqs, _ptr(cu), T, _ptr(q), _ptr(k), _ptr(v), DTYPES[io_dtype],
                                 _ptr(g), _ptr(beta), float(scale), _ptr(o))
    return dst_pool, o, err


def q8_tile_bytes(dk, dv, n_hp):
    """Bytes of one (slot, head) tile in the mixed INT8 / BF16 ("q8") format."""
    return int(lib().lao_q8_tile_bytes(dk, dv, n_hp))


def _u32(masks):
    return np.ascontiguousarray(masks, dtype=np.uint32)


def q8_encode(x, n_hp, masks):
    """x float32 [n, H, d_k, d_v] -> uint8 [n, H, tile bytes]; masks uint32 [H, d_k / 32]
    (bit i of a head's mask: key channel i is kept in BF16)."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    n, H, dk, dv = x.shape
    out = np.zeros((n, H, q8_tile_bytes(dk, dv, n_hp)), dtype=np.uint8)
    m = _u32(masks)
    assert lib().lao_q8_encode(_ptr(x), n, H, dk, dv, n_hp, _ptr(m), _ptr(out)) == 0, "mask rows != n_hp"
    return out


def q8_decode(b, dk, dv, n_hp, masks):
    """uint8 [n, H, tile bytes] -> float32 [n, H, d_k, d_v]."""
    b = np.ascontiguousarray(b, dtype=np.uint8)
    n, H, _ = b.shape
    x = np.zeros((n, H, dk, dv), dtype=np.float32)
    m = _u32(masks)
    assert lib().lao_q8_decode(_ptr(b), n, H, dk, dv, n_hp, _ptr(m), _ptr(x)) == 0, "mask rows != n_hp"
    return x


def step_q8(rule, n_qk_heads, src_pool, q, k, v, g=None, beta=None, scale=1.0, *, masks,
            dst_pool=None, io_dtype="f64", read_slot=None, write_slot=None):
    """Decode step whose new states are stored in the q8 format (returned as decoded values)."""
    src = _f64(src_pool)
    dst = src.copy() if dst_pool is None else dst_pool
    n_src, hv, dk, dv = src.shape
    q, k, v = _f64(q), _f64(k), _f64(v)
    B = q.shape[0]
    g = None if g is None else _f64(g)
    beta = None if beta is None else _f64(beta)
    o = np.zeros((B, hv, dv), dtype=np.float64)
    m = _u32(masks)
    err = lib().lao_step_q8(RULES[rule], n_qk_heads, hv, dk, dv, _ptr(src), n_src, _ptr(dst), dst.shape[0],
                            _ptr(_i32(read_slot)), _ptr(_i32(write_slot)), B, _ptr(q), _ptr(k), _ptr(v),
                            DTYPES[io_dtype], _ptr(g), _ptr(beta), float(scale), _ptr(o), _ptr(m))
    return dst, o, err


def scan_q8(rule, n_qk_heads, cu_seqlens, q, k, v, g=None, beta=None, scale=1.0, *, masks,
            src_pool=None, read_slot=None, dst_pool=None, write_slot=None, io_dtype="f64", ckpt_every=0,
            ckpt_cu=None, ckpt_slots=None):
    """Scan whose final states (and checkpoints) are stored in the q8 format."""
    cu = _i32(cu_seqlens)
    n_seqs = cu.shape[0] - 1
    q, k, v = _f64(q), _f64(k), _f64(v)
    T, _, dk = q.shape
    hv, dv = v.shape[1], v.shape[2]
    if dst_pool is None:
        dst_pool = np.zeros((n_seqs, hv, dk, dv), dtype=np.float64)
    src = None if src_pool is None else _f64(src_pool)
    n_src = 0 if src is None else src.shape[0]
    g = None if g is None else _f64(g)
    beta = None if beta is None else _f64(beta)
    o = np.zeros((T, hv, dv), dtype=np.float64)
    m = _u32(masks)
    err = lib().lao_scan_q8(RULES[rule], n_qk_heads, hv, dk, dv, _ptr(src), n_src, _ptr(_i32(read_slot)),
                            _ptr(dst_pool), dst_pool.shape[0], _ptr(_i32(write_slot)), n_seqs, _ptr(cu), T,
                            _ptr(q), _ptr(k), _ptr(v), DTYPES[io_dtype], _ptr(g), _ptr(beta), float(scale), _ptr(o),
                            int(ckpt_every), _ptr(_i32(ckpt_cu)), _ptr(_i32(ckpt_slots)), _ptr(m))
    return dst_pool, o, err


def conv(n_qk_heads, xq, xk, xv, wq, wk, wv, hist, *, act=0, l2norm=0):
    """The short causal convolution alone (see la_oracle.c): xq, xk [B, H_qk, d_k], xv
    [B, H_v, d_v], weights [heads, channels, W], hist [B, H_v, 2 d_k + d_v, W - 1].
    Returns (q, k [B, H_v, d_k], v [B, H_v, d_v], new hist)."""
    xq, xk, xv, wq, wk, wv, hist = (_f64(a) for a in (xq, xk, xv, wq, wk, wv, hist))
    B, hv, dv = xv.shape
    dk = xq.shape[2]
    W = wq.shape[2]
    q = np.zeros((B, hv, dk)); k = np.zeros((B, hv, dk)); v = np.zeros((B, hv, dv))
    out = np.zeros_like(hist)
    lib().lao_conv(n_qk_heads, hv, dk, dv, W, int(act), int(l2norm), B, _ptr(xq), _ptr(xk), _ptr(xv), _ptr(wq),
                   _ptr(wk), _ptr(wv), _ptr(hist), _ptr(out), _ptr(q), _ptr(k), _ptr(v))
    return q, k, v, out


def step_conv(rule, n_qk_heads, src_pool, xq, xk, xv, g, beta, scale, wq, wk, wv, conv_src, *, act=0, l2norm=0,
              dst_pool=None, conv_dst=None, dst_dtype="f64", io_dtype="f64", read_slot=None, write_slot=None):
    """Decode step with the convolution fused ahead of it.  Returns (dst_pool, conv_dst, o, err)."""
    src = _f64(src_pool)
    dst = src.copy() if dst_pool is None else dst_pool
    csrc = _f64(conv_src)
    cdst = csrc.copy() if conv_dst is None else conv_dst
    n_src, hv, dk, dv = src.shape
    xq, xk, xv, wq, wk, wv = (_f64(a) for a in (xq, xk, xv, wq, wk, wv))
    B = xq.shape[0]
    g = None if g is None else _f64(g)
    beta = None if beta is None else _f64(beta)
    o = np.zeros((B, hv, dv))
    err = lib().lao_step_conv(RULES[rule], n_qk_heads, hv, dk, dv, _ptr(src), n_src, _ptr(dst), dst.shape[0],
                              DTYPES[dst_dtype], _ptr(_i32(read_slot)), _ptr(_i32(write_slot)), B, _ptr(xq), _ptr(xk),
                              _ptr(xv), DTYPES[io_dtype], _ptr(g), _ptr(beta), float(scale), _ptr(o), wq.shape[2],
                              int(act), int(l2norm), _ptr(wq), _ptr(wk), _ptr(wv), _ptr(csrc), _ptr(cdst))
    return dst, cdst, o, err


def scan_conv(rule, n_qk_heads, cu_seqlens, xq, xk, xv, g, beta, scale, wq, wk, wv, *, act=0, l2norm=0,
              conv_src=None, src_pool=None, read_slot=None, dst_pool=None, conv_dst=None, write_slot=None,
              dst_dtype="f64", io_dtype="f64"):
    """Token-serial scan with the convolution ahead of every token (see la_oracle.c).
    conv_src: histories [slots, H_v, 2 d_k + d_v, W - 1] read at read_slot (zeros when
    read_slot is None).  Returns (dst_pool, conv_dst, o, err_bits)."""
    cu = _i32(cu_seqlens)
    n_seqs = cu.shape[0] - 1
    xq, xk, xv, wq, wk, wv = (_f64(a) for a in (xq, xk, xv, wq, wk, wv))
    T, _, dk = xq.shape
    hv, dv = xv.shape[1], xv.shape[2]
    W = wq.shape[2]
    if dst_pool is None:
        dst_pool = np.zeros((n_seqs, hv, dk, dv))
    if conv_dst is None:
        conv_dst = np.zeros((dst_pool.shape[0], hv, 2 * dk + dv, W - 1))
    src = None if src_pool is None else _f64(src_pool)
    csrc = np.zeros((1, hv, 2 * dk + dv, W - 1)) if conv_src is None else _f64(conv_src)
    n_src = 0 if src is None else src.shape[0]
    g = None if g is None else _f64(g)
    beta = None if beta is None else _f64(beta)
    o = np.zeros((T, hv, dv))
    err = lib().lao_scan_conv(RULES[rule], n_qk_heads, hv, dk, dv, _ptr(src), n_src, _ptr(_i32(read_slot)),
                              _ptr(dst_pool), dst_pool.shape[0], DTYPES[dst_dtype], _ptr(_i32(write_slot)), n_seqs,
                              _ptr(cu), T, _ptr(xq), _ptr(xk), _ptr(xv), DTYPES[io_dtype], _ptr(g), _ptr(beta),
                              float(scale), _ptr(o), W, int(act), int(l2norm), _ptr(wq), _ptr(wk), _ptr(wv),
                              _ptr(csrc), _ptr(conv_dst))
    return dst_pool, conv_dst, o, err


def readout_rearranged(rule, n_qk_heads, state, q, k, v, g=None, beta=None, scale=1.0):
    """o of one decode step in the rearranged form; state [B, H_v, d_k, d_v] (dense)."""
    S = _f64(state)
    B, hv, dk, dv = S.shape
    q, k, v = _f64(q), _f64(k), _f64(v)
    g = None if g is None else _f64(g)
    beta = None if beta is None else _f64(beta)
    o = np.zeros((B, hv, dv), dtype=np.float64)
    lib().lao_readout_rearranged(RULES[rule], n_qk_heads, hv, dk, dv, _ptr(S), B,
                                 _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), float(scale), _ptr(o))
    return o


def scan(rule, n_qk_heads, cu_seqlens, q, k, v, g=None, beta=None, scale=1.0, *,
         src_pool=None, read_slot=None, dst_pool=None, dst_dtype="f64", write_slot=None,
         io_dtype="f64", n_v_heads=None, d_v=None, ckpt_every=0, ckpt_cu=None, ckpt_slots=None):
    """Token-serial scan over packed sequences.  Initial state from src_pool[read_slot]
    (zero when read_slot is None).  With ckpt_every > 0, the state after every ckpt_every
    tokens of sequence s goes to dst_pool[ckpt_slots[ckpt_cu[s] + j]] (see la_oracle.c).
    Returns (dst_pool, o, err_bits)."""
    cu = _i32(cu_seqlens)
    n_seqs = cu.shape[0] - 1
    q, k, v = _f64(q), _f64(k), _f64(v)
    T, _, dk = q.shape
    hv, dv = v.shape[1], v.shape[2]
    if dst_pool is None:
        dst_pool = np.zeros((n_seqs, hv, dk, dv), dtype=np.float64)
    assert dst_pool.dtype == np.float64 and dst_pool.flags.c_contiguous
    src = None if src_pool is None else _f64(src_pool)
    n_src = 0 if src is None else src.shape[0]
    g = None if g is None else _f64(g)
    beta = None if beta is None else _f64(beta)
    o = np.zeros((T, hv, dv), dtype=np.float64)
    args = (RULES[rule], n_qk_heads, hv, dk, dv, _ptr(src), n_src, _ptr(_i32(read_slot)),
            _ptr(dst_pool), dst_pool.shape[0], DTYPES[dst_dtype], _ptr(_i32(write_slot)),
            n_seqs, _ptr(cu), T, _ptr(q), _ptr(k), _ptr(v), DTYPES[io_dtype],
            _ptr(g), _ptr(beta), float(scale), _ptr(o))
    if ckpt_every > 0:
        ccu, csl = _i32(ckpt_cu), _i32(ckpt_slots)
        err = lib().lao_scan_ckpt(*args, int(ckpt_every), _ptr(ccu), _ptr(csl))
    else:
        err = lib().lao_scan(*args)
    return dst_pool, o, err


def _u8(pool):
    assert pool.flags.c_contiguous
    return pool.view(np.uint8).reshape(pool.shape[0], -1)


def pool_copy(pool, src_slots, dst_slots):
    """Bit copy of whole slots, pool is any contiguous numpy array [n_slots, ...]."""
    b = _u8(pool)
    s, d = _i32(src_slots), _i32(dst_slots)
    return lib().lao_pool_copy(_ptr(b), b.shape[1], b.shape[0], s.shape[0], _ptr(s), _ptr(d))


def pool_gather(pool, slots):
    b = _u8(pool)
    s = _i32(slots)
    dense = np.zeros((s.shape[0],) + pool.shape[1:], dtype=pool.dtype)
    err = lib().lao_pool_gather(_ptr(b), b.shape[1], b.shape[0], s.shape[0], _ptr(s), _ptr(_u8(dense)))
    return dense, err


def pool_scatter(pool, slots, dense):
    b = _u8(pool)
    s = _i32(slots)
    dense = np.ascontiguousarray(dense, dtype=pool.dtype)
    return lib().lao_pool_scatter(_ptr(b), b.shape[1], b.shape[0], s.shape[0], _ptr(s), _ptr(_u8(dense)))


def pool_zero(pool, slots):
    b = _u8(pool)
    s = _i32(slots)
    return lib().lao_pool_zero(_ptr(b), b.shape[1], b.shape[0], s.shape[0], _ptr(s))


def num_threads():
    return lib().lao_num_threads()


def set_threads(n):
    lib().lao_set_threads(int(n))


__all__ = ["round_bf16", "round_to", "step", "readout_rearranged", "scan", "pool_copy",
           "pool_gather", "pool_scatter", "pool_zero", "num_threads", "set_threads", "RULES", "DTYPES",
           "step_qgroups", "scan_qgroups", "q8_tile_bytes", "q8_encode", "q8_decode", "step_q8", "scan_q8", "conv",
           "step_conv", "scan_conv"]

if os.environ.get("LAO_THREADS"):
    set_threads(int(os.environ["LAO_THREADS"]))
