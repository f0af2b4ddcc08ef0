"""CPU oracle for the group-wise 4-bit decode path (ctypes binding of ``fg_oracle.c``).

TEST INFRASTRUCTURE.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package.  It shares no code
with the CUDA library and never imports it.

Every function cites the passage it follows in ``fg_oracle.c``; see that
file's header for the readings taken where the pages are silent.

Arrays of fp16 values are passed as ``numpy.float16`` (or their ``uint16``
bit patterns); results of the float64 layer evaluation come back as
``numpy.float64``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import time

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "fg_oracle.c")
_LIB = os.path.join(_HERE, "liboracle_fg.so")
GROUP = 64


def build(force: bool = False) -> str:
    """Compiles the oracle with gcc (no fast-math, no FMA contraction)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math",
                               "-fPIC", "-shared", "-pthread", _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        P = ctypes.c_void_p
        I64, I, D = ctypes.c_int64, ctypes.c_int, ctypes.c_double
        _lib.oracle_f16_to_f64.restype = D
        _lib.oracle_f16_to_f64.argtypes = [ctypes.c_uint16]
        _lib.oracle_f64_to_f16.restype = ctypes.c_uint16
        _lib.oracle_f64_to_f16.argtypes = [D]
        _lib.oracle_f32_to_f16.restype = ctypes.c_uint16
        _lib.oracle_f32_to_f16.argtypes = [ctypes.c_float]
        _lib.oracle_f16_to_f64_array.argtypes = [P, P, I64]
        _lib.oracle_f64_to_f16_array.argtypes = [P, P, I64]
        _lib.oracle_quantize.restype = I
        _lib.oracle_quantize.argtypes = [P, I64, I64, I64, P, P, P]
        _lib.oracle_dequantize.restype = I
        _lib.oracle_dequantize.argtypes = [P, P, P, I64, I64, I64, P]
        _lib.oracle_linear.restype = I
        _lib.oracle_linear.argtypes = [P, I, I, P, P, P, I, P, P, I, I, D, P]
        _lib.oracle_quantize_g.restype = I
        _lib.oracle_quantize_g.argtypes = [P, I64, I64, I64, P, P, P, I]
        _lib.oracle_dequantize_g.restype = I
        _lib.oracle_dequantize_g.argtypes = [P, P, P, I64, I64, I64, P, I]
        _lib.oracle_quantize_gb.restype = I
        _lib.oracle_quantize_gb.argtypes = [P, I64, I64, I64, P, P, P, I, I]
        _lib.oracle_dequantize_gb.restype = I
        _lib.oracle_dequantize_gb.argtypes = [P, P, P, I64, I64, I64, P, I, I]
        _lib.oracle_linear_g.restype = I
        _lib.oracle_linear_g.argtypes = [P, I, I, P, P, P, I, P, P, I, I, D, P, I]
        _lib.oracle_layernorm.restype = I
        _lib.oracle_layernorm.argtypes = [P, I, I, P, P, D, P]
        _lib.oracle_kv_append_g.restype = I
        _lib.oracle_kv_append_g.argtypes = [P, P, I64, I, P, P, P, P, P, P, P, P, I, I, I, I, I]
        _lib.oracle_attention_x.restype = I
        _lib.oracle_attention_x.argtypes = [P, I64, I, P, P, P, P, P, P, P, P, I, I, I, I, P, I, I]
        _lib.oracle_w4a8_quantize_weight.restype = I
        _lib.oracle_w4a8_quantize_weight.argtypes = [P, I, I, P, P, P, P]
        _lib.oracle_w4a8_weight_int8.restype = I
        _lib.oracle_w4a8_weight_int8.argtypes = [P, P, P, I, I, P]
        _lib.oracle_act8_quantize.restype = I
        _lib.oracle_act8_quantize.argtypes = [P, I, I, P, P]
        _lib.oracle_linear_w4a8.restype = I
        _lib.oracle_linear_w4a8.argtypes = [P, P, I, I, P, P, P, P, I, P, P, I, I, D, P, P]
        _lib.oracle_layer_rows_w4a8.restype = I
        _lib.oracle_layer_rows_w4a8.argtypes = ([P, D, P] + [P] * 8 + [P] * 6 + [I, I] + [P, I, P, P, I, P, P, I])
        _lib.oracle_layer_rows.restype = I
        _lib.oracle_layer_rows.argtypes = ([P, D] + [P] * 16 + [P] * 4 + [P] * 6 + [I, I] + [P, I, P, P, I, P, P, I])
    return _lib


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _u16(a) -> np.ndarray:
    a = np.ascontiguousarray(a)
    if a.dtype == np.float16:
        return a.view(np.uint16)
    assert a.dtype == np.uint16, a.dtype
    return a


# --------------------------------------------------------------------------------------
# binary16 conversions (IEEE 754 format definition)
# --------------------------------------------------------------------------------------

def f16_to_f64(h) -> np.ndarray:
    h = _u16(h)
    out = np.empty(h.shape, dtype=np.float64)
    lib().oracle_f16_to_f64_array(_p(h), _p(out), h.size)
    return out


def f64_to_f16(x) -> np.ndarray:
    """Round to nearest binary16, ties to even; returns float16."""
    x = np.ascontiguousarray(x, dtype=np.float64)
    out = np.empty(x.shape, dtype=np.uint16)
    lib().oracle_f64_to_f16_array(_p(x), _p(out), x.size)
    return out.view(np.float16)


# --------------------------------------------------------------------------------------
# Group-wise 4-bit quantisation ("FlexGen Guide", section 3)
# --------------------------------------------------------------------------------------

class Packed:
    """Planar quantised tensor: codes uint8 (dim x bits / 8: two 4-bit codes or one 8-bit code
    per byte), mins/scales float16 (dim / group)."""

    def __init__(self, codes, mins, scales, shape, dim, group: int = GROUP, bits: int = 4):
        self.codes, self.mins, self.scales = codes, mins, scales
        self.shape, self.dim, self.group, self.bits = tuple(shape), dim, group, bits


def _split(shape, dim):
    dim = dim % len(shape)
    outer = int(np.prod(shape[:dim])) if dim else 1
    inner = int(np.prod(shape[dim + 1:])) if dim + 1 < len(shape) else 1
    return dim, outer, int(shape[dim]), inner


def quantize(x, dim: int = -1, group: int = GROUP, bits: int = 4) -> Packed:
    """Group-wise asymmetric min-max quantisation along ``dim``, groups of 64 or 128
    consecutive elements ("FlexGen Guide", section 3: 4 bits, groups of 64 or 128); bits = 8
    is the same scheme with 255 steps (INT8 among the post-training formats of the
    "Optimizing LLM for low memory usage" page)."""
    x = _u16(x)
    dim, outer, n, inner = _split(x.shape, dim)
    if group not in (64, 128):
        raise ValueError("group must be 64 or 128")
    if bits not in (4, 8):
        raise ValueError("bits must be 4 or 8")
    if n % group:
        raise ValueError(f"size along dim must be a multiple of {group}")
    cshape = list(x.shape); cshape[dim] = n * bits // 8
    mshape = list(x.shape); mshape[dim] = n // group
    codes = np.empty(cshape, dtype=np.uint8)
    mins = np.empty(mshape, dtype=np.uint16)
    scales = np.empty(mshape, dtype=np.uint16)
    rc = lib().oracle_quantize_gb(_p(x), outer, n, inner, _p(codes), _p(mins), _p(scales), group, bits)
    assert rc == 0
    return Packed(codes, mins.view(np.float16), scales.view(np.float16), x.shape, dim, group, bits)


def dequantize(q: Packed) -> np.ndarray:
    dim, outer, n, inner = _split(q.shape, q.dim)
    y = np.empty(q.shape, dtype=np.uint16)
    rc = lib().oracle_dequantize_gb(_p(np.ascontiguousarray(q.codes)), _p(_u16(q.mins)), _p(_u16(q.scales)),
                                    outer, n, inner, _p(y), q.group, getattr(q, "bits", 4))
    assert rc == 0
    return y.view(np.float16)


# --------------------------------------------------------------------------------------
# Layer pieces (float64)
# --------------------------------------------------------------------------------------

def linear(x, w: Packed, bias=None, residual=None, relu: bool = False,
           qscale_cols: int = 0, qscale: float = 1.0) -> np.ndarray:
    """``epi(x @ deq(w).T + bias)`` in float64; w is ``[N, K]`` packed along K."""
    x = _u16(x)
    M, K = x.shape
    N = w.shape[0]
    assert w.shape == (N, K) and w.dim == 1
    y = np.empty((M, N), dtype=np.float64)
    rc = lib().oracle_linear_g(_p(x), M, K, _p(np.ascontiguousarray(w.codes)), _p(_u16(w.mins)), _p(_u16(w.scales)),
                               N, _p(None if bias is None else _u16(bias)),
                               _p(None if residual is None else _u16(residual)),
                               int(relu), int(qscale_cols), float(qscale), _p(y), w.group)
    assert rc == 0
    return y


# --------------------------------------------------------------------------------------
# W4A8: two-level 4-bit weights and per-row 8-bit activations, integer products (the QServe
# W4A8KV4 entry of the PIPO paper's references, by title; "Optimizing LLM for low memory
# usage", Quantization and Weight Compression).  The scheme is a reading: fg_oracle.c states it.
# --------------------------------------------------------------------------------------

class W4A8Weight:
    """codes uint8 [N, K/2] (low nibble = even k), gmin int8 [N, K/64], gstep uint8 [N, K/64],
    cscale float32 [N]; the product's 8-bit weight is gmin + code * gstep, the real weight
    cscale * that."""

    def __init__(self, codes, gmin, gstep, cscale):
        self.codes, self.gmin, self.gstep, self.cscale = codes, gmin, gstep, cscale
        self.N, self.K = codes.shape[0], codes.shape[1] * 2


def w4a8_quantize_weight(w) -> W4A8Weight:
    w = _u16(w)
    N, K = w.shape
    if K % GROUP:
        raise ValueError("K must be a multiple of 64")
    codes = np.empty((N, K // 2), np.uint8)
    gmin = np.empty((N, K // GROUP), np.int8)
    gstep = np.empty((N, K // GROUP), np.uint8)
    cscale = np.empty(N, np.float32)
    assert lib().oracle_w4a8_quantize_weight(_p(w), N, K, _p(codes), _p(gmin), _p(gstep), _p(cscale)) == 0
    return W4A8Weight(codes, gmin, gstep, cscale)


def w4a8_weight_int8(q: W4A8Weight) -> np.ndarray:
    """The 8-bit weights [N, K] the integer product uses."""
    w8 = np.empty((q.N, q.K), np.int8)
    assert lib().oracle_w4a8_weight_int8(_p(np.ascontiguousarray(q.codes)), _p(np.ascontiguousarray(q.gmin)),
                                         _p(np.ascontiguousarray(q.gstep)), q.N, q.K, _p(w8)) == 0
    return w8


def act8_quantize(x):
    """Per-row symmetric 8-bit activations: (a8 int8 [M, K], ascale float32 [M])."""
    x = _u16(x)
    M, K = x.shape
    a8 = np.empty((M, K), np.int8)
    ascale = np.empty(M, np.float32)
    assert lib().oracle_act8_quantize(_p(x), M, K, _p(a8), _p(ascale)) == 0
    return a8, ascale


def linear_w4a8(a8, ascale, w: W4A8Weight, bias=None, residual=None, relu: bool = False,
                qscale_cols: int = 0, qscale: float = 1.0, with_acc: bool = False):
    """``epi(acc * ascale[t] * cscale[n] + bias)`` in float64 with the exact integer sums
    ``acc = a8 @ w8.T``; with ``with_acc`` also returns acc (int64)."""
    a8 = np.ascontiguousarray(a8, dtype=np.int8)
    ascale = np.ascontiguousarray(ascale, dtype=np.float32)
    M, K = a8.shape
    assert K == w.K
    y = np.empty((M, w.N), np.float64)
    acc = np.empty((M, w.N), np.int64) if with_acc else None
    rc = lib().oracle_linear_w4a8(_p(a8), _p(ascale), M, K, _p(np.ascontiguousarray(w.codes)),
                                  _p(np.ascontiguousarray(w.gmin)), _p(np.ascontiguousarray(w.gstep)),
                                  _p(np.ascontiguousarray(w.cscale)), w.N,
                                  _p(None if bias is None else _u16(bias)),
                                  _p(None if residual is None else _u16(residual)),
                                  int(relu), int(qscale_cols), float(qscale), _p(y), _p(acc))
    assert rc == 0
    return (y, acc) if with_acc else y


def layernorm(x, gamma=None, beta=None, eps: float = 1e-5) -> np.ndarray:
    x = _u16(x)
    M, h = x.shape
    y = np.empty((M, h), dtype=np.float64)
    lib().oracle_layernorm(_p(x), M, h, _p(None if gamma is None else _u16(gamma)),
                           _p(None if beta is None else _u16(beta)), float(eps), _p(y))
    return y


class KVCache:
    """4-bit KV cache of one layer: codes [S,H,maxL,d/2], mins/scales [S,H,maxL,d/group], head_dim
    quantised in groups of 64 or 128 ("FlexGen Guide", section 3)."""

    def __init__(self, S: int, H: int, d: int, maxL: int, group: int = GROUP):
        if group not in (64, 128) or d % group:
            raise ValueError("group must be 64 or 128 and divide head_dim")
        self.S, self.H, self.d, self.maxL, self.group = S, H, d, maxL, group
        ng = d // group
        self.kc = np.zeros((S, H, maxL, d // 2), dtype=np.uint8)
        self.vc = np.zeros((S, H, maxL, d // 2), dtype=np.uint8)
        self.km = np.zeros((S, H, maxL, ng), dtype=np.uint16)
        self.ks = np.zeros((S, H, maxL, ng), dtype=np.uint16)
        self.vm = np.zeros((S, H, maxL, ng), dtype=np.uint16)
        self.vs = np.zeros((S, H, maxL, ng), dtype=np.uint16)

    def arrays(self):
        return [self.kc, self.km, self.ks, self.vc, self.vm, self.vs]

    def ptrs(self):
        return [_p(a) for a in self.arrays()]


def kv_append(cache: KVCache, k, v, seq_of_row, pos_of_row, ld: int | None = None) -> None:
    """Quantises fp16 k, v rows ``[R, H*d]`` into the cache (groups of cache.group along head_dim)."""
    k = _u16(k); v = _u16(v)
    R = k.shape[0]
    ld = k.shape[1] if ld is None else ld
    sr = np.ascontiguousarray(seq_of_row, dtype=np.int32)
    pr = np.ascontiguousarray(pos_of_row, dtype=np.int32)
    rc = lib().oracle_kv_append_g(_p(k), _p(v), ld, R, _p(sr), _p(pr), *cache.ptrs(),
                                  cache.S, cache.H, cache.d, cache.maxL, cache.group)
    assert rc == 0, rc


def attention(cache: KVCache, q, seq_of_row, len_of_row, exact_dequant: bool = False) -> np.ndarray:
    """Softmax attention of fp16 query rows ``[R, H*d]`` (already scaled) over the cache.

    K and V are the dequantised fp16 values (``exact_dequant=False``, the layer's reading), or
    ``min + code * scale`` before that rounding (``exact_dequant=True``)."""
    q = _u16(q)
    R = q.shape[0]
    out = np.empty((R, cache.H * cache.d), dtype=np.float64)
    sr = np.ascontiguousarray(seq_of_row, dtype=np.int32)
    lr = np.ascontiguousarray(len_of_row, dtype=np.int32)
    rc = lib().oracle_attention_x(_p(q), q.shape[1], R, _p(sr), _p(lr), *cache.ptrs(),
                                  cache.S, cache.H, cache.d, cache.maxL, _p(out), cache.group, int(exact_dequant))
    assert rc == 0, rc
    return out


class LayerWeights:
    """One OPT layer's weights, quantised by the oracle along the input dim in groups of 64 or 128."""

    def __init__(self, w16: dict, group: int = GROUP):
        self.group = group
        self.wqkv = quantize(w16["wqkv"], 1, group)
        self.wo = quantize(w16["wo"], 1, group)
        self.w1 = quantize(w16["w1"], 1, group)
        self.w2 = quantize(w16["w2"], 1, group)
        self.b = {k: _u16(w16[k]) for k in ("bqkv", "bo", "b1", "b2", "ln1_g", "ln1_b", "ln2_g", "ln2_b")}
        self.hidden = self.wqkv.shape[1]
        self.ffn = self.w1.shape[0]


def layer_rows(weights: LayerWeights, heads: int, cache: KVCache, x, seq_of_row, pos_of_row,
               kv_only: bool = False, eps: float = 1e-5, nthreads: int = 1, want_attn: bool = False):
    """Runs the OPT layer on hidden-state rows ``x [R, h]`` in order.

    Row r belongs to sequence ``seq_of_row[r]`` and is the token at cache
    position ``pos_of_row[r]``: its k, v are appended there, then it attends
    over positions ``0..pos``.  The weights' group size is the cache's.
    Returns ``(out [R,h] float64, attn [R,h] or None)``.
    """
    x = _u16(x)
    R, h = x.shape
    d = h // heads
    if cache.group != weights.group:
        raise ValueError("the layer's weights and KV cache use one group size")
    dims = np.array([h, heads, d, weights.ffn, weights.group], dtype=np.int32)
    out = np.zeros((R, h), dtype=np.float64)
    attn = np.zeros((R, h), dtype=np.float64) if want_attn else None
    sr = np.ascontiguousarray(seq_of_row, dtype=np.int32)
    pr = np.ascontiguousarray(pos_of_row, dtype=np.int32)
    w = weights
    args = [_p(dims), float(eps)]
    for t, b in ((w.wqkv, "bqkv"), (w.wo, "bo"), (w.w1, "b1"), (w.w2, "b2")):
        args += [_p(np.ascontiguousarray(t.codes)), _p(_u16(t.mins)), _p(_u16(t.scales)), _p(w.b[b])]
    args += [_p(w.b["ln1_g"]), _p(w.b["ln1_b"]), _p(w.b["ln2_g"]), _p(w.b["ln2_b"])]
    args += cache.ptrs() + [cache.S, cache.maxL]
    args += [_p(x), R, _p(sr), _p(pr), int(kv_only), _p(out), _p(attn), int(nthreads)]
    rc = lib().oracle_layer_rows(*args)
    assert rc == 0, rc
    return out, attn


class W4A8LayerWeights:
    """One OPT layer's weights in the W4A8 form (w4a8_quantize_weight of each matrix); the KV
    cache stays 4-bit in groups of 64."""

    def __init__(self, w16: dict):
        self.group = GROUP
        self.wqkv = w4a8_quantize_weight(w16["wqkv"])
        self.wo = w4a8_quantize_weight(w16["wo"])
        self.w1 = w4a8_quantize_weight(w16["w1"])
        self.w2 = w4a8_quantize_weight(w16["w2"])
        self.b = {k: _u16(w16[k]) for k in ("bqkv", "bo", "b1", "b2", "ln1_g", "ln1_b", "ln2_g", "ln2_b")}
        self.hidden = self.wqkv.K
        self.ffn = self.w1.N


def layer_rows_w4a8(weights: W4A8LayerWeights, heads: int, cache: KVCache, x, seq_of_row, pos_of_row,
                    kv_only: bool = False, eps: float = 1e-5, nthreads: int = 1, want_attn: bool = False):
    """``layer_rows`` with the four products in the W4A8 form (the reading in fg_oracle.c): each
    product's fp16 input row is quantised to int8 with one scale and multiplied as integers."""
    x = _u16(x)
    R, h = x.shape
    d = h // heads
    if cache.group != GROUP:
        raise ValueError("the W4A8 layer's KV cache uses groups of 64")
    dims = np.array([h, heads, d, weights.ffn], dtype=np.int32)
    out = np.zeros((R, h), dtype=np.float64)
    attn = np.zeros((R, h), dtype=np.float64) if want_attn else None
    sr = np.ascontiguousarray(seq_of_row, dtype=np.int32)
    pr = np.ascontiguousarray(pos_of_row, dtype=np.int32)
    w = weights
    keep = []
    for t in (w.wqkv, w.wo, w.w1, w.w2):
        keep += [np.ascontiguousarray(t.codes), np.ascontiguousarray(t.gmin), np.ascontiguousarray(t.gstep),
                 np.ascontiguousarray(t.cscale, dtype=np.float32)]
    mats = (ctypes.c_void_p * 16)(*[a.ctypes.data for a in keep])
    args = [_p(dims), float(eps), ctypes.cast(mats, ctypes.c_void_p)]
    args += [_p(w.b["bqkv"]), _p(w.b["bo"]), _p(w.b["b1"]), _p(w.b["b2"])]
    args += [_p(w.b["ln1_g"]), _p(w.b["ln1_b"]), _p(w.b["ln2_g"]), _p(w.b["ln2_b"])]
    args += cache.ptrs() + [cache.S, cache.maxL]
    args += [_p(x), R, _p(sr), _p(pr), int(kv_only), _p(out), _p(attn), int(nthreads)]
    rc = lib().oracle_layer_rows_w4a8(*args)
    assert rc == 0, rc
    return out, attn


def timed(fn, *a, **k):
    t0 = time.perf_counter()
    r = fn(*a, **k)
    return r, time.perf_counter() - t0
