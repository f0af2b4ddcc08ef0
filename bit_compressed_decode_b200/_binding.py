"""ctypes binding of ``libfg_b200.so`` (the C ABI in ``include/fg.h``).

Argument marshalling only: torch provides device memory and streams, every
step of the computation runs in the library's CUDA kernels.  The function
names are those of the C ABI.  A missing library raises at import time; there
is no fallback path.
"""
from __future__ import annotations

import ctypes
import os
from ctypes import POINTER, Structure, c_char_p, c_float, c_int, c_int32, c_int64, c_size_t, c_uint16, c_void_p

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libfg_b200.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is not built; run `python -m bit_compressed_decode_b200.build`")
_lib = ctypes.CDLL(LIB_PATH)

STATUS = {0: "FG_OK", 1: "FG_ERR_INVALID", 2: "FG_ERR_SHAPE", 3: "FG_ERR_UNSUPPORTED", 4: "FG_ERR_RANGE",
          5: "FG_ERR_CUDA", 6: "FG_ERR_TIMEOUT", 7: "FG_ERR_WORKSPACE"}
FG_EPI_RELU = 1
FG_EPI_RESIDUAL = 2
FG_GEMM_PERSISTENT = 4


class FgError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        msg = f"{where}: {STATUS.get(code, code)}"
        if code == 5:
            msg += f" ({_lib.fg_last_cuda_error().decode()})"
        super().__init__(msg)


class fg_qtensor(Structure):
    _fields_ = [("codes", c_void_p), ("mins", c_void_p), ("scales", c_void_p), ("ndim", c_int32),
                ("shape", c_int64 * 4), ("dim", c_int32), ("bits", c_int32), ("group", c_int32)]


class fg_kv_cache(Structure):
    _fields_ = [("k_codes", c_void_p), ("k_mins", c_void_p), ("k_scales", c_void_p),
                ("v_codes", c_void_p), ("v_mins", c_void_p), ("v_scales", c_void_p),
                ("num_seqs", c_int32), ("num_heads", c_int32), ("head_dim", c_int32), ("max_len", c_int32),
                ("group", c_int32)]


class fg_layer_config(Structure):
    _fields_ = [("hidden", c_int32), ("num_heads", c_int32), ("head_dim", c_int32), ("ffn", c_int32),
                ("ln_eps", c_float), ("group", c_int32), ("act_bits", c_int32)]


class fg_layer_weights(Structure):
    _fields_ = [("wqkv", fg_qtensor), ("wo", fg_qtensor), ("w1", fg_qtensor), ("w2", fg_qtensor)] + [
        (n, c_void_p) for n in ("bqkv", "bo", "b1", "b2", "ln1_g", "ln1_b", "ln2_g", "ln2_b")] + [
        ("cscale", c_void_p * 4)]


class fg_w4a8_weight(Structure):
    _fields_ = [("codes", c_void_p), ("gmin", c_void_p), ("gstep", c_void_p), ("cscale", c_void_p),
                ("N", c_int64), ("K", c_int64)]


def _decl(name, restype, *args):
    f = getattr(_lib, name)
    f.restype = restype
    f.argtypes = list(args)
    return f


P = c_void_p
_decl("fg_status_string", c_char_p, c_int)
_decl("fg_sync_status", c_int, P)
_decl("fg_last_cuda_error", c_char_p)
_decl("fg_qtensor_bytes", c_int, c_int, POINTER(c_int64), c_int, c_int, c_int, POINTER(c_size_t), POINTER(c_size_t))
_decl("fg_quantize", c_int, P, c_int, POINTER(c_int64), c_int, c_int, c_int, POINTER(fg_qtensor), P)
_decl("fg_dequantize", c_int, POINTER(fg_qtensor), P, P)
_decl("fg_kv_cache_bytes", c_int, c_int, c_int, c_int, c_int, c_int, POINTER(c_size_t), POINTER(c_size_t))
_decl("fg_kv_append", c_int, POINTER(fg_kv_cache), P, P, c_int64, c_int, c_int, P, P)
_decl("fg_attention_decode", c_int, POINTER(fg_kv_cache), P, c_int64, P, c_int64, c_int, c_int, P, P)
_decl("fg_attention_decode_append", c_int, POINTER(fg_kv_cache), P, c_int64, P, P, c_int64, P, c_int64, c_int, P, P)
_decl("fg_linear_workspace_bytes", c_size_t, c_int, c_int, c_int)
_decl("fg_linear_plan", c_int, c_int, c_int, c_int, POINTER(c_int), POINTER(c_int), POINTER(c_int))
_decl("fg_linear_w4a16", c_int, P, c_int, c_int, POINTER(fg_qtensor), P, P, c_int, c_int, c_float, P, P, c_size_t, P)
_decl("fg_layernorm", c_int, P, c_int, c_int, P, P, c_float, P, P)
_decl("fg_w4a8_quantize_weight", c_int, P, POINTER(fg_w4a8_weight), P)
_decl("fg_act8_quantize", c_int, P, c_int, c_int, P, P, P)
_decl("fg_linear_w4a8", c_int, P, P, c_int, c_int, POINTER(fg_w4a8_weight), P, P, c_int, c_int, c_float, P, P,
      c_size_t, P)
_decl("fg_linear_w4a8_workspace_bytes", c_size_t, c_int, c_int, c_int)
_decl("fg_linear_w4a8_plan", c_int, c_int, c_int, c_int, POINTER(c_int), POINTER(c_int))
_decl("fg_layer_blob_bytes", c_size_t, POINTER(fg_layer_config))
_decl("fg_layer_weights_from_blob", c_int, POINTER(fg_layer_config), P, POINTER(fg_layer_weights))
_decl("fg_layer_workspace_bytes", c_size_t, POINTER(fg_layer_config), c_int)
_decl("fg_layer_decode", c_int, POINTER(fg_layer_config), POINTER(fg_layer_weights), POINTER(fg_kv_cache), P, P, P,
      c_int, c_int, P, c_size_t, P)
_decl("fg_layer_prefill", c_int, POINTER(fg_layer_config), POINTER(fg_layer_weights), POINTER(fg_kv_cache), P, P, P,
      c_int, c_int, c_int, P, c_size_t, P)
_decl("fg_layer_decode_noalloc", c_int, POINTER(fg_layer_config), POINTER(fg_layer_weights), POINTER(fg_kv_cache),
      P, P, P, c_int, c_int, P)
_decl("fg_profile_enable", c_int, c_int)
_decl("fg_profile_collect", c_int, POINTER(c_float), POINTER(c_int), c_int)
_decl("fg_stack_create", c_int, POINTER(fg_layer_config), c_int, POINTER(c_void_p), P, P, POINTER(c_void_p))
_decl("fg_stack_decode", c_int, P, POINTER(fg_kv_cache), P, P, P, c_int, c_int, P, c_size_t, P, P)
_decl("fg_stack_prefill", c_int, P, POINTER(fg_kv_cache), P, P, P, c_int, c_int, c_int, P, c_size_t, P, P)
_decl("fg_stack_decode_host_kv", c_int, P, POINTER(fg_kv_cache), POINTER(fg_kv_cache), c_int, c_int, c_int, P, P, P,
      c_int, c_int, P, c_size_t, P, P)
_decl("fg_stack_inject_copy_failure", c_int, P, c_int)
_decl("fg_test_gemm_stall", c_int, c_int, ctypes.c_uint64)
_decl("fg_stack_destroy", c_int, P)
_decl("fg_stack_one_buffer_bytes", c_size_t, POINTER(fg_layer_config))


def lib():
    return _lib


def _check(rc: int, where: str) -> None:
    if rc != 0:
        raise FgError(rc, where)


def _stream(stream=None):
    if stream is None:
        if not torch.cuda.is_available():
            return None
        stream = torch.cuda.current_stream()
    return c_void_p(stream.cuda_stream)


def _ptr(t):
    return None if t is None else c_void_p(t.data_ptr())


def _need(t: torch.Tensor, dtype, name: str) -> None:
    if t.dtype != dtype or not t.is_cuda or not t.is_contiguous():
        raise ValueError(f"{name}: expected a contiguous CUDA {dtype} tensor, got {t.dtype} on {t.device}")


# ---------------------------------------------------------------------------------------
# packed tensors
# ---------------------------------------------------------------------------------------

class QTensor:
    """Packed tensor (device): codes uint8 (two 4-bit or one 8-bit code per byte), mins/scales
    float16, grouped along ``dim``."""

    def __init__(self, codes, mins, scales, shape, dim, group: int = 64, bits: int = 4):
        self.codes, self.mins, self.scales = codes, mins, scales
        self.shape, self.dim, self.group, self.bits = tuple(int(s) for s in shape), dim, group, bits

    def struct(self) -> fg_qtensor:
        s = fg_qtensor()
        s.codes, s.mins, s.scales = self.codes.data_ptr(), self.mins.data_ptr(), self.scales.data_ptr()
        s.ndim = len(self.shape)
        for i in range(4):
            s.shape[i] = self.shape[i] if i < len(self.shape) else 1
        s.dim, s.bits, s.group = self.dim, self.bits, self.group
        return s


def fg_qtensor_bytes(shape, dim=-1, bits=4, group=64):
    shape = tuple(int(s) for s in shape)
    dim = dim % len(shape)
    cb, mb = c_size_t(), c_size_t()
    arr = (c_int64 * len(shape))(*shape)
    _check(_lib.fg_qtensor_bytes(len(shape), arr, dim, bits, group, ctypes.byref(cb), ctypes.byref(mb)),
           "fg_qtensor_bytes")
    return cb.value, mb.value


def fg_quantize(x: torch.Tensor, dim: int = -1, bits: int = 4, group: int = 64, stream=None,
                out: QTensor | None = None) -> QTensor:
    _need(x, torch.float16, "x")
    shape = tuple(x.shape)
    dim = dim % len(shape)
    fg_qtensor_bytes(shape, dim, bits, group)
    if out is None:
        cs = list(shape); cs[dim] = cs[dim] * bits // 8
        ms = list(shape); ms[dim] //= group
        out = QTensor(torch.empty(cs, dtype=torch.uint8, device=x.device),
                      torch.empty(ms, dtype=torch.float16, device=x.device),
                      torch.empty(ms, dtype=torch.float16, device=x.device), shape, dim, group, bits)
    out.bits = bits
    s = out.struct()
    arr = (c_int64 * len(shape))(*shape)
    _check(_lib.fg_quantize(_ptr(x), len(shape), arr, dim, bits, group, ctypes.byref(s), _stream(stream)),
           "fg_quantize")
    out.group = group
    return out


def fg_dequantize(q: QTensor, stream=None) -> torch.Tensor:
    y = torch.empty(q.shape, dtype=torch.float16, device=q.codes.device)
    s = q.struct()
    _check(_lib.fg_dequantize(ctypes.byref(s), _ptr(y), _stream(stream)), "fg_dequantize")
    return y


# ---------------------------------------------------------------------------------------
# KV cache
# ---------------------------------------------------------------------------------------

class KVCache:
    """4-bit KV cache of one layer, allocated with torch on ``device``; head_dim quantised in
    groups of ``group`` (64 or 128)."""

    def __init__(self, num_seqs, num_heads, head_dim, max_len, device="cuda", arrays=None, pin_memory=False,
                 group: int = 64):
        """``pin_memory=True`` with ``device="cpu"`` allocates page-locked host arrays, the form
        fg_stack_decode_host_kv copies from and back to."""
        self.num_seqs, self.num_heads, self.head_dim, self.max_len = num_seqs, num_heads, head_dim, max_len
        self.group = group
        cb, mb = c_size_t(), c_size_t()
        _check(_lib.fg_kv_cache_bytes(num_seqs, num_heads, head_dim, max_len, group, ctypes.byref(cb),
                                      ctypes.byref(mb)), "fg_kv_cache_bytes")
        ng = head_dim // group
        if arrays is None:
            cshape = (num_seqs, num_heads, max_len, head_dim // 2)
            mshape = (num_seqs, num_heads, max_len, ng)
            kw = {"pin_memory": True} if pin_memory else {}
            arrays = [torch.zeros(cshape, dtype=torch.uint8, device=device, **kw),
                      torch.zeros(mshape, dtype=torch.float16, device=device, **kw),
                      torch.zeros(mshape, dtype=torch.float16, device=device, **kw),
                      torch.zeros(cshape, dtype=torch.uint8, device=device, **kw),
                      torch.zeros(mshape, dtype=torch.float16, device=device, **kw),
                      torch.zeros(mshape, dtype=torch.float16, device=device, **kw)]
        self.k_codes, self.k_mins, self.k_scales, self.v_codes, self.v_mins, self.v_scales = arrays

    def arrays(self):
        return [self.k_codes, self.k_mins, self.k_scales, self.v_codes, self.v_mins, self.v_scales]

    def view(self, s0: int, n: int) -> "KVCache":
        """The cache of sequences [s0, s0+n) (shares memory)."""
        return KVCache(n, self.num_heads, self.head_dim, self.max_len,
                       arrays=[a[s0:s0 + n] for a in self.arrays()], group=self.group)

    def struct(self) -> fg_kv_cache:
        s = fg_kv_cache()
        (s.k_codes, s.k_mins, s.k_scales, s.v_codes, s.v_mins, s.v_scales) = [a.data_ptr() for a in self.arrays()]
        s.num_seqs, s.num_heads, s.head_dim, s.max_len = self.num_seqs, self.num_heads, self.head_dim, self.max_len
        s.group = self.group
        return s

    def nbytes(self) -> int:
        return sum(a.numel() * a.element_size() for a in self.arrays())


def fg_kv_append(cache: KVCache, k: torch.Tensor, v: torch.Tensor, positions: torch.Tensor,
                 rows_per_seq: int = 1, ld: int | None = None, stream=None) -> None:
    rows = k.shape[0]
    ld = k.stride(0) if ld is None else ld
    _need(positions, torch.int32, "positions")
    s = cache.struct()
    _check(_lib.fg_kv_append(ctypes.byref(s), _ptr(k), _ptr(v), ld, rows, rows_per_seq, _ptr(positions),
                             _stream(stream)), "fg_kv_append")


def fg_attention_decode(cache: KVCache, q: torch.Tensor, positions: torch.Tensor, rows_per_seq: int = 1,
                        out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    rows = q.shape[0]
    hd = cache.num_heads * cache.head_dim
    if out is None:
        out = torch.empty((rows, hd), dtype=torch.float16, device=q.device)
    s = cache.struct()
    _check(_lib.fg_attention_decode(ctypes.byref(s), _ptr(q), q.stride(0), _ptr(out), out.stride(0), rows,
                                    rows_per_seq, _ptr(positions), _stream(stream)), "fg_attention_decode")
    return out


def fg_attention_decode_append(cache: KVCache, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                               positions: torch.Tensor, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Append k, v at ``positions`` and attend with q, one launch (decode rows: one per sequence)."""
    rows = q.shape[0]
    hd = cache.num_heads * cache.head_dim
    if k.stride(0) != v.stride(0):
        raise ValueError("k and v must share a row stride")
    _need(positions, torch.int32, "positions")
    if out is None:
        out = torch.empty((rows, hd), dtype=torch.float16, device=q.device)
    s = cache.struct()
    _check(_lib.fg_attention_decode_append(ctypes.byref(s), _ptr(q), q.stride(0), _ptr(k), _ptr(v), k.stride(0),
                                           _ptr(out), out.stride(0), rows, _ptr(positions), _stream(stream)),
           "fg_attention_decode_append")
    return out


# ---------------------------------------------------------------------------------------
# linear / layernorm
# ---------------------------------------------------------------------------------------

def fg_linear_workspace_bytes(M: int, N: int, K: int) -> int:
    return int(_lib.fg_linear_workspace_bytes(M, N, K))


def fg_linear_plan(M: int, N: int, K: int) -> tuple:
    """(tokens per output tile, k splits) of the classic launch fg_linear_w4a16 makes for this
    shape (see fg_linear_plan_pairs for the persistent launch)."""
    t, s, p = c_int(), c_int(), c_int()
    _check(_lib.fg_linear_plan(M, N, K, ctypes.byref(t), ctypes.byref(s), ctypes.byref(p)), "fg_linear_plan")
    return t.value, s.value


def fg_linear_plan_pairs(M: int, N: int, K: int) -> int:
    """CTA pairs of the persistent launch fg_linear_w4a16(..., persistent=True) takes for this
    shape given fg_linear_workspace_bytes of scratch (0: not available, the classic launch)."""
    t, s, p = c_int(), c_int(), c_int()
    _check(_lib.fg_linear_plan(M, N, K, ctypes.byref(t), ctypes.byref(s), ctypes.byref(p)), "fg_linear_plan")
    return p.value


def fg_linear_classic_scratch_bytes(M: int, N: int, K: int, flags: bool = True) -> int:
    """Scratch the classic launch's split k-range adds its partial sums through (0 without a
    split): the fp32 partials and, with flags, the flags that let the split ranks run as
    separate clusters; with less than the partials it adds them on chip."""
    t, s = fg_linear_plan(M, N, K)
    if M <= 256 or s < 2:
        return 0
    tiles = -(-N // 256) * -(-M // t)
    return tiles * s * t * 256 * 4 + (tiles * s * 2 * 8 if flags else 0)


def fg_linear_w4a16(x: torch.Tensor, w: QTensor, bias=None, residual=None, relu: bool = False,
                    qscale_cols: int = 0, qscale: float = 1.0, out=None, workspace=None, stream=None,
                    persistent: bool = False):
    _need(x, torch.float16, "x")
    M, K = x.shape
    N = w.shape[0]
    if out is None:
        out = torch.empty((M, N), dtype=torch.float16, device=x.device)
    need = fg_linear_workspace_bytes(M, N, K)
    if workspace is None and need:
        workspace = torch.empty(need, dtype=torch.uint8, device=x.device)
    flags = ((FG_EPI_RELU if relu else 0) | (FG_EPI_RESIDUAL if residual is not None else 0) |
             (FG_GEMM_PERSISTENT if persistent else 0))
    s = w.struct()
    _check(_lib.fg_linear_w4a16(_ptr(x), M, K, ctypes.byref(s), _ptr(bias), _ptr(residual), flags, qscale_cols,
                                qscale, _ptr(out), _ptr(workspace), 0 if workspace is None else workspace.numel(),
                                _stream(stream)), "fg_linear_w4a16")
    return out


# ---------------------------------------------------------------------------------------
# W4A8: 4-bit weights, 8-bit activations, integer products ([Q8] in fg.h)
# ---------------------------------------------------------------------------------------

class W4A8Weight:
    """Device W4A8 weight: codes uint8 [N, K/2], gmin int8 [N, K/64], gstep uint8 [N, K/64],
    cscale float32 [N]."""

    def __init__(self, N: int, K: int, device="cuda"):
        self.N, self.K = N, K
        self.codes = torch.empty((N, K // 2), dtype=torch.uint8, device=device)
        self.gmin = torch.empty((N, K // 64), dtype=torch.int8, device=device)
        self.gstep = torch.empty((N, K // 64), dtype=torch.uint8, device=device)
        self.cscale = torch.empty(N, dtype=torch.float32, device=device)

    def struct(self) -> fg_w4a8_weight:
        return fg_w4a8_weight(self.codes.data_ptr(), self.gmin.data_ptr(), self.gstep.data_ptr(),
                              self.cscale.data_ptr(), self.N, self.K)


def fg_w4a8_quantize_weight(w: torch.Tensor, out: W4A8Weight = None, stream=None) -> W4A8Weight:
    _need(w, torch.float16, "w")
    N, K = w.shape
    if out is None:
        out = W4A8Weight(N, K, device=w.device)
    s = out.struct()
    _check(_lib.fg_w4a8_quantize_weight(_ptr(w), ctypes.byref(s), _stream(stream)), "fg_w4a8_quantize_weight")
    return out


def fg_act8_quantize(x: torch.Tensor, a8=None, ascale=None, stream=None):
    """(a8 int8 [M, K], ascale float32 [M])."""
    _need(x, torch.float16, "x")
    M, K = x.shape
    if a8 is None:
        a8 = torch.empty((M, K), dtype=torch.int8, device=x.device)
    if ascale is None:
        ascale = torch.empty(M, dtype=torch.float32, device=x.device)
    _check(_lib.fg_act8_quantize(_ptr(x), M, K, _ptr(a8), _ptr(ascale), _stream(stream)), "fg_act8_quantize")
    return a8, ascale


def fg_linear_w4a8_plan(M: int, N: int, K: int) -> tuple:
    t, s = c_int(), c_int()
    _check(_lib.fg_linear_w4a8_plan(M, N, K, ctypes.byref(t), ctypes.byref(s)), "fg_linear_w4a8_plan")
    return t.value, s.value


def fg_linear_w4a8_workspace_bytes(M: int, N: int, K: int) -> int:
    return int(_lib.fg_linear_w4a8_workspace_bytes(M, N, K))


def fg_linear_w4a8(a8: torch.Tensor, ascale: torch.Tensor, w: W4A8Weight, bias=None, residual=None,
                   relu: bool = False, qscale_cols: int = 0, qscale: float = 1.0, out=None, workspace=None,
                   stream=None):
    """``workspace``: None allocates the scratch the CTA-pair launch can use; a tensor is passed
    as given (a 0-element one means none: k splits are then added on chip)."""
    _need(a8, torch.int8, "a8")
    _need(ascale, torch.float32, "ascale")
    M, K = a8.shape
    if out is None:
        out = torch.empty((M, w.N), dtype=torch.float16, device=a8.device)
    if workspace is None:
        need = fg_linear_w4a8_workspace_bytes(M, w.N, K)
        workspace = torch.empty(need, dtype=torch.uint8, device=a8.device) if need else None
    flags = (FG_EPI_RELU if relu else 0) | (FG_EPI_RESIDUAL if residual is not None else 0)
    s = w.struct()
    _check(_lib.fg_linear_w4a8(_ptr(a8), _ptr(ascale), M, K, ctypes.byref(s), _ptr(bias), _ptr(residual), flags,
                               qscale_cols, qscale, _ptr(out), _ptr(workspace),
                               0 if workspace is None else workspace.numel(), _stream(stream)), "fg_linear_w4a8")
    return out


def fg_layernorm(x: torch.Tensor, gamma=None, beta=None, eps: float = 1e-5, out=None, stream=None):
    _need(x, torch.float16, "x")
    M, h = x.shape
    if out is None:
        out = torch.empty_like(x)
    _check(_lib.fg_layernorm(_ptr(x), M, h, _ptr(gamma), _ptr(beta), eps, _ptr(out), _stream(stream)),
           "fg_layernorm")
    return out


# ---------------------------------------------------------------------------------------
# layer
# ---------------------------------------------------------------------------------------

class LayerConfig:
    def __init__(self, hidden: int, num_heads: int, ffn: int, ln_eps: float = 1e-5, group: int = 64,
                 act_bits: int = 16):
        """``group``: the 4-bit group of the layer's weights and KV cache (64 or 128);
        ``act_bits``: 16 (W4A16) or 8 (W4A8 products, weights in the W4A8 form, group 64)."""
        self.hidden, self.num_heads, self.ffn, self.ln_eps, self.group = hidden, num_heads, ffn, ln_eps, group
        self.act_bits = act_bits
        self.head_dim = hidden // num_heads

    def struct(self) -> fg_layer_config:
        return fg_layer_config(self.hidden, self.num_heads, self.head_dim, self.ffn, self.ln_eps, self.group,
                               self.act_bits)

    def blob_bytes(self) -> int:
        c = self.struct()
        n = int(_lib.fg_layer_blob_bytes(ctypes.byref(c)))
        if n == 0:
            raise FgError(3, "fg_layer_blob_bytes")
        return n

    def workspace_bytes(self, rows: int) -> int:
        c = self.struct()
        return int(_lib.fg_layer_workspace_bytes(ctypes.byref(c), rows))


_MATS = ("wqkv", "wo", "w1", "w2")
_VECS = ("bqkv", "bo", "b1", "b2", "ln1_g", "ln1_b", "ln2_g", "ln2_b")


def weights_struct(cfg: LayerConfig, blob: torch.Tensor) -> fg_layer_weights:
    """fg_layer_weights pointing into ``blob`` (device or host)."""
    c = cfg.struct()
    w = fg_layer_weights()
    _check(_lib.fg_layer_weights_from_blob(ctypes.byref(c), c_void_p(blob.data_ptr()), ctypes.byref(w)),
           "fg_layer_weights_from_blob")
    return w


class LayerWeights:
    """One layer's 4-bit weights in a single device blob (see fg_layer_blob_bytes)."""

    def __init__(self, cfg: LayerConfig, blob: torch.Tensor):
        self.cfg, self.blob = cfg, blob
        self._w = weights_struct(cfg, blob)

    def struct(self) -> fg_layer_weights:
        return self._w

    def matrix(self, name: str) -> QTensor:
        """QTensor view of one packed matrix inside the blob."""
        q = getattr(self._w, name)
        base = self.blob.data_ptr()
        n, k = q.shape[0], q.shape[1]
        def sub(ptr, nbytes):
            off = ptr - base
            return self.blob[off:off + nbytes]
        G = self.cfg.group
        codes = sub(q.codes, n * k // 2).view(n, k // 2)
        mins = sub(q.mins, n * k // G * 2).view(torch.float16).view(n, k // G)
        scales = sub(q.scales, n * k // G * 2).view(torch.float16).view(n, k // G)
        return QTensor(codes, mins, scales, (n, k), 1, G)

    def w4a8_matrix(self, name: str) -> "W4A8Weight":
        """W4A8Weight view of one matrix inside the blob of a W4A8 layer."""
        i = _MATS.index(name)
        q = getattr(self._w, name)
        base = self.blob.data_ptr()
        n, k = q.shape[0], q.shape[1]
        def sub(ptr, nbytes):
            off = ptr - base
            return self.blob[off:off + nbytes]
        m = W4A8Weight.__new__(W4A8Weight)
        m.N, m.K = n, k
        m.codes = sub(q.codes, n * k // 2).view(n, k // 2)
        m.gmin = sub(q.mins, n * k // 64).view(torch.int8).view(n, k // 64)
        m.gstep = sub(q.scales, n * k // 64).view(n, k // 64)
        m.cscale = sub(self._w.cscale[i], n * 4).view(torch.float32)
        return m

    def vector(self, name: str) -> torch.Tensor:
        ptr = getattr(self._w, name)
        off = ptr - self.blob.data_ptr()
        n = {"bqkv": 3 * self.cfg.hidden, "b1": self.cfg.ffn}.get(name, self.cfg.hidden)
        return self.blob[off:off + 2 * n].view(torch.float16)

    @staticmethod
    def from_fp16(cfg: LayerConfig, w16: dict, device="cuda", stream=None) -> "LayerWeights":
        """Quantises fp16 weights (``[out, in]`` orientation) into a new device blob with fg_quantize."""
        blob = torch.empty(cfg.blob_bytes(), dtype=torch.uint8, device=device)
        lw = LayerWeights(cfg, blob)
        for name in _MATS:
            x = torch.as_tensor(w16[name]).to(device=device, dtype=torch.float16).contiguous()
            if cfg.act_bits == 8:
                fg_w4a8_quantize_weight(x, out=lw.w4a8_matrix(name), stream=stream)
            else:
                fg_quantize(x, dim=1, group=cfg.group, stream=stream, out=lw.matrix(name))
        for name in _VECS:
            lw.vector(name).copy_(torch.as_tensor(w16[name]).to(device=device, dtype=torch.float16))
        return lw


def fg_layer_decode(cfg: LayerConfig, w: LayerWeights, cache: KVCache, x: torch.Tensor, positions: torch.Tensor,
                    num_gpu_batches: int = 1, gpu_batch_size: int | None = None, out=None, workspace=None,
                    stream=None):
    S = x.shape[0]
    if gpu_batch_size is None:
        gpu_batch_size = S // num_gpu_batches
    if out is None:
        out = torch.empty_like(x)
    if workspace is None:
        workspace = torch.empty(cfg.workspace_bytes(S), dtype=torch.uint8, device=x.device)
    c = cfg.struct()
    ws = w.struct()
    kv = cache.struct()
    _check(_lib.fg_layer_decode(ctypes.byref(c), ctypes.byref(ws), ctypes.byref(kv), _ptr(x), _ptr(out),
                                _ptr(positions), num_gpu_batches, gpu_batch_size, _ptr(workspace),
                                workspace.numel(), _stream(stream)), "fg_layer_decode")
    return out


NOALLOC_SCRATCH_BYTES = 96 << 20


def fg_layer_decode_noalloc(cfg: LayerConfig, w: LayerWeights, cache: KVCache, x: torch.Tensor,
                            positions: torch.Tensor, num_gpu_batches: int = 1, gpu_batch_size: int | None = None,
                            out=None, stream=None):
    """fg_layer_decode with the library's static scratch instead of a caller workspace."""
    S = x.shape[0]
    if gpu_batch_size is None:
        gpu_batch_size = S // num_gpu_batches
    if out is None:
        out = torch.empty_like(x)
    c = cfg.struct()
    ws = w.struct()
    kv = cache.struct()
    _check(_lib.fg_layer_decode_noalloc(ctypes.byref(c), ctypes.byref(ws), ctypes.byref(kv), _ptr(x), _ptr(out),
                                        _ptr(positions), num_gpu_batches, gpu_batch_size, _stream(stream)),
           "fg_layer_decode_noalloc")
    return out


def fg_layer_prefill(cfg: LayerConfig, w: LayerWeights, cache: KVCache, x: torch.Tensor, positions: torch.Tensor,
                     num_gpu_batches: int = 1, gpu_batch_size: int | None = None, out=None, workspace=None,
                     stream=None, max_workspace_rows: int = 65536):
    S, P = x.shape[0], x.shape[1]
    if gpu_batch_size is None:
        gpu_batch_size = S // num_gpu_batches
    if out is None:
        out = torch.empty_like(x)
    if workspace is None:
        seqs = max(1, min(S, max_workspace_rows // P))
        workspace = torch.empty(cfg.workspace_bytes(seqs * P), dtype=torch.uint8, device=x.device)
    c = cfg.struct()
    ws = w.struct()
    kv = cache.struct()
    _check(_lib.fg_layer_prefill(ctypes.byref(c), ctypes.byref(ws), ctypes.byref(kv), _ptr(x), _ptr(out),
                                 _ptr(positions), P, num_gpu_batches, gpu_batch_size, _ptr(workspace),
                                 workspace.numel(), _stream(stream)), "fg_layer_prefill")
    return out


PROFILE_SLOTS = ("ln1", "qkv_gemm", "kv_append", "attention", "out_gemm", "ln2", "fc1_gemm", "fc2_gemm",
                 "qkv_act8", "out_act8", "fc1_act8", "fc2_act8")


def fg_profile_enable(enable: bool = True) -> None:
    _check(_lib.fg_profile_enable(1 if enable else 0), "fg_profile_enable")


def fg_profile_collect() -> dict:
    """{slot name: (total ms, launches)} of the kernels timed since the last collect."""
    n = len(PROFILE_SLOTS)
    ms = (c_float * n)()
    cnt = (c_int * n)()
    _check(_lib.fg_profile_collect(ms, cnt, n), "fg_profile_collect")
    return {PROFILE_SLOTS[i]: (float(ms[i]), int(cnt[i])) for i in range(n)}


def fg_test_gemm_stall(count: int, wait_limit_ns: int) -> None:
    """Test hook: the next `count` one-SM GEMM launches stall their first pipeline stage and give
    up after wait_limit_ns (see fg_test_gemm_stall in fg.h)."""
    _check(_lib.fg_test_gemm_stall(count, wait_limit_ns), "fg_test_gemm_stall")


def fg_sync_status(stream=None) -> None:
    _check(_lib.fg_sync_status(_stream(stream)), "fg_sync_status")


def fg_status_string(code: int) -> str:
    return _lib.fg_status_string(code).decode()


# ---------------------------------------------------------------------------------------
# stack with weights streamed from pinned host memory
# ---------------------------------------------------------------------------------------

class Stack:
    """A stack of layers whose blobs live in (pinned) host tensors; see fg_stack_create."""

    def __init__(self, cfg: LayerConfig, host_blobs, device="cuda", staging_buffers: int = 2):
        """``staging_buffers``: 2 (layers alternate between two device blobs) or 1 (one blob,
        refilled slice by slice as the layer before finishes with each slice)."""
        if staging_buffers not in (1, 2):
            raise ValueError("staging_buffers must be 1 or 2")
        self.cfg = cfg
        self.host_blobs = list(host_blobs)
        c0 = cfg.struct()
        nbytes = cfg.blob_bytes() if staging_buffers == 2 else int(_lib.fg_stack_one_buffer_bytes(ctypes.byref(c0)))
        self.staging = [torch.empty(nbytes, dtype=torch.uint8, device=device) for _ in range(staging_buffers)]
        arr = (c_void_p * len(self.host_blobs))(*[b.data_ptr() for b in self.host_blobs])
        self._arr = arr
        h = c_void_p()
        c = cfg.struct()
        _check(_lib.fg_stack_create(ctypes.byref(c), len(self.host_blobs), arr, _ptr(self.staging[0]),
                                    _ptr(self.staging[-1]), ctypes.byref(h)), "fg_stack_create")
        self._h = h

    def workspace_bytes(self, rows: int) -> int:
        act = (rows * self.cfg.hidden * 2 + 255) // 256 * 256
        return 2 * act + self.cfg.workspace_bytes(rows)

    def decode(self, caches, x, positions, num_gpu_batches=1, gpu_batch_size=None, out=None, workspace=None,
               compute_stream=None, copy_stream=None):
        S = x.shape[0]
        gbs = S // num_gpu_batches if gpu_batch_size is None else gpu_batch_size
        if out is None:
            out = torch.empty_like(x)
        if workspace is None:
            workspace = torch.empty(self.workspace_bytes(S), dtype=torch.uint8, device=x.device)
        kv = (fg_kv_cache * len(caches))(*[c.struct() for c in caches])
        cs = _stream(compute_stream)
        ps = _stream(copy_stream) if copy_stream is not None else c_void_p(torch.cuda.Stream().cuda_stream)
        _check(_lib.fg_stack_decode(self._h, kv, _ptr(x), _ptr(out), _ptr(positions), num_gpu_batches, gbs,
                                    _ptr(workspace), workspace.numel(), cs, ps), "fg_stack_decode")
        return out

    def prefill(self, caches, x, positions, num_gpu_batches=1, gpu_batch_size=None, out=None, workspace=None,
                compute_stream=None, copy_stream=None):
        S, P = x.shape[0], x.shape[1]
        gbs = S // num_gpu_batches if gpu_batch_size is None else gpu_batch_size
        if out is None:
            out = torch.empty_like(x)
        if workspace is None:
            workspace = torch.empty(self.workspace_bytes(S * P), dtype=torch.uint8, device=x.device)
        kv = (fg_kv_cache * len(caches))(*[c.struct() for c in caches])
        cs = _stream(compute_stream)
        ps = _stream(copy_stream) if copy_stream is not None else c_void_p(torch.cuda.Stream().cuda_stream)
        _check(_lib.fg_stack_prefill(self._h, kv, _ptr(x), _ptr(out), _ptr(positions), P, num_gpu_batches, gbs,
                                     _ptr(workspace), workspace.numel(), cs, ps), "fg_stack_prefill")
        return out

    def decode_host_kv(self, host_caches, staging_caches, x, positions, fill_len, wb_begin, wb_end,
                       num_gpu_batches=1, gpu_batch_size=None, out=None, workspace=None, compute_stream=None,
                       copy_stream=None):
        """One decode step with every layer's cache in pinned host memory (fg_stack_decode_host_kv):
        ``host_caches`` one pinned KVCache per layer, ``staging_caches`` two device KVCaches of the same
        geometry; positions [0, fill_len) are filled before each layer and [wb_begin, wb_end) written
        back after it."""
        S = x.shape[0]
        gbs = S // num_gpu_batches if gpu_batch_size is None else gpu_batch_size
        if out is None:
            out = torch.empty_like(x)
        if workspace is None:
            workspace = torch.empty(self.workspace_bytes(S), dtype=torch.uint8, device=x.device)
        hk = (fg_kv_cache * len(host_caches))(*[c.struct() for c in host_caches])
        dk = (fg_kv_cache * 2)(*[c.struct() for c in staging_caches])
        cs = _stream(compute_stream)
        ps = _stream(copy_stream) if copy_stream is not None else c_void_p(torch.cuda.Stream().cuda_stream)
        _check(_lib.fg_stack_decode_host_kv(self._h, hk, dk, fill_len, wb_begin, wb_end, _ptr(x), _ptr(out),
                                            _ptr(positions), num_gpu_batches, gbs, _ptr(workspace),
                                            workspace.numel(), cs, ps), "fg_stack_decode_host_kv")
        return out

    def inject_copy_failure(self, count: int = 1) -> None:
        _check(_lib.fg_stack_inject_copy_failure(self._h, count), "fg_stack_inject_copy_failure")

    def close(self) -> None:
        if self._h:
            _lib.fg_stack_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
