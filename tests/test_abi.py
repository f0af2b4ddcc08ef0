"""The C ABI library loads, exports every symbol include/fg.h declares, and validates
arguments on the host (CPU only: no call here reaches a CUDA launch)."""
import ctypes
import os
import re
import subprocess

import numpy as np
import pytest

import bit_compressed_decode_b200 as fg
from bit_compressed_decode_b200 import _binding as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "fg.h")


def declared():
    with open(HEADER) as f:
        text = f.read()
    return sorted(set(re.findall(r"FG_API\s+[\w\s\*]*?\b(fg_\w+)\s*\(", text)))


def test_header_declares_the_entry_points():
    names = declared()
    for must in ("fg_quantize", "fg_dequantize", "fg_kv_append", "fg_layer_decode", "fg_layer_prefill",
                 "fg_attention_decode", "fg_linear_w4a16", "fg_sync_status", "fg_stack_decode",
                 "fg_layer_decode_noalloc", "fg_stack_decode_host_kv"):
        assert must in names


def test_library_exports_every_declared_symbol():
    out = subprocess.run(["nm", "-D", "--defined-only", fg.LIB_PATH], capture_output=True, text=True).stdout
    exported = set(re.findall(r" T (fg_\w+)", out))
    missing = [n for n in declared() if n not in exported]
    assert not missing, missing
    for n in declared():
        assert hasattr(B.lib(), n)


def test_status_strings():
    for code, name in B.STATUS.items():
        assert fg.fg_status_string(code) == name
    assert fg.fg_status_string(99) == "FG_ERR_UNKNOWN"


def _rc(fn, *args):
    return getattr(B.lib(), fn)(*args)


def test_qtensor_bytes_and_errors():
    assert fg.fg_qtensor_bytes((8, 4096)) == (8 * 4096 // 2, 8 * 4096 // 64 * 2)
    assert fg.fg_qtensor_bytes((6, 128, 5), dim=1) == (6 * 128 * 5 // 2, 6 * 2 * 5 * 2)
    with pytest.raises(fg.FgError, match="SHAPE"):
        fg.fg_qtensor_bytes((8, 96))
    assert fg.fg_qtensor_bytes((8, 64), bits=8) == (8 * 64, 8 * 2)        # 8-bit codes: one per byte
    assert fg.fg_qtensor_bytes((6, 128, 5), dim=1, bits=8, group=128) == (6 * 128 * 5, 6 * 5 * 2)
    for bits in (2, 3, 16):
        with pytest.raises(fg.FgError, match="UNSUPPORTED"):
            fg.fg_qtensor_bytes((8, 64), bits=bits)
    assert fg.fg_qtensor_bytes((8, 256), group=128) == (8 * 256 // 2, 8 * 2 * 2)   # groups of 128
    with pytest.raises(fg.FgError, match="SHAPE"):
        fg.fg_qtensor_bytes((8, 192), group=128)
    with pytest.raises(fg.FgError, match="UNSUPPORTED"):
        fg.fg_qtensor_bytes((8, 256), group=32)
    with pytest.raises(fg.FgError, match="INVALID"):
        fg.fg_qtensor_bytes((1, 2, 3, 4, 64))


def test_quantize_validates_before_launch():
    q = B.fg_qtensor()
    shape = (ctypes.c_int64 * 2)(4, 96)
    assert _rc("fg_quantize", None, 2, shape, 1, 4, 64, ctypes.byref(q), None) == 2   # SHAPE
    shape = (ctypes.c_int64 * 2)(4, 64)
    assert _rc("fg_quantize", None, 2, shape, 1, 4, 64, ctypes.byref(q), None) == 1   # null buffers
    assert _rc("fg_quantize", None, 2, shape, 1, 4, 64, None, None) == 1
    misaligned = ctypes.c_void_p(0x1008)
    q.codes, q.mins, q.scales = 0x1000, 0x2000, 0x3000
    assert _rc("fg_quantize", misaligned, 2, shape, 1, 4, 64, ctypes.byref(q), None) == 1


def test_kv_cache_bytes_rules():
    cb, mb = ctypes.c_size_t(), ctypes.c_size_t()
    assert _rc("fg_kv_cache_bytes", 512, 32, 128, 576, 64, ctypes.byref(cb), ctypes.byref(mb)) == 0
    assert cb.value == 512 * 32 * 576 * 64 and mb.value == 512 * 32 * 576 * 2 * 2
    assert _rc("fg_kv_cache_bytes", 512, 32, 128, 576, 0, ctypes.byref(cb), ctypes.byref(mb)) == 0   # 0 = 64
    assert mb.value == 512 * 32 * 576 * 2 * 2
    # groups of 128 along head_dim ("FlexGen Guide", section 3: groups of 64 or 128)
    assert _rc("fg_kv_cache_bytes", 512, 32, 128, 576, 128, ctypes.byref(cb), ctypes.byref(mb)) == 0
    assert cb.value == 512 * 32 * 576 * 64 and mb.value == 512 * 32 * 576 * 1 * 2
    assert _rc("fg_kv_cache_bytes", 4, 12, 64, 64, 128, ctypes.byref(cb), ctypes.byref(mb)) == 2    # G > head_dim
    assert _rc("fg_kv_cache_bytes", 4, 12, 64, 64, 32, ctypes.byref(cb), ctypes.byref(mb)) == 3     # group 32
    assert _rc("fg_kv_cache_bytes", 4, 12, 96, 64, 64, ctypes.byref(cb), ctypes.byref(mb)) == 3     # head_dim
    assert _rc("fg_kv_cache_bytes", 4, 12, 64, 100, 64, ctypes.byref(cb), ctypes.byref(mb)) == 2    # max_len % 64


def _align(x, a=256):
    return (x + a - 1) // a * a


@pytest.mark.parametrize("h,H,F", [(768, 12, 3072), (4096, 32, 16384), (7168, 56, 28672), (12288, 96, 49152)])
def test_layer_blob_layout(h, H, F):
    cfg = fg.LayerConfig(h, H, F)
    # the blob holds 4 packed matrices (codes n*k/2, mins and scales n*k/64*2 each) and
    # 8 fp16 vectors, every array 256-byte aligned
    want = 0
    for n, k in ((3 * h, h), (h, h), (F, h), (h, F)):
        want += _align(n * k // 2) + 2 * _align(n * k // 64 * 2)
    for n in (3 * h, h, F, h, h, h, h, h):
        want += _align(2 * n)
    assert cfg.blob_bytes() == want
    blob = np.zeros(want + 256, dtype=np.uint8)
    base = (blob.ctypes.data + 255) // 256 * 256
    w = B.fg_layer_weights()
    c = cfg.struct()
    assert _rc("fg_layer_weights_from_blob", ctypes.byref(c), ctypes.c_void_p(base), ctypes.byref(w)) == 0
    spans = []
    for name, (n, k) in zip(("wqkv", "wo", "w1", "w2"), ((3 * h, h), (h, h), (F, h), (h, F))):
        t = getattr(w, name)
        assert (t.shape[0], t.shape[1], t.dim, t.bits, t.group) == (n, k, 1, 4, 64)
        spans += [(t.codes, n * k // 2), (t.mins, n * k // 32), (t.scales, n * k // 32)]
    for name, n in zip(("bqkv", "bo", "b1", "b2", "ln1_g", "ln1_b", "ln2_g", "ln2_b"),
                       (3 * h, h, F, h, h, h, h, h)):
        spans.append((getattr(w, name), 2 * n))
    spans.sort()
    for (p, nbytes), (q, _) in zip(spans, spans[1:]):
        assert p % 256 == 0 and p + nbytes <= q
    assert spans[-1][0] + spans[-1][1] <= base + want


def test_layer_blob_layout_group128():
    # groups of 128: the same codes, half the metadata of groups of 64
    h, H, F = 4096, 32, 16384
    c64, c128 = fg.LayerConfig(h, H, F), fg.LayerConfig(h, H, F, group=128)
    want = 0
    for n, k in ((3 * h, h), (h, h), (F, h), (h, F)):
        want += _align(n * k // 2) + 2 * _align(n * k // 128 * 2)
    for n in (3 * h, h, F, h, h, h, h, h):
        want += _align(2 * n)
    assert c128.blob_bytes() == want < c64.blob_bytes()
    blob = np.zeros(want + 256, dtype=np.uint8)
    base = (blob.ctypes.data + 255) // 256 * 256
    w = B.fg_layer_weights()
    c = c128.struct()
    assert _rc("fg_layer_weights_from_blob", ctypes.byref(c), ctypes.c_void_p(base), ctypes.byref(w)) == 0
    assert w.wqkv.group == w.w2.group == 128
    bad = fg.LayerConfig(768, 12, 3072, group=128).struct()  # head_dim 64 cannot hold a group of 128
    assert B.lib().fg_layer_blob_bytes(ctypes.byref(bad)) == 0


def test_opt6p7b_sizes():
    cfg = fg.LayerConfig(4096, 32, 16384)
    # 12 h^2 parameters at 4.5 bits (codes + fp16 min and scale per 64): 113.2 MB + vectors
    assert abs(cfg.blob_bytes() - 12 * 4096 ** 2 * (0.5 + 4 / 64)) < 0.2e6
    # scratch per decode step: a, o, h1 [S,h] + qkv [S,3h] + ffn [S,F] in fp16, then the
    # largest split-k scratch of the four GEMMs (0 without a GPU to plan the splits for)
    h, F = 4096, 16384
    g = max(fg.fg_linear_workspace_bytes(512, n, k) for n, k in ((3 * h, h), (h, h), (F, h), (h, F)))
    assert cfg.workspace_bytes(512) == 512 * (6 * h + F) * 2 + (g + 255) // 256 * 256


def test_layer_entry_points_validate_config():
    bad = B.fg_layer_config(4096, 32, 100, 16384, 1e-5, 64)     # head_dim inconsistent
    assert B.lib().fg_layer_blob_bytes(ctypes.byref(bad)) == 0
    w = B.fg_layer_weights()
    kv = B.fg_kv_cache()
    rc = _rc("fg_layer_decode", ctypes.byref(bad), ctypes.byref(w), ctypes.byref(kv), None, None, None, 1, 1, None,
             0, None)
    assert rc == 3


def test_noalloc_rejects_oversized_block_on_host():
    cfg = fg.LayerConfig(4096, 32, 16384)
    c = cfg.struct()
    w = B.fg_layer_weights()
    kv = B.fg_kv_cache()
    assert cfg.workspace_bytes(2048) > fg.NOALLOC_SCRATCH_BYTES
    rc = _rc("fg_layer_decode_noalloc", ctypes.byref(c), ctypes.byref(w), ctypes.byref(kv), None, None, None, 1,
             2048, None)
    assert rc == 7                                          # FG_ERR_WORKSPACE, before any CUDA call


def test_noalloc_rejects_row_count_overflow_on_host():
    cfg = fg.LayerConfig(4096, 32, 16384)
    c = cfg.struct()
    w = B.fg_layer_weights()
    kv = B.fg_kv_cache()
    rc = _rc("fg_layer_decode_noalloc", ctypes.byref(c), ctypes.byref(w), ctypes.byref(kv), None, None, None, 65536,
             65536, None)
    assert rc == 2                                          # FG_ERR_SHAPE: 2^32 rows, before any CUDA call


def test_gemm_stall_hook_validates():
    assert _rc("fg_test_gemm_stall", -1, 1000) == 1
    assert _rc("fg_test_gemm_stall", 1, 0) == 1             # a zero limit
    assert _rc("fg_test_gemm_stall", 1, 3_000_000_000) == 1  # above the normal 2 s limit
    assert _rc("fg_test_gemm_stall", 0, 1000) == 0           # disarm


def test_stack_create_validates():
    cfg = fg.LayerConfig(768, 12, 3072)
    c = cfg.struct()
    h = ctypes.c_void_p()
    blobs = (ctypes.c_void_p * 2)(None, None)
    assert _rc("fg_stack_create", ctypes.byref(c), 2, blobs, ctypes.c_void_p(256), ctypes.c_void_p(512),
               ctypes.byref(h)) == 1
    assert _rc("fg_stack_create", ctypes.byref(c), 0, blobs, ctypes.c_void_p(256), ctypes.c_void_p(512),
               ctypes.byref(h)) == 1


def test_stack_decode_host_kv_validates_before_cuda():
    kv = (B.fg_kv_cache * 2)()
    assert _rc("fg_stack_decode_host_kv", None, kv, kv, 0, 0, 1, None, None, None, 1, 1, None, 0, None,
               None) == 1                                    # no stack: FG_ERR_INVALID


def _fake_kv(S=4, H=2, d=128, maxL=64):
    """A cache descriptor with aligned, never dereferenced addresses: for checks that must
    fail on the host, before any CUDA call."""
    kv = B.fg_kv_cache()
    for i, name in enumerate(("k_codes", "k_mins", "k_scales", "v_codes", "v_mins", "v_scales")):
        setattr(kv, name, 0x100000 * (i + 1))
    kv.num_seqs, kv.num_heads, kv.head_dim, kv.max_len, kv.group = S, H, d, maxL, 64
    return kv


def test_attention_decode_append_validates_on_host():
    kv = _fake_kv()
    P = 0x800000                                            # aligned, never dereferenced
    args = lambda **o: [ctypes.byref(o.get("kv", kv)), o.get("q", P), o.get("ldq", 256), o.get("k", P + 512),
                        o.get("v", P + 1024), o.get("ldkv", 768), o.get("out", P * 2), o.get("ldo", 256),
                        o.get("rows", 4), o.get("pos", P * 3), None]
    assert _rc("fg_attention_decode_append", *args(rows=5)) == 2       # more rows than sequences: SHAPE
    assert _rc("fg_attention_decode_append", *args(rows=-1)) == 2
    assert _rc("fg_attention_decode_append", *args(rows=0)) == 0       # nothing to do
    assert _rc("fg_attention_decode_append", *args(k=None)) == 1       # INVALID
    assert _rc("fg_attention_decode_append", *args(v=P + 1026)) == 1   # misaligned v
    assert _rc("fg_attention_decode_append", *args(pos=None)) == 1
    assert _rc("fg_attention_decode_append", *args(ldkv=128)) == 2     # row stride below heads x head_dim
    assert _rc("fg_attention_decode_append", *args(ldq=260)) == 2      # stride not a multiple of 8
    bad = _fake_kv(maxL=100)                                           # max_len not a multiple of 64
    assert _rc("fg_attention_decode_append", *args(kv=bad)) == 2


def _fake_w4a8(N=256, K=512):
    w = B.fg_w4a8_weight()
    w.codes, w.gmin, w.gstep, w.cscale = 0x100000, 0x200000, 0x300000, 0x400000
    w.N, w.K = N, K
    return w


def test_w4a8_entry_points_validate_on_host():
    P = 0x800000                                            # aligned, never dereferenced
    w = _fake_w4a8()
    lin = lambda **o: [o.get("a8", P), o.get("ascale", P * 2), o.get("M", 8), o.get("K", 512),
                       ctypes.byref(o.get("w", w)), None, o.get("res", None), o.get("flags", 0), 0, 1.0,
                       o.get("y", P * 3), None, 0, None]
    assert _rc("fg_linear_w4a8", *lin(K=448)) == 2                     # K differs from the weight's
    assert _rc("fg_linear_w4a8", *lin(w=_fake_w4a8(K=448), K=448)) == 2  # K not a multiple of 128
    assert _rc("fg_linear_w4a8", *lin(w=_fake_w4a8(K=65536 + 128), K=65536 + 128)) == 2  # int32 sums
    assert _rc("fg_linear_w4a8", *lin(w=_fake_w4a8(N=192))) == 2       # N not a multiple of 128
    assert _rc("fg_linear_w4a8", *lin(M=-1)) == 1
    assert _rc("fg_linear_w4a8", *lin(M=0)) == 0                       # nothing to do
    assert _rc("fg_linear_w4a8", *lin(flags=4)) == 1                   # no persistent launch here
    assert _rc("fg_linear_w4a8", *lin(flags=2)) == 1                   # residual flag without residual
    assert _rc("fg_linear_w4a8", *lin(a8=P + 8)) == 1                  # misaligned activations
    assert _rc("fg_linear_w4a8", *lin(y=None)) == 1
    odd = _fake_w4a8()
    odd.gmin = 0x200001                                                # metadata read 2 bytes at a time
    assert _rc("fg_linear_w4a8", *lin(w=odd)) == 1
    odd = _fake_w4a8()
    odd.cscale = 0x400002                                              # fp32 row scales
    assert _rc("fg_linear_w4a8", *lin(w=odd)) == 1
    assert _rc("fg_linear_w4a8", *lin(ascale=P * 2 + 2)) == 1          # fp32 token scales
    assert _rc("fg_act8_quantize", P, 4, 96, P * 2, P * 3, None) == 2  # K not a multiple of 64
    assert _rc("fg_act8_quantize", P, 0, 128, P * 2, P * 3, None) == 0
    assert _rc("fg_act8_quantize", P + 2, 4, 128, P * 2, P * 3, None) == 1
    assert _rc("fg_w4a8_quantize_weight", P, ctypes.byref(_fake_w4a8(K=96)), None) == 2
    assert _rc("fg_w4a8_quantize_weight", P, ctypes.byref(_fake_w4a8(N=0)), None) == 2
    assert _rc("fg_w4a8_quantize_weight", None, ctypes.byref(w), None) == 1
    t, s = ctypes.c_int(), ctypes.c_int()
    assert B.lib().fg_linear_w4a8_plan(8, 256, 448, ctypes.byref(t), ctypes.byref(s)) == 1


def test_w4a8_layer_config_rules():
    # the W4A8 form of the layer: group 64 only, act_bits 16 (or 0) or 8
    h, H, F = 768, 12, 3072
    w16 = fg.LayerConfig(h, H, F).blob_bytes()
    w8 = fg.LayerConfig(h, H, F, act_bits=8).blob_bytes()
    # per matrix: codes N*K/2, int8 minima and uint8 steps N*K/64 each, fp32 row scales 4N (each
    # array 256-byte aligned) in place of fp16 mins and scales N*K/64 * 2 each
    a = lambda x: (x + 255) // 256 * 256
    mats = [(3 * h, h), (h, h), (F, h), (h, F)]
    vecs = sum(a(n * 2) for n in (3 * h, h, F, h, h, h, h, h))
    assert w16 == sum(a(n * k // 2) + 2 * a(n * k // 64 * 2) for n, k in mats) + vecs
    assert w8 == sum(a(n * k // 2) + 2 * a(n * k // 64) + a(4 * n) for n, k in mats) + vecs
    with pytest.raises(fg.FgError):
        fg.LayerConfig(1024, 8, 4096, group=128, act_bits=8).blob_bytes()
    with pytest.raises(fg.FgError):
        fg.LayerConfig(h, H, F, act_bits=4).blob_bytes()
    assert fg.LayerConfig(h, H, F, act_bits=8).workspace_bytes(16) > fg.LayerConfig(h, H, F).workspace_bytes(16)


def test_stack_one_buffer_bytes():
    # one staging buffer: the blob, then a second slot for the vectors (biases, LayerNorm parameters)
    for act_bits in (16, 8):
        cfg = fg.LayerConfig(768, 12, 3072, act_bits=act_bits)
        c = cfg.struct()
        vec = sum((n * 2 + 255) // 256 * 256 for n in (3 * 768, 768, 3072, 768, 768, 768, 768, 768))
        assert B.lib().fg_stack_one_buffer_bytes(ctypes.byref(c)) == cfg.blob_bytes() + vec
    bad = fg.LayerConfig(768, 12, 3072, act_bits=4).struct()
    assert B.lib().fg_stack_one_buffer_bytes(ctypes.byref(bad)) == 0
