"""GPU parity of the individual kernels against the CPU oracle (through the C ABI).

Bit-exact: quantise (codes, mins, scales), dequantise, KV append.
Tolerance (floating point): attention, W4A16 linear, LayerNorm -- the fp16
output rounding (2^-11 relative) plus fp32 accumulation, checked as
max|gpu - oracle| <= tol * max|oracle|.
"""
import os
import subprocess
import sys

import numpy as np
import pytest
import torch

import oracle
import seeded_inputs as si

pytestmark = pytest.mark.gpu

fg = None


@pytest.fixture(autouse=True)
def _bind_library(fg_lib):
    global fg
    fg = fg_lib


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def host(t):
    return t.cpu().numpy()


def u16(a):
    return np.ascontiguousarray(a).view(np.uint16)


# ------------------------------------------------------------------ quantise ----------

def _check_quant_equal(x16, dim=-1, group=64, bits=4):
    q = fg.fg_quantize(dev(x16), dim=dim, group=group, bits=bits)
    r = oracle.quantize(x16, dim=dim, group=group, bits=bits)
    torch.cuda.synchronize()
    assert np.array_equal(host(q.codes), r.codes)
    assert np.array_equal(u16(host(q.mins)), u16(r.mins))
    assert np.array_equal(u16(host(q.scales)), u16(r.scales))
    y = fg.fg_dequantize(q)
    assert np.array_equal(u16(host(y)), u16(oracle.dequantize(r)))
    return q


@pytest.mark.parametrize("rows,cols", [(1, 64), (3, 128), (17, 4096), (256, 4096), (5, 768 * 4)])
def test_quantize_lastdim_bit_exact(rows, cols):
    _check_quant_equal(si.sweep_tensor(7, rows * cols, row=cols) if cols % 64 == 0 and rows * cols >= 128
                       else si.normal_f16(7, 1, (rows, cols), 0.02))


def test_quantize_sweep_2pow20_bit_exact():
    _check_quant_equal(si.sweep_tensor(0, 1 << 20, row=4096))


def test_quantize_wide_ranges_and_specials():
    rng = np.random.default_rng(5)
    x = (rng.standard_normal((2048, 64)) * 10.0 ** rng.integers(-7, 4, (2048, 1))).astype(np.float16)
    x[0] = 0
    x[1] = -0.0
    x[2] = np.where(np.arange(64) % 3 == 0, np.float16(-0.0), np.float16(0.0))
    x[3] = 65504
    x[4, :32] = -65504
    x[4, 32:] = 65504
    x[5] = np.arange(64)
    _check_quant_equal(x)


def test_quantize_every_fp16_range_bit_exact():
    # one group per positive finite fp16 value v: {0, v} and {-v, v} ranges with the other
    # elements spread between them -- every reachable scale, including the fp16 subnormal
    # ones, goes through the quantizer's division and reciprocal
    v = np.arange(1, 0x7C00, dtype=np.uint16).view(np.float16).astype(np.float64)
    t = np.linspace(0.0, 1.0, 64)
    a = (v[:, None] * t[None, :]).astype(np.float16)                  # min 0, max v
    b = (v[:, None] * (2.0 * t[None, :] - 1.0)).astype(np.float16)    # min -v, max v
    b[:, 0] = (-v).astype(np.float16)
    b[:, -1] = v.astype(np.float16)
    _check_quant_equal(np.concatenate([a, b], axis=0))


@pytest.mark.parametrize("shape,dim", [((6, 128, 5), 1), ((64, 3), 0), ((2, 3, 192, 4), 2)])
def test_quantize_strided_dims_bit_exact(shape, dim):
    _check_quant_equal(si.normal_f16(8, 2, shape, 1.0), dim=dim)


def test_quantize_empty_and_errors():
    x = torch.empty((0, 64), dtype=torch.float16, device="cuda")
    q = fg.fg_quantize(x)
    assert q.codes.numel() == 0
    with pytest.raises(fg.FgError, match="SHAPE"):
        fg.fg_quantize(torch.zeros((2, 96), dtype=torch.float16, device="cuda"))
    for bits in (2, 3, 16):
        with pytest.raises(fg.FgError, match="UNSUPPORTED"):
            fg.fg_quantize(torch.zeros((2, 64), dtype=torch.float16, device="cuda"), bits=bits)


# ------------------------------------------------------------------ 8-bit codes -----
# the same min-max scheme with 255 steps, one code per byte

@pytest.mark.parametrize("rows,cols,group", [(1, 64, 64), (3, 128, 64), (17, 4096, 64), (5, 768 * 4, 64),
                                             (1, 128, 128), (33, 4096, 128), (1000, 384, 128)])
def test_quantize_b8_lastdim_bit_exact(rows, cols, group):
    x = si.sweep_tensor(11, rows * cols, row=cols) if rows * cols >= 4096 else si.normal_f16(11, 1, (rows, cols), 0.02)
    q = _check_quant_equal(x, group=group, bits=8)
    assert tuple(q.codes.shape) == (rows, cols)


def test_quantize_b8_sweep_2pow20_bit_exact():
    _check_quant_equal(si.sweep_tensor(3, 1 << 20, row=4096), bits=8)


def test_quantize_b8_every_fp16_range_bit_exact():
    # every positive finite fp16 range v, from 0 and from -v: every reachable scale (fp16
    # subnormal ones included) through the 8-bit division by 255 and the reciprocal
    v = np.arange(1, 0x7C00, dtype=np.uint16).view(np.float16).astype(np.float64)
    t = np.linspace(0.0, 1.0, 64)
    a = (v[:, None] * t[None, :]).astype(np.float16)
    b = (v[:, None] * (2.0 * t[None, :] - 1.0)).astype(np.float16)
    b[:, 0] = (-v).astype(np.float16)
    b[:, -1] = v.astype(np.float16)
    _check_quant_equal(np.concatenate([a, b], axis=0), bits=8)


def test_quantize_b8_specials():
    x = np.full((6, 64), 3.0, dtype=np.float16)
    x[0] = 0
    x[1] = np.where(np.arange(64) % 3 == 0, np.float16(-0.0), np.float16(0.0))
    x[2] = 65504
    x[3, :32] = -65504
    x[3, 32:] = 65504
    x[4] = np.concatenate([[0.0, 255.0], np.arange(1, 63)]).astype(np.float16)   # step exactly 1
    x[5, :8] = [0.0, 255.0, 0.5, 1.5, 2.5, 3.5, 128.5, 254.5]                  # half-even ties
    q = _check_quant_equal(x, bits=8)
    assert list(host(q.codes)[5, :8]) == [0, 255, 0, 2, 2, 4, 128, 254]


@pytest.mark.parametrize("shape,dim,group", [((6, 128, 5), 1, 64), ((64, 3), 0, 64), ((2, 3, 256, 4), 2, 128)])
def test_quantize_b8_strided_dims_bit_exact(shape, dim, group):
    _check_quant_equal(si.normal_f16(12, 2, shape, 1.0), dim=dim, group=group, bits=8)


def test_linear_rejects_8bit_weights():
    wq = fg.fg_quantize(torch.zeros((256, 256), dtype=torch.float16, device="cuda"), dim=1, bits=8)
    with pytest.raises(fg.FgError, match="UNSUPPORTED"):
        fg.fg_linear_w4a16(torch.zeros((4, 256), dtype=torch.float16, device="cuda"), wq)


@pytest.mark.slow
def test_quantize_2pow30_sampled_bit_exact():
    # full-size sweep point, in the launch the benchmark times; sampled groups checked by the oracle
    n = 1 << 30
    x = si.sweep_tensor(0, n, row=4096)
    q = fg.fg_quantize(dev(x))
    torch.cuda.synchronize()
    G = n // 64
    rng = np.random.default_rng(1)
    sel = np.unique(np.concatenate([[0, 1, 2, G - 1], rng.integers(0, G, 20000)]))
    xs = x.reshape(-1, 64)[sel]
    r = oracle.quantize(xs)
    codes = q.codes.view(-1, 32)[torch.from_numpy(sel).cuda()].cpu().numpy()
    assert np.array_equal(codes, r.codes)
    assert np.array_equal(u16(q.mins.view(-1)[torch.from_numpy(sel).cuda()].cpu().numpy()), u16(r.mins[:, 0]))
    assert np.array_equal(u16(q.scales.view(-1)[torch.from_numpy(sel).cuda()].cpu().numpy()), u16(r.scales[:, 0]))
    y = fg.fg_dequantize(q).view(-1, 64)[torch.from_numpy(sel).cuda()].cpu().numpy()
    assert np.array_equal(u16(y), u16(oracle.dequantize(r)))


# ------------------------------------------------------------------ groups of 128 -----

@pytest.mark.parametrize("rows,cols", [(1, 128), (3, 256), (17, 4096), (5, 768 * 4), (1000, 384)])
def test_quantize_group128_lastdim_bit_exact(rows, cols):
    _check_quant_equal(si.sweep_tensor(9, rows * cols, row=cols) if rows * cols >= 256
                       else si.normal_f16(9, 1, (rows, cols), 0.02), group=128)


def test_quantize_group128_wide_ranges_bit_exact():
    rng = np.random.default_rng(6)
    x = (rng.standard_normal((1024, 128)) * 10.0 ** rng.integers(-7, 4, (1024, 1))).astype(np.float16)
    x[0] = 0
    x[1, :64] = -65504
    x[1, 64:] = 65504
    x[2] = (np.arange(128) / 2).astype(np.float16)
    _check_quant_equal(x, group=128)


@pytest.mark.parametrize("shape,dim", [((6, 256, 5), 1), ((128, 3), 0), ((2, 3, 384, 4), 2)])
def test_quantize_group128_strided_bit_exact(shape, dim):
    _check_quant_equal(si.normal_f16(10, 2, shape, 1.0), dim=dim, group=128)


def test_quantize_group128_errors():
    with pytest.raises(fg.FgError, match="SHAPE"):
        fg.fg_quantize(torch.zeros((2, 192), dtype=torch.float16, device="cuda"), group=128)
    with pytest.raises(fg.FgError, match="UNSUPPORTED"):
        fg.fg_quantize(torch.zeros((2, 192), dtype=torch.float16, device="cuda"), group=96)


@pytest.mark.parametrize("M,N,K", [(7, 256, 1024), (200, 384, 2048), (300, 512, 4096), (600, 640, 2048),
                                   (512, 4096, 4096)])
def test_linear_group128_weights(M, N, K):
    # W4 weights in groups of 128 along K on both GEMM kernels (one SM per tile for M <= 256,
    # CTA pairs above, with k splits for the long-k shapes)
    x = si.normal_f16(19, 1, (M, K), 1.0)
    w16 = si.normal_f16(19, 2, (N, K), 0.02)
    b = si.normal_f16(19, 3, (N,), 0.1)
    r = si.normal_f16(19, 4, (M, N), 1.0)
    wq = fg.fg_quantize(dev(w16), dim=1, group=128)
    wo = oracle.quantize(w16, 1, group=128)
    assert np.array_equal(host(wq.codes), wo.codes)
    y = fg.fg_linear_w4a16(dev(x), wq, bias=dev(b), residual=dev(r))
    rows = np.unique(np.concatenate([np.arange(min(M, 8)), [M // 2, M - 1]]))
    ref = oracle.linear(x[rows], wo, bias=b, residual=r[rows])
    got = host(y)[rows].astype(np.float64)
    assert np.max(np.abs(got - ref)) <= 2e-3 * np.max(np.abs(ref))


# ------------------------------------------------------------------ KV append ---------

@pytest.mark.parametrize("H,d", [(2, 64), (3, 128), (1, 256)])
def test_kv_append_bit_exact(H, d):
    S, maxL = 5, 128
    g = fg.KVCache(S, H, d, maxL)
    o = oracle.KVCache(S, H, d, maxL)
    pos = np.array([0, 7, 63, 64, 127], dtype=np.int32)
    k = si.normal_f16(9, 1, (S, 3 * H * d), 1.0)      # rows with a stride, like the QKV buffer
    kk, vv = k[:, H * d:2 * H * d], k[:, 2 * H * d:]
    kd = dev(k)
    fg.fg_kv_append(g, kd[:, H * d:], kd[:, 2 * H * d:], dev(pos), ld=3 * H * d)
    oracle.kv_append(o, kk, vv, np.arange(S), pos)
    fg.fg_sync_status()
    for a, b in zip(g.arrays(), o.arrays()):
        assert np.array_equal(u16(host(a)) if a.dtype == torch.float16 else host(a), b)


@pytest.mark.parametrize("H,d", [(3, 128), (2, 256)])
def test_kv_append_group128_bit_exact(H, d):
    # head_dim quantised in groups of 128 ("FlexGen Guide", section 3: groups of 64 or 128)
    S, maxL = 4, 128
    g = fg.KVCache(S, H, d, maxL, group=128)
    o = oracle.KVCache(S, H, d, maxL, group=128)
    pos = np.array([0, 63, 64, 127], dtype=np.int32)
    k = si.normal_f16(26, 1, (S, 3 * H * d), 1.0)
    kd = dev(k)
    fg.fg_kv_append(g, kd[:, H * d:], kd[:, 2 * H * d:], dev(pos), ld=3 * H * d)
    oracle.kv_append(o, k[:, H * d:2 * H * d], k[:, 2 * H * d:], np.arange(S), pos)
    fg.fg_sync_status()
    for a, b in zip(g.arrays(), o.arrays()):
        assert np.array_equal(u16(host(a)) if a.dtype == torch.float16 else host(a), b)


@pytest.mark.parametrize("H,d,P", [(2, 128, 1), (2, 256, 1), (3, 128, 90)])
def test_attention_group128_matches_oracle(H, d, P):
    # decode rows (P = 1) through the row kernel, prompt rows through the tiled prefill kernel
    # (head_dim 128), the cache in groups of 128 along head_dim
    S = 3
    starts = np.array([0, 70, 200], dtype=np.int32)
    lens = starts + P
    maxL = int((lens.max() + 63) // 64 * 64)
    o, g = _cache_pair(S, H, d, maxL, lens, seed=27, group=128)
    _garbage_past(g, lens, 28)
    q = (si.normal_f16(27, 1, (S * P, H * d), 1.0).astype(np.float32) / np.sqrt(d)).astype(np.float16)
    out = fg.fg_attention_decode(g, dev(q), dev(starts), rows_per_seq=P)
    fg.fg_sync_status()
    seq = np.repeat(np.arange(S), P)
    ref = oracle.attention(o, q, seq, starts[seq] + np.tile(np.arange(P), S) + 1)
    got = host(out).astype(np.float64)
    for h in range(H):
        sl = slice(h * d, (h + 1) * d)
        err = np.max(np.abs(got[:, sl] - ref[:, sl]), axis=1)
        assert np.all(err <= 2e-3 * np.max(np.abs(ref[:, sl]), axis=1) + 1e-4), (h, err.max())


def test_kv_append_prompt_rows_and_range_error():
    S, H, d, maxL, P = 3, 2, 128, 64, 10
    g = fg.KVCache(S, H, d, maxL)
    o = oracle.KVCache(S, H, d, maxL)
    k = si.normal_f16(10, 1, (S * P, H * d), 1.0)
    v = si.normal_f16(10, 2, (S * P, H * d), 1.0)
    start = np.array([0, 5, 58], dtype=np.int32)        # the last sequence runs past max_len (58+9 > 63)
    fg.fg_kv_append(g, dev(k), dev(v), dev(start), rows_per_seq=P)
    with pytest.raises(fg.FgError, match="RANGE"):
        fg.fg_sync_status()
    fg.fg_sync_status()                                  # the error word was cleared
    seq = np.repeat(np.arange(S), P)
    pos = start[seq] + np.tile(np.arange(P), S)
    ok = pos < maxL
    oracle.kv_append(o, k[ok], v[ok], seq[ok], pos[ok])
    for a, b in zip(g.arrays(), o.arrays()):
        assert np.array_equal(u16(host(a)) if a.dtype == torch.float16 else host(a), b)


# ------------------------------------------------------------------ attention ---------

def _cache_pair(S, H, d, maxL, lens, seed, group=64):
    o = oracle.KVCache(S, H, d, maxL, group=group)
    for s in range(S):
        L = lens[s]
        k = si.normal_f16(seed, 100 + s, (L, H * d), 1.0)
        v = si.normal_f16(seed, 200 + s, (L, H * d), 1.0)
        oracle.kv_append(o, k, v, np.full(L, s), np.arange(L))
    arrays = [dev(a.view(np.float16) if a.dtype == np.uint16 else a) for a in o.arrays()]
    return o, fg.KVCache(S, H, d, maxL, arrays=arrays, group=group)


@pytest.mark.parametrize("H,d", [(4, 64), (3, 128), (2, 256)])
def test_attention_decode_matches_oracle(H, d):
    S, maxL = 6, 320
    lens = np.array([1, 2, 63, 64, 65, 300], dtype=np.int32)   # ragged: 1 token, chunk edges, several chunks
    o, g = _cache_pair(S, H, d, maxL, lens, seed=11)
    q = (si.normal_f16(11, 1, (S, H * d), 1.0).astype(np.float32) / np.sqrt(d)).astype(np.float16)
    out = fg.fg_attention_decode(g, dev(q), dev(lens - 1))
    ref = oracle.attention(o, q, np.arange(S), lens)
    got = host(out).astype(np.float64)
    for s in range(S):
        for h in range(H):
            sl = slice(h * d, (h + 1) * d)
            err = np.max(np.abs(got[s, sl] - ref[s, sl]))
            assert err <= 2e-3 * np.max(np.abs(ref[s, sl])) + 1e-4, (s, h, err)


def _seeded_cache(S, H, d, maxL, lens, seed, group):
    """Oracle cache with lens[s] tokens per sequence (0 allowed), and its device copy."""
    o = oracle.KVCache(S, H, d, maxL, group=group)
    for s in range(S):
        L = int(lens[s])
        if L:
            k = si.normal_f16(seed, 100 + s, (L, H * d), 1.0)
            v = si.normal_f16(seed, 200 + s, (L, H * d), 1.0)
            oracle.kv_append(o, k, v, np.full(L, s), np.arange(L))
    arrays = [dev(a.view(np.float16) if a.dtype == np.uint16 else a) for a in o.arrays()]
    return o, fg.KVCache(S, H, d, maxL, arrays=arrays, group=group)


@pytest.mark.parametrize("H,d,group", [(4, 64, 64), (3, 128, 64), (2, 256, 64), (3, 128, 128), (2, 256, 128)])
def test_attention_decode_append_fused(H, d, group):
    # One launch appends each sequence's new k, v row and attends over the cache with it.
    # New rows inside the first chunks the kernel streams (positions < 256) and past them;
    # garbage in every slot from the new position on (the append must overwrite it, the
    # attention must not read beyond it).  The cache must hold the oracle's append bits,
    # the output must equal the append-then-attend launches bit for bit and the oracle's
    # attention within the decode-attention tolerance.
    S, maxL = 8, 384
    pos = np.array([0, 1, 63, 127, 128, 255, 256, 300], dtype=np.int32)
    o, g = _seeded_cache(S, H, d, maxL, pos, seed=31 + d + group, group=group)
    _garbage_past(g, pos, 32)
    g2 = fg.KVCache(S, H, d, maxL, arrays=[a.clone() for a in g.arrays()], group=group)
    Hd = H * d
    qkv = si.normal_f16(33, 1, (S, 3 * Hd), 1.0)
    qkv[:, :Hd] = (qkv[:, :Hd].astype(np.float32) / np.sqrt(d)).astype(np.float16)
    qd, pd = dev(qkv), dev(pos)
    out = fg.fg_attention_decode_append(g, qd[:, :Hd], qd[:, Hd:2 * Hd], qd[:, 2 * Hd:], pd)
    fg.fg_kv_append(g2, qd[:, Hd:2 * Hd], qd[:, 2 * Hd:], pd, ld=3 * Hd)
    out2 = fg.fg_attention_decode(g2, qd[:, :Hd], pd)
    fg.fg_sync_status()
    assert torch.equal(out, out2)
    for a, b in zip(g.arrays(), g2.arrays()):   # bytes: the planted garbage holds NaNs
        assert torch.equal(a.view(torch.uint8), b.view(torch.uint8))
    oracle.kv_append(o, qkv[:, Hd:2 * Hd], qkv[:, 2 * Hd:], np.arange(S), pos)
    for a, b in zip(g.arrays(), o.arrays()):
        ha = u16(host(a)) if a.dtype == torch.float16 else host(a)
        for s in range(S):
            assert np.array_equal(ha[s, :, :pos[s] + 1], b[s, :, :pos[s] + 1]), s
    ref = oracle.attention(o, qkv[:, :Hd], np.arange(S), pos + 1)
    got = host(out).astype(np.float64)
    for s in range(S):
        for h in range(H):
            sl = slice(h * d, (h + 1) * d)
            err = np.max(np.abs(got[s, sl] - ref[s, sl]))
            assert err <= 2e-3 * np.max(np.abs(ref[s, sl])) + 1e-4, (s, h, err)


def test_attention_decode_append_range_error():
    # a position at max_len: nothing appended for that sequence, zeros out, FG_ERR_RANGE;
    # the other sequences are appended and attended as usual
    S, H, d, maxL = 3, 2, 128, 128
    pos = np.array([5, 128, 127], dtype=np.int32)
    o, g = _seeded_cache(S, H, d, maxL, np.minimum(pos, maxL), seed=34, group=64)
    before = [a.clone() for a in g.arrays()]
    qkv = si.normal_f16(35, 1, (S, 3 * H * d), 1.0)
    qd = dev(qkv)
    Hd = H * d
    out = fg.fg_attention_decode_append(g, qd[:, :Hd], qd[:, Hd:2 * Hd], qd[:, 2 * Hd:], dev(pos))
    with pytest.raises(fg.FgError, match="RANGE"):
        fg.fg_sync_status()
    assert not host(out)[1].any()
    for a, b in zip(g.arrays(), before):
        assert torch.equal(a[1].view(torch.uint8), b[1].view(torch.uint8))   # sequence 1 untouched
    ok = pos < maxL
    oracle.kv_append(o, qkv[ok, Hd:2 * Hd], qkv[ok, 2 * Hd:], np.arange(S)[ok], pos[ok])
    for a, b in zip(g.arrays(), o.arrays()):
        ha = u16(host(a)) if a.dtype == torch.float16 else host(a)
        assert np.array_equal(ha[[0, 2]], b[[0, 2]])


def test_attention_peaked_scores():
    # large query norms make the softmax nearly one-hot: catches masking and max handling
    S, H, d, maxL = 2, 2, 128, 256
    lens = np.array([130, 200], dtype=np.int32)
    o, g = _cache_pair(S, H, d, maxL, lens, seed=12)
    q = si.normal_f16(12, 1, (S, H * d), 3.0)
    out = fg.fg_attention_decode(g, dev(q), dev(lens - 1))
    ref = oracle.attention(o, q, np.arange(S), lens)
    assert np.max(np.abs(host(out).astype(np.float64) - ref)) <= 5e-3 * np.max(np.abs(ref))


def test_attention_prompt_rows_causal():
    S, H, d, maxL, P = 2, 2, 128, 128, 70
    lens = np.array([P, P], dtype=np.int32)
    o, g = _cache_pair(S, H, d, maxL, lens, seed=13)
    q = (si.normal_f16(13, 1, (S * P, H * d), 1.0).astype(np.float32) / np.sqrt(d)).astype(np.float16)
    out = fg.fg_attention_decode(g, dev(q), dev(np.zeros(S, np.int32)), rows_per_seq=P)
    seq = np.repeat(np.arange(S), P)
    ref = oracle.attention(o, q, seq, np.tile(np.arange(P), S) + 1)
    assert np.max(np.abs(host(out).astype(np.float64) - ref)) <= 2e-3 * np.max(np.abs(ref))


def _garbage_past(g, lens, seed):
    """Random bytes (NaN and inf metadata included) in every cache slot at or past each
    sequence's length: attention must never let them reach its output."""
    gen = torch.Generator(device="cuda").manual_seed(seed)
    for a in g.arrays():
        u8 = a.view(torch.uint8)
        noise = torch.randint(0, 256, u8.shape, dtype=torch.uint8, device="cuda", generator=gen)
        for s, L in enumerate(lens):
            u8[s, :, L:] = noise[s, :, L:]


@pytest.mark.parametrize("H,d,P", [(2, 128, 70), (3, 64, 130), (1, 128, 512), (2, 64, 17), (2, 256, 40)])
def test_attention_prefill_tiles_match_oracle(H, d, P):
    # prompt rows through the tiled prefill kernel (head_dim 64 / 128; 256 takes the row kernel):
    # sequences that start at position 0 and sequences that continue an earlier prompt
    # (positions 5 and 64), prompt lengths that end mid-tile, garbage in the slots past them
    S = 3
    starts = np.array([0, 5, 64], dtype=np.int32)
    lens = starts + P
    maxL = int((lens.max() + 63) // 64 * 64)
    o, g = _cache_pair(S, H, d, maxL, lens, seed=30 + d)
    _garbage_past(g, lens, 31)
    q = (si.normal_f16(30, 1, (S * P, H * d), 1.0).astype(np.float32) / np.sqrt(d)).astype(np.float16)
    out = fg.fg_attention_decode(g, dev(q), dev(starts), rows_per_seq=P)
    fg.fg_sync_status()
    seq = np.repeat(np.arange(S), P)
    ref = oracle.attention(o, q, seq, starts[seq] + np.tile(np.arange(P), S) + 1)
    got = host(out).astype(np.float64)
    for h in range(H):
        sl = slice(h * d, (h + 1) * d)
        err = np.max(np.abs(got[:, sl] - ref[:, sl]), axis=1)
        assert np.all(err <= 2e-3 * np.max(np.abs(ref[:, sl]), axis=1) + 1e-4), (h, err.max())


@pytest.mark.parametrize("prompt", [False, True])
def test_attention_mixed_token_magnitudes(prompt):
    # K and V rows whose magnitudes span 1e-3 .. 1e1 from token to token (groups with very
    # small and very large scales side by side, scores spread over hundreds of log units),
    # through the decode and the prefill kernels.  The decode kernel multiplies fp16 operands
    # without forming the dequantised fp16 K/V value (its p * scale operand is the fp16 one
    # under test here), so it is held to the oracle's exact-dequantisation form; the prefill
    # kernel dequantises to fp16 like the layer's reading and is held to that form.
    S, H, d = 2, 2, 128
    P = 96 if prompt else 1
    lens = np.array([150, 200], dtype=np.int32) if not prompt else np.array([P, P + 40], dtype=np.int32)
    maxL = 256
    o = oracle.KVCache(S, H, d, maxL)
    rng = np.random.default_rng(41)
    for s in range(S):
        L = int(lens[s])
        mag = 10.0 ** rng.uniform(-3, 1, size=(L, 1))
        k = (si.normal_f16(41, 100 + s, (L, H * d), 1.0).astype(np.float64) * mag).astype(np.float16)
        v = (si.normal_f16(41, 200 + s, (L, H * d), 1.0).astype(np.float64) * mag).astype(np.float16)
        oracle.kv_append(o, k, v, np.full(L, s), np.arange(L))
    g = fg.KVCache(S, H, d, maxL, arrays=[dev(a.view(np.float16) if a.dtype == np.uint16 else a) for a in o.arrays()])
    starts = lens - P
    q = (si.normal_f16(41, 1, (S * P, H * d), 0.3).astype(np.float32)).astype(np.float16)
    out = fg.fg_attention_decode(g, dev(q), dev(starts.astype(np.int32)), rows_per_seq=P)
    fg.fg_sync_status()
    seq = np.repeat(np.arange(S), P)
    ref = oracle.attention(o, q, seq, starts[seq] + np.tile(np.arange(P), S) + 1, exact_dequant=not prompt)
    got = host(out).astype(np.float64)
    for h in range(H):
        sl = slice(h * d, (h + 1) * d)
        err = np.max(np.abs(got[:, sl] - ref[:, sl]), axis=1)
        assert np.all(err <= 2e-3 * np.max(np.abs(ref[:, sl]), axis=1) + 1e-4), (h, err.max())


# ------------------------------------------------------------------ linear -------------

@pytest.mark.parametrize("M,N,K", [(1, 128, 64), (4, 256, 768), (16, 384, 128), (17, 256, 192), (100, 512, 1024),
                                   (256, 768, 768), (300, 1280, 512), (512, 2304, 768), (40, 768, 3072),
                                   # M > 256: two-SM (CTA pair) tiles of 256 features x 512 tokens, with a
                                   # ragged last token tile, a last pair holding only 128 features, and
                                   # (long k) the split-k cluster reduction
                                   (257, 256, 128), (600, 640, 2048), (1100, 384, 1024), (520, 640, 4096)])
def test_linear_matches_oracle(M, N, K):
    x = si.normal_f16(14, 1, (M, K), 1.0)
    w16 = si.normal_f16(14, 2, (N, K), 0.02)
    b = si.normal_f16(14, 3, (N,), 0.1)
    wq = fg.fg_quantize(dev(w16), dim=1)
    ref = oracle.linear(x, oracle.quantize(w16, 1), bias=b)
    # the classic launch with its scratch; for M > 256 also without scratch (partial sums added
    # on chip) and the persistent launch where it is available
    runs = [dict()]
    if M > 256:
        runs.append(dict(workspace=torch.empty(16, dtype=torch.uint8, device="cuda")))
        if fg.fg_linear_plan_pairs(M, N, K) > 0:
            runs.append(dict(persistent=True))
    for kw in runs:
        y = fg.fg_linear_w4a16(dev(x), wq, bias=dev(b), **kw)
        err = np.max(np.abs(host(y).astype(np.float64) - ref))
        assert err <= 2e-3 * np.max(np.abs(ref)), (err, kw)


@pytest.mark.parametrize("M,K", [(70, 256), (300, 256), (300, 2048)])
def test_linear_epilogues(M, K):
    N = 512
    x = si.normal_f16(15, 1, (M, K), 1.0)
    w16 = si.normal_f16(15, 2, (N, K), 0.05)
    b = si.normal_f16(15, 3, (N,), 0.1)
    r = si.normal_f16(15, 4, (M, N), 1.0)
    wq = fg.fg_quantize(dev(w16), dim=1)
    wo = oracle.quantize(w16, 1)
    for kw, okw in [(dict(relu=True), dict(relu=True)), (dict(residual=dev(r)), dict(residual=r)),
                    (dict(qscale_cols=128, qscale=0.125), dict(qscale_cols=128, qscale=0.125))]:
        y = fg.fg_linear_w4a16(dev(x), wq, bias=dev(b), **kw)
        ref = oracle.linear(x, wo, bias=b, **okw)
        assert np.max(np.abs(host(y).astype(np.float64) - ref)) <= 2e-3 * np.max(np.abs(ref)), kw


def test_bounded_wait_timeout_is_reported_and_the_gpu_stays_usable():
    # Failure detection without a GPU fault: one launch of the one-SM GEMM (a CTA on each of
    # 148 SMs) whose dequantising warps withhold their first-stage arrival, with every pipeline
    # wait limited to 50 ms.  The MMA issuer's wait gives up, the launch drains its copies,
    # frees its tensor memory and flags FG_ERR_TIMEOUT; the same GEMM then runs normally on
    # every SM and matches the oracle.
    M, N, K = 16, 148 * 256, 512
    x = si.normal_f16(23, 1, (M, K), 1.0)
    w16 = si.normal_f16(23, 2, (N, K), 0.02)
    wq = fg.fg_quantize(dev(w16), dim=1)
    assert fg.fg_linear_plan(M, N, K) == (16, 1)
    xd = dev(x)
    y = torch.empty((M, N), dtype=torch.float16, device="cuda")
    fg.fg_sync_status()
    fg.fg_test_gemm_stall(1, 50_000_000)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    fg.fg_linear_w4a16(xd, wq, out=y)
    e1.record()
    with pytest.raises(fg.FgError, match="TIMEOUT"):
        fg.fg_sync_status()
    assert 40.0 <= e0.elapsed_time(e1) < 1000.0          # gave up after about the 50 ms limit
    fg.fg_sync_status()                                  # the error word was cleared
    y = fg.fg_linear_w4a16(xd, wq, out=y)
    fg.fg_sync_status()
    ref = oracle.linear(x, oracle.quantize(w16, 1))
    assert np.max(np.abs(host(y).astype(np.float64) - ref)) <= 2e-3 * np.max(np.abs(ref))


def test_linear_permutation_weight_exact():
    # weights {0, 15} per group are stored exactly; y = 15 * x[:, cols] + b up to the fp16 output rounding
    M, N, K = 33, 256, 512
    cols = np.random.default_rng(2).integers(0, K, N)
    w16 = np.zeros((N, K), np.float16)
    w16[np.arange(N), cols] = 15
    x = si.normal_f16(16, 1, (M, K), 1.0)
    y = fg.fg_linear_w4a16(dev(x), fg.fg_quantize(dev(w16), dim=1))
    assert np.array_equal(host(y), (15.0 * x.astype(np.float64)[:, cols]).astype(np.float16))


@pytest.mark.parametrize("M,N,K", [(8, 256, 8192), (512, 4096, 4096), (40, 384, 16384)])
def test_linear_split_k_deterministic(M, N, K):
    # few output tiles and a long k-range take the cluster split-k path; two runs give identical bits
    xs = si.normal_f16(17, 1, (M, K), 1.0)
    x = dev(xs)
    w16 = si.normal_f16(17, 2, (N, K), 0.02)
    wq = fg.fg_quantize(dev(w16), dim=1)
    y1 = fg.fg_linear_w4a16(x, wq)
    y2 = fg.fg_linear_w4a16(x, wq)
    assert torch.equal(y1, y2)
    ref = oracle.linear(xs, oracle.quantize(w16, 1))
    assert np.max(np.abs(host(y1).astype(np.float64) - ref)) <= 2e-3 * np.max(np.abs(ref))
    if M <= 256:
        assert fg.fg_linear_workspace_bytes(M, N, K) == 0   # one-SM tiles add partials on chip
    else:
        # CTA pairs: the classic launch's split k-range through the scratch (L2) and on chip
        # (no scratch) add the splits in the same order: the same bits
        assert fg.fg_linear_workspace_bytes(M, N, K) > 0
        y3 = fg.fg_linear_w4a16(x, wq, workspace=torch.empty(16, dtype=torch.uint8, device="cuda"))
        assert torch.equal(y1, y3)
        cb = fg.fg_linear_classic_scratch_bytes(M, N, K)
        if cb:
            # partials and flags (split ranks as separate clusters when the grid is one wave),
            # and partials only (split ranks in one cluster): the same bits again
            y4 = fg.fg_linear_w4a16(x, wq, workspace=torch.empty(cb, dtype=torch.uint8, device="cuda"))
            assert torch.equal(y1, y4)
            cp = fg.fg_linear_classic_scratch_bytes(M, N, K, flags=False)
            y5 = fg.fg_linear_w4a16(x, wq, workspace=torch.empty(cp, dtype=torch.uint8, device="cuda"))
            assert torch.equal(y1, y5)


@pytest.mark.parametrize("M,N,K", [(520, 4096, 4096), (600, 7680, 1024), (530, 5120, 1536), (512, 4096, 16384)])
def test_linear_split_k_residual_sampled(M, N, K):
    # output-projection / FC2 shapes with a residual: few CTA-pair tiles, so the k-range is
    # split over a cluster and the partial sums are pushed between ranks; two runs give
    # identical bits, and sampled rows (the oracle is slow at this size) match the oracle
    x = si.normal_f16(18, 1, (M, K), 1.0)
    w16 = si.normal_f16(18, 2, (N, K), 0.02)
    b = si.normal_f16(18, 3, (N,), 0.1)
    r = si.normal_f16(18, 4, (M, N), 1.0)
    wq = fg.fg_quantize(dev(w16), dim=1)
    y1 = fg.fg_linear_w4a16(dev(x), wq, bias=dev(b), residual=dev(r))
    y2 = fg.fg_linear_w4a16(dev(x), wq, bias=dev(b), residual=dev(r))
    assert torch.equal(y1, y2)
    if K >= 4096:
        assert fg.fg_linear_workspace_bytes(M, N, K) > 0        # these shapes split the k-range
    outs = [y1]
    if fg.fg_linear_classic_scratch_bytes(M, N, K):
        # partial sums through the scratch (above: the split ranks as separate clusters meeting
        # through flags when the grid is one wave), through the scratch within one cluster, or,
        # with too little scratch, on chip over distributed shared memory: the same order of
        # additions, the same bits
        y3 = fg.fg_linear_w4a16(dev(x), wq, bias=dev(b), residual=dev(r),
                                workspace=torch.empty(16, dtype=torch.uint8, device="cuda"))
        assert torch.equal(y1, y3)
        cp = fg.fg_linear_classic_scratch_bytes(M, N, K, flags=False)
        y4 = fg.fg_linear_w4a16(dev(x), wq, bias=dev(b), residual=dev(r),
                                workspace=torch.empty(cp, dtype=torch.uint8, device="cuda"))
        assert torch.equal(y1, y4)
    if fg.fg_linear_plan_pairs(M, N, K) > 0:
        outs.append(fg.fg_linear_w4a16(dev(x), wq, bias=dev(b), residual=dev(r), persistent=True))
    rows = np.unique(np.concatenate([np.random.default_rng(M).choice(M, 20, replace=False), [0, 255, 256, 511, M - 1]]))
    ref = oracle.linear(x[rows], oracle.quantize(w16, 1), bias=b, residual=r[rows])
    for y in outs:
        got = host(y)[rows].astype(np.float64)
        assert np.max(np.abs(got - ref)) <= 2e-3 * np.max(np.abs(ref))


@pytest.mark.parametrize("M,N,K,epi", [
    (512, 12288, 4096, "qscale"),      # QKV of the OPT-6.7B block: 48 tiles over the pairs, split tiles
    (512, 4096, 4096, "residual"),     # output projection: every tile split between several pairs
    (512, 16384, 4096, "relu"),        # FC1
    (512, 4096, 16384, "residual"),    # FC2: long k-ranges
    (700, 12288, 4096, "relu"),        # a ragged second token tile
    (513, 4224, 4096, "none"),         # a last feature pair holding 128 features, 2 token tiles
    (4096, 2048, 1024, "residual"),    # many whole tiles per pair (a prompt-sized M)
])
def test_linear_persistent_launch_matches_oracle(M, N, K, epi):
    # the persistent stream-K launch (FG_GEMM_PERSISTENT with the full scratch): whole tiles,
    # split tiles finished by the pair holding their first k-segment, every epilogue;
    # deterministic, and sampled rows against the oracle
    assert fg.fg_linear_plan_pairs(M, N, K) > 0
    x = si.normal_f16(24, 1, (M, K), 1.0)
    w16 = si.normal_f16(24, 2, (N, K), 0.02)
    b = si.normal_f16(24, 3, (N,), 0.1)
    r = si.normal_f16(24, 4, (M, N), 1.0)
    wq = fg.fg_quantize(dev(w16), dim=1)
    kw = {"qscale": dict(qscale_cols=N // 3, qscale=0.125), "residual": dict(residual=dev(r)),
          "relu": dict(relu=True), "none": {}}[epi]
    okw = {"qscale": dict(qscale_cols=N // 3, qscale=0.125), "residual": dict(residual=r),
           "relu": dict(relu=True), "none": {}}[epi]
    y1 = fg.fg_linear_w4a16(dev(x), wq, bias=dev(b), persistent=True, **kw)
    y2 = fg.fg_linear_w4a16(dev(x), wq, bias=dev(b), persistent=True, **kw)
    fg.fg_sync_status()
    assert torch.equal(y1, y2)
    rows = np.unique(np.concatenate([np.random.default_rng(M + N).choice(M, 24, replace=False),
                                     [0, 255, 256, 511, M - 1]]))
    okw_rows = dict(okw)
    if "residual" in okw_rows:
        okw_rows["residual"] = r[rows]
    ref = oracle.linear(x[rows], oracle.quantize(w16, 1), bias=b, **okw_rows)
    got = host(y1)[rows].astype(np.float64)
    assert np.max(np.abs(got - ref)) <= 2e-3 * np.max(np.abs(ref))


def test_linear_persistent_launch_group128():
    M, N, K = 512, 4096, 4096
    assert fg.fg_linear_plan_pairs(M, N, K) > 0
    x = si.normal_f16(25, 1, (M, K), 1.0)
    w16 = si.normal_f16(25, 2, (N, K), 0.02)
    wq = fg.fg_quantize(dev(w16), dim=1, group=128)
    y = fg.fg_linear_w4a16(dev(x), wq, persistent=True)
    rows = np.array([0, 100, 300, 511])
    ref = oracle.linear(x[rows], oracle.quantize(w16, 1, group=128))
    assert np.max(np.abs(host(y)[rows].astype(np.float64) - ref)) <= 2e-3 * np.max(np.abs(ref))


def test_linear_errors():
    x = torch.zeros((4, 64), dtype=torch.float16, device="cuda")
    w = fg.fg_quantize(torch.zeros((64, 64), dtype=torch.float16, device="cuda"), dim=1)
    with pytest.raises(fg.FgError, match="SHAPE"):
        fg.fg_linear_w4a16(x, w)                             # N = 64 is not a multiple of 128


# ------------------------------------------------------------------ layernorm ----------

@pytest.mark.parametrize("M,h", [(1, 768), (7, 4096), (3, 12288), (5, 64)])
def test_layernorm_matches_oracle(M, h):
    x = si.normal_f16(18, 1, (M, h), 1.0)
    g = (1 + si.normal_f16(18, 2, (h,), 0.1).astype(np.float32)).astype(np.float16)
    b = si.normal_f16(18, 3, (h,), 0.1)
    y = fg.fg_layernorm(dev(x), dev(g), dev(b))
    ref = oracle.layernorm(x, g, b)
    assert np.max(np.abs(host(y).astype(np.float64) - ref)) <= 2e-3 * np.max(np.abs(ref))


def test_linear_plan_in_a_fresh_process_before_any_launch():
    # the split-k plan (and so the scratch size) must not depend on whether a GEMM has run in
    # the process yet: query it first thing in a new interpreter, then after a launch
    code = (
        "import torch, bit_compressed_decode_b200 as fg\n"
        "torch.cuda.init()\n"
        "a = fg.fg_linear_workspace_bytes(512, 4096, 4096)\n"
        "x = torch.zeros((512, 4096), dtype=torch.float16, device='cuda')\n"
        "w = fg.fg_quantize(torch.zeros((4096, 4096), dtype=torch.float16, device='cuda'), dim=1)\n"
        "fg.fg_linear_w4a16(x, w)\n"
        "torch.cuda.synchronize()\n"
        "print(a, fg.fg_linear_workspace_bytes(512, 4096, 4096))\n")
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    out = subprocess.run([sys.executable, "-c", code], cwd=root, capture_output=True, text=True, timeout=300)
    assert out.returncode == 0, out.stderr[-2000:]
    before, after = map(int, out.stdout.split()[-2:])
    assert before == after > 0


def test_linear_parity_shapes_cover_every_pair_plan():
    # the shapes the parity tests above run reach both pair tile sizes (256 and 512 tokens),
    # each with and without a k split
    shapes = [(257, 256, 128), (600, 640, 2048), (1100, 384, 1024), (520, 640, 4096), (300, 512, 256),
              (300, 512, 2048), (512, 4096, 4096), (520, 4096, 4096), (600, 7680, 1024), (530, 5120, 1536),
              (512, 4096, 16384), (512, 2304, 768), (300, 1280, 512)]
    plans = {(M, N, K): fg.fg_linear_plan(M, N, K) for M, N, K in shapes}
    seen = {(t, s > 1) for t, s in plans.values()}
    for want in [(256, False), (256, True), (512, False), (512, True)]:
        assert want in seen, (want, plans)
