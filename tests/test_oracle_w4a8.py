"""Pins of the oracle's W4A8 path (CPU only).

The pages name W4A8 only through the QServe W4A8KV4 title in the PIPO paper's references and the
INT8/INT4 formats of the "Optimizing LLM for low memory usage" page (Quantization and Weight
Compression); the scheme itself is a reading, stated in ``oracle/fg_oracle.c``.  Nothing here
compares the oracle with itself: the expected values are hand-derived fixtures (tests/golden),
exhaustive integer invariants of the scheme, closed forms, numpy's integer matrix product as an
independent check of the oracle's accumulation loop, and -- for the W4A8 layer -- the OPT layer's
wiring written out in Python from those pinned pieces.
"""
import json
import os

import numpy as np
import pytest

import oracle


def _load(golden_dir, name):
    with open(os.path.join(golden_dir, name)) as f:
        return json.load(f)


def _nib(codes):
    b = np.asarray(codes, dtype=np.uint8)
    out = np.empty(b.shape[:-1] + (b.shape[-1] * 2,), dtype=np.int64)
    out[..., 0::2] = b & 15
    out[..., 1::2] = b >> 4
    return out


# ------------------------------------------------------------------ weights -------------

def test_w4a8_ramp_row_golden(golden_dir):
    g = _load(golden_dir, "w4a8_ramp_row.json")
    w = (np.arange(64) - 32).astype(np.float16)[None, :]
    q = oracle.w4a8_quantize_weight(w)
    assert q.gmin[0, 0] == g["gmin"] and q.gstep[0, 0] == g["gstep"]
    assert q.cscale[0] == np.float32(g["cscale_num"]) / np.float32(g["cscale_den"])
    codes = _nib(q.codes)[0]
    w8 = oracle.w4a8_weight_int8(q)[0]
    for k, c, wi in zip(g["ks"], g["codes"], g["int8_weight"]):
        assert codes[k] == c, k
        assert w8[k] == wi, k


def test_w4a8_tie_groups_golden(golden_dir):
    g = _load(golden_dir, "w4a8_tie_groups.json")
    row = np.zeros(128, np.float16)
    row[0] = 113
    head = g["input_group1_head"]
    row[64:64 + len(head)] = head
    row[64 + len(head):] = g["input_group1_tail_value"]
    q = oracle.w4a8_quantize_weight(row[None, :])
    assert q.cscale[0] == np.float32(g["cscale"])
    assert list(q.gmin[0]) == g["gmin"] and list(q.gstep[0]) == g["gstep"]
    codes = _nib(q.codes)[0]
    assert list(codes[:2]) == g["group0_codes_head"]
    assert list(codes[64:64 + len(head)]) == g["group1_codes_head"]
    assert np.all(codes[64 + len(head):] == g["group1_code_tail"])
    w8 = oracle.w4a8_weight_int8(q)[0]
    assert list(w8[64:64 + len(head)]) == g["group1_int8_head"]


def _exhaustive_rows():
    """Every integer group (mn, mx) with -113 <= mn <= mx <= 113 and every value between them,
    laid out as groups of 64: each group holds mn, mx and up to 62 values of [mn, mx]; every row
    starts with a group holding +-113 so that amax = 113 (inv = 1, cscale = 1) and w8 = x."""
    groups, vals = [], []
    for mn in range(-113, 114):
        for mx in range(mn, 114):
            span = list(range(mn, mx + 1))
            for i in range(0, len(span), 62):
                chunk = span[i:i + 62]
                chunk = chunk + [mn] * (62 - len(chunk))
                groups.append([mn, mx] + chunk)
    per_row = 1000
    rows = []
    for r0 in range(0, len(groups), per_row):
        gs = groups[r0:r0 + per_row]
        gs = gs + [[0] * 64] * (per_row - len(gs))
        setter = [113] + [-113] + [0] * 62
        rows.append(np.array([setter] + gs, dtype=np.int64).reshape(-1))
    return np.stack(rows), len(groups)


def test_w4a8_level2_every_integer_group():
    x, ngroups = _exhaustive_rows()
    q = oracle.w4a8_quantize_weight(x.astype(np.float16))
    assert np.all(q.cscale == np.float32(1.0))
    w8 = oracle.w4a8_weight_int8(q).astype(np.int64)        # the oracle refuses values outside int8
    G = x.reshape(x.shape[0], -1, 64)[:, 1:, :]            # drop the amax setter groups
    W = w8.reshape(x.shape[0], -1, 64)[:, 1:, :]
    mn, mx = G.min(axis=2), G.max(axis=2)
    step = q.gstep.astype(np.int64)[:, 1:]
    assert np.all(q.gmin.astype(np.int64)[:, 1:] == mn)
    # the step is the smallest one whose 16 levels span the group, and every value is within
    # half a step of its 8-bit weight
    assert np.all(15 * step >= mx - mn)
    assert np.all((step == 1) | (15 * (step - 1) < mx - mn))
    err = np.abs(W - G)
    assert np.all(2 * err <= step[:, :, None])
    # a value exactly half-way between two levels takes the upper one
    half = (2 * (G - mn[:, :, None]) % (2 * step[:, :, None])) == step[:, :, None]
    assert np.all(W[half] > G[half])
    assert ngroups > 25000


def test_w4a8_row_scale_and_bound():
    rng = np.random.default_rng(3)
    w = (rng.standard_normal((9, 256)) * rng.uniform(1e-3, 10, (9, 1))).astype(np.float16)
    w[4] = 0                                                  # an all-zero row
    w[5, 7] = -w[5].astype(np.float32).__abs__().max() * 2    # the row's largest magnitude negative
    w[6] = (rng.standard_normal(256) * 2e-6).astype(np.float16)  # fp16 subnormals only
    q = oracle.w4a8_quantize_weight(w)
    wf = w.astype(np.float64)
    amax = np.abs(wf).max(axis=1)
    w8 = oracle.w4a8_weight_int8(q).astype(np.float64)
    assert q.cscale[4] == 0 and np.all(w8[4] == 0)
    for n in range(9):
        if amax[n] == 0:
            continue
        assert q.cscale[n] == np.float32(np.float32(amax[n]) / np.float32(113))
        # level 1 puts the largest magnitude on +-113; level 2 moves a value by at most half a
        # step (<= 8 levels); so |w - cscale * w8| <= cscale * (1/2 + step/2) + rounding
        step = np.repeat(q.gstep[n].astype(np.float64), 64)
        bound = q.cscale[n] * (0.5 + step / 2) * (1 + 1e-6)
        assert np.all(np.abs(wf[n] - q.cscale[n] * w8[n]) <= bound)
    assert np.abs(w8).max() <= 127


# ------------------------------------------------------------------ activations ---------

def test_act8_hand_values():
    x = np.zeros((3, 64), np.float16)
    x[0, :7] = [127, -0.5, 0.5, 1.5, 2.5, -2.5, 126.5]      # amax 127: inv = 1, scale = 1
    x[2, :5] = [2, 1, -1, 0.5, -2]                          # amax 2: inv = 63.5
    a8, s = oracle.act8_quantize(x)
    assert s[0] == np.float32(1.0)
    assert list(a8[0, :7]) == [127, 0, 0, 2, 2, -2, 126]    # halves to even
    assert s[1] == 0 and np.all(a8[1] == 0)                 # an all-zero row
    assert s[2] == np.float32(2) / np.float32(127)
    assert list(a8[2, :5]) == [127, 64, -64, 32, -127]      # 63.5 -> 64 (even), 31.75 -> 32


def test_act8_bound_random():
    rng = np.random.default_rng(4)
    x = (rng.standard_normal((16, 320)) * rng.uniform(1e-4, 50, (16, 1))).astype(np.float16)
    a8, s = oracle.act8_quantize(x)
    xf = x.astype(np.float64)
    assert np.all(np.abs(a8.astype(np.int64)) <= 127)
    assert np.all(np.abs(a8).max(axis=1) == 127)            # the largest magnitude maps to 127
    err = np.abs(xf - a8.astype(np.float64) * s[:, None].astype(np.float64))
    assert np.all(err <= s[:, None] * 0.5 * (1 + 1e-5))


# ------------------------------------------------------------------ product --------------

def test_linear_w4a8_integer_sum_matches_numpy():
    rng = np.random.default_rng(5)
    M, N, K = 7, 24, 448
    w = (rng.standard_normal((N, K)) * 0.02).astype(np.float16)
    x = rng.standard_normal((M, K)).astype(np.float16)
    q = oracle.w4a8_quantize_weight(w)
    a8, s = oracle.act8_quantize(x)
    y, acc = oracle.linear_w4a8(a8, s, q, with_acc=True)
    w8 = oracle.w4a8_weight_int8(q)
    assert np.array_equal(acc, a8.astype(np.int64) @ w8.astype(np.int64).T)
    # a transposed or shifted operand would not match
    assert not np.array_equal(acc[:, 1:], (a8.astype(np.int64) @ w8.astype(np.int64).T)[:, :-1])


def test_linear_w4a8_closed_form_epilogue():
    # a8 = 1 everywhere and every 8-bit weight 3 (integer rows 3 and amax 3 -> w8 = 113, one level),
    # so acc = 113 K; y = acc * ascale * cscale + bias, q-scaled, ReLU'd, + residual
    M, N, K = 3, 4, 128
    x = np.ones((M, K), np.float16)
    w = np.full((N, K), 3.0, np.float16)
    w[1] = -3.0
    q = oracle.w4a8_quantize_weight(w)
    a8, s = oracle.act8_quantize(x)
    assert np.all(a8 == 127) and s[0] == np.float32(1) / np.float32(127)
    bias = np.array([0.5, 0.25, -1.0, 2.0], np.float16)
    res = np.full((M, N), 0.125, np.float16)
    y, acc = oracle.linear_w4a8(a8, s, q, bias=bias, residual=res, relu=True, qscale_cols=2, qscale=0.5,
                                with_acc=True)
    assert np.all(acc[:, [0, 2, 3]] == 127 * 113 * K) and np.all(acc[:, 1] == -127 * 113 * K)
    cs = float(s[0]) * float(q.cscale[0])
    base = 127 * 113 * K * cs                                # ~= 3 K = 384
    assert base == pytest.approx(3 * K, rel=1e-6)
    expect = np.array([(base + 0.5) * 0.5, max(0.0, (-base + 0.25) * 0.5), base - 1.0, base + 2.0]) + 0.125
    assert np.allclose(y, expect[None, :], rtol=0, atol=1e-9)


def test_linear_w4a8_close_to_the_real_product():
    # the whole scheme against the fp64 product of the unquantised operands: the error is bounded
    # by the two quantisation errors (8-bit activations, two-level 4-bit weights)
    rng = np.random.default_rng(6)
    M, N, K = 5, 16, 512
    w = (rng.standard_normal((N, K)) * 0.02).astype(np.float16)
    x = rng.standard_normal((M, K)).astype(np.float16)
    q = oracle.w4a8_quantize_weight(w)
    a8, s = oracle.act8_quantize(x)
    y = oracle.linear_w4a8(a8, s, q)
    ref = x.astype(np.float64) @ w.astype(np.float64).T
    wq = q.cscale[:, None].astype(np.float64) * oracle.w4a8_weight_int8(q).astype(np.float64)
    xq = s[:, None].astype(np.float64) * a8.astype(np.float64)
    bound = np.abs(x.astype(np.float64) - xq) @ np.abs(wq).T + np.abs(x.astype(np.float64)) @ np.abs(
        w.astype(np.float64) - wq).T
    assert np.all(np.abs(y - ref) <= bound * (1 + 1e-9) + 1e-12)
    assert np.max(np.abs(y - ref)) / np.max(np.abs(ref)) < 0.2


# ------------------------------------------------------------------ the W4A8 layer ------

def _f16(a):
    return oracle.f64_to_f16(np.asarray(a, dtype=np.float64))


def _compose_layer(w16, wq, heads, cache, x_rows, seq, pos):
    """The W4A8 layer written out from its pinned pieces (LayerNorm, the activation quantiser,
    the W4A8 product, the KV append and attention), row by row in order: the wiring of an OPT
    pre-LN decoder layer ([OPT]) with every activation handed on in fp16."""
    h = x_rows.shape[1]
    d = h // heads
    outs = []
    for r in range(x_rows.shape[0]):
        x = x_rows[r:r + 1]
        a = _f16(oracle.layernorm(x, w16["ln1_g"], w16["ln1_b"]))
        a8, s = oracle.act8_quantize(a)
        qkv = oracle.linear_w4a8(a8, s, wq.wqkv, bias=w16["bqkv"], qscale_cols=h, qscale=1.0 / np.sqrt(d))
        qkv16 = _f16(qkv)
        oracle.kv_append(cache, qkv16[:, h:2 * h], qkv16[:, 2 * h:], [seq[r]], [pos[r]])
        o = _f16(oracle.attention(cache, qkv16[:, :h], [seq[r]], [pos[r] + 1]))
        o8, so = oracle.act8_quantize(o)
        h1 = _f16(oracle.linear_w4a8(o8, so, wq.wo, bias=w16["bo"], residual=x))
        a2 = _f16(oracle.layernorm(h1, w16["ln2_g"], w16["ln2_b"]))
        a28, s2 = oracle.act8_quantize(a2)
        f = _f16(oracle.linear_w4a8(a28, s2, wq.w1, bias=w16["b1"], relu=True))
        f8, sf = oracle.act8_quantize(f)
        y = oracle.linear_w4a8(f8, sf, wq.w2, bias=w16["b2"], residual=h1)
        outs.append(y[0])
    return np.stack(outs)


def test_w4a8_layer_equals_its_pinned_pieces():
    import seeded_inputs as si
    h, H, F = 128, 2, 256
    w16 = si.layer_weights_f16(41, h, F, std=0.05, bias_std=0.05, ln_random=True)
    wq = oracle.W4A8LayerWeights(w16)
    S, maxL = 2, 64
    c_layer = oracle.KVCache(S, H, h // H, maxL)
    c_pieces = oracle.KVCache(S, H, h // H, maxL)
    seq = np.array([0, 1, 0, 0, 1])
    pos = np.array([0, 0, 1, 2, 1])
    x = si.normal_f16(41, 9, (len(seq), h), 1.0)
    got, _ = oracle.layer_rows_w4a8(wq, H, c_layer, x, seq, pos)
    ref = _compose_layer(w16, wq, H, c_pieces, x, seq, pos)
    assert np.allclose(got, ref, rtol=1e-12, atol=1e-12)
    for a, b in zip(c_layer.arrays(), c_pieces.arrays()):
        assert np.array_equal(a, b)


def test_w4a8_layer_close_to_the_w4a16_layer():
    # a sanity bound, not a pin: both forms quantise the same weights with independent errors of
    # similar size (the W4A8 one with 8-bit activations and integer group steps), so their layer
    # updates differ by about the quantisation noise -- a dropped term or a wrong sign would not
    import seeded_inputs as si
    h, H, F = 256, 4, 1024
    w16 = si.layer_weights_f16(42, h, F, std=0.02)
    S, maxL = 3, 64
    seq = np.array([0, 1, 2])
    pos = np.array([0, 0, 0])
    x = si.normal_f16(42, 9, (S, h), 1.0)
    a, _ = oracle.layer_rows_w4a8(oracle.W4A8LayerWeights(w16), H, oracle.KVCache(S, H, h // H, maxL), x, seq, pos)
    b, _ = oracle.layer_rows(oracle.LayerWeights(w16), H, oracle.KVCache(S, H, h // H, maxL), x, seq, pos)
    dx = x.astype(np.float64)
    assert np.max(np.abs((a - dx) - (b - dx))) <= 0.5 * np.max(np.abs(b - dx))
