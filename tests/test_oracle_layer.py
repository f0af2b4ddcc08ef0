"""Pins of the oracle's LayerNorm, linear, attention and OPT-layer wiring (CPU only).

Expected values come from closed forms (LayerNorm of a +-a row, permutation
weights that 4-bit groups store exactly, one-token and uniform softmax, the
two-element softmax = logistic function) and from invariances the pages fix
(rows are independent of the batch split: "FlexGen Guide", section 2, The
Zig-Zag Block Schedule).  Model family: OPT (pre-LayerNorm, ReLU FFN).
"""
import math

import numpy as np
import pytest

import oracle
import seeded_inputs as si


def f16(a):
    return np.asarray(a, dtype=np.float64).astype(np.float16)


def perm_weight(n_out, n_in, cols, value=15.0):
    """[n_out, n_in] with `value` at (i, cols[i]), zero elsewhere.

    Every 64-group along the input dim is {0, 15} or all zero, which the
    4-bit format stores exactly (min 0, scale 1, codes 0/15)."""
    w = np.zeros((n_out, n_in), dtype=np.float16)
    w[np.arange(n_out), cols] = value
    return w


# ------------------------------------------------------------------ LayerNorm ----------

def test_layernorm_alternating_row_closed_form():
    h, a, eps = 256, 3.0, 1e-5
    x = f16(np.where(np.arange(h) % 2 == 0, a, -a)).reshape(1, h)
    y = oracle.layernorm(x, eps=eps)
    want = np.where(np.arange(h) % 2 == 0, a, -a) / math.sqrt(a * a + eps)
    assert np.allclose(y[0], want, rtol=0, atol=1e-14)


def test_layernorm_constant_row_gives_beta_and_affine():
    h = 128
    beta = si.normal_f16(1, 5, (h,), 0.5)
    gamma = si.normal_f16(1, 6, (h,), 1.0)
    y = oracle.layernorm(np.full((1, h), 2.5, dtype=np.float16), gamma, beta)
    assert np.array_equal(y[0], beta.astype(np.float64))
    x = si.normal_f16(1, 7, (3, h), 1.0)
    n = oracle.layernorm(x)                    # gamma 1, beta 0
    y = oracle.layernorm(x, gamma, beta)
    assert np.allclose(y, n * gamma.astype(np.float64) + beta.astype(np.float64), atol=1e-13)
    # normalised rows have mean 0 and variance var/(var+eps) ~ 1
    assert np.allclose(n.mean(axis=1), 0, atol=1e-12)
    assert np.allclose((n * n).mean(axis=1), 1, atol=1e-4)


# ------------------------------------------------------------------ linear -------------

def test_linear_permutation_exact():
    M, K, N = 5, 192, 128
    rng = np.random.default_rng(0)
    cols = rng.integers(0, K, N)                # not symmetric: catches a transposed W
    w = oracle.quantize(perm_weight(N, K, cols), 1)
    assert np.array_equal(oracle.dequantize(w).astype(np.float64), perm_weight(N, K, cols).astype(np.float64))
    x = si.normal_f16(2, 1, (M, K), 1.0)
    b = si.normal_f16(2, 2, (N,), 1.0)
    y = oracle.linear(x, w, bias=b)
    want = 15.0 * x.astype(np.float64)[:, cols] + b.astype(np.float64)
    assert np.array_equal(y, want)


def test_linear_epilogues_closed_form():
    M, K, N = 3, 128, 64
    cols = (np.arange(N) * 7) % K
    w = oracle.quantize(perm_weight(N, K, cols), 1)
    x = si.normal_f16(3, 1, (M, K), 1.0)
    b = si.normal_f16(3, 2, (N,), 1.0)
    r = si.normal_f16(3, 3, (M, N), 1.0)
    base = 15.0 * x.astype(np.float64)[:, cols] + b.astype(np.float64)
    assert np.array_equal(oracle.linear(x, w, bias=b, relu=True), np.maximum(base, 0))
    assert np.array_equal(oracle.linear(x, w, bias=b, residual=r), base + r.astype(np.float64))
    qs = 1 / math.sqrt(64)
    got = oracle.linear(x, w, bias=b, qscale_cols=20, qscale=qs)
    want = base.copy(); want[:, :20] *= qs
    assert np.array_equal(got, want)


def test_linear_random_against_dequantized_matmul_sizes():
    # ragged M, several groups along K: agrees with a float64 matmul of the dequantised weight
    M, K, N = 7, 320, 96
    x = si.normal_f16(4, 1, (M, K), 1.0)
    w = oracle.quantize(si.normal_f16(4, 2, (N, K), 0.02), 1)
    wd = oracle.dequantize(w).astype(np.float64)
    assert np.allclose(oracle.linear(x, w), x.astype(np.float64) @ wd.T, rtol=1e-12, atol=1e-12)


# ------------------------------------------------------------------ attention ----------

def _random_cache(S, H, d, maxL, L, seed=5):
    c = oracle.KVCache(S, H, d, maxL)
    for pos in range(L):
        k = si.normal_f16(seed, 100 + pos, (S, H * d), 1.0)
        v = si.normal_f16(seed, 200 + pos, (S, H * d), 1.0)
        oracle.kv_append(c, k, v, np.arange(S), np.full(S, pos))
    return c


def _deq_v(c, s, h, pos):
    q = oracle.Packed(c.vc[s, h, pos][None], c.vm[s, h, pos][None].view(np.float16),
                      c.vs[s, h, pos][None].view(np.float16), (1, c.d), 1)
    return oracle.dequantize(q).astype(np.float64)[0]


def test_attention_single_token_returns_v():
    S, H, d = 2, 3, 128
    c = _random_cache(S, H, d, 64, 1)
    q = si.normal_f16(6, 1, (S, H * d), 1.0)
    o = oracle.attention(c, q, np.arange(S), np.ones(S, dtype=np.int32))
    for s in range(S):
        for h in range(H):
            assert np.array_equal(o[s, h * d:(h + 1) * d], _deq_v(c, s, h, 0))


def test_attention_zero_query_is_mean_of_v():
    S, H, d, L = 2, 2, 64, 9
    c = _random_cache(S, H, d, 64, L)
    q = np.zeros((S, H * d), dtype=np.float16)
    o = oracle.attention(c, q, np.arange(S), np.full(S, L))
    for s in range(S):
        for h in range(H):
            mean = np.mean([_deq_v(c, s, h, j) for j in range(L)], axis=0)
            assert np.allclose(o[s, h * d:(h + 1) * d], mean, rtol=0, atol=1e-13)


def test_attention_exact_dequant_single_token_rounds_to_the_fp16_form():
    # one cached token: the exact form returns min + code * scale, the fp16 form that value
    # rounded to fp16 -- so rounding the exact output gives the fp16 output bit for bit
    S, H, d = 2, 3, 128
    c = _random_cache(S, H, d, 64, 1)
    q = si.normal_f16(7, 1, (S, H * d), 1.0)
    o16 = oracle.attention(c, q, np.arange(S), np.ones(S, dtype=np.int32))
    ox = oracle.attention(c, q, np.arange(S), np.ones(S, dtype=np.int32), exact_dequant=True)
    assert np.array_equal(oracle.f64_to_f16(ox).astype(np.float64), o16)
    assert np.all(np.abs(ox - o16) <= 2.0 ** -11 * np.abs(o16))
    assert not np.array_equal(ox, o16)                       # the two forms do differ


@pytest.mark.parametrize("group", [64, 128])
def test_attention_exact_dequant_equals_fp16_form_on_representable_groups(group):
    # groups built as min + code * 2^e (codes 0 and 15 present, min a multiple of 2^e): the
    # quantiser stores scale 2^e and the codes exactly, and every min + code * scale is an fp16
    # value, so both forms read the same K and V and agree bit for bit for any query
    S, H, d, L = 2, 2, 128, 37
    rng = np.random.default_rng(8)
    c = oracle.KVCache(S, H, d, 64, group=group)
    for s in range(S):
        rows = []
        for _ in range(2 * L):
            e = rng.integers(-8, 0, size=d // group)
            codes = rng.integers(0, 16, size=(d // group, group))
            codes[:, 0], codes[:, 1] = 0, 15
            mins = rng.integers(-64, 64, size=d // group) * 2.0 ** e
            rows.append((mins[:, None] + codes * (2.0 ** e)[:, None]).reshape(d))
        kv = np.array(rows).astype(np.float16).reshape(2, L, d)
        k, v = np.tile(kv[0], (1, H)), np.tile(kv[1], (1, H))
        oracle.kv_append(c, k, v, np.full(L, s), np.arange(L))
    q = si.normal_f16(8, 1, (S, H * d), 1.0)
    lens = np.array([L, 20], dtype=np.int32)
    assert np.array_equal(oracle.attention(c, q, np.arange(S), lens),
                          oracle.attention(c, q, np.arange(S), lens, exact_dequant=True))


def test_attention_two_tokens_logistic():
    # K_0 = 0 (constant group), K_1 = constant c: scores 0 and c*sum(q); softmax of two is logistic
    S, H, d = 1, 1, 64
    cache = oracle.KVCache(S, H, d, 64)
    k = np.stack([np.zeros(d), np.full(d, 0.25)]).astype(np.float16)
    v = si.normal_f16(7, 1, (2, d), 1.0)
    oracle.kv_append(cache, k[:1], v[:1], [0], [0])
    oracle.kv_append(cache, k[1:], v[1:], [0], [1])
    q = si.normal_f16(7, 2, (1, d), 1.0)
    o = oracle.attention(cache, q, [0], [2])[0]
    s1 = 0.25 * q.astype(np.float64).sum()
    p1 = 1.0 / (1.0 + math.exp(-s1))
    want = (1 - p1) * _deq_v(cache, 0, 0, 0) + p1 * _deq_v(cache, 0, 0, 1)
    assert np.allclose(o, want, rtol=0, atol=1e-12)


def test_attention_reads_only_first_len_positions():
    S, H, d = 1, 2, 64
    c = _random_cache(S, H, d, 64, 5)
    q = si.normal_f16(8, 1, (1, H * d), 1.0)
    a = oracle.attention(c, q, [0], [3])
    big = np.full((1, H * d), 1000.0, dtype=np.float16)
    oracle.kv_append(c, big, big, [0], [3])
    oracle.kv_append(c, big, big, [0], [4])
    assert np.array_equal(a, oracle.attention(c, q, [0], [3]))


def test_attention_peaked_selects_token():
    S, H, d = 1, 1, 64
    cache = oracle.KVCache(S, H, d, 64)
    for j in range(4):
        k = np.full((1, d), 4.0 if j == 2 else 0.0, dtype=np.float16)
        oracle.kv_append(cache, k, si.normal_f16(9, j, (1, d), 1.0), [0], [j])
    q = np.full((1, d), 1.0, dtype=np.float16)   # score 256 for token 2, 0 elsewhere
    o = oracle.attention(cache, q, [0], [4])[0]
    assert np.allclose(o, _deq_v(cache, 0, 0, 2), rtol=0, atol=1e-100 + 1e-12)


@pytest.mark.parametrize("d", [128, 256])
def test_kv_append_group128_layout_matches_quantize(d):
    # groups of 128 along head_dim ("FlexGen Guide", section 3: groups of 64 or 128): the cache
    # slot of (sequence, head, position) holds quantize(row, groups of 128) of that head's values
    S, H, maxL = 2, 2, 64
    c = oracle.KVCache(S, H, d, maxL, group=128)
    assert c.km.shape == (S, H, maxL, d // 128)
    k = si.normal_f16(20, 1, (3, H * d), 1.0)
    v = si.normal_f16(20, 2, (3, H * d), 1.0)
    oracle.kv_append(c, k, v, [1, 0, 1], [3, 9, 63])
    qk = oracle.quantize(k.reshape(3, H, d), dim=-1, group=128)
    qv = oracle.quantize(v.reshape(3, H, d), dim=-1, group=128)
    for r, (s, p) in enumerate([(1, 3), (0, 9), (1, 63)]):
        assert np.array_equal(c.kc[s, :, p], qk.codes[r]) and np.array_equal(c.vc[s, :, p], qv.codes[r])
        assert np.array_equal(c.ks[s, :, p], qk.scales.view(np.uint16)[r])
        assert np.array_equal(c.vm[s, :, p], qv.mins.view(np.uint16)[r])
    with pytest.raises(ValueError):
        oracle.KVCache(S, H, 64, maxL, group=128)            # a group must fit in head_dim


def test_kv_append_layout_matches_quantize():
    S, H, d, maxL = 3, 2, 128, 64
    c = oracle.KVCache(S, H, d, maxL)
    k = si.normal_f16(10, 1, (2, H * d), 1.0)
    v = si.normal_f16(10, 2, (2, H * d), 1.0)
    oracle.kv_append(c, k, v, [2, 0], [5, 7])
    qk = oracle.quantize(k.reshape(2, H, d), dim=-1)
    qv = oracle.quantize(v.reshape(2, H, d), dim=-1)
    assert np.array_equal(c.kc[2, :, 5], qk.codes[0]) and np.array_equal(c.kc[0, :, 7], qk.codes[1])
    assert np.array_equal(c.vs[2, :, 5], qv.scales.view(np.uint16)[0])
    assert np.array_equal(c.km[0, :, 7], qk.mins.view(np.uint16)[1])
    assert c.kc[1].sum() == 0 and c.kc[2, :, 4].sum() == 0


# ------------------------------------------------------------------ layer wiring -------

H_, D_ = 2, 64
HID = H_ * D_
FFN = 4 * HID


def _wiring_weights(qk_zero: bool, HID=HID, FFN=FFN):
    """Permutation-structured layer whose output has a closed form."""
    rng = np.random.default_rng(11)
    pv, po, p1 = rng.permutation(HID), rng.permutation(HID), rng.integers(0, HID, FFN)
    p2 = rng.permutation(FFN)[:HID]
    wq = np.zeros((HID, HID), np.float16) if qk_zero else si.normal_f16(12, 1, (HID, HID), 0.05)
    wk = np.zeros((HID, HID), np.float16) if qk_zero else si.normal_f16(12, 2, (HID, HID), 0.05)
    w16 = {
        "wqkv": np.concatenate([wq, wk, perm_weight(HID, HID, pv)]),
        "wo": perm_weight(HID, HID, po),
        "w1": perm_weight(FFN, HID, p1),
        "w2": perm_weight(HID, FFN, p2),
        "bqkv": np.concatenate([np.zeros(2 * HID), si.normal_f16(12, 3, (HID,), 0.5)]).astype(np.float16),
        "bo": si.normal_f16(12, 4, (HID,), 0.5),
        "b1": si.normal_f16(12, 5, (FFN,), 3.0),
        "b2": si.normal_f16(12, 6, (HID,), 0.5),
        "ln1_g": (1 + si.normal_f16(12, 7, (HID,), 0.1).astype(np.float32)).astype(np.float16),
        "ln1_b": si.normal_f16(12, 8, (HID,), 0.1),
        "ln2_g": (1 + si.normal_f16(12, 9, (HID,), 0.1).astype(np.float32)).astype(np.float16),
        "ln2_b": si.normal_f16(12, 10, (HID,), 0.1),
    }
    return w16, (pv, po, p1, p2)


def r16(a):
    """Value of the nearest fp16 (an activation the FP16 layer stores), as float64."""
    return f16(a).astype(np.float64)


def _closed_form(w16, perms, x_rows, o_rows):
    """y = h1 + 15*r16(relu(15*r16(LN2(h1))[p1] + b1))[p2] + b2, h1 = r16(x + 15*o[po] + bo).

    r16 marks the activations an FP16 layer hands from op to op (rounded to fp16)."""
    pv, po, p1, p2 = perms
    x = x_rows.astype(np.float64)
    h1 = r16(x + 15.0 * o_rows[:, po] + w16["bo"].astype(np.float64))
    a2 = r16(oracle.layernorm(f16(h1), w16["ln2_g"], w16["ln2_b"]))   # h1 is exactly an fp16 value
    f = r16(np.maximum(15.0 * a2[:, p1] + w16["b1"].astype(np.float64), 0.0))
    return h1 + 15.0 * f[:, p2] + w16["b2"].astype(np.float64)


def _v_rows(w16, perms, x_rows):
    """v = fp16(15*fp16(LN1(x))[pv] + bv) (what is appended to the cache)."""
    pv = perms[0]
    hid = x_rows.shape[1]
    a = r16(oracle.layernorm(x_rows, w16["ln1_g"], w16["ln1_b"]))
    return f16(15.0 * a[:, pv] + w16["bqkv"].astype(np.float64)[2 * hid:])


def test_layer_single_token_closed_form():
    w16, perms = _wiring_weights(qk_zero=False)
    W = oracle.LayerWeights(w16)
    S = 3
    x = si.normal_f16(13, 1, (S, HID), 1.0)
    cache = oracle.KVCache(S, H_, D_, 64)
    y, attn = oracle.layer_rows(W, H_, cache, x, np.arange(S), np.zeros(S), want_attn=True)
    # one cached token: attention returns the dequantised 4-bit v of that token
    v = _v_rows(w16, perms, x)
    o = oracle.dequantize(oracle.quantize(v.reshape(S, H_, D_), -1)).astype(np.float64).reshape(S, HID)
    assert np.array_equal(attn, r16(o))
    assert np.allclose(y, _closed_form(w16, perms, x, r16(o)), rtol=0, atol=1e-9)


def test_layer_group128_single_token_and_uniform_prompt_closed_forms():
    # The layer with weights and KV cache in groups of 128 (2 heads x 128): the permutation
    # weights are still stored exactly ({0, 15} per group), one cached token returns its
    # dequantised group-128 v, and q = k = 0 averages the group-128 v of the prefix.
    H, D = 2, 128
    hid, ffn = H * D, 4 * H * D
    w16, perms = _wiring_weights(qk_zero=True, HID=hid, FFN=ffn)
    W = oracle.LayerWeights(w16, group=128)
    S, P = 2, 4
    x = si.normal_f16(21, 1, (S, P, hid), 1.0)
    cache = oracle.KVCache(S, H, D, 64, group=128)
    rows = x.transpose(1, 0, 2).reshape(P * S, hid)
    seq, pos = np.tile(np.arange(S), P), np.repeat(np.arange(P), S)
    y, attn = oracle.layer_rows(W, H, cache, rows, seq, pos, want_attn=True)
    v = _v_rows(w16, perms, rows)
    vd = oracle.dequantize(oracle.quantize(v.reshape(-1, H, D), -1, group=128)).astype(np.float64).reshape(-1, hid)
    for r in range(P * S):
        mine = (seq == seq[r]) & (pos <= pos[r])
        o = vd[mine].mean(axis=0)
        # the attention output is o rounded to fp16 (its sum order differs from numpy's mean, so
        # allow half an fp16 ulp; a wrong group would be off by up to half a quantisation step)
        assert np.all(np.abs(attn[r] - o) <= 2.0 ** -11 * np.abs(o) + 1e-12)
        assert np.allclose(y[r], _closed_form(w16, perms, rows[r:r + 1], attn[r][None])[0], rtol=0, atol=1e-9)
    assert np.array_equal(attn[:S], r16(vd[:S]))          # position 0: the one cached token
    with pytest.raises(ValueError):
        oracle.layer_rows(W, H, oracle.KVCache(S, H, D, 64), rows, seq, pos)   # groups must agree


def test_layer_uniform_attention_over_prompt():
    w16, perms = _wiring_weights(qk_zero=True)
    W = oracle.LayerWeights(w16)
    S, P = 2, 5
    x = si.normal_f16(14, 1, (S, P, HID), 1.0)
    cache = oracle.KVCache(S, H_, D_, 64)
    rows = x.transpose(1, 0, 2).reshape(P * S, HID)          # token-major: all seqs at t=0, then t=1 ...
    seq = np.tile(np.arange(S), P)
    pos = np.repeat(np.arange(P), S)
    y, attn = oracle.layer_rows(W, H_, cache, rows, seq, pos, want_attn=True)
    v = _v_rows(w16, perms, rows)
    vd = oracle.dequantize(oracle.quantize(v.reshape(-1, H_, D_), -1)).astype(np.float64).reshape(-1, HID)
    for r in range(P * S):
        s, t = seq[r], pos[r]
        mine = (seq == s) & (pos <= t)
        o = vd[mine].mean(axis=0)                         # q = k = 0: softmax is uniform over 0..t
        assert np.allclose(attn[r], r16(o), rtol=0, atol=1e-12)
        o = attn[r]
        assert np.allclose(y[r], _closed_form(w16, perms, rows[r:r + 1], o[None])[0], rtol=0, atol=1e-9)


def test_layer_query_scale_two_tokens():
    # Wq = 15*I and Wk = 15*I with zero v-weights: score_j = d^-1/2 * q.k_j,
    # softmax over two tokens is the logistic of the score difference
    d = D_
    w16, perms = _wiring_weights(qk_zero=True)
    eye = perm_weight(HID, HID, np.arange(HID))
    w16["wqkv"] = np.concatenate([eye, eye, w16["wqkv"][2 * HID:]])
    W = oracle.LayerWeights(w16)
    x = si.normal_f16(15, 1, (2, HID), 1.0)
    cache = oracle.KVCache(1, H_, D_, 64)
    _, attn = oracle.layer_rows(W, H_, cache, x, [0, 0], [0, 1], want_attn=True)
    a = r16(oracle.layernorm(x, w16["ln1_g"], w16["ln1_b"]))
    q1 = r16(15.0 * a[1] / math.sqrt(d))
    kq = oracle.dequantize(oracle.quantize(f16(15.0 * a).reshape(2, H_, D_), -1)).astype(np.float64).reshape(2, HID)
    v = _v_rows(w16, perms, x)
    vd = oracle.dequantize(oracle.quantize(v.reshape(-1, H_, D_), -1)).astype(np.float64).reshape(-1, HID)
    for h in range(H_):
        sl = slice(h * d, (h + 1) * d)
        s0, s1 = q1[sl] @ kq[0, sl], q1[sl] @ kq[1, sl]
        p1 = 1.0 / (1.0 + math.exp(s0 - s1))
        want = (1 - p1) * vd[0, sl] + p1 * vd[1, sl]
        assert np.allclose(attn[1, sl], r16(want), rtol=0, atol=2e-3 * np.abs(want).max())


def test_layer_rows_independent_of_block_split_and_threads():
    rng = np.random.default_rng(3)
    h, H, F = 128, 2, 256
    w16 = si.layer_weights_f16(16, h, F, std=0.05, bias_std=0.1, ln_random=True)
    W = oracle.LayerWeights(w16)
    S, P = 6, 3
    x = si.normal_f16(16, 2, (P, S, h), 1.0).reshape(P * S, h)
    seq = np.tile(np.arange(S), P)
    pos = np.repeat(np.arange(P), S)
    c1 = oracle.KVCache(S, H, h // H, 64)
    y1, _ = oracle.layer_rows(W, H, c1, x, seq, pos, nthreads=1)
    c2 = oracle.KVCache(S, H, h // H, 64)
    y2, _ = oracle.layer_rows(W, H, c2, x, seq, pos, nthreads=4)
    assert np.array_equal(y1, y2)
    # one sequence at a time (a block of batches of size 1) gives identical rows
    c3 = oracle.KVCache(S, H, h // H, 64)
    order = rng.permutation(S)
    y3 = np.zeros_like(y1)
    for s in order:
        m = seq == s
        y3[m], _ = oracle.layer_rows(W, H, c3, x[m], seq[m], pos[m])
    assert np.array_equal(y1, y3)
    for a, b in zip(c1.arrays(), c3.arrays()):
        assert np.array_equal(a, b)


def test_layer_kv_only_fills_same_cache():
    h, H, F = 128, 2, 256
    w16 = si.layer_weights_f16(17, h, F, std=0.05, bias_std=0.1)
    W = oracle.LayerWeights(w16)
    x = si.normal_f16(17, 2, (4, h), 1.0)
    c1 = oracle.KVCache(2, H, h // H, 64)
    c2 = oracle.KVCache(2, H, h // H, 64)
    oracle.layer_rows(W, H, c1, x, [0, 1, 0, 1], [0, 0, 1, 1])
    oracle.layer_rows(W, H, c2, x, [0, 1, 0, 1], [0, 0, 1, 1], kv_only=True)
    for a, b in zip(c1.arrays(), c2.arrays()):
        assert np.array_equal(a, b)


def test_layer_rejects_bad_positions():
    h, H, F = 128, 2, 256
    W = oracle.LayerWeights(si.layer_weights_f16(18, h, F))
    c = oracle.KVCache(1, H, h // H, 64)
    with pytest.raises(AssertionError):
        oracle.layer_rows(W, H, c, np.zeros((1, h), np.float16), [0], [64])
