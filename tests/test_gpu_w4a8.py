"""GPU parity of the W4A8 path (fg_w4a8_quantize_weight, fg_act8_quantize, fg_linear_w4a8)
against the CPU oracle, through the C ABI.

Bit-exact: the weight codes, group minima and steps, the row scales, the activation codes and
scales (integers decided in fp32 on both sides, one IEEE operation at a time).
The product: the integer sums are exact on both sides, so the only difference left is the
epilogue: the GPU's fp32 operations (scale product, acc * it, + bias, q-scale, + residual, each
rounded to 2^-24 relative) and its final fp16 rounding, against the oracle's float64 epilogue.
The test bound is one fp16 ulp of the result plus 2^-21 of the magnitudes that enter the sums.
"""
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


def _weights(seed, N, K):
    """N(0, 0.02) weights with rows of very different magnitudes, an all-zero row, a row with one
    outlier, a constant group and a row of fp16 subnormals (trained-like weights with outliers)."""
    w = si.normal_f16(seed, 1, (N, K), 0.02).astype(np.float32)
    w *= np.float32(10.0) ** si.normal_f16(seed, 2, (N, 1), 1.0).astype(np.float32).clip(-3, 1)
    w = w.astype(np.float16)
    w[1] = 0
    w[2, K // 3] = 8.0
    w[3, 64:128] = 0.5
    if N > 5:
        w[5] = (w[5].astype(np.float32) * np.float32(5e-5)).astype(np.float16)   # fp16 subnormals
    return w


def _acts(seed, M, K):
    x = si.normal_f16(seed, 3, (M, K), 1.0).astype(np.float32)
    x *= np.float32(10.0) ** si.normal_f16(seed, 4, (M, 1), 1.0).astype(np.float32).clip(-3, 1)
    x = x.astype(np.float16)
    if M > 1:
        x[1] = 0
    if M > 2:
        x[2] = (x[2].astype(np.float32) * np.float32(1e-5)).astype(np.float16)   # fp16 subnormals
    return x


def _check_weight(wq, ref, rows=None):
    sel = slice(None) if rows is None else torch.from_numpy(rows).cuda()
    r = slice(None) if rows is None else rows
    assert np.array_equal(host(wq.codes[sel]), ref.codes[r])
    assert np.array_equal(host(wq.gmin[sel]), ref.gmin[r])
    assert np.array_equal(host(wq.gstep[sel]), ref.gstep[r])
    assert np.array_equal(host(wq.cscale[sel]).view(np.uint32), ref.cscale[r].view(np.uint32))


@pytest.mark.parametrize("N,K", [(4, 64), (7, 192), (256, 512), (130, 4096)])
def test_w4a8_weight_quantiser_bit_exact(N, K):
    w = _weights(31, N, K)
    wq = fg.fg_w4a8_quantize_weight(dev(w))
    _check_weight(wq, oracle.w4a8_quantize_weight(w))


@pytest.mark.parametrize("M,K", [(1, 64), (5, 4096), (300, 1024), (2, 7168), (2, 16384), (2, 28672), (3, 49152)])
def test_act8_quantiser_bit_exact(M, K):
    x = _acts(32, M, K)
    a8, s = fg.fg_act8_quantize(dev(x))
    ra8, rs = oracle.act8_quantize(x)
    assert np.array_equal(host(a8), ra8)
    assert np.array_equal(host(s).view(np.uint32), rs.view(np.uint32))


def _bound(acc, ascale, cscale, bias, res, qcols, qscale, ref):
    cs = ascale[:, None].astype(np.float64) * cscale[None, :].astype(np.float64)
    qs = np.ones(cs.shape[1])
    qs[:qcols] = abs(qscale)
    mag = (np.abs(acc.astype(np.float64)) * cs + (0 if bias is None else np.abs(bias.astype(np.float64)))) * qs
    if res is not None:
        mag = mag + np.abs(res.astype(np.float64))
    tiny = 2.0 ** -24
    ulp = np.maximum(np.spacing(np.abs(ref).astype(np.float16)).astype(np.float64), tiny)
    return ulp + mag * 2.0 ** -21 + tiny


def _run_and_check(M, N, K, seed, rows=None, relu=False, qcols=0, qscale=1.0, with_res=True):
    w = _weights(seed, N, K)
    x = _acts(seed, M, K)
    b = si.normal_f16(seed, 5, (N,), 0.1)
    r = si.normal_f16(seed, 6, (M, N), 1.0) if with_res else None
    wq = fg.fg_w4a8_quantize_weight(dev(w))
    a8, s = fg.fg_act8_quantize(dev(x))
    y = fg.fg_linear_w4a8(a8, s, wq, bias=dev(b), residual=None if r is None else dev(r), relu=relu,
                          qscale_cols=qcols, qscale=qscale)
    fg.fg_sync_status()
    rows = np.arange(M) if rows is None else rows
    ref_w = oracle.w4a8_quantize_weight(w)
    _check_weight(wq, ref_w)
    ra8, rs = oracle.act8_quantize(x[rows])
    assert np.array_equal(host(a8)[rows], ra8)
    ref, acc = oracle.linear_w4a8(ra8, rs, ref_w, bias=b, residual=None if r is None else r[rows], relu=relu,
                                  qscale_cols=qcols, qscale=qscale, with_acc=True)
    got = host(y)[rows].astype(np.float64)
    tol = _bound(acc, rs, ref_w.cscale, b, None if r is None else r[rows], qcols, qscale, ref)
    bad = np.abs(got - ref) > tol
    assert not bad.any(), (int(bad.sum()), np.argwhere(bad)[:4], got[bad][:4], ref[bad][:4])
    return y


@pytest.mark.parametrize("M,N,K", [(1, 256, 128), (5, 384, 640), (40, 512, 1024), (130, 256, 4096),
                                   (300, 768, 2048), (16, 256, 16384), (600, 256, 768)])
def test_linear_w4a8_matches_oracle(M, N, K):
    # (600, 256, 768): more than 256 tokens with K / 64 = 12 metadata columns per row, which the
    # pair launch's 16-column tensor copies do not take: the one-SM kernel over 3 token tiles
    _run_and_check(M, N, K, seed=33)


def test_linear_w4a8_epilogues():
    _run_and_check(70, 384, 768, seed=34, relu=True, qcols=128, qscale=0.125)
    _run_and_check(70, 384, 768, seed=35, with_res=False)


def test_linear_w4a8_plans_agree_bit_for_bit():
    # a k split sums int32 partials, exactly: rows computed under different plans are equal
    M, N, K = 512, 16384, 4096
    w = _weights(36, N, K)
    x = _acts(36, M, K)
    wq = fg.fg_w4a8_quantize_weight(dev(w))
    a8, s = fg.fg_act8_quantize(dev(x))
    big = fg.fg_linear_w4a8(a8, s, wq)
    small = fg.fg_linear_w4a8(a8[:16].contiguous(), s[:16].contiguous(), wq)
    assert fg.fg_linear_w4a8_plan(M, N, K)[1] == 1 and fg.fg_linear_w4a8_plan(16, N, K)[1] > 1
    assert torch.equal(big[:16], small)


@pytest.mark.parametrize("N,K", [(12288, 4096), (4096, 16384)])
def test_linear_w4a8_decode_shapes_sampled(N, K):
    # the OPT-6.7B decode block's QKV and FC2 shapes at 512 tokens, in the launch the benchmark
    # times; the oracle checks sampled rows (one per 64-token stretch, first and last included)
    M = 512
    rows = np.unique(np.concatenate([np.arange(0, M, 64), [1, 255, 256, M - 1]]))
    _run_and_check(M, N, K, seed=37, rows=rows)


def test_linear_w4a8_pair_split_modes_agree():
    # the CTA-pair launch's k split (FC2's shape: 4 split ranks) through the scratch with flags,
    # through the scratch at a cluster barrier, and over distributed shared memory: the int32
    # partials add exactly, so all three give the same bits
    M, N, K = 512, 4096, 16384
    t, splits = fg.fg_linear_w4a8_plan(M, N, K)
    assert t in (256, 512) and splits > 1
    w = _weights(38, N, K)
    x = _acts(38, M, K)
    r = dev(si.normal_f16(38, 6, (M, N), 1.0))
    wq = fg.fg_w4a8_quantize_weight(dev(w))
    a8, s = fg.fg_act8_quantize(dev(x))
    tiles = -(-N // 256) * -(-M // t)
    part = tiles * splits * t * 256 * 4
    full = fg.fg_linear_w4a8_workspace_bytes(M, N, K)
    assert full == part + tiles * splits * 2 * 8
    outs = []
    for nbytes in (full, part, 0):
        ws = torch.empty(max(nbytes, 1), dtype=torch.uint8, device="cuda")[:nbytes]
        outs.append(fg.fg_linear_w4a8(a8, s, wq, residual=r, workspace=ws))
    fg.fg_sync_status()
    assert torch.equal(outs[0], outs[1]) and torch.equal(outs[0], outs[2])
    rows = np.array([0, 100, 511])
    ref_w = oracle.w4a8_quantize_weight(w)
    ra8, rs = oracle.act8_quantize(x[rows])
    rr = host(r)[rows]
    ref, acc = oracle.linear_w4a8(ra8, rs, ref_w, residual=rr, with_acc=True)
    tol = _bound(acc, rs, ref_w.cscale, None, rr, 0, 1.0, ref)
    assert np.all(np.abs(host(outs[0])[rows].astype(np.float64) - ref) <= tol)
