"""GPU parity of the OPT layer in its W4A8 form (fg_layer_config.act_bits = 8) against the
oracle's W4A8 layer, through the C ABI.

The W4A8 weights are bit-exact with the oracle's. Two kinds of check:

- Stage by stage (test_w4a8_decode_step_stage_by_stage): every stage of a decode step against
  the oracle's pieces applied to the GPU's own input of that stage, read from the workspace
  (fg.h states its layout): the activation codes and scales bit-exact, each product within its
  epilogue bound, attention at the fp16 attention tolerance.
- The whole layer against the oracle's whole W4A8 layer, on D = x_out - x_in. Each product's
  int8 input is decided in fp32 on both sides, but from fp16 rows that already carry the
  fp32-versus-float64 differences of the steps before. One ulp on a row's largest value moves
  that row's scale by 2^-11 and every code by up to 127 * 2^-11 = 0.06, so about one code in
  sixteen flips by a step, all in the same direction; through four products this adds up to
  about 1e-2 of max|D| (1.01e-2 measured on a 4-sequence decode step whose every stage agrees
  to an ulp). The W4A8 layer is therefore held to 2e-2, the W4A16 layer's 1e-2 doubled for
  this one extra rounding decision per product. A 4-bit K/V code can flip the same way, and one
  flipped code of the current token's v moves the attention output by a quantisation step
  (0.14 seen at a prompt's third token), so the oracle attends over the GPU's cache (the
  reading on KV codes in full-layer runs): each comparison starts from a copy of the GPU's
  cache after the call and runs the oracle's layer without its append (keep_cache). The KV
  append itself is held bit-exact by its own tests.
"""
import numpy as np
import pytest
import torch

import oracle
import seeded_inputs as si

pytestmark = pytest.mark.gpu
fg = None
TOL = 2e-2
MATS = ("wqkv", "wo", "w1", "w2")


@pytest.fixture(autouse=True)
def _bind_library(fg_lib):
    global fg
    fg = fg_lib


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def delta_err(out_gpu, x16, ref):
    x = x16.astype(np.float64)
    return np.max(np.abs((out_gpu.astype(np.float64) - x) - (ref - x))) / np.max(np.abs(ref - x))


def _gpu_cache(gc, sample, maxL):
    """The oracle's cache for the sampled sequences, a copy of the GPU's."""
    H, d = gc.arrays()[0].shape[1], gc.arrays()[0].shape[3] * 2
    oc = oracle.KVCache(len(sample), H, d, maxL)
    idx = torch.from_numpy(np.asarray(sample)).cuda()
    for a, b in zip(oc.arrays(), gc.arrays()):
        a[...] = b[idx].cpu().numpy().view(a.dtype)
    return oc


def _prompt_ref(ow, H, gc, prompt, sample, maxL):
    """The oracle's prefill rows of the sampled sequences over the GPU's K/V codes."""
    P, h = prompt.shape[1], prompt.shape[2]
    oc = _gpu_cache(gc, sample, maxL)
    ref, _ = oracle.layer_rows_w4a8(ow, H, oc, prompt[sample].reshape(-1, h), np.repeat(np.arange(len(sample)), P),
                                    np.tile(np.arange(P), len(sample)), nthreads=len(sample), keep_cache=True)
    return ref


def _decode_ref(ow, H, gc, x_rows, sample, p, maxL):
    oc = _gpu_cache(gc, sample, maxL)
    r, _ = oracle.layer_rows_w4a8(ow, H, oc, x_rows, np.arange(len(sample)), np.full(len(sample), p),
                                  nthreads=len(sample), keep_cache=True)
    return r


def _layer(h, H, F, seed, **kw):
    cfg = fg.LayerConfig(h, H, F, act_bits=8)
    w16 = si.layer_weights_f16(seed, h, F, **kw)
    gw = fg.LayerWeights.from_fp16(cfg, w16)
    ow = oracle.W4A8LayerWeights(w16)
    for name in MATS:  # the GPU's W4A8 weights equal the oracle's bit for bit
        m, r = gw.w4a8_matrix(name), getattr(ow, name)
        assert np.array_equal(m.codes.cpu().numpy(), r.codes)
        assert np.array_equal(m.gmin.cpu().numpy(), r.gmin)
        assert np.array_equal(m.gstep.cpu().numpy(), r.gstep)
        assert np.array_equal(m.cscale.cpu().numpy().view(np.uint32), r.cscale.view(np.uint32))
    return cfg, gw, ow


@pytest.mark.parametrize("S", [4, 300])
def test_w4a8_layer_prefill_and_decode(S):
    # 8 heads x 128, a prompt of 40 tokens, then 3 decode steps; S = 300 runs the products on CTA
    # pairs (the prompt's 12000 rows and the decode block), S = 4 the decode products on one SM
    # per tile
    h, H, F, P = 1024, 8, 4096, 40
    cfg, gw, ow = _layer(h, H, F, 23, std=0.03, bias_std=0.05, ln_random=True)
    gc = fg.KVCache(S, H, h // H, 64)
    prompt = si.hidden_block(23, si.STREAM["prompt"], S, P, h)
    sample = np.array([0, S // 2, S - 1]) if S > 4 else np.arange(S)
    out = fg.fg_layer_prefill(cfg, gw, gc, dev(prompt), dev(np.zeros(S, np.int32)), num_gpu_batches=2)
    fg.fg_sync_status()
    rows = prompt[sample].reshape(-1, h)
    ref = _prompt_ref(ow, H, gc, prompt, sample, 64)
    assert delta_err(out.cpu().numpy()[sample].reshape(-1, h), rows, ref) <= TOL
    for t in range(3):
        x = si.decode_inputs(23, t, S, h)
        y = fg.fg_layer_decode(cfg, gw, gc, dev(x), dev(np.full(S, P + t, np.int32)), num_gpu_batches=2)
        fg.fg_sync_status()
        r = _decode_ref(ow, H, gc, x[sample], sample, P + t, 64)
        assert delta_err(y.cpu().numpy()[sample], x[sample], r) <= TOL, t


def test_w4a8_layer_block_split_invariance():
    # one product launch per step over the whole block: 8 x 16 and 1 x 128 give the same bits
    h, H, F, S, P = 768, 12, 3072, 128, 8
    cfg, gw, _ = _layer(h, H, F, 24, std=0.05, bias_std=0.05)
    x = dev(si.decode_inputs(24, 0, S, h))
    pos = dev(np.full(S, P, np.int32))
    outs = []
    for nb in (8, 1):
        c = fg.KVCache(S, H, h // H, 64)
        fg.fg_layer_prefill(cfg, gw, c, dev(si.hidden_block(24, si.STREAM["prompt"], S, P, h)),
                            dev(np.zeros(S, np.int32)), num_gpu_batches=nb)
        outs.append(fg.fg_layer_decode(cfg, gw, c, x, pos, num_gpu_batches=nb))
    fg.fg_sync_status()
    assert torch.equal(outs[0], outs[1])


def test_w4a8_opt6p7b_block_decode_sampled_sequences():
    # the OPT-6.7B-shaped block (8 x 64 sequences, prompt 512) in the W4A8 form, decode steps at
    # positions 512 and 513; the oracle checks sampled sequences
    h, H, F, nb, gbs, P = 4096, 32, 16384, 8, 64, 512
    S = nb * gbs
    maxL = 576
    cfg, gw, ow = _layer(h, H, F, 25)
    gc = fg.KVCache(S, H, h // H, maxL)
    prompt = si.hidden_block(25, si.STREAM["prompt"], S, P, h)
    fg.fg_layer_prefill(cfg, gw, gc, dev(prompt), dev(np.zeros(S, np.int32)), num_gpu_batches=nb)
    fg.fg_sync_status()
    sample = np.array([0, 130, 301, 511])
    del prompt
    for t in range(2):
        x = si.decode_inputs(25, t, S, h)
        y = fg.fg_layer_decode(cfg, gw, gc, dev(x), dev(np.full(S, P + t, np.int32)), num_gpu_batches=nb)
        fg.fg_sync_status()
        r = _decode_ref(ow, H, gc, x[sample], sample, P + t, maxL)
        assert delta_err(y.cpu().numpy()[sample], x[sample], r) <= TOL, t


def _ws_taps(ws, R, h, F):
    """The activations a decode call leaves in its workspace (the layout fg.h states)."""
    al = lambda x: (x + 255) // 256 * 256
    wsn = ws.cpu().numpy()
    off, p = {}, 0
    for name, n in (("a", R * h * 2), ("qkv", R * 3 * h * 2), ("o", R * h * 2), ("h1", R * h * 2), ("f", R * F * 2)):
        off[name] = p
        p = al(p + n)
    off["a8"] = p
    p = al(p + R * max(F, h))
    off["as"] = p
    f16 = lambda n, c: wsn[off[n]:off[n] + R * c * 2].view(np.float16).reshape(R, c)
    return dict(qkv=f16("qkv", 3 * h), o=f16("o", h), h1=f16("h1", h), f=f16("f", F),
                a8=wsn[off["a8"]:off["a8"] + R * F].view(np.int8).reshape(R, F),
                as_=wsn[off["as"]:off["as"] + R * 4].view(np.float32))


def _close(got, ref, mag):
    """One fp16 ulp of the reference plus 2^-21 of the magnitudes that enter its sums (the W4A8
    product's epilogue bound, as in the product's own tests)."""
    ulp = np.maximum(np.spacing(np.abs(ref).astype(np.float16)).astype(np.float64), 2.0 ** -24)
    return np.all(np.abs(got.astype(np.float64) - ref) <= ulp + mag * 2.0 ** -21 + 2.0 ** -24)


@pytest.mark.parametrize("S", [4, 300])
def test_w4a8_decode_step_stage_by_stage(S):
    # every stage of a W4A8 decode step against the oracle's pieces applied to the GPU's own input
    # of that stage: the activation codes and scales bit-exact, each product within its epilogue
    # bound, attention over the GPU's cache at the fp16 attention tolerance
    h, H, F, P = 1024, 8, 4096, 40
    d = h // H
    cfg, gw, ow = _layer(h, H, F, 26, std=0.03, bias_std=0.05, ln_random=True)
    w16 = si.layer_weights_f16(26, h, F, std=0.03, bias_std=0.05, ln_random=True)
    gc = fg.KVCache(S, H, d, 64)
    fg.fg_layer_prefill(cfg, gw, gc, dev(si.hidden_block(26, si.STREAM["prompt"], S, P, h)),
                        dev(np.zeros(S, np.int32)), num_gpu_batches=2)
    x = si.decode_inputs(26, 0, S, h)
    ws = torch.zeros(cfg.workspace_bytes(S), dtype=torch.uint8, device="cuda")
    y = fg.fg_layer_decode(cfg, gw, gc, dev(x), dev(np.full(S, P, np.int32)), num_gpu_batches=2, workspace=ws)
    fg.fg_sync_status()
    t = _ws_taps(ws, S, h, F)
    f16 = oracle.f64_to_f16
    # QKV from the LayerNorm of x (fp16 rows both sides decide the same codes unless LN differs by an ulp)
    a8, s = oracle.act8_quantize(f16(oracle.layernorm(x, w16["ln1_g"], w16["ln1_b"])))
    rq, acc = oracle.linear_w4a8(a8, s, ow.wqkv, bias=w16["bqkv"], qscale_cols=h, qscale=1 / np.sqrt(d), with_acc=True)
    assert np.max(np.abs(t["qkv"].astype(np.float64) - rq)) <= 4 * np.max(np.spacing(np.abs(rq).astype(np.float16)))
    # attention over the GPU's cache with the GPU's q
    oc = _gpu_cache(gc, np.arange(S), 64)
    ro = oracle.attention(oc, t["qkv"][:, :h], np.arange(S), np.full(S, P + 1))
    assert np.max(np.abs(t["o"].astype(np.float64) - ro)) <= 2e-3 * np.max(np.abs(ro))
    # output projection + residual from the GPU's o
    o8, so = oracle.act8_quantize(t["o"])
    r1, acc1 = oracle.linear_w4a8(o8, so, ow.wo, bias=w16["bo"], residual=x, with_acc=True)
    mag1 = (np.abs(acc1) * (so[:, None].astype(np.float64) * ow.wo.cscale[None, :]) + np.abs(x.astype(np.float64))
            + np.abs(w16["bo"].astype(np.float64))[None, :])
    assert _close(t["h1"], r1, mag1)
    # FC1 + ReLU from the GPU's h1
    a28, s2 = oracle.act8_quantize(f16(oracle.layernorm(t["h1"], w16["ln2_g"], w16["ln2_b"])))
    rf = oracle.linear_w4a8(a28, s2, ow.w1, bias=w16["b1"], relu=True)
    assert np.max(np.abs(t["f"].astype(np.float64) - rf)) <= 4 * np.max(np.spacing(np.abs(rf).astype(np.float16)))
    # FC2's int8 input: bit-exact with the oracle's quantiser on the GPU's f
    f8, sf = oracle.act8_quantize(t["f"])
    assert np.array_equal(t["a8"], f8) and np.array_equal(t["as_"].view(np.uint32), sf.view(np.uint32))
    # FC2 + residual from the GPU's f and h1
    ry, acc2 = oracle.linear_w4a8(f8, sf, ow.w2, bias=w16["b2"], residual=t["h1"], with_acc=True)
    mag2 = np.abs(acc2) * (sf[:, None].astype(np.float64) * ow.w2.cscale[None, :]) + np.abs(t["h1"].astype(np.float64))
    assert _close(y.cpu().numpy(), ry, mag2 + np.abs(w16["b2"].astype(np.float64))[None, :])


def test_w4a8_stack_streamed_equals_resident_layers():
    # the W4A8 blobs streamed from pinned host memory in slices (the stack's sliced prefetch) give
    # the same bits as the same layers run from resident device blobs
    nl, h, H, F, S, P = 3, 256, 4, 512, 8, 12
    cfg = fg.LayerConfig(h, H, F, act_bits=8)
    w16 = [si.layer_weights_f16(27 + l, h, F, std=0.05, bias_std=0.05, ln_random=True) for l in range(nl)]
    dev_w = [fg.LayerWeights.from_fp16(cfg, w) for w in w16]
    host = [torch.empty(cfg.blob_bytes(), dtype=torch.uint8, pin_memory=True) for _ in range(nl)]
    for hb, dw in zip(host, dev_w):
        hb.copy_(dw.blob)
    st = fg.Stack(cfg, host)
    caches = [fg.KVCache(S, H, h // H, 64) for _ in range(nl)]
    st.prefill(caches, dev(si.hidden_block(27, si.STREAM["prompt"], S, P, h)), dev(np.zeros(S, np.int32)))
    x = dev(si.decode_inputs(27, 0, S, h))
    pos = dev(np.full(S, P, np.int32))
    snap = [[a.clone() for a in c.arrays()] for c in caches]
    y = st.decode(caches, x, pos, num_gpu_batches=2)
    torch.cuda.synchronize()
    after = [[a.clone() for a in c.arrays()] for c in caches]
    for c, s in zip(caches, snap):
        for a, b in zip(c.arrays(), s):
            a.copy_(b)
    z = x
    for l in range(nl):
        z = fg.fg_layer_decode(cfg, dev_w[l], caches[l], z, pos, num_gpu_batches=2)
    fg.fg_sync_status()
    assert torch.equal(y, z)
    for c, s in zip(caches, after):
        for a, b in zip(c.arrays(), s):
            assert torch.equal(a, b)
    st.close()
