"""GPU parity of the whole OPT layer (prefill + decode), the block schedule and the stack.

Tolerance (the stated layer bound): max relative error 1e-2 of the layer output
against the oracle's float64 evaluation of the same dequantised weights, read
as max|gpu - ref| <= 1e-2 * max|ref| on D = x_out - x_in (the residual
stream would otherwise hide errors in the attention and FFN branches).
"""
import numpy as np
import pytest
import torch

import oracle
import seeded_inputs as si

pytestmark = pytest.mark.gpu
fg = None
TOL = 1e-2


@pytest.fixture(autouse=True)
def _bind_library(fg_lib):
    global fg
    fg = fg_lib


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def delta_err(out_gpu, x16, ref):
    """max|D_gpu - D_ref| / max|D_ref| with D = out - x."""
    x = x16.astype(np.float64)
    d_gpu = out_gpu.astype(np.float64) - x
    d_ref = ref - x
    return np.max(np.abs(d_gpu - d_ref)) / np.max(np.abs(d_ref))


class Layer:
    """A layer set up identically on the GPU and in the oracle."""

    def __init__(self, h, H, F, S, maxL, seed=0, std=0.02, bias_std=0.0, ln_random=False, group=64):
        self.h, self.H, self.F, self.S, self.maxL = h, H, F, S, maxL
        self.cfg = fg.LayerConfig(h, H, F, group=group)
        self.w16 = si.layer_weights_f16(seed, h, F, std=std, bias_std=bias_std, ln_random=ln_random)
        self.gw = fg.LayerWeights.from_fp16(self.cfg, self.w16)
        self.ow = oracle.LayerWeights(self.w16, group=group)
        # the GPU's packed weights equal the oracle's bit for bit
        for name in ("wqkv", "wo", "w1", "w2"):
            m = self.gw.matrix(name)
            assert np.array_equal(m.codes.cpu().numpy(), getattr(self.ow, name).codes)
            assert np.array_equal(m.scales.cpu().numpy().view(np.uint16), getattr(self.ow, name).scales.view(np.uint16))
        self.gc = fg.KVCache(S, H, h // H, maxL, group=group)
        self.oc = oracle.KVCache(S, H, h // H, maxL, group=group)


def run_opt125m(bias_std=0.0, ln_random=False, nb=1):
    # OPT-125M-shaped layer: hidden 768, 12 heads x 64, FFN 3072; batch 4, prompt 32, 8 decode steps
    h, H, F, S, P, steps = 768, 12, 3072, 4, 32, 8
    L = Layer(h, H, F, S, 64, seed=0, bias_std=bias_std, ln_random=ln_random)
    prompt = si.hidden_block(0, si.STREAM["prompt"], S, P, h)
    out = fg.fg_layer_prefill(L.cfg, L.gw, L.gc, dev(prompt), dev(np.zeros(S, np.int32)), num_gpu_batches=nb)
    fg.fg_sync_status()
    rows = prompt.reshape(S * P, h)
    ref, _ = oracle.layer_rows(L.ow, H, L.oc, rows, np.repeat(np.arange(S), P), np.tile(np.arange(P), S),
                               nthreads=4)
    errs = [delta_err(out.cpu().numpy().reshape(S * P, h), rows, ref)]
    for t in range(steps):
        x = si.decode_inputs(0, t, S, h)
        pos = np.full(S, P + t, np.int32)
        y = fg.fg_layer_decode(L.cfg, L.gw, L.gc, dev(x), dev(pos), num_gpu_batches=nb)
        fg.fg_sync_status()
        r, _ = oracle.layer_rows(L.ow, H, L.oc, x, np.arange(S), pos)
        errs.append(delta_err(y.cpu().numpy(), x, r))
    return errs


def test_opt125m_prefill_and_8_decode_steps():
    errs = run_opt125m()
    assert max(errs) <= TOL, errs


def test_opt125m_with_biases_and_layernorm_params():
    errs = run_opt125m(bias_std=0.1, ln_random=True, nb=2)
    assert max(errs) <= TOL, errs


@pytest.mark.parametrize("S", [4, 300])
def test_layer_group128_prefill_and_decode(S):
    # weights and KV cache in groups of 128 ("FlexGen Guide", section 3: groups of 64 or 128):
    # 8 heads x 128, a prompt of 40 tokens, then 3 decode steps; S = 300 takes the CTA-pair
    # GEMM launches with their group-128 metadata
    h, H, F, P = 1024, 8, 4096, 40
    L = Layer(h, H, F, S, 64, seed=22, std=0.03, bias_std=0.05, ln_random=True, group=128)
    assert L.gw.matrix("w1").mins.shape == (F, h // 128)
    prompt = si.hidden_block(22, si.STREAM["prompt"], S, P, h)
    sample = np.array([0, S // 2, S - 1]) if S > 4 else np.arange(S)
    out = fg.fg_layer_prefill(L.cfg, L.gw, L.gc, dev(prompt), dev(np.zeros(S, np.int32)), num_gpu_batches=2)
    fg.fg_sync_status()
    oc = oracle.KVCache(len(sample), H, h // H, 64, group=128)
    rows = prompt[sample].reshape(-1, h)
    ref, _ = oracle.layer_rows(L.ow, H, oc, rows, np.repeat(np.arange(len(sample)), P),
                               np.tile(np.arange(P), len(sample)), nthreads=len(sample))
    assert delta_err(out.cpu().numpy()[sample].reshape(-1, h), rows, ref) <= TOL
    for t in range(3):
        x = si.decode_inputs(22, t, S, h)
        y = fg.fg_layer_decode(L.cfg, L.gw, L.gc, dev(x), dev(np.full(S, P + t, np.int32)), num_gpu_batches=2)
        fg.fg_sync_status()
        r, _ = oracle.layer_rows(L.ow, H, oc, x[sample], np.arange(len(sample)), np.full(len(sample), P + t),
                                 nthreads=len(sample))
        assert delta_err(y.cpu().numpy()[sample], x[sample], r) <= TOL, t


def test_ragged_positions_and_peaked_attention():
    # sequences at different cache positions; larger weights sharpen the softmax
    h, H, F, S = 256, 2, 512, 5
    L = Layer(h, H, F, S, 192, seed=3, std=0.08, bias_std=0.1, ln_random=True)
    starts = np.array([0, 1, 63, 64, 130], np.int32)
    for s in range(S):
        if starts[s]:
            p = si.hidden_rows(3, si.STREAM["prompt"], [s], 192, h, 0, int(starts[s]))[0]
            fg.fg_layer_prefill(L.cfg, L.gw, L.gc.view(s, 1), dev(p[None]), dev(np.zeros(1, np.int32)))
            oracle.layer_rows(L.ow, H, L.oc, p, np.full(len(p), s), np.arange(len(p)))
    x = si.decode_inputs(3, 0, S, h)
    y = fg.fg_layer_decode(L.cfg, L.gw, L.gc, dev(x), dev(starts))
    fg.fg_sync_status()
    r, _ = oracle.layer_rows(L.ow, H, L.oc, x, np.arange(S), starts)
    assert delta_err(y.cpu().numpy(), x, r) <= TOL


def test_block_split_invariance():
    # "FlexGen Guide" section 2: the block's batches share the loaded weights; the same
    # block split as 8 x 16 or 1 x 128 gives identical bits, and batch-by-batch calls agree
    h, H, F, S, P = 512, 4, 1024, 128, 16
    L = Layer(h, H, F, S, 64, seed=4)
    prompt = dev(si.hidden_block(4, si.STREAM["prompt"], S, P, h))
    fg.fg_layer_prefill(L.cfg, L.gw, L.gc, prompt, dev(np.zeros(S, np.int32)))
    x = dev(si.decode_inputs(4, 0, S, h))
    pos = dev(np.full(S, P, np.int32))
    snapshot = [a.clone() for a in L.gc.arrays()]
    y1 = fg.fg_layer_decode(L.cfg, L.gw, L.gc, x, pos, num_gpu_batches=8, gpu_batch_size=16)
    for a, b in zip(L.gc.arrays(), snapshot):
        a.copy_(b)
    y2 = fg.fg_layer_decode(L.cfg, L.gw, L.gc, x, pos, num_gpu_batches=1, gpu_batch_size=128)
    assert torch.equal(y1, y2)
    for a, b in zip(L.gc.arrays(), snapshot):
        a.copy_(b)
    parts = []
    for j in range(8):
        sl = slice(16 * j, 16 * (j + 1))
        parts.append(fg.fg_layer_decode(L.cfg, L.gw, L.gc.view(16 * j, 16), x[sl].contiguous(),
                                        pos[sl].contiguous()))
    y3 = torch.cat(parts)
    xd = x.double()
    d1, d3 = (y1.double() - xd), (y3.double() - xd)
    assert (d1 - d3).abs().max().item() <= TOL * d1.abs().max().item()


def test_prefill_equals_token_by_token_decode():
    h, H, F, S, P = 256, 4, 512, 3, 20
    L = Layer(h, H, F, S, 64, seed=5, bias_std=0.1)
    prompt = si.hidden_block(5, si.STREAM["prompt"], S, P, h)
    a = fg.fg_layer_prefill(L.cfg, L.gw, L.gc, dev(prompt), dev(np.zeros(S, np.int32))).cpu().numpy()
    c2 = fg.KVCache(S, H, h // H, 64)
    outs = []
    for t in range(P):
        outs.append(fg.fg_layer_decode(L.cfg, L.gw, c2, dev(prompt[:, t]), dev(np.full(S, t, np.int32))).cpu().numpy())
    b = np.stack(outs, axis=1)
    x = prompt.astype(np.float64)
    assert np.max(np.abs((a - x) - (b - x))) <= TOL * np.max(np.abs(a - x))


def test_decode_rejects_bad_arguments():
    h, H, F, S = 256, 4, 512, 2
    L = Layer(h, H, F, S, 64)
    x = dev(si.decode_inputs(6, 0, S, h))
    with pytest.raises(fg.FgError, match="SHAPE"):
        fg.fg_layer_decode(L.cfg, L.gw, L.gc, x, dev(np.zeros(S, np.int32)), num_gpu_batches=3, gpu_batch_size=1)
    with pytest.raises(fg.FgError, match="WORKSPACE"):
        fg.fg_layer_decode(L.cfg, L.gw, L.gc, x, dev(np.zeros(S, np.int32)),
                           workspace=torch.empty(1024, dtype=torch.uint8, device="cuda"))
    fg.fg_layer_decode(L.cfg, L.gw, L.gc, x, dev(np.full(S, 64, np.int32)))   # position == max_len
    with pytest.raises(fg.FgError, match="RANGE"):
        fg.fg_sync_status()


# ------------------------------------------------------------------ stack ---------------

def _stack_setup(nlayers=3, h=256, H=4, F=512, S=8, P=12, seed=7):
    cfg = fg.LayerConfig(h, H, F)
    w16 = [si.layer_weights_f16(seed + l, h, F, std=0.05, bias_std=0.05, ln_random=True) for l in range(nlayers)]
    dev_w = [fg.LayerWeights.from_fp16(cfg, w) for w in w16]
    host = [torch.empty(cfg.blob_bytes(), dtype=torch.uint8, pin_memory=True) for _ in range(nlayers)]
    for hb, dw in zip(host, dev_w):
        hb.copy_(dw.blob)
    return cfg, w16, dev_w, host


def _oracle_chain(w16, H, prompt, xs, P):
    """The oracle's layers chained through fp16 activations: a prompt of P tokens per sequence,
    then one decode step per entry of `xs` at positions P, P+1, ...  Returns, per layer l, the
    fp16 prompt rows that enter layer l, the fp16 decode inputs of layer l (one per step) and
    the layer's float64 decode outputs (one per step)."""
    nl, S, h = len(w16), prompt.shape[0], prompt.shape[2]
    oc = [oracle.KVCache(S, H, h // H, 64) for _ in range(nl)]
    ow = [oracle.LayerWeights(w) for w in w16]
    rows = prompt.reshape(S * P, h)
    seq, tpos = np.repeat(np.arange(S), P), np.tile(np.arange(P), S)
    prompt_in, dec_in, dec_out = [], [[] for _ in range(nl)], [[] for _ in range(nl)]
    for l in range(nl):
        prompt_in.append(rows.reshape(S, P, h))
        r, _ = oracle.layer_rows(ow[l], H, oc[l], rows, seq, tpos)
        rows = oracle.f64_to_f16(r)
    for t, x in enumerate(xs):
        xin = x
        for l in range(nl):
            r, _ = oracle.layer_rows(ow[l], H, oc[l], xin, np.arange(S), np.full(S, P + t))
            dec_in[l].append(xin)
            dec_out[l].append(r)
            xin = oracle.f64_to_f16(r)
    return prompt_in, dec_in, dec_out


def _chain_bound(dec_in, dec_out, t):
    """Tolerance of a chain of layers compared end to end (step t): each layer's Delta may be off
    by 1e-2 of its own largest magnitude, and the residual stream carries an earlier layer's
    error on to the output unchanged (to first order), so the budgets add up."""
    return TOL * sum(np.max(np.abs(dec_out[l][t] - dec_in[l][t].astype(np.float64))) for l in range(len(dec_in)))


def test_stack_streamed_equals_resident_layers_and_oracle():
    nl, h, H, F, S, P = 3, 256, 4, 512, 8, 12
    cfg, w16, dev_w, host = _stack_setup(nl, h, H, F, S, P)
    st = fg.Stack(cfg, host)
    caches = [fg.KVCache(S, H, h // H, 64) for _ in range(nl)]
    prompt = si.hidden_block(8, si.STREAM["prompt"], S, P, h)
    st.prefill(caches, dev(prompt), dev(np.zeros(S, np.int32)))
    x = si.decode_inputs(8, 0, S, h)
    pos = dev(np.full(S, P, np.int32))
    snap = [[a.clone() for a in c.arrays()] for c in caches]
    y = st.decode(caches, dev(x), pos, num_gpu_batches=2)
    torch.cuda.synchronize()
    # the same layers run one by one from resident device blobs give the same bits
    for c, s in zip(caches, snap):
        for a, b in zip(c.arrays(), s):
            a.copy_(b)
    z = dev(x)
    for l in range(nl):
        z = fg.fg_layer_decode(cfg, dev_w[l], caches[l], z, pos, num_gpu_batches=2)
    assert torch.equal(y, z)
    # Each layer of the chain against the oracle at the layer bound: GPU layer l is given the
    # oracle's own fp16 inputs to layer l (its prompt rows, to fill its cache, and its decode
    # rows); with the bit equalities above this covers every layer of the streamed stack.
    prompt_in, dec_in, dec_out = _oracle_chain(w16, H, prompt, [x], P)
    for l in range(nl):
        c = fg.KVCache(S, H, h // H, 64)
        fg.fg_layer_prefill(cfg, dev_w[l], c, dev(prompt_in[l]), dev(np.zeros(S, np.int32)))
        yl = fg.fg_layer_decode(cfg, dev_w[l], c, dev(dec_in[l][0]), pos, num_gpu_batches=2)
        fg.fg_sync_status()
        assert delta_err(yl.cpu().numpy(), dec_in[l][0], dec_out[l][0]) <= TOL, l
    # the streamed stack end to end against the oracle's chain, at the chain's summed bound
    err = np.max(np.abs(y.cpu().numpy().astype(np.float64) - dec_out[-1][0]))
    assert err <= _chain_bound(dec_in, dec_out, 0)


def test_pipeline_stage_runs_its_layers_on_the_gpu():
    # Pipeline parallelism ("A 175B-parameter model on one GPU, if you can wait", key
    # highlights): one stage holding all three layers (world size 1, so no send or receive),
    # the block cut into two micro-batches.  Its layer_runner must give what the same layers
    # give over the whole block, and the oracle's chained layers within the chain's bound.
    from bit_compressed_decode_b200 import pipeline
    nl, h, H, F, S, P = 3, 256, 4, 512, 8, 12
    cfg, w16, dev_w, _ = _stack_setup(nl, h, H, F, S, P, seed=17)
    prompt = si.hidden_block(12, si.STREAM["prompt"], S, P, h)
    caches = [fg.KVCache(S, H, h // H, 64) for _ in range(nl)]
    z = dev(prompt)
    for l in range(nl):
        z = fg.fg_layer_prefill(cfg, dev_w[l], caches[l], z, dev(np.zeros(S, np.int32)))
    snap = [[a.clone() for a in c.arrays()] for c in caches]
    x = si.decode_inputs(12, 0, S, h)
    pos = dev(np.full(S, P, np.int32))
    parts = pipeline.micro_batches(S, 2)
    ws = torch.empty(cfg.workspace_bytes(max(n for _, n in parts)), dtype=torch.uint8, device="cuda")
    stage = pipeline.PipelineStage(pipeline.layer_runner(cfg, dev_w, caches, pos, ws), h, rank=0, world=1)
    y = stage.step(dev(x), parts)
    fg.fg_sync_status()
    for c, sn in zip(caches, snap):
        for a, b in zip(c.arrays(), sn):
            a.copy_(b)
    z = dev(x)
    for l in range(nl):
        z = fg.fg_layer_decode(cfg, dev_w[l], caches[l], z, pos)
    xd = dev(x).double()
    assert (y.double() - z.double()).abs().max().item() <= TOL * (z.double() - xd).abs().max().item()
    _, dec_in, dec_out = _oracle_chain(w16, H, prompt, [x], P)
    err = np.max(np.abs(y.cpu().numpy().astype(np.float64) - dec_out[-1][0]))
    assert err <= _chain_bound(dec_in, dec_out, 0)


def test_stack_copy_failure_is_reported_and_recoverable():
    nl, h, H, F, S, P = 3, 256, 4, 512, 4, 4
    cfg, _, _, host = _stack_setup(nl, h, H, F, S, P)
    st = fg.Stack(cfg, host)
    caches = [fg.KVCache(S, H, h // H, 64) for _ in range(nl)]
    x = dev(si.decode_inputs(9, 0, S, h))
    pos = dev(np.zeros(S, np.int32))
    st.inject_copy_failure(1)
    with pytest.raises(fg.FgError, match="CUDA"):
        st.decode(caches, x, pos)
    y = st.decode(caches, x, pos)        # the next step runs normally
    fg.fg_sync_status()
    assert torch.isfinite(y.float()).all()
    st.close()


@pytest.mark.parametrize("ragged", [False, True])
def test_stack_host_kv_equals_device_kv(ragged):
    # Caches spilled to pinned host memory, filled into two device staging caches layer by
    # layer, give the same bits as the caches resident in HBM: the output of two decode
    # steps and, after the write-back of the new slots, the host caches themselves.
    nl, h, H, F, S, P, maxL = 3, 256, 4, 512, 8, 12, 64
    cfg, w16, _, host = _stack_setup(nl, h, H, F, S, P)
    st = fg.Stack(cfg, host)
    caches = [fg.KVCache(S, H, h // H, maxL) for _ in range(nl)]
    st.prefill(caches, dev(si.hidden_block(10, si.STREAM["prompt"], S, P, h)), dev(np.zeros(S, np.int32)))
    torch.cuda.synchronize()
    hcaches = [fg.KVCache(S, H, h // H, maxL, device="cpu", pin_memory=True) for _ in range(nl)]
    for hc, c in zip(hcaches, caches):
        for a, b in zip(hc.arrays(), c.arrays()):
            a.copy_(b)
    # staging caches start with arbitrary bytes (NaN and inf metadata included): slots past a
    # sequence's length are never read
    g = torch.Generator(device="cuda").manual_seed(3)
    staging = [fg.KVCache(S, H, h // H, maxL) for _ in range(2)]
    for c in staging:
        for a in c.arrays():
            a.view(torch.uint8).copy_(torch.randint(0, 256, a.view(torch.uint8).shape, dtype=torch.uint8,
                                                    device="cuda", generator=g))
    cs, ps = torch.cuda.Stream(), torch.cuda.Stream()
    zs = []
    for t in range(2):
        p = np.full(S, P + t, np.int32) + (np.arange(S, dtype=np.int32) % 3 if ragged else 0)
        x = dev(si.decode_inputs(10, t, S, h))
        y = st.decode(caches, x, dev(p), num_gpu_batches=2)
        torch.cuda.synchronize()
        # ragged: slots that some sequences skip are filled so the write-back returns them intact
        fill = int(p.max()) + (1 if ragged else 0)
        z = st.decode_host_kv(hcaches, staging, x, dev(p), fill, int(p.min()), int(p.max()) + 1,
                              num_gpu_batches=2, compute_stream=cs, copy_stream=ps)
        ps.synchronize()
        cs.synchronize()
        fg.fg_sync_status()
        assert torch.equal(y, z)
        zs.append(z.cpu().numpy())
    for hc, c in zip(hcaches, caches):
        for a, b in zip(hc.arrays(), c.arrays()):
            assert torch.equal(a, b.cpu())
    st.close()
    if not ragged:
        # both decode steps of the host-KV stack against the oracle's chained layers, at the
        # chain's summed bound (the per-layer bound is checked on the same kernels above)
        xs = [si.decode_inputs(10, t, S, h) for t in range(2)]
        _, dec_in, dec_out = _oracle_chain(w16, H, si.hidden_block(10, si.STREAM["prompt"], S, P, h), xs, P)
        for t in range(2):
            err = np.max(np.abs(zs[t].astype(np.float64) - dec_out[-1][t]))
            assert err <= _chain_bound(dec_in, dec_out, t), t


def test_stack_host_kv_rejects_bad_ranges():
    nl, h, H, F, S = 2, 256, 4, 512, 4
    cfg, _, _, host = _stack_setup(nl, h, H, F, S, 4)
    st = fg.Stack(cfg, host)
    hc = [fg.KVCache(S, H, h // H, 64, device="cpu", pin_memory=True) for _ in range(nl)]
    dc = [fg.KVCache(S, H, h // H, 64) for _ in range(2)]
    x, pos = dev(si.decode_inputs(11, 0, S, h)), dev(np.zeros(S, np.int32))
    with pytest.raises(fg.FgError, match="INVALID"):
        st.decode_host_kv(hc, dc, x, pos, 65, 0, 1)          # fill past max_len
    with pytest.raises(fg.FgError, match="INVALID"):
        st.decode_host_kv(hc, dc, x, pos, 0, 2, 1)           # empty-reversed write-back range
    short = [fg.KVCache(S, H, h // H, 128) for _ in range(2)]
    with pytest.raises(fg.FgError, match="SHAPE"):
        st.decode_host_kv(hc, short, x, pos, 0, 0, 1)        # staging geometry differs
    hfew = [fg.KVCache(2, H, h // H, 64, device="cpu", pin_memory=True) for _ in range(nl)]
    few = [fg.KVCache(2, H, h // H, 64) for _ in range(2)]
    with pytest.raises(fg.FgError, match="SHAPE"):
        st.decode_host_kv(hfew, few, x, pos, 0, 0, 1)        # block larger than the caches
    st.close()


# ------------------------------------------------------------------ full size -----------

@pytest.mark.slow
def test_opt6p7b_block_decode_sampled_sequences():
    # OPT-6.7B-shaped layer at full size: 8 x 64 sequences, prompt 512, decode steps at
    # positions 512 and 513 in the launch configuration the benchmark times; the oracle
    # checks sampled sequences (first, last and one per 128-row tile).
    h, H, F, nb, gbs, P = 4096, 32, 16384, 8, 64, 512
    S = nb * gbs
    maxL = 576
    L = Layer(h, H, F, S, maxL, seed=0)
    prompt = si.hidden_block(0, si.STREAM["prompt"], S, P, h)
    fg.fg_layer_prefill(L.cfg, L.gw, L.gc, dev(prompt), dev(np.zeros(S, np.int32)), num_gpu_batches=nb)
    fg.fg_sync_status()
    sample = np.array([0, 130, 301, 511])
    oc = oracle.KVCache(len(sample), H, h // H, maxL)
    rows = prompt[sample].reshape(-1, h)
    oracle.layer_rows(L.ow, H, oc, rows, np.repeat(np.arange(len(sample)), P),
                      np.tile(np.arange(P), len(sample)), kv_only=True, nthreads=len(sample))
    del prompt
    for t in range(2):
        x = si.decode_inputs(0, t, S, h)
        y = fg.fg_layer_decode(L.cfg, L.gw, L.gc, dev(x), dev(np.full(S, P + t, np.int32)), num_gpu_batches=nb)
        fg.fg_sync_status()
        r, _ = oracle.layer_rows(L.ow, H, oc, x[sample], np.arange(len(sample)), np.full(len(sample), P + t),
                                 nthreads=len(sample))
        assert delta_err(y.cpu().numpy()[sample], x[sample], r) <= TOL


@pytest.mark.slow
@pytest.mark.parametrize("shape", ["opt-30b", "opt-175b"])
def test_large_layer_shapes_sampled_sequences(shape):
    # One layer of the OPT-30B shape (hidden 7168, 56 heads, FFN 28672; block 4 x 64) and of the
    # OPT-175B shape (hidden 12288, 96 heads, FFN 49152; block 8 x 32): 256 sequences, so every
    # GEMM gets the launch plan (tile, k splits) of the stack workloads.  Both sides start from
    # the same 4-bit cache: 64 cached positions of seeded k and v appended by each side's own
    # quantiser (bit-equal, checked), drawn with the spread the layer's own k and v have
    # (N(0, (0.02 sqrt(h))^2): unit-variance LayerNorm rows times N(0, 0.02^2) weights over h
    # inputs); then two decode steps.  The oracle checks sampled sequences, one from each quarter
    # of the block.
    h, H, F, nb, gbs = {"opt-30b": (7168, 56, 28672, 4, 64), "opt-175b": (12288, 96, 49152, 8, 32)}[shape]
    S, P, maxL = nb * gbs, 64, 128
    d = h // H
    kv_std = 0.02 * np.sqrt(h)
    L = Layer(h, H, F, S, maxL, seed=0)
    sample = np.array([0, S // 3, (2 * S) // 3 + 1, S - 1])
    oc = oracle.KVCache(len(sample), H, d, maxL)
    for i, s in enumerate(sample):
        k = si.normal_f16(0, si.STREAM["k_new"], (P, h), kv_std, start=int(s) * P * h)
        v = si.normal_f16(0, si.STREAM["v_new"], (P, h), kv_std, start=int(s) * P * h)
        oracle.kv_append(oc, k, v, np.full(P, i), np.arange(P))
    kall = si.normal_f16(0, si.STREAM["k_new"], (S * P, h), kv_std)
    vall = si.normal_f16(0, si.STREAM["v_new"], (S * P, h), kv_std)
    fg.fg_kv_append(L.gc, dev(kall), dev(vall), dev(np.zeros(S, np.int32)), rows_per_seq=P)
    fg.fg_sync_status()
    del kall, vall
    for a, b in zip(L.gc.arrays(), oc.arrays()):
        got = a[torch.from_numpy(sample).cuda()].cpu().numpy()
        assert np.array_equal(got.view(np.uint16) if got.dtype == np.float16 else got, b)
    for t in range(2):
        x = si.decode_inputs(0, t, S, h)
        y = fg.fg_layer_decode(L.cfg, L.gw, L.gc, dev(x), dev(np.full(S, P + t, np.int32)), num_gpu_batches=nb)
        fg.fg_sync_status()
        r, _ = oracle.layer_rows(L.ow, H, oc, x[sample], np.arange(len(sample)), np.full(len(sample), P + t),
                                 nthreads=len(sample))
        assert delta_err(y.cpu().numpy()[sample], x[sample], r) <= TOL, t


def test_stack_one_staging_buffer_equals_resident_layers():
    # one staging blob, refilled slice by slice as the layer before finishes with each slice:
    # prefill and decode give the same bits as the layers run from resident device blobs
    nl, h, H, F, S, P = 3, 256, 4, 512, 8, 12
    cfg, w16, dev_w, host = _stack_setup(nl, h, H, F, S, P, seed=17)
    st = fg.Stack(cfg, host, staging_buffers=1)
    caches = [fg.KVCache(S, H, h // H, 64) for _ in range(nl)]
    prompt = dev(si.hidden_block(17, si.STREAM["prompt"], S, P, h))
    yp = st.prefill(caches, prompt, dev(np.zeros(S, np.int32)))
    ref_caches = [fg.KVCache(S, H, h // H, 64) for _ in range(nl)]
    z = prompt
    for l in range(nl):
        z = fg.fg_layer_prefill(cfg, dev_w[l], ref_caches[l], z, dev(np.zeros(S, np.int32)))
    torch.cuda.synchronize()
    assert torch.equal(yp, z)
    x = dev(si.decode_inputs(17, 0, S, h))
    pos = dev(np.full(S, P, np.int32))
    y = st.decode(caches, x, pos, num_gpu_batches=2)
    z = x
    for l in range(nl):
        z = fg.fg_layer_decode(cfg, dev_w[l], ref_caches[l], z, pos, num_gpu_batches=2)
    fg.fg_sync_status()
    assert torch.equal(y, z)
    for c, r in zip(caches, ref_caches):
        for a, b in zip(c.arrays(), r.arrays()):
            assert torch.equal(a, b)
    st.close()


@pytest.mark.parametrize("buffers", [2, 1])
def test_stack_with_resident_layers_equals_streamed(buffers):
    # layers whose blobs sit in device memory are read in place (no copy, no staging buffer);
    # mixed with streamed ones, prefill and decode give the bits of the all-streamed stack
    nl, h, H, F, S, P = 4, 256, 4, 512, 8, 12
    cfg, w16, dev_w, host = _stack_setup(nl, h, H, F, S, P, seed=19)
    mixed = [dw.blob if l in (0, 2) else hb for l, (dw, hb) in enumerate(zip(dev_w, host))]
    runs = []
    for blobs in (host, mixed):
        st = fg.Stack(cfg, blobs, staging_buffers=buffers)
        caches = [fg.KVCache(S, H, h // H, 64) for _ in range(nl)]
        yp = st.prefill(caches, dev(si.hidden_block(19, si.STREAM["prompt"], S, P, h)), dev(np.zeros(S, np.int32)))
        y = st.decode(caches, dev(si.decode_inputs(19, 0, S, h)), dev(np.full(S, P, np.int32)), num_gpu_batches=2)
        fg.fg_sync_status()
        runs.append((yp.clone(), y.clone(), [[a.clone() for a in c.arrays()] for c in caches]))
        st.close()
    assert torch.equal(runs[0][0], runs[1][0]) and torch.equal(runs[0][1], runs[1][1])
    for c0, c1 in zip(runs[0][2], runs[1][2]):
        for a, b in zip(c0, c1):
            assert torch.equal(a, b)


def test_stack_host_kv_with_resident_layers():
    # host-spilled caches with the weights of layers 0 and 2 resident in device memory (read in
    # place; their KV caches still filled into the staging caches and written back): the same
    # bits as the HBM-resident caches and all-streamed weights
    nl, h, H, F, S, P, maxL = 3, 256, 4, 512, 8, 12, 64
    cfg, w16, dev_w, host = _stack_setup(nl, h, H, F, S, P, seed=21)
    st = fg.Stack(cfg, host)
    caches = [fg.KVCache(S, H, h // H, maxL) for _ in range(nl)]
    st.prefill(caches, dev(si.hidden_block(21, si.STREAM["prompt"], S, P, h)), dev(np.zeros(S, np.int32)))
    torch.cuda.synchronize()
    hcaches = [fg.KVCache(S, H, h // H, maxL, device="cpu", pin_memory=True) for _ in range(nl)]
    for hc, c in zip(hcaches, caches):
        for a, b in zip(hc.arrays(), c.arrays()):
            a.copy_(b)
    mixed = fg.Stack(cfg, [dev_w[0].blob, host[1], dev_w[2].blob])
    staging = [fg.KVCache(S, H, h // H, maxL) for _ in range(2)]
    cs, ps = torch.cuda.Stream(), torch.cuda.Stream()
    p = np.full(S, P, np.int32)
    x = dev(si.decode_inputs(21, 0, S, h))
    y = st.decode(caches, x, dev(p), num_gpu_batches=2)
    z = mixed.decode_host_kv(hcaches, staging, x, dev(p), P, P, P + 1, num_gpu_batches=2, compute_stream=cs,
                             copy_stream=ps)
    ps.synchronize()
    cs.synchronize()
    fg.fg_sync_status()
    assert torch.equal(y, z)
    for hc, c in zip(hcaches, caches):
        for a, b in zip(hc.arrays(), c.arrays()):
            assert torch.equal(a, b.cpu())
    st.close()
    mixed.close()
