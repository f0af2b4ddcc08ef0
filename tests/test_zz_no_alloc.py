"""The allocation-free layer decode (fg_layer_decode_noalloc) against fg_layer_decode.

For callers that can't allocate device memory while decoding (all memory reserved
up front, or hosts that only pass pointers they own), the library offers a decode
entry point whose scratch is a static device array.  It accepts a block only when the
block's whole layer workspace fits the array, so both entry points run the same kernels
with the same launch plans in the same order, and their outputs and caches must agree
bit for bit.  This file is collected last on purpose: if it fails, a run that stops at
the first failure has run everything else.  It must pass alone in a fresh process and
after the other tests.
"""
import numpy as np
import pytest
import torch

import seeded_inputs as si

pytestmark = pytest.mark.gpu


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def test_noalloc_decode_matches_workspace_decode_two_calls(fg_lib):
    fg = fg_lib
    h, H, F, S, P = 768, 12, 3072, 16, 24
    cfg = fg.LayerConfig(h, H, F)
    w16 = si.layer_weights_f16(21, h, F, std=0.05, bias_std=0.05, ln_random=True)
    lw = fg.LayerWeights.from_fp16(cfg, w16)
    ref_cache = fg.KVCache(S, H, h // H, 64)
    fg.fg_layer_prefill(cfg, lw, ref_cache, _dev(si.hidden_block(21, si.STREAM["prompt"], S, P, h)),
                        _dev(np.zeros(S, np.int32)), num_gpu_batches=2)
    na_cache = fg.KVCache(S, H, h // H, 64, arrays=[a.clone() for a in ref_cache.arrays()])
    assert cfg.workspace_bytes(S) <= fg.NOALLOC_SCRATCH_BYTES
    # every tensor the calls touch exists before the first call, so torch allocates nothing later
    xs = [_dev(si.decode_inputs(21, step, S, h)) for step in range(3)]
    ps = [_dev(np.full(S, P + step, np.int32)) for step in range(3)]
    y_ref, y_na = torch.empty_like(xs[0]), torch.empty_like(xs[0])
    ws = torch.empty(cfg.workspace_bytes(S), dtype=torch.uint8, device="cuda")
    for step in range(3):                                   # set-up call, then two calls in a row
        fg.fg_layer_decode(cfg, lw, ref_cache, xs[step], ps[step], num_gpu_batches=2, out=y_ref, workspace=ws)
        torch.cuda.synchronize()
        free_before = torch.cuda.mem_get_info()[0]
        fg.fg_layer_decode_noalloc(cfg, lw, na_cache, xs[step], ps[step], num_gpu_batches=2, out=y_na)
        fg.fg_sync_status()
        free_after = torch.cuda.mem_get_info()[0]
        if step > 0:                                        # after the set-up call nothing is allocated
            assert free_after == free_before, (free_before, free_after)
        assert torch.equal(y_ref, y_na)
        for a, b in zip(ref_cache.arrays(), na_cache.arrays()):
            assert torch.equal(a, b)


def test_noalloc_opt6p7b_block_equals_workspace_decode(fg_lib):
    # The OPT-6.7B-shaped block of 512 sequences: its whole workspace (40 MiB of activations and
    # the GEMMs' split-k scratch) fits the static array; both calls take the same launches.
    fg = fg_lib
    h, H, F, S, P = 4096, 32, 16384, 512, 4
    cfg = fg.LayerConfig(h, H, F)
    assert cfg.workspace_bytes(S) <= fg.NOALLOC_SCRATCH_BYTES
    g = torch.Generator(device="cuda").manual_seed(5)
    lw = fg.LayerWeights(cfg, torch.empty(cfg.blob_bytes(), dtype=torch.uint8, device="cuda"))
    for name, shape in (("wqkv", (3 * h, h)), ("wo", (h, h)), ("w1", (F, h)), ("w2", (h, F))):
        w = torch.randn(shape, generator=g, device="cuda", dtype=torch.float16) * 0.02
        fg.fg_quantize(w, dim=1, out=lw.matrix(name))
    for name in ("bqkv", "bo", "b1", "b2", "ln1_b", "ln2_b"):
        lw.vector(name).normal_(0.0, 0.05, generator=g)
    lw.vector("ln1_g").fill_(1.0)
    lw.vector("ln2_g").fill_(1.0)
    cache = fg.KVCache(S, H, h // H, 64)
    fg.fg_layer_prefill(cfg, lw, cache, torch.randn((S, P, h), generator=g, device="cuda", dtype=torch.float16),
                        torch.zeros(S, dtype=torch.int32, device="cuda"), num_gpu_batches=8)
    snap = [a.clone() for a in cache.arrays()]
    for step in range(2):
        x = torch.randn((S, h), generator=g, device="cuda", dtype=torch.float16)
        pos = torch.full((S,), P + step, dtype=torch.int32, device="cuda")
        y_ref = fg.fg_layer_decode(cfg, lw, cache, x, pos, num_gpu_batches=8)
        ref_arrays = [a.clone() for a in cache.arrays()]
        for a, b in zip(cache.arrays(), snap):
            a.copy_(b)
        y_na = fg.fg_layer_decode_noalloc(cfg, lw, cache, x, pos, num_gpu_batches=8)
        fg.fg_sync_status()
        assert torch.equal(y_ref, y_na)
        for a, b in zip(cache.arrays(), ref_arrays):
            assert torch.equal(a, b)
        snap = ref_arrays


def test_noalloc_rejects_blocks_beyond_the_scratch(fg_lib):
    fg = fg_lib
    h, H, F = 4096, 32, 16384
    cfg = fg.LayerConfig(h, H, F)
    S = 2048                                                # needs ~200 MB of scratch
    assert cfg.workspace_bytes(S) > fg.NOALLOC_SCRATCH_BYTES
    lw = fg.LayerWeights(cfg, torch.zeros(cfg.blob_bytes(), dtype=torch.uint8, device="cuda"))
    cache = fg.KVCache(S, H, h // H, 64)
    x = torch.zeros((S, h), dtype=torch.float16, device="cuda")
    with pytest.raises(fg.FgError, match="WORKSPACE"):
        fg.fg_layer_decode_noalloc(cfg, lw, cache, x, torch.zeros(S, dtype=torch.int32, device="cuda"))


def test_noalloc_w4a8_layer_equals_workspace_decode(fg_lib):
    # the W4A8 form of the layer through the allocation-free entry: same kernels, same bits
    fg = fg_lib
    h, H, F, S, P = 768, 12, 3072, 16, 24
    cfg = fg.LayerConfig(h, H, F, act_bits=8)
    w16 = si.layer_weights_f16(28, h, F, std=0.05, bias_std=0.05, ln_random=True)
    lw = fg.LayerWeights.from_fp16(cfg, w16)
    ref_cache = fg.KVCache(S, H, h // H, 64)
    fg.fg_layer_prefill(cfg, lw, ref_cache, _dev(si.hidden_block(28, si.STREAM["prompt"], S, P, h)),
                        _dev(np.zeros(S, np.int32)), num_gpu_batches=2)
    na_cache = fg.KVCache(S, H, h // H, 64, arrays=[a.clone() for a in ref_cache.arrays()])
    assert cfg.workspace_bytes(S) <= fg.NOALLOC_SCRATCH_BYTES
    x = _dev(si.decode_inputs(28, 0, S, h))
    pos = _dev(np.full(S, P, np.int32))
    y_ref = fg.fg_layer_decode(cfg, lw, ref_cache, x, pos, num_gpu_batches=2)
    y_na = fg.fg_layer_decode_noalloc(cfg, lw, na_cache, x, pos, num_gpu_batches=2)
    fg.fg_sync_status()
    assert torch.equal(y_ref, y_na)
    for a, b in zip(ref_cache.arrays(), na_cache.arrays()):
        assert torch.equal(a, b)
