"""The allocation-free layer decode (fg_layer_decode_noalloc) against fg_layer_decode.

For callers that can't allocate device memory while decoding (all memory reserved
up front, or hosts that only pass pointers they own), the library offers a decode
entry point whose scratch is a static device array.  This file is collected last on
purpose: if it fails, a run that stops at the first failure has run everything else.
It must pass alone in a fresh process and after the other tests.
"""
import numpy as np
import pytest
import torch

import seeded_inputs as si

pytestmark = pytest.mark.gpu
TOL = 1e-2


def test_noalloc_decode_matches_workspace_decode_two_calls(fg_lib):
    fg = fg_lib
    h, H, F, S, P = 768, 12, 3072, 16, 24
    cfg = fg.LayerConfig(h, H, F)
    w16 = si.layer_weights_f16(21, h, F, std=0.05, bias_std=0.05, ln_random=True)
    lw = fg.LayerWeights.from_fp16(cfg, w16)
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    ref_cache = fg.KVCache(S, H, h // H, 64)
    fg.fg_layer_prefill(cfg, lw, ref_cache, dev(si.hidden_block(21, si.STREAM["prompt"], S, P, h)),
                        dev(np.zeros(S, np.int32)), num_gpu_batches=2)
    na_cache = fg.KVCache(S, H, h // H, 64, arrays=[a.clone() for a in ref_cache.arrays()])
    assert cfg.workspace_bytes(S) <= fg.NOALLOC_SCRATCH_BYTES
    for step in range(2):                                   # two calls in a row
        x = dev(si.decode_inputs(21, step, S, h))
        pos = dev(np.full(S, P + step, np.int32))
        y_ref = fg.fg_layer_decode(cfg, lw, ref_cache, x, pos, num_gpu_batches=2)
        y_na = fg.fg_layer_decode_noalloc(cfg, lw, na_cache, x, pos, num_gpu_batches=2)
        fg.fg_sync_status()
        xd = x.double()
        d_ref, d_na = y_ref.double() - xd, y_na.double() - xd
        assert (d_ref - d_na).abs().max().item() <= TOL * d_ref.abs().max().item()
        for a, b in zip(ref_cache.arrays(), na_cache.arrays()):
            assert torch.equal(a, b)


def test_noalloc_rejects_blocks_beyond_the_scratch(fg_lib):
    fg = fg_lib
    h, H, F = 4096, 32, 16384
    cfg = fg.LayerConfig(h, H, F)
    S = 1024                                                # needs ~80 MiB of scratch
    assert cfg.workspace_bytes(S) > fg.NOALLOC_SCRATCH_BYTES
    lw = fg.LayerWeights(cfg, torch.zeros(cfg.blob_bytes(), dtype=torch.uint8, device="cuda"))
    cache = fg.KVCache(S, H, h // H, 64)
    x = torch.zeros((S, h), dtype=torch.float16, device="cuda")
    with pytest.raises(fg.FgError, match="WORKSPACE"):
        fg.fg_layer_decode_noalloc(cfg, lw, cache, x, torch.zeros(S, dtype=torch.int32, device="cuda"))
