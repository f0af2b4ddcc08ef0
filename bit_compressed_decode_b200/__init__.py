"""B200 (sm_100a) group-wise 4-bit decode library: Python binding of ``include/fg.h``.

The CUDA library ``libfg_b200.so`` is built in-tree by
``python -m bit_compressed_decode_b200.build``; importing this package without
it raises ImportError (there is no CPU path).
"""
from ._binding import (  # noqa: F401
    FG_EPI_RELU, FG_EPI_RESIDUAL, FG_GEMM_PERSISTENT, LIB_PATH, STATUS, FgError, KVCache, LayerConfig, LayerWeights, QTensor, Stack,
    fg_attention_decode, fg_attention_decode_append, fg_dequantize, fg_kv_append, fg_layer_decode, fg_layer_prefill, fg_layernorm,
    fg_linear_w4a16, fg_linear_plan, fg_linear_workspace_bytes, fg_qtensor_bytes, fg_quantize, fg_status_string, fg_sync_status,
    fg_profile_enable, fg_profile_collect, PROFILE_SLOTS, fg_layer_decode_noalloc, NOALLOC_SCRATCH_BYTES,
    fg_linear_plan_pairs, fg_linear_classic_scratch_bytes, fg_test_gemm_stall,
    W4A8Weight, fg_w4a8_quantize_weight, fg_act8_quantize, fg_linear_w4a8, fg_linear_w4a8_plan, fg_linear_w4a8_workspace_bytes,
    lib, weights_struct,
)
