"""B200-native (sm_100a) deterministic mixture-of-experts layer.

The computation lives in libmok.so (CUDA, C ABI, include/mok.h); this package
is its thin binding (``abi``), torch buffer plumbing (``layer``), the
expert-parallel buffers and phase order (``ep``), the build helper
(``build``) and the seeded input generator (``synth``).
"""
from .abi import (MOK_DTYPE_BF16, MOK_DTYPE_MXFP8, MOK_SCORE_SIGMOID, MOK_SCORE_SOFTMAX, MokError,
                  moe_bwd, moe_bwd_host, moe_cfg, moe_fwd, moe_fwd_host, moe_grads,
                  moe_host_scratch_size, moe_params, moe_quantize_mxfp8, moe_quantize_mxfp8_weights,
                  moe_quantize_mxfp8_weights_both, moe_quantize_mxfp8_weights_t, moe_routing, moe_status, moe_strerror, moe_trace_events,
                  moe_workspace_size)
from .ep import EPRank, EPWorld, exchange_pointers, new_rank_grads, split_params
from .layer import (MoELayer, cfg_for, make_cfg, quantize_mxfp8, quantize_mxfp8_weights,
                    quantize_mxfp8_weights_both, quantize_mxfp8_weights_t)

__all__ = [
    "MOK_DTYPE_BF16", "MOK_DTYPE_MXFP8", "MOK_SCORE_SIGMOID", "MOK_SCORE_SOFTMAX", "MokError",
    "moe_bwd", "moe_bwd_host", "moe_cfg", "moe_fwd", "moe_fwd_host", "moe_grads",
    "moe_host_scratch_size", "moe_params", "moe_quantize_mxfp8", "moe_quantize_mxfp8_weights",
    "moe_quantize_mxfp8_weights_both", "moe_quantize_mxfp8_weights_t", "moe_routing", "moe_status", "moe_strerror", "moe_trace_events",
    "moe_workspace_size", "MoELayer", "cfg_for", "make_cfg", "quantize_mxfp8", "quantize_mxfp8_weights",
    "quantize_mxfp8_weights_both", "quantize_mxfp8_weights_t", "EPRank", "EPWorld", "exchange_pointers",
    "new_rank_grads", "split_params",
]
