"""B200-native Hierarchical Global Attention (HGA): two-level routed sparse
attention behind the C ABI of libhga.so.

Method source: the article "BMW's 16 GB GPU just did what needs an A100"
(seventnews.com), section "What HGA does differently".  The public calls
(``build_summaries``, ``route_chunks``, ``route_groups``, ``attn_fwd``,
``attn_bwd``, ``stage_routed`` ...) mirror the C ABI one to one; ``Buffers``
holds the device buffers of one problem shape and runs a whole segment step;
``StagedKV`` runs the attention on history kept in host memory;
``DecodeState`` generates token by token (hga_decode); ``CausalBuffers``
runs the strictly causal variant (routing per query position);
``StepPipeline`` overlaps host copies with the compute of segment steps.
"""
from .pipeline import StepPipeline
from .binding import (CHECKED_LIB_PATH, EXPORTS, HGA_ALL, HGA_BF16, HGA_ERR_CUDA, HGA_ERR_DEVICE_CHECK,
                      HGA_ERR_INVALID_ARG,
                      HGA_ERR_UNSUPPORTED, HGA_FP32, HGA_OK, LIB_PATH, NOALLOC_MAX_ROWS, Buffers,
                      CausalBuffers, DecodeState, HGAError, Params, StagedKV, attn_bwd_causal, attn_fwd_causal, route_causal,
                      causal_schedule, causal_sched_size,
                      attn_bwd, attn_bwd_noalloc, attn_fwd, build_summaries, decode, build_summaries_rows, device_status, load, route, route_chunks, route_groups,
                      route_attn_fwd, route_widths, selftest_wait, stage_params, stage_routed, version, workspace_size,
                      checked_build, device_check, use_library)

__all__ = ["CHECKED_LIB_PATH", "HGA_ERR_DEVICE_CHECK", "checked_build", "device_check", "use_library",
           "EXPORTS", "HGA_ALL", "HGA_BF16", "HGA_FP32", "HGA_OK", "HGA_ERR_CUDA",
           "HGA_ERR_INVALID_ARG", "HGA_ERR_UNSUPPORTED", "LIB_PATH", "NOALLOC_MAX_ROWS", "Buffers", "HGAError",
           "CausalBuffers", "DecodeState", "Params", "StepPipeline", "attn_bwd_causal", "attn_fwd_causal", "route_causal",
           "causal_schedule", "causal_sched_size", "StagedKV", "decode", "stage_params", "stage_routed", "attn_bwd", "attn_bwd_noalloc", "attn_fwd", "build_summaries", "build_summaries_rows", "device_status", "load", "route", "route_chunks",
           "route_attn_fwd", "route_groups", "route_widths", "selftest_wait", "version", "workspace_size"]
