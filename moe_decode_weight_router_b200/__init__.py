"""B200-native (sm_100a) batch-1 MXFP4 mixture-of-experts decode step.

The computation lives in libmoe_decode.so (CUDA kernels behind the C ABI in
include/moe_decode.h); ``binding`` exposes its entry points under the same names.
``synth`` holds the seeded synthetic-input generators.  Importing this package
does not load the library; the first call does, and raises if it is missing.
"""
from .binding import (DecodeGraph, DecodeModel, MoeError, abi_version, decode_step,  # noqa: F401
                      decode_step_launch_names, decode_step_workspace_bytes, lm_head_bf16_gemv, lm_head_fp8_gemv,
                      lm_head_fp8_gemv_noalloc, lm_head_fp8_quantize, lm_head_fp8_verify,
                      lm_head_workspace_bytes, moe_experts_workspace_bytes, moe_mxfp4_experts, moe_mxfp8_quantize, moe_sample,
                      moe_prefill_layer, moe_prefill_workspace_bytes, moe_route, moe_route_workspace_bytes, moe_selfcheck,
                      workspace_status)
