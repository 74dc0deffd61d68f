"""CPU oracle for the NVFP4 hot path -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
and reference legs may import this package.  It shares no code with the CUDA
library and never imports it.  See ``oracle/nvfp4_ref.py`` for the definitions
and the tests that pin each function.
"""
from .nvfp4_ref import *  # noqa: F401,F403
from .nvfp4_ref import (  # noqa: F401  (explicit re-exports for readers)
    ACT_GELU_TANH, ACT_NONE, BLOCK, E2M1_GRID, E4M3_MAX, G_MAX, G_MIN, dequantize,
    dequantize_to_bf16, dynamic_scale, e2m1_decode, e2m1_encode, e4m3_decode, e4m3_encode_sat,
    epilogue_ref, gelu_tanh, gemm_ref, linear_w4a16_ref, gemm_tolerance, global_scale, pack_codes,
    quantize_dynamic, quantize_nvfp4, round_to_bf16,
    sf_offset, sf_padded_shape, swizzle_sf, tensor_amax, unpack_codes, unswizzle_sf,
)
from . import mxfp8_ref  # noqa: F401,E402  (the MXFP8 variant: 32-element blocks, E8M0 scales)
from . import fp8row_ref  # noqa: F401,E402  (row-wise FP8: E4M3 with one fp32 scale per row)
