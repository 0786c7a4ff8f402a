"""CPU oracle of the FlashDecoder streaming step (test infrastructure only).

Only tests/, the smoke check and the benchmark's CPU-baseline leg may import
this package. The product path never does.
"""
from .flashdec_oracle import (E4M3_MAX, OracleDecoder, attention,  # noqa: F401
                              calibrate_fp8, decode_video, e4m3_round,
                              full_sequence, gelu, linear, mlp, patchify,
                              quantize_act, quantize_weight, rms_norm,
                              rope_3d, rope_rotate, rope_split, unpatchify,
                              weight_scale)
