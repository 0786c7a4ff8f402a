"""CPU oracle of the FlashDecoder streaming step (test infrastructure only).

Only tests/, the smoke check and the benchmark's CPU-baseline leg may import
this package. The product path never does.
"""
from .flashdec_oracle import (OracleDecoder, attention, decode_video,  # noqa: F401
                              full_sequence, gelu, linear, patchify,
                              rms_norm, rope_3d, rope_rotate, rope_split,
                              unpatchify)
