"""weight_dequantization_b200: on-device decoding of compressed tensors on
NVIDIA B200 (sm_100a).

The compute lives in ``liblt_decode.so`` (CUDA kernels behind the C ABI of
``include/lt_decode.h``); :mod:`.lt_decode` is its Python binding and
:mod:`.synth` builds seeded synthetic inputs.
"""
from .lt_decode import (LT_ERR_CORRUPT_STREAM, LT_ERR_CUDA, LT_ERR_INVALID_ARG, LT_ERR_MISALIGNED,
                        LT_ERR_SIZE_MISMATCH, LT_ERR_UNSUPPORTED, LT_OK, LT_SCALE_PER_ROW, LT_SCALE_PER_TENSOR,
                        LtError, abi_version, load_library, lt_dequant_int4, lt_dequant_int8, lt_lz4_decode,
                        lt_lz4_int4_decode, lt_lz4_int4_decode_batch, lt_zrle_decode, status_string)

__all__ = [
    "LT_OK", "LT_ERR_INVALID_ARG", "LT_ERR_MISALIGNED", "LT_ERR_UNSUPPORTED", "LT_ERR_CORRUPT_STREAM",
    "LT_ERR_SIZE_MISMATCH", "LT_ERR_CUDA", "LT_SCALE_PER_TENSOR", "LT_SCALE_PER_ROW", "LtError", "abi_version",
    "load_library", "status_string", "lt_dequant_int4", "lt_dequant_int8", "lt_zrle_decode", "lt_lz4_int4_decode",
    "lt_lz4_int4_decode_batch", "lt_lz4_decode",
]
