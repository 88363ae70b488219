"""int6_int8_weight_b200: B200-native int6/int8 weight quantization.

The product is ``libgq.so`` (CUDA kernels for sm_100a behind the C ABI of
``include/gq.h``); ``gq`` is its thin Python binding.  Importing the package
raises if the library has not been built (``python -m
int6_int8_weight_b200.build``): there is no CPU fallback.
"""
from . import gq  # noqa: F401
from .gq import (FakeQuantSTE, GQError, Quantized, Request, dequant,  # noqa: F401
                 export_pack, export_state_dict, fakequant, row_clip_select, ste_bwd)
