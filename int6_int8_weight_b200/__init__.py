"""int6_int8_weight_b200: B200-native int6/int8 weight quantization.

The product is ``libgq.so`` (CUDA kernels for sm_100a behind the C ABI of
``include/gq.h``); ``gq`` is its thin Python binding.  The binding is loaded
on first use (``from int6_int8_weight_b200 import gq``, or any of the names
below) and raises if the library has not been built (``python -m
int6_int8_weight_b200.build``): there is no CPU fallback.
"""
_EXPORTS = ("FakeQuantSTE", "GQError", "Quantized", "Request", "dequant", "export_pack",
            "export_state_dict", "fakequant", "row_clip_select", "ste_bwd")


def __getattr__(name):
    if name == "gq" or name in _EXPORTS:
        import importlib
        mod = importlib.import_module(".gq", __name__)
        return mod if name == "gq" else getattr(mod, name)
    raise AttributeError(name)
