"""ConvRot W4A4 quantized linear for NVIDIA B200 (sm_100a).

The computation lives in libck.so (C ABI in include/ck.h); ``ck`` is its thin
Python binding and ``workloads`` draws the seeded synthetic inputs.
"""
__all__ = ["ck", "workloads", "ck_rotate_quant", "ck_w4a4_linear", "ck_unpack_w4"]


def __getattr__(name):
    if name in ("ck_rotate_quant", "ck_w4a4_linear", "ck_unpack_w4"):
        from . import ck
        return getattr(ck, name)
    raise AttributeError(name)
