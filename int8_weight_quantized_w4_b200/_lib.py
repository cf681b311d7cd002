"""ctypes declarations of libw4b200.so (the C ABI in include/w4.h).

Loading fails loudly when the library has not been built: there is no
fallback implementation of any entry point.
"""

from __future__ import annotations

import ctypes as C
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libw4b200.so")

STATUS = {
    0: "W4_OK",
    1: "W4_ERR_NULL",
    2: "W4_ERR_SHAPE",
    3: "W4_ERR_ALIGN",
    4: "W4_ERR_DEVICE",
    5: "W4_ERR_CUDA",
    6: "W4_ERR_TIMEOUT",
    7: "W4_ERR_WORKSPACE",
    8: "W4_ERR_VALUE",
}
W4_OK, W4_ERR_NULL, W4_ERR_SHAPE, W4_ERR_ALIGN, W4_ERR_DEVICE, W4_ERR_CUDA, W4_ERR_TIMEOUT, W4_ERR_WORKSPACE, \
    W4_ERR_VALUE = range(9)
PATHS = {"auto": 0, "gemv": 1, "generic": 2, "tc": 3}
ACTS = {"none": 0, "gelu_tanh": 1, "gelu_erf": 2}
ABI_VERSION = 6
GROUP_MAX = 48


class W4Desc(C.Structure):
    _fields_ = [
        ("x", C.c_void_p),
        ("ldx", C.c_int64),
        ("qw", C.c_void_p),
        ("scales", C.c_void_p),
        ("zp", C.c_void_p),
        ("y", C.c_void_p),
        ("ldy", C.c_int64),
        ("M", C.c_int64),
        ("K", C.c_int64),
        ("N", C.c_int64),
        ("bias", C.c_void_p),
        ("residual", C.c_void_p),
        ("ldr", C.c_int64),
        ("act", C.c_int32),
        ("reserved", C.c_int32),
    ]


class W4RDesc(C.Structure):
    """w4r_desc: one decode matmul on a weight in the streaming layout."""
    _fields_ = [
        ("x", C.c_void_p),
        ("ldx", C.c_int64),
        ("wr", C.c_void_p),
        ("y", C.c_void_p),
        ("ldy", C.c_int64),
        ("M", C.c_int64),
        ("K", C.c_int64),
        ("N", C.c_int64),
        ("bias", C.c_void_p),
        ("residual", C.c_void_p),
        ("ldr", C.c_int64),
        ("act", C.c_int32),
        ("reserved", C.c_int32),
    ]


# name -> (restype, argtypes)
SIGNATURES = {
    "w4_matmul_workspace_size": (C.c_size_t, [C.c_int64, C.c_int64, C.c_int64]),
    "w4_matmul": (C.c_int, [C.c_void_p, C.c_int64, C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p, C.c_int64,
                            C.c_int64, C.c_int64, C.c_int64, C.c_void_p, C.c_size_t, C.c_void_p]),
    "w4_matmul_path": (C.c_int, [C.c_void_p, C.c_int64, C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p, C.c_int64,
                                 C.c_int64, C.c_int64, C.c_int64, C.c_void_p, C.c_size_t, C.c_int, C.c_void_p]),
    "w4_matmul_noalloc": (C.c_int, [C.c_void_p, C.c_int64, C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p,
                                    C.c_int64, C.c_int64, C.c_int64, C.c_int64, C.c_void_p]),
    "w4_matmul_desc": (C.c_int, [C.POINTER(W4Desc), C.c_void_p, C.c_size_t, C.c_int, C.c_void_p]),
    "w4_matmul_grouped_workspace_size": (C.c_size_t, [C.POINTER(W4Desc), C.c_int32]),
    "w4_matmul_grouped": (C.c_int, [C.POINTER(W4Desc), C.c_int32, C.c_void_p, C.c_size_t, C.c_void_p]),
    "w4_repacked_bytes": (C.c_size_t, [C.c_int64, C.c_int64]),
    "w4_repack": (C.c_int, [C.c_void_p, C.c_void_p, C.c_void_p, C.c_int64, C.c_int64, C.c_void_p, C.c_void_p]),
    "w4_repack_restore": (C.c_int, [C.c_void_p, C.c_int64, C.c_int64, C.c_void_p, C.c_void_p, C.c_void_p,
                                    C.c_void_p]),
    "w4r_matmul": (C.c_int, [C.POINTER(W4RDesc), C.c_void_p]),
    "w4t_repacked_bytes": (C.c_size_t, [C.c_int64, C.c_int64]),
    "w4t_repack": (C.c_int, [C.c_void_p, C.c_void_p, C.c_void_p, C.c_int64, C.c_int64, C.c_void_p, C.c_void_p]),
    "w4t_repack_restore": (C.c_int, [C.c_void_p, C.c_int64, C.c_int64, C.c_void_p, C.c_void_p, C.c_void_p,
                                     C.c_void_p]),
    "w4t_workspace_size": (C.c_size_t, [C.POINTER(W4RDesc), C.c_int32]),
    "w4t_matmul_grouped": (C.c_int, [C.POINTER(W4RDesc), C.c_int32, C.c_void_p, C.c_size_t, C.c_void_p]),
    "w4t_matmul": (C.c_int, [C.POINTER(W4RDesc), C.c_void_p, C.c_size_t, C.c_void_p]),
    "w4i_workspace_size": (C.c_size_t, [C.POINTER(W4RDesc), C.c_int32]),
    "w4i_matmul_grouped": (C.c_int, [C.POINTER(W4RDesc), C.c_int32, C.c_void_p, C.c_size_t, C.c_void_p]),
    "w4i_matmul": (C.c_int, [C.POINTER(W4RDesc), C.c_void_p, C.c_size_t, C.c_void_p]),
    "w4r_matmul_grouped": (C.c_int, [C.POINTER(W4RDesc), C.c_int32, C.c_void_p]),
    "i8_head_repacked_bytes": (C.c_size_t, [C.c_int64, C.c_int64]),
    "i8_head_repack": (C.c_int, [C.c_void_p, C.c_int64, C.c_void_p, C.c_int64, C.c_int64, C.c_void_p, C.c_void_p]),
    "i8_head_repack_restore": (C.c_int, [C.c_void_p, C.c_int64, C.c_int64, C.c_void_p, C.c_int64, C.c_void_p,
                                         C.c_void_p]),
    "i8r_head_logits": (C.c_int, [C.c_void_p, C.c_void_p, C.c_int64, C.c_int64, C.c_void_p, C.c_void_p]),
    "w4r_decode_step": (C.c_int, [C.POINTER(W4RDesc), C.c_int32, C.c_void_p, C.c_void_p, C.c_int64, C.c_int64,
                                  C.c_void_p, C.c_void_p]),
    "w4r_decode_step_argmax": (C.c_int, [C.POINTER(W4RDesc), C.c_int32, C.c_void_p, C.c_void_p, C.c_int64,
                                         C.c_int64, C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p]),
    "i8t_head_repacked_bytes": (C.c_size_t, [C.c_int64, C.c_int64]),
    "i8t_head_repack": (C.c_int, [C.c_void_p, C.c_int64, C.c_void_p, C.c_int64, C.c_int64, C.c_void_p, C.c_void_p]),
    "i8t_head_repack_restore": (C.c_int, [C.c_void_p, C.c_int64, C.c_int64, C.c_void_p, C.c_int64, C.c_void_p,
                                          C.c_void_p]),
    "i8t_head_logits": (C.c_int, [C.c_void_p, C.c_int64, C.c_void_p, C.c_int64, C.c_int64, C.c_int64, C.c_void_p,
                                  C.c_int64, C.c_void_p]),
    "i8t_head_argmax": (C.c_int, [C.c_void_p, C.c_int64, C.c_void_p, C.c_int64, C.c_int64, C.c_int64, C.c_void_p,
                                  C.c_void_p, C.c_void_p, C.c_void_p]),
    "i8r_head_argmax": (C.c_int, [C.c_void_p, C.c_void_p, C.c_int64, C.c_int64, C.c_void_p, C.c_void_p,
                                  C.c_void_p, C.c_void_p]),
    "i8_head_workspace_size": (C.c_size_t, [C.c_int64, C.c_int64, C.c_int64]),
    "i8_head_argmax_workspace_size": (C.c_size_t, [C.c_int64, C.c_int64, C.c_int64]),
    "i8_head_argmax": (C.c_int, [C.c_void_p, C.c_int64, C.c_void_p, C.c_int64, C.c_void_p, C.c_int64, C.c_int64,
                                 C.c_int64, C.c_void_p, C.c_void_p, C.c_void_p, C.c_size_t, C.c_void_p]),
    "i8_embed_lookup": (C.c_int, [C.c_void_p, C.c_int64, C.c_void_p, C.c_void_p, C.c_int64, C.c_void_p,
                                  C.c_int64, C.c_int64, C.c_int64, C.c_void_p]),
    "i8_head_logits": (C.c_int, [C.c_void_p, C.c_int64, C.c_void_p, C.c_int64, C.c_void_p, C.c_void_p, C.c_int64,
                                 C.c_int64, C.c_int64, C.c_int64, C.c_void_p, C.c_size_t, C.c_void_p]),
    "i8_head_logits_path": (C.c_int, [C.c_void_p, C.c_int64, C.c_void_p, C.c_int64, C.c_void_p, C.c_void_p,
                                      C.c_int64, C.c_int64, C.c_int64, C.c_int64, C.c_void_p, C.c_size_t, C.c_int,
                                      C.c_void_p]),
    "w4_quantize": (C.c_int, [C.c_void_p, C.c_int64, C.c_int64, C.c_int64, C.c_int32, C.c_int32, C.c_void_p,
                              C.c_void_p, C.c_void_p, C.c_void_p]),
    "i8_quantize_head": (C.c_int, [C.c_void_p, C.c_int64, C.c_int64, C.c_int64, C.c_void_p, C.c_int64, C.c_void_p,
                                   C.c_void_p]),
    "w4_pack_nibbles": (C.c_int, [C.c_void_p, C.c_int64, C.c_void_p]),
    "w4_unpack_nibbles": (C.c_int, [C.c_void_p, C.c_int64, C.c_void_p]),
    "w4_status_string": (C.c_char_p, [C.c_int]),
    "w4_last_error": (C.c_char_p, []),
    "w4_device_error": (C.c_int, [C.POINTER(C.c_int32), C.c_int32]),
    "w4_set_wait_timeout_ns": (C.c_int, [C.c_uint64]),
    "w4_debug_wait_timeout": (C.c_int, [C.c_uint64, C.c_void_p]),
    "w4_abi_version": (C.c_int32, []),
}

_lib = None


class W4LibraryMissing(ImportError):
    pass


def load():
    """The loaded library (built in-tree by int8_weight_quantized_w4_b200.build)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise W4LibraryMissing(
            f"{LIB_PATH} is missing; build it with `python -m int8_weight_quantized_w4_b200.build` "
            "(there is no CPU or fallback implementation)")
    lib = C.CDLL(LIB_PATH)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    if lib.w4_abi_version() != ABI_VERSION:
        raise W4LibraryMissing(f"{LIB_PATH} has ABI version {lib.w4_abi_version()}, this binding needs "
                               f"{ABI_VERSION}: rebuild it")
    _lib = lib
    return lib
