"""ctypes mirror of include/lla.h: status codes, parameter structs, prototypes.

Loading fails loudly (``LibraryMissing``) when liblla.so is absent: there is no
CPU or Python fallback for any entry point.
"""

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "liblla.so")

LLA_OK = 0
LLA_ERR_NULL = 1
LLA_ERR_SHAPE = 2
LLA_ERR_DTYPE = 3
LLA_ERR_ALIGN = 4
LLA_ERR_WORKSPACE = 5
LLA_ERR_UNSUPPORTED = 6
LLA_ERR_CUDA = 7

LLA_F32 = 0
LLA_BF16 = 1
LLA_FP8_E4M3 = 2

LLA_WRITE_HLA = 0
LLA_WRITE_PERHEAD = 1
LLA_WRITE_FOLDED = 2

c_i32 = ctypes.c_int32
c_i64 = ctypes.c_int64
c_f32 = ctypes.c_float
c_f64 = ctypes.c_double
c_vp = ctypes.c_void_p


class WriteParams(ctypes.Structure):
    _fields_ = [
        ("mode", c_i32), ("B", c_i32), ("n", c_i32), ("pos0", c_i32),
        ("T", c_i32), ("H", c_i32), ("d_h", c_i32), ("D", c_i32),
        ("r_k", c_i32), ("r_v", c_i32), ("r_1", c_i32), ("rotate_keys", c_i32),
        ("rope_base", c_f64),
        ("x", c_vp), ("xv", c_vp),
        ("x_stride_b", c_i64), ("x_stride_n", c_i64), ("x_stride_t", c_i64),
        ("E_main", c_vp), ("E_1", c_vp), ("E_K", c_vp), ("E_V", c_vp),
        ("out0", c_vp), ("out1", c_vp),
        ("out_dtype", c_i32), ("Ncap", c_i32),
        ("out_stride_b", c_i64), ("out_stride_h", c_i64), ("out_stride_n", c_i64),
        ("out1_stride_b", c_i64), ("out1_stride_n", c_i64),
    ]


class LlaDecodeParams(ctypes.Structure):
    _fields_ = [
        ("B", c_i32), ("H", c_i32), ("d_h", c_i32), ("r", c_i32),
        ("T", c_i32), ("t0", c_i32), ("nt", c_i32),
        ("N", c_i32), ("W", c_i32),
        ("cK", c_vp), ("cV", c_vp),
        ("lat_dtype", c_i32),
        ("lat_stride_b", c_i64), ("lat_stride_h", c_i64),
        ("UK", c_vp), ("UV", c_vp),
        ("q", c_vp),
        ("q_stride_b", c_i64),
        ("win_k", c_vp), ("win_v", c_vp),
        ("win_dtype", c_i32), ("Wcap", c_i32),
        ("win_stride_b", c_i64),
        ("out", c_vp),
        ("out_stride_b", c_i64),
        ("scale", c_f32),
        ("timing_events", c_vp),
    ]


class HlaDecodeParams(ctypes.Structure):
    _fields_ = [
        ("B", c_i32), ("H", c_i32), ("d_h", c_i32),
        ("T", c_i32), ("t0", c_i32), ("nt", c_i32),
        ("N", c_i32), ("W", c_i32),
        ("r_k", c_i32), ("r_v", c_i32),
        ("lat", c_vp),
        ("lat_dtype", c_i32),
        ("lat_stride_b", c_i64), ("lat_stride_n", c_i64),
        ("A", c_vp), ("Bm", c_vp),
        ("q", c_vp),
        ("q_stride_b", c_i64),
        ("rotate_query", c_i32),
        ("rope_base", c_f64),
        ("win_k", c_vp), ("win_v", c_vp),
        ("win_dtype", c_i32), ("Wcap", c_i32),
        ("win_stride_b", c_i64),
        ("out", c_vp),
        ("out_stride_b", c_i64),
        ("scale", c_f32),
        ("timing_events", c_vp),
        ("nq", c_i32),
        ("win_stream", c_vp),
        ("win_events", c_vp),
    ]


# Every symbol include/lla.h declares, with its ctypes prototype.
PROTOTYPES = {
    "lla_abi_version": (ctypes.c_int, []),
    "lla_status_str": (ctypes.c_char_p, [ctypes.c_int]),
    "lla_last_cuda_error": (ctypes.c_int, []),
    "lla_cuda_error_name": (ctypes.c_char_p, [ctypes.c_int]),
    "lla_write_workspace_bytes": (ctypes.c_size_t, [ctypes.POINTER(WriteParams)]),
    "lla_write_latents": (ctypes.c_int, [ctypes.POINTER(WriteParams), c_vp, ctypes.c_size_t, c_vp]),
    "lla_decode_workspace_bytes": (ctypes.c_size_t, [ctypes.POINTER(LlaDecodeParams)]),
    "lla_decode_attn": (ctypes.c_int, [ctypes.POINTER(LlaDecodeParams), c_vp, ctypes.c_size_t, c_vp]),
    "hla_decode_workspace_bytes": (ctypes.c_size_t, [ctypes.POINTER(HlaDecodeParams)]),
    "hla_decode_attn": (ctypes.c_int, [ctypes.POINTER(HlaDecodeParams), c_vp, ctypes.c_size_t, c_vp]),
    "hla_decode_attn_noalloc": (ctypes.c_int, [ctypes.POINTER(HlaDecodeParams), c_vp]),
}

# Size of the library's static scratch used by hla_decode_attn_noalloc.
NOALLOC_SCRATCH_BYTES = 32 * 1024 * 1024


class LibraryMissing(RuntimeError):
    pass


_lib = None


def load():
    """Load liblla.so (once) and attach prototypes."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise LibraryMissing(
            f"{LIB_PATH} is missing; build it with `python -m looped_transformer_latent_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    for name, (res, args) in PROTOTYPES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib
