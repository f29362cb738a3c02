"""ctypes view of libmla.so: the C structs and function signatures of include/mla.h."""
from __future__ import annotations

import ctypes
import os
from ctypes import POINTER, c_char_p, c_float, c_int32, c_int64, c_size_t, c_void_p

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libmla.so")

MLA_OK = 0
MLA_ERR_INVALID_ARG = 1
MLA_ERR_UNSUPPORTED = 2
MLA_ERR_WORKSPACE = 3
MLA_ERR_CUDA = 4
MLA_ERR_TIMEOUT = 5
MLA_ERR_DEVICE_CHECK = 6

MLA_F32 = 0
MLA_BF16 = 1


class MlaDims(ctypes.Structure):
    _fields_ = [("H", c_int32), ("D", c_int32), ("d_r", c_int32), ("d_c", c_int32), ("d_v", c_int32),
                ("g", c_int32), ("page_size", c_int32), ("sm_scale", c_float), ("rms_eps", c_float),
                ("rope_base", c_float)]


class MlaLatentCache(ctypes.Structure):
    _fields_ = [("latent", c_void_p), ("latent_stride", c_int64), ("rope", c_void_p),
                ("rope_stride", c_int64), ("num_pages", c_int32)]


class MlaGqaCache(ctypes.Structure):
    _fields_ = [("k", c_void_p), ("k_stride", c_int64), ("v", c_void_p), ("v_stride", c_int64),
                ("rope", c_void_p), ("rope_stride", c_int64), ("num_pages", c_int32)]


class MlaLatentCacheFp8(ctypes.Structure):
    _fields_ = [("codes", c_void_p), ("code_stride", c_int64), ("scales", c_void_p), ("rope", c_void_p),
                ("rope_stride", c_int64), ("num_pages", c_int32)]


PD = POINTER(MlaDims)
PI = c_void_p  # int32 device pointers travel as void*

# name -> (restype, argtypes); exactly the functions include/mla.h declares
SIGNATURES = {
    "mla_append_workspace_size": (c_size_t, [PD, c_int32, c_int32, c_int32]),
    "mla_append_cache": (c_int32, [PD, c_int32, c_int32, c_int32, c_void_p, c_int32, c_void_p, c_void_p,
                                   PI, PI, c_int32, POINTER(MlaLatentCache), c_void_p, c_size_t, c_void_p]),
    "mla_append_cache_noalloc": (c_int32, [PD, c_int32, c_int32, c_int32, c_void_p, c_int32, c_void_p, c_void_p,
                                           PI, PI, c_int32, POINTER(MlaLatentCache), c_void_p]),
    "mla_query_workspace_size": (c_size_t, [PD, c_int32, c_int32, c_int32, c_int32]),
    "mla_project_query": (c_int32, [PD, c_int32, c_int32, c_int32, c_void_p, c_int32, c_int32, c_void_p, c_void_p,
                                    c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_size_t, c_void_p]),
    "mla_absorb_q": (c_int32, [PD, c_int32, c_int32, c_int32, c_void_p, c_void_p, c_void_p, PI, c_void_p,
                               c_void_p]),
    "mla_append_cache_absorb_q": (c_int32, [PD, c_int32, c_int32, c_int32, c_void_p, c_int32, c_void_p, c_void_p,
                                            c_void_p, c_void_p, c_void_p, PI, PI, c_int32,
                                            POINTER(MlaLatentCache), c_void_p, c_void_p, c_size_t, c_void_p]),
    "mla_decode_workspace_size": (c_size_t, [PD, c_int32, c_int32, c_int32, c_int32]),
    "mla_decode_absorbed": (c_int32, [PD, c_int32, c_int32, c_int32, c_void_p, POINTER(MlaLatentCache), PI,
                                      c_int32, PI, c_void_p, c_void_p, c_void_p, c_size_t, c_void_p]),
    "mla_decode_absorbed_hinted": (c_int32, [PD, c_int32, c_int32, c_int32, c_void_p, POINTER(MlaLatentCache), PI,
                                             c_int32, PI, c_void_p, c_void_p, c_void_p, c_void_p, c_size_t,
                                             c_void_p]),
    "mla_out_proj": (c_int32, [PD, c_int32, c_int32, c_int32, c_void_p, c_void_p, c_void_p, c_void_p, c_int32,
                               c_void_p, c_void_p]),
    "mla_gqla_workspace_size": (c_size_t, [PD, c_int32, c_int32, c_int32, c_int32]),
    "mla_decode_gqla_grouped": (c_int32, [PD, c_int32, c_int32, c_int32, c_void_p, c_void_p,
                                          POINTER(MlaGqaCache), PI, c_int32, PI, c_void_p, c_void_p, c_void_p,
                                          c_size_t, c_void_p]),
    "mla_gqa_append_workspace_size": (c_size_t, [PD, c_int32, c_int32, c_int32]),
    "mla_append_gqa_cache": (c_int32, [PD, c_int32, c_int32, c_int32, c_void_p, c_int32, c_void_p, c_void_p, c_void_p,
                                       c_void_p, PI, PI, c_int32, POINTER(MlaGqaCache), c_void_p, c_size_t, c_void_p]),
    "mla_preabsorb_out_weights": (c_int32, [PD, c_int32, c_void_p, c_void_p, c_int32, c_void_p, c_void_p]),
    "mla_out_proj_preabsorbed": (c_int32, [PD, c_int32, c_int32, c_int32, c_void_p, c_void_p, c_int32, c_void_p,
                                           c_void_p]),
    "mla_quantize_latent_fp8": (c_int32, [PD, c_int32, c_void_p, c_int64, c_int64, c_void_p, c_int64, c_void_p,
                                          c_void_p]),
    "mla_decode_fp8_workspace_size": (c_size_t, [PD, c_int32, c_int32, c_int32]),
    "mla_decode_absorbed_fp8": (c_int32, [PD, c_int32, c_int32, c_int32, c_void_p, POINTER(MlaLatentCacheFp8), PI,
                                          c_int32, PI, c_void_p, c_void_p, c_void_p, c_size_t, c_void_p]),
    "mla_check_status": (c_int32, [c_void_p]),
    "mla_status_string": (c_char_p, [c_int32]),
    "mla_build_info": (c_char_p, []),
    "mla_launch_count": (ctypes.c_uint64, []),
}

_lib = None


def load(path: str = LIB_PATH):
    """Load libmla.so (built in-tree by mla_compressed_latent_b200.build). Fails loudly if absent."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise FileNotFoundError(
            f"{path} is missing: build it with `python -m mla_compressed_latent_b200.build` "
            "(nvcc, sm_100a). There is no fallback implementation.")
    lib = ctypes.CDLL(path)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib
