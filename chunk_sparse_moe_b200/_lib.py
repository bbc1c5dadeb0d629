"""ctypes declarations of libblockffn.so (include/blockffn.h).

Argument marshalling only: every step of the layer runs in the library's CUDA
kernels.  Importing this module loads the in-tree shared library and raises
if it is missing -- there is no other implementation to fall back to.
"""
from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libblockffn.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python -m chunk_sparse_moe_b200.build` "
        "(nvcc, sm_100a). The package has no CPU implementation.")

lib = ctypes.CDLL(LIB_PATH)

c_void_p, c_int, c_float, c_size_t = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
c_uint64 = ctypes.c_uint64
c_int32_p = ctypes.POINTER(ctypes.c_int32)



class LayerOpts(ctypes.Structure):
    """blockffn_layer_opts: optional expert biases and closing LayerNorm."""
    _fields_ = [("b_in", c_void_p), ("b_out", c_void_p), ("ln_weight", c_void_p),
                ("ln_bias", c_void_p), ("ln_eps", c_float)]


# name -> (restype, argtypes); every symbol include/blockffn.h declares
SIGNATURES = {
    "blockffn_status_string": (ctypes.c_char_p, [c_int]),
    "blockffn_last_error_message": (ctypes.c_char_p, []),
    "blockffn_version": (c_int, []),
    "blockffn_route": (c_int, [c_void_p, c_void_p, c_void_p, c_void_p, c_float, c_int, c_int,
                               c_int, c_int, c_void_p, c_void_p]),
    "blockffn_chunk_union": (c_int, [c_void_p, c_int, c_int, c_int, c_void_p, c_void_p,
                                     c_void_p, c_void_p]),
    "blockffn_residual_layernorm": (c_int, [c_void_p, c_void_p, c_void_p, c_void_p, c_float, c_int,
                                            c_int, c_int, c_void_p, c_void_p]),
    "blockffn_forward_workspace_bytes": (c_size_t, [c_int, c_int, c_int, c_int, c_int, c_int,
                                                    c_int]),
    "blockffn_workspace_reset": (c_int, [c_void_p, c_size_t, c_void_p]),
    "blockffn_forward": (c_int, [c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_float,
                                 c_void_p, c_void_p, c_void_p,
                                 c_void_p, c_void_p, c_int, c_int, c_int, c_int, c_int, c_int,
                                 c_void_p, c_void_p, c_void_p, c_size_t, c_void_p]),
    "blockffn_get_device_status": (c_int, [c_void_p, c_void_p, c_int32_p]),
    "blockffn_forward_noalloc": (c_int, [c_void_p, c_void_p, c_void_p, c_void_p, c_int, c_int,
                                         c_int, c_int, c_int, c_void_p, c_void_p]),
    "blockffn_set_wait_limit_ns": (None, [c_uint64]),
    "blockffn_num_sms": (c_int, []),
    "blockffn_debug_skip_flag": (None, [c_int]),
    "blockffn_debug_set_trace": (None, [c_void_p]),
}

for _name, (_res, _args) in SIGNATURES.items():
    _fn = getattr(lib, _name)
    _fn.restype = _res
    _fn.argtypes = _args

# status codes and dtypes (include/blockffn.h)
OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_CUDA, ERR_TIMEOUT, ERR_WORKSPACE = range(6)
F32, BF16 = 0, 1
# workspace-size flags
WS_ROUTER, WS_EXPERT_BIAS = 1, 2
