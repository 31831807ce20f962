"""ctypes loading of libomnimoe.so and the prototypes of its C ABI (include/omnimoe.h)."""
from __future__ import annotations

import ctypes as C
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libomnimoe.so")

OMNI_OK = 0
OMNI_ERR_INVALID_ARG = 1
OMNI_ERR_UNSUPPORTED = 2
OMNI_ERR_WORKSPACE = 3
OMNI_ERR_CUDA = 4

OMNI_DEV_TIMEOUT = 1
OMNI_DEV_BAD_INDEX = 2

OMNI_F32 = 0
OMNI_BF16 = 1
OMNI_FLAG_ROUTER_SIMT = 1
OMNI_FLAG_STAGED_SMALL = 2
OMNI_FLAG_DENSE_TENSOR_CORES = 4

OMNI_WS_ROUTE = 0
OMNI_WS_SCHEDULE = 1
OMNI_WS_EXPERT = 2
OMNI_WS_FUSED = 3
OMNI_WS_TOKEN = 4
OMNI_WS_SELECT = 5
OMNI_WS_BACKWARD = 6

# every function the header declares, with its argument types
_P = C.c_void_p
_I64 = C.c_int64
SIGNATURES = {
    "omni_abi_version": ([], C.c_int),
    "omni_status_string": ([C.c_int], C.c_char_p),
    "omni_last_cuda_error_name": ([], C.c_char_p),
    "omni_workspace_size": ([_P, C.c_int, C.POINTER(C.c_size_t)], C.c_int),
    "omni_route": ([_P] * 11 + [C.c_size_t, _P], C.c_int),
    "omni_route_select": ([_P] * 9 + [C.c_size_t, _P], C.c_int),
    "omni_router_logits": ([_P] * 7 + [C.c_size_t, _P], C.c_int),
    "omni_schedule": ([_P] * 10 + [C.c_size_t, _P], C.c_int),
    "omni_expert_forward": ([_P] * 12 + [C.c_size_t, _P], C.c_int),
    "omni_expert_forward_noalloc": ([_P] * 12, C.c_int),
    "omni_moe_forward": ([_P] * 13 + [C.c_size_t, _P], C.c_int),
    "omni_token_centric_forward": ([_P] * 9 + [C.c_size_t, _P], C.c_int),
    "omni_expert_forward_glu": ([_P] * 13 + [C.c_size_t, _P], C.c_int),
    "omni_moe_forward_glu": ([_P] * 14 + [C.c_size_t, _P], C.c_int),
    "omni_token_centric_forward_glu": ([_P] * 10 + [C.c_size_t, _P], C.c_int),
    "omni_moe_forward_shard": ([_P, _I64, _I64] + [_P] * 13 + [C.c_size_t, _P], C.c_int),
    "omni_cast_output": ([_P] * 4, C.c_int),
    "omni_moe_forward_shard_routed": ([_P, _I64, _I64] + [_P] * 9 + [C.c_size_t, _P], C.c_int),
    "omni_moe_backward": ([_P] * 16 + [C.c_int, _P, _P, C.c_size_t, _P], C.c_int),
    "omni_wait_selftest": ([_P, _P], C.c_int),
    "omni_shared_mlp": ([_P, _I64, _P, _P, _P, _P, C.c_int, _P, _P, C.c_size_t, _P], C.c_int),
    "omni_moe_mlp_forward": ([_P, _I64] + [_P] * 14 + [C.c_size_t, _P], C.c_int),
    "omni_mlp_workspace_size": ([_P, _I64, C.c_int, C.POINTER(C.c_size_t)], C.c_int),
}


class Dims(C.Structure):
    _fields_ = [("L", C.c_int64), ("d", C.c_int64), ("Nr", C.c_int64), ("Nc", C.c_int64),
                ("k", C.c_int64), ("K", C.c_int64), ("B", C.c_int64), ("dtype", C.c_int32),
                ("flags", C.c_int32)]


_lib = None


def load(path: str = LIB_PATH):
    """Load the library (once).  Raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(path):
            raise RuntimeError(
                f"{path} is missing: build the CUDA library first "
                "(python -m atomic_expert_routing_b200.build)")
        lib = C.CDLL(path)
        for name, (args, res) in SIGNATURES.items():
            fn = getattr(lib, name)
            fn.argtypes = args
            fn.restype = res
        _lib = lib
    return _lib


class OmniError(RuntimeError):
    def __init__(self, fn: str, code: int):
        msg = load().omni_status_string(code).decode()
        if code == OMNI_ERR_CUDA:
            msg += f" [{load().omni_last_cuda_error_name().decode()}]"
        super().__init__(f"{fn} failed: {msg} (code {code})")
        self.code = code


def check(fn: str, code: int) -> None:
    if code != OMNI_OK:
        raise OmniError(fn, code)
