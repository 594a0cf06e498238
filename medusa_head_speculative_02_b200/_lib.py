"""ctypes loader for libmedusa.so (the C ABI of include/medusa.h).

With MEDUSA_DEBUG=1 in the environment the MEDUSA_DEBUG build
(libmedusa_debug.so: device-side index checks reported as
MEDUSA_ERR_BOUNDS) is loaded instead.  Loading fails loudly: there is no CPU
or Python fallback for any call.
"""
from __future__ import annotations

import ctypes as C
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
DEBUG = os.environ.get("MEDUSA_DEBUG", "0") == "1"
LIB_PATH = os.path.join(_HERE, "libmedusa_debug.so" if DEBUG else "libmedusa.so")

OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_CUDA, ERR_TIMEOUT, ERR_BOUNDS = 0, -1, -2, -3, -4, -5
F32, BF16 = 0, 1
MAX_K, MAX_S, MAX_N = 8, 16, 256

vp, i32p, u32p, f32p = C.c_void_p, C.POINTER(C.c_int32), C.POINTER(C.c_uint32), C.POINTER(C.c_float)
ci, cf, csz = C.c_int, C.c_float, C.c_size_t

# name -> (restype, argtypes); every symbol include/medusa.h declares
SIGNATURES = {
    "medusa_last_error": (C.c_char_p, []),
    "medusa_version": (C.c_char_p, []),
    "medusa_device_status": (ci, [C.POINTER(ci), ci]),
    "medusa_selftest_wait_timeout": (ci, [ci, vp]),
    "medusa_topk_merge": (ci, [vp, vp, C.c_longlong, vp, ci, ci, ci, ci, vp, vp, vp]),
    "medusa_sample_next": (ci, [vp, ci, vp, vp, ci, ci, ci, ci, C.c_float, C.c_uint64,
                                C.c_uint64, vp, vp, vp]),
    "medusa_tree_plan_host": (ci, [ci, ci, ci, vp, vp, vp, vp]),
    "medusa_tree_create": (ci, [ci, ci, ci, C.POINTER(vp)]),
    "medusa_tree_destroy": (ci, [vp]),
    "medusa_tree_info": (ci, [vp, C.POINTER(ci), C.POINTER(ci), C.POINTER(ci), vp, vp, vp, vp]),
    "medusa_heads_workspace_size": (csz, [ci, ci, ci, ci, ci, ci]),
    "medusa_heads_forward": (ci, [vp, vp, vp, vp, ci, ci, ci, ci, ci, vp, ci, vp, vp, vp, csz,
                                  vp]),
    "medusa_topk": (ci, [vp, ci, ci, ci, ci, vp, vp, vp]),
    "medusa_build_tree": (ci, [vp, vp, vp, vp, ci, vp, vp, vp]),
    "medusa_tree_attention_workspace_size": (csz, [vp, ci, ci, ci, ci, ci]),
    "medusa_tree_attention_chunks": (ci, [vp, ci, ci, ci, ci, ci, ci]),
    "medusa_tree_attention_launches": (ci, [vp, ci, ci, ci, ci, ci, ci]),
    "medusa_tree_attention_tiles_per_cta": (ci, [vp, ci, ci, ci, ci, ci, ci]),
    "medusa_tree_attention": (ci, [vp, vp, vp, vp, vp, ci, ci, ci, ci, ci, cf, ci, vp, vp, csz,
                                   vp]),
    "medusa_accept_workspace_size": (csz, [vp, ci, ci]),
    "medusa_accept_greedy": (ci, [vp, ci, vp, vp, ci, ci, vp, vp, vp, vp, csz, vp]),
    "medusa_accept_typical": (ci, [vp, ci, vp, vp, ci, ci, cf, cf, cf, vp, vp, vp, vp, csz, vp]),
    "medusa_accept_greedy_typical": (ci, [vp, ci, vp, vp, ci, ci, cf, cf, cf, vp, vp, vp, vp, vp,
                                          vp, vp, csz, vp]),
    "medusa_accept_typical_per_head": (ci, [vp, ci, vp, vp, ci, ci, f32p, cf, cf, vp, vp, vp, vp,
                                            csz, vp]),
    "medusa_accept_greedy_noalloc": (ci, [vp, ci, vp, vp, ci, ci, vp, vp, vp, vp]),
    "medusa_kv_compact": (ci, [vp, vp, vp, vp, vp, ci, ci, ci, ci, ci, ci, vp, vp]),
    "medusa_kv_compact_layers": (ci, [vp, vp, ci, C.c_longlong, vp, vp, vp, ci, ci, ci, ci, ci,
                                      ci, vp, vp]),
}

_lib = None


class MedusaError(RuntimeError):
    def __init__(self, code: int, where: str, msg: str):
        super().__init__(f"{where} failed with status {code}: {msg}")
        self.code = code


def lib() -> C.CDLL:
    """The loaded library; raises if libmedusa.so has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing: build it with "
                "`python -m medusa_head_speculative_02_b200.build` (no fallback exists)")
        L = C.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def check(code: int, where: str) -> None:
    if code != OK:
        raise MedusaError(code, where, lib().medusa_last_error().decode())
