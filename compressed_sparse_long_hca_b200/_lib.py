"""ctypes declarations of the C ABI in include/csa.h (argument marshalling only).

The shared library is built in-tree (``build.py``).  Loading fails loudly
when it is missing: there is no fallback implementation.
"""
from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libcsa.so")

CSA_OK = 0
STATUS_NAMES = {0: "CSA_OK", -1: "CSA_ERR_ARG", -2: "CSA_ERR_CAPACITY", -3: "CSA_ERR_CUDA",
                -4: "CSA_ERR_DEVICE_TIMEOUT", -5: "CSA_ERR_DEVICE_BOUNDS"}
VARIANT_AUTO, VARIANT_HIGH_OCC, VARIANT_LOW_OCC = 0, 1, 2
ATTN_STATE_READY = 0x100        # flag OR-ed into csa_hca_decode_attn's variant
REGION_KV, REGION_INDEX, REGION_WINDOW = 0, 1, 2
FMT_MIXED, FMT_F32 = 0, 1


class GemmOut(ctypes.Structure):
    _fields_ = [("rows", ctypes.c_int32), ("bf16", ctypes.c_int32), ("y", ctypes.c_void_p)]


class CsaCfg(ctypes.Structure):
    _fields_ = [("n_csa_layers", ctypes.c_int32), ("n_hca_layers", ctypes.c_int32),
                ("H", ctypes.c_int32), ("D", ctypes.c_int32), ("D_rope", ctypes.c_int32),
                ("H_I", ctypes.c_int32), ("d_I", ctypes.c_int32), ("window", ctypes.c_int32),
                ("max_requests", ctypes.c_int32), ("max_pages_per_request", ctypes.c_int32),
                ("pool_pages", ctypes.c_int32), ("rope_base", ctypes.c_float), ("fmt", ctypes.c_int32)]


# exported symbol -> (restype, argtypes)
_P, _I32, _I64, _SZ, _F = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t, ctypes.c_float
SIGNATURES = {
    "csa_cache_required_bytes": (_SZ, [ctypes.POINTER(CsaCfg)]),
    "csa_cache_init": (_I32, [ctypes.POINTER(CsaCfg), _P, _SZ, _P, _P, _P, ctypes.POINTER(_P)]),
    "csa_cache_destroy": (None, [_P]),
    "csa_request_alloc": (_I32, [_P, _I32, _I64]),
    "csa_request_free": (_I32, [_P, _I32]),
    "csa_compress_append": (_I32, [_P, _I32, _I32, _P, _I32, _P, _P, _P, _P, _P]),
    "csa_index_scores": (_I32, [_P, _I32, _I32, _P, _P, _P, _P, _I64, _P, _I32, _P]),
    "csa_topk": (_I32, [_P, _I64, _P, _I32, _I32, _P, _I32, _P]),
    "csa_index_topk_workspace_bytes": (_SZ, [_P, _I32, _I64]),
    "csa_index_topk": (_I32, [_P, _I32, _I32, _P, _P, _P, _P, _I64, _P, _I32, _P, _P, _SZ, _I32, _P]),
    "csa_attn_workspace_bytes": (_SZ, [_P, _I32, _I32, _I32]),
    "csa_hca_decode_attn": (_I32, [_P, _I32, _I32, _P, _P, _P, _I32, _P, _F, _P, _P, _SZ, _I32, _P]),
    "csa_hca_decode_attn_noalloc": (_I32, [_P, _I32, _I32, _P, _P, _P, _I32, _P, _F, _P, _P]),
    "csa_check_device_error": (_I32, [_P, _P]),
    "csa_last_error": (ctypes.c_char_p, []),
    "csa_launch_count": (ctypes.c_uint64, []),
    "csa_debug_row_bytes": (_SZ, [_P, _I32]),
    "csa_debug_rows": (_I32, [_P, _I32, _I32, _I32, _I64, _I64, _P, _I32]),
    "csa_debug_set_length": (_I32, [_P, _I32, _I32, _I64]),
    "csa_debug_get_length": (_I64, [_P, _I32, _I32]),
    "csa_debug_wait_timeout": (_I32, [_P, _I32, _P]),
    "csa_decode_step_input_bytes": (_SZ, [_P, _I32, _I32]),
    "csa_decode_step_dev_bytes": (_SZ, [_P, _I32, _I32, _I32]),
    "csa_decode_step": (_I32, [_P, _I32, _I32, _P, _I32, _P, _F, _P, _P, _P, _SZ, _P]),
    "csa_prefill_workspace_bytes": (_SZ, [_P, _I32, _I32, _I32, _I32, _I32]),
    "csa_prefill_chunk": (_I32, [_P, _I32, _I32, _P, _I32, _P, _P, _P, _P, _P, _P, _P, _I32, _P, _F, _P, _P, _P,
                                 _SZ, _I32, _P]),
    "csa_gemm_weight_bytes": (_SZ, [_I32, _I32, _I32]),
    "csa_gemm_pack_weight": (_I32, [_P, _I32, _I32, _I32, _P, _SZ]),
    "csa_gemm_workspace_bytes": (_SZ, [_I32, _I32, _I32, _I32]),
    "csa_gemm_bf16": (_I32, [_P, _I32, _I32, _I32, _P, _I32, _I32, _P, _P, _SZ, _P]),
    "csa_gemm_check_device_error": (_I32, [_P]),
}

_lib = None


def load():
    """Load libcsa.so and declare every exported function."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"libcsa.so is not built ({LIB_PATH}); run "
                           "`python -c 'import __graft_entry__ as g; g.build()'`")
    lib = ctypes.CDLL(LIB_PATH)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


class CsaError(RuntimeError):
    def __init__(self, status: int, where: str):
        lib = load()
        msg = lib.csa_last_error().decode(errors="replace")
        super().__init__(f"{where}: {STATUS_NAMES.get(status, status)}: {msg}")
        self.status = status


def check(status: int, where: str) -> None:
    if status != CSA_OK:
        raise CsaError(status, where)
