"""ctypes binding of ``libfa_sm100.so`` (the C ABI in ``include/fa.h``): argument marshalling only.

Every step of the computation runs in the library's CUDA kernels.  Loading fails loudly when the
library is missing; there is no fallback.
"""
import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libfa_sm100.so")

FA_OK, FA_ERR_INVALID_ARG, FA_ERR_UNSUPPORTED, FA_ERR_CUDA, FA_ERR_TIMEOUT, FA_ERR_INTERNAL = range(6)
STATUS_NAMES = {0: "FA_OK", 1: "FA_ERR_INVALID_ARG", 2: "FA_ERR_UNSUPPORTED", 3: "FA_ERR_CUDA",
                4: "FA_ERR_TIMEOUT", 5: "FA_ERR_INTERNAL"}

# name -> (restype, argtypes)
_P, _I, _F, _U64, _SZ = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_uint64, ctypes.c_size_t
SIGNATURES = {
    "fa_fwd": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _F, _I, _P, _F, _U64, _P]),
    "fa_fwd_f32": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _F, _I, _P, _F, _U64, _P]),
    "fa_bwd_workspace_size": (_SZ, [_I, _I, _I, _I]),
    "fa_bwd": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _F, _I, _P, _F, _U64, _P, _SZ, _P]),
    "fa_bwd_split": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _F, _I, _P, _F, _U64, _P, _SZ, _P]),
    "fa_bwd_prep": (_I, [_P, _P, _I, _I, _I, _I, _P, _SZ, _P]),
    "fa_bwd_main": (_I, [_P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _F, _I, _P, _F, _U64, _P, _SZ, _P]),
    "fa_bwd_dq_convert": (_I, [_P, _I, _I, _I, _I, _F, _P, _SZ, _P]),
    "fa_bwd_noalloc": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _F, _I, _P, _F, _U64, _P]),
    "fa_bwd_noalloc_max_scratch": (_SZ, []),
    "fa_fwd_decode_workspace_size": (_SZ, [_I, _I, _I, _I, _I]),
    "fa_fwd_decode_split": (_I, [_I, _I, _I, _I]),
    "fa_fwd_decode": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _F, _I, _P, _P, _SZ, _P]),
    "fa_bwd_head_group": (_I, [_I, _I, _SZ]),
    "fa_dropout_mask": (_I, [_P, _I, _I, _I, _F, _U64, _P]),
    "fa_test_exp2_fma": (_I, [_P, _P, _I, _P]),
    "fa_check": (_I, [_P]),
    "fa_get_error": (ctypes.c_char_p, []),
    "fa_set_wait_limit_ns": (None, [_U64]),
    "fa_debug_set_flags": (None, [_I]),
    "fa_version": (ctypes.c_char_p, []),
}

_lib = None


class FAError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {message}")
        self.status = status


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load the library once and attach the C signatures."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"CUDA library {path} is missing: build it with "
                           "`python -m exact_io_aware_68_b200.build` (there is no fallback)")
    lib = ctypes.CDLL(path)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def call(name: str, *args) -> int:
    """Call an fa_* entry point that returns fa_status; raise FAError unless FA_OK."""
    lib = load()
    st = getattr(lib, name)(*args)
    if st != FA_OK:
        raise FAError(st, lib.fa_get_error().decode())
    return st


def status(name: str, *args) -> int:
    """Call an fa_* entry point and return its status without raising."""
    return getattr(load(), name)(*args)
