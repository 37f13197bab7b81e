"""ctypes binding of libdsa.so (the C ABI in include/dsa.h).

Argument marshalling only.  Loading fails loudly when the library has not
been built: there is no fallback implementation.
"""
from __future__ import annotations

import ctypes
import os
import threading

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libdsa.so")

DSA_OK, DSA_ERR_INVALID_ARG, DSA_ERR_UNSUPPORTED, DSA_ERR_CUDA, DSA_ERR_DEVICE = range(5)
DSA_F32, DSA_BF16 = 0, 1
DSA_OP_POOL_SCORE, DSA_OP_SELECT_TOPP = 0, 1
DSA_OP_POOL_SCORE_HIER2, DSA_OP_POOL_SCORE_HIER4, DSA_OP_ATTN_BWD = 2, 3, 4
DSA_MAX_BLOCKS = 1024
DSA_STATIC_MAX_ROWS = 32768

STATUS_NAMES = {0: "DSA_OK", 1: "DSA_ERR_INVALID_ARG", 2: "DSA_ERR_UNSUPPORTED",
                3: "DSA_ERR_CUDA", 4: "DSA_ERR_DEVICE"}

# Every entry point declared in include/dsa.h: name -> (restype, argtypes)
_vp, _i, _f, _sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
SIGNATURES = {
    "dsa_workspace_size": (_sz, [_i, _i, _i, _i, _i, _i]),
    "dsa_pool_score": (_i, [_vp, _vp, _i, _i, _i, _i, _i, _i, _f, _vp, _vp, _vp, _vp, _sz, _vp]),
    "dsa_select_topp": (_i, [_vp, _i, _i, _f, _vp, _vp, _vp, _vp, _vp, _sz, _vp]),
    "dsa_row_order": (_i, [_vp, _i, _i, _i, _vp, _vp]),
    "dsa_attn_fwd": (_i, [_vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _f, _vp, _vp, _vp, _vp, _vp, _vp]),
    "dsa_attn_fwd_ordered": (_i, [_vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _f, _vp, _vp, _vp, _vp,
                                  _vp, _vp, _vp]),
    "dsa_block_mass": (_i, [_vp, _vp, _i, _i, _i, _i, _vp, _vp, _vp]),
    "dsa_attn_bwd": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _f, _vp, _vp,
                          _vp, _vp, _vp, _vp, _sz, _vp]),
    "dsa_mass_to_probs": (_i, [_vp, _vp, _vp, _i, _i, _vp, _vp]),
    "dsa_pool_score_hier": (_i, [_vp, _vp, _i, _i, _i, _i, _i, _i, _i, _f, _vp, _vp, _sz, _vp]),
    "dsa_hilbert_order": (_i, [_i, _i, _i, _i, _vp]),
    "dsa_gilbert_order": (_i, [_i, _i, _i, _i, _vp]),
    "dsa_permute_tokens": (_i, [_vp, _vp, _i, _i, _i, _i, _i, _vp, _i, _vp]),
    "dsa_select_topp_static": (_i, [_vp, _i, _i, _f, _vp, _vp, _vp, _vp, _vp]),
    "dsa_selftest_wait_timeout": (_i, [ctypes.c_ulonglong, _vp]),
    "dsa_selftest_exp2_poly": (_i, [_vp, _vp, _i, _vp]),
    "dsa_sparse_attention_host": (_i, [_vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _f, _f, _i, _vp, _vp,
                                       _sz, _vp]),
    "dsa_host_pipeline_workspace_size": (_sz, [_i, _i, _i, _i, _i, _i, _i]),
    "dsa_device_status": (_i, [_vp]),
    "dsa_last_error": (ctypes.c_char_p, []),
    "dsa_version": (_i, []),
}

_lock = threading.Lock()
_lib = None


class DSAError(RuntimeError):
    """A libdsa call returned an error status."""

    def __init__(self, status: int, where: str, message: str):
        super().__init__(f"{where}: {STATUS_NAMES.get(status, status)}: {message}")
        self.status = status


def lib() -> ctypes.CDLL:
    """The loaded library (built in place by dynamic_block_sparse_pool_b200.build)."""
    global _lib
    if _lib is None:
        with _lock:
            if _lib is None:
                if not os.path.exists(LIB_PATH):
                    raise RuntimeError(
                        f"{LIB_PATH} is missing: build it with "
                        "`python -m dynamic_block_sparse_pool_b200.build` (no fallback exists)")
                h = ctypes.CDLL(LIB_PATH)
                for name, (res, args) in SIGNATURES.items():
                    fn = getattr(h, name)
                    fn.restype = res
                    fn.argtypes = args
                _lib = h
    return _lib


def check(status: int, where: str) -> None:
    if status != DSA_OK:
        msg = lib().dsa_last_error()
        raise DSAError(status, where, msg.decode() if msg else "")
