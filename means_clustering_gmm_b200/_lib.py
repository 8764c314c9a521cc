"""ctypes loader for libgmm_b200.so (the C-ABI library in include/gmm_b200.h).

There is no fallback: if the library is missing this raises, telling the user
to build it (``python -m means_clustering_gmm_b200.build``).
"""
from __future__ import annotations

import ctypes
import os
import threading

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "_lib", "libgmm_b200.so")

GMM_OK = 0
GMM_ERR_INVALID_ARG = 1
GMM_ERR_UNSUPPORTED = 2
GMM_ERR_CUDA = 3
GMM_ERR_TIMEOUT = 4
GMM_ERR_NONFINITE = 5
GMM_ERR_RANGE = 6

GMM_F32, GMM_BF16, GMM_F16 = 0, 1, 2

GMM_FLAG_NONE = 0
GMM_FLAG_FORCE_TWO_SWEEP = 1
GMM_FLAG_FORCE_SIMT = 2
GMM_FLAG_TEST_STALL = 4

# Every symbol include/gmm_b200.h declares, with its ctypes signature.
_vp, _sz, _i64, _i32, _u32 = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int64, ctypes.c_int, \
    ctypes.c_uint32
SIGNATURES = {
    "gmm_status_string": (ctypes.c_char_p, [_i32]),
    "gmm_version": (_i32, []),
    "gmm_workspace_init": (_i32, [_vp, _sz, _vp]),
    "gmm_workspace_size": (_sz, [_i64, _i32, _i32, _i32]),
    "gmm_regime": (_i32, [_i64, _i32, _i32, _i32, _u32]),
    "gmm_em_step": (_i32, [_vp, _i32, _i64, _i32, _i32, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _sz,
                           _u32, _vp]),
    "gmm_finalize": (_i32, [_vp, _i64, _i32, _i32, ctypes.c_float, _vp, _vp, _vp, _vp, _sz,
                            _vp]),
    "kmeans_workspace_size": (_sz, [_i32, _i64, _i32, _i32]),
    "kmeans_step": (_i32, [_vp, _i32, _i32, _i64, _i32, _i32, _vp, _vp, _vp, _vp, _vp, _vp, _sz,
                           _u32, _vp]),
    "gmm_em_step_static": (_i32, [_vp, _i32, _i64, _i32, _i32, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                                  _u32, _vp]),
    "gmm_last_error": (_i32, [_vp, _vp]),
    "gmm_set_kernel_timer": (_i32, [_vp, _vp]),
    "gmm_kernel_timer_begin": (_i32, []),
    "gmm_kernel_timer_end": (_i32, [_vp, _i64, _vp]),
    "gmm_point_chunk": (_i64, [_i64, _i32, _i32, _i32, _u32]),
    "gmm_set_point_chunk": (_i32, [_i64]),
    "gmm_kernel_launch_count": (ctypes.c_uint64, []),
    "gmm_device_binary_version": (_i32, []),
    "gmm_fit_workspace_size": (_sz, [_i64, _i32, _i32, _i32]),
    "gmm_fit": (_i32, [_vp, _i32, _i64, _i32, _i32, _vp, _vp, _vp, _i32, ctypes.c_double,
                       ctypes.c_float, _vp, _vp, _vp, _sz, _u32, _vp]),
    "gmm_soft_assign": (_i32, [_vp, _i32, _i64, _i32, _i32, _vp, _vp, _vp, _i32, ctypes.c_float,
                               _vp, _vp, _vp, _vp, _sz, _u32, _vp]),
    "gmm_batched_workspace_size": (_sz, [_i32, _i64, _i32, _i32, _i32]),
    "gmm_batched_workspace_init": (_i32, [_vp, _i32, _i64, _i32, _i32, _i32, _vp]),
    "gmm_em_step_batched": (_i32, [_vp, _i32, _i32, _i64, _i32, _i32, _vp, _vp, _vp, _vp, _vp,
                                   _vp, _vp, _sz, _u32, _vp]),
    "gmm_finalize_batched": (_i32, [_vp, _i32, _i64, _i32, _i32, ctypes.c_float, _vp, _vp, _vp,
                                    _vp, _sz, _vp]),
    "gmm_init_kmeans_workspace_size": (_sz, [_i64, _i32, _i32]),
    "gmm_init_kmeans": (_i32, [_vp, _i32, _i64, _i32, _i32, _i32, ctypes.c_float, _vp, _vp, _vp,
                               _vp, _vp, _sz, _vp]),
}

_lock = threading.Lock()
_lib = None


class GmmError(RuntimeError):
    def __init__(self, fn: str, code: int):
        self.code = code
        super().__init__(f"{fn} failed: {status_string(code)} ({code})")


def load() -> ctypes.CDLL:
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise ImportError(
                    f"libgmm_b200.so not found at {LIB_PATH}; build it with "
                    "`python -m means_clustering_gmm_b200.build` (nvcc, sm_100a)")
            lib = ctypes.CDLL(LIB_PATH)
            for name, (res, args) in SIGNATURES.items():
                fn = getattr(lib, name)
                fn.restype = res
                fn.argtypes = args
            _lib = lib
    return _lib


def status_string(code: int) -> str:
    return load().gmm_status_string(int(code)).decode()


def check(fn: str, code: int) -> None:
    if code != GMM_OK:
        raise GmmError(fn, code)
