"""ctypes loader of ``libgdn.so`` (the C ABI of ``include/gdn.h``).

There is no fallback: if the library is missing or cannot be loaded, importing the binding
raises. Build it with ``python -m frame_wise_gated_deltanet_b200.build``.
"""
from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libgdn.so")
# the same sources with the device-side address, size and coordinate checks (include/gdn.h)
DEBUG_LIB_PATH = os.path.join(HERE, "libgdn_debug.so")

STATUS = {
    0: "GDN_OK",
    1: "GDN_ERR_INVALID_ARG",
    2: "GDN_ERR_UNSUPPORTED",
    3: "GDN_ERR_MISALIGNED",
    4: "GDN_ERR_NO_MEMORY",
    5: "GDN_ERR_CUDA",
    6: "GDN_ERR_TIMEOUT",
    7: "GDN_ERR_SCRATCH_LIMIT",
}

# Every symbol include/gdn.h declares, with (restype, argtypes).
_P = ctypes.c_void_p
_I = ctypes.c_int
_F = ctypes.c_float
SIGNATURES = {
    "gdn_frame_forward": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _F, _P]),
    "gdn_frame_forward_noalloc": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _F, _P]),
    "gdn_frame_forward_host": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _F, _P]),
    "gdn_frame_forward_fp8": (_I, [_P] * 11 + [_I, _I, _I, _I, _I, _F, _P]),
    "gdn_frame_forward_rope": (_I, [_P] * 8 + [_I, _I, _I, _I, _I, _F, _I, _I, _F, _I, _P]),
    "gdn_frame_step": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _F, _P]),
    "gdn_frame_backward": (_I, [_P] * 14 + [_I, _I, _I, _I, _I, _F, _P]),
    "gdn_backward_workspace_bytes": (ctypes.c_size_t, [_I, _I, _I, _I, _I]),
    "gdn_train_saved_bytes": (ctypes.c_size_t, [_I, _I, _I, _I, _I]),
    "gdn_frame_forward_train": (_I, [_P] * 9 + [_I, _I, _I, _I, _I, _F, _P]),
    "gdn_frame_backward_saved": (_I, [_P] * 15 + [_I, _I, _I, _I, _I, _F, _P]),
    "gdn_rope_3d": (_I, [_P, _P, _I, _I, _I, _I, _I, _I, _I, _F, _I, _P]),
    "gdn_softmax_attention": (_I, [_P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _F, _P]),
    "gdn_frame_stats": (_I, [_P, _P, _P, _P, _I, _I, _I, _I, _I, _F, _P]),
    "gdn_block_causal_la": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _P]),
    "gdn_workspace_bytes": (ctypes.c_size_t, [_I, _I, _I, _I, _I]),
    "gdn_la_workspace_bytes": (ctypes.c_size_t, [_I, _I, _I, _I]),
    "gdn_status_string": (ctypes.c_char_p, [_I]),
    "gdn_sync_status": (_I, [_P]),
    "gdn_release_workspace": (None, []),
    "gdn_version": (_I, []),
    "gdn_debug_checks": (_I, []),
    "gdn_debug_report": (_I, [ctypes.POINTER(ctypes.c_int), ctypes.POINTER(ctypes.c_longlong)]),
    "gdn_profile_arm": (_I, [_P, _I]),
    "gdn_set_forward_mode": (_I, [_I]),
    "gdn_profile_count": (_I, []),
    "gdn_profile_kernel": (ctypes.c_char_p, [_I]),
}


class GdnError(RuntimeError):
    def __init__(self, fn: str, code: int, msg: str):
        super().__init__(f"{fn} failed: {STATUS.get(code, code)} ({msg})")
        self.code = code


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    if not os.path.exists(path):
        raise ImportError(
            f"{path} is missing; build it with `python -m frame_wise_gated_deltanet_b200.build`")
    lib = ctypes.CDLL(path)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


LIB = load()


def check(fn: str, code: int) -> None:
    if code != 0:
        raise GdnError(fn, code, LIB.gdn_status_string(code).decode())
