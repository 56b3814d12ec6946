"""ctypes view of libhsa_b200.so (the C ABI in include/hsa.h).

Argument marshalling only.  Every step of the method runs in the CUDA library.
There is no fallback: if the library is missing or fails to load, every call
raises.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
# HSA_DEBUG=1 selects the debug build (every kernel-derived index checked on the device)
DEBUG = os.environ.get("HSA_DEBUG", "0") not in ("", "0")
LIB_PATH = os.path.join(_HERE, "libhsa_b200_debug.so" if DEBUG else "libhsa_b200.so")

HSA_OK, HSA_ERR_INVALID_ARG, HSA_ERR_UNSUPPORTED, HSA_ERR_WORKSPACE, HSA_ERR_CUDA, HSA_ERR_TIMEOUT = range(6)
HSA_F32, HSA_BF16 = 0, 1
HSA_FLAG_LANDMARKS_READY = 1
HSA_FLAG_SIMT = 2
HSA_FLAG_TEST_STALL = 4
HSA_FLAG_QUEST = 8

EXPORTED = ("hsa_workspace_size", "hsa_landmarks", "hsa_select", "hsa_attend", "hsa_forward",
            "hsa_get_device_status", "hsa_plan", "hsa_status_string", "hsa_last_error", "hsa_abi_version",
            "hsa_select_noalloc", "hsa_decode_append", "hsa_attend_partials", "hsa_merge_partials",
            "hsa_backward_workspace_size", "hsa_backward", "hsa_noalloc_status", "hsa_landmarks_refined",
            "hsa_debug_checks", "hsa_forward_host_bytes", "hsa_forward_host")
PATH_NAMES = {0: "none", 1: "simt_rows", 2: "simt_split", 3: "tensor", 4: "mma_split"}


class hsa_problem_t(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int32), ("Tq", ctypes.c_int32), ("Tkv", ctypes.c_int32),
                ("H", ctypes.c_int32), ("Hkv", ctypes.c_int32), ("d", ctypes.c_int32),
                ("S", ctypes.c_int32), ("k", ctypes.c_int32), ("q_pos0", ctypes.c_int64),
                ("tau", ctypes.c_float), ("dtype", ctypes.c_int32), ("flags", ctypes.c_uint32),
                ("kv_cap", ctypes.c_int32)]


class hsa_plan_t(ctypes.Structure):
    _fields_ = [("landmark_path", ctypes.c_int32), ("select_path", ctypes.c_int32),
                ("attend_path", ctypes.c_int32), ("landmark_kernels", ctypes.c_int32),
                ("select_kernels", ctypes.c_int32), ("attend_kernels", ctypes.c_int32),
                ("forward_fused", ctypes.c_int32)]


class HSAError(RuntimeError):
    def __init__(self, status: int, where: str, detail: str):
        self.status = status
        super().__init__(f"{where}: {detail}")


_lib = None


def lib() -> ctypes.CDLL:
    """Load the library once.  Raises if it is missing.  There is no other path."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"HSA CUDA library not built: {LIB_PATH} is missing "
                           "(run landmark_guided_chunk_b200/build.py [--debug] or __graft_entry__.build())")
    L = ctypes.CDLL(LIB_PATH)
    P, Z, I32p, Fp = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p, ctypes.c_void_p
    prob = ctypes.POINTER(hsa_problem_t)
    L.hsa_workspace_size.argtypes = [prob, ctypes.POINTER(ctypes.c_size_t)]
    L.hsa_landmarks.argtypes = [prob, P, P, P, P]
    L.hsa_select.argtypes = [prob, P, P, I32p, Fp, I32p, P, Z, P]
    L.hsa_attend.argtypes = [prob, P, P, P, I32p, Fp, I32p, P, P, Z, P]
    L.hsa_forward.argtypes = [prob, P, P, P, P, P, I32p, Fp, I32p, P, P, Z, P]
    L.hsa_forward_host_bytes.argtypes = [prob, ctypes.POINTER(ctypes.c_size_t)]
    L.hsa_forward_host.argtypes = [prob, P, P, P, P, P, P, Z, P, Z, P]
    L.hsa_get_device_status.argtypes = [P, Z, P]
    L.hsa_plan.argtypes = [prob, ctypes.POINTER(hsa_plan_t)]
    L.hsa_select_noalloc.argtypes = [prob, P, P, I32p, Fp, I32p, P]
    L.hsa_decode_append.argtypes = [prob, P, P, P, P, P, P, P]
    L.hsa_attend_partials.argtypes = [prob, P, P, P, I32p, I32p, Fp, P, Z, P]
    L.hsa_merge_partials.argtypes = [prob, ctypes.c_int, Fp, I32p, I32p, Fp, P, I32p, Fp, I32p, P]
    L.hsa_noalloc_status.argtypes = [P]
    L.hsa_landmarks_refined.argtypes = [prob, P, P, P, P, P, P, P]
    L.hsa_backward_workspace_size.argtypes = [prob, ctypes.POINTER(ctypes.c_size_t)]
    L.hsa_backward.argtypes = [prob, P, P, P, P, P, I32p, Fp, I32p, P, Fp, Fp, Fp, Fp, P, Z, P]
    L.hsa_status_string.argtypes = [ctypes.c_int]
    L.hsa_status_string.restype = ctypes.c_char_p
    L.hsa_last_error.argtypes = []
    L.hsa_last_error.restype = ctypes.c_char_p
    L.hsa_abi_version.argtypes = []
    L.hsa_abi_version.restype = ctypes.c_int
    L.hsa_debug_checks.argtypes = []
    L.hsa_debug_checks.restype = ctypes.c_int
    for f in ("hsa_workspace_size", "hsa_landmarks", "hsa_select", "hsa_attend", "hsa_forward",
              "hsa_get_device_status", "hsa_plan", "hsa_select_noalloc", "hsa_decode_append",
              "hsa_attend_partials", "hsa_merge_partials", "hsa_backward_workspace_size", "hsa_backward",
              "hsa_noalloc_status", "hsa_landmarks_refined", "hsa_forward_host_bytes", "hsa_forward_host"):
        getattr(L, f).restype = ctypes.c_int
    _lib = L
    return L


def check(status: int, where: str) -> None:
    if status != HSA_OK:
        L = lib()
        detail = L.hsa_last_error().decode() or L.hsa_status_string(status).decode()
        raise HSAError(status, where, f"{L.hsa_status_string(status).decode()} -- {detail}")
