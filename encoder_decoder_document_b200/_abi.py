"""ctypes view of libkalm.so (the C ABI declared in include/kalm.h).

Loading never falls back to anything: if the library is missing or the device
is not an sm_100 part, calls raise ``KalmError``.
"""
from __future__ import annotations

import ctypes
import os
import threading

from . import _build

c_i32, c_i64, c_u32, c_u64, c_f32, c_vp = (ctypes.c_int32, ctypes.c_int64, ctypes.c_uint32,
                                          ctypes.c_uint64, ctypes.c_float, ctypes.c_void_p)

STATUS = {
    0: "KALM_OK", 1: "KALM_ERR_INVALID_ARG", 2: "KALM_ERR_UNSUPPORTED", 3: "KALM_ERR_NO_DEVICE",
    4: "KALM_ERR_CUDA", 5: "KALM_ERR_TIMEOUT", 6: "KALM_ERR_DEVICE_ARG",
}

# name -> argtypes (restype is int32 status unless listed in _RESTYPE)
SIGNATURES = {
    "kalm_version": [],
    "kalm_status_string": [c_i32],
    "kalm_last_error": [],
    "kalm_device_check": [],
    "kalm_check_device_errors": [c_vp, ctypes.POINTER(c_u32)],
    "kalm_ragged_offsets": [c_vp, c_i32, c_i32, c_vp, c_vp, c_vp],
    "kalm_chunk_pool": [c_vp, c_i64, c_vp, c_vp, c_i32, c_i32, c_i32, c_vp, c_i64, c_vp, c_i64, c_vp],
    "kalm_linear": [c_vp, c_i64, c_vp, c_i64, c_vp, c_i64, c_vp, c_i64, c_i64, c_i32, c_i32, c_vp],
    "kalm_linear_chain": [c_vp, c_i64, c_vp, c_i64, c_vp, c_i64, c_vp, c_i64, c_vp, c_i64, c_i64, c_i32, c_i32,
                          c_i32, c_vp, c_i64, c_vp],
    "kalm_linear_chain_sync_len": [c_i64],
    "kalm_linear_chain_rope": [c_vp, c_i64, c_vp, c_i64, c_vp, c_i64, c_vp, c_i64, c_vp, c_i64, c_i64, c_i32, c_i32,
                               c_i32, c_i32, c_i32, c_vp, c_i32, c_vp, c_vp, c_i64, c_vp],
    "kalm_cross_kv_proj": [c_vp, c_i64, c_i64, c_i32, c_vp, c_i32, c_i32, c_i32, c_vp, c_vp],
    "kalm_merged_attention": [c_vp, c_i64, c_vp, c_vp, c_i64, c_vp, c_vp, c_i64, c_vp, c_vp, c_i64, c_vp, c_i32,
                              c_i32, c_i64, c_i64, c_i32, c_i32, c_i32, c_f32, c_i32, c_vp, c_vp, c_i64, c_vp,
                              c_vp],
    "kalm_merged_attention_out_proj": [c_vp, c_i64, c_vp, c_vp, c_i64, c_vp, c_vp, c_i64, c_vp, c_vp, c_i64, c_vp,
                                       c_i32, c_i32, c_i64, c_i64, c_i32, c_i32, c_i32, c_f32, c_vp, c_vp, c_i64,
                                       c_vp, c_i64, c_vp, c_i64, c_i32, c_vp, c_i64, c_vp],
    "kalm_attention_out_proj_sync_len": [c_i32, c_i32, c_i32],
    "kalm_merged_attention_out_proj_static": [c_vp, c_i64, c_vp, c_vp, c_i64, c_vp, c_vp, c_i64, c_vp, c_vp, c_i64,
                                              c_vp, c_i32, c_i32, c_i64, c_i64, c_i32, c_i32, c_i32, c_f32, c_vp, c_vp,
                                              c_i64, c_vp, c_i64, c_vp, c_i64, c_i32, c_vp],
    "kalm_attention_items": [c_i32, c_i32, c_i32, c_i32, c_i32],
    "kalm_attention_schedule": [c_vp, c_vp, c_i32, c_i32, c_i32, c_i32, c_i32, c_vp, c_i64, c_vp],
    "kalm_yes_no_score": [c_vp, c_i64, c_vp, c_i32, c_i32, c_vp, c_vp, c_vp, c_vp, c_vp, c_vp, c_vp],
    "kalm_broadcast_rows": [c_vp, c_i64, c_i32, c_i32, c_vp, c_i32, c_vp, c_i64, c_vp],
    "kalm_selftest_wait_timeout": [c_u64, c_vp],
    "kalm_rope": [c_vp, c_i64, c_i64, c_i32, c_i32, c_vp, c_i32, c_f32, c_vp],
    "kalm_linear_rope": [c_vp, c_i64, c_vp, c_i64, c_vp, c_i64, c_i64, c_i32, c_i32, c_i32, c_i32, c_vp, c_i32,
                         c_vp, c_vp],
    "kalm_rope_table": [c_f32, c_i32, c_vp, c_vp],
}
_RESTYPE = {"kalm_version": c_i32, "kalm_attention_items": c_i64, "kalm_attention_out_proj_sync_len": c_i64, "kalm_linear_chain_sync_len": c_i64, "kalm_status_string": ctypes.c_char_p, "kalm_last_error": ctypes.c_char_p}


class KalmError(RuntimeError):
    def __init__(self, status: int, where: str, detail: str = ""):
        self.status = status
        self.name = STATUS.get(status, f"status {status}")
        super().__init__(f"{where}: {self.name}" + (f" ({detail})" if detail else ""))


_lib = None
_lock = threading.Lock()


def library_path() -> str:
    return _build.LIB


def load() -> ctypes.CDLL:
    """Load libkalm.so (built in-tree).  Raises if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    with _lock:
        if _lib is not None:
            return _lib
        path = library_path()
        if not os.path.exists(path):
            raise KalmError(3, "load", f"{path} is not built; run __graft_entry__.build() "
                                       "(there is no CPU fallback)")
        lib = ctypes.CDLL(path)
        for name, args in SIGNATURES.items():
            fn = getattr(lib, name)
            fn.argtypes = args
            fn.restype = _RESTYPE.get(name, c_i32)
        _lib = lib
    return _lib


def call(name: str, *args) -> None:
    """Call an entry point and raise KalmError on a non-zero status."""
    lib = load()
    st = getattr(lib, name)(*args)
    if st != 0:
        raise KalmError(st, name, lib.kalm_last_error().decode(errors="replace"))
