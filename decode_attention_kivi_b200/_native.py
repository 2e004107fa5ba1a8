"""ctypes declarations of libkivi.so (include/kivi.h).  Argument marshalling only."""
from __future__ import annotations

import ctypes
import os

# KIVI_LIBRARY selects another in-tree build (the debug library in its tests)
_LIB_PATH = os.environ.get("KIVI_LIBRARY") or os.path.join(
    os.path.dirname(os.path.abspath(__file__)), "libkivi.so")


class KiviConfig(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in (
        "batch", "num_layers", "num_kv_heads", "num_q_heads", "head_dim", "bits",
        "group_size", "residual", "max_tokens")]


class KiviSizes(ctypes.Structure):
    _fields_ = [(n, ctypes.c_size_t) for n in (
        "records_bytes", "resid_k_bytes", "resid_v_bytes", "workspace_bytes")]


class KiviBuffers(ctypes.Structure):
    _fields_ = [("records", ctypes.c_void_p), ("resid_k", ctypes.c_void_p),
                ("resid_v", ctypes.c_void_p), ("workspace", ctypes.c_void_p),
                ("sizes", KiviSizes)]


STATUS = {0: "KIVI_OK", 1: "KIVI_ERR_INVALID_ARG", 2: "KIVI_ERR_UNSUPPORTED",
          3: "KIVI_ERR_BUFFER_TOO_SMALL", 4: "KIVI_ERR_CAPACITY", 5: "KIVI_ERR_STATE",
          6: "KIVI_ERR_CUDA", 7: "KIVI_ERR_DEVICE", 8: "KIVI_ERR_SCRATCH_LIMIT"}

STATIC_SCRATCH_BYTES = 8 << 20  # KIVI_STATIC_SCRATCH_BYTES

_lib = None


def lib() -> ctypes.CDLL:
    """Loads the in-tree libkivi.so; raises if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(_LIB_PATH):
        raise RuntimeError(
            f"{_LIB_PATH} is missing: build it with `python -m decode_attention_kivi_b200.build` "
            "(there is no CPU fallback)")
    L = ctypes.CDLL(_LIB_PATH)
    P, I32, F32 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_float
    st = ctypes.c_int
    sig = {
        "kivi_required_bytes": (st, [ctypes.POINTER(KiviConfig), ctypes.POINTER(KiviSizes)]),
        "kivi_record_layout": (st, [ctypes.POINTER(KiviConfig), ctypes.POINTER(ctypes.c_size_t),
                                    ctypes.POINTER(I32)]),
        "kivi_cache_create": (st, [ctypes.POINTER(KiviConfig), ctypes.POINTER(KiviBuffers),
                                   ctypes.POINTER(P)]),
        "kivi_cache_destroy": (None, [P]),
        "kivi_cache_length": (st, [P, I32, ctypes.POINTER(I32), ctypes.POINTER(I32)]),
        "kivi_cache_reset": (st, [P, I32]),
        "kivi_quantize_prefill": (st, [P, I32, P, P, I32, P]),
        "kivi_append_token": (st, [P, I32, P, P, P]),
        "kivi_quantize_prefill_ragged": (st, [P, I32, P, P, I32, ctypes.POINTER(I32), P]),
        "kivi_cache_lengths": (st, [P, I32, ctypes.POINTER(I32)]),
        "kivi_decode_attention": (st, [P, I32, P, P, F32, P]),
        "kivi_check_device_status": (st, [P, P, ctypes.POINTER(ctypes.c_uint32)]),
        "kivi_cache_bytes": (st, [ctypes.POINTER(KiviConfig), I32,
                                  ctypes.POINTER(ctypes.c_double),
                                  ctypes.POINTER(ctypes.c_double),
                                  ctypes.POINTER(ctypes.c_double)]),
        "kivi_status_string": (ctypes.c_char_p, [st]),
        "kivi_decode_attention_static_scratch": (st, [ctypes.POINTER(KiviConfig), P, P, P, I32,
                                                      I32, P, P, F32, P]),
        "kivi_static_scratch_status": (st, [P, ctypes.POINTER(ctypes.c_uint32)]),
        "kivi_bf16_workspace_bytes": (st, [I32, I32, I32, I32, ctypes.POINTER(ctypes.c_size_t)]),
        "kivi_bf16_decode_attention": (st, [P, P, I32, I32, I32, I32, I32, I32, P, P, F32, P,
                                            ctypes.c_size_t, P]),
        "kivi_bf16_status": (st, [P, I32, I32, P, ctypes.POINTER(ctypes.c_uint32)]),
        "kivi_fake_quant_keys": (st, [P, ctypes.c_int64, I32, I32, I32, P, P]),
        "kivi_prefill_attention": (st, [P, I32, P, P, P, I32, P, F32, P]),
        "kivi_causal_attention": (st, [P, P, P, I32, I32, I32, I32, I32, P, F32, P, P]),
    }
    if hasattr(L, "kivi_debug_overstate_copies"):  # debug build only
        sig["kivi_debug_overstate_copies"] = (st, [ctypes.c_uint32])
    for name, (res, args) in sig.items():
        fn = getattr(L, name)
        fn.restype = res
        fn.argtypes = args
    _lib = L
    return L


class KiviError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        self.status = STATUS.get(code, str(code))
        text = lib().kivi_status_string(code).decode()
        super().__init__(f"{where}: {self.status} ({text})")


def check(code: int, where: str) -> None:
    if code != 0:
        raise KiviError(code, where)
