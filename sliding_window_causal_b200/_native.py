"""ctypes binding of the C ABI in include/swa.h (argument marshalling only).

The library is sliding_window_causal_b200/_swa.so, built in-tree by build.py. There
is no fallback: if it is missing or cannot be loaded, every call raises.
"""
import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "_swa.so")

# every exported symbol of include/swa.h
EXPORTS = ("swa_forward", "swa_forward_ex", "swa_forward_host", "swa_band_weights", "swa_decode", "swa_decode_noalloc",
           "swa_chunk_forward", "swa_ring_append", "swa_mha_forward", "swa_mha_workspace_bytes",
           "swa_forward_lse", "swa_backward", "swa_backward_workspace_bytes", "swa_device_status", "swa_last_error", "swa_prefill_tile_class", "swa_prefill_work_item", "swa_backward_cta_tile", "swa_decode_valid_slots", "swa_decode_split_plan",
           "swa_set_wait_limit_ns", "swa_timeout_probe", "swa_set_prefill_mode", "swa_prefill_auto_state")

SWA_F32, SWA_BF16 = 0, 1
STATUS_NAMES = {0: "SWA_OK", 1: "SWA_ERR_INVALID_ARG", 2: "SWA_ERR_UNSUPPORTED",
                3: "SWA_ERR_MISALIGNED", 4: "SWA_ERR_CUDA", 5: "SWA_ERR_TIMEOUT"}

_lib = None


class SwaError(RuntimeError):
    def __init__(self, code, message):
        super().__init__(f"{STATUS_NAMES.get(code, code)}: {message}")
        self.code = code


def lib(path=None):
    """Load (once) and return the ctypes handle of the CUDA library."""
    global _lib
    if _lib is not None and path is None:
        return _lib
    p = path or LIB_PATH
    if not os.path.exists(p):
        raise ImportError(f"CUDA library {p} is missing: build it with "
                          "`python -m sliding_window_causal_b200.build`")
    h = ctypes.CDLL(p)
    i64, vp, i32 = ctypes.c_int64, ctypes.c_void_p, ctypes.c_int
    h.swa_forward.argtypes = [vp, vp, vp, vp, i64, i64, i64, i64, i64, i32, vp]
    h.swa_forward.restype = i32
    h.swa_forward_ex.argtypes = [vp, vp, vp, vp, i64, i64, i64, i64, i64, ctypes.c_double,
                                 ctypes.POINTER(i64), i32, vp]
    h.swa_forward_ex.restype = i32
    h.swa_forward_host.argtypes = [vp] * 8 + [i64] * 6 + [i32, vp]
    h.swa_forward_host.restype = i32
    h.swa_band_weights.argtypes = [vp, vp, vp, i64, i64, i64, i64, i64, ctypes.c_double,
                                   ctypes.POINTER(i64), i32, vp]
    h.swa_band_weights.restype = i32
    h.swa_decode.argtypes = [vp, vp, vp, vp, vp, i64, i64, i64, i64, vp]
    h.swa_decode.restype = i32
    h.swa_chunk_forward.argtypes = [vp, vp, vp, vp, vp, vp, vp, i64, i64, i64, i64, i64, vp]
    h.swa_chunk_forward.restype = i32
    h.swa_ring_append.argtypes = [vp, vp, vp, vp, vp, i64, i64, i64, i64, i64, vp]
    h.swa_ring_append.restype = i32
    h.swa_mha_forward.argtypes = [vp] * 11 + [i64] * 6 + [i32, vp]
    h.swa_mha_forward.restype = i32
    h.swa_mha_workspace_bytes.argtypes = [i64, i64, i64, i32]
    h.swa_mha_workspace_bytes.restype = i64
    h.swa_forward_lse.argtypes = [vp] * 5 + [i64] * 5 + [ctypes.c_double, i32, vp]
    h.swa_forward_lse.restype = i32
    h.swa_backward.argtypes = [vp] * 10 + [i64] * 6 + [ctypes.c_double, i32, vp]
    h.swa_backward.restype = i32
    h.swa_backward_workspace_bytes.argtypes = [i64, i64, i64]
    h.swa_backward_workspace_bytes.restype = i64
    h.swa_decode_noalloc.argtypes = [vp, vp, vp, vp, vp, i64, i64, i64, i64, vp]
    h.swa_decode_noalloc.restype = i32
    h.swa_device_status.argtypes = [vp]
    h.swa_device_status.restype = i32
    h.swa_last_error.argtypes = []
    h.swa_last_error.restype = ctypes.c_char_p
    h.swa_prefill_tile_class.argtypes = [i64] * 6
    h.swa_prefill_tile_class.restype = i32
    pi64 = ctypes.POINTER(i64)
    h.swa_prefill_work_item.argtypes = [i64] * 5 + [pi64] * 3
    h.swa_prefill_work_item.restype = i32
    h.swa_backward_cta_tile.argtypes = [i64] * 5 + [i32] + [pi64] * 3
    h.swa_backward_cta_tile.restype = i32
    h.swa_set_prefill_mode.argtypes = [i32]
    h.swa_set_prefill_mode.restype = i32
    h.swa_prefill_auto_state.argtypes = [i32]
    h.swa_prefill_auto_state.restype = i32
    h.swa_decode_valid_slots.argtypes = [i64, i64]
    h.swa_decode_valid_slots.restype = i64
    h.swa_decode_split_plan.argtypes = [i64, i64, i64, i64, ctypes.POINTER(ctypes.c_int32),
                                        ctypes.POINTER(ctypes.c_int32)]
    h.swa_decode_split_plan.restype = i32
    h.swa_set_wait_limit_ns.argtypes = [ctypes.c_uint64]
    h.swa_set_wait_limit_ns.restype = ctypes.c_uint64
    h.swa_timeout_probe.argtypes = [vp]
    h.swa_timeout_probe.restype = i32
    if path is None:
        _lib = h
    return h


def check(rc):
    if rc != 0:
        msg = lib().swa_last_error()
        raise SwaError(rc, msg.decode() if msg else "")
    return rc
