"""ctypes declarations of the C ABI in include/dg.h (argument marshalling only)."""

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libdg.so")

DG_OK, DG_EINVAL, DG_ECUDA, DG_EUNSUPPORTED, DG_ETIMEOUT, DG_ENOMEM = 0, -1, -2, -3, -4, -5

# every symbol include/dg.h declares
EXPORTS = ("dg_params_default", "dg_temperature", "dg_workspace_size", "dg_canvas_init", "dg_denoise_step",
           "dg_stop_check", "dg_stub_hidden", "dg_status_string", "dg_last_launch_count", "dg_plan",
           "dg_profile_enable", "dg_profile_collect", "dg_denoise_stats_noalloc", "dg_debug_set_error",
           "dg_partial_bytes", "dg_denoise_partial", "dg_denoise_merge", "dg_debug_set_counter_wait_limit",
           "dg_quantize_e4m3", "dg_last_sm_clock", "dg_tile_head")


class DgParams(ctypes.Structure):
    _fields_ = [("n_canvas", ctypes.c_int), ("canvas_len", ctypes.c_int), ("vocab", ctypes.c_int),
                ("hidden", ctypes.c_int), ("max_steps", ctypes.c_int), ("t_start", ctypes.c_float),
                ("t_end", ctypes.c_float), ("eb_bound", ctypes.c_float), ("stop_thresh", ctypes.c_float),
                ("stability", ctypes.c_int), ("tied", ctypes.c_int), ("group", ctypes.c_int),
                ("accept_mode", ctypes.c_int), ("accept_rule", ctypes.c_int), ("logits_format", ctypes.c_int),
                ("w_scale_exp", ctypes.c_int), ("head_layout", ctypes.c_int)]


class DgError(RuntimeError):
    def __init__(self, fn, status, msg):
        super().__init__(f"{fn} failed: {msg} ({status})")
        self.status = status


_lib = None


def lib():
    """Load libdg.so (raises if it is missing: there is no fallback path)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"CUDA library {LIB_PATH} is missing; build it with "
                              "`python -m discrete_diffusion_decoding_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        P = ctypes.POINTER(DgParams)
        vp, sz, i32 = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int
        L.dg_params_default.argtypes = [P, i32, i32, i32]
        L.dg_params_default.restype = None
        L.dg_temperature.argtypes = [P, i32]
        L.dg_temperature.restype = ctypes.c_float
        L.dg_workspace_size.argtypes = [P]
        L.dg_workspace_size.restype = sz
        L.dg_canvas_init.argtypes = [P, vp, vp, vp, sz, vp]
        L.dg_canvas_init.restype = i32
        L.dg_denoise_step.argtypes = [P, i32, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
        L.dg_denoise_step.restype = i32
        L.dg_stop_check.argtypes = [P, vp, sz, vp, vp, vp, vp]
        L.dg_stop_check.restype = i32
        L.dg_debug_set_error.argtypes = [P, vp, sz, i32, vp]
        L.dg_debug_set_error.restype = i32
        L.dg_stub_hidden.argtypes = [P, i32, ctypes.c_float, ctypes.c_float, vp, vp, vp, vp, vp, sz, vp]
        L.dg_stub_hidden.restype = i32
        L.dg_status_string.argtypes = [i32]
        L.dg_status_string.restype = ctypes.c_char_p
        L.dg_last_launch_count.argtypes = []
        L.dg_last_launch_count.restype = i32
        L.dg_plan.argtypes = [P, ctypes.POINTER(i32), ctypes.POINTER(i32), ctypes.POINTER(i32)]
        L.dg_plan.restype = i32
        L.dg_denoise_stats_noalloc.argtypes = [P, i32, vp, vp, vp, vp, vp, vp, vp, vp]
        L.dg_denoise_stats_noalloc.restype = i32
        L.dg_partial_bytes.argtypes = [P]
        L.dg_partial_bytes.restype = sz
        L.dg_denoise_partial.argtypes = [P, i32, i32, i32, vp, vp, vp, vp, vp, vp, sz, vp]
        L.dg_denoise_partial.restype = i32
        L.dg_denoise_merge.argtypes = [P, i32, i32, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
        L.dg_denoise_merge.restype = i32
        L.dg_debug_set_counter_wait_limit.argtypes = [ctypes.c_ulonglong]
        L.dg_debug_set_counter_wait_limit.restype = i32
        L.dg_quantize_e4m3.argtypes = [vp, ctypes.c_longlong, i32, i32, vp, vp, vp]
        L.dg_quantize_e4m3.restype = i32
        L.dg_last_sm_clock.argtypes = [P, vp, sz, ctypes.POINTER(ctypes.c_float), vp]
        L.dg_last_sm_clock.restype = i32
        L.dg_tile_head.argtypes = [vp, vp, ctypes.c_longlong, i32, i32, vp]
        L.dg_tile_head.restype = i32
        L.dg_profile_enable.argtypes = [i32]
        L.dg_profile_enable.restype = i32
        L.dg_profile_collect.argtypes = [ctypes.POINTER(i32), ctypes.POINTER(ctypes.c_float),
                                         ctypes.POINTER(ctypes.c_float)]
        L.dg_profile_collect.restype = i32
        _lib = L
    return _lib


def check(fn, status):
    if status != DG_OK:
        raise DgError(fn, status, lib().dg_status_string(status).decode())
    return status
