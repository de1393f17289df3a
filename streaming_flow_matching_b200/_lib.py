"""ctypes declarations of libsfm's C ABI (include/sfm.h), same names and arguments.

Loading fails loudly when the library has not been built: there is no other
implementation of these calls in this package.
"""
from __future__ import annotations

import ctypes as C
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libsfm.so")

SFM_OK, SFM_EINVAL, SFM_ECAPACITY, SFM_ESESSION, SFM_ECUDA, SFM_ENOMEM, SFM_EUNSUPPORTED = (
    0, -1, -2, -3, -4, -5, -6)
SFM_EDEVICE = -7
SFM_FAULT_NONE, SFM_FAULT_ATTN_NO_LOADS, SFM_FAULT_GEMM_NO_LOADS = 0, 1, 2
SFM_DTYPE_BF16, SFM_DTYPE_FP32 = 0, 1
SFM_MLP_GELU, SFM_MLP_SWIGLU = 0, 1
SFM_ROPE_1D, SFM_ROPE_3D = 0, 1
SFM_NOALLOC_SCRATCH_BYTES = 64 << 20
SFM_LINEAR_F32, SFM_LINEAR_OUT, SFM_LINEAR_GELU, SFM_LINEAR_RESID = 0, 1, 2, 3


class sfm_config(C.Structure):
    _fields_ = [("n_layers", C.c_int), ("d_model", C.c_int), ("n_heads", C.c_int),
                ("head_dim", C.c_int), ("d_mlp", C.c_int), ("c_lat", C.c_int),
                ("n_video", C.c_int), ("n_audio", C.c_int), ("unit_kv_tokens", C.c_int),
                ("max_sessions", C.c_int), ("pool_tokens", C.c_longlong), ("dtype", C.c_int),
                ("ring", C.c_int), ("rope_theta", C.c_double), ("rms_eps", C.c_double),
                ("mlp", C.c_int), ("rope", C.c_int), ("grid_w", C.c_int)]


_PP = C.POINTER(C.c_void_p)


class sfm_weights(C.Structure):
    _fields_ = [("w_in", C.c_void_p), ("e_mod", C.c_void_p), ("g_final", C.c_void_p),
                ("w_out", C.c_void_p), ("g_attn", _PP), ("w_qkv", _PP), ("w_o", _PP),
                ("g_mlp", _PP), ("w_1", _PP), ("w_2", _PP)]


class sfm_session_info(C.Structure):
    _fields_ = [("cache_units", C.c_int), ("units_appended", C.c_longlong),
                ("valid_tokens", C.c_longlong), ("p0", C.c_longlong), ("base_row", C.c_longlong)]


class sfm_plan(C.Structure):
    _fields_ = [("block_n", C.c_int * 4), ("pair", C.c_int * 4), ("k_splits", C.c_int * 4),
                ("fused_norm", C.c_int)]


class SfmError(RuntimeError):
    def __init__(self, status, what=""):
        self.status = status
        msg = lib.sfm_strerror(status).decode() if lib is not None else str(status)
        if status == SFM_ECUDA:
            msg += f" (cudaError {lib.sfm_last_cuda_error()})"
        super().__init__(f"{what}: {msg} [{status}]" if what else f"{msg} [{status}]")


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"libsfm.so is not built ({LIB_PATH}); build it with "
            "`python streaming_flow_matching_b200/build.py`")
    L = C.CDLL(LIB_PATH)
    vp, i, ll, f, sz = C.c_void_p, C.c_int, C.c_longlong, C.c_float, C.c_size_t
    sig = {
        "sfm_create": (i, [C.POINTER(sfm_config), C.POINTER(sfm_weights), C.POINTER(vp)]),
        "sfm_destroy": (None, [vp]),
        "sfm_session_open": (i, [vp, i, C.POINTER(i)]),
        "sfm_session_reset": (i, [vp, i]),
        "sfm_session_get_info": (i, [vp, i, C.POINTER(sfm_session_info)]),
        "sfm_kvcache_append": (i, [vp, i, vp, vp, i, vp]),
        "sfm_kvcache_append_heads": (i, [vp, i, vp, vp, i, i, i, vp]),
        "sfm_kvcache_read": (i, [vp, i, i, ll, ll, vp, vp, vp]),
        "sfm_denoise_step": (i, [vp, i, vp, f, f, vp, vp]),
        "sfm_fm_solve": (i, [vp, i, vp, C.POINTER(f), i, vp]),
        "sfm_fm_solve_batched": (i, [vp, i, C.POINTER(i), C.POINTER(vp), C.POINTER(f), i, vp]),
        "sfm_fm_solve_guided": (i, [vp, i, i, vp, C.POINTER(f), i, f, vp]),
        "sfm_fm_solve_guided_batched": (i, [vp, i, C.POINTER(i), C.POINTER(i), C.POINTER(vp),
                                            C.POINTER(f), i, f, C.POINTER(vp), vp]),
        "sfm_velocity_units": (i, [vp, i, i, C.POINTER(vp), C.POINTER(f), C.POINTER(vp), i, vp]),
        "sfm_set_graph_mode": (i, [vp, i]),
        "sfm_attention_workspace_bytes": (sz, [i, i, i, i, i]),
        "sfm_attention": (i, [vp, vp, vp, vp, i, i, i, i, i, vp, sz, vp]),
        "sfm_attention_block_causal": (i, [vp, vp, vp, vp, i, i, i, i, i, i, vp, sz, vp]),
        "sfm_attention_noalloc": (i, [vp, vp, vp, vp, i, i, i, i, i, vp]),
        "sfm_linear": (i, [vp, vp, vp, i, i, i, i, i, vp]),
        "sfm_check_device_error": (i, [vp, C.POINTER(i)]),
        "sfm_clear_device_error": (i, [vp]),
        "sfm_check_call_error": (i, [C.POINTER(i)]),
        "sfm_test_fault": (i, [vp, i, ll]),
        "sfm_get_plan": (i, [vp, C.POINTER(sfm_plan)]),
        "sfm_attention_batch_splits": (i, [i, i, C.POINTER(ll), i, i, C.POINTER(i)]),
        "sfm_euler_update": (i, [vp, vp, f, ll, vp]),
        "sfm_fm_solve_exact_velocity": (i, [vp, vp, vp, C.POINTER(f), i, vp]),
        "sfm_profile_begin": (i, [i]),
        "sfm_profile_end": (i, [C.POINTER(C.c_double), C.POINTER(ll)]),
        "sfm_kernel_launch_count": (C.c_ulonglong, []),
        "sfm_strerror": (C.c_char_p, [i]),
        "sfm_last_cuda_error": (i, []),
    }
    for name, (res, args) in sig.items():
        fn = getattr(L, name)
        fn.restype = res
        fn.argtypes = args
    return L


lib = None
lib = _load()

# Every symbol declared in include/sfm.h, in declaration order.
EXPORTS = ["sfm_create", "sfm_destroy", "sfm_session_open", "sfm_session_reset",
           "sfm_session_get_info", "sfm_kvcache_append", "sfm_kvcache_append_heads",
           "sfm_kvcache_read", "sfm_denoise_step",
           "sfm_fm_solve", "sfm_fm_solve_batched", "sfm_fm_solve_guided",
           "sfm_fm_solve_guided_batched", "sfm_velocity_units", "sfm_set_graph_mode",
           "sfm_attention_workspace_bytes", "sfm_attention", "sfm_attention_block_causal",
           "sfm_attention_noalloc", "sfm_linear", "sfm_euler_update", "sfm_fm_solve_exact_velocity",
           "sfm_profile_begin", "sfm_profile_end", "sfm_kernel_launch_count",
           "sfm_check_device_error", "sfm_clear_device_error", "sfm_check_call_error",
           "sfm_test_fault", "sfm_get_plan", "sfm_attention_batch_splits", "sfm_strerror",
           "sfm_last_cuda_error"]

PROF_KINDS = ["append", "attention", "attention_merge", "gemm_qkv", "gemm_o", "gemm_up",
              "gemm_down", "rowops", "head_euler"]


def attention_batch_splits(rows_per_session, n_keys, n_heads, sms=148):
    """The split counts the batched attention gives each session (host only)."""
    n = len(n_keys)
    keys = (C.c_longlong * max(1, n))(*n_keys)
    out = (C.c_int * max(1, n))()
    check(lib.sfm_attention_batch_splits(n, rows_per_session, keys, n_heads, sms, out),
          "sfm_attention_batch_splits")
    return list(out[:n])


def profile_begin(max_launches=1 << 16):
    check(lib.sfm_profile_begin(max_launches), "sfm_profile_begin")


def profile_end():
    """Per kernel class: (summed device ms, launches) since profile_begin."""
    ms = (C.c_double * len(PROF_KINDS))()
    n = (C.c_longlong * len(PROF_KINDS))()
    check(lib.sfm_profile_end(ms, n), "sfm_profile_end")
    return {k: (ms[i], n[i]) for i, k in enumerate(PROF_KINDS)}


def check_call_error():
    """Synchronises the current device; returns and clears the standalone calls' error word."""
    code = C.c_int()
    check(lib.sfm_check_call_error(C.byref(code)), "sfm_check_call_error")
    return code.value


def set_call_fault(faults, wait_ns=0):
    """Test-only: fault bits and wait bound of the standalone calls (0, 0 = normal)."""
    check(lib.sfm_test_fault(None, faults, wait_ns), "sfm_test_fault")


def check(status, what=""):
    if status != SFM_OK:
        raise SfmError(status, what)
    return status
