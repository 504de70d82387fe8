"""ctypes declarations of libttt.so — the same names and arguments as include/ttt.h.

Nothing here computes: every entry point marshals integers (device pointers, sizes,
stream handles) into the C library. If the library is missing or fails to load, the
import raises; there is no fallback path.
"""

from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "lib", "libttt.so")

TTT_OK = 0
TTT_ERR_INVALID_ARG = 1
TTT_ERR_UNSUPPORTED = 2
TTT_ERR_OOM = 3
TTT_ERR_CUDA = 4
TTT_ERR_TIMEOUT = 5
TTT_ERR_DEVICE = 6
STATUS_NAMES = {0: "TTT_OK", 1: "TTT_ERR_INVALID_ARG", 2: "TTT_ERR_UNSUPPORTED", 3: "TTT_ERR_OOM",
                4: "TTT_ERR_CUDA", 5: "TTT_ERR_TIMEOUT", 6: "TTT_ERR_DEVICE"}

TTT_RULE_INPLACE_HEBBIAN = 0
TTT_RULE_LINEAR_GD = 1
TTT_RULE_LINEAR_LN_GD = 2
TTT_RULE_MLP_GD = 3
TTT_F32 = 0
TTT_BF16 = 1

TTT_OPT_LINEAR_CHUNK = 1
TTT_OPT_WAIT_LIMIT_NS = 2
TTT_OPT_INJECT_STALL = 3
TTT_OPT_INPLACE_PREFIX = 4
TTT_OPT_SM_PAIR = 5
TTT_OPT_GATE_TOKENS = 6


class ttt_config(ctypes.Structure):
    _fields_ = [
        ("rule", ctypes.c_int32),
        ("io_dtype", ctypes.c_int32),
        ("batch", ctypes.c_int32),
        ("heads", ctypes.c_int32),
        ("d_key", ctypes.c_int32),
        ("d_val", ctypes.c_int32),
        ("chunk", ctypes.c_int32),
        ("eta", ctypes.c_float),
        ("target_mode", ctypes.c_int32),
        ("conv_pad_mode", ctypes.c_int32),
        ("conv_taps", ctypes.c_int32),
        ("gate_enable", ctypes.c_int32),
        ("gate_chunk", ctypes.c_int32),
        ("cache_capacity", ctypes.c_int32),
        ("gate_pct", ctypes.c_float),
        ("gate_ema_old", ctypes.c_float),
        ("gate_ema_new", ctypes.c_float),
        ("gate_mean_num", ctypes.c_int32),
        ("gate_mean_den", ctypes.c_int32),
        ("ln_eps", ctypes.c_float),
        ("token_weights", ctypes.c_int32),
    ]


_vp = ctypes.c_void_p
_st = ctypes.c_int
_SIGNATURES = {
    "ttt_abi_version": (ctypes.c_int32, []),
    "ttt_config_init": (_st, [ctypes.POINTER(ttt_config), ctypes.c_int32]),
    "ttt_state_create": (_st, [ctypes.POINTER(ttt_config), _vp, _vp, _vp, _vp, ctypes.POINTER(_vp)]),
    "ttt_chunk_scan": (_st, [_vp, _vp, _vp, _vp, ctypes.c_int64, _vp, _vp, _vp]),
    "ttt_chunk_scan_host": (_st, [_vp, _vp, _vp, _vp, ctypes.c_int64, _vp, _vp, _vp]),
    "ttt_chunk_scan_docs": (_st, [_vp, _vp, _vp, ctypes.c_int64, _vp, _vp, ctypes.c_int32, ctypes.c_float, _vp]),
    "ttt_chunk_scan_packed": (_st, [_vp, _vp, _vp, _vp, ctypes.c_int64, _vp, _vp, _vp, _vp, _vp]),
    "ttt_surprisal_route": (_st, [_vp, _vp, ctypes.c_int64, _vp]),
    "ttt_state_reset": (_st, [_vp, _vp]),
    "ttt_state_get_weights": (_st, [_vp, _vp, _vp]),
    "ttt_state_set_weights": (_st, [_vp, _vp, _vp]),
    "ttt_add_f32": (_st, [_vp, _vp, ctypes.c_float, ctypes.c_int64, _vp]),
    "ttt_state_set_layernorm": (_st, [_vp, _vp, _vp, _vp]),
    "ttt_cache_read": (_st, [_vp, _vp, _vp, _vp]),
    "ttt_gate_read": (_st, [_vp, _vp, _vp, _vp]),
    "ttt_state_set_option": (_st, [_vp, ctypes.c_int32, ctypes.c_int64]),
    "ttt_cache_attention": (_st, [_vp, _vp, _vp, _vp, _vp, _vp, ctypes.c_int64, _vp, _vp]),
    "ttt_state_poll": (_st, [_vp]),
    "ttt_state_launch_count": (ctypes.c_int64, [_vp]),
    "ttt_state_destroy": (_st, [_vp]),
    "ttt_last_error_string": (ctypes.c_char_p, []),
    "ttt_target_values_noalloc": (_st, [_vp, _vp, _vp, ctypes.c_int64, ctypes.c_int32, ctypes.c_int32,
                                        ctypes.c_int32, ctypes.c_int32, _vp, _vp, _vp]),
}

_lib = None


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libttt.so (once) and declare every entry point; raises if it is missing."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"libttt.so not found at {path}; build it with "
                           "`python -m chunked_weight_layers_b200.build`")
    lib = ctypes.CDLL(path)
    for name, (res, args) in _SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def exported_symbols() -> list[str]:
    return list(_SIGNATURES)


class TTTError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {message}")
        self.status = status


def check(status: int) -> None:
    if status != TTT_OK:
        msg = load().ttt_last_error_string()
        raise TTTError(status, msg.decode() if msg else "")
