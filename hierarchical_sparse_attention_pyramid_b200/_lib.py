"""ctypes view of liblh.so (the C ABI declared in include/lh.h).

Loading is lazy and loud: if the shared library is missing the first call
raises; there is no fallback implementation.
"""

from __future__ import annotations

import ctypes
import os
from ctypes import POINTER, c_char_p, c_int, c_int32, c_int64, c_size_t, c_void_p

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "liblh.so")
MAX_LEVELS = 16
ERR_WORD_BYTES = 256
SELFTEST_WS_BYTES = 131072

LH_OK = 0
STATUS_NAMES = {0: "LH_OK", 1: "LH_ERR_INVALID_ARG", 2: "LH_ERR_UNSUPPORTED", 3: "LH_ERR_WORKSPACE",
                4: "LH_ERR_CUDA", 5: "LH_ERR_TIMEOUT", 6: "LH_ERR_DEVICE"}
DTYPES = {"bf16": 0, "fp32": 1}
SCORERS = {"qk_sum": 0, "k": 1, "q": 2}
SELECTIONS = {"parents": 0, "direct": 1, "nested": 2}


class LhConfig(ctypes.Structure):
    _fields_ = [("B", c_int64), ("H", c_int64), ("N", c_int64), ("d", c_int32), ("L", c_int32), ("p", c_int32),
                ("k", c_int32), ("chunk", c_int32), ("dtype", c_int32), ("scorer", c_int32),
                ("selection", c_int32)]


_SIZES = ["pyr_bytes", "norms_bytes", "topk_ws_bytes", "sel_bytes", "seq_bytes", "os_bytes", "seq_map_bytes", "slot_of_bytes",
          "lse_bytes", "grad_seq_bytes", "attn_bwd_ws_bytes", "ctx_bytes", "ws_bytes",
          "ctx_off_sel", "ctx_off_seq_map", "ctx_off_slot_of", "ctx_off_qs", "ctx_off_ks", "ctx_off_vs",
          "ctx_off_os", "ctx_off_lse",
          "ws_off_pyr_q", "ws_off_pyr_k", "ws_off_pyr_v", "ws_off_norms", "ws_off_topk",
          "ws_off_dos", "ws_off_delta", "ws_off_dqs", "ws_off_dks", "ws_off_dvs"]


class LhPlanInfo(ctypes.Structure):
    _fields_ = ([("S", c_int64), ("pyr_entries", c_int64), ("level_len", c_int64 * MAX_LEVELS),
                 ("level_off", c_int64 * MAX_LEVELS), ("upper_off", c_int64 * MAX_LEVELS),
                 ("upper_entries", c_int64), ("kprime", c_int32 * MAX_LEVELS), ("sel_off", c_int64 * MAX_LEVELS),
                 ("sel_per_head", c_int64)]
                + [(n, c_size_t) for n in _SIZES] + [("first_level", c_int32)])


class LhPisaConfig(ctypes.Structure):
    _fields_ = [("B", c_int64), ("H", c_int64), ("N", c_int64), ("d", c_int32), ("p", c_int32), ("L", c_int32),
                ("block", c_int32), ("group", c_int32), ("topk", c_int32)]


class LhPisaInfo(ctypes.Structure):
    _fields_ = [("n_groups", c_int64), ("blocks", c_int64 * MAX_LEVELS), ("level_off", c_int64 * MAX_LEVELS),
                ("upper_entries", c_int64), ("pyr_bytes", c_size_t), ("kept_elems", c_size_t),
                ("max_candidates", c_int32)]


_P = c_void_p
_CFG = POINTER(LhConfig)
_PCFG = POINTER(LhPisaConfig)
# name -> argument types (all return lh_status unless listed in _RESTYPES)
SIGNATURES = {
    "lh_plan": [_CFG, POINTER(LhPlanInfo)],
    "lh_pyramid_pool": [_CFG, _P, _P, _P, _P, _P, _P, _P, _P],
    "lh_pyramid_pool_from": [_CFG, c_int32, _P, _P, _P, _P, _P, _P, _P, _P],
    "lh_score_topk": [_CFG, _P, _P, _P, _P],
    "lh_score_topk_static": [_CFG, _P, _P, _P],
    "lh_gather": [_CFG, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P],
    "lh_gather_from": [_CFG, c_int32, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P],
    "lh_attn_fwd": [_CFG, c_int64, _P, _P, _P, _P, _P, _P, _P],
    "lh_attn_bwd": [_CFG, c_int64, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P],
    "lh_gather_shard": [_CFG, c_int64, c_int64, _P, c_int64, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P],
    "lh_scatter_back_shard": [_CFG, c_int64, _P, _P, _P, _P, _P],
    "lh_scatter_back_adjoint_shard": [_CFG, c_int64, _P, _P, _P, _P, _P, _P, _P],
    "lh_pool_adjoint_shard": [_CFG, c_int64, _P, _P, _P, _P, _P, _P, _P, _P],
    "lh_head_sums": [_CFG, _P, _P, _P],
    "lh_attn_fwd_rows": [_CFG, c_int64, c_int64, c_int64, _P, _P, _P, _P, _P, _P, _P],
    "lh_attn_bwd_rows": [_CFG, c_int64, c_int64, c_int64, c_int64, c_int64, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P],
    "lh_scatter_back": [_CFG, _P, _P, _P, _P],
    "lh_scatter_back_adjoint": [_CFG, _P, _P, _P, _P, _P, _P],
    "lh_pool_adjoint": [_CFG, _P, _P, _P, _P, _P, _P, _P, _P],
    "lh_forward": [_CFG, _P, _P, _P, _P, _P, c_size_t, _P, c_size_t, _P],
    "lh_backward": [_CFG, _P, _P, c_size_t, _P, _P, _P, _P, c_size_t, _P],
    "lh_pisa_plan": [_PCFG, POINTER(LhPisaInfo)],
    "lh_pisa_pool_keys": [_PCFG, _P, _P, _P],
    "lh_pisa_select": [_PCFG, _P, _P, _P, _P, _P, _P, _P],
    "lh_selftest_wait_timeout": [_P, c_size_t, c_int64, _P],
    "lh_check_error": [_P, _P],
    "lh_clear_error": [_P, _P],
    "lh_status_string": [c_int],
    "lh_last_error_message": [],
}
_RESTYPES = {"lh_status_string": c_char_p, "lh_last_error_message": c_char_p}

_lib = None


def load(path: str = LIB_PATH):
    """Load liblh.so once and attach the prototypes."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"liblh.so not found at {path}: run `python -m hierarchical_sparse_attention_pyramid_b200.build`")
    lib = ctypes.CDLL(path)
    for name, args in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = _RESTYPES.get(name, c_int)
    _lib = lib
    return lib


class LhError(RuntimeError):
    def __init__(self, status: int, call: str):
        lib = load()
        self.status = status
        msg = lib.lh_last_error_message().decode()
        super().__init__(f"{call} -> {STATUS_NAMES.get(status, status)} ({lib.lh_status_string(status).decode()}): {msg}")


def call(name: str, *args) -> None:
    status = getattr(load(), name)(*args)
    if status != LH_OK:
        raise LhError(status, name)
