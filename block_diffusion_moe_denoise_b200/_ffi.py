"""ctypes declarations of the libdg C ABI (include/dg.h, include/dg_ops.h)."""
from __future__ import annotations

import ctypes as C
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libdg.so")

DG_OK = 0
ERRORS = {-1: "DG_E_ARG", -2: "DG_E_STATE", -3: "DG_E_CAPACITY", -4: "DG_E_CUDA", -5: "DG_E_DEVICE",
          -6: "DG_E_UNSUPPORTED"}
DG_MAX_REQUESTS = 8


class dg_config(C.Structure):
    _fields_ = [(n, C.c_int) for n in ("n_layers", "d_model", "n_q_heads", "n_kv_heads", "head_dim", "n_experts",
                                       "top_k", "ffn_expert", "ffn_shared", "vocab", "canvas", "max_steps",
                                       "min_accept")] + \
               [("entropy_thresh", C.c_float), ("rope_theta", C.c_float), ("norm_eps", C.c_float),
                ("sampler", C.c_int), ("entropy_budget", C.c_float), ("stop_entropy", C.c_float),
                ("temperature", C.c_float), ("ffn_selfcond", C.c_int), ("selfcond_topk", C.c_int),
                ("expert_fp8", C.c_int)]


class dg_layer_weights(C.Structure):
    _fields_ = [(n, C.c_void_p) for n in ("attn_norm", "w_qkv", "w_o", "ffn_norm", "w_router", "w_gate", "w_up",
                                          "w_down", "ws_gate", "ws_up", "ws_down", "w_gate_scale", "w_up_scale",
                                          "w_down_scale")]


class dg_weights(C.Structure):
    _fields_ = [("embed", C.c_void_p), ("final_norm", C.c_void_p), ("layers", C.POINTER(dg_layer_weights)),
                ("sc_gate", C.c_void_p), ("sc_up", C.c_void_p), ("sc_down", C.c_void_p)]


class DGError(RuntimeError):
    def __init__(self, code: int, what: str):
        super().__init__(f"{what}: {ERRORS.get(code, code)} ({code})")
        self.code = code


_lib = None

_SIGS = {
    "dg_workspace_size": (C.c_size_t, [C.POINTER(dg_config), C.c_int, C.c_int64]),
    "dg_init": (C.c_int, [C.POINTER(dg_config), C.POINTER(dg_weights), C.c_int, C.c_int64, C.c_void_p, C.c_size_t,
                          C.c_void_p, C.POINTER(C.c_void_p)]),
    "dg_destroy": (None, [C.c_void_p]),
    "dg_strerror": (C.c_char_p, [C.c_int]),
    "dg_prefill": (C.c_int, [C.c_void_p, C.c_int, C.c_void_p, C.c_int]),
    "dg_set_kv": (C.c_int, [C.c_void_p, C.c_int, C.c_int, C.c_int64, C.c_int64, C.c_void_p, C.c_void_p]),
    "dg_get_kv": (C.c_int, [C.c_void_p, C.c_int, C.c_int, C.c_int64, C.c_int64, C.c_void_p, C.c_void_p]),
    "dg_set_kv_len": (C.c_int, [C.c_void_p, C.c_int, C.c_int64]),
    "dg_kv_len": (C.c_int64, [C.c_void_p, C.c_int]),
    "dg_open_canvas": (C.c_int, [C.c_void_p, C.c_int, C.c_uint64, C.c_int]),
    "dg_denoise_step": (C.c_int, [C.c_void_p, C.c_int, C.POINTER(C.c_int), C.c_void_p]),
    "dg_read_remaining": (C.c_int, [C.c_void_p, C.c_int, C.POINTER(C.c_int32)]),
    "dg_commit_block": (C.c_int, [C.c_void_p, C.c_int]),
    "dg_generate": (C.c_int, [C.c_void_p, C.c_int, C.c_void_p, C.c_int, C.c_int, C.c_uint64, C.c_void_p,
                              C.POINTER(C.c_int)]),
    "dg_get_canvas": (C.c_int, [C.c_void_p, C.c_int, C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p]),
    "dg_set_canvas": (C.c_int, [C.c_void_p, C.c_int, C.c_void_p, C.c_void_p, C.c_int]),
    "dg_sync": (C.c_int, [C.c_void_p]),
    "dg_op_philox_tokens": (C.c_int, [C.c_uint64, C.c_int, C.c_int, C.c_int, C.c_int64, C.c_int64, C.c_int,
                                      C.c_void_p, C.c_void_p]),
    "dg_op_route_topk": (C.c_int, [C.c_void_p, C.c_int, C.c_int, C.c_int, C.c_void_p, C.c_void_p, C.c_void_p]),
    "dg_op_route_group": (C.c_int, [C.c_void_p, C.c_void_p, C.c_void_p, C.c_int, C.c_void_p, C.c_void_p,
                                    C.c_void_p]),
    "dg_op_sample": (C.c_int, [C.c_void_p, C.c_int, C.c_void_p, C.c_void_p, C.c_void_p, C.c_int]),
    "dg_op_lm_head": (C.c_int, [C.c_void_p, C.c_void_p, C.c_int, C.c_void_p, C.c_void_p, C.c_void_p]),
    "dg_op_selfcond": (C.c_int, [C.c_void_p, C.c_int, C.c_void_p, C.c_int, C.c_void_p, C.c_void_p]),
    "dg_op_lm_sample": (C.c_int, [C.c_void_p, C.c_void_p, C.c_int, C.c_float, C.c_uint64, C.c_int, C.c_int, C.c_int,
                                  C.c_void_p, C.c_void_p, C.c_void_p]),
    "dg_profile": (C.c_int, [C.c_void_p, C.c_int]),
    "dg_profile_read": (C.c_int, [C.c_void_p, C.c_char_p, C.POINTER(C.c_double), C.POINTER(C.c_int64)]),
    "dg_launch_count": (C.c_int64, [C.c_void_p]),
    "dg_op_lm_head_noalloc": (C.c_int, [C.c_void_p, C.c_void_p, C.c_void_p, C.c_int, C.c_int, C.c_int,
                                        C.c_float, C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p]),
    "dg_debug_forward": (C.c_int, [C.c_void_p, C.c_int, C.c_void_p, C.c_int, C.c_int]),
    "dg_debug_forward_hidden": (C.c_int, [C.c_void_p, C.c_int, C.c_void_p, C.c_void_p, C.c_int, C.c_int,
                                          C.c_int]),
    "dg_debug_buffer": (C.c_int, [C.c_void_p, C.c_char_p, C.POINTER(C.c_size_t), C.POINTER(C.c_size_t)]),
}


def exported_symbols():
    return list(_SIGS)


def load():
    """Load libdg.so (built in-tree).  Raises if it is missing: there is no fallback."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"libdg.so not built at {LIB_PATH}; run block_diffusion_moe_denoise_b200/build.py")
    lib = C.CDLL(LIB_PATH)
    for name, (res, args) in _SIGS.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def check(code: int, what: str) -> None:
    if code != DG_OK:
        raise DGError(code, what)
