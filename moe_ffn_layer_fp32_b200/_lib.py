"""ctypes view of libmmoe.so (the C ABI declared in include/mmoe.h).

Only argument marshalling lives here.  The library must have been built
(``moe_ffn_layer_fp32_b200.build.build()``); there is no fallback of any kind:
loading fails loudly when the shared object is missing.
"""
from __future__ import annotations

import ctypes as C
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
SO_PATH = os.path.join(_PKG, "libmmoe.so")

MMOE_OK = 0
STATUS_NAMES = {0: "OK", 1: "INVALID_ARG", 2: "NOT_LOADED", 3: "OOM", 4: "CUDA", 5: "TIMEOUT", 6: "UNIMPLEMENTED"}

GATE_SOFTMAX = 0
GATE_SIGMOID_TOPK_NORM = 1
GATE_SIGMOID_TOPK_NORM_SEL_BIAS = 2
FLAG_DETERMINISTIC = 1
FLAG_CUDA_CORES = 2
FLAG_NO_DECODE = 4
FLAG_ATOMIC_COMBINE = 8
FLAG_TC_INT8 = 16
FLAG_NO_FUSED_DECODE = 32
FLAG_FUSED_REQUANT = 64

STAGE_XQ, STAGE_SX, STAGE_OFFSETS, STAGE_ROW_SRC, STAGE_SLOT_ROW, STAGE_HQ, STAGE_SH, STAGE_LOGITS = range(8)

# every symbol include/mmoe.h declares
EXPORTS = ("mmoe_create", "mmoe_load_quantized_weights", "mmoe_forward", "mmoe_forward_host", "mmoe_destroy",
           "mmoe_last_error", "mmoe_quantize_int4", "mmoe_debug_copy_stage", "mmoe_debug_partials",
           "mmoe_profile_enable", "mmoe_profile_read", "mmoe_forward_static_scratch", "mmoe_debug_host_chunks",
           "mmoe_debug_set_wait_limit", "mmoe_debug_fail_alloc", "mmoe_forward_chain")
MAX_CHAIN_LAYERS = 32

STATIC_SCRATCH_BYTES = 8 * 1024 * 1024

PROF_STAGES = ("zero_y", "router", "permute", "gate_up", "requant", "down", "combine", "decode_fused")


class MMoEError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"mmoe status {status} ({STATUS_NAMES.get(status, '?')}): {message}")
        self.status = status


class Config(C.Structure):
    _fields_ = [("d_model", C.c_int32), ("n_experts", C.c_int32), ("top_k", C.c_int32),
                ("expert_hidden", C.c_int32), ("shared_hidden", C.c_int32), ("group_size", C.c_int32),
                ("max_tokens", C.c_int32), ("gating", C.c_int32), ("has_router_bias", C.c_int32),
                ("flags", C.c_uint32)]


class Weights(C.Structure):
    _fields_ = [("w_router", C.c_void_p), ("router_bias", C.c_void_p), ("w_gate_up", C.c_void_p),
                ("s_gate_up", C.c_void_p), ("w_down", C.c_void_p), ("s_down", C.c_void_p),
                ("on_device", C.c_int32)]


_lib = None


def lib() -> C.CDLL:
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(SO_PATH):
        raise RuntimeError(f"{SO_PATH} is missing: build the CUDA library first "
                           "(python -m moe_ffn_layer_fp32_b200.build or __graft_entry__.build())")
    L = C.CDLL(SO_PATH)
    vp, i64, i32, st = C.c_void_p, C.c_int64, C.c_int32, C.c_int
    L.mmoe_create.argtypes = [C.POINTER(Config), C.c_int, C.POINTER(vp)]
    L.mmoe_load_quantized_weights.argtypes = [vp, C.POINTER(Weights), vp]
    L.mmoe_forward.argtypes = [vp, vp, i64, vp, vp, vp, vp, vp]
    L.mmoe_forward_host.argtypes = [vp, vp, i64, vp, vp]
    L.mmoe_destroy.argtypes = [vp]
    L.mmoe_last_error.argtypes = []
    L.mmoe_last_error.restype = C.c_char_p
    L.mmoe_quantize_int4.argtypes = [vp, i64, i64, vp, vp, vp]
    L.mmoe_debug_copy_stage.argtypes = [vp, i32, vp, C.c_size_t, vp]
    L.mmoe_debug_partials.argtypes = [vp, i32, i64, i64, vp, vp]
    L.mmoe_profile_enable.argtypes = [vp, i32]
    L.mmoe_profile_read.argtypes = [vp, vp, vp, i32]
    L.mmoe_forward_static_scratch.argtypes = [C.POINTER(Config), C.POINTER(Weights), vp, i64, vp, vp]
    L.mmoe_debug_host_chunks.argtypes = [i64, vp, i32, vp]
    L.mmoe_debug_set_wait_limit.argtypes = [vp, i64, i32]
    L.mmoe_debug_fail_alloc.argtypes = [i64]
    L.mmoe_forward_chain.argtypes = [C.POINTER(vp), i32, vp, i64, C.POINTER(vp), vp]
    for name in EXPORTS:
        if name != "mmoe_last_error":
            getattr(L, name).restype = st
    _lib = L
    return L


def check(status: int) -> None:
    if status != MMOE_OK:
        raise MMoEError(status, lib().mmoe_last_error().decode(errors="replace"))
