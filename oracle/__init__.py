"""CPU oracle of the fused MoE FFN layer -- TEST INFRASTRUCTURE ONLY.

Plain C (mmoe_oracle.c) behind ctypes.  Only tests/, ``__graft_entry__.smoke()``
and the CPU-baseline leg of bench.py may import this package; the library in
``moe_ffn_layer_fp32_b200`` never does, and the two share no code.

Every function follows the MobileMoE pages (paper-archivist reading):
Eq. (*) for the layer, Eq. (6) for the INT4 weights, section "QAT" for the
dynamic INT8 activations, "MoE training stability techniques" for the FP32
router.  See mmoe_oracle.c for the precision of every step.
"""
from __future__ import annotations

import ctypes as C
import os
import subprocess
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "mmoe_oracle.c")
_BUILD = os.path.join(_HERE, "_build")
_SO = os.path.join(_BUILD, "liboracle.so")
GROUP = 32


def compile_oracle(src: str, out: str) -> None:
    """gcc -O2 with OpenMP over tokens and no fused multiply-adds: the oracle's build flags."""
    cmd = ["gcc", "-O2", "-march=native", "-fopenmp", "-ffp-contract=off", "-fno-fast-math",
           "-std=c11", "-Wall", "-shared", "-fPIC", "-o", out, src, "-lm"]
    subprocess.run(cmd, check=True)


def build(force: bool = False) -> str:
    """Compile the oracle (see compile_oracle) into oracle/_build if it is out of date."""
    if not force and os.path.exists(_SO) and os.path.getmtime(_SO) >= os.path.getmtime(_SRC):
        return _SO
    os.makedirs(_BUILD, exist_ok=True)
    tmp = _SO + f".{os.getpid()}.tmp"
    compile_oracle(_SRC, tmp)
    os.replace(tmp, _SO)
    return _SO


class _Layer(C.Structure):
    _fields_ = [("d", C.c_int64), ("h", C.c_int64), ("hs", C.c_int64), ("E", C.c_int64),
                ("k", C.c_int64), ("gating", C.c_int64),
                ("w_router", C.c_void_p), ("router_bias", C.c_void_p),
                ("w_gate_up", C.c_void_p), ("s_gate_up", C.c_void_p),
                ("w_down", C.c_void_p), ("s_down", C.c_void_p)]


class _Dumps(C.Structure):
    _fields_ = [(n, C.c_void_p) for n in
                ("logits", "probs", "idx", "gate", "xq", "sx", "pg", "pu", "hq", "sh", "pd", "o")]


_lib = None


def lib():
    global _lib
    if _lib is None:
        # MMOE_ORACLE_SO: another build of the oracle source (the pin tests' mutation check
        # points it at copies with one planted mistake each)
        _lib = C.CDLL(os.environ.get("MMOE_ORACLE_SO") or build())
        i64, vp = C.c_int64, C.c_void_p
        _lib.oracle_quantize_int4.argtypes = [vp, i64, i64, vp, vp]
        _lib.oracle_quantize_act.argtypes = [vp, i64, i64, vp, vp]
        _lib.oracle_router.argtypes = [C.POINTER(_Layer), vp, i64, vp, vp, vp, vp]
        _lib.oracle_expert_gate_up.argtypes = [C.POINTER(_Layer), i64, vp, C.c_float, vp, vp, vp, vp]
        _lib.oracle_expert_down.argtypes = [C.POINTER(_Layer), i64, vp, C.c_float, vp, vp]
        _lib.oracle_moe_layer.argtypes = [C.POINTER(_Layer), vp, i64, vp, C.POINTER(_Dumps)]
        _lib.oracle_moe_tokens.argtypes = [C.POINTER(_Layer), vp, i64, vp, i64, vp]
        _lib.oracle_num_threads.argtypes = []
        _lib.oracle_set_num_threads.argtypes = [C.c_int]
        for f in ("oracle_quantize_int4", "oracle_quantize_act", "oracle_router",
                  "oracle_expert_gate_up", "oracle_expert_down", "oracle_moe_layer",
                  "oracle_moe_tokens", "oracle_num_threads", "oracle_set_num_threads"):
            getattr(_lib, f).restype = C.c_int
    return _lib


def _p(a):
    return None if a is None else a.ctypes.data


def num_threads() -> int:
    return int(lib().oracle_num_threads())


def set_num_threads(n: int) -> int:
    """OpenMP threads of the following oracle calls; returns the count now in effect."""
    return int(lib().oracle_set_num_threads(int(n)))


def quantize_int4(W: np.ndarray):
    """Eq. (6) on W[rows, K] (FP32) -> (packed uint8 [rows, K/2], scales float32 [rows, K/32])."""
    W = np.ascontiguousarray(W, dtype=np.float32)
    rows, K = W.shape
    packed = np.zeros((rows, K // 2), dtype=np.uint8)
    scales = np.zeros((rows, K // GROUP), dtype=np.float32)
    if lib().oracle_quantize_int4(_p(W), rows, K, _p(packed), _p(scales)):
        raise ValueError("oracle_quantize_int4: K must be a multiple of 32")
    return packed, scales


def quantize_act(x_bf16: np.ndarray):
    """Per-token INT8 of BF16 x[T, d] -> (xq int8 [T, d], sx float32 [T])."""
    x = np.ascontiguousarray(x_bf16, dtype=np.uint16)
    T, d = x.shape
    xq = np.zeros((T, d), dtype=np.int8)
    sx = np.zeros(T, dtype=np.float32)
    if lib().oracle_quantize_act(_p(x), T, d, _p(xq), _p(sx)):
        raise MemoryError
    return xq, sx


def unpack_int4(packed: np.ndarray) -> np.ndarray:
    """Packed INT4 (low nibble = even index) -> int8 codes."""
    p = np.asarray(packed, dtype=np.uint8)
    lo = (p & 15).astype(np.int8)
    hi = (p >> 4).astype(np.int8)
    out = np.empty(p.shape[:-1] + (p.shape[-1] * 2,), dtype=np.int8)
    out[..., 0::2] = np.where(lo >= 8, lo - 16, lo)
    out[..., 1::2] = np.where(hi >= 8, hi - 16, hi)
    return out


@dataclass
class QuantizedLayer:
    """A layer in the interchange format the library also loads.

    w_gate_up: uint8, expert g's [2*hid, d/2] block at byte g*2h*d/2 (shared expert = index E)
    s_gate_up: float32, expert g's [2*hid, d/32] block at g*2h*d/32
    w_down:    uint8, expert g's [d, hid/2] block at byte g*d*h/2
    s_down:    float32, expert g's [d, hid/32] block at g*d*h/32
    """
    d: int
    h: int
    hs: int
    E: int
    k: int
    gating: int
    w_router: np.ndarray
    router_bias: np.ndarray | None
    w_gate_up: np.ndarray
    s_gate_up: np.ndarray
    w_down: np.ndarray
    s_down: np.ndarray

    def struct(self) -> _Layer:
        return _Layer(self.d, self.h, self.hs, self.E, self.k, self.gating,
                      _p(self.w_router), _p(self.router_bias), _p(self.w_gate_up),
                      _p(self.s_gate_up), _p(self.w_down), _p(self.s_down))

    def expert_codes(self, g: int):
        """(gate_up int8 codes [2*hid, d], gate_up scales, down codes [d, hid], down scales) of expert g."""
        d, h = self.d, self.h
        hid = h if g < self.E else self.hs
        wgu = self.w_gate_up[g * 2 * h * d // 2:][: 2 * hid * d // 2].reshape(2 * hid, d // 2)
        sgu = self.s_gate_up[g * 2 * h * d // GROUP:][: 2 * hid * d // GROUP].reshape(2 * hid, d // GROUP)
        wd = self.w_down[g * d * h // 2:][: d * hid // 2].reshape(d, hid // 2)
        sd = self.s_down[g * d * h // GROUP:][: d * hid // GROUP].reshape(d, hid // GROUP)
        return unpack_int4(wgu), sgu, unpack_int4(wd), sd


def quantize_layer(lw, k: int = 4, gating: int = 0) -> QuantizedLayer:
    """Quantise the FP32 weights of one layer (synth.LayerWeights) with Eq. (6)."""
    gu_w, gu_s, dn_w, dn_s = [], [], [], []
    for g in range(lw.E + 1):
        p, s = quantize_int4(lw.w_gate_up[g])
        gu_w.append(p.ravel()); gu_s.append(s.ravel())
        p, s = quantize_int4(lw.w_down[g])
        dn_w.append(p.ravel()); dn_s.append(s.ravel())
    bias = None if lw.router_bias is None else np.ascontiguousarray(lw.router_bias, dtype=np.float32)
    return QuantizedLayer(lw.d, lw.h, lw.hs, lw.E, k, gating,
                          np.ascontiguousarray(lw.w_router, dtype=np.float32), bias,
                          np.concatenate(gu_w), np.concatenate(gu_s),
                          np.concatenate(dn_w), np.concatenate(dn_s))


def router(q: QuantizedLayer, x_bf16: np.ndarray):
    """-> (logits [T,E], probs [T,E], idx int32 [T,k], gate [T,k])."""
    x = np.ascontiguousarray(x_bf16, dtype=np.uint16)
    T = x.shape[0]
    logits = np.zeros((T, q.E), np.float32)
    probs = np.zeros((T, q.E), np.float32)
    idx = np.zeros((T, q.k), np.int32)
    gate = np.zeros((T, q.k), np.float32)
    L = q.struct()
    if lib().oracle_router(C.byref(L), _p(x), T, _p(logits), _p(probs), _p(idx), _p(gate)):
        raise ValueError("oracle_router: invalid layer description or allocation failure")
    return logits, probs, idx, gate


def expert_gate_up(q: QuantizedLayer, g: int, xq_row: np.ndarray, sx: float, partials: bool = False):
    """One expert's gate/up + SwiGLU + requantisation for one token -> (hq, sh[, pg, pu])."""
    hid = q.h if g < q.E else q.hs
    xq_row = np.ascontiguousarray(xq_row, dtype=np.int8)
    hq = np.zeros(hid, np.int8)
    sh = np.zeros(1, np.float32)
    ng = q.d // GROUP
    pg = np.zeros((hid, ng), np.int32) if partials else None
    pu = np.zeros((hid, ng), np.int32) if partials else None
    L = q.struct()
    sh_c = C.c_float()
    if lib().oracle_expert_gate_up(C.byref(L), g, _p(xq_row), C.c_float(float(sx)), _p(pg), _p(pu),
                                   _p(hq), C.addressof(sh_c)):
        raise MemoryError
    return (hq, sh_c.value, pg, pu) if partials else (hq, sh_c.value)


def expert_down(q: QuantizedLayer, g: int, hq_row: np.ndarray, sh: float, partials: bool = False):
    """One expert's down projection for one token -> (o[, pd])."""
    hid = q.h if g < q.E else q.hs
    hq_row = np.ascontiguousarray(hq_row[:hid], dtype=np.int8)
    o = np.zeros(q.d, np.float32)
    pd = np.zeros((q.d, hid // GROUP), np.int32) if partials else None
    L = q.struct()
    if lib().oracle_expert_down(C.byref(L), g, _p(hq_row), C.c_float(float(sh)), _p(pd), _p(o)):
        raise MemoryError
    return (o, pd) if partials else o


def moe_layer(q: QuantizedLayer, x_bf16: np.ndarray, dumps: bool = False, partials: bool = False):
    """y[T, d] of the whole layer; with dumps=True also every stage's values (dict)."""
    x = np.ascontiguousarray(x_bf16, dtype=np.uint16)
    T = x.shape[0]
    y = np.zeros((T, q.d), np.float32)
    D = _Dumps()
    out = {}
    if dumps:
        hm = max(q.h, q.hs)
        s = q.k + 1
        out = dict(logits=np.zeros((T, q.E), np.float32), probs=np.zeros((T, q.E), np.float32),
                   idx=np.zeros((T, q.k), np.int32), gate=np.zeros((T, q.k), np.float32),
                   xq=np.zeros((T, q.d), np.int8), sx=np.zeros(T, np.float32),
                   hq=np.zeros((T, s, hm), np.int8), sh=np.zeros((T, s), np.float32),
                   o=np.zeros((T, s, q.d), np.float32))
        if partials:
            out.update(pg=np.zeros((T, s, hm, q.d // GROUP), np.int32),
                       pu=np.zeros((T, s, hm, q.d // GROUP), np.int32),
                       pd=np.zeros((T, s, q.d, hm // GROUP), np.int32))
        for name, arr in out.items():
            setattr(D, name, arr.ctypes.data)
    L = q.struct()
    if lib().oracle_moe_layer(C.byref(L), _p(x), T, _p(y), C.byref(D)):
        raise ValueError("oracle_moe_layer: invalid layer description")
    return (y, out) if dumps else y


def moe_tokens(q: QuantizedLayer, x_bf16: np.ndarray, toks) -> np.ndarray:
    """Layer output rows for the token ids in toks only."""
    x = np.ascontiguousarray(x_bf16, dtype=np.uint16)
    toks = np.ascontiguousarray(toks, dtype=np.int64)
    y = np.zeros((len(toks), q.d), np.float32)
    L = q.struct()
    if lib().oracle_moe_tokens(C.byref(L), _p(x), x.shape[0], _p(toks), len(toks), _p(y)):
        raise ValueError("oracle_moe_tokens: bad layer or token id")
    return y
