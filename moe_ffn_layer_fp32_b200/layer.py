"""Python face of the fused MoE FFN layer: a thin wrapper over the C ABI.

PyTorch provides device memory and streams; every step of the layer runs in
libmmoe.so.  Tensors are passed by pointer, nothing is computed here.
"""
from __future__ import annotations

import ctypes as C

import numpy as np
import torch

from . import _lib
from ._lib import check, lib

GROUP = 32


def _stream_ptr(stream) -> int | None:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, torch.Tensor):
        if not t.is_contiguous():
            raise ValueError("tensors passed to the library must be contiguous")
        return t.data_ptr()
    if isinstance(t, np.ndarray):
        if not t.flags["C_CONTIGUOUS"]:
            raise ValueError("arrays passed to the library must be C-contiguous")
        return t.ctypes.data
    raise TypeError(f"expected a torch.Tensor or numpy.ndarray, got {type(t).__name__}")


def quantize_int4(w: torch.Tensor, stream=None):
    """Eq. (6) on the device: FP32 W[rows, K] (cuda) -> (packed uint8 [rows, K/2], scales FP32 [rows, K/32])."""
    if w.dtype != torch.float32 or not w.is_cuda or w.dim() != 2:
        raise ValueError("w must be a 2-D float32 CUDA tensor")
    rows, K = w.shape
    if K % GROUP:
        raise ValueError("K must be a multiple of 32")
    packed = torch.empty((rows, K // 2), dtype=torch.uint8, device=w.device)
    scales = torch.empty((rows, K // GROUP), dtype=torch.float32, device=w.device)
    with torch.cuda.device(w.device):
        check(lib().mmoe_quantize_int4(_ptr(w.contiguous()), rows, K, _ptr(packed), _ptr(scales),
                                       _stream_ptr(stream)))
    return packed, scales


class MoELayer:
    """One fused MoE FFN layer (Eq. (*) of the MobileMoE pages) on one CUDA device."""

    def __init__(self, d_model: int, expert_hidden: int, *, shared_hidden: int | None = None,
                 n_experts: int = 60, top_k: int = 4, max_tokens: int = 4096, gating: int = 0,
                 has_router_bias: bool = False, deterministic: bool = False, cuda_cores: bool = False,
                 decode: bool = True, atomic_combine: bool = False, tc_int8: bool = False,
                 fused_decode: bool = True, fused_requant: bool = False, device: int = 0):
        """decode=False keeps small batches (T <= 64) on the prefill kernels instead of the
        weight-streaming decode kernels; cuda_cores=True runs every expert GEMM on CUDA cores;
        tc_int8=True runs the prefill expert GEMMs on the kind::i8 tensor-core kernels instead of the
        default kind::f16 ones; fused_decode=False keeps batches of at most 8 tokens on the four-launch
        decode kernels instead of the one-launch decode; fused_requant=True requantises the SwiGLU output
        inside the prefill gate/up GEMM (thread-block clusters); deterministic=True adds the expert outputs
        into y in the fixed order of Eq. (*) (bit-reproducible y, an [R, d] workspace) instead of with FP32
        atomics; atomic_combine is the default and changes nothing."""
        flags = ((_lib.FLAG_DETERMINISTIC if deterministic else 0) | (_lib.FLAG_CUDA_CORES if cuda_cores else 0)
                 | (0 if decode else _lib.FLAG_NO_DECODE) | (_lib.FLAG_ATOMIC_COMBINE if atomic_combine else 0)
                 | (_lib.FLAG_TC_INT8 if tc_int8 else 0) | (0 if fused_decode else _lib.FLAG_NO_FUSED_DECODE)
                 | (_lib.FLAG_FUSED_REQUANT if fused_requant else 0))
        self.cfg = _lib.Config(d_model, n_experts, top_k, expert_hidden,
                               expert_hidden if shared_hidden is None else shared_hidden, GROUP, max_tokens,
                               gating, int(has_router_bias), flags)
        self.device = device
        self._h = C.c_void_p()
        check(lib().mmoe_create(C.byref(self.cfg), device, C.byref(self._h)))

    @property
    def d_model(self):
        return self.cfg.d_model

    def close(self):
        if self._h:
            h, self._h = self._h, C.c_void_p()
            check(lib().mmoe_destroy(h))

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def load(self, w_router, router_bias, w_gate_up, s_gate_up, w_down, s_down, stream=None):
        """Weights in the interchange layout (include/mmoe.h), all CUDA tensors or all numpy arrays."""
        arrs = [w_router, router_bias, w_gate_up, s_gate_up, w_down, s_down]
        on_dev = isinstance(w_router, torch.Tensor) and w_router.is_cuda
        w = _lib.Weights(*[_ptr(a) for a in arrs], 1 if on_dev else 0)
        check(lib().mmoe_load_quantized_weights(self._h, C.byref(w), _stream_ptr(stream)))
        self._keep = arrs  # source buffers stay alive until the stream has copied them
        if not on_dev:
            torch.cuda.synchronize(self.device)

    def forward(self, x: torch.Tensor, y: torch.Tensor | None = None, *, stream=None, topk_idx=None,
                topk_gate=None, expert_counts=None) -> torch.Tensor:
        """y[T, d] (FP32) from x[T, d] (BF16), both CUDA tensors on this layer's device."""
        if x.dtype != torch.bfloat16 or x.dim() != 2 or x.shape[1] != self.cfg.d_model:
            raise ValueError("x must be a [T, d_model] bfloat16 tensor")
        T = x.shape[0]
        if y is None:
            y = torch.empty((T, self.cfg.d_model), dtype=torch.float32, device=x.device)
        check(lib().mmoe_forward(self._h, _ptr(x), T, _ptr(y), _stream_ptr(stream), _ptr(topk_idx),
                                 _ptr(topk_gate), _ptr(expert_counts)))
        return y

    __call__ = forward

    @staticmethod
    def forward_chain(layers, x: torch.Tensor, ys, stream=None) -> list:
        """Layers one after another on the same tokens: layer 0 reads x (BF16 [T, d]); layer l + 1 reads
        layer l's y rounded to BF16.  ys: one FP32 [T, d] CUDA tensor per layer (filled; returned).  For
        up to 8 tokens on the decode path the whole stack is one kernel launch."""
        if x.dtype != torch.bfloat16 or x.dim() != 2:
            raise ValueError("x must be a [T, d_model] bfloat16 tensor")
        n = len(layers)
        if len(ys) != n:
            raise ValueError("one output tensor per layer")
        hs = (C.c_void_p * n)(*[L._h.value for L in layers])
        yp = (C.c_void_p * n)(*[_ptr(y) for y in ys])
        check(lib().mmoe_forward_chain(hs, n, _ptr(x), x.shape[0], yp, _stream_ptr(stream)))
        return list(ys)

    def forward_host(self, x: np.ndarray, y: np.ndarray | None = None, stream=None) -> np.ndarray:
        """Same layer with host buffers: x uint16 (BF16 bits) [T, d] -> y float32 [T, d]; waits for the result."""
        x = np.ascontiguousarray(x, dtype=np.uint16)
        T = x.shape[0]
        if y is None:
            y = np.empty((T, self.cfg.d_model), dtype=np.float32)
        check(lib().mmoe_forward_host(self._h, _ptr(x), T, _ptr(y), _stream_ptr(stream)))
        return y

    def set_wait_limit(self, clocks: int, stall_next: bool = False) -> None:
        """SM clocks a bounded wait of the prefill tensor-core GEMMs lasts before giving up (0: default);
        stall_next=True makes the next prefill forward stall on purpose (failure-detection tests)."""
        check(lib().mmoe_debug_set_wait_limit(self._h, int(clocks), 1 if stall_next else 0))

    def profile(self, enable: bool) -> None:
        """Start (and clear) or stop per-stage event timing of the following forwards."""
        check(lib().mmoe_profile_enable(self._h, 1 if enable else 0))

    def profile_read(self) -> dict:
        """{stage: (kernel launches, summed device ms)} since the last profile(True)."""
        n = len(_lib.PROF_STAGES)
        launches = (C.c_int32 * n)()
        ms = (C.c_double * n)()
        check(lib().mmoe_profile_read(self._h, launches, ms, n))
        return {name: (int(launches[i]), float(ms[i])) for i, name in enumerate(_lib.PROF_STAGES)}

    def stage(self, stage: int, shape, dtype, stream=None) -> torch.Tensor:
        """Copy of an internal buffer of the last forward (include/mmoe.h, MMOE_STAGE_*)."""
        out = torch.empty(shape, dtype=dtype, device=f"cuda:{self.device}")
        check(lib().mmoe_debug_copy_stage(self._h, stage, _ptr(out), out.numel() * out.element_size(),
                                          _stream_ptr(stream)))
        return out

    def partials(self, which: int, row0: int, nrows: int, stream=None) -> torch.Tensor:
        """INT32 group partials of rows [row0, row0+nrows) of the last forward (0: gate/up, 1: down)."""
        c = self.cfg
        hmax = max(c.expert_hidden, c.shared_hidden)
        shape = (nrows, 2 * hmax, c.d_model // GROUP) if which == 0 else (nrows, c.d_model, hmax // GROUP)
        out = torch.zeros(shape, dtype=torch.int32, device=f"cuda:{self.device}")
        check(lib().mmoe_debug_partials(self._h, which, row0, nrows, _ptr(out), _stream_ptr(stream)))
        return out
