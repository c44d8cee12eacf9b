"""The forward that allocates nothing (mmoe_forward_static_scratch).

Some callers cannot let the library allocate device memory: a host framework
that owns all of the GPU's memory through its own pool, or a serving loop that
may not block on cudaMalloc once it runs.  This entry point keeps its scratch
in one array that the library declares in device memory, and reads the
caller's device-resident weights in place.  Its output must agree with
mmoe_forward's, within the tolerance of the other parity tests, on two calls
in a row (the second call finds the first call's data in the shared array).
This file is collected last and also passes on its own in a fresh process.
"""
import ctypes as C

import numpy as np
import pytest
import torch

from moe_ffn_layer_fp32_b200 import _lib, build, synth
from tests.gpu_util import Y_TOL

pytestmark = pytest.mark.gpu


def _device_weights(w, dev):
    from moe_ffn_layer_fp32_b200.layer import quantize_int4
    lw = synth.workload_layer(w)
    parts = {"gu_w": [], "gu_s": [], "dn_w": [], "dn_s": []}
    for g in range(w.E + 1):
        p, s = quantize_int4(torch.from_numpy(lw.w_gate_up[g]).to(dev))
        parts["gu_w"].append(p.reshape(-1)); parts["gu_s"].append(s.reshape(-1))
        p, s = quantize_int4(torch.from_numpy(lw.w_down[g]).to(dev))
        parts["dn_w"].append(p.reshape(-1)); parts["dn_s"].append(s.reshape(-1))
    wr = torch.from_numpy(lw.w_router).to(dev)
    bias = None if lw.router_bias is None else torch.from_numpy(lw.router_bias).to(dev)
    return [wr, bias, torch.cat(parts["gu_w"]), torch.cat(parts["gu_s"]), torch.cat(parts["dn_w"]),
            torch.cat(parts["dn_s"])]


def _ptr(t):
    return None if t is None else t.data_ptr()


def _static_call(L, cfg, wts, x, T, d, dev):
    y = torch.full((T, d), float("nan"), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev).cuda_stream
    _lib.check(L.mmoe_forward_static_scratch(C.byref(cfg), C.byref(wts), x.data_ptr(), T, y.data_ptr(), stream))
    torch.cuda.synchronize()
    return y


@pytest.mark.parametrize("name,flags", [("c0", 0), ("c4dec", 0), ("c4dec", _lib.FLAG_DETERMINISTIC),
                                        ("c4dec", _lib.FLAG_ATOMIC_COMBINE)])
def test_static_scratch_forward_matches_mmoe_forward(name, flags):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    build.build()
    from moe_ffn_layer_fp32_b200.layer import MoELayer
    L = _lib.lib()
    w = synth.WORKLOADS[name]
    dev = torch.device("cuda", 0)
    tensors = _device_weights(w, dev)
    x = torch.from_numpy(synth.workload_x(w).view(np.int16)).to(dev).view(torch.bfloat16)
    T = x.shape[0]

    ref_layer = MoELayer(w.d, w.h, shared_hidden=w.hs, max_tokens=T,
                         deterministic=bool(flags & _lib.FLAG_DETERMINISTIC), has_router_bias=tensors[1] is not None)
    ref_layer.load(*tensors)
    y_ref = ref_layer.forward(x)
    torch.cuda.synchronize()

    cfg = _lib.Config(w.d, w.E, w.k, w.h, w.hs, 32, T, 0, int(tensors[1] is not None), flags)
    wts = _lib.Weights(*[_ptr(t) for t in tensors], 1)
    scale = y_ref.abs().max().item()
    outs = []
    for _ in range(2):
        y = _static_call(L, cfg, wts, x, T, w.d, dev)
        err = (y - y_ref).abs().max().item()
        assert err <= Y_TOL * scale, (err, scale)
        outs.append(y)
    assert (outs[0] - outs[1]).abs().max().item() <= Y_TOL * scale
    if not flags & _lib.FLAG_ATOMIC_COMBINE:
        # the fixed-order combine (the default) makes y bit-reproducible from call to call
        assert torch.equal(outs[0], outs[1])
    ref_layer.close()


@pytest.mark.parametrize("name,sizes,flags", [("c4dec", (64, 80, 64), 0),
                                              ("c4dec", (64, 140, 64), _lib.FLAG_ATOMIC_COMBINE),
                                              ("c3b", (37, 100, 37), 0)])
def test_static_scratch_calls_of_changing_size(name, sizes, flags):
    # A larger call moves every buffer inside the shared array; the smaller call after it finds
    # the larger call's data where its own buffers now lie.  Each call must still match
    # mmoe_forward on the same tokens.  c3b carries a per-expert router bias.
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    build.build()
    from moe_ffn_layer_fp32_b200.layer import MoELayer
    L = _lib.lib()
    w = synth.WORKLOADS[name]
    dev = torch.device("cuda", 0)
    tensors = _device_weights(w, dev)
    bias = tensors[1] is not None
    assert bias == (w.bias_coef is not None)
    Tmax = max(sizes)
    ref_layer = MoELayer(w.d, w.h, shared_hidden=w.hs, max_tokens=Tmax, has_router_bias=bias)
    ref_layer.load(*tensors)
    wts = _lib.Weights(*[_ptr(t) for t in tensors], 1)
    xs = torch.from_numpy(synth.workload_x(w, T=Tmax).view(np.int16)).to(dev).view(torch.bfloat16)
    for T in sizes:
        x = xs[:T].contiguous()
        y_ref = ref_layer.forward(x)
        torch.cuda.synchronize()
        cfg = _lib.Config(w.d, w.E, w.k, w.h, w.hs, 32, T, 0, int(bias), flags)
        y = _static_call(L, cfg, wts, x, T, w.d, dev)
        scale = y_ref.abs().max().item()
        err = (y - y_ref).abs().max().item()
        assert err <= Y_TOL * scale, (T, err, scale)
    ref_layer.close()


def test_static_scratch_rejects_calls_that_do_not_fit():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    build.build()
    L = _lib.lib()
    w = synth.WORKLOADS["c4dec"]
    cfg = _lib.Config(w.d, w.E, w.k, w.h, w.hs, 32, 1, 0, 0, 0)
    dummy = torch.zeros(16, dtype=torch.uint8, device="cuda")
    wts = _lib.Weights(*([dummy.data_ptr()] * 6), 1)
    st = L.mmoe_forward_static_scratch(C.byref(cfg), C.byref(wts), dummy.data_ptr(), 4096, dummy.data_ptr(), None)
    assert st == 1 and b"static scratch" in L.mmoe_last_error()
