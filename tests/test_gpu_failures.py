"""Failure detection on the GPU without a GPU fault.

A device-side wait that runs out is made on purpose (a one-shot injected
stall: a wait on a barrier that nothing signals, bounded by a short limit);
the kernel drains its copies in flight and returns, the context stays usable,
the next call reports MMOE_ERR_TIMEOUT and the call after it is correct again.
Allocation failures are injected on the host (a countdown in the library's
allocator) and must leave no device memory behind.
"""
import numpy as np
import pytest
import torch

import oracle
from moe_ffn_layer_fp32_b200 import _lib, synth
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    gu.ensure_built()


def _c0():
    w = synth.WORKLOADS["c0"]
    q = oracle.quantize_layer(synth.workload_layer(w))
    return w, q, synth.workload_x(w)


def test_injected_stall_times_out_and_the_next_forward_recovers():
    w, q, x = _c0()
    L = gu.make_gpu_layer(q, w.T, decode=False)       # the prefill tensor-core GEMMs
    yref = oracle.moe_layer(q, x)
    # about 20 us of SM clock for each bounded wait, and one wait that can never complete
    L.set_wait_limit(40000, stall_next=True)
    xd = gu.x_to_device(x)
    L.forward(xd)                                      # enqueues; the stall happens on the device
    torch.cuda.synchronize()                           # the context is still usable
    L.set_wait_limit(0)
    with pytest.raises(_lib.MMoEError) as ei:
        L.forward(xd)
    assert ei.value.status == 5                        # TIMEOUT, reported once
    out = gu.run_gpu(L, q, x, stages=False)           # and the layer is correct again
    rep = {}
    gu.check_y(out["y"], yref, rep)
    L.close()


def test_short_wait_limit_alone_keeps_results_correct():
    # a tight but satisfiable limit: whether or not a wait gives up, no wrong result is reported
    # as a success, and the default limit restores normal operation
    w, q, x = _c0()
    L = gu.make_gpu_layer(q, w.T, decode=False)
    yref = oracle.moe_layer(q, x)
    xd = gu.x_to_device(x)
    L.set_wait_limit(1)
    L.forward(xd)
    torch.cuda.synchronize()
    L.set_wait_limit(0)
    try:
        y = L.forward(xd)
        torch.cuda.synchronize()
        gave_up = False
    except _lib.MMoEError as e:
        assert e.status == 5
        gave_up = True
    if gave_up:
        y = L.forward(xd)
        torch.cuda.synchronize()
    rep = {}
    gu.check_y(y.cpu().numpy(), yref, rep)
    L.close()


@pytest.mark.parametrize("after", [0, 3, 11, 25])
def test_allocation_failure_in_create_leaks_nothing(after):
    import ctypes as C
    w, q, x = _c0()
    Lb = _lib.lib()
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info()[0]
    cfg = _lib.Config(q.d, q.E, q.k, q.h, q.hs, 32, 4096, 0, 0, 0)
    h = C.c_void_p()
    assert Lb.mmoe_debug_fail_alloc(after) == 0
    st = Lb.mmoe_create(C.byref(cfg), 0, C.byref(h))
    Lb.mmoe_debug_fail_alloc(-1)
    assert st == 3 and not h.value, (st, Lb.mmoe_last_error())
    torch.cuda.synchronize()
    assert abs(torch.cuda.mem_get_info()[0] - free0) <= 4 << 20
    # without the injection the same handle is created and works
    L = gu.make_gpu_layer(q, 4096)
    out = gu.run_gpu(L, q, x, stages=False)
    gu.check_y(out["y"], oracle.moe_layer(q, x), {})
    L.close()


def test_allocation_failure_in_host_forward():
    w, q, x = _c0()
    L = gu.make_gpu_layer(q, w.T, deterministic=True)
    Lb = _lib.lib()
    assert Lb.mmoe_debug_fail_alloc(0) == 0           # the first staging buffer fails
    with pytest.raises(_lib.MMoEError) as ei:
        L.forward_host(x)
    Lb.mmoe_debug_fail_alloc(-1)
    assert ei.value.status == 3
    y = L.forward_host(x)                              # the next call allocates and runs
    gu.check_y(y, oracle.moe_layer(q, x), {})
    L.close()
