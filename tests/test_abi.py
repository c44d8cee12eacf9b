"""The C ABI without a GPU: the library loads, exports every symbol that
include/mmoe.h declares, and rejects bad arguments before touching a device."""
import ctypes as C
import os
import re

import pytest

from moe_ffn_layer_fp32_b200 import _lib, build
from tests.conftest import ROOT


@pytest.fixture(scope="module")
def L():
    build.build()
    return _lib.lib()


def header_functions():
    src = open(os.path.join(ROOT, "include", "mmoe.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:mmoe_status|const char\*)\s+(mmoe_\w+)\s*\(", src, flags=re.M)))


def test_header_declares_the_exports():
    assert header_functions() == sorted(_lib.EXPORTS)


def test_every_declared_symbol_is_exported(L):
    for name in header_functions():
        assert hasattr(L, name), name


def valid_cfg(**kw):
    c = dict(d_model=256, n_experts=60, top_k=4, expert_hidden=128, shared_hidden=128, group_size=32,
             max_tokens=64, gating=0, has_router_bias=0, flags=0)
    c.update(kw)
    return _lib.Config(**c)


@pytest.mark.parametrize("kw", [dict(d_model=250), dict(d_model=32), dict(n_experts=0), dict(n_experts=65),
                                dict(top_k=0), dict(top_k=9), dict(n_experts=3, top_k=4),
                                dict(expert_hidden=100), dict(shared_hidden=0), dict(group_size=64),
                                dict(max_tokens=0), dict(gating=3), dict(has_router_bias=2), dict(flags=128),
                                dict(flags=0x80000000)])
def test_create_rejects_bad_config(L, kw):
    h = C.c_void_p()
    st = L.mmoe_create(C.byref(valid_cfg(**kw)), 0, C.byref(h))
    assert st == 1 and not h.value
    assert L.mmoe_last_error()


def test_null_arguments(L):
    h = C.c_void_p()
    assert L.mmoe_create(None, 0, C.byref(h)) == 1
    assert L.mmoe_create(C.byref(valid_cfg()), 0, None) == 1
    assert L.mmoe_destroy(None) == 0
    assert L.mmoe_forward(None, None, 1, None, None, None, None, None) == 1
    assert L.mmoe_forward_host(None, None, 1, None, None) == 1
    assert L.mmoe_load_quantized_weights(None, None, None) == 1
    assert L.mmoe_debug_copy_stage(None, 0, None, 0, None) == 1
    assert L.mmoe_debug_partials(None, 0, 0, 0, None, None) == 1


def test_forward_chain_validates_before_any_device_work(L):
    # the stack of layers: argument checks need no device
    VP = C.c_void_p
    hs = (VP * 2)(None, None)
    ys = (VP * 2)(16, 32)
    assert L.mmoe_forward_chain(None, 1, None, 1, ys, None) == 1
    assert L.mmoe_forward_chain(hs, 1, None, 1, None, None) == 1
    assert L.mmoe_forward_chain(hs, 0, None, 1, ys, None) == 1
    assert L.mmoe_forward_chain(hs, 33, None, 1, ys, None) == 1
    assert L.mmoe_forward_chain(hs, 2, None, 1, ys, None) == 1
    assert b"NULL" in L.mmoe_last_error()
    # two layers writing the same buffer: refused before the handles are looked at
    same = (VP * 2)(64, 64)
    assert L.mmoe_forward_chain(hs, 2, None, 1, same, None) == 1
    assert b"same buffer" in L.mmoe_last_error()


def test_quantize_validates_before_launch(L):
    assert L.mmoe_quantize_int4(None, 4, 48, None, None, None) == 1
    assert L.mmoe_quantize_int4(None, -1, 32, None, None, None) == 1
    assert L.mmoe_quantize_int4(None, 0, 32, None, None, None) == 0
    assert L.mmoe_quantize_int4(None, 2, 32, None, None, None) == 1
    assert b"NULL" in L.mmoe_last_error()


def test_create_without_a_device_is_an_error_not_a_crash(L):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    h = C.c_void_p()
    assert L.mmoe_create(C.byref(valid_cfg()), 0, C.byref(h)) == 1
    assert b"device" in L.mmoe_last_error()


def test_static_scratch_forward_validates_before_any_device_work(L):
    cfg = valid_cfg(d_model=2048, expert_hidden=1024, shared_hidden=1024)
    fake = C.c_void_p(0x1000)
    w = _lib.Weights(fake, None, fake, fake, fake, fake, 1)
    # too many tokens for the static array: rejected before touching a device
    st = L.mmoe_forward_static_scratch(C.byref(cfg), C.byref(w), fake, 100000, fake, None)
    assert st == 1 and b"static scratch" in L.mmoe_last_error()
    # host weights are refused (nothing is copied)
    wh = _lib.Weights(fake, None, fake, fake, fake, fake, 0)
    assert L.mmoe_forward_static_scratch(C.byref(cfg), C.byref(wh), fake, 1, fake, None) == 1
    assert L.mmoe_forward_static_scratch(C.byref(cfg), C.byref(w), fake, -1, fake, None) == 1
    assert L.mmoe_forward_static_scratch(C.byref(cfg), C.byref(w), fake, 0, fake, None) == 0
    assert L.mmoe_forward_static_scratch(None, C.byref(w), fake, 1, fake, None) == 1
    # more than 2^20 tokens: rejected before the scratch size is worked out
    assert L.mmoe_forward_static_scratch(C.byref(cfg), C.byref(w), fake, (1 << 20) + 1, fake, None) == 1
    assert b"2^20" in L.mmoe_last_error()


@pytest.mark.parametrize("field,offset,msg", [("w_gate_up", 8, b"16-byte"), ("w_down", 4, b"16-byte"),
                                              ("w_router", 2, b"4-byte"), ("router_bias", 1, b"4-byte"),
                                              ("s_gate_up", 2, b"4-byte"), ("s_down", 3, b"4-byte")])
def test_static_scratch_rejects_misaligned_weights(L, field, offset, msg):
    # the weights are read in place with vector loads: a misaligned slice of a caller's pool is an
    # argument error, found before anything is launched (no device is needed to see it)
    cfg = valid_cfg(has_router_bias=1)
    ptrs = {f: 0x10000 + 0x1000 * i for i, f in enumerate(("w_router", "router_bias", "w_gate_up", "s_gate_up",
                                                            "w_down", "s_down"))}
    ptrs[field] += offset
    w = _lib.Weights(*[C.c_void_p(ptrs[f]) for f in ("w_router", "router_bias", "w_gate_up", "s_gate_up",
                                                     "w_down", "s_down")], 1)
    fake = C.c_void_p(0x1000)
    assert L.mmoe_forward_static_scratch(C.byref(cfg), C.byref(w), fake, 1, fake, None) == 1
    assert msg in L.mmoe_last_error()


def test_failure_injection_entry_points_validate(L):
    # the allocation-failure and stall hooks of the failure-detection tests: arguments checked
    # without a device; an armed allocation hook that never fires is turned off again
    assert L.mmoe_debug_fail_alloc(-2) == 1
    assert L.mmoe_debug_fail_alloc(3) == 0
    assert L.mmoe_debug_fail_alloc(-1) == 0
    assert L.mmoe_debug_set_wait_limit(None, 100, 1) == 1
    assert b"NULL" in L.mmoe_last_error()


def host_chunks(L, T, cap=8):
    b = (C.c_int64 * cap)()
    n = C.c_int32()
    assert L.mmoe_debug_host_chunks(T, b, cap, C.byref(n)) == 0
    return list(b[:n.value + 1])


@pytest.mark.parametrize("T", [0, 1, 64, 65, 8191, 8192, 16383, 16384, 16385, 24576, 24653, 32767, 32768, 32832,
                               40000, 65536, 100003, 1 << 20])
def test_host_forward_chunks(L, T):
    # the split of a host-buffer forward: ordered, complete, on 128-token boundaries, with
    # n = min(4, T // 8192) chunks and end chunks a third of the middle ones when n >= 3
    b = host_chunks(L, T)
    n = len(b) - 1
    assert n == max(1, min(4, T // 8192))
    assert b[0] == 0 and b[-1] == T
    assert all(x % 128 == 0 for x in b[1:-1])
    sizes = [b[i + 1] - b[i] for i in range(n)]
    if T > 0:
        assert all(s > 0 for s in sizes)
    if n >= 2:
        assert min(sizes) > 64  # every chunk stays on the prefill kernels, like the unsplit batch
    if n >= 3:
        unit = T / (3 * n - 4)
        for i, s in enumerate(sizes):
            w = 1 if i in (0, n - 1) else 3
            assert abs(s - w * unit) <= 256, (i, s, w * unit)


def test_host_chunks_rejects_bad_arguments(L):
    b = (C.c_int64 * 8)()
    n = C.c_int32()
    assert L.mmoe_debug_host_chunks(-1, b, 8, C.byref(n)) == 1
    assert L.mmoe_debug_host_chunks(40000, None, 8, C.byref(n)) == 1
    assert L.mmoe_debug_host_chunks(40000, b, 8, None) == 1
    assert L.mmoe_debug_host_chunks(40000, b, 4, C.byref(n)) == 1  # 4 chunks need 5 boundaries
    assert b"cap" in L.mmoe_last_error()
