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
                                dict(max_tokens=0), dict(gating=2), dict(has_router_bias=2), dict(flags=16),
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
