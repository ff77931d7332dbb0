"""The C-ABI library loads, exports every entry point of include/spava.h and rejects
bad plans on the host before touching a device (no GPU needed)."""

import ctypes
import os
import re

import pytest
import torch

from sequence_approximate_attention_b200 import _lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "spava.h")


def _declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\s*\**\s*(spava_[a-z0-9_]+)\s*\(", text, flags=re.M)
    return sorted(set(names))


def test_header_and_binding_agree():
    declared = _declared_functions()
    assert len(declared) >= 12
    assert sorted(_lib.SIGNATURES) == declared


def test_library_exports_every_symbol(lib):
    for name in _declared_functions():
        assert hasattr(lib, name), name


def test_status_strings(lib):
    assert lib.spava_status_string(0) == b"SPAVA_OK"
    assert lib.spava_status_string(4) == b"SPAVA_ERR_TIMEOUT"
    assert lib.spava_status_string(5) == b"SPAVA_ERR_DEVICE_CHECK"


def _create(lib, **kw):
    args = dict(n_visual=512, n_text=0, n_hosts=2, sizes=None, anchor=64, passing=32, probe_r=16,
                hq=4, hkv=2, head_dim=64, scale=0.0)
    args.update(kw)
    h = ctypes.c_void_p()
    sizes = None
    if args["sizes"] is not None:
        arr = (ctypes.c_int32 * len(args["sizes"]))(*args["sizes"])
        sizes = ctypes.cast(arr, ctypes.POINTER(ctypes.c_int32))
    st = lib.spava_plan_create(ctypes.byref(h), args["n_visual"], args["n_text"], args["n_hosts"], sizes,
                               args["anchor"], args["passing"], args["probe_r"], args["hq"], args["hkv"],
                               args["head_dim"], ctypes.c_float(args["scale"]))
    if st == 0:
        lib.spava_plan_destroy(h)
    return st, lib.spava_last_error().decode()


@pytest.mark.parametrize("kw,status", [
    (dict(hq=5, hkv=2), _lib.SPAVA_ERR_INVALID_ARG),           # hq % hkv
    (dict(hq=34, hkv=2), _lib.SPAVA_ERR_UNSUPPORTED),          # G > 16
    (dict(head_dim=96), _lib.SPAVA_ERR_UNSUPPORTED),
    (dict(n_visual=513), _lib.SPAVA_ERR_INVALID_ARG),          # equal split
    (dict(sizes=[200, 300]), _lib.SPAVA_ERR_INVALID_ARG),      # sum != N
    (dict(sizes=[512, 0]), _lib.SPAVA_ERR_INVALID_ARG),
    (dict(anchor=240, passing=32), _lib.SPAVA_ERR_INVALID_ARG),  # A + P > B_0
    (dict(probe_r=300), _lib.SPAVA_ERR_INVALID_ARG),           # R > B_h
    (dict(probe_r=24), _lib.SPAVA_ERR_UNSUPPORTED),            # R % 16
    (dict(n_hosts=0), _lib.SPAVA_ERR_INVALID_ARG),
    (dict(passing=-1), _lib.SPAVA_ERR_INVALID_ARG),
])
def test_plan_rejects_bad_sizes_on_host(lib, kw, status):
    st, msg = _create(lib, **kw)
    assert st == status, msg
    assert msg


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-device path")
def test_valid_plan_without_device_reports_cuda_error(lib):
    st, msg = _create(lib)
    assert st == _lib.SPAVA_ERR_CUDA
    assert "device" in msg.lower()


def test_null_arguments(lib):
    assert lib.spava_workspace_bytes(None) == 0
    assert lib.spava_plan_destroy(None) == 0
    assert lib.spava_attn_prefill(None, None, None, None, None, None, None, None, None, None) == \
        _lib.SPAVA_ERR_INVALID_ARG
    assert lib.spava_plan_offsets(None, None) == -1
    assert lib.spava_plan_set_score_reduce(None, 0) == _lib.SPAVA_ERR_INVALID_ARG
