"""The C-ABI library builds, loads and exports every entry point the header
declares; host-side validation answers without a GPU.  No compute calls."""
import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "rankmixer.h")


def _declared():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(rm_[a-z0-9_]+)\s*\(", src)))


@pytest.fixture(scope="module")
def lib_path():
    from token_mixing_feature_b200 import build
    return str(build.build())


def test_header_declares_the_boundary():
    names = _declared()
    for required in ("rm_create", "rm_token_mix", "rm_pffn_forward", "rm_moe_forward",
                     "rm_block_forward", "rm_stack_forward", "rm_destroy"):
        assert required in names


def test_library_exports_every_declared_symbol(lib_path):
    lib = ctypes.CDLL(lib_path)
    out = subprocess.run(["nm", "-D", "--defined-only", lib_path], capture_output=True, text=True).stdout
    exported = set(re.findall(r"\sT\s(rm_\w+)", out))
    for name in _declared():
        assert hasattr(lib, name), name
        assert name in exported, name


def test_binding_mirrors_header(lib_path):
    from token_mixing_feature_b200 import rankmixer as rm
    assert sorted(rm.EXPORTED) == _declared()
    for name in rm.EXPORTED:
        assert callable(getattr(rm, name))


def test_host_validation_without_gpu(lib_path):
    from token_mixing_feature_b200 import rankmixer as rm
    lib = rm._lib
    assert rm.status_string(rm.RM_ERR_DEVICE_TIMEOUT) == "a bounded device-side wait ran out"
    out = ctypes.c_void_p()
    assert lib.rm_create(None, ctypes.byref(out)) == rm.RM_ERR_INVALID_ARG
    # H = T needs D divisible by T: rejected before any device call
    cfg = rm.rm_config(64, 3, 64, 256, 2, 0, rm.RM_BF16, 1e-5, 0)
    assert lib.rm_create(ctypes.byref(cfg), ctypes.byref(out)) == rm.RM_ERR_UNSUPPORTED
    cfg = rm.rm_config(64, 8, 72, 256, 2, 0, rm.RM_BF16, 1e-5, 0)      # D % 16 != 0 for bf16
    assert lib.rm_create(ctypes.byref(cfg), ctypes.byref(out)) == rm.RM_ERR_UNSUPPORTED
    cfg = rm.rm_config(0, 8, 64, 256, 2, 0, rm.RM_BF16, 1e-5, 0)       # B_max < 1
    assert lib.rm_create(ctypes.byref(cfg), ctypes.byref(out)) == rm.RM_ERR_INVALID_ARG
    cfg = rm.rm_config(64, 8, 64, 256, 2, 4, rm.RM_F32, 1e-5, 0)       # MoE needs bf16
    assert lib.rm_create(ctypes.byref(cfg), ctypes.byref(out)) == rm.RM_ERR_UNSUPPORTED
    # limits of the staged kernels, all rejected before any device call
    for fields, status in [
        ((64, 65, 65 * 16, 256, 2, 0, rm.RM_BF16, 1e-5, 0, 1), rm.RM_ERR_UNSUPPORTED),   # T > 64
        ((64, 8, 128, 256, 2, 33, rm.RM_BF16, 1e-5, 0, 1), rm.RM_ERR_UNSUPPORTED),       # more than 32 experts
        ((64, 16, 1536, 256, 2, 32, rm.RM_BF16, 1e-5, 0, 1), rm.RM_ERR_UNSUPPORTED),     # router rows beyond 160 KB
        ((64, 16, 4096, 256, 2, 0, rm.RM_BF16, 1e-5, 0, 1), rm.RM_ERR_UNSUPPORTED),      # D above 2048 (bf16)
        ((64, 8, 2048, 256, 2, 0, rm.RM_F32, 1e-5, 0, 1), rm.RM_ERR_UNSUPPORTED),        # D above 1024 (fp32)
        ((64, 64, 2048, 256, 2, 0, rm.RM_BF16, 1e-5, 0, 1), rm.RM_ERR_UNSUPPORTED),      # a sample exceeds shared memory
        ((64, 8, 64, 256, 2, 0, rm.RM_BF16, 1e-5, 3, 1), rm.RM_ERR_INVALID_ARG),         # unknown activation
        ((64, 8, 64, 256, 2, 0, rm.RM_BF16, 1e-5, 0, 2), rm.RM_ERR_INVALID_ARG),         # mix_addnorm not 0/1
        ((64, 8, 64, 256, 2, 0, rm.RM_BF16, 0.0, 0, 1), rm.RM_ERR_INVALID_ARG),          # eps must be > 0
        ((64, 8, 64, 256, 0, 0, rm.RM_BF16, 1e-5, 0, 1), rm.RM_ERR_INVALID_ARG),         # L < 1
    ]:
        cfg = rm.rm_config(*fields)
        assert lib.rm_create(ctypes.byref(cfg), ctypes.byref(out)) == status, fields
    assert out.value is None
    assert lib.rm_token_mix(None, None, None, 1, None) == rm.RM_ERR_INVALID_ARG
