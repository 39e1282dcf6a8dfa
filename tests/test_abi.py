"""The C-ABI library loads and exports every entry point its header declares.

No compute call here: these run without a GPU. Shape validation happens
before any device query, so unsupported shapes are rejected on any machine.
"""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe_b200.h")


def _declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[A-Za-z_][\w\s\*]*?\b(moe_\w+)\s*\(", src, flags=re.M)
    return sorted(set(names))


@pytest.fixture(scope="module")
def lib():
    from moe_megakernel_b200 import build, load_library
    build.build()
    return load_library()


def test_header_declares_the_boundary():
    names = _declared_functions()
    for required in ["moe_plan_create", "moe_plan_workspace_bytes", "moe_plan_bind_workspace", "moe_forward",
                     "moe_forward_host", "moe_route", "moe_check", "moe_plan_destroy", "moe_status_string",
                     "moe_plan_get_routing"]:
        assert required in names


def test_library_exports_every_declared_symbol(lib):
    for name in _declared_functions():
        assert hasattr(lib, name), f"{name} declared in moe_b200.h but not exported"


def test_binding_signatures_cover_the_header():
    from moe_megakernel_b200 import SIGNATURES
    assert sorted(SIGNATURES) == _declared_functions()


def test_status_strings(lib):
    for s in range(9):
        assert lib.moe_status_string(s)
    assert lib.moe_status_string(0) == b"ok"


@pytest.mark.parametrize("shape", [
    (0, 128, 128, 8, 2),      # T_max < 1
    (64, 100, 256, 8, 2),     # H % 128
    (64, 128, 200, 8, 2),     # I % 128
    (64, 128, 256, 12, 2),    # E % 8
    (64, 128, 256, 512, 2),   # E > 256
    (64, 128, 256, 8, 9),     # k > 8
    (64, 128, 256, 8, 0),     # k < 1
])
def test_unsupported_shapes_rejected_without_device(lib, shape):
    plan = ctypes.c_void_p()
    rc = lib.moe_plan_create(ctypes.byref(plan), *shape, 0, 0)
    assert rc == 2 and not plan.value


def test_bad_block_m_rejected(lib):
    plan = ctypes.c_void_p()
    assert lib.moe_plan_create(ctypes.byref(plan), 64, 128, 256, 8, 2, 48, 0) == 2


def test_null_plan_arguments(lib):
    assert lib.moe_plan_create(None, 64, 128, 256, 8, 2, 0, 0) == 1
    assert lib.moe_plan_workspace_bytes(None) == 0
    assert lib.moe_forward(None, None, None, None, None, None, None, 0, None, None) == 1
    assert lib.moe_check(None, None, None) == 1
    lib.moe_plan_destroy(None)


def test_kernel_count(lib):
    assert lib.moe_forward_kernel_count() == 5
