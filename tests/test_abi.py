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


def test_null_plan_arguments_of_the_newer_entries(lib):
    """The FP8, pipelined and shared-expert entries reject a null plan before touching a device."""
    assert lib.moe_plan_set_fp8(None, 1) == 1
    assert lib.moe_forward_fp8(None, None, None, None, None, None, None, None, None, None, 0, None, None) == 1
    assert lib.moe_forward_host_pipelined(None, None, None, None, None, None, None, 0, None, None) == 1
    assert lib.moe_host_pipeline_after(None, None) == 1
    assert lib.moe_host_pipeline_join(None, None) == 1
    assert lib.moe_plan_set_cta_pairs(None, 1) == 1
    assert lib.moe_plan_forward_launches(None, 0) == -1
    assert lib.moe_plan_forward_launches(None, 1) == -1


@pytest.mark.parametrize("args", [
    (1, 100, 128),    # K % 64
    (1, 128, 100),    # N % 64
    (0, 128, 128),    # E < 1
])
def test_weight_quantizer_rejects_bad_sizes_without_device(lib, args):
    E, K, N = args
    assert lib.moe_quantize_weights_fp8(None, None, None, E, K, N, None) == 1


def test_quantizer_bindings_check_shapes_before_calling(lib):
    import torch

    from moe_megakernel_b200 import quantize_weights_fp8, quantize_x_fp8
    with pytest.raises(TypeError):
        quantize_weights_fp8(torch.zeros(4, 4, dtype=torch.bfloat16))     # not [E, K, N]
    with pytest.raises(TypeError):
        quantize_x_fp8(torch.zeros(2, 2, 2, dtype=torch.bfloat16))        # not [T, H]
    with pytest.raises(ValueError):
        quantize_weights_fp8(torch.zeros(1, 64, 64, dtype=torch.float32))  # not bf16


def test_bench_source_hash_ignores_comments():
    """bench.py's check that measured counters belong to the current expert-GEMM code: comment
    and blank-line edits do not change the hash, code edits do."""
    import sys
    sys.path.insert(0, ROOT)
    import bench
    a = "int f(int x) {\n  return x + 1;  // add one\n}\n"
    b = "/* header\n   text */\nint f(int x) {\n\n  return x + 1;\n}  // end\n"
    c = "int f(int x) {\n  return x + 2;\n}\n"
    assert bench.code_text(a) == bench.code_text(b)
    assert bench.code_text(a) != bench.code_text(c)


def test_readme_c_example_compiles_against_the_header(tmp_path):
    """The C usage example in the README stays in step with include/moe_b200.h (syntax and types)."""
    import re
    import shutil
    import subprocess
    cc = shutil.which("gcc") or shutil.which("cc")
    cuda_inc = "/usr/local/cuda/include"
    if cc is None or not os.path.exists(os.path.join(cuda_inc, "cuda_runtime.h")):
        pytest.skip("no C compiler or CUDA headers")
    readme = open(os.path.join(ROOT, "README.md")).read()
    code = re.search(r"```c\n(.*?)```", readme, re.S).group(1).replace('#include "moe_b200.h"', "")
    src = tmp_path / "example.c"
    src.write_text("#include <stdio.h>\n#include <cuda_runtime.h>\n#include \"moe_b200.h\"\n"
                   "int example(int T_max, int H, int I, int E, int k, int T, const void* x, const void* Wg,\n"
                   "            const void* W1, const void* W3, const void* W2, void* y, void* stream) {\n"
                   + code + "\n  return st;\n}\n")
    r = subprocess.run([cc, "-fsyntax-only", "-Wall", "-I", os.path.join(ROOT, "include"), "-I", cuda_inc, str(src)],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
