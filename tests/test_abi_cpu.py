"""CPU-only checks of the C ABI library: it builds for sm_100a, loads without
a GPU, exports every function include/moe.h declares, and rejects bad
arguments before touching the device."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def abi():
    from block_diffusion_moe_router_b200 import build
    build.build()
    from block_diffusion_moe_router_b200 import _abi
    return _abi


def declared_functions():
    names = []
    for h in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if h.endswith(".h"):
            src = open(os.path.join(ROOT, "include", h)).read()
            names += re.findall(r"^\s*(?:moe_status_t|void|const char\s*\*)\s*(moe_\w+)\s*\(",
                                src, re.M)
    return names


def test_header_declares_the_boundary():
    names = declared_functions()
    for n in ("moe_plan_create", "moe_forward", "moe_route", "moe_plan_destroy",
              "moe_plan_sync_status", "moe_status_str"):
        assert n in names


def test_library_exports_every_declared_symbol(abi):
    lib = abi.lib()
    missing = [n for n in declared_functions() if not hasattr(lib, n)]
    assert not missing, missing
    assert set(abi.EXPORTS) >= set(declared_functions()) - set()


def test_status_strings(abi):
    assert abi.status_str(abi.MOE_OK) == "MOE_OK"
    assert "TIMEOUT" in abi.status_str(abi.MOE_ERR_TIMEOUT)
    assert "unknown" in abi.status_str(99)


def test_plan_create_rejects_bad_shapes_without_device(abi):
    lib = abi.lib()
    h = ctypes.c_void_p()
    for E, k, d, f, wd in [(0, 1, 256, 64, 0), (16, 0, 256, 64, 0), (16, 17, 256, 64, 0),
                           (300, 8, 256, 64, 0), (16, 2, 200, 64, 0), (16, 2, 256, 96, 0),
                           (16, 2, 8192, 64, 0), (16, 33, 256, 64, 0), (16, 2, 256, 64, 7)]:
        assert lib.moe_plan_create(E, k, d, f, wd, ctypes.byref(h)) == abi.MOE_ERR_UNSUPPORTED
        assert h.value is None
    assert lib.moe_plan_create(16, 2, 256, 64, 0, None) == abi.MOE_ERR_INVALID_ARG


def test_null_plan_calls_are_rejected(abi):
    lib = abi.lib()
    assert lib.moe_plan_set_option(None, 0, 1e-6) == abi.MOE_ERR_INVALID_ARG
    assert lib.moe_plan_reserve(None, 16) == abi.MOE_ERR_INVALID_ARG
    assert lib.moe_forward(None, 4, *([None] * 12)) == abi.MOE_ERR_INVALID_ARG
    assert lib.moe_route(None, 4, *([None] * 8)) == abi.MOE_ERR_INVALID_ARG
    assert lib.moe_plan_sync_status(None, None) == abi.MOE_ERR_INVALID_ARG
    lib.moe_plan_destroy(None)


def test_product_path_has_no_oracle_dependency():
    """The package and its C/CUDA sources never reference the oracle."""
    pkg = os.path.join(ROOT, "block_diffusion_moe_router_b200")
    for dp, _, fs in os.walk(pkg):
        for fn in fs:
            if fn.endswith((".py", ".cu", ".cuh", ".h")):
                src = open(os.path.join(dp, fn)).read()
                assert "oracle" not in src.replace("CPU oracle", ""), fn


def test_lmhead_create_rejects_bad_shapes_without_device(abi):
    lib = abi.lib()
    h = ctypes.c_void_p()
    for V, d in [(0, 256), (1 << 25, 256), (1000, 32), (1000, 100), (1000, 16384)]:
        assert lib.moe_lmhead_create(V, d, ctypes.byref(h)) == abi.MOE_ERR_UNSUPPORTED
        assert h.value is None
    assert lib.moe_lmhead_create(1000, 256, None) == abi.MOE_ERR_INVALID_ARG
    assert lib.moe_lmhead_forward(None, 4, None, None, 1.0, 0.0, None, 0.1, None, None, None,
                                  None, None) == abi.MOE_ERR_INVALID_ARG
    assert lib.moe_lmhead_sync_status(None, None) == abi.MOE_ERR_INVALID_ARG
    lib.moe_lmhead_destroy(None)


def test_binding_constants_match_the_header(abi):
    """Every status, weight format, option and limit the header defines has the
    same value in the Python binding."""
    src = open(os.path.join(ROOT, "include", "moe.h")).read()
    enums = dict((n, int(v)) for n, v in re.findall(r"\b(MOE_(?:ERR_\w+|OK|W_\w+|OPT_\w+|K_\w+))"
                                                    r"\s*=\s*(\d+)", src))
    assert len(enums) >= 25
    for name, val in enums.items():
        if name == "MOE_K_COUNT":
            continue
        assert getattr(abi, name) == val, name
    defines = dict(re.findall(r"#define\s+(MOE_MAX_\w+)\s+\(?([^)\n]+)\)?", src))
    assert eval(defines["MOE_MAX_T"]) == abi.MOE_MAX_T
    assert eval(defines["MOE_MAX_ASSIGNMENTS"].replace("(", "").replace(")", "")) == \
        abi.MOE_MAX_ASSIGNMENTS
