"""Host-only checks of the C ABI: the library loads without a GPU, exports
every entry point include/fwpkm.h declares, and rejects bad arguments on the
host with the documented status codes (before any CUDA call)."""
import ctypes
import os
import re

import pytest

from sparse_weight_memory_b200 import build as fwbuild
from sparse_weight_memory_b200 import fwpkm

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "fwpkm.h")


@pytest.fixture(scope="module")
def lib():
    fwbuild.build()
    return fwpkm.load_library()


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(fwpkm_[a-z_]+)\s*\(", src)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ("fwpkm_state_init", "fwpkm_step", "fwpkm_state_get", "fwpkm_state_set",
                     "fwpkm_state_free", "fwpkm_last_error"):
        assert required in names


def test_every_declared_symbol_is_exported(lib):
    for name in declared_functions():
        assert hasattr(lib, name), f"{name} declared in fwpkm.h but not exported"


@pytest.mark.parametrize("N,dq,dv,topk,chunk,heads", [
    (1000, 64, 64, 4, 32, 1),      # N not a perfect square
    (9, 64, 64, 2, 32, 1),         # n = 3 < 4
    (1024, 10, 64, 4, 32, 1),      # dq not a multiple of 16
    (1024, 64, 6, 4, 32, 1),       # dv not a multiple of 4
    (1024, 64, 64, 33, 32, 1),     # topk > 32
    (16 * 16, 64, 64, 17, 32, 1),  # topk > n
    (1024, 64, 64, 0, 32, 1),      # topk < 1
    (1024, 64, 64, 4, 0, 1),       # chunk < 1
    (1024, 64, 64, 4, 32, 0),      # heads < 1
    (4096 * 4096, 64, 64, 4, 32, 1),  # n > 1024
    (1025 * 1025, 64, 64, 4, 32, 1),  # n > 1024 (the selection masks hold 32 entries per lane)
    (1024, 2064, 64, 4, 32, 1),    # dq/2 > 1024
    (1024, 64, 2052, 4, 32, 1),    # dv > 2048
    (1024, 64, 64, 4, (1 << 20) + 1, 1),  # chunk > 2^20
    (1024, 64, 64, 4, 32, 17),     # heads > 16
])
def test_state_init_rejects_bad_shapes(lib, N, dq, dv, topk, chunk, heads):
    h = ctypes.c_void_p()
    rc = lib.fwpkm_state_init(N, dq, dv, topk, chunk, heads, ctypes.byref(h))
    assert rc == fwpkm.FWPKM_ESHAPE
    assert h.value is None
    assert lib.fwpkm_last_error().decode()


def test_null_arguments_are_rejected(lib):
    assert lib.fwpkm_state_init(1024, 64, 64, 4, 32, 1, None) == fwpkm.FWPKM_EINVAL
    assert lib.fwpkm_state_init_batched(1024, 64, 64, 4, 32, 1, 2, None) == fwpkm.FWPKM_EINVAL
    assert lib.fwpkm_step(None, 1, 1, None, 0, None, 0, None, 1.0, 0.0, None, None) == \
        fwpkm.FWPKM_EINVAL
    assert lib.fwpkm_state_get(None, None, None, None) == fwpkm.FWPKM_EINVAL
    assert lib.fwpkm_state_set(None, None, None, None) == fwpkm.FWPKM_EINVAL
    assert lib.fwpkm_state_set_eps(None, 1e-3) == fwpkm.FWPKM_EINVAL
    assert lib.fwpkm_record_selection(None, None, None) == fwpkm.FWPKM_EINVAL
    assert lib.fwpkm_force_selection(None, None, None) == fwpkm.FWPKM_EINVAL
    assert lib.fwpkm_read_stats(None, None, None, None, None, None, 0, None) == fwpkm.FWPKM_EINVAL
    assert lib.fwpkm_step_host(None, 1, 1, None, 0, None, 0, None, 1.0, 0.0, None, None) == \
        fwpkm.FWPKM_EINVAL
    assert lib.fwpkm_set_graphs(None, 1) == fwpkm.FWPKM_EINVAL
    assert lib.fwpkm_set_profiling(None, 1) == fwpkm.FWPKM_EINVAL
    assert lib.fwpkm_profile_read(None, None, None, None, 0, None, None) == fwpkm.FWPKM_EINVAL
    assert lib.fwpkm_select_noalloc(None, 1, 1, None, 0, None, None, None, None) == \
        fwpkm.FWPKM_EINVAL
    assert lib.fwpkm_set_wait_limits(None, 0, 0) == fwpkm.FWPKM_EINVAL
    assert lib.fwpkm_state_set_options(None, 0) == fwpkm.FWPKM_EINVAL
    assert lib.fwpkm_step_ex(None, 1, 1, None, 0, None, 0, None, None, 0, 1.0, 0.0, None,
                             None) == fwpkm.FWPKM_EINVAL
    assert lib.fwpkm_step_host_ex(None, 1, 1, None, 0, None, 0, None, None, 0, 1.0, 0.0, None,
                                  None) == fwpkm.FWPKM_EINVAL
    lib.fwpkm_inject_alloc_failures(0)  # takes no state; 0 disarms
    lib.fwpkm_state_free(None)  # no-op


def test_every_entry_point_rejects_a_null_state(lib):
    """Each fwpkm_* call that takes a state is covered by the NULL checks above."""
    src = open(os.path.join(ROOT, "tests", "test_abi_cpu.py")).read()
    body = src[src.index("def test_null_arguments_are_rejected"):
               src.index("def test_every_entry_point_rejects_a_null_state")]
    for name in declared_functions():
        if name in ("fwpkm_last_error",):
            continue
        assert f"lib.{name}(" in body, f"{name} has no NULL-argument check"


def test_product_path_has_no_oracle_or_fallback():
    """The library package never imports the oracle (test infrastructure)."""
    pkg = os.path.join(ROOT, "sparse_weight_memory_b200")
    pat = re.compile(r"^\s*(from|import)\s+oracle\b|ctypes\.CDLL\(.*oracle", re.M)
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith(".py"):
                assert not pat.search(open(os.path.join(dirpath, f)).read()), f


def test_injected_allocation_failure_is_enomem(lib):
    """An injected device-allocation failure makes state_init return ENOMEM
    with no state, before any table exists; the injection is consumed."""
    h = ctypes.c_void_p()
    lib.fwpkm_inject_alloc_failures(1)
    try:
        rc = lib.fwpkm_state_init(1024, 64, 64, 4, 32, 1, ctypes.byref(h))
    finally:
        lib.fwpkm_inject_alloc_failures(0)
    assert rc == fwpkm.FWPKM_ENOMEM
    assert h.value is None
    assert "allocation" in lib.fwpkm_last_error().decode()


@pytest.mark.parametrize("memories", [0, -1, 2048])
def test_batched_init_rejects_bad_memory_counts(lib, memories):
    """memories >= 1, and every value and sub-key row of all memories must
    have a 32-bit group id (2048 memories of 1M slots do not)."""
    h = ctypes.c_void_p()
    rc = lib.fwpkm_state_init_batched(1024 * 1024, 64, 64, 4, 32, 1, memories, ctypes.byref(h))
    assert rc == fwpkm.FWPKM_ESHAPE
    assert h.value is None


def test_binding_constants_equal_the_header():
    """Every status code, dtype code, option bit and flag the binding passes
    through equals the header's value (a mismatch would select another reading
    of the method without any error)."""
    src = re.sub(r"/\*.*?\*/", "", open(HEADER).read(), flags=re.S)
    values = {name: int(val) for name, val in
              re.findall(r"#define\s+(FWPKM_[A-Z_]+)\s+(-?\d+)u?\b", src)}
    values.update({name: int(val) for name, val in
                   re.findall(r"\b(FWPKM_[A-Z0-9_]+)\s*=\s*(-?\d+)", src)})
    binding = [name for name in dir(fwpkm) if name.startswith("FWPKM_")]
    for name in binding:  # every constant of the binding is the header's
        assert name in values, f"{name} is not in the header"
        assert getattr(fwpkm, name) == values[name], name
    for name in ("FWPKM_OK", "FWPKM_ECUDA", "FWPKM_BF16", "FWPKM_LOOKAHEAD", "FWPKM_HEADS_SUM",
                 "FWPKM_AGG_COUNT", "FWPKM_AGG_SUM", "FWPKM_SCORE_DOT"):
        assert name in binding, name
