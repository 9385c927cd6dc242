"""The C ABI library loads, exports every entry point include/moe.h declares,
and rejects bad arguments on the host (CPU only: none of these calls reaches
the GPU)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe.h")


def declared_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^MOE_API\s+[\w\s\*]+?\b(moe_\w+)\s*\(", text, re.M)))


@pytest.fixture(scope="module")
def m():
    from conftest import build_library
    build_library()
    import sparse_mixture_experts_24_b200 as m
    return m


def test_header_declares_the_entry_points():
    syms = declared_symbols()
    assert {"moe_create", "moe_forward", "moe_destroy", "moe_last_error"} <= set(syms)
    assert len(syms) >= 11


def test_library_exports_every_declared_symbol(m):
    lib = ctypes.CDLL(m.LIB_PATH)
    for s in declared_symbols():
        assert hasattr(lib, s), "symbol %s declared in moe.h is not exported" % s
    assert set(declared_symbols()) == set(m.EXPORTED)
    assert "sm_100a" in m.moe_version()


@pytest.mark.parametrize("args,msg", [
    ((0, 1, 128, 256, 1), "n = 0"),
    ((257, 2, 128, 256, 1), "n = 257"),
    ((8, 0, 128, 256, 1), "K = 0"),
    ((8, 9, 128, 256, 1), "K = 9"),
    ((8, 2, 100, 256, 1), "d = 100"),
    ((8, 2, 0, 256, 1), "d = 0"),
    ((8, 2, 128, 96, 1), "ffn = 96"),
    ((8, 2, 128, 256, 7), "dtype = 7"),
])
def test_create_rejects_bad_shapes(m, args, msg):
    with pytest.raises(m.MoEError) as ei:
        m.moe_create(*args)
    assert ei.value.status == m.MOE_ERR_INVALID_ARG
    assert msg in str(ei.value)


def test_create_destroy_without_gpu(m):
    for dt in (m.MOE_F32, m.MOE_BF16):
        h = m.moe_create(8, 2, 4096, 14336, dt)
        assert h
        m.moe_destroy(h)
    m.moe_destroy(None)  # NULL is allowed
    h = m.moe_create(256, 256, 64, 64, m.MOE_BF16)  # extremes are accepted
    m.moe_destroy(h)


def test_forward_rejects_bad_arguments_on_the_host(m):
    h = m.moe_create(8, 2, 128, 256, m.MOE_BF16)
    try:
        good = 1 << 20  # 16-byte aligned stand-in address; never dereferenced
        with pytest.raises(m.MoEError) as ei:
            m.moe_forward(None, 4, good, good, good, good, good, good, good, good, 0)
        assert ei.value.status == m.MOE_ERR_INVALID_ARG and "null handle" in str(ei.value)
        with pytest.raises(m.MoEError) as ei:
            m.moe_forward(h, -1, good, good, good, good, good, good, good, good, 0)
        assert "T = -1" in str(ei.value)
        with pytest.raises(m.MoEError) as ei:
            m.moe_forward(h, 4, None, good, good, good, good, good, good, good, 0)
        assert "x is NULL" in str(ei.value)
        with pytest.raises(m.MoEError) as ei:
            m.moe_forward(h, 4, good, good, good + 8, good, good, good, good, good, 0)
        assert "w1 is not 16-byte aligned" in str(ei.value)
        with pytest.raises(m.MoEError) as ei:
            m.moe_forward(h, 1 << 31, good, good, good, good, good, good, good, good, 0)
        assert "exceeds" in str(ei.value)
        with pytest.raises(m.MoEError) as ei:
            m.moe_route(h, 4, good, good, None, good, 0)
        assert "topk_idx is NULL" in str(ei.value)
        with pytest.raises(m.MoEError) as ei:
            m.moe_forward_with_routing(h, 4, good, good, good, good, good, None, good, 0)
        assert "w2 is NULL" in str(ei.value)
        with pytest.raises(m.MoEError) as ei:
            m.moe_dispatch(h, 4, None)
        assert "topk_idx is NULL" in str(ei.value)
        # T = 0 is a no-op that touches nothing
        m.moe_forward(h, 0, None, None, None, None, None, None, None, None, 0)
        with pytest.raises(m.MoEError) as ei:
            m.moe_workspace_view(h, "H")
        assert "no workspace" in str(ei.value)
        assert m.moe_last_error() != ""
    finally:
        m.moe_destroy(h)


def test_capacity_and_stats_argument_checks_on_the_host(m):
    h = m.moe_create(8, 2, 128, 256, m.MOE_BF16)
    try:
        m.moe_set_capacity_factor(h, 1.25)
        m.moe_set_capacity_factor(h, 0.0)
        for bad in (-1.0, float("nan"), float("inf")):
            with pytest.raises(m.MoEError) as ei:
                m.moe_set_capacity_factor(h, bad)
            assert ei.value.status == m.MOE_ERR_INVALID_ARG
        good = 1 << 20
        with pytest.raises(m.MoEError) as ei:
            m.moe_router_stats(h, 0, good, good, good, 0.01, good, good, good, 0)
        assert "T = 0" in str(ei.value)
        with pytest.raises(m.MoEError) as ei:
            m.moe_router_stats(h, 4, good, good, good, 0.01, good, None, good, 0)
        assert "P is NULL" in str(ei.value)
    finally:
        m.moe_destroy(h)


def test_header_is_plain_c():
    """include/moe.h is a C header (C99, no C++ or CUDA types): a C compiler
    accepts it on its own."""
    import shutil
    import subprocess
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler on this host")
    r = subprocess.run([cc, "-fsyntax-only", "-std=c99", "-Wall", "-Werror", "-x", "c", HEADER],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
