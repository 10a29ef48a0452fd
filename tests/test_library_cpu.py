"""CPU-only checks of the C ABI: the library loads, exports every symbol the header
declares, and rejects bad configurations before touching CUDA."""
import ctypes
import os
import re

import pytest

from titans_long_term_b200 import mem

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    src = open(os.path.join(ROOT, "include", "titans_mem.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(titans_[a-z_]+)\s*\(", src)))


def test_header_declares_the_binding_surface():
    assert declared_functions() == sorted(mem.EXPORTED)


def test_library_exports_every_declared_symbol():
    L = mem.lib()
    for name in declared_functions():
        assert hasattr(L, name), name
    assert L.titans_mem_version() == 100


def test_debug_library_exports_every_declared_symbol():
    """The bounds-checked variant (TITANS_DEBUG) has the same C ABI as the release library."""
    from titans_long_term_b200 import build
    L = ctypes.CDLL(build.build(debug=True))
    for name in declared_functions():
        assert hasattr(L, name), name
    L.titans_mem_version.restype = ctypes.c_int
    assert L.titans_mem_version() == 100


@pytest.mark.parametrize("d,h,chunk,mode,B,H,status", [
    (96, 0, 16, mem.FP32, 1, 1, mem.EUNSUPPORTED),
    (64, 128, 16, mem.FP32, 1, 1, mem.EUNSUPPORTED),
    (64, 256, 0, mem.BF16, 1, 1, mem.EUNSUPPORTED),
    (64, 256, 129, mem.BF16, 1, 1, mem.EUNSUPPORTED),
    (64, 256, 64, mem.BF16, 0, 1, mem.EINVAL),
    (64, 256, 64, mem.BF16, 1, -2, mem.EINVAL),
    (64, 256, 64, 7, 1, 1, mem.EINVAL),
])
def test_init_rejects_bad_configs(d, h, chunk, mode, B, H, status):
    cfg = mem.Config(d, h, chunk, mode, B, H, 0)
    out = ctypes.c_void_p()
    assert mem.lib().titans_mem_init(ctypes.byref(cfg), ctypes.byref(out)) == status
    assert out.value is None
    assert mem.lib().titans_last_error_string().decode()


def test_null_arguments():
    L = mem.lib()
    assert L.titans_mem_init(None, None) == mem.EINVAL
    assert L.titans_mem_destroy(None) == mem.EINVAL
    assert L.titans_mem_sync_status(None, None) == mem.EINVAL
    assert L.titans_mem_path(None, 64, 0) == -1
    rc = L.titans_mem_forward(None, None, None, None, None, None, None, 16, 16, None, None, None, None, None, None)
    assert rc == mem.EINVAL
    rc = L.titans_mem_step(None, None, None, None, None, None, None, None, None, None, None, None, None)
    assert rc == mem.EINVAL


def test_host_staged_forward_rejects_null_handle_and_buffers():
    L = mem.lib()
    rc = L.titans_mem_forward_host(None, None, None, None, None, None, None, 16, 16, None, None, None, None, None,
                                   None, 0, None)
    assert rc == mem.EINVAL
    assert "handle" in L.titans_last_error_string().decode()


def test_noalloc_rejects_bad_config_before_cuda():
    L = mem.lib()
    assert L.titans_mem_forward_noalloc(None, None, None, None, None, None, None, 16, 16, None, None, None, None,
                                        None, None) == mem.EINVAL
    cfg = mem.Config(96, 0, 16, mem.FP32, 1, 1, 0)  # unsupported d
    rc = L.titans_mem_forward_noalloc(ctypes.byref(cfg), None, None, None, None, None, None, 16, 16, None, None,
                                      None, None, None, None)
    assert rc in (mem.EINVAL, mem.EUNSUPPORTED)


def test_noalloc_rejects_too_many_units_before_cuda():
    """B*H above 2^30 units is refused before the scratch size is computed (it could wrap)."""
    L = mem.lib()
    cfg = mem.Config(64, 256, 64, mem.BF16, 1 << 16, 1 << 15, 0)  # 2^31 units
    rc = L.titans_mem_forward_noalloc(ctypes.byref(cfg), None, None, None, None, None, None, 16, 16, None, None,
                                      None, None, None, None)
    assert rc == mem.EINVAL
    assert "units" in L.titans_last_error_string().decode()


@pytest.mark.parametrize("d,h,layers,status", [
    (64, 256, 9, mem.EUNSUPPORTED),   # too deep
    (64, 256, 1, mem.EUNSUPPORTED),   # below two layers
    (64, 0, 3, mem.EINVAL),           # a deep memory needs hidden layers
    (96, 384, 3, mem.EUNSUPPORTED),   # unsupported width, as for titans_mem_init
])
def test_init_deep_rejects_bad_configs(d, h, layers, status):
    cfg = mem.Config(d, h, 64, mem.FP32, 1, 1, 0)
    out = ctypes.c_void_p()
    assert mem.lib().titans_mem_init_deep(ctypes.byref(cfg), layers, ctypes.byref(out)) == status
    assert out.value is None


def test_deep_forward_rejects_null_handle():
    L = mem.lib()
    rc = L.titans_mem_forward_deep(None, None, None, None, None, None, None, 16, 16, None, None, None, None, None)
    assert rc == mem.EINVAL


def test_binding_argument_counts_match_the_header():
    """Every function the binding declares takes as many arguments as the header says."""
    src = open(os.path.join(ROOT, "include", "titans_mem.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    L = mem.lib()
    for name, params in re.findall(r"\b(titans_[a-z_]+)\s*\(([^;{]*?)\)\s*;", src):
        params = params.strip()
        n = 0 if params in ("", "void") else params.count(",") + 1
        argtypes = getattr(L, name).argtypes
        if argtypes is None:
            assert n == 0, f"{name}: the header declares {n} parameters, the binding none"
            continue
        assert len(argtypes) == n, f"{name}: header {n} parameters, binding {len(argtypes)}"
